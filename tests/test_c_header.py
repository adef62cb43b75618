"""The header is a plain C interface: a C99 program (and a C++ one) that
includes it compiles with warnings as errors, links against libarops.so and
runs the library's host-side paths (version, status strings, argument
validation, empty problems).  No GPU is needed: nothing here launches."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "swiglu_ar_tts_b200")

PROGRAM = r"""
#include <stdio.h>
#include "arops.h"

int main(void)
{
    arops_status st;
    int32_t sections[3] = {24, 20, 20};
    printf("version %d\n", (int)arops_version());
    st = arops_rmsnorm(NULL, NULL, NULL, 4, 1024, 1e-6f, AROPS_BF16, NULL);
    printf("null %d %s\n", (int)st, arops_status_string(st));
    printf("reason %s\n", arops_last_error());
    st = arops_mrope_qk(NULL, NULL, NULL, NULL, NULL, 5, 16, 8, 127, sections, 1e6f,
                        AROPS_BF16, NULL);
    printf("odd %d\n", (int)st);
    st = arops_swiglu(NULL, NULL, NULL, 0, 6144, AROPS_BF16, NULL);
    printf("empty %d\n", (int)st);
    return 0;
}
"""


def _build_and_run(tmp_path, compiler, flags, suffix):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not found")
    from swiglu_ar_tts_b200 import build

    build.build()
    src = tmp_path / f"use_arops.{suffix}"
    src.write_text(PROGRAM)
    exe = tmp_path / f"use_arops_{suffix}"
    subprocess.run([compiler, *flags, "-Wall", "-Wextra", "-Werror", "-pedantic",
                    f"-I{os.path.join(ROOT, 'include')}", str(src), "-o", str(exe),
                    f"-L{LIBDIR}", "-larops", f"-Wl,-rpath,{LIBDIR}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    lines = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert lines["version"] == "20200"
    assert lines["null"].startswith("1 ")  # AROPS_ERR_INVALID before any launch
    assert lines["reason"].strip()
    assert lines["odd"] == "1"  # odd head_dim
    assert lines["empty"] == "0"  # zero rows: a no-op


def test_header_is_c99(tmp_path):
    _build_and_run(tmp_path, "gcc", ["-std=c99"], "c")


def test_header_is_cxx(tmp_path):
    _build_and_run(tmp_path, "g++", ["-std=c++11"], "cpp")
