"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host without launching anything (no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

import swiglu_ar_tts_b200 as ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"AROPS_API\s+[\w\s\*]+?\b(arops_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    from swiglu_ar_tts_b200 import build

    build.build()
    return ops.lib()


def test_header_declares_the_operators():
    names = _declared_symbols()
    for n in ("arops_rmsnorm", "arops_add_rmsnorm", "arops_mrope_qk", "arops_swiglu",
              "arops_status_string", "arops_last_error"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in _declared_symbols():
        assert hasattr(L, n), n
    assert L.arops_version() == 20200


def test_status_strings(L):
    for code, text in ((0, b"ok"), (1, b"invalid argument"), (2, b"unsupported size"),
                       (3, b"CUDA error"), (99, b"unknown status")):
        assert L.arops_status_string(code) == text


SEC = (ctypes.c_int32 * 3)(24, 20, 20)


@pytest.mark.parametrize("call,expect", [
    (lambda L: L.arops_rmsnorm(None, None, None, 4, 2048, 1e-6, 1, None), 1),
    (lambda L: L.arops_rmsnorm(1, 1, 1, 4, 2048, 1e-6, 7, None), 1),
    (lambda L: L.arops_rmsnorm(1, 1, 1, 4, 0, 1e-6, 1, None), 1),
    (lambda L: L.arops_rmsnorm(1, 1, 1, -1, 2048, 1e-6, 1, None), 1),
    (lambda L: L.arops_rmsnorm(1, 1, 1, 4, 2048, -1.0, 1, None), 1),
    (lambda L: L.arops_rmsnorm(1, 1, 1, 4, 2048, float("nan"), 1, None), 1),
    (lambda L: L.arops_rmsnorm(None, None, None, 0, 2048, 1e-6, 1, None), 0),
    (lambda L: L.arops_add_rmsnorm(1, None, 1, 1, 1, 4, 2048, 1e-6, 1, None), 1),
    (lambda L: L.arops_add_rmsnorm(1, 1, 2, 1, 2, 4, 2048, 1e-6, 1, None), 1),  # y == residual_out
    (lambda L: L.arops_add_rmsnorm(None, None, None, None, None, 0, 2048, 1e-6, 1, None), 0),
    (lambda L: L.arops_mrope_qk(1, 1, 1, 1, 1, 4, 16, 8, 127, SEC, 1e6, 1, None), 1),
    (lambda L: L.arops_mrope_qk(1, 1, 1, 1, 1, 4, 16, 8, 126, SEC, 1e6, 1, None), 1),
    (lambda L: L.arops_mrope_qk(1, 1, 1, 1, 1, 4, 16, 8, 1024, (ctypes.c_int32 * 3)(256, 128, 128),
                                1e6, 1, None), 2),
    (lambda L: L.arops_mrope_qk(1, 1, 1, 1, 1, 4, 16, 8, 128, None, 1e6, 1, None), 1),
    (lambda L: L.arops_mrope_qk(1, 1, 1, 1, 1, 4, 16, 8, 128, SEC, 0.0, 1, None), 1),
    (lambda L: L.arops_mrope_qk(1, 1, 1, 1, 1, 4, 16, 8, 128, SEC, float("inf"), 1, None), 1),
    (lambda L: L.arops_mrope_qk(1, 1, 1, 1, 1, 4, 16, 8, 128, (ctypes.c_int32 * 3)(24, 20, -1),
                                1e6, 1, None), 1),
    (lambda L: L.arops_mrope_qk(None, None, None, None, None, 4, 16, 8, 128, SEC, 1e6, 1, None), 1),
    (lambda L: L.arops_mrope_qk(1, None, 1, None, 1, 4, 16, 8, 128, SEC, 1e6, 1, None), 1),
    (lambda L: L.arops_mrope_qk(None, None, None, None, None, 0, 16, 8, 128, SEC, 1e6, 1, None), 0),
    (lambda L: L.arops_swiglu(None, 1, 1, 4, 6144, 1, None), 1),
    (lambda L: L.arops_swiglu(1, 1, 1, 4, 0, 1, None), 1),
    (lambda L: L.arops_swiglu(1, 1, 1, 1 << 40, 1 << 40, 1, None), 1),
    (lambda L: L.arops_swiglu(None, None, None, 0, 6144, 1, None), 0),
])
def test_argument_errors_launch_nothing(L, call, expect):
    before = L.arops_launch_count()
    assert call(L) == expect, L.arops_last_error()
    assert L.arops_launch_count() == before
    if expect != 0:
        assert L.arops_last_error() != b""


def test_python_binding_rejects_cpu_tensors():
    import torch

    x = torch.zeros(2, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.rmsnorm(x, torch.ones(8, dtype=torch.bfloat16))


def test_topk_sample_argument_errors(L):
    import ctypes as C

    n = C.c_size_t(0)
    assert L.arops_topk_sample_workspace(5, 151936, 50, C.byref(n)) == 0
    assert n.value == (1 << 18) + 5 * 38 * 50 * 8  # arrival counters, then candidates
    assert L.arops_topk_sample_workspace(5, 100, 0, C.byref(n)) == 1
    assert L.arops_topk_sample_workspace(5, 100, 101, C.byref(n)) == 1
    assert L.arops_topk_sample_workspace(5, 1000, 65, C.byref(n)) == 2
    assert L.arops_topk_sample_workspace(5, 262145, 5, C.byref(n)) == 2
    before = L.arops_launch_count()
    # workspace too small, null pointers, bad temperature: nothing launched
    assert L.arops_topk_sample(1, 1, 1, 1, 5, 1000, 5, 1.0, 1, 8, 16, None) == 1
    assert L.arops_topk_sample(None, 1, 1, 1, 5, 1000, 5, 1.0, 1, 8, 1 << 20, None) == 1
    assert L.arops_topk_sample(1, 1, 1, 1, 5, 1000, 5, 0.0, 1, 8, 1 << 20, None) == 1
    assert L.arops_topk_sample(1, 1, 1, 1, 5, 1000, 5, 1.0, 1, 9, 1 << 20, None) == 1  # misaligned
    assert L.arops_topk_sample(None, None, None, None, 0, 1000, 5, 1.0, 1, None, 0, None) == 0
    L.arops_topk_sample_prepare.argtypes = [C.c_void_p, C.c_size_t, C.c_void_p]
    assert L.arops_topk_sample_prepare(None, 1 << 20, None) == 1
    assert L.arops_topk_sample_prepare(16, (1 << 18) - 1, None) == 1  # smaller than the counters
    assert L.arops_launch_count() == before


def test_sampling_kernel_selection_is_clamped(L):
    """arops_set_topk_cluster takes 0 (slice), 1 (default), 2 (shared-memory
    cluster) and 3 (streaming), clamps anything else, and returns the old
    mode; a host setting, so no GPU is needed."""
    old = ops.set_topk_cluster(1)
    try:
        for mode, kept in ((0, 0), (2, 2), (3, 3), (7, 3), (-4, 0), (1, 1)):
            ops.set_topk_cluster(mode)
            assert ops.set_topk_cluster(mode) == kept, mode
    finally:
        ops.set_topk_cluster(old)
