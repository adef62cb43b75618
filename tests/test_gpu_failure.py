"""Failure detection without a GPU fault: a bounded wait that is made to run
out reports an error status the host reads, and the context stays usable."""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
import swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports():
    L = ops.lib()
    L.arops_selftest_wait_timeout.argtypes = [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
    L.arops_selftest_wait_timeout.restype = ctypes.c_int
    ops.device_errors(clear=True)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    st = L.arops_selftest_wait_timeout(5_000_000, flag.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)  # 5 ms
    assert st == 0, L.arops_last_error()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(flag.item()) == 1  # the wait gave up
    assert ops.device_errors(clear=True) == 1  # AROPS_DEVICE_ERR_TIMEOUT
    assert elapsed < 5.0
    # the context is still usable: an operator runs and matches the oracle
    a = inputs.add_rmsnorm_inputs(4, 2048, "bf16", 3)
    y, r = ops.add_rmsnorm(a["x"].cuda(), a["residual"].cuda().clone(), a["gamma"].cuda())
    torch.cuda.synchronize()
    _, r_e = oracle.get().add_rmsnorm(a["x"], a["residual"], a["gamma"], 1e-6, "bf16")
    assert np.array_equal(r.cpu().double().numpy(), r_e)


def test_selftest_rejects_bad_limits():
    L = ops.lib()
    L.arops_selftest_wait_timeout.argtypes = [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
    assert L.arops_selftest_wait_timeout(0, 8, None) == 1
    assert L.arops_selftest_wait_timeout(3_000_000_000, 8, None) == 1
    assert L.arops_selftest_wait_timeout(1000, None, None) == 1
