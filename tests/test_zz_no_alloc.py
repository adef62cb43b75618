"""The allocation-free top-k sampling entry point, through the C ABI.

arops_topk_sample_noalloc serves callers that cannot allocate device memory
(for example code inside a host application's real-time audio callback, where
cudaMalloc may block and synchronise the device, or a plugin that only receives
buffers from a host that owns all device memory): it takes its scratch from an
array the library keeps in device memory (arrival counters, then 1 MiB of
candidates).  This file is collected last
(after every other test) and also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs
from tolerance import to_f64

pytestmark = pytest.mark.gpu

_vp = ctypes.c_void_p
_DT = {"f32": 0, "bf16": 1}


def _lib():
    L = ops.lib()
    f = L.arops_topk_sample_noalloc
    f.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                  ctypes.c_float, ctypes.c_int, _vp]
    f.restype = ctypes.c_int
    return L


def _noalloc(L, logits, gumbel, rows, vocab, k, temp, dtype, stream):
    tok = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    prob = torch.zeros(rows, dtype=torch.float32, device="cuda")
    st = L.arops_topk_sample_noalloc(logits.data_ptr(), gumbel.data_ptr(), tok.data_ptr(),
                                     prob.data_ptr(), rows, vocab, k, temp, _DT[dtype], stream)
    assert st == 0, L.arops_last_error()
    return tok, prob


def _with_workspace(L, logits, gumbel, rows, vocab, k, temp, dtype, stream):
    n = ctypes.c_size_t(0)
    assert L.arops_topk_sample_workspace(rows, vocab, k, ctypes.byref(n)) == 0
    ws = torch.zeros(n.value, dtype=torch.uint8, device="cuda")  # counters start at zero
    tok = torch.empty(rows, dtype=torch.int32, device="cuda")
    prob = torch.empty(rows, dtype=torch.float32, device="cuda")
    st = L.arops_topk_sample(logits.data_ptr(), gumbel.data_ptr(), tok.data_ptr(), prob.data_ptr(),
                             rows, vocab, k, temp, _DT[dtype], ws.data_ptr(), n.value, stream)
    assert st == 0, L.arops_last_error()
    return tok, prob


def test_noalloc_setup_call_launches_nothing():
    """rows == 0 is the set-up call: it resolves the array in the current
    context and launches nothing."""
    L = _lib()
    before = L.arops_launch_count()
    st = L.arops_topk_sample_noalloc(None, None, None, None, 0, 151936, 50, 1.0, 1, None)
    assert st == 0, L.arops_last_error()
    assert L.arops_launch_count() == before


@pytest.mark.parametrize("kernel", ["slice", "cluster"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_two_calls_match_workspace_entry_point_and_oracle(dtype, kernel):
    """Two calls in a row, each compared with the workspace entry point and with
    the oracle, on each kernel (these few-row calls take the cluster kernel by
    default, which uses no scratch; the slice kernel is the one that does).
    The first call's logits sit 100 above the second's, so a key the second
    call read from the first call's leftover scratch (instead of writing it
    first) would outrank every real candidate and change the token."""
    old = ops.set_topk_cluster(kernel == "cluster")
    try:
        _two_calls(dtype)
    finally:
        ops.set_topk_cluster(old)


def _two_calls(dtype):
    L = _lib()
    stream = torch.cuda.current_stream().cuda_stream
    orc = oracle.get()
    cases = ((5, 151936, 50, 0.8, 1, 100.0), (17, 30000, 64, 1.3, 2, 0.0))
    for rows, vocab, k, temp, seed, shift in cases:
        inp = inputs.topk_inputs(rows, vocab, k, dtype, seed=seed)
        logits_host = (inp["logits"].float() + shift).to(inp["logits"].dtype)
        logits = logits_host.cuda()
        gumbel = inp["gumbel"].cuda()
        tok, prob = _noalloc(L, logits, gumbel, rows, vocab, k, temp, dtype, stream)
        torch.cuda.synchronize()
        assert ops.device_errors(clear=True) == 0
        t_ws, p_ws = _with_workspace(L, logits, gumbel, rows, vocab, k, temp, dtype, stream)
        torch.cuda.synchronize()
        t_orc, p_orc = orc.topk_sample(logits_host, inp["gumbel"], k, temp)
        assert np.array_equal(tok.cpu().numpy(), t_orc)
        np.testing.assert_allclose(to_f64(prob), p_orc, rtol=1e-5, atol=0)
        assert torch.equal(tok, t_ws)
        assert torch.equal(prob, p_ws)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    L = _lib()
    before = L.arops_launch_count()
    # 200 rows x 38 slices x 50 x 8 bytes = 3.04 MB > 1 MiB
    st = L.arops_topk_sample_noalloc(8, 8, 8, 8, 200, 151936, 50, 1.0, 1, None)
    assert st == 2  # AROPS_ERR_UNSUPPORTED
    assert b"1048576" in L.arops_last_error()
    assert L.arops_launch_count() == before
