"""The allocation-free top-k sampling entry point, through the C ABI.

arops_topk_sample_noalloc serves callers that cannot allocate device memory
(for example code inside a host application's real-time audio callback, where
cudaMalloc may block and synchronise the device): it takes its scratch from a
1 MiB array the library keeps in device memory.  This file is collected last
(after every other test) and also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs

pytestmark = pytest.mark.gpu

_vp = ctypes.c_void_p


def _lib():
    L = ops.lib()
    f = L.arops_topk_sample_noalloc
    f.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                  ctypes.c_float, ctypes.c_int, _vp]
    f.restype = ctypes.c_int
    return L


def _with_workspace(L, logits, gumbel, rows, vocab, k, temp, stream):
    n = ctypes.c_size_t(0)
    assert L.arops_topk_sample_workspace(rows, vocab, k, ctypes.byref(n)) == 0
    ws = torch.empty(n.value, dtype=torch.uint8, device="cuda")
    tok = torch.empty(rows, dtype=torch.int32, device="cuda")
    prob = torch.empty(rows, dtype=torch.float32, device="cuda")
    st = L.arops_topk_sample(logits.data_ptr(), gumbel.data_ptr(), tok.data_ptr(), prob.data_ptr(),
                             rows, vocab, k, temp, 1, ws.data_ptr(), n.value, stream)
    assert st == 0, L.arops_last_error()
    return tok, prob


def test_noalloc_matches_workspace_entry_point_two_calls():
    L = _lib()
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row, different shapes: the second runs on the first's
    # leftover scratch contents
    for rows, vocab, k, temp, seed in ((5, 151936, 50, 0.8, 1), (17, 30000, 64, 1.3, 2)):
        inp = inputs.topk_inputs(rows, vocab, k, "bf16", seed=seed)
        logits = inp["logits"].cuda()
        gumbel = inp["gumbel"].cuda()
        tok = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
        prob = torch.zeros(rows, dtype=torch.float32, device="cuda")
        st = L.arops_topk_sample_noalloc(logits.data_ptr(), gumbel.data_ptr(), tok.data_ptr(),
                                         prob.data_ptr(), rows, vocab, k, temp, 1, stream)
        assert st == 0, L.arops_last_error()
        t_ref, p_ref = _with_workspace(L, logits, gumbel, rows, vocab, k, temp, stream)
        torch.cuda.synchronize()
        assert torch.equal(tok, t_ref)
        np.testing.assert_allclose(prob.cpu().numpy(), p_ref.cpu().numpy(), rtol=1e-5, atol=0)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    L = _lib()
    before = L.arops_launch_count()
    # 200 rows x 38 slices x 50 x 8 bytes = 3.04 MB > 1 MiB
    st = L.arops_topk_sample_noalloc(8, 8, 8, 8, 200, 151936, 50, 1.0, 1, None)
    assert st == 2  # AROPS_ERR_UNSUPPORTED
    assert b"1048576" in L.arops_last_error()
    assert L.arops_launch_count() == before
