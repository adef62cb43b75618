"""M-RoPE fused with the KV-cache append on the GPU against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs
from gpu_util import dev
from tolerance import check, to_f64

pytestmark = pytest.mark.gpu


def _pair_scale(x):
    half = x.shape[-1] // 2
    m = np.maximum(np.abs(x[..., :half]), np.abs(x[..., half:]))
    return np.concatenate([m, m], axis=-1)


def _case(tokens, hq, hk, d, rows, max_seq, dtype, seed, loc=None, pos=None):
    rng = np.random.default_rng(seed)
    q = inputs.normal((tokens, hq, d), seed, dtype=dtype)
    k = inputs.normal((tokens, hk, d), seed + 1, dtype=dtype)
    v = inputs.normal((tokens, hk, d), seed + 2, dtype=dtype)
    kc = inputs.normal((rows, hk, max_seq, d), seed + 3, dtype=dtype)
    vc = inputs.normal((rows, hk, max_seq, d), seed + 4, dtype=dtype)
    if pos is None:
        pos = torch.from_numpy(rng.integers(0, 2000, size=(3, tokens)).astype(np.int32))
    if loc is None:
        # distinct slots: token t -> row t % rows, position t // rows
        t = np.arange(tokens)
        loc = torch.from_numpy(np.stack([t % rows, (t // rows) % max_seq]).astype(np.int32))
    return q, k, v, kc, vc, pos, loc


def _run_and_check(q, k, v, kc, vc, pos, loc, dtype, sections=(24, 20, 20), what=""):
    d = q.shape[-1]
    qd, kcd, vcd = dev(q), dev(kc), dev(vc)
    q_out = torch.empty_like(qd)
    ops.mrope_kv_append(qd, dev(k), dev(v), dev(pos), dev(loc), kcd, vcd, sections, 1e6, q_out=q_out)
    torch.cuda.synchronize()
    q_e, kc_e, vc_e = oracle.get().mrope_kv_append(q, k, v, pos, loc, kc, vc, sections, 1e6)
    check(q_out, q_e, dtype, _pair_scale(to_f64(q)), what=f"{what} q")
    # the cache: untouched and v slots bit-exact, k slots within tolerance
    kc_scale = np.full(kc_e.shape, np.inf)
    kc_scale_src = to_f64(kc).copy()
    ln = loc.numpy()
    kn = to_f64(k)
    for t in range(q.shape[0]):
        b, s = ln[0, t], ln[1, t]
        if 0 <= b < kc.shape[0] and 0 <= s < kc.shape[2]:
            kc_scale_src[b, :, s] = kn[t]
    check(kcd, kc_e, dtype, _pair_scale(kc_scale_src), what=f"{what} k_cache")
    assert np.array_equal(to_f64(vcd), vc_e), f"{what} v_cache"
    return kcd, vcd


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
# 2400 tokens hold more (token, head-pass) units than warps resident at once,
# the others fewer: both layouts of the launcher
@pytest.mark.parametrize("tokens,rows,max_seq", [(5, 5, 300), (256, 256, 4), (1000, 4, 512), (1, 1, 1),
                                                 (2400, 8, 512)])
def test_kv_append_shapes(dtype, tokens, rows, max_seq):
    case = _case(tokens, 16, 8, 128, rows, max_seq, dtype, seed=tokens + rows)
    _run_and_check(*case, dtype, what=f"{dtype} T={tokens}")


@pytest.mark.parametrize("d,sections", [(64, (16, 8, 8)), (96, (16, 16, 16)), (256, (48, 40, 40)), (10, (2, 2, 1))])
def test_kv_append_head_dims(d, sections):
    case = _case(9, 3, 2, d, 4, 6, "bf16", seed=d)
    _run_and_check(*case, "bf16", sections=sections, what=f"D={d}")


def test_kv_append_decode_step_positions_and_untouched_slots():
    """Decode: 5 candidates at step 17 (all rows = 17) write slot 17 of their
    own cache row; every other slot keeps its bits."""
    t = np.arange(5)
    loc = torch.from_numpy(np.stack([t, np.full(5, 17)]).astype(np.int32))
    pos = torch.full((3, 5), 17, dtype=torch.int32)
    case = _case(5, 16, 8, 128, 5, 64, "bf16", seed=5, loc=loc, pos=pos)
    kcd, vcd = _run_and_check(*case, "bf16", what="decode")
    kc0, vc0 = case[3], case[4]
    mask = torch.ones(kc0.shape, dtype=torch.bool)
    mask[:, :, 17] = False
    assert torch.equal(kcd.cpu()[mask], kc0[mask]) and torch.equal(vcd.cpu()[mask], vc0[mask])


def test_kv_append_out_of_range_slots_are_skipped_and_flagged():
    loc = torch.tensor([[0, 7, 1, -1], [3, 0, 99, 2]], dtype=torch.int32)  # tokens 1, 2, 3 invalid
    case = _case(4, 4, 2, 128, 2, 8, "bf16", seed=6, loc=loc)
    ops.device_errors(clear=True)
    _run_and_check(*case, "bf16", what="out of range")
    assert ops.device_errors(clear=True) == 2  # AROPS_DEVICE_ERR_BAD_INDEX
