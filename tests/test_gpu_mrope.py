"""M-RoPE on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs
from gpu_util import Guarded, dev, misaligned, resident_threads
from tolerance import check, to_f64

pytestmark = pytest.mark.gpu

SECTIONS = inputs.SECTIONS
THETA = inputs.THETA


def _pair_scale(x: np.ndarray) -> np.ndarray:
    """max(|a|, |b|) of the rotated pair of each element (the cancellation scale)."""
    half = x.shape[-1] // 2
    m = np.maximum(np.abs(x[..., :half]), np.abs(x[..., half:]))
    return np.concatenate([m, m], axis=-1)


def _compare(q_out, k_out, inp, sections=SECTIONS, theta=THETA, dtype="bf16", what=""):
    qe, ke = oracle.get().mrope_qk(inp["q"], inp["k"], inp["pos"], sections, theta)
    sq = check(q_out, qe, dtype, _pair_scale(to_f64(inp["q"])), what=f"{what} q")
    sk = check(k_out, ke, dtype, _pair_scale(to_f64(inp["k"])), what=f"{what} k")
    return sq, sk


def _run(inp, sections=SECTIONS, theta=THETA, in_place=False):
    q, k, pos = dev(inp["q"]), dev(inp["k"]), dev(inp["pos"])
    qo = q if in_place else torch.empty_like(q)
    ko = k if in_place else torch.empty_like(k)
    ops.mrope_qk(q, k, pos, sections, theta, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    return qo, ko


@pytest.mark.parametrize("in_place", [False, True])
def test_mrope_4096_tokens(in_place, family):
    """The M-RoPE workload: q [4096 x 16 x 128], k [4096 x 8 x 128], theta 1e6,
    sections [24, 20, 20]; 1024 text tokens then a 48 x 8 x 8 t/h/w grid."""
    inp = inputs.mrope_inputs(4096)
    qo, ko = _run(inp, in_place=in_place)
    _compare(qo, ko, inp, what="mrope 4096")
    # token 0 sits at position 0 in all rows: bit-identical to its input
    assert torch.equal(qo[0].cpu(), inp["q"][0]) and torch.equal(ko[0].cpu(), inp["k"][0])


def test_mrope_positions_layout():
    pos = inputs.mrope_positions(4096)
    assert pos.dtype == torch.int32 and tuple(pos.shape) == (3, 4096)
    assert torch.equal(pos[0, :1024], torch.arange(1024, dtype=torch.int32))
    assert torch.equal(pos[0, :1024], pos[1, :1024]) and torch.equal(pos[0, :1024], pos[2, :1024])
    assert int(pos[0, 1024]) == 1024 and int(pos[0, -1]) == 1024 + 3071 // 64
    assert int(pos[1, 1024 + 8]) == 1 and int(pos[2, 1024 + 9]) == 1


def test_mrope_section_masks_bit_exact(family):
    """Only one of t/h/w nonzero: pairs outside that row's section are returned
    bit for bit; pairs inside move."""
    inp = inputs.mrope_inputs(3, seed=40)
    bounds = [(0, 24), (24, 44), (44, 64)]
    for row, (lo, hi) in enumerate(bounds):
        pos = torch.zeros(3, 3, dtype=torch.int32)
        pos[row, :] = torch.tensor([5, 77, 1071], dtype=torch.int32)
        qo, ko = _run({"q": inp["q"], "k": inp["k"], "pos": pos})
        for out, src in ((qo.cpu(), inp["q"]), (ko.cpu(), inp["k"])):
            for j in range(64):
                same = torch.equal(out[..., j], src[..., j]) and torch.equal(out[..., j + 64], src[..., j + 64])
                if lo <= j < hi:
                    assert not same, (row, j)
                else:
                    assert same, (row, j)
        _compare(qo, ko, {"q": inp["q"], "k": inp["k"], "pos": pos}, what=f"mask row {row}")


def test_mrope_equal_rows_is_1d_rope_and_large_positions(family):
    inp = inputs.mrope_inputs(64, seed=41)
    p = torch.tensor([0, 1, 2, 3, 1000, 1071, 4095, 65535, 1 << 20, (1 << 31) - 1, -5, -1000] + list(range(52)),
                     dtype=torch.int32)
    inp["pos"] = torch.stack([p, p, p])
    qo, ko = _run(inp)
    _compare(qo, ko, inp, what="equal rows")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("head_dim,sections", [
    (128, (24, 20, 20)), (128, (64, 0, 0)), (128, (0, 0, 64)), (64, (16, 8, 8)), (256, (48, 40, 40)),
    (16, (4, 2, 2)), (32, (8, 4, 4)), (512, (128, 64, 64)), (96, (16, 16, 16)), (2, (1, 0, 0)),
    (10, (2, 2, 1)),
])
def test_mrope_head_dims(dtype, head_dim, sections, family):
    inp = inputs.mrope_inputs(37, n_q_heads=5, n_k_heads=3, head_dim=head_dim, dtype=dtype, seed=head_dim)
    qo, ko = _run(inp, sections=sections)
    _compare(qo, ko, inp, sections=sections, dtype=dtype, what=f"D={head_dim} {dtype}")


@pytest.mark.parametrize("hq,hk", [(16, 0), (0, 8), (1, 1), (7, 5), (32, 4), (40, 40)])
def test_mrope_head_counts(hq, hk, family):
    inp = inputs.mrope_inputs(19, n_q_heads=hq, n_k_heads=hk, seed=hq * 10 + hk)
    q, k, pos = dev(inp["q"]), dev(inp["k"]), dev(inp["pos"])
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    ops.mrope_qk(q, k, pos, SECTIONS, THETA, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    _compare(qo, ko, inp, what=f"hq={hq} hk={hk}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hq,hk", [(1, 1), (7, 5), (16, 8), (40, 40)])
def test_mrope_head_counts_past_one_wave(dtype, hq, hk):
    """More (token, head-pass) units than warps resident at once: each warp then
    takes whole tokens, U head passes at a time, instead of one pass each."""
    heads_per_pass = 4 if dtype == "bf16" else 2  # head_dim 128: 32 lanes / (64 / E)
    passes = -(-(hq + hk) // heads_per_pass)
    tokens = (resident_threads() // 32) // passes + 5
    inp = inputs.mrope_inputs(tokens, n_q_heads=hq, n_k_heads=hk, dtype=dtype, seed=hq + 100 * hk)
    qo, ko = _run(inp)
    _compare(qo, ko, inp, dtype=dtype, what=f"{dtype} {tokens} tokens hq={hq} hk={hk}")


def test_mrope_theta_values():
    for theta in (10000.0, 1e6, 5e5):
        inp = inputs.mrope_inputs(50, seed=int(theta) % 1000)
        qo, ko = _run(inp, theta=theta)
        _compare(qo, ko, inp, theta=theta, what=f"theta={theta}")


def test_mrope_misaligned_and_guarded():
    inp = inputs.mrope_inputs(11, seed=43)
    q = misaligned(dev(inp["q"]))
    k = misaligned(dev(inp["k"]), 2)
    qo = Guarded(tuple(inp["q"].shape), torch.bfloat16, offset=3)
    ko = Guarded(tuple(inp["k"].shape), torch.bfloat16)
    ops.mrope_qk(q, k, dev(inp["pos"]), SECTIONS, THETA, q_out=qo.t, k_out=ko.t)
    torch.cuda.synchronize()
    qo.check()
    ko.check()
    _compare(qo.t, ko.t, inp, what="misaligned")


def test_mrope_guarded_vector_path(family):
    inp = inputs.mrope_inputs(33, seed=44)
    qo = Guarded(tuple(inp["q"].shape), torch.bfloat16)
    ko = Guarded(tuple(inp["k"].shape), torch.bfloat16)
    ops.mrope_qk(dev(inp["q"]), dev(inp["k"]), dev(inp["pos"]), SECTIONS, THETA, q_out=qo.t, k_out=ko.t)
    torch.cuda.synchronize()
    qo.check()
    ko.check()
    _compare(qo.t, ko.t, inp)


def test_mrope_empty():
    q = torch.empty(0, 16, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    pos = torch.empty(3, 0, dtype=torch.int32, device="cuda")
    ops.mrope_qk(q, k, pos)
    torch.cuda.synchronize()
