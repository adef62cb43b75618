"""Fused softmax + top-k sampling on the GPU against the oracle: the sampled
token bit for bit (the decision is taken in fp32 on both sides), its
probability within the fp32 bound."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs
from gpu_util import Guarded, dev
from tolerance import to_f64

pytestmark = pytest.mark.gpu


def _run(inp, k, temp):
    tok, prob = ops.topk_sample(dev(inp["logits"]), dev(inp["gumbel"]), k, temp)
    torch.cuda.synchronize()
    return tok.cpu().numpy(), to_f64(prob)


def _check(inp, k, temp, what=""):
    tok, prob = _run(inp, k, temp)
    t_ref, p_ref = oracle.get().topk_sample(inp["logits"], inp["gumbel"], k, temp)
    assert np.array_equal(tok, t_ref), f"{what}: tokens differ at {np.flatnonzero(tok != t_ref)[:5]}"
    np.testing.assert_allclose(prob, p_ref, rtol=1e-5, atol=0, err_msg=what)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("vocab,k", [(1, 1), (63, 5), (4096, 50), (4097, 64), (3072, 1),
                                     (151936, 50), (262144, 64), (10000, 20)])
def test_topk_sample_shapes(dtype, vocab, k):
    inp = inputs.topk_inputs(5, vocab, k, dtype, seed=vocab + k)
    _check(inp, k, 0.8, f"{dtype} V={vocab} k={k}")


@pytest.mark.parametrize("temp", [0.3, 1.0, 1.7])
def test_topk_sample_temperatures_many_rows(temp):
    inp = inputs.topk_inputs(257, 20000, 40, "bf16", seed=int(temp * 10))
    _check(inp, 40, temp, f"T={temp}")


def test_topk_sample_ties_go_to_lower_index():
    """Coarse logits (multiples of 0.5) tie constantly; the candidates and ranks
    must follow (logit desc, index asc) exactly."""
    rng = np.random.default_rng(3)
    lg = torch.from_numpy(np.round(rng.standard_normal((16, 30000)) * 2) / 2).float()
    for dt in (torch.bfloat16, torch.float32):
        inp = {"logits": lg.to(dt), "gumbel": torch.from_numpy(rng.gumbel(size=(16, 64)).astype(np.float32))}
        _check(inp, 64, 1.0, f"ties {dt}")
        inp["gumbel"] = torch.zeros(16, 64)
        tok, _ = _run(inp, 64, 1.0)  # no noise: greedy, first index of the maximum
        assert np.array_equal(tok, np.argmax(lg.to(dt).float().numpy(), axis=1))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_topk_sample_flat_spread_and_outlier_rows(dtype):
    """Rows whose k largest values are not all near the largest one, and rows
    where one value repeats everywhere: constant logits (the k lowest indices
    win), three outliers far above N(0,1) noise (fewer than k values within
    two binades of the largest), magnitudes spread over 2^-60 .. 2^60 of both
    signs, and all-negative logits."""
    rng = np.random.default_rng(17)
    v, k = 20000, 50
    lg = np.empty((5, v))
    lg[0] = 1.25
    lg[1] = rng.standard_normal(v)
    lg[1, [7, 5000, 19999]] = [9000.0, 8000.0, 7000.0]
    lg[2] = rng.choice([-1.0, 1.0], v) * np.exp2(rng.uniform(-60, 60, v))
    lg[3] = -np.abs(rng.standard_normal(v)) * 4 - 1.0
    lg[4] = np.round(rng.standard_normal(v) * 3)
    inp = {"logits": torch.from_numpy(lg).float().to(dtype),
           "gumbel": torch.from_numpy(rng.gumbel(size=(5, k)).astype(np.float32))}
    _check(inp, k, 1.0, f"flat/spread/outliers {dtype}")


def test_topk_sample_winner_in_last_slice_and_greedy():
    inp = inputs.topk_inputs(4, 151936, 8, "bf16", seed=9)
    lg = inp["logits"].clone()
    lg[0, -1] = 40.0
    lg[1, 4095] = 40.0
    lg[2, 4096] = 40.0
    lg[3, 0] = 40.0
    inp["logits"] = lg
    tok, prob = _run({"logits": lg, "gumbel": torch.zeros(4, 1)}, 1, 1.0)
    assert list(tok) == [151935, 4095, 4096, 0] and np.all(prob == 1.0)
    _check(inp, 8, 1.0, "winners at slice edges")


def test_topk_sample_distribution():
    """Over 20,000 rows of one logit vector with fresh draws, the GPU's token
    frequencies match the top-k softmax (chi-square)."""
    rng = np.random.default_rng(11)
    base = rng.standard_normal(1000) * 2
    n, k, temp = 20000, 6, 0.9
    lg = torch.from_numpy(np.tile(base, (n, 1))).float()
    g = torch.from_numpy(rng.gumbel(size=(n, k)).astype(np.float32))
    tok, _ = _run({"logits": lg, "gumbel": g}, k, temp)
    top = np.argsort(-base.astype(np.float32), kind="stable")[:k]
    p = np.exp(base[top] / temp - base[top].max() / temp)
    p /= p.sum()
    counts = np.array([np.count_nonzero(tok == t) for t in top])
    assert counts.sum() == n
    chi2 = np.sum((counts - n * p) ** 2 / (n * p))
    assert chi2 < 25.0, (counts, n * p)


COUNTER_BYTES = 1 << 18  # the workspace's arrival counters (one per row, up to 65535 rows)


def test_topk_sample_workspace_is_exact_and_guarded():
    rows, vocab, k = 5, 50000, 32
    need = ops.topk_sample_workspace(rows, vocab, k)
    assert need == COUNTER_BYTES + rows * ((vocab + 4095) // 4096) * k * 8
    ws = Guarded((need // 4,), torch.float32)  # canaries on both sides of the workspace
    w8 = ws.t.view(torch.uint8)
    ops.topk_sample_prepare(w8)
    inp = inputs.topk_inputs(rows, vocab, k, "bf16", seed=12)
    tok, prob = ops.topk_sample(dev(inp["logits"]), dev(inp["gumbel"]), k, 1.1, workspace=w8)
    torch.cuda.synchronize()
    ws.check()
    assert not w8[:COUNTER_BYTES].any()  # the call left its counters at zero
    t_ref, p_ref = oracle.get().topk_sample(inp["logits"], inp["gumbel"], k, 1.1)
    assert np.array_equal(tok.cpu().numpy(), t_ref)


def test_topk_sample_one_workspace_for_many_shapes():
    """The counters sit at a fixed place and every call leaves them at zero, so
    one prepared workspace serves calls of any shape in turn."""
    shapes = ((5, 151936, 50), (33, 70000, 64), (3, 4096, 7), (64, 151936, 50), (1, 100, 1))
    need = max(ops.topk_sample_workspace(r, v, k) for r, v, k in shapes)
    w8 = ops.topk_sample_prepare(torch.empty(need, dtype=torch.uint8, device="cuda"))
    for i, (r, v, k) in enumerate(shapes):
        inp = inputs.topk_inputs(r, v, k, "bf16", seed=40 + i)
        tok, prob = ops.topk_sample(dev(inp["logits"]), dev(inp["gumbel"]), k, 0.9, workspace=w8)
        t_ref, p_ref = oracle.get().topk_sample(inp["logits"], inp["gumbel"], k, 0.9)
        assert np.array_equal(tok.cpu().numpy(), t_ref), (r, v, k)
        np.testing.assert_allclose(to_f64(prob), p_ref, rtol=1e-5, atol=0)
    assert not w8[:COUNTER_BYTES].any()


def test_topk_sample_flags_a_workspace_whose_counters_were_not_cleared():
    """Counters left non-zero (a workspace never prepared) are reported in the
    device error word; the kernel still completes."""
    rows, vocab, k = 2, 10000, 8
    w8 = torch.full((ops.topk_sample_workspace(rows, vocab, k),), 0xA5, dtype=torch.uint8,
                    device="cuda")
    inp = inputs.topk_inputs(rows, vocab, k, "bf16", seed=3)
    ops.topk_sample(dev(inp["logits"]), dev(inp["gumbel"]), k, 1.0, workspace=w8)
    torch.cuda.synchronize()
    assert ops.device_errors(clear=True) == 4  # AROPS_DEVICE_ERR_WORKSPACE


def test_topk_sample_empty_rows():
    lg = torch.empty(0, 100, dtype=torch.bfloat16, device="cuda")
    tok, prob = ops.topk_sample(lg, torch.empty(0, 4, device="cuda"), 4, 1.0)
    torch.cuda.synchronize()
    assert tok.numel() == 0
