"""Fused softmax + top-k sampling on the GPU against the oracle: the sampled
token bit for bit (the decision is taken in fp32 on both sides), its
probability within the fp32 bound.  Every kernel is run: the cluster kernels
(registers or shared memory), the streaming kernel (one CTA a row) and the
slice kernel."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs
from gpu_util import Guarded, dev
from tolerance import to_f64

pytestmark = pytest.mark.gpu


MODES = {"slice": 0, "cluster": 1, "smem": 2, "row": 3}  # arops_set_topk_cluster


@pytest.fixture(params=["cluster", "smem", "row", "slice"])
def kernel(request):
    old = ops.set_topk_cluster(MODES[request.param])
    yield request.param
    ops.set_topk_cluster(old)


@pytest.fixture
def slice_kernel():
    old = ops.set_topk_cluster(False)
    yield
    ops.set_topk_cluster(old)


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
def test_topk_sample_shapes(dtype, vocab, k, kernel):
    inp = inputs.topk_inputs(5, vocab, k, dtype, seed=vocab + k)
    _check(inp, k, 0.8, f"{dtype} V={vocab} k={k}")


@pytest.mark.parametrize("temp", [0.3, 1.0, 1.7])
def test_topk_sample_temperatures_many_rows(temp, kernel):
    inp = inputs.topk_inputs(257, 20000, 40, "bf16", seed=int(temp * 10))
    _check(inp, 40, temp, f"T={temp}")


def test_topk_sample_ties_go_to_lower_index(kernel):
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
def test_topk_sample_flat_spread_and_outlier_rows(dtype, kernel):
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


def test_topk_sample_winner_in_last_slice_and_greedy(kernel):
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


def test_topk_sample_distribution(kernel):
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


def test_topk_sample_workspace_is_exact_and_guarded(slice_kernel):
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


def test_topk_sample_one_workspace_for_many_shapes(kernel):
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


def test_topk_sample_flags_a_workspace_whose_counters_were_not_cleared(slice_kernel):
    """Counters left non-zero (a workspace never prepared) are reported in the
    device error word; the kernel still completes."""
    rows, vocab, k = 2, 10000, 8
    w8 = torch.full((ops.topk_sample_workspace(rows, vocab, k),), 0xA5, dtype=torch.uint8,
                    device="cuda")
    inp = inputs.topk_inputs(rows, vocab, k, "bf16", seed=3)
    ops.topk_sample(dev(inp["logits"]), dev(inp["gumbel"]), k, 1.0, workspace=w8)
    torch.cuda.synchronize()
    assert ops.device_errors(clear=True) == 4  # AROPS_DEVICE_ERR_WORKSPACE


def test_topk_sample_empty_rows(kernel):
    lg = torch.empty(0, 100, dtype=torch.bfloat16, device="cuda")
    tok, prob = ops.topk_sample(lg, torch.empty(0, 4, device="cuda"), 4, 1.0)
    torch.cuda.synchronize()
    assert tok.numel() == 0


# Cluster sizes 1 .. 16 and their edges (a CTA per 4096 logits up to 16 CTAs,
# then up to 16384 logits a CTA), rows of 16-byte-aligned and unaligned starts.
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("vocab", [8, 4096, 4104, 8192, 8200, 16385, 32769, 65536, 65544,
                                   131080, 196608, 262136])
def test_topk_sample_cluster_sizes(dtype, vocab):
    k = min(64, vocab)
    inp = inputs.topk_inputs(3, vocab, k, dtype, seed=vocab)
    _check(inp, k, 0.7, f"{dtype} V={vocab}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_topk_sample_unaligned_rows(kernel, dtype):
    """Logits that start 2 or 4 bytes past a 16-byte boundary take the
    element-by-element loads."""
    rows, vocab = 4, 151936
    inp = inputs.topk_inputs(rows, vocab, 50, "f32", seed=5)
    lg = inp["logits"].to(dtype)
    flat = torch.empty(rows * vocab + 1, dtype=dtype, device="cuda")
    view = flat[1:].view(rows, vocab)  # contiguous rows, start one element past the boundary
    view.copy_(dev(lg))
    assert view.data_ptr() % 16 != 0
    tok, prob = ops.topk_sample(view, dev(inp["gumbel"]), 50, 1.0)
    t_ref, p_ref = oracle.get().topk_sample(lg, inp["gumbel"], 50, 1.0)
    assert np.array_equal(tok.cpu().numpy(), t_ref)
    np.testing.assert_allclose(to_f64(prob), p_ref, rtol=1e-5, atol=0)


def test_topk_sample_cluster_kernel_leaves_the_workspace_alone():
    """A few rows of up to 32768 logits always take the cluster kernel (clusters
    of at most 8 CTAs, the portable size, dozens of which a B200 holds at
    once); it reads no workspace byte and writes none."""
    rows, vocab, k = 6, 32768, 64
    w8 = torch.full((ops.topk_sample_workspace(rows, vocab, k),), 0x5A, dtype=torch.uint8,
                    device="cuda")
    inp = inputs.topk_inputs(rows, vocab, k, "bf16", seed=21)
    tok, _ = ops.topk_sample(dev(inp["logits"]), dev(inp["gumbel"]), k, 1.0, workspace=w8)
    torch.cuda.synchronize()
    assert bool((w8 == 0x5A).all())
    assert ops.device_errors(clear=True) == 0
    t_ref, _ = oracle.get().topk_sample(inp["logits"], inp["gumbel"], k, 1.0)
    assert np.array_equal(tok.cpu().numpy(), t_ref)


@pytest.mark.parametrize("rows", [1, 7, 12, 64, 300])
def test_topk_sample_kernels_agree_bit_for_bit(rows):
    """The four kernels give the same tokens and the same probabilities, bit
    for bit, over many rows (mode 1 at 12 rows of 151,936: the register kernel
    on 8-CTA clusters; mode 3 at 300 rows: two rows and more a CTA)."""
    inp = inputs.topk_inputs(rows, 151936, 50, "bf16", seed=rows)
    lg, g = dev(inp["logits"]), dev(inp["gumbel"])
    out = {}
    for mode in (1, 2, 3, 0):
        old = ops.set_topk_cluster(mode)
        try:
            tok, prob = ops.topk_sample(lg, g, 50, 0.8)
            torch.cuda.synchronize()
        finally:
            ops.set_topk_cluster(old)
        out[mode] = (tok.cpu(), prob.cpu())
    for mode in (1, 2, 3):
        assert torch.equal(out[mode][0], out[0][0]), mode
        assert torch.equal(out[mode][1], out[0][1]), mode


@pytest.mark.parametrize("rows", [5, 20, 100])
def test_topk_sample_in_a_graph_with_pdl(rows):
    """Sampling captured in a CUDA graph behind another kernel, with
    programmatic dependent launch (the end of a decode step): the register
    cluster kernel (5 rows), the shared-memory one (20 rows) and the streaming
    one (100 rows) replayed on new logits and draws each time, every replay
    against the oracle."""
    vocab, k = 151936, 50
    lg = torch.empty(rows, vocab, dtype=torch.bfloat16, device="cuda")
    g = torch.empty(rows, k, dtype=torch.float32, device="cuda")
    x = torch.randn(rows, 2048, device="cuda").to(torch.bfloat16)
    res = torch.randn(rows, 2048, device="cuda").to(torch.bfloat16)
    gamma = torch.ones(2048, device="cuda").to(torch.bfloat16)
    y = torch.empty_like(x)
    tok = torch.empty(rows, dtype=torch.int32, device="cuda")
    prob = torch.empty(rows, dtype=torch.float32, device="cuda")
    ws = ops.topk_sample_prepare(torch.empty(ops.topk_sample_workspace(rows, vocab, k),
                                             dtype=torch.uint8, device="cuda"))
    old = ops.set_pdl(True)
    try:
        def step():
            ops.add_rmsnorm(x, res, gamma, 1e-6, y=y)
            ops.topk_sample(lg, g, k, 0.9, workspace=ws, token_out=tok, prob_out=prob)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            lg.zero_()
            g.zero_()
            step()  # warm-up outside the capture
        torch.cuda.current_stream().wait_stream(s)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for rep in range(3):
            inp = inputs.topk_inputs(rows, vocab, k, "bf16", seed=100 + rep)
            lg.copy_(inp["logits"])
            g.copy_(inp["gumbel"])
            graph.replay()
            torch.cuda.synchronize()
            t_ref, p_ref = oracle.get().topk_sample(inp["logits"], inp["gumbel"], k, 0.9)
            assert np.array_equal(tok.cpu().numpy(), t_ref), f"replay {rep}"
            np.testing.assert_allclose(to_f64(prob), p_ref, rtol=1e-5, atol=0)
        assert ops.device_errors(clear=True) == 0
    finally:
        ops.set_pdl(old)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_topk_sample_ties_across_cta_boundaries(kernel, dtype):
    """Equal maxima that straddle the boundary between two CTAs' chunks (the
    cluster kernel cuts a 151,936-logit row into chunks of 9,496): the
    candidates must be the lowest indices, crossing the boundary in order.  A
    run of 11 ties is taken whole by the first round; a run of 100 with k = 50
    splits the boundary bin and takes the digit rounds."""
    rng = np.random.default_rng(23)
    vocab, rows = 151936, 4
    lg = rng.standard_normal((rows, vocab))
    lg[0, 9490:9501] = 50.0   # 11 ties over the boundary at 9,496
    lg[1, 9446:9546] = 50.0   # 100 ties, 50 on each side
    lg[2, 18980:19000] = 50.0  # 20 ties over the boundary at 18,992
    lg[3, 151900:] = 50.0     # ties at the end of the last chunk
    for k in (8, 50):
        g = rng.gumbel(size=(rows, k)).astype(np.float32)
        inp = {"logits": torch.from_numpy(lg).float().to(dtype), "gumbel": torch.from_numpy(g)}
        _check(inp, k, 1.0, f"boundary ties k={k} {dtype}")
        tok, _ = _run({"logits": inp["logits"], "gumbel": torch.zeros(rows, k)}, k, 1.0)
        assert list(tok) == [9490, 9446, 18980, 151900]  # greedy: the first index of the maximum


@pytest.mark.parametrize("mode,touched", [(1, False), (2, False), (3, False), (0, True)])
def test_topk_sample_workspace_use_by_kernel(mode, touched):
    """The cluster kernels (one row: registers; 64 rows, more than a B200 holds
    clusters of 16 CTAs at once: shared memory) leave the workspace as it was;
    the slice kernel's candidates land in it."""
    vocab, k = 151936, 50
    old = ops.set_topk_cluster(mode)
    try:
        _workspace_use(vocab, k, touched)
    finally:
        ops.set_topk_cluster(old)


def _workspace_use(vocab, k, touched):
    for rows in (1, 64):
        n = ops.topk_sample_workspace(rows, vocab, k)
        w8 = torch.full((n,), 0xA5, dtype=torch.uint8, device="cuda")
        w8[:COUNTER_BYTES] = 0
        inp = inputs.topk_inputs(rows, vocab, k, "bf16", seed=rows)
        tok, _ = ops.topk_sample(dev(inp["logits"]), dev(inp["gumbel"]), k, 1.0, workspace=w8)
        torch.cuda.synchronize()
        assert bool((w8[COUNTER_BYTES:] != 0xA5).any()) == touched, rows
        assert not w8[:COUNTER_BYTES].any()
        t_ref, _ = oracle.get().topk_sample(inp["logits"], inp["gumbel"], k, 1.0)
        assert np.array_equal(tok.cpu().numpy(), t_ref)


_FIRST_CALL_CAPTURED = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import oracle, swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs
rows, vocab, k = {rows}, 151936, 50
inp = inputs.topk_inputs(rows, vocab, k, "bf16", seed=rows)
lg, g = inp["logits"].cuda(), inp["gumbel"].cuda()
tok = torch.empty(rows, dtype=torch.int32, device="cuda")
prob = torch.empty(rows, dtype=torch.float32, device="cuda")
ws = ops.topk_sample_prepare(torch.empty(ops.topk_sample_workspace(rows, vocab, k), dtype=torch.uint8, device="cuda"))
torch.cuda.synchronize()
graph = torch.cuda.CUDAGraph()
with torch.cuda.graph(graph):  # the process's first sampling call
    ops.topk_sample(lg, g, k, 0.9, workspace=ws, token_out=tok, prob_out=prob)
graph.replay()
torch.cuda.synchronize()
t_ref, _ = oracle.get().topk_sample(inp["logits"], inp["gumbel"], k, 0.9)
assert np.array_equal(tok.cpu().numpy(), t_ref)
print("ok")
"""


@pytest.mark.parametrize("rows", [5, 40, 100])
def test_topk_sample_first_call_inside_a_graph_capture(rows):
    """A fresh process whose first sampling call is made while a CUDA graph is
    being captured (the one-time occupancy lookup and kernel attributes of the
    cluster kernels run inside the capture): register kernel (5 rows),
    shared-memory kernel (40 rows) and streaming kernel (100 rows)."""
    import os
    import subprocess
    import sys

    tests = os.path.dirname(os.path.abspath(__file__))
    code = _FIRST_CALL_CAPTURED.format(root=os.path.dirname(tests), tests=tests, rows=rows)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stderr[-2000:]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("offset", [0, 1])
def test_topk_sample_ten_rows(dtype, offset):
    """Ten rows of 151,936 logits, 16-byte-aligned or one element past the
    boundary: more rows than a B200 holds 16-CTA clusters of the register
    kernel at once, so the default takes it on 8-CTA clusters (40 logits a
    thread)."""
    rows, vocab, k = 10, 151936, 50
    inp = inputs.topk_inputs(rows, vocab, k, "f32", seed=77 + offset)
    lg = inp["logits"].to(dtype)
    flat = torch.empty(rows * vocab + offset, dtype=dtype, device="cuda")
    view = flat[offset:].view(rows, vocab)
    view.copy_(dev(lg))
    tok, prob = ops.topk_sample(view, dev(inp["gumbel"]), k, 0.7)
    t_ref, p_ref = oracle.get().topk_sample(lg, inp["gumbel"], k, 0.7)
    assert np.array_equal(tok.cpu().numpy(), t_ref)
    np.testing.assert_allclose(to_f64(prob), p_ref, rtol=1e-5, atol=0)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows", [4, 160])
def test_topk_sample_streaming_list_overflow(dtype, rows):
    """The streaming kernel's candidate list running full, against the oracle:
    ascending rows (every stage beats the ones before it), a first stage far
    below the rest (its floor lets all of the next stage through), constant
    rows (every key ties), and coarse values with long runs of ties; 4 rows,
    and 160 (more rows than SMs: CTAs that walk two rows)."""
    rng = np.random.default_rng(31 + rows)
    v, k = 151936, 50
    lg = np.empty((rows, v))
    for r in range(rows):
        kind = r % 4
        if kind == 0:
            lg[r] = np.linspace(-4.0, 4.0, v) + r * 1e-3
        elif kind == 1:
            lg[r] = rng.standard_normal(v)
            lg[r, :16384] = -30.0 + rng.standard_normal(16384) * 0.01
        elif kind == 2:
            lg[r] = 0.5 + r
        else:
            lg[r] = np.round(rng.standard_normal(v) * 2) / 2
    inp = {"logits": torch.from_numpy(lg).float().to(dtype),
           "gumbel": torch.from_numpy(rng.gumbel(size=(rows, k)).astype(np.float32))}
    old = ops.set_topk_cluster(3)
    try:
        _check(inp, k, 1.0, f"list overflow {dtype} rows={rows}")
        tok, _ = _run({"logits": inp["logits"], "gumbel": torch.zeros(rows, k)}, k, 1.0)
        assert np.array_equal(tok, np.argmax(inp["logits"].float().numpy(), axis=1))
        assert ops.device_errors(clear=True) == 0
    finally:
        ops.set_topk_cluster(old)
