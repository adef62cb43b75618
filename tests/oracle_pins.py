"""Pins for the fp64 oracle: checks that tie it to something other than itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` build and raises
AssertionError when the build disagrees with a closed form, an invariant, a
textbook special case or a library routine.  ``test_oracle_pins.py`` runs every
pin on the real oracle; ``test_oracle_mutants.py`` runs them on builds with one
planted mistake each and requires that some pin fails.

None of these re-types the oracle's own formula: each compares against an
independent statement (a closed form worked out by hand, an identity the
operator must satisfy, the complex-exponential form of a rotation, the logistic
function written through tanh, or torch's own dtype casts).
"""
from __future__ import annotations

import math

import numpy as np
import torch

# ---------------------------------------------------------------------------
# bf16 rounding and decoding
# ---------------------------------------------------------------------------


def _torch_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def _torch_f32_to_bf16_bits(v32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(v32.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().astype(np.uint16)


def pin_bf16_decode_matches_torch(orc):
    """Decoding every finite bf16 pattern agrees with torch's exact widening."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    mine = orc.bf16_value(bits)
    ref = _torch_bits_to_f64(bits)
    finite = np.isfinite(ref)
    assert np.array_equal(mine[finite], ref[finite])
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.array_equal(np.isinf(mine), np.isinf(ref))


def pin_bf16_round_trip(orc):
    """Every finite bf16 value rounds to itself."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = _torch_bits_to_f64(bits)
    finite = np.isfinite(vals)
    back = orc.round_bf16(vals[finite])
    assert np.array_equal(back, bits[finite])


def pin_bf16_round_matches_torch_on_fp32_values(orc):
    """For values that are exact in fp32, direct fp64->bf16 rounding must agree
    with torch's fp32->bf16 round-to-nearest-even cast, across all binades,
    subnormals and exact ties."""
    rng = np.random.default_rng(1234)
    raw = rng.integers(0, 1 << 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    v32 = raw.view(np.float32)
    v32 = v32[np.isfinite(v32)]
    # exact ties: bf16 value + half an ulp (low 16 bits = 0x8000)
    ties = ((raw[:20_000] & 0xFFFF0000) | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    v32 = np.concatenate([v32, ties])
    mine = orc.round_bf16(v32.astype(np.float64))
    ref = _torch_f32_to_bf16_bits(v32)
    ok = ~np.isnan(v32)
    assert np.array_equal(mine[ok], ref[ok])


def pin_bf16_round_special_cases(orc):
    """Hand-worked cases, including ones where rounding through fp32 first
    would give a different (double-rounded) answer."""
    cases = [
        (1.0, 0x3F80),
        (-2.0, 0xC000),
        (1.0 + 2.0 ** -8, 0x3F80),               # tie -> even (mantissa 0)
        (1.0 + 3 * 2.0 ** -8, 0x3F82),           # tie -> even (mantissa 2)
        (1.0 + 2.0 ** -8 + 2.0 ** -30, 0x3F81),  # just above a tie: direct rounding goes up
        (1.0 + 2.0 ** -8 - 2.0 ** -40, 0x3F80),  # just below a tie
        (2.0 ** -133, 0x0001),                   # smallest subnormal
        (2.0 ** -134, 0x0000),                   # tie between 0 and the smallest subnormal
        (1.5 * 2.0 ** -134, 0x0001),
        (2.0 ** -126 - 2.0 ** -140, 0x0080),     # rounds up into the smallest normal
        ((2 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),  # largest finite
        ((2 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),  # tie above the largest finite -> inf
        ((2 - 2.0 ** -8 - 2.0 ** -20) * 2.0 ** 127, 0x7F7F),
        (-0.0, 0x8000),
        (float("inf"), 0x7F80),
        (float("-inf"), 0xFF80),
    ]
    vals = np.array([c[0] for c in cases], dtype=np.float64)
    want = np.array([c[1] for c in cases], dtype=np.uint16)
    got = orc.round_bf16(vals)
    bad = [(cases[i][0], hex(got[i]), hex(want[i])) for i in range(len(cases)) if got[i] != want[i]]
    assert not bad, bad
    nan_bits = orc.round_bf16(np.array([float("nan")]))[0]
    assert (nan_bits & 0x7F80) == 0x7F80 and (nan_bits & 0x7F) != 0


# ---------------------------------------------------------------------------
# RMSNorm
# ---------------------------------------------------------------------------


def pin_rmsnorm_constant_rows(orc):
    """Row of constant value a: y_i = gamma_i * a / sqrt(a^2 + eps)."""
    H = 64
    rng = np.random.default_rng(5)
    gamma = 1.0 + 0.1 * rng.standard_normal(H)
    a = np.array([1.0, -3.0, 0.25, 1e-3, 7.5])
    x = np.repeat(a[:, None], H, axis=1)
    for eps in (1e-6, 0.0, 0.5):
        y = orc.rmsnorm(x, gamma, eps)
        want = gamma[None, :] * (a / np.sqrt(a * a + eps))[:, None]
        np.testing.assert_allclose(y, want, rtol=1e-14, atol=0)


def pin_rmsnorm_one_hot(orc):
    """One nonzero entry a at index k: y_k = gamma_k * a / sqrt(a^2/H + eps),
    every other output exactly 0."""
    H = 48
    gamma = np.linspace(0.5, 1.5, H)
    eps = 1e-6
    for k, a in ((0, 2.0), (17, -0.75), (47, 30.0)):
        x = np.zeros((1, H))
        x[0, k] = a
        y = orc.rmsnorm(x, gamma, eps)
        want = gamma[k] * a / math.sqrt(a * a / H + eps)
        assert abs(y[0, k] - want) <= 1e-14 * abs(want)
        rest = np.delete(y[0], k)
        assert np.all(rest == 0.0)


def pin_rmsnorm_small_closed_form(orc):
    """x = (3, 4), eps = 0: mean(x^2) = 25/2, so y = x * sqrt(2)/5."""
    y = orc.rmsnorm(np.array([[3.0, 4.0]]), np.array([1.0, 1.0]), 0.0)
    np.testing.assert_allclose(y[0], [3 * math.sqrt(2) / 5, 4 * math.sqrt(2) / 5], rtol=1e-15)
    y = orc.rmsnorm(np.array([[3.0, 4.0]]), np.array([2.0, -1.0]), 0.0)
    np.testing.assert_allclose(y[0], [6 * math.sqrt(2) / 5, -4 * math.sqrt(2) / 5], rtol=1e-15)


def pin_rmsnorm_unit_rms(orc):
    """gamma = 1: rms(y) = sqrt(m / (m + eps)) with m = mean(x^2); = 1 at eps = 0."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((16, 1000)) * rng.uniform(0.01, 10, size=(16, 1))
    gamma = np.ones(1000)
    for eps in (0.0, 1e-6, 1e-2):
        y = orc.rmsnorm(x, gamma, eps)
        m = np.mean(x * x, axis=1)
        rms = np.sqrt(np.mean(y * y, axis=1))
        np.testing.assert_allclose(rms, np.sqrt(m / (m + eps)), rtol=1e-13)


def pin_rmsnorm_zero_row(orc):
    y = orc.rmsnorm(np.zeros((2, 32)), np.ones(32), 1e-6)
    assert np.all(y == 0.0)


def pin_rmsnorm_scale_invariance(orc):
    """eps = 0: y(2^k x) == y(x) bit for bit (power-of-two scaling is exact)."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((4, 256))
    gamma = 1 + 0.1 * rng.standard_normal(256)
    y0 = orc.rmsnorm(x, gamma, 0.0)
    for k in (-20, -3, 5, 40):
        assert np.array_equal(orc.rmsnorm(x * 2.0 ** k, gamma, 0.0), y0)


def pin_rmsnorm_equivariance(orc):
    """Permuting rows permutes outputs; permuting channels together with gamma
    permutes outputs; scaling gamma scales outputs."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((6, 128))
    gamma = 1 + 0.1 * rng.standard_normal(128)
    y = orc.rmsnorm(x, gamma, 1e-6)
    rp = rng.permutation(6)
    np.testing.assert_allclose(orc.rmsnorm(x[rp], gamma, 1e-6), y[rp], rtol=1e-14)
    cp = rng.permutation(128)
    np.testing.assert_allclose(orc.rmsnorm(x[:, cp], gamma[cp], 1e-6), y[:, cp], rtol=1e-13)
    np.testing.assert_allclose(orc.rmsnorm(x, 2 * gamma, 1e-6), 2 * y, rtol=1e-15)


# ---------------------------------------------------------------------------
# residual add + RMSNorm
# ---------------------------------------------------------------------------


def _bf16_tensor(shape, seed, std=1.0):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal(shape) * std).float().bfloat16()


def pin_add_rmsnorm_residual_exact(orc):
    """residual_out is the bf16 rounding of the exact sum x + residual; torch's
    fp32 add (exact for these operands) followed by its bf16 cast gives it."""
    x = _bf16_tensor((8, 512), 10)
    r = _bf16_tensor((8, 512), 11, std=2.0)
    gamma = _bf16_tensor((512,), 12) * 0.1 + 1
    _, res_out = orc.add_rmsnorm(x, r, gamma.bfloat16(), 1e-6, "bf16")
    want = (x.float() + r.float()).bfloat16().double().numpy()
    assert np.array_equal(res_out, want)
    # fp32 activations: the fp32 sum of two fp32 numbers, rounded once
    xf = torch.from_numpy(np.random.default_rng(13).standard_normal((4, 256))).float()
    rf = torch.from_numpy(np.random.default_rng(14).standard_normal((4, 256)) * 3).float()
    _, res_f = orc.add_rmsnorm(xf, rf, torch.ones(256), 1e-6, "f32")
    assert np.array_equal(res_f, (xf + rf).double().numpy())


def pin_add_rmsnorm_is_add_then_norm(orc):
    """y == RMSNorm(bf16(x + residual)), and x = 0 reduces to RMSNorm(residual)."""
    x = _bf16_tensor((8, 512), 20)
    r = _bf16_tensor((8, 512), 21, std=2.0)
    gamma = (_bf16_tensor((512,), 22) * 0.1 + 1).bfloat16()
    y, res_out = orc.add_rmsnorm(x, r, gamma, 1e-6, "bf16")
    summed = (x.float() + r.float()).bfloat16()
    np.testing.assert_array_equal(y, orc.rmsnorm(summed, gamma, 1e-6))
    y0, res0 = orc.add_rmsnorm(torch.zeros_like(r), r, gamma, 1e-6, "bf16")
    assert np.array_equal(res0, r.double().numpy())
    np.testing.assert_array_equal(y0, orc.rmsnorm(r, gamma, 1e-6))


# ---------------------------------------------------------------------------
# LayerNorm
# ---------------------------------------------------------------------------


def pin_layernorm_two_element_closed_form(orc):
    """x = (a, b): mean (a+b)/2, variance ((a-b)/2)^2, so at eps = 0 the row
    normalises to (+1, -1) * sign(a-b): y = (gamma_0 + beta_0, -gamma_1 + beta_1)."""
    gamma = np.array([1.5, -0.5])
    beta = np.array([0.25, 2.0])
    for a, b in ((3.0, 1.0), (-2.0, 7.0), (1e-3, -4e-3)):
        y = orc.layernorm(np.array([[a, b]]), gamma, beta, 0.0)
        sgn = 1.0 if a > b else -1.0
        np.testing.assert_allclose(y[0], [sgn * gamma[0] + beta[0], -sgn * gamma[1] + beta[1]],
                                   rtol=1e-14, atol=1e-14)
    # with eps: the deviation is divided by sqrt(d^2 + eps), d = (a - b)/2
    y = orc.layernorm(np.array([[3.0, 1.0]]), np.ones(2), np.zeros(2), 0.5)
    np.testing.assert_allclose(y[0], [1 / math.sqrt(1.5), -1 / math.sqrt(1.5)], rtol=1e-15)


def pin_layernorm_constant_row_is_beta(orc):
    """A constant row has zero deviation: y = beta exactly (eps > 0)."""
    beta = np.linspace(-1, 1, 32)
    y = orc.layernorm(np.full((3, 32), 7.25), np.full(32, 3.0), beta, 1e-6)
    assert np.array_equal(y, np.tile(beta, (3, 1)))


def pin_layernorm_moments(orc):
    """gamma = 1, beta = 0, eps = 0: every output row has mean 0 and population
    variance 1; shifting the input row by a constant changes nothing."""
    rng = np.random.default_rng(60)
    x = rng.standard_normal((8, 500)) * 3 + 11
    y = orc.layernorm(x, np.ones(500), np.zeros(500), 0.0)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-13)
    np.testing.assert_allclose(y.var(axis=1), 1, rtol=1e-12)
    np.testing.assert_allclose(orc.layernorm(x + 100.0, np.ones(500), np.zeros(500), 0.0), y,
                               atol=1e-11)


def pin_layernorm_zero_mean_is_rmsnorm_plus_beta(orc):
    """On rows with mean exactly 0, LayerNorm is RMSNorm followed by + beta."""
    rng = np.random.default_rng(61)
    h = rng.standard_normal((4, 64))
    x = np.concatenate([h, -h], axis=1)  # every row sums to exactly 0
    gamma = 1 + 0.1 * rng.standard_normal(128)
    beta = rng.standard_normal(128)
    np.testing.assert_allclose(orc.layernorm(x, gamma, beta, 1e-6),
                               orc.rmsnorm(x, gamma, 1e-6) + beta, rtol=1e-13, atol=1e-14)


def pin_add_layernorm_is_add_then_norm(orc):
    x = _bf16_tensor((8, 256), 62)
    r = _bf16_tensor((8, 256), 63, std=2.0)
    gamma = (_bf16_tensor((256,), 64) * 0.1 + 1).bfloat16()
    beta = (_bf16_tensor((256,), 65) * 0.1).bfloat16()
    y, res_out = orc.add_layernorm(x, r, gamma, beta, 1e-6, "bf16")
    summed = (x.float() + r.float()).bfloat16()
    assert np.array_equal(res_out, summed.double().numpy())
    np.testing.assert_array_equal(y, orc.layernorm(summed, gamma, beta, 1e-6))


# ---------------------------------------------------------------------------
# fused softmax + top-k sampling
# ---------------------------------------------------------------------------


def pin_topk_greedy_cases(orc):
    """k = 1, or zero noise, is greedy decoding: the (first) largest logit, with
    probability 1 for k = 1; ties go to the lower index."""
    rng = np.random.default_rng(70)
    lg = rng.standard_normal((4, 300))
    lg[2, 17] = lg[2, 200] = 9.0  # a tie for the maximum
    g = rng.gumbel(size=(4, 1)).astype(np.float32)
    tok, prob = orc.topk_sample(lg, g, 1, 0.7)
    assert list(tok) == [int(np.argmax(r)) for r in lg] and tok[2] == 17
    assert np.all(prob == 1.0)
    tok, _ = orc.topk_sample(lg, np.zeros((4, 40), np.float32), 40, 1.3)
    assert list(tok) == [int(np.argmax(r)) for r in lg]


def pin_topk_probability_closed_form(orc):
    """Logits (0, ln 2, ln 3, -inf-ish ...) with k = 3, T = 1: the top-3 softmax is
    (3, 2, 1)/6 for indices (2, 1, 0); a dominant noise on rank j picks rank j."""
    lg = np.array([[0.0, math.log(2.0), math.log(3.0), -50.0, -60.0]])
    for j, (idx, p) in enumerate(((2, 0.5), (1, 1 / 3), (0, 1 / 6))):
        g = np.zeros((1, 3), np.float32)
        g[0, j] = 100.0
        tok, prob = orc.topk_sample(lg, g, 3, 1.0)
        assert tok[0] == idx
        assert abs(prob[0] - p) < 1e-15
    # temperature 2 on logits (0, ln 4): top-2 softmax of (0, ln 2) = (1/3, 2/3)
    g = np.array([[0.0, 100.0]], np.float32)
    tok, prob = orc.topk_sample(np.array([[0.0, math.log(4.0)]]), g, 2, 2.0)
    assert tok[0] == 0 and abs(prob[0] - 1 / 3) < 1e-15


def pin_topk_gumbel_max_distribution(orc):
    """Gumbel-max with i.i.d. Gumbel(0,1) draws samples the top-k softmax: over
    40,000 draws the token frequencies match the probabilities (chi-square)."""
    rng = np.random.default_rng(71)
    lg = np.array([[1.0, 0.2, 2.0, -1.0, 1.5, 0.0, -3.0, 0.7]])
    k, T, n = 5, 0.8, 40_000
    top = np.argsort(-lg[0], kind="stable")[:k]
    p = np.exp(lg[0, top] / T - np.max(lg[0, top] / T))
    p /= p.sum()
    counts = np.zeros(k)
    toks, _ = orc.topk_sample(np.repeat(lg, n, axis=0), rng.gumbel(size=(n, k)).astype(np.float32), k, T)
    for i, t in enumerate(top):
        counts[i] = np.count_nonzero(toks == t)
    assert counts.sum() == n  # only top-k tokens are ever drawn
    chi2 = np.sum((counts - n * p) ** 2 / (n * p))
    assert chi2 < 20.0, (counts, n * p, chi2)  # 4 degrees of freedom: p(chi2 > 20) < 1e-3


def pin_topk_candidate_set(orc):
    """Only the k largest logits can be drawn, whatever the noise."""
    rng = np.random.default_rng(72)
    lg = rng.standard_normal((64, 1000))
    k = 7
    toks, _ = orc.topk_sample(lg, (rng.gumbel(size=(64, k)) * 5).astype(np.float32), k, 1.0)
    for r in range(64):
        assert lg[r, toks[r]] >= np.sort(lg[r])[-k]


# ---------------------------------------------------------------------------
# M-RoPE
# ---------------------------------------------------------------------------
SECTIONS = (24, 20, 20)
THETA = 1e6
D = 128


def _rand_qk(tokens, hq=4, hk=2, d=D, seed=30):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((tokens, hq, d)), rng.standard_normal((tokens, hk, d))


def pin_mrope_position_zero_identity(orc):
    """At position 0 every angle is 0, so the output is the input, bit for bit."""
    q, k = _rand_qk(3)
    pos = np.zeros((3, 3), dtype=np.int32)
    qo, ko = orc.mrope_qk(q, k, pos, SECTIONS, THETA)
    assert np.array_equal(qo, q) and np.array_equal(ko, k)


def pin_mrope_pair_norm(orc):
    """A rotation preserves a^2 + b^2 for every pair (j, j + D/2)."""
    q, k = _rand_qk(5, seed=31)
    pos = np.array([[0, 5, 100, 1071, 77], [3, 5, 7, 0, 1], [9, 5, 0, 7, 1000]], dtype=np.int32)
    qo, ko = orc.mrope_qk(q, k, pos, SECTIONS, THETA)
    for x, o in ((q, qo), (k, ko)):
        n_in = x[..., :D // 2] ** 2 + x[..., D // 2:] ** 2
        n_out = o[..., :D // 2] ** 2 + o[..., D // 2:] ** 2
        np.testing.assert_allclose(n_out, n_in, rtol=1e-12)


def pin_mrope_section_mask(orc):
    """With only one of the rows t/h/w nonzero, exactly the pairs of that row's
    section move; all other pairs are bit-identical to the input."""
    q, k = _rand_qk(1, seed=32)
    bounds = [(0, 24), (24, 44), (44, 64)]
    for row, (lo, hi) in enumerate(bounds):
        pos = np.zeros((3, 1), dtype=np.int32)
        pos[row, 0] = 7
        qo, _ = orc.mrope_qk(q, k, pos, SECTIONS, THETA)
        for j in range(D // 2):
            same = qo[0, :, j] == q[0, :, j]
            same2 = qo[0, :, j + D // 2] == q[0, :, j + D // 2]
            if lo <= j < hi:
                assert not same.any() and not same2.any(), (row, j)
            else:
                assert same.all() and same2.all(), (row, j)


def _rope_1d_complex(x, p, theta):
    """Textbook 1-D RoPE as a complex multiplication: (a + ib) * e^(i p w_j),
    w_j = exp(-(2j/D) ln theta)."""
    d = x.shape[-1]
    j = np.arange(d // 2)
    w = np.exp(-(2.0 * j / d) * math.log(theta))
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    z = z * np.exp(1j * p[:, None, None] * w[None, None, :])
    return np.concatenate([z.real, z.imag], axis=-1)


def pin_mrope_equal_rows_is_rope_1d(orc):
    """When rows t, h and w hold the same position, M-RoPE is plain 1-D RoPE."""
    q, k = _rand_qk(6, seed=33)
    p = np.array([0, 1, 2, 31, 500, 1071], dtype=np.int32)
    pos = np.stack([p, p, p])
    qo, ko = orc.mrope_qk(q, k, pos, SECTIONS, THETA)
    np.testing.assert_allclose(qo, _rope_1d_complex(q, p.astype(np.float64), THETA), rtol=0, atol=1e-11)
    np.testing.assert_allclose(ko, _rope_1d_complex(k, p.astype(np.float64), THETA), rtol=0, atol=1e-11)


def pin_mrope_closed_form_angles(orc):
    """Pair j = 0 has frequency 1, so position p turns (1, 0) into (cos p, sin p);
    pair j = 32 has frequency 1e6^(-1/2) = 1e-3, so p = 1000 turns it by 1 rad."""
    x = np.zeros((1, 1, D))
    x[0, 0, 0] = 1.0
    x[0, 0, 32] = 1.0
    for p in (1, 2, 3, 1000):
        pos = np.full((3, 1), p, dtype=np.int32)
        qo, _ = orc.mrope_qk(x, np.zeros((1, 1, D)), pos, SECTIONS, THETA)
        assert abs(qo[0, 0, 0] - math.cos(p)) < 1e-14
        assert abs(qo[0, 0, 64] - math.sin(p)) < 1e-14
        if p == 1000:
            assert abs(qo[0, 0, 32] - math.cos(1.0)) < 1e-12
            assert abs(qo[0, 0, 96] - math.sin(1.0)) < 1e-12


def pin_mrope_relative_position(orc):
    """<R(m) q, R(n) k> depends only on m - n (all three rows shifted alike)."""
    rng = np.random.default_rng(34)
    qv = rng.standard_normal((1, 1, D))
    kv = rng.standard_normal((1, 1, D))

    def dot(m, n):
        pm = np.array([[m[0]], [m[1]], [m[2]]], dtype=np.int32)
        pn = np.array([[n[0]], [n[1]], [n[2]]], dtype=np.int32)
        qo, _ = orc.mrope_qk(qv, kv, pm, SECTIONS, THETA)
        ko, _ = orc.mrope_qk(kv, qv, pn, SECTIONS, THETA)
        return float(np.sum(qo * ko))

    base = dot((10, 3, 5), (4, 1, 2))
    for shift in ((1, 1, 1), (100, 0, 0), (0, 7, 0), (0, 0, 9), (500, 3, 2)):
        got = dot((10 + shift[0], 3 + shift[1], 5 + shift[2]), (4 + shift[0], 1 + shift[1], 2 + shift[2]))
        assert abs(got - base) < 1e-9 * max(1.0, abs(base))
    # and it does change when the offset changes
    assert abs(dot((11, 3, 5), (4, 1, 2)) - base) > 1e-6


def _kv_case(seed, tokens=4, hq=3, hk=2, rows=3, max_seq=8):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((tokens, hq, D))
    k = rng.standard_normal((tokens, hk, D))
    v = rng.standard_normal((tokens, hk, D))
    kc = rng.standard_normal((rows, hk, max_seq, D))
    vc = rng.standard_normal((rows, hk, max_seq, D))
    return q, k, v, kc, vc


def pin_kv_append_is_plain_append_at_position_zero(orc):
    """With every position 0 the rotation is the identity and the operation is
    the pages' KV-cache append: cache[row][head][slot][:] = new k / v, bit for
    bit; q passes through; every other slot keeps its contents."""
    q, k, v, kc, vc = _kv_case(80)
    pos = np.zeros((3, 4), np.int32)
    loc = np.array([[0, 2, 1, 2], [5, 0, 7, 3]], np.int32)
    qo, kc2, vc2 = orc.mrope_kv_append(q, k, v, pos, loc, kc, vc, SECTIONS, THETA)
    assert np.array_equal(qo, q)
    want_k, want_v = kc.copy(), vc.copy()
    for t in range(4):
        want_k[loc[0, t], :, loc[1, t], :] = k[t]
        want_v[loc[0, t], :, loc[1, t], :] = v[t]
    assert np.array_equal(kc2, want_k) and np.array_equal(vc2, want_v)


def pin_kv_append_rotates_k_like_q(orc):
    """The cached k is the rotation M-RoPE gives k at the token's positions (the
    same rotation q gets); v is copied unrotated; out-of-range slots are skipped."""
    q, k, v, kc, vc = _kv_case(81)
    pos = np.array([[3, 100, 7, 0], [1, 2, 3, 4], [9, 9, 9, 9]], np.int32)
    loc = np.array([[1, 0, 3, 2], [2, 6, 0, -1]], np.int32)  # tokens 2, 3 out of range
    qo, kc2, vc2 = orc.mrope_kv_append(q, k, v, pos, loc, kc, vc, SECTIONS, THETA)
    q_ref, k_ref = orc.mrope_qk(q, k, pos, SECTIONS, THETA)
    assert np.array_equal(qo, q_ref)
    assert np.array_equal(kc2[1, :, 2], k_ref[0]) and np.array_equal(kc2[0, :, 6], k_ref[1])
    assert np.array_equal(vc2[1, :, 2], v[0]) and np.array_equal(vc2[0, :, 6], v[1])
    kc2[1, :, 2] = kc[1, :, 2]
    kc2[0, :, 6] = kc[0, :, 6]
    vc2[1, :, 2] = vc[1, :, 2]
    vc2[0, :, 6] = vc[0, :, 6]
    assert np.array_equal(kc2, kc) and np.array_equal(vc2, vc)
    # the cached k of token 1 is k rotated: its pair norms are those of k
    half = D // 2
    n_in = k[1, :, :half] ** 2 + k[1, :, half:] ** 2
    n_out = kc[0, :, 6, :half] ** 2 + kc[0, :, 6, half:] ** 2
    assert not np.allclose(n_in, n_out)  # the old slot contents differ ...
    c = orc.mrope_kv_append(q, k, v, pos, loc, kc, vc, SECTIONS, THETA)[1]
    np.testing.assert_allclose(c[0, :, 6, :half] ** 2 + c[0, :, 6, half:] ** 2, n_in, rtol=1e-12)


# ---------------------------------------------------------------------------
# SwiGLU
# ---------------------------------------------------------------------------


def _silu_tanh(g):
    """silu through the logistic identity sigma(g) = (1 + tanh(g/2)) / 2."""
    return g * 0.5 * (1.0 + np.tanh(0.5 * g))


def pin_swiglu_known_values(orc):
    """silu(0) = 0, silu(1) = 0.7310585786300049, silu(-1) = -0.2689414213699951,
    silu(2) = 1.7615941559557646 (values of the logistic function)."""
    g = np.array([0.0, 1.0, -1.0, 2.0])
    out = orc.swiglu(g, np.ones(4))
    want = np.array([0.0, 0.7310585786300049, -0.2689414213699951, 1.7615941559557646])
    np.testing.assert_allclose(out, want, rtol=2e-16, atol=0)
    assert orc.swiglu(np.array([0.0]), np.array([-3.0]))[0] == 0.0


def pin_swiglu_odd_part_identity(orc):
    """silu(g) - silu(-g) = g for every g."""
    g = np.random.default_rng(40).standard_normal(1000) * 4
    u = np.ones_like(g)
    d = orc.swiglu(g, u) - orc.swiglu(-g, u)
    np.testing.assert_allclose(d, g, rtol=1e-14, atol=1e-15)


def pin_swiglu_tanh_form_and_limits(orc):
    """Matches the tanh form of the logistic function on random inputs; tends to
    g*u for large g and to 0 for very negative g; linear in up."""
    rng = np.random.default_rng(41)
    g = rng.standard_normal(5000) * 2
    u = rng.standard_normal(5000)
    out = orc.swiglu(g, u)
    np.testing.assert_allclose(out, _silu_tanh(g) * u, rtol=1e-13, atol=1e-300)
    assert np.array_equal(orc.swiglu(g, 2 * u), 2 * out)
    big = np.array([40.0, 60.0])
    np.testing.assert_allclose(orc.swiglu(big, np.array([1.5, -2.0])), big * [1.5, -2.0], rtol=1e-15)
    tiny = orc.swiglu(np.array([-40.0, -700.0, -1000.0]), np.array([1.0, 1.0, 1.0]))
    assert np.all(np.abs(tiny) < 1e-15) and np.all(tiny <= 0)


# ---------------------------------------------------------------------------
# decode-step chain
# ---------------------------------------------------------------------------


def _rmsnorm_torch_fp64(x, weight, eps):
    """RMSNorm as the module of "Optimising autoregressive speech models", §09
    ("How to swap") computes it, restated here and run by torch in fp64 on the
    CPU: the reciprocal square root (torch.rsqrt) of the row's mean square plus
    eps scales the row, then the weight multiplies each channel."""
    xt = torch.as_tensor(np.asarray(x, dtype=np.float64))
    w = torch.as_tensor(np.asarray(weight, dtype=np.float64))
    scale = torch.rsqrt(xt.square().mean(dim=-1, keepdim=True) + eps)
    return (xt * scale * w).numpy()


def pin_rmsnorm_matches_section09_module_in_torch(orc):
    """The oracle agrees with the §09 RMSNorm module run in torch fp64 (its
    rsqrt-then-multiply order against the oracle's divide by sqrt) to ~1e-15,
    and with torch's own fp64 rms_norm routine, on rows of mixed scale."""
    rng = np.random.default_rng(60)
    for rows, hidden, eps in ((7, 2048, 1e-6), (5, 1024, 1e-6), (3, 96, 0.25), (4, 33, 0.0)):
        x = rng.standard_normal((rows, hidden)) * rng.uniform(1e-3, 30, size=(rows, 1))
        w = 1.0 + 0.1 * rng.standard_normal(hidden)
        y = orc.rmsnorm(x, w, eps)
        np.testing.assert_allclose(y, _rmsnorm_torch_fp64(x, w, eps), rtol=4e-15, atol=1e-300)
        lib = torch.nn.functional.rms_norm(torch.from_numpy(x), (hidden,), torch.from_numpy(w),
                                           eps).numpy()
        np.testing.assert_allclose(y, lib, rtol=4e-15, atol=1e-300)


def pin_layernorm_matches_torch_layer_norm(orc):
    """The oracle's LayerNorm agrees with torch's fp64 layer_norm (population
    variance, eps inside the root, gamma and beta per channel)."""
    rng = np.random.default_rng(61)
    for rows, hidden, eps in ((6, 2048, 1e-6), (3, 40, 1e-2)):
        x = rng.standard_normal((rows, hidden)) * 3 + rng.uniform(-5, 5, size=(rows, 1))
        g = 1.0 + 0.1 * rng.standard_normal(hidden)
        b = 0.1 * rng.standard_normal(hidden)
        lib = torch.nn.functional.layer_norm(torch.from_numpy(x), (hidden,), torch.from_numpy(g),
                                             torch.from_numpy(b), eps).numpy()
        np.testing.assert_allclose(orc.layernorm(x, g, b, eps), lib, rtol=1e-13, atol=1e-14)


def _half_ulp_close(got, exact, what):
    """got is exact rounded to bf16: within half a bf16 ulp, i.e. 2^-8 |exact|
    (plus a floor far below any value used here)."""
    exact = np.asarray(exact, dtype=np.float64)
    assert got.shape == exact.shape, (what, got.shape, exact.shape)
    bad = np.abs(got - exact) > 2.0 ** -8 * np.abs(exact) + 1e-30
    assert not bad.any(), f"{what}: {np.count_nonzero(bad)} elements off"


def pin_decode_chain(orc):
    """Every output of the oracle's decode step against statements that do not
    use the oracle's operators, over several steps of a small chain:
      residual  the bf16 rounding, after every add, of the running sum (torch
                fp32 add + bf16 cast);
      y_attn    the §09 RMSNorm module in torch fp64 of the residual after the
                attention-side add, with that layer's attention weights;
      y_mlp     the same of the residual after the MLP-side add, with the MLP
                weights;
      q, k      1-D RoPE at position s written as a complex multiplication (all
                three position rows equal the step s);
      act       silu(gate) * up with the logistic written through tanh."""
    rng = np.random.default_rng(50)
    B, H, I, hq, hk, d, L = 2, 64, 96, 2, 1, 16, 3
    sections = (3, 3, 2)
    eps = 1e-6

    def bf(shape, std=1.0, mean=0.0):
        return torch.from_numpy(rng.standard_normal(shape) * std + mean).float().bfloat16()

    inp = {key: [] for key in ("x_attn", "gamma_attn", "q", "k", "x_mlp", "gamma_mlp", "gate", "up")}
    for _ in range(L):
        inp["x_attn"].append(bf((B, H)))
        inp["gamma_attn"].append(bf((H,), 0.1, 1.0))
        inp["q"].append(bf((B, hq, d)))
        inp["k"].append(bf((B, hk, d)))
        inp["x_mlp"].append(bf((B, H)))
        inp["gamma_mlp"].append(bf((H,), 0.1, 1.0))
        inp["gate"].append(bf((B, I), 2.0))
        inp["up"].append(bf((B, I)))
    res0 = bf((B, H), 2.0)
    res = res0.double().numpy()
    run = res0.clone()
    f64 = lambda t: t.double().numpy()  # noqa: E731
    for step in range(4):
        prev = res
        res, outs = orc.decode_step(res, inp, step, eps, 1e6, sections, "bf16")
        p = np.full(B, float(step))
        for layer in range(L):
            run_attn = (inp["x_attn"][layer].float() + run.float()).bfloat16()
            _half_ulp_close(outs["y_attn"][layer],
                            _rmsnorm_torch_fp64(f64(run_attn), f64(inp["gamma_attn"][layer]), eps),
                            f"y_attn step {step} layer {layer}")
            run = (inp["x_mlp"][layer].float() + run_attn.float()).bfloat16()
            _half_ulp_close(outs["y_mlp"][layer],
                            _rmsnorm_torch_fp64(f64(run), f64(inp["gamma_mlp"][layer]), eps),
                            f"y_mlp step {step} layer {layer}")
            _half_ulp_close(outs["q"][layer], _rope_1d_complex(f64(inp["q"][layer]), p, 1e6),
                            f"q step {step} layer {layer}")
            _half_ulp_close(outs["k"][layer], _rope_1d_complex(f64(inp["k"][layer]), p, 1e6),
                            f"k step {step} layer {layer}")
            _half_ulp_close(outs["act"][layer],
                            _silu_tanh(f64(inp["gate"][layer])) * f64(inp["up"][layer]),
                            f"act step {step} layer {layer}")
        assert np.array_equal(res, run.double().numpy())
        # the residual-only form of the step (outputs=False) carries the same residual
        res_only, none = orc.decode_step(prev, inp, step, eps, 1e6, sections, "bf16",
                                         outputs=False)
        assert none == {} and np.array_equal(res_only, res)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
