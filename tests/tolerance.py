"""Comparison of GPU outputs with the fp64 oracle.

Floating-point bar (the workload definition: max relative error <= 1e-5 for fp32
outputs; <= 8e-3 with cosine >= 0.99999 for bf16 outputs, both against the fp64
oracle rounded to the output dtype).  Relative error has no meaning where the
exact result is ~0, so the bf16 check is applied element by element as:

  |gpu - round_bf16(exact)| <= 1 bf16 ulp of round_bf16(exact)

Adjacent bf16 numbers differ by at most 2^-7 of their magnitude (< 8e-3), so
this is at least as strict as the relative bound wherever that bound means
anything.  The one exception is cancellation in M-RoPE (a cos - b sin ~ 0):
there the fp32 kernel's absolute error is set by the size of the operands, not
of the result.  Its bound, from the arithmetic: cos/sin of the fp64-reduced
angle carry <= ~1.2e-7 (fp32 rounding of the reduced angle) + 1 ulp of sincosf;
two products and a sum in fp32 add <= 3 * 2^-24 relative; in total less than
2^-20 * max(|a|, |b|).  Those elements therefore pass when
|gpu - exact| <= 2^-19 * max(|a|, |b|) (twice the derived bound).

The same cancellation allowance applies to fp32 M-RoPE outputs, whose other
elements must meet the 1e-5 relative bound.  fp32 relative errors are taken
against max(|exact|, 2^-126): subnormal fp32 numbers are spaced more coarsely
than 1e-5 of their size.

On top of the element-wise check, every comparison also requires
cosine(gpu, exact) >= 0.99999 in fp64 and max relative error <= 8e-3 (bf16) or
1e-5 (fp32) over the elements with |exact| >= 1e-3 * rms(exact) and, where a
cancellation scale is given, |exact| >= band * scale, i.e. away from
cancellation.  For M-RoPE band = 0.05 (an output that keeps a twentieth of its
operands' size).  LayerNorm passes band = LN_BAND = 0.5: its fp32 outputs are
held to 1e-5 relative, and at |exact| = 0.05 * scale its cancellation
allowance 2^-19 * scale alone is 3.8e-5 of the output, so the relative bar
there would contradict the allowance derived from the arithmetic; at 0.5 *
scale the allowance is 3.8e-6 of the output, inside the 1e-5 bar.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (v a bf16 value, as fp64)."""
    a = np.abs(v)
    _, e = np.frexp(a)
    ulp = np.ldexp(1.0, e - 8)
    return np.maximum(ulp, 2.0 ** -133)


def cosine(a: np.ndarray, b: np.ndarray) -> float:
    a = a.ravel()
    b = b.ravel()
    na = np.linalg.norm(a)
    nb = np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(np.dot(a, b) / (na * nb))


# relative-error band of the LayerNorm comparisons (see the module docstring)
LN_BAND = 0.5


def check(gpu: torch.Tensor, exact: np.ndarray, dtype: str, cancel_scale: np.ndarray | None = None,
          what: str = "", band: float = 0.05) -> dict:
    """Assert that ``gpu`` matches the unrounded fp64 oracle result ``exact``."""
    g = to_f64(gpu)
    exact = np.asarray(exact, dtype=np.float64)
    assert g.shape == exact.shape, (what, g.shape, exact.shape)
    orc = oracle.get()
    stats = {"n": int(g.size)}
    if g.size == 0:
        return stats
    assert np.array_equal(np.isnan(g), np.isnan(exact)), f"{what}: NaN pattern differs"
    fin = np.isfinite(exact)
    g, exact_f = g[fin], exact[fin]
    if dtype == "bf16":
        o_hat = orc.round_to(exact_f, "bf16")
        err = np.abs(g - o_hat)
        ok = err <= bf16_ulp(o_hat)
        if cancel_scale is not None:
            cs = np.asarray(cancel_scale, dtype=np.float64)[fin]
            ok |= np.abs(g - exact_f) <= 2.0 ** -19 * cs
        bad = np.flatnonzero(~ok)
        assert bad.size == 0, (
            f"{what}: {bad.size} of {g.size} elements beyond 1 bf16 ulp; first: "
            f"gpu={g[bad[:5]]} oracle={exact_f[bad[:5]]}")
        stats["ulp_mismatch"] = int(np.count_nonzero(g != o_hat))
        stats["max_ulp"] = float(np.max(err / bf16_ulp(o_hat)))
    elif dtype == "f32":
        err = np.abs(g - exact_f)
        # relative to max(|exact|, smallest normal fp32): below 2^-126 the fp32
        # grid itself is coarser than 1e-5 relative
        ok = err <= 1e-5 * np.maximum(np.abs(exact_f), 2.0 ** -126)
        if cancel_scale is not None:
            cs = np.asarray(cancel_scale, dtype=np.float64)[fin]
            ok |= err <= 2.0 ** -19 * cs
        bad = np.flatnonzero(~ok)
        assert bad.size == 0, (
            f"{what}: {bad.size} elements beyond rel 1e-5; first gpu={g[bad[:5]]} "
            f"oracle={exact_f[bad[:5]]}")
        stats["max_rel"] = float(np.max(err / (np.abs(exact_f) + 1e-300)))
    else:
        raise ValueError(dtype)
    cos = cosine(g, exact_f)
    assert cos >= 0.99999, f"{what}: cosine {cos}"
    rms = np.sqrt(np.mean(exact_f ** 2))
    big = np.abs(exact_f) >= 1e-3 * rms
    if cancel_scale is not None:
        # away from cancellation: the result keeps `band` of its operands' size
        big &= np.abs(exact_f) >= band * np.asarray(cancel_scale, dtype=np.float64)[fin]
    if big.any():
        rel = np.max(np.abs(g[big] - exact_f[big]) / np.abs(exact_f[big]))
        assert rel <= (8e-3 if dtype == "bf16" else 1e-5), f"{what}: max rel err {rel}"
        stats["max_rel_big"] = float(rel)
    stats["cosine"] = cos
    return stats
