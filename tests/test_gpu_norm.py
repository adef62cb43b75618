"""RMSNorm and residual-add + RMSNorm on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_ar_tts_b200 as ops
from swiglu_ar_tts_b200 import inputs
from gpu_util import Guarded, dev, misaligned, resident_threads
from tolerance import LN_BAND, check, to_f64

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _run_rmsnorm(rows, hidden, dtype, seed=0, eps=EPS):
    inp = inputs.rmsnorm_inputs(rows, hidden, dtype, seed)
    x, g = dev(inp["x"]), dev(inp["gamma"])
    y = ops.rmsnorm(x, g, eps)
    torch.cuda.synchronize()
    exact = oracle.get().rmsnorm(inp["x"], inp["gamma"], eps)
    return y, exact


def test_rmsnorm_f32_64x1024(family):
    """The fp32 workload: 64 rows x 1024, gamma = 1 + 0.1 N(0,1), eps 1e-6."""
    y, exact = _run_rmsnorm(64, 1024, "f32")
    st = check(y, exact, "f32", what="rmsnorm f32 64x1024")
    assert st["max_rel"] <= 1e-5


# hidden sizes cover every kernel variant: 1/2/4/8 vectors per lane with one
# warp per row, 2/4/8/16 warps per row, the looped vector kernel (> 4096
# vectors) and the element-wise kernel (hidden not a multiple of the vector).
# With few rows (as here) rows of 33 to 512 vectors take one vector per lane
# over 2 to 16 warps, some lanes idle for 264, 1000 and 4000.
HIDDEN = [8, 16, 24, 40, 256, 264, 512, 1000, 1024, 2048, 4000, 4104, 8192, 16384, 32768, 40000,
          100, 2050, 40001]

# Row widths whose layout depends on the row count, run with just more rows
# than one wave of one vector per thread holds: 8 / 4 vectors per lane, one warp
# per row, or 2 warps per row for 512 vectors.
HIDDEN_WIDE = [264, 512, 1000, 1024, 2048, 4000]


def rows_past_one_wave(hidden: int, dtype: str) -> int:
    nvec = hidden // (8 if dtype == "bf16" else 4)
    return resident_threads() // nvec + 3


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hidden", HIDDEN)
def test_rmsnorm_shapes(dtype, hidden, family):
    rows = 37 if hidden <= 16384 else 5
    y, exact = _run_rmsnorm(rows, hidden, dtype, seed=hidden)
    check(y, exact, dtype, what=f"rmsnorm {dtype} {rows}x{hidden}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hidden", HIDDEN_WIDE)
def test_rmsnorm_shapes_past_one_wave(dtype, hidden):
    rows = rows_past_one_wave(hidden, dtype)
    y, exact = _run_rmsnorm(rows, hidden, dtype, seed=hidden + 2)
    check(y, exact, dtype, what=f"rmsnorm {dtype} {rows}x{hidden}")


def _sm_count() -> int:
    return torch.cuda.get_device_properties(0).multi_processor_count


# Decode-size problems with at least one row per SM (256 decode candidates)
# take two vectors per lane over hidden/512 warps (bf16); fewer rows take one
# vector per lane.  Widths on both sides of each warp count, rows at the SM
# count and above, all four norms.
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hidden", [264, 1000, 1024, 2048, 4000, 8192])
@pytest.mark.parametrize("extra_rows", [0, 57])
def test_norms_with_a_row_per_sm(dtype, hidden, extra_rows):
    nvec = hidden // (8 if dtype == "bf16" else 4)
    rows = _sm_count() + extra_rows
    if rows * nvec > _sm_count() * 2048:
        rows = _sm_count() * 2048 // nvec  # still within one vector per resident thread
    orc = oracle.get()
    inp = _ln_inputs(rows, hidden, dtype, hidden + extra_rows)
    x, r, g, b = dev(inp["x"]), dev(inp["residual"]), dev(inp["gamma"]), dev(inp["beta"])
    y = ops.rmsnorm(x, g, EPS)
    y2, r_out = ops.add_rmsnorm(x, r, g, EPS, residual_out=torch.empty_like(r))
    y3 = ops.layernorm(x, g, b, EPS)
    y4, r_out4 = ops.add_layernorm(x, r, g, b, EPS, residual_out=torch.empty_like(r))
    torch.cuda.synchronize()
    check(y, orc.rmsnorm(inp["x"], inp["gamma"], EPS), dtype, what=f"rmsnorm {rows}x{hidden}")
    y2_e, r_e = orc.add_rmsnorm(inp["x"], inp["residual"], inp["gamma"], EPS, dtype)
    assert np.array_equal(to_f64(r_out), r_e) and np.array_equal(to_f64(r_out4), r_e)
    check(y2, y2_e, dtype, what=f"add_rmsnorm {rows}x{hidden}")
    xr = to_f64(inp["x"])
    check(y3, orc.layernorm(inp["x"], inp["gamma"], inp["beta"], EPS), dtype,
          _ln_scale(xr, to_f64(inp["gamma"]), to_f64(inp["beta"]), EPS),
          what=f"layernorm {rows}x{hidden}", band=LN_BAND)
    y4_e, _ = orc.add_layernorm(inp["x"], inp["residual"], inp["gamma"], inp["beta"], EPS, dtype)
    check(y4, y4_e, dtype, _ln_scale(r_e, to_f64(inp["gamma"]), to_f64(inp["beta"]), EPS),
          what=f"add_layernorm {rows}x{hidden}", band=LN_BAND)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rmsnorm_large_bf16_prefill(dtype, family):
    y, exact = _run_rmsnorm(4096, 2048, dtype, seed=3)
    check(y, exact, dtype, what="rmsnorm 4096x2048")


def test_rmsnorm_single_row_and_empty():
    y, exact = _run_rmsnorm(1, 2048, "bf16")
    check(y, exact, "bf16")
    x = torch.empty(0, 2048, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(2048, dtype=torch.bfloat16, device="cuda")
    assert ops.rmsnorm(x, g).shape == (0, 2048)


def test_rmsnorm_zero_row_and_in_place():
    inp = inputs.rmsnorm_inputs(8, 2048, "bf16", 9)
    x = inp["x"].clone()
    x[3] = 0
    xd, g = dev(x), dev(inp["gamma"])
    ops.rmsnorm(xd, g, EPS, out=xd)  # in place
    torch.cuda.synchronize()
    assert bool((xd[3] == 0).all())
    check(xd, oracle.get().rmsnorm(x, inp["gamma"], EPS), "bf16", what="in-place")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rmsnorm_misaligned(dtype):
    inp = inputs.rmsnorm_inputs(9, 2048, dtype, 11)
    x = misaligned(dev(inp["x"]))
    g = misaligned(dev(inp["gamma"]))
    y = ops.rmsnorm(x, g, EPS)
    torch.cuda.synchronize()
    check(y, oracle.get().rmsnorm(inp["x"], inp["gamma"], EPS), dtype, what="misaligned")


@pytest.mark.parametrize("hidden", [2048, 100, 40000])
def test_rmsnorm_guard_bands(hidden, family):
    inp = inputs.rmsnorm_inputs(7, hidden, "bf16", 12)
    out = Guarded((7, hidden), torch.bfloat16)
    ops.rmsnorm(dev(inp["x"]), dev(inp["gamma"]), EPS, out=out.t)
    torch.cuda.synchronize()
    out.check()
    check(out.t, oracle.get().rmsnorm(inp["x"], inp["gamma"], EPS), "bf16")


def test_rmsnorm_eps_values():
    for eps in (0.0, 1e-6, 1e-2, 1.0):
        y, exact = _run_rmsnorm(16, 2048, "f32", seed=13, eps=eps)
        check(y, exact, "f32", what=f"eps={eps}")


# ---------------------------------------------------------------------------
# residual add + RMSNorm
# ---------------------------------------------------------------------------


def _run_add(rows, hidden, dtype, seed=0, in_place=False, eps=EPS):
    inp = inputs.add_rmsnorm_inputs(rows, hidden, dtype, seed)
    x, r, g = dev(inp["x"]), dev(inp["residual"]), dev(inp["gamma"])
    r_out = r if in_place else torch.empty_like(r)
    y, r_out = ops.add_rmsnorm(x, r, g, eps, residual_out=r_out)
    torch.cuda.synchronize()
    y_exact, r_exact = oracle.get().add_rmsnorm(inp["x"], inp["residual"], inp["gamma"], eps, dtype)
    return y, r_out, y_exact, r_exact


@pytest.mark.parametrize("in_place", [False, True])
def test_add_rmsnorm_bf16_4096x2048(in_place, family):
    """The fused add+norm workload: x ~ N(0,1), residual ~ N(0,2^2), [4096 x 2048]."""
    y, r_out, y_exact, r_exact = _run_add(4096, 2048, "bf16", in_place=in_place)
    assert np.array_equal(to_f64(r_out), r_exact), "residual_out must be bit-exact"
    check(y, y_exact, "bf16", what="add_rmsnorm 4096x2048")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hidden", HIDDEN)
def test_add_rmsnorm_shapes(dtype, hidden, family):
    rows = 21 if hidden <= 16384 else 3
    y, r_out, y_exact, r_exact = _run_add(rows, hidden, dtype, seed=hidden + 1)
    assert np.array_equal(to_f64(r_out), r_exact)
    check(y, y_exact, dtype, what=f"add_rmsnorm {dtype} {rows}x{hidden}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hidden", HIDDEN_WIDE)
def test_add_rmsnorm_shapes_past_one_wave(dtype, hidden):
    rows = rows_past_one_wave(hidden, dtype)
    y, r_out, y_exact, r_exact = _run_add(rows, hidden, dtype, seed=hidden + 4)
    assert np.array_equal(to_f64(r_out), r_exact)
    check(y, y_exact, dtype, what=f"add_rmsnorm {dtype} {rows}x{hidden}")


def test_add_rmsnorm_is_add_then_norm_on_gpu(family):
    """The fused kernel equals the add written back, then RMSNorm of it, both on
    the GPU (bit for bit: the norm sees exactly the written residual)."""
    inp = inputs.add_rmsnorm_inputs(64, 2048, "bf16", 21)
    x, r, g = dev(inp["x"]), dev(inp["residual"]), dev(inp["gamma"])
    y, r_out = ops.add_rmsnorm(x, r.clone(), g, EPS)
    y2 = ops.rmsnorm(r_out, g, EPS)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


def test_add_rmsnorm_misaligned_and_guarded(family):
    inp = inputs.add_rmsnorm_inputs(5, 2048, "bf16", 22)
    x = misaligned(dev(inp["x"]))
    r = misaligned(dev(inp["residual"]))
    y = Guarded((5, 2048), torch.bfloat16, offset=1)
    r_out = Guarded((5, 2048), torch.bfloat16)
    ops.add_rmsnorm(x, r, dev(inp["gamma"]), EPS, y=y.t, residual_out=r_out.t)
    torch.cuda.synchronize()
    y.check()
    r_out.check()
    y_exact, r_exact = oracle.get().add_rmsnorm(inp["x"], inp["residual"], inp["gamma"], EPS, "bf16")
    assert np.array_equal(to_f64(r_out.t), r_exact)
    check(y.t, y_exact, "bf16")


def test_add_rmsnorm_x_zero_reduces_to_rmsnorm():
    inp = inputs.add_rmsnorm_inputs(16, 2048, "bf16", 23)
    r, g = dev(inp["residual"]), dev(inp["gamma"])
    y, r_out = ops.add_rmsnorm(torch.zeros_like(r), r.clone(), g, EPS)
    y2 = ops.rmsnorm(r, g, EPS)
    torch.cuda.synchronize()
    assert torch.equal(r_out, r) and torch.equal(y, y2)


# ---------------------------------------------------------------------------
# LayerNorm and residual add + LayerNorm
# ---------------------------------------------------------------------------


def _ln_scale(xr: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float) -> np.ndarray:
    """(|x - mean| r + 1) |gamma| + |beta|, r = 1/sqrt(var + eps): the size of the
    operands of each output, used as its cancellation scale (tolerance.check).
    The kernel sums the row shifted by its first element, so the fp32 error of
    x - mean is of the order of the row's spread (the "+ 1", one standard
    deviation times r), whatever the row's offset."""
    mean = xr.mean(axis=-1, keepdims=True)
    r = 1.0 / np.sqrt(((xr - mean) ** 2).mean(axis=-1, keepdims=True) + eps)
    return (np.abs(xr - mean) * r + 1.0) * np.abs(gamma) + np.abs(beta)


def _ln_inputs(rows, hidden, dtype, seed):
    inp = inputs.add_rmsnorm_inputs(rows, hidden, dtype, seed)
    inp["beta"] = inputs.normal((hidden,), seed + 3, std=0.1, dtype=dtype)
    return inp


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hidden", HIDDEN)
def test_layernorm_shapes(dtype, hidden):
    rows = 21 if hidden <= 16384 else 3
    inp = _ln_inputs(rows, hidden, dtype, hidden + 7)
    # a shifted input (mean far from 0) exercises the two-pass variance
    x = (inp["x"].float() + 3.0).to(inp["x"].dtype)
    y = ops.layernorm(dev(x), dev(inp["gamma"]), dev(inp["beta"]), EPS)
    torch.cuda.synchronize()
    exact = oracle.get().layernorm(x, inp["gamma"], inp["beta"], EPS)
    scale = _ln_scale(to_f64(x), to_f64(inp["gamma"]), to_f64(inp["beta"]), EPS)
    check(y, exact, dtype, scale, what=f"layernorm {dtype} {rows}x{hidden}", band=LN_BAND)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hidden", HIDDEN_WIDE)
def test_add_layernorm_shapes_past_one_wave(dtype, hidden):
    rows = rows_past_one_wave(hidden, dtype)
    inp = _ln_inputs(rows, hidden, dtype, hidden + 13)
    x = (inp["x"].float() + 3.0).to(inp["x"].dtype)
    y, r_out = ops.add_layernorm(dev(x), dev(inp["residual"]), dev(inp["gamma"]),
                                 dev(inp["beta"]), EPS, residual_out=torch.empty_like(dev(x)))
    torch.cuda.synchronize()
    y_exact, r_exact = oracle.get().add_layernorm(x, inp["residual"], inp["gamma"],
                                                  inp["beta"], EPS, dtype)
    assert np.array_equal(to_f64(r_out), r_exact)
    scale = _ln_scale(r_exact, to_f64(inp["gamma"]), to_f64(inp["beta"]), EPS)
    check(y, y_exact, dtype, scale, what=f"add_layernorm {dtype} {rows}x{hidden}", band=LN_BAND)


@pytest.mark.parametrize("in_place", [False, True])
def test_add_layernorm_bf16_4096x2048(in_place):
    inp = _ln_inputs(4096, 2048, "bf16", 0)
    x, r = dev(inp["x"]), dev(inp["residual"])
    r_out = r if in_place else torch.empty_like(r)
    y, r_out = ops.add_layernorm(x, r, dev(inp["gamma"]), dev(inp["beta"]), EPS, residual_out=r_out)
    torch.cuda.synchronize()
    y_exact, r_exact = oracle.get().add_layernorm(inp["x"], inp["residual"], inp["gamma"],
                                                  inp["beta"], EPS, "bf16")
    assert np.array_equal(to_f64(r_out), r_exact), "residual_out must be bit-exact"
    scale = _ln_scale(r_exact, to_f64(inp["gamma"]), to_f64(inp["beta"]), EPS)
    check(y, y_exact, "bf16", scale, what="add_layernorm 4096x2048", band=LN_BAND)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hidden", [8, 264, 1000, 2048, 4000, 100, 40000, 16384])
def test_add_layernorm_shapes(dtype, hidden):
    rows = 9
    inp = _ln_inputs(rows, hidden, dtype, hidden + 11)
    y, r_out = ops.add_layernorm(dev(inp["x"]), dev(inp["residual"]), dev(inp["gamma"]),
                                 dev(inp["beta"]), EPS, residual_out=torch.empty_like(dev(inp["x"])))
    torch.cuda.synchronize()
    y_exact, r_exact = oracle.get().add_layernorm(inp["x"], inp["residual"], inp["gamma"],
                                                  inp["beta"], EPS, dtype)
    assert np.array_equal(to_f64(r_out), r_exact)
    scale = _ln_scale(r_exact, to_f64(inp["gamma"]), to_f64(inp["beta"]), EPS)
    check(y, y_exact, dtype, scale, what=f"add_layernorm {dtype} {rows}x{hidden}", band=LN_BAND)


def test_layernorm_constant_rows_give_beta_and_guarded():
    """A constant row normalises to exactly beta (zero deviation)."""
    hidden = 2048
    beta = inputs.normal((hidden,), 5, std=0.1, dtype="bf16")
    x = torch.full((6, hidden), 1.75, dtype=torch.bfloat16)
    out = Guarded((6, hidden), torch.bfloat16, offset=1)
    ops.layernorm(dev(x), dev(torch.ones(hidden, dtype=torch.bfloat16)), dev(beta), EPS, out=out.t)
    torch.cuda.synchronize()
    out.check()
    assert torch.equal(out.t.cpu(), beta.expand(6, hidden))


def test_layernorm_misaligned():
    inp = _ln_inputs(5, 2048, "bf16", 31)
    y = ops.layernorm(misaligned(dev(inp["x"])), dev(inp["gamma"]), misaligned(dev(inp["beta"])), EPS)
    torch.cuda.synchronize()
    exact = oracle.get().layernorm(inp["x"], inp["gamma"], inp["beta"], EPS)
    check(y, exact, "bf16", _ln_scale(to_f64(inp["x"]), to_f64(inp["gamma"]), to_f64(inp["beta"]), EPS),
          band=LN_BAND)
