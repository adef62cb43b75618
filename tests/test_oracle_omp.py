"""The row-parallel (OpenMP) build of the oracle, timed as the multi-core CPU
baseline, computes exactly what the plain build computes: each parallel loop
splits independent rows, tokens or elements, and every row's arithmetic runs in
the same order on one thread."""
import numpy as np

import oracle
from swiglu_ar_tts_b200 import inputs


def test_omp_build_equals_plain_build_bit_for_bit():
    plain = oracle.get()
    omp = oracle.get_omp()
    assert plain.threads() == 1 and omp.threads() >= 1
    f64 = lambda t: t.double().numpy()  # noqa: E731
    a = inputs.add_rmsnorm_inputs(300, 2048, "bf16", 3)
    y0, r0 = plain.add_rmsnorm(a["x"], a["residual"], a["gamma"], 1e-6, "bf16")
    y1, r1 = omp.add_rmsnorm(a["x"], a["residual"], a["gamma"], 1e-6, "bf16")
    assert np.array_equal(y0, y1) and np.array_equal(r0, r1)
    n = inputs.rmsnorm_inputs(64, 1024, "f32", 0)
    assert np.array_equal(plain.rmsnorm(n["x"], n["gamma"]), omp.rmsnorm(n["x"], n["gamma"]))
    beta = inputs.normal((2048,), 9, std=0.1)
    assert np.array_equal(plain.layernorm(a["x"], a["gamma"], beta),
                          omp.layernorm(a["x"], a["gamma"], beta))
    s = inputs.swiglu_inputs(64, 6144, "bf16", 0)
    assert np.array_equal(plain.swiglu(s["gate"], s["up"]), omp.swiglu(s["gate"], s["up"]))
    m = inputs.mrope_inputs(256)
    for x0, x1 in zip(plain.mrope_qk(m["q"], m["k"], m["pos"]), omp.mrope_qk(m["q"], m["k"], m["pos"])):
        assert np.array_equal(x0, x1)
    v = np.random.default_rng(4).standard_normal(100_000) * 10
    assert np.array_equal(plain.round_bf16(v), omp.round_bf16(v))
    shape = inputs.ChainShape(batch=3, layers=2)
    c = inputs.decode_chain_inputs(shape, seed=5)
    host = {k: [f64(t) for t in val] for k, val in c.items() if k != "residual"}
    r0, o0 = plain.decode_step(f64(c["residual"]), host, 7)
    r1, o1 = omp.decode_step(f64(c["residual"]), host, 7)
    assert np.array_equal(r0, r1)
    for key in o0:
        for u, w in zip(o0[key], o1[key]):
            assert np.array_equal(u, w)
