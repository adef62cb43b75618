"""Checks against values the source pages print (tests/golden/)."""
import json
import os

import numpy as np

import oracle
from swiglu_ar_tts_b200.inputs import ChainShape, decode_chain_inputs, normal

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# row reductions per norm, from the two formulas of the LayerNorm -> RMSNorm
# section: LayerNorm needs the mean and then the variance, RMSNorm only the
# mean of squares
REDUCTIONS = {"layer": 2, "rms": 1}


def test_reduction_count_of_the_norm_swap_matches_the_decode_step():
    """The pages count the reductions the swap saves over a 30-layer, 300-step
    decode; the decode step's norms per layer (counted by running the oracle's
    step) must reproduce that count."""
    fx = json.load(open(os.path.join(GOLDEN, "layernorm_to_rmsnorm_reductions.json")))
    shape = ChainShape(batch=1, layers=fx["layers"], hidden=8, inter=8, n_q_heads=1,
                       n_k_heads=1, head_dim=8)
    inp = decode_chain_inputs(shape, "f32", seed=0)
    inp["beta_attn"] = [normal((8,), 900 + l, std=0.1, dtype="f32") for l in range(shape.layers)]
    inp["beta_mlp"] = [normal((8,), 950 + l, std=0.1, dtype="f32") for l in range(shape.layers)]
    orc = oracle.Oracle(0)
    calls = {"rms": 0, "layer": 0}
    add_rms, add_ln = orc.add_rmsnorm, orc.add_layernorm

    def count_rms(*a, **kw):
        calls["rms"] += 1
        return add_rms(*a, **kw)

    def count_ln(*a, **kw):
        calls["layer"] += 1
        return add_ln(*a, **kw)

    orc.add_rmsnorm, orc.add_layernorm = count_rms, count_ln
    for norm in ("rms", "layer"):
        res, _ = orc.decode_step(inp["residual"], inp, step=3, sections=(2, 1, 1), dtype="f32",
                                 norm=norm)
        assert np.all(np.isfinite(res))
    per_step = {n: calls[n] * REDUCTIONS[n] for n in calls}
    assert calls["rms"] == calls["layer"] == 2 * fx["layers"]
    fewer = (per_step["layer"] - per_step["rms"]) * fx["decode_steps"]
    assert fewer == fx["fewer_reductions"]
