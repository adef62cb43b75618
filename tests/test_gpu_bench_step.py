"""The benchmark's own step, in the launch configuration bench.py times, against
the oracle: every configuration at full size, all 228 launches captured as one
CUDA graph with programmatic dependent launch, two replays (decode positions 0
and 1).  RMSNorm f32 64 x 1024, add+RMSNorm bf16 4096 x 2048, SwiGLU bf16
8192 x 6144 and M-RoPE bf16 4096 tokens are compared element by element; the
two 28-layer decode steps (batch 5 and 256) keep their residual bit-exact and
every output of every layer is compared at the second step."""
import numpy as np
import pytest
import torch

import oracle
from swiglu_ar_tts_b200.step import Step
from tolerance import check, to_f64

pytestmark = pytest.mark.gpu


def _pair_scale(x):
    half = x.shape[-1] // 2
    m = np.maximum(np.abs(x[..., :half]), np.abs(x[..., half:]))
    return np.concatenate([m, m], axis=-1)


def _chain_inputs(chain):
    return {k: [to_f64(t) for t in v] for k, v in chain.host_inputs.items() if k != "residual"}


def _check_chain_outputs(chain, outs, what):
    for l in range(chain.shape.layers):
        check(chain.y_attn[l], outs["y_attn"][l], "bf16", what=f"{what} y_attn[{l}]")
        check(chain.y_mlp[l], outs["y_mlp"][l], "bf16", what=f"{what} y_mlp[{l}]")
        check(chain.act[l], outs["act"][l], "bf16", what=f"{what} act[{l}]")
        check(chain.q_out[l], outs["q"][l], "bf16", _pair_scale(to_f64(chain.host_inputs["q"][l])),
              what=f"{what} q[{l}]")
        check(chain.k_out[l], outs["k"][l], "bf16", _pair_scale(to_f64(chain.host_inputs["k"][l])),
              what=f"{what} k[{l}]")


def test_bench_step_graph_against_oracle():
    step = Step(torch.device("cuda", torch.cuda.current_device()))
    step.capture()
    orc = oracle.get()
    chains = {"b5": step.chain5, "b256": step.chain256}
    res = {k: to_f64(c.residual0.cpu()) for k, c in chains.items()}
    assert all(np.array_equal(to_f64(c.residual), res[k]) for k, c in chains.items())
    inp = {k: _chain_inputs(c) for k, c in chains.items()}
    for s in range(2):
        step.run()  # positions = s, then one replay of the step graph
        torch.cuda.synchronize()
        for k, c in chains.items():
            res[k], outs = orc.decode_step(res[k], inp[k], s, c.eps, c.theta, c.sections, "bf16",
                                           outputs=s == 1)
            assert np.array_equal(to_f64(c.residual), res[k]), f"decode {k}: residual at step {s}"
            if s == 1:
                _check_chain_outputs(c, outs, f"decode {k}")

    h = step.host
    rn = h["rmsnorm"]
    check(step.rn["y"], orc.rmsnorm(rn["x"], rn["gamma"], 1e-6), "f32", what="rmsnorm 64x1024")
    an = h["add_rmsnorm"]
    y_e, r_e = orc.add_rmsnorm(an["x"], an["residual"], an["gamma"], 1e-6, "bf16")
    assert np.array_equal(to_f64(step.an["residual_out"]), r_e), "add_rmsnorm residual_out"
    check(step.an["y"], y_e, "bf16", what="add_rmsnorm 4096x2048")
    sw = h["swiglu"]
    check(step.sw["out"], orc.swiglu(sw["gate"], sw["up"]), "bf16", what="swiglu 8192x6144")
    mr = h["mrope_qk"]
    q_e, k_e = orc.mrope_qk(mr["q"], mr["k"], mr["pos"], (24, 20, 20), 1e6)
    check(step.mr["q_out"], q_e, "bf16", _pair_scale(to_f64(mr["q"])), what="mrope q")
    check(step.mr["k_out"], k_e, "bf16", _pair_scale(to_f64(mr["k"])), what="mrope k")
