"""One pass of the whole hot path on one GPU, as a CUDA graph.

The step runs every operator once at its workload size: RMSNorm fp32
[64 x 1024], residual add + RMSNorm bf16 [4096 x 2048], SwiGLU bf16
[8192 x 6144], M-RoPE bf16 on q [4096 x 16 x 128] and k [4096 x 8 x 128], and
one 28-layer decode step (add + RMSNorm, M-RoPE, add + RMSNorm, SwiGLU per
layer) at batch 5 and at batch 256.  ``Step`` owns the device buffers (seeded
synthetic inputs from ``inputs``) and captures the step's 228 launches as one
CUDA graph with programmatic dependent launch; it also carries the
end-to-end form of the step (host buffers in, results back to the host).
``bench.py`` times it.

    python -m swiglu_ar_tts_b200.step [--replays N]

replays the step graph N times inside an NVTX range named "step" (the driver
of the step's ncu launch list).
"""
from __future__ import annotations

import argparse

import torch

STEP_CONFIGS = ("rmsnorm", "add_rmsnorm", "swiglu", "mrope_qk", "decode_b5", "decode_b256")


def step_bytes() -> dict:
    """Algorithmic HBM bytes of each operator of the step (every operand read
    once, every output written once)."""
    per_row_layer = 2 * 4 * 2048 * 2 + 2 * (16 + 8) * 128 * 2 + 3 * 4 + 3 * 6144 * 2  # 81,932
    gammas = 2 * 2048 * 2  # two norm weights per layer
    return {
        "rmsnorm": (2 * 64 * 1024 + 1024) * 4,
        "add_rmsnorm": (4 * 4096 * 2048 + 2048) * 2,
        "swiglu": 3 * 8192 * 6144 * 2,
        "mrope_qk": 2 * 4096 * (16 + 8) * 128 * 2 + 3 * 4096 * 4,
        "decode_b5": 28 * (5 * per_row_layer + gammas),
        "decode_b256": 28 * (256 * per_row_layer + gammas),
    }


class Step:
    """Device buffers and launches of one hot-path step."""

    OPS = ("rmsnorm", "add_rmsnorm", "swiglu", "mrope_qk", "decode_b5", "decode_b256")

    def __init__(self, device: torch.device, pdl: bool = True, like: "Step | None" = None):
        """``like``: take the host inputs of that step instead of drawing them
        again (a second set of device buffers for the same workload)."""
        import swiglu_ar_tts_b200 as ops

        from . import inputs
        from .chain import DecodeChain

        self.ops = ops
        self.device = device
        self.host = like.host if like is not None else {
            "rmsnorm": inputs.rmsnorm_inputs(64, 1024, "f32", 0),
            "add_rmsnorm": inputs.add_rmsnorm_inputs(4096, 2048, "bf16", 0),
            "swiglu": inputs.swiglu_inputs(8192, 6144, "bf16", 0),
            "mrope_qk": inputs.mrope_inputs(4096),
        }
        d = device
        h = self.host
        self.rn = {k: v.to(d) for k, v in h["rmsnorm"].items()}
        self.rn["y"] = torch.empty_like(self.rn["x"])
        self.an = {k: v.to(d) for k, v in h["add_rmsnorm"].items()}
        self.an["y"] = torch.empty_like(self.an["x"])
        self.an["residual_out"] = torch.empty_like(self.an["residual"])
        self.sw = {k: v.to(d) for k, v in h["swiglu"].items()}
        self.sw["out"] = torch.empty_like(self.sw["gate"])
        self.mr = {k: v.to(d) for k, v in h["mrope_qk"].items()}
        self.mr["q_out"] = torch.empty_like(self.mr["q"])
        self.mr["k_out"] = torch.empty_like(self.mr["k"])
        self.chain5 = DecodeChain(inputs.ChainShape(batch=5), device=d, pdl=pdl,
                                  host_inputs=like.chain5.host_inputs if like else None)
        self.chain256 = DecodeChain(inputs.ChainShape(batch=256), device=d, seed=1000, pdl=pdl,
                                    host_inputs=like.chain256.host_inputs if like else None)
        self.chain5.capture()
        self.chain256.capture()
        self.pdl = pdl
        self.graph = None
        self.decode_step_index = 0
        self.bytes = step_bytes()
        assert self.bytes["decode_b5"] == self.chain5.bytes_per_step()
        assert self.bytes["decode_b256"] == self.chain256.bytes_per_step()
        # rows (tokens) one launch of each operator processes
        self.rows = {"rmsnorm": 64, "add_rmsnorm": 4096, "swiglu": 8192, "mrope_qk": 4096,
                     "decode_b5": 5, "decode_b256": 256}
        # kernels of this library launched per step (graph replays bypass the
        # launch counter, so their kernels are counted from the capture)
        self.kernels_per_step = 4 + self.chain5.launches_per_step + self.chain256.launches_per_step

    def prepare_op(self, name: str) -> None:
        """Host-side set-up that precedes an operator: the decode step's position
        ids (a 24-byte fill, outside the operator's timed window)."""
        if name == "decode_b5":
            self.chain5.set_position(self.decode_step_index % 300)
        elif name == "decode_b256":
            self.chain256.set_position(self.decode_step_index % 300)

    def run_op(self, name: str) -> None:
        ops = self.ops
        if name == "rmsnorm":
            ops.rmsnorm(self.rn["x"], self.rn["gamma"], 1e-6, out=self.rn["y"])
        elif name == "add_rmsnorm":
            ops.add_rmsnorm(self.an["x"], self.an["residual"], self.an["gamma"], 1e-6,
                            y=self.an["y"], residual_out=self.an["residual_out"])
        elif name == "swiglu":
            ops.swiglu(self.sw["gate"], self.sw["up"], out=self.sw["out"])
        elif name == "mrope_qk":
            ops.mrope_qk(self.mr["q"], self.mr["k"], self.mr["pos"], (24, 20, 20), 1e6,
                         q_out=self.mr["q_out"], k_out=self.mr["k_out"])
        elif name == "decode_b5":
            self.chain5._graph.replay()
        elif name == "decode_b256":
            self.chain256._graph.replay()

    def launch_op(self, name: str) -> None:
        """Enqueue operator ``name``'s kernels on the current stream (the decode
        steps' 112 launches each, through their pre-bound calls)."""
        if name == "decode_b5":
            self.chain5.launch_step()
        elif name == "decode_b256":
            self.chain256.launch_step()
        else:
            self.run_op(name)

    def capture(self, without: str | None = None) -> torch.cuda.CUDAGraph:
        """The whole step as one CUDA graph: the four prefill launches and both
        decode steps' 224 launches, every kernel launched with programmatic
        dependent launch (unless --no-pdl), so each one is scheduled while its
        predecessor drains, across operator boundaries too.  The decode
        residuals are put back after the warm-up and capture.  With
        ``without`` the graph leaves that operator out (for step_marginals)
        and is returned; otherwise it becomes the step's graph."""
        ops = self.ops
        names = [n for n in self.OPS if n != without]
        cur = torch.cuda.current_stream(self.device)
        saved = [self.chain5.residual.clone(), self.chain256.residual.clone()]
        old = ops.set_pdl(self.pdl)
        try:
            side = torch.cuda.Stream(self.device)
            side.wait_stream(cur)
            with torch.cuda.stream(side):  # warm-up outside the capture
                for name in names:
                    self.launch_op(name)
            cur.wait_stream(side)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for name in names:
                    self.launch_op(name)
        finally:
            ops.set_pdl(old)
        self.chain5.residual.copy_(saved[0])
        self.chain256.residual.copy_(saved[1])
        if without is None:
            self.graph = g
        return g

    def run(self, events=None) -> None:
        """One step: the step's set-up (the decode position ids), then one
        replay of the step graph between ``events[0]`` and ``events[1]``."""
        for name in self.OPS:
            self.prepare_op(name)
        if self.graph is None:
            self.capture()
        if events is not None:
            events[0].record()
        self.graph.replay()
        if events is not None:
            events[1].record()
        self.decode_step_index += 1

    # -- end to end: host buffers in, results back to the host ------------------
    def setup_e2e(self, share: "Step | None" = None) -> None:
        """Pinned host copies of every input and pinned host buffers for every
        output, and the two copy streams.  With ``share`` (a step of the same
        workload) this step becomes a second set of device buffers that uses
        ``share``'s host buffers and copy streams (run_e2e_pipelined)."""
        if share is not None:
            self.h_in, self.h_out = share.h_in, share.h_out
            self.h2d_bytes, self.d2h_bytes = share.h2d_bytes, share.d2h_bytes
            self.s_h2d, self.s_d2h = share.s_h2d, share.s_d2h
            return
        pin = lambda t: t.detach().cpu().pin_memory()  # noqa: E731
        self.h_in = {
            "rn": {k: pin(v) for k, v in self.host["rmsnorm"].items()},
            "an": {k: pin(v) for k, v in self.host["add_rmsnorm"].items()},
            "sw": {k: pin(v) for k, v in self.host["swiglu"].items()},
            "mr": {k: pin(v) for k, v in self.host["mrope_qk"].items()},
            "c5": [pin(t) for t in self._chain_inputs(self.chain5)],
            "c256": [pin(t) for t in self._chain_inputs(self.chain256)],
        }
        self.h_out = {
            "rn": [pin(torch.empty_like(self.rn["y"], device="cpu"))],
            "an": [pin(torch.empty_like(self.an["y"], device="cpu")),
                   pin(torch.empty_like(self.an["residual_out"], device="cpu"))],
            "sw": [pin(torch.empty_like(self.sw["out"], device="cpu"))],
            "mr": [pin(torch.empty_like(self.mr["q_out"], device="cpu")),
                   pin(torch.empty_like(self.mr["k_out"], device="cpu"))],
            "c5": [pin(torch.empty_like(t, device="cpu")) for t in self._chain_outputs(self.chain5)],
            "c256": [pin(torch.empty_like(t, device="cpu")) for t in self._chain_outputs(self.chain256)],
        }
        nbytes = lambda ts: sum(t.numel() * t.element_size() for t in ts)  # noqa: E731
        self.h2d_bytes = (sum(nbytes(v.values()) for k, v in self.h_in.items() if isinstance(v, dict))
                          + nbytes(self.h_in["c5"]) + nbytes(self.h_in["c256"]))
        self.d2h_bytes = sum(nbytes(v) for v in self.h_out.values())
        self.s_h2d = torch.cuda.Stream(self.device)
        self.s_d2h = torch.cuda.Stream(self.device)

    @staticmethod
    def _chain_inputs(c):
        """A decode step's inputs: the residual and the flat buffer holding
        every layer's inputs (one copy each)."""
        return [c.residual, c.flat_in]

    @staticmethod
    def _chain_outputs(c):
        """A decode step's outputs: the residual and the flat buffer holding
        every layer's outputs."""
        return [c.residual, c.flat_out]

    # operators with the most output first: their copies back overlap the
    # later operators' copies in, and the pipeline ends on small copies
    E2E_GROUPS = (("c256", "decode_b256"), ("sw", "swiglu"), ("an", "add_rmsnorm"),
                  ("mr", "mrope_qk"), ("c5", "decode_b5"), ("rn", "rmsnorm"))

    def _e2e_in(self, g: str) -> list:
        """(device input, pinned host source) pairs of operator group ``g``."""
        if g in ("c5", "c256"):
            c = self.chain5 if g == "c5" else self.chain256
            return list(zip(self._chain_inputs(c), self.h_in[g]))
        dev = {"rn": self.rn, "an": self.an, "sw": self.sw, "mr": self.mr}[g]
        return [(dev[k], v) for k, v in self.h_in[g].items()]

    def _e2e_out(self, g: str) -> list:
        """(pinned host destination, device output) pairs of operator group ``g``."""
        dev = {"rn": [self.rn["y"]], "an": [self.an["y"], self.an["residual_out"]],
               "sw": [self.sw["out"]], "mr": [self.mr["q_out"], self.mr["k_out"]]}
        if g in ("c5", "c256"):
            srcs = self._chain_outputs(self.chain5 if g == "c5" else self.chain256)
        else:
            srcs = dev[g]
        return list(zip(self.h_out[g], srcs))

    def run_e2e(self, after: dict | None = None, serial: bool = True) -> dict:
        """Host->device copies of every input, the step, device->host copies of
        every output.  Three streams form a pipeline over the operators: the
        inputs of operator i+1 cross PCIe while operator i computes and the
        results of operator i-1 cross back (the two copy directions run at the
        same time).  Events order each operator's copy-in, compute and
        copy-out.  ``serial`` (one step at a time): the copies in wait for
        everything enqueued before, and the compute stream ends waiting for
        the copies back.  Otherwise (run_e2e_pipelined) the copies in of an
        operator wait only for ``after[group]``, the end of the previous use
        of this set's buffers of that operator.  Returns, per group, the event
        that ends this step's use of them (its copy back, which followed its
        compute)."""
        nb = dict(non_blocking=True)
        cur = torch.cuda.current_stream()
        h2d, d2h = self.s_h2d, self.s_d2h
        if serial:
            h2d.wait_stream(cur)
        used = {}
        for g, name in self.E2E_GROUPS:
            if after is not None:
                h2d.wait_event(after[g])
            with torch.cuda.stream(h2d):
                for dst, src in self._e2e_in(g):
                    dst.copy_(src, **nb)
            arrived = torch.cuda.Event()
            arrived.record(h2d)
            cur.wait_event(arrived)
            self.prepare_op(name)
            self.run_op(name)
            done = torch.cuda.Event()
            done.record(cur)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                for dst, src in self._e2e_out(g):
                    dst.copy_(src, **nb)
            used[g] = torch.cuda.Event()
            used[g].record(d2h)
        if serial:
            cur.wait_stream(d2h)
        self.decode_step_index += 1
        return used


def run_e2e_pipelined(sets: list, steps: int) -> None:
    """``steps`` end-to-end steps on alternating sets of device buffers (Steps
    of one workload sharing host buffers and copy streams; step i runs on set
    i % len(sets)).  Each copy direction runs in order on its own stream, so
    step i+1's inputs cross PCIe while step i computes and its results drain;
    a set's buffers of an operator are refilled only after the previous step
    on that set has computed and copied back that operator.  The compute
    stream ends waiting for the last copy back."""
    cur = torch.cuda.current_stream()
    sets[0].s_h2d.wait_stream(cur)
    after = [None] * len(sets)
    for i in range(steps):
        j = i % len(sets)
        after[j] = sets[j].run_e2e(after[j], serial=False)
    cur.wait_stream(sets[0].s_d2h)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--replays", type=int, default=2)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args()
    device = torch.device("cuda", torch.cuda.current_device())
    step = Step(device)
    step.capture()
    for _ in range(a.warmup):
        step.graph.replay()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("step")
    for _ in range(a.replays):
        step.graph.replay()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    print(f"step: {a.replays} replays of {step.kernels_per_step} launches")


if __name__ == "__main__":
    main()
