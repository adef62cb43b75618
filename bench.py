"""Benchmark of the decode-operator hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of every operator of the hot path over one batch of
synthetic input:
  * RMSNorm fp32 [64 x 1024]
  * residual add + RMSNorm bf16 [4096 x 2048]
  * SwiGLU bf16, gate and up [8192 x 6144]
  * M-RoPE bf16, q [4096 x 16 x 128], k [4096 x 8 x 128], sections [24, 20, 20]
  * one 28-layer decode step (add+norm, M-RoPE, add+norm, SwiGLU per layer) at
    batch 5 and at batch 256, each replayed from a CUDA graph.
The step is captured once as a CUDA graph of its 228 launches, each launched
with programmatic dependent launch, and every timed step is one replay of it
between two CUDA events.  ``value`` is the step's algorithmic HBM bytes (every
operand read once, every output written once) divided by its device time, in
GB/s, summed over ranks.  The JSON line also gives each operator alone
(``ops_isolated``: median of 100 event-bracketed launches over inputs rotated
through >= 512 MB, and the per-launch time back to back), the step time split
among the operators in proportion to what each adds to the step graph's time
(``ops``),
microseconds per decode step, the time, share and GB/s of each kernel type
(each decode step split across its kernels by timing each operator's launches
as a graph of its own), the roofline of the dominant kernel and of the largest
single launch (SwiGLU), an end-to-end figure with host buffers, and the oracle
timed on the host cores.

L2: the step touches ~1 GB of distinct data, 8x the 126 MB L2, and no operator
reuses data of another, so every operator's inputs were last touched hundreds
of MB of traffic earlier and come from DRAM ("inputs larger than L2").  No
flush buffer is written between steps: its dirty lines would be written back
during, and charged to, the next step's first kernels.

Multi-GPU (torchrun, one process per GPU): every rank runs the same step on its
own GPU (replicas; the operators have no exchange step).  Times are the max
over ranks; value is the total bytes of all ranks over that time.

``--impl reference`` times the plain single-threaded fp64 CPU oracle instead, on
the same whole step (rank 0 only; other ranks exit at once).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from swiglu_ar_tts_b200.step import (STEP_CONFIGS, Step, run_e2e_pipelined,  # noqa: E402
                                     step_bytes)

METRIC = "fused-op HBM GB/s & % of B200 peak; µs per decode step (5 candidates)"
UNIT = "GB/s"
WORKLOAD = ("hot-path pass: RMSNorm f32 64x1024; add+RMSNorm bf16 4096x2048; SwiGLU bf16 "
            "8192x6144; M-RoPE bf16 4096 tok x (16q+8k) heads x 128, sections [24,20,20]; "
            "28-layer decode step at batch 5 and at batch 256")
FALLBACK_HBM_GBS = 6650.0
L2_NOTE = ("inputs larger than L2: the step streams ~1 GB of distinct data (8x L2) and no "
           "operator reuses another's data; no flush buffer")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
# B200 HBM3e specification (DGX figure); fractions of it are reported beside
# the fractions of the measured copy peak
SPEC_HBM_GBS = 8000.0


def measured_hbm_peak() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest(*rel: str) -> str:
    """Digest of the code of the given sources: `//` comments, trailing blanks
    and blank lines are left out (the sources keep no `//` inside string
    literals), so an edit to comments alone keeps the digest and any change to
    the code itself changes it."""
    h = hashlib.sha256()
    for r in rel:
        with open(os.path.join(ROOT, r), encoding="utf-8") as f:
            for line in f.read().splitlines():
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, sources: tuple[str, ...]) -> float | None:
    """Memory traffic per launch recorded from an ncu capture
    (profiles/traffic.json): DRAM reads plus the bytes the kernel wrote into L2
    (all of which reach DRAM once; most are still in L2 when the kernel ends),
    or None when absent or when the kernel's sources changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    if rec.get("source_digest") != source_digest(*sources):
        return None
    return float(rec.get("traffic_bytes_per_launch", rec["dram_bytes_per_launch"]))


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this process's GPU, sampled
    every 5 ms through NVML on a background thread while the timed steps run."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device: torch.device):
        self.device = device
        self.samples: list[tuple[float, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._err = None

    def _handle(self):
        import pynvml

        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
            except Exception:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def start(self):
        try:
            import pynvml

            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons",
                                  None) or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # no NVML: report that, do not guess
            self._err = f"nvml unavailable: {e}"
            return

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                         int(get_reasons(h))))
                except Exception as e:
                    self._err = str(e)
                    return
                time.sleep(0.005)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self) -> dict:
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=2)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": [self._err or "no samples"], "samples": 0}
        reasons = set()
        for _, bits in self.samples:
            for bit, name in self.REASONS.items():
                if bits & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml, 5 ms"}


def step_marginals(step, reps: int = 20, rounds: int = 5) -> tuple[dict, float]:
    """What each operator adds to the step, in µs: the step graph's time minus
    the time of the same graph with that operator left out (each graph
    replayed ``reps`` times back to back between two events, the median of
    ``rounds`` interleaved rounds).  Returns ({op: µs}, µs of the whole step
    measured the same way)."""
    graphs = {None: step.graph}
    for name in step.OPS:
        graphs[name] = step.capture(without=name)
    times = {k: [] for k in graphs}
    for _ in range(rounds):
        for k, g in graphs.items():
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            times[k].append(1e3 * e0.elapsed_time(e1) / reps)
    full = statistics.median(times[None])
    marg = {name: full - statistics.median(times[name]) for name in step.OPS}
    del graphs
    return marg, full


def reduce_max(x: float, pg=None, device=None) -> float:
    """Max of ``x`` over the ranks of process group ``pg`` (identity without one).
    Used for every time in a multi-GPU run, so ranks agree on the slowest."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world: int, step_bytes: int, steps: int, total_ms_max: float) -> float:
    """Whole-job GB/s: every rank processed ``step_bytes`` per step (replicas),
    over the slowest rank's device time."""
    return world * step_bytes * steps / (total_ms_max * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# attribution of the decode graphs to kernel types
# ---------------------------------------------------------------------------
KERNEL_OF = {"add_rmsnorm": "norm_rows_kernel", "rmsnorm": "norm_rows_kernel",
             "mrope_qk": "mrope_vec_kernel", "swiglu": "swiglu_vec_kernel"}


OP_OF_SYMBOL = {"arops_add_rmsnorm": "add_rmsnorm", "arops_add_layernorm": "add_layernorm",
                "arops_mrope_qk": "mrope_qk", "arops_swiglu": "swiglu"}
KERNEL_OF["add_layernorm"] = "norm_rows_kernel"


def group_decode_calls(chain) -> dict:
    """The decode step's pre-bound calls grouped by operator (symbol name)."""
    groups: dict[str, list] = {}
    for fn, a in chain._calls:
        groups.setdefault(OP_OF_SYMBOL[fn.__name__], []).append((fn, a))
    return groups


def decode_split(chain, reps: int = 10) -> dict:
    """Fraction of a decode step spent in each operator's kernels.

    The step's launches are grouped by operator (56 add+RMSNorm, 28 M-RoPE, 28
    SwiGLU for 28 layers); each group is captured as a graph of its own and
    timed, and the step's measured time is split in proportion.  Returns
    {op: (fraction, launches, algorithmic bytes)}."""
    from swiglu_ar_tts_b200 import lib

    L = lib()
    groups = group_decode_calls(chain)
    sh = chain.shape
    e = chain.residual.element_size()
    per_launch_bytes = {
        "add_rmsnorm": (4 * sh.batch * sh.hidden + sh.hidden) * e,
        "add_layernorm": (4 * sh.batch * sh.hidden + 2 * sh.hidden) * e,
        "mrope_qk": 2 * sh.batch * (sh.n_q_heads + sh.n_k_heads) * sh.head_dim * e + 3 * sh.batch * 4,
        "swiglu": 3 * sh.batch * sh.inter * e,
    }
    saved = chain.residual.clone()
    times = {}
    old = L.arops_set_pdl(1 if chain.pdl else 0)
    try:
        for key, calls in groups.items():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                st = torch.cuda.current_stream().cuda_stream
                for fn, a in calls:
                    fn(*a, st)
            for _ in range(2):
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            times[key] = e0.elapsed_time(e1) / reps
            del g
    finally:
        L.arops_set_pdl(old)
    chain.residual.copy_(saved)
    total = sum(times.values())
    return {k: (times[k] / total, len(groups[k]), len(groups[k]) * per_launch_bytes[k]) for k in times}


# ---------------------------------------------------------------------------
# each operator alone, inputs rotated through >= 4x L2
# ---------------------------------------------------------------------------
ISOLATED = (("rmsnorm", "rmsnorm"), ("add_rmsnorm", "add_rmsnorm"), ("swiglu", "swiglu"),
            ("mrope_qk", "mrope_qk"), ("decode5", "decode_b5"), ("decode256", "decode_b256"))


def _time_alone(op: str, rows, device, peak: float, peak_kind: str, launches: int) -> dict:
    """One operator on its own (see isolated_ops)."""
    import swiglu_ar_tts_b200 as ops
    from swiglu_ar_tts_b200 import opbench

    fns, nbytes, desc = opbench.make_rotation(op, rows, device, None)
    ops.set_pdl(False)
    us = opbench.time_op(fns, launches)
    ops.set_pdl(True)
    for f in fns:
        f()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    # a head start long enough for the host to queue every launch before the
    # first one runs (~50 ms), so that the figure is the device's alone
    torch.cuda._sleep(int(1e8))
    e0.record()
    for i in range(launches):
        fns[i % len(fns)]()
    e1.record()
    torch.cuda.synchronize()
    b2b = 1e3 * e0.elapsed_time(e1) / launches
    med = statistics.median(us)
    gbs = nbytes / (med * 1e-6) / 1e9
    gbs_b2b = nbytes / (b2b * 1e-6) / 1e9
    del fns
    torch.cuda.empty_cache()
    return {"shape": desc, "bytes": nbytes, "launches": launches,
            "us_median": round(med, 3), "us_min": round(min(us), 3),
            "gbs_median": round(gbs, 1),
            "frac_of_" + peak_kind + "_hbm": round(gbs / peak, 4),
            "us_back_to_back": round(b2b, 3), "gbs_back_to_back": round(gbs_b2b, 1),
            "frac_back_to_back": round(gbs_b2b / peak, 4)}


def isolated_ops(device, peak: float, peak_kind: str, launches: int = 100) -> dict:
    """Each operator on its own, outside the timed steps: enough copies of its
    buffers to cover 512 MB (4x L2; a decode step at batch 256 is 588 MB in one
    copy), launches cycling through them so every launch reads from DRAM and
    pays for earlier launches' write-backs.  ``us_median``: the median over
    ``launches`` launches, each bracketed by its own CUDA events (launched
    without programmatic dependent launch, so each starts on an idle GPU).
    ``us_back_to_back``: the same launches enqueued back to back with
    programmatic dependent launch between one pair of events, per launch (each
    launch overlaps its predecessor's drain, as inside a step)."""
    import swiglu_ar_tts_b200 as ops

    out = {}
    old = ops.set_pdl(False)
    try:
        for op, key in ISOLATED:
            out[key] = _time_alone(op, None, device, peak, peak_kind, launches)
    finally:
        ops.set_pdl(old)
    return out


def sampling_ops(device, peak: float, peak_kind: str, launches: int = 100) -> dict:
    """The fused softmax + top-k sampler (top 50 of 151,936 bf16 logits a row)
    timed the same way, at the decode step's two batch sizes: 5 candidates
    (the register cluster kernel) and 256 rows (the shared-memory one)."""
    import swiglu_ar_tts_b200 as ops

    out = {}
    old = ops.set_pdl(False)
    try:
        for rows in (5, 256):
            out[f"rows{rows}"] = _time_alone("topk_sample", rows, device, peak, peak_kind, launches)
    finally:
        ops.set_pdl(old)
    return out


# ---------------------------------------------------------------------------
# CPU oracle timings
# ---------------------------------------------------------------------------
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


class OracleStep:
    """The whole step (every configuration at full size) on the fp64 CPU
    oracle, from the same seeded inputs as the GPU step, widened to fp64 once
    up front (the oracle's input format).  ``run`` returns seconds per
    configuration; each output is rounded to its dtype as the GPU writes it."""

    def __init__(self):
        from swiglu_ar_tts_b200 import inputs

        f64 = lambda t: t.detach().to(torch.float64).numpy()  # noqa: E731
        self.rn = {k: f64(v) for k, v in inputs.rmsnorm_inputs(64, 1024, "f32", 0).items()}
        self.an = {k: f64(v) for k, v in inputs.add_rmsnorm_inputs(4096, 2048, "bf16", 0).items()}
        self.sw = {k: f64(v) for k, v in inputs.swiglu_inputs(8192, 6144, "bf16", 0).items()}
        mr = inputs.mrope_inputs(4096)
        self.pos = mr["pos"].numpy()
        self.mr = {k: f64(v) for k, v in mr.items() if k != "pos"}
        self.chains = {}
        for name, batch, seed in (("decode_b5", 5, 0), ("decode_b256", 256, 1000)):
            c = inputs.decode_chain_inputs(inputs.ChainShape(batch=batch), seed=seed)
            self.chains[name] = (f64(c["residual"]),
                                 {k: [f64(t) for t in v] for k, v in c.items() if k != "residual"})
        self.bytes = step_bytes()
        self.sample = ("the whole step at full size: rmsnorm f32 64x1024, add_rmsnorm bf16 "
                       "4096x2048, swiglu bf16 8192x6144, mrope bf16 4096 tokens, one 28-layer "
                       "decode step at batch 5 and at batch 256 (every output of every layer)")

    def run(self, orc) -> dict:
        t = {}
        c0 = time.perf_counter()
        orc.round_to(orc.rmsnorm(self.rn["x"], self.rn["gamma"], 1e-6), "f32")
        c1 = time.perf_counter()
        t["rmsnorm"] = c1 - c0
        y, _ = orc.add_rmsnorm(self.an["x"], self.an["residual"], self.an["gamma"], 1e-6, "bf16")
        orc.round_bf16(y)
        c2 = time.perf_counter()
        t["add_rmsnorm"] = c2 - c1
        orc.round_bf16(orc.swiglu(self.sw["gate"], self.sw["up"]))
        c3 = time.perf_counter()
        t["swiglu"] = c3 - c2
        qo, ko = orc.mrope_qk(self.mr["q"], self.mr["k"], self.pos, (24, 20, 20), 1e6)
        orc.round_bf16(qo)
        orc.round_bf16(ko)
        c4 = time.perf_counter()
        t["mrope_qk"] = c4 - c3
        for name in ("decode_b5", "decode_b256"):
            res, layer_inputs = self.chains[name]
            c5 = time.perf_counter()
            orc.decode_step(res, layer_inputs, 0)
            t[name] = time.perf_counter() - c5
        return t


def cpu_baseline_report(ostep: "OracleStep") -> dict:
    """The oracle as it stands, timed on this host's cores on the whole step:
    the plain single-threaded build (the reported value) and the row-parallel
    OpenMP build of the same source on every core, with ms per configuration."""
    import oracle

    runs = {}
    for kind, orc in (("single", oracle.get()), ("omp", oracle.get_omp())):
        t = ostep.run(orc)
        total = sum(t.values())
        runs[kind] = {"value": sum(ostep.bytes.values()) / total / 1e9, "unit": UNIT,
                      "threads": orc.threads(), "ms_per_step": round(1e3 * total, 1),
                      "per_config_ms": {k: round(1e3 * v, 2) for k, v in t.items()}}
    single = runs["single"]
    return {"value": single["value"], "unit": UNIT, "cores": single["threads"], "kind": "oracle",
            "sample": ostep.sample + f"; plain single-threaded C oracle, fp64 "
                                     f"({single['ms_per_step'] / 1e3:.1f} s)",
            "single": single, "omp": runs["omp"],
            "per_config_ms": single["per_config_ms"],
            "nproc": os.cpu_count(), "affinity_cores": len(os.sched_getaffinity(0)),
            "cpu_model": cpu_model()}


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    ostep = OracleStep()
    orc = oracle.get()
    times = []
    per_config = {k: 0.0 for k in STEP_CONFIGS}
    for i in range(args.warmup + args.steps):
        t = ostep.run(orc)
        if i >= args.warmup:
            times.append(sum(t.values()))
            for k, v in t.items():
                per_config[k] += v
    total = sum(times)
    value = sum(ostep.bytes.values()) * len(times) / total / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": None, "parallelism": "replicas x1",
                   "l2": L2_NOTE},
        "method": {"sample": ostep.sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.threads(), "kind": "oracle",
                         "sample": ostep.sample + "; plain single-threaded C oracle, fp64",
                         "per_config_ms": {k: round(1e3 * v / len(times), 2)
                                           for k, v in per_config.items()},
                         "nproc": os.cpu_count(), "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-pdl", action="store_true", help="launch without programmatic dependent launch")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=6)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        run_reference(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, pg, device)

    import swiglu_ar_tts_b200 as ops

    ops.lib()
    step = Step(device, pdl=not args.no_pdl)
    step.capture()

    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(device)
    sampler.start()
    launches0 = ops.launch_count()
    barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    # a bounded device-side delay lets the host queue every timed step before
    # the GPU reaches it, so no host latency shows up inside the events
    torch.cuda._sleep(int(2e7))
    for k in range(args.steps):
        step.run(events[k])
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - wall0
    eager_launches = ops.launch_count() - launches0
    clocks = sampler.stop()

    step_ms = [ev[0].elapsed_time(ev[1]) for ev in events]
    total_ms = max_over_ranks(float(sum(step_ms)))
    ms_per_step = total_ms / args.steps
    step_bytes = sum(step.bytes[o] for o in Step.OPS)
    value = aggregate_value(world, step_bytes, args.steps, total_ms)
    step_us = 1e3 * ms_per_step

    # The step runs its operators back to back in one graph, so no event can sit
    # between two of them without breaking programmatic dependent launch.  Its
    # device time is split among them in proportion to what each adds to it
    # (step_marginals, outside the timed steps); each operator is also timed
    # alone (isolated_ops).
    peak, peak_kind = measured_hbm_peak()
    marg, marg_full = step_marginals(step)
    scale = step_us / sum(marg.values())
    ops_report = {}
    for name in Step.OPS:
        us = marg[name] * scale
        gbs = step.bytes[name] / (us * 1e-6) / 1e9
        ops_report[name] = {"us": round(us, 3), "bytes": step.bytes[name], "gbs": round(gbs, 1),
                            "frac_of_" + peak_kind + "_hbm": round(gbs / peak, 4),
                            "frac_of_spec_hbm": round(gbs / SPEC_HBM_GBS, 4),
                            "rows_per_s": round(step.rows[name] / (us * 1e-6)),
                            "us_marginal": round(marg[name], 3)}
    iso = isolated_ops(device, peak, peak_kind)
    sampling = sampling_ops(device, peak, peak_kind)
    # time per kernel type in the step: prefill operators are one launch each;
    # each decode step is split across its operators' kernels (decode_split)
    kernels: dict[str, dict] = {}

    def add_time(kernel, us, launches, nbytes):
        k = kernels.setdefault(kernel, {"us": 0.0, "launches": 0, "bytes": 0})
        k["us"] += us
        k["launches"] += launches
        k["bytes"] += nbytes

    for name in ("rmsnorm", "add_rmsnorm", "swiglu", "mrope_qk"):
        add_time(KERNEL_OF[name], ops_report[name]["us"], 1, step.bytes[name])
    decode_launch_us: dict[str, dict] = {}  # µs per decode launch, per kernel and batch
    for name, chain in (("decode_b5", step.chain5), ("decode_b256", step.chain256)):
        for op, (frac, launches, nbytes) in decode_split(chain).items():
            add_time(KERNEL_OF[op], frac * ops_report[name]["us"], launches, nbytes)
            decode_launch_us.setdefault(KERNEL_OF[op], {})[name] = round(
                frac * ops_report[name]["us"] / launches, 3)
    step_us = 1e3 * ms_per_step
    for kname, k in kernels.items():
        k["share"] = round(k["us"] / step_us, 4)
        k["gbs"] = round(k["bytes"] / (k["us"] * 1e-6) / 1e9, 1)
        k["us"] = round(k["us"], 2)
        k["us_per_decode_launch"] = decode_launch_us.get(kname, {})
    dominant = max(kernels, key=lambda k: kernels[k]["us"])
    dk = kernels[dominant]
    # traffic: DRAM bytes per launch averaged over the step's launches of the
    # kernel, from one ncu capture per launch size (profiles/traffic.json)
    dom_traffic = None
    if dominant == "norm_rows_kernel":
        dom_traffic = ncu_traffic("norm_rows_kernel", ("swiglu_ar_tts_b200/csrc/norm.cu",
                                                       "swiglu_ar_tts_b200/csrc/common.cuh"))
    roofline = {"kernel": dominant, "bound": "hbm", "achieved": dk["gbs"], "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dk["gbs"] / peak, 4),
                "traffic": dom_traffic, "launches_per_step": dk["launches"],
                "algorithmic_bytes_per_step": dk["bytes"],
                "algorithmic_bytes_per_launch": round(dk["bytes"] / dk["launches"]),
                "us_per_decode_launch": decode_launch_us.get(dominant, {}),
                "note": "dominant by share of step time; achieved = its algorithmic bytes per "
                        "step / its time per step; traffic = DRAM reads + bytes written into "
                        "L2 per launch (ncu, profiles/traffic.json), averaged over the step's "
                        "prefill and decode launches; all but 2 of its launches are "
                        "decode launches of 45 KB to 4.2 MB, bound by the latency of a "
                        "dependent launch (us_per_decode_launch) rather than by bandwidth"}
    sw_us = ops_report["swiglu"]["us"]
    sw_gbs = step.bytes["swiglu"] / (sw_us * 1e-6) / 1e9
    roofline_swiglu = {"kernel": "swiglu_vec_kernel<bf16> 8192x6144 (largest single launch)",
                       "bound": "hbm", "achieved": round(sw_gbs, 1), "peak": peak,
                       "peak_kind": peak_kind, "unit": "GB/s", "frac": round(sw_gbs / peak, 4),
                       "traffic": ncu_traffic("swiglu_vec_kernel",
                                              ("swiglu_ar_tts_b200/csrc/swiglu.cu",
                                               "swiglu_ar_tts_b200/csrc/common.cuh")),
                       "algorithmic_bytes": step.bytes["swiglu"]}

    # the LayerNorm -> RMSNorm swap of "Optimising autoregressive speech models"
    # §09: the same decode step with add + LayerNorm in every norm, timed alone
    # (outside the timed steps) against the add + RMSNorm step
    swap = {}
    for batch, chain in ((5, step.chain5), (256, step.chain256)):
        from swiglu_ar_tts_b200.chain import DecodeChain
        from swiglu_ar_tts_b200.inputs import ChainShape

        ln = DecodeChain(ChainShape(batch=batch), device=device, seed=2000 + batch,
                         pdl=not args.no_pdl, norm="layer")
        ln.capture()
        t = {}
        for name, c in (("rmsnorm", chain), ("layernorm", ln)):
            c.set_position(3)
            for _ in range(3):
                c._graph.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(20):
                c._graph.replay()
            e1.record()
            torch.cuda.synchronize()
            t[name] = 1e3 * e0.elapsed_time(e1) / 20
        swap[f"batch{batch}"] = {"us_rmsnorm_step": round(t["rmsnorm"], 2),
                                 "us_layernorm_step": round(t["layernorm"], 2),
                                 "rmsnorm_saves": round(1 - t["rmsnorm"] / t["layernorm"], 4)}
        del ln

    # a decoding run: 300 consecutive steps (positions 0..299, as the 300 decode
    # steps of an utterance), replaying the captured step graph and launching
    # the 112 operators one by one from the host loop, outside the timed steps
    run300 = {}
    for batch, chain in ((5, step.chain5), (256, step.chain256)):
        saved = chain.residual.clone()
        t = {}
        for mode in ("graph", "eager"):
            go = chain.replay if mode == "graph" else chain.step
            for s in range(3):
                go(s)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for s in range(300):
                go(s)
            e1.record()
            torch.cuda.synchronize()
            t[mode] = 1e3 * e0.elapsed_time(e1) / 300
        chain.residual.copy_(saved)
        run300[f"batch{batch}"] = {"graph_us_per_step": round(t["graph"], 2),
                                   "eager_us_per_step": round(t["eager"], 2)}

    # end to end: pinned host buffers in and out, through the same public
    # calls, on two sets of device buffers so that one step's inputs cross
    # PCIe while the previous step's results drain
    step.setup_e2e()
    step_b = Step(device, pdl=not args.no_pdl, like=step)
    step_b.setup_e2e(share=step)
    sets = [step, step_b]
    torch.cuda.synchronize()
    run_e2e_pipelined(sets, 2)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    run_e2e_pipelined(sets, args.e2e_steps)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    # the copies hand back exactly what the device holds (the last step's set)
    last = sets[(args.e2e_steps - 1) % len(sets)]
    for g, _ in last.E2E_GROUPS:
        for dst, src in last._e2e_out(g):
            if not torch.equal(dst, src.cpu()):
                raise SystemExit(f"e2e: host copy of {g} differs from the device result")
    e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / args.e2e_steps
    e2e = {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
           "ms_per_step": e2e_ms, "h2d_bytes_per_step": step.h2d_bytes,
           "d2h_bytes_per_step": step.d2h_bytes,
           "pipeline": "two device buffer sets; each step's inputs cross while the previous "
                       "step's results drain"}
    del step_b, sets, last

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_report(OracleStep())

    if pg is not None:
        pg.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": None, "parallelism": f"replicas x{world}",
                   "l2": L2_NOTE},
        "method": {"pdl": not args.no_pdl,
                   "timing": "each step is one replay of a CUDA graph of all 228 launches "
                             "(4 prefill, 112 + 112 decode), CUDA events around the replay; "
                             "ops[*].us = the step time split in proportion to what each "
                             "operator adds to the step graph's time (us_marginal: the "
                             "graph's time minus that of the graph without the operator)",
                   "step_split_scale": round(scale, 4),
                   "step_us_in_marginal_runs": round(marg_full, 2)},
        "us_per_decode_step": {"batch5": ops_report["decode_b5"]["us"],
                               "batch256": ops_report["decode_b256"]["us"]},
        "ops": ops_report,
        "ops_isolated": iso,
        "sampling": sampling,
        "roofline": roofline,
        "roofline_swiglu": roofline_swiglu,
        "kernels": kernels,
        "layernorm_to_rmsnorm": swap,
        "decode_300_steps": run300,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "gpu_launches": eager_launches + args.steps * step.kernels_per_step,
        "clocks": clocks,
        "wall_s_timed": wall,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
