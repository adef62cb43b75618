"""Per-operator timing on one GPU (CUDA events; inputs rotated through > 4x L2).

    python -m swiglu_ar_tts_b200.opbench --op swiglu --iters 50
    python -m swiglu_ar_tts_b200.opbench --op all

Shapes are the operators' workload sizes (add+RMSNorm bf16 4096x2048, SwiGLU
bf16 8192x6144, M-RoPE bf16 4096 tokens x 16/8 heads x 128, RMSNorm fp32
64x1024, decode steps at batch 5 and 256); ``--rows`` scales the row count.
Prints one line per operator: median and minimum microseconds per launch (each
launch between its own pair of events), the per-launch time of the same
launches back to back, and the algorithmic HBM GB/s (every operand read once,
every output written once) of both.

Each operator gets enough copies of its buffers to cover 512 MB (4x the L2) and
successive launches cycle through them, so every launch reads from DRAM and
pays for the write-back of earlier launches, as it does in steady state.  With
``--copies 1`` it is also the small driver used for ncu captures.
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

from . import (add_layernorm, add_rmsnorm, layernorm, mrope_qk, rmsnorm, set_pdl, set_streaming,
               set_topk_cluster, mrope_kv_append, swiglu, topk_sample, topk_sample_prepare,
               topk_sample_workspace)
from . import inputs as I
from .chain import DecodeChain

OPS = ("rmsnorm", "add_rmsnorm", "swiglu", "mrope_qk", "decode5", "decode256")
EXTRA_OPS = ("layernorm", "add_layernorm", "decode5_ln", "decode256_ln", "topk_sample",
             "mrope_kv_append", "copy_add_rmsnorm", "copy_mrope_qk", "copy_swiglu")
# Size-matched device copies: a plain device-to-device copy (torch's copy
# kernel, not this library's) that reads half and writes half of an
# operator's algorithmic bytes at the workload size, as the ceiling a kernel
# of that size and launch pattern can reach.
COPY_OF = {"copy_add_rmsnorm": (4 * 4096 * 2048 + 2048) * 2,
           "copy_mrope_qk": 2 * 4096 * 24 * 128 * 2 + 3 * 4096 * 4,
           "copy_swiglu": 3 * 8192 * 6144 * 2}


CHAIN_PDL = True


def make(op: str, rows: int | None, dev: torch.device, seed: int = 0):
    """Returns (launch callable, algorithmic bytes, shape description) for one
    copy of the operator's buffers."""
    if op == "rmsnorm":
        r = rows or 64
        t = {k: v.to(dev) for k, v in I.rmsnorm_inputs(r, 1024, "f32", seed).items()}
        y = torch.empty_like(t["x"])
        return (lambda: rmsnorm(t["x"], t["gamma"], I.EPS, out=y)), (2 * r * 1024 + 1024) * 4, f"f32 {r}x1024"
    if op == "add_rmsnorm":
        r = rows or 4096
        t = {k: v.to(dev) for k, v in I.add_rmsnorm_inputs(r, I.HIDDEN, "bf16", seed).items()}
        y, ro = torch.empty_like(t["x"]), torch.empty_like(t["x"])
        return ((lambda: add_rmsnorm(t["x"], t["residual"], t["gamma"], I.EPS, y=y, residual_out=ro)),
                (4 * r * I.HIDDEN + I.HIDDEN) * 2, f"bf16 {r}x{I.HIDDEN}")
    if op == "swiglu":
        r = rows or 8192
        t = {k: v.to(dev) for k, v in I.swiglu_inputs(r, I.INTER, "bf16", seed).items()}
        o = torch.empty_like(t["gate"])
        return (lambda: swiglu(t["gate"], t["up"], out=o)), 3 * r * I.INTER * 2, f"bf16 {r}x{I.INTER}"
    if op == "mrope_qk":
        r = rows or 4096
        t = {k: v.to(dev) for k, v in I.mrope_inputs(r, seed=seed).items()}
        qo, ko = torch.empty_like(t["q"]), torch.empty_like(t["k"])
        nb = 2 * r * (I.N_Q_HEADS + I.N_K_HEADS) * I.HEAD_DIM * 2 + 3 * r * 4
        return ((lambda: mrope_qk(t["q"], t["k"], t["pos"], I.SECTIONS, I.THETA, q_out=qo, k_out=ko)),
                nb, f"bf16 {r} tokens")
    if op == "layernorm":
        r = rows or 4096
        t = {k: v.to(dev) for k, v in I.rmsnorm_inputs(r, I.HIDDEN, "bf16", seed).items()}
        beta = I.normal((I.HIDDEN,), seed + 9, std=0.1).to(dev)
        y = torch.empty_like(t["x"])
        return ((lambda: layernorm(t["x"], t["gamma"], beta, I.EPS, out=y)),
                (2 * r * I.HIDDEN + 2 * I.HIDDEN) * 2, f"bf16 {r}x{I.HIDDEN}")
    if op == "add_layernorm":
        r = rows or 4096
        t = {k: v.to(dev) for k, v in I.add_rmsnorm_inputs(r, I.HIDDEN, "bf16", seed).items()}
        beta = I.normal((I.HIDDEN,), seed + 9, std=0.1).to(dev)
        y, ro = torch.empty_like(t["x"]), torch.empty_like(t["x"])
        return ((lambda: add_layernorm(t["x"], t["residual"], t["gamma"], beta, I.EPS, y=y,
                                       residual_out=ro)),
                (4 * r * I.HIDDEN + 2 * I.HIDDEN) * 2, f"bf16 {r}x{I.HIDDEN}")
    if op == "mrope_kv_append":
        r = rows or 4096
        hq, hk, d = I.N_Q_HEADS, I.N_K_HEADS, I.HEAD_DIM
        q = I.normal((r, hq, d), seed).to(dev)
        k = I.normal((r, hk, d), seed + 1).to(dev)
        v = I.normal((r, hk, d), seed + 2).to(dev)
        qo = torch.empty_like(q)
        cache_rows, max_seq = (r, 512) if r <= 256 else (1, r)
        kc = torch.zeros(cache_rows, hk, max_seq, d, dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        t = torch.arange(r, dtype=torch.int32)
        loc = (torch.stack([t, torch.full_like(t, 7)]) if r <= 256
               else torch.stack([torch.zeros_like(t), t])).to(dev)
        pos = I.mrope_positions(r).to(dev)
        nb = (2 * r * hq * d + 4 * r * hk * d) * 2 + 3 * r * 4 + 2 * r * 4
        return ((lambda: mrope_kv_append(q, k, v, pos, loc, kc, vc, I.SECTIONS, I.THETA, q_out=qo)),
                nb, f"bf16 {r} tokens, cache [{cache_rows},{hk},{max_seq},{d}]")
    if op == "topk_sample":
        r = rows or 5
        t = {k: v.to(dev) for k, v in I.topk_inputs(r, 151936, 50, "bf16", seed).items()}
        ws = topk_sample_prepare(torch.empty(topk_sample_workspace(r, 151936, 50),
                                             dtype=torch.uint8, device=dev))
        tok = torch.empty(r, dtype=torch.int32, device=dev)
        prob = torch.empty(r, dtype=torch.float32, device=dev)
        return ((lambda: topk_sample(t["logits"], t["gumbel"], 50, 0.8, workspace=ws,
                                     token_out=tok, prob_out=prob)),
                r * 151936 * 2 + r * 50 * 4 + r * 8, f"bf16 {r}x151936, top-50")
    if op in COPY_OF:
        half = COPY_OF[op] // 2 // 16 * 16
        src = torch.randint(0, 255, (half,), dtype=torch.uint8, device=dev)
        dst = torch.empty_like(src)
        return (lambda: dst.copy_(src)), 2 * half, f"device copy of {half} B"
    if op.startswith("decode"):
        b = rows or (5 if op.startswith("decode5") else 256)
        norm = "layer" if op.endswith("_ln") else "rms"
        c = DecodeChain(I.ChainShape(batch=b), device=dev, seed=seed, pdl=CHAIN_PDL, norm=norm)
        c.capture()
        c.set_position(7)
        return (lambda: c._graph.replay()), c.bytes_per_step(), f"28 layers, batch {b}, {norm}norm, graph"
    raise ValueError(op)


def make_rotation(op: str, rows: int | None, dev: torch.device, copies: int | None):
    fn, nbytes, desc = make(op, rows, dev)
    n = copies if copies is not None else max(1, min(64, -(-(512 << 20) // nbytes)))
    fns = [fn] + [make(op, rows, dev, seed=100 + i)[0] for i in range(n - 1)]
    return fns, nbytes, f"{desc}, {n} copies"


def time_op(fns, iters: int) -> list[float]:
    for f in fns:
        f()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    torch.cuda._sleep(int(5e7))  # let the host queue ahead of the device
    for i, (a, b) in enumerate(ev):
        a.record()
        fns[i % len(fns)]()
        b.record()
    torch.cuda.synchronize()
    return [1e3 * a.elapsed_time(b) for a, b in ev]


def time_back_to_back(fns, iters: int) -> float:
    """Microseconds per launch of ``iters`` launches enqueued back to back
    between one pair of events (with programmatic dependent launch when it is
    enabled, each launch overlaps its predecessor's drain)."""
    for f in fns:
        f()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(int(5e7))
    e0.record()
    for i in range(iters):
        fns[i % len(fns)]()
    e1.record()
    torch.cuda.synchronize()
    return 1e3 * e0.elapsed_time(e1) / iters


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", default="all", choices=("all",) + OPS + EXTRA_OPS)
    ap.add_argument("--iters", type=int, default=50)
    ap.add_argument("--rows", type=int, default=None)
    ap.add_argument("--copies", type=int, default=None,
                    help="buffer copies to rotate through (default: enough for 512 MB)")
    ap.add_argument("--pdl", action="store_true")
    ap.add_argument("--streaming", action="store_true",
                    help="shared-memory streaming kernels instead of the default register kernels")
    ap.add_argument("--no-chain-pdl", action="store_true",
                    help="decode steps without programmatic dependent launch")
    ap.add_argument("--topk-mode", type=int, default=1, choices=(0, 1, 2, 3),
                    help="top-k kernels: 0 slice, 1 cluster (default), 2 shared-memory cluster")
    ap.add_argument("--json", action="store_true")
    a = ap.parse_args()
    dev = torch.device("cuda", torch.cuda.current_device())
    global CHAIN_PDL
    CHAIN_PDL = not a.no_chain_pdl
    set_pdl(a.pdl)
    set_streaming(a.streaming)
    set_topk_cluster(a.topk_mode)
    for op in (OPS if a.op == "all" else (a.op,)):
        fns, nbytes, desc = make_rotation(op, a.rows, dev, a.copies)
        us = time_op(fns, a.iters)
        b2b = time_back_to_back(fns, a.iters)
        med = statistics.median(us)
        rec = {"op": op, "shape": desc, "bytes": nbytes, "us_median": round(med, 3),
               "us_mean": round(statistics.fmean(us), 3), "us_min": round(min(us), 3),
               "gbs_median": round(nbytes / (med * 1e-6) / 1e9, 1),
               "us_back_to_back": round(b2b, 3),
               "gbs_back_to_back": round(nbytes / (b2b * 1e-6) / 1e9, 1)}
        print(json.dumps(rec) if a.json else
              f"{op:12s} {desc:40s} median {med:9.3f} us  min {min(us):9.3f} us  "
              f"{rec['gbs_median']:8.1f} GB/s  back to back {b2b:9.3f} us "
              f"{rec['gbs_back_to_back']:8.1f} GB/s", flush=True)


if __name__ == "__main__":
    main()
