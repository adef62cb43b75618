"""Decode-step chain over the library's operators.

One decode step of an autoregressive speech decoder (one new token for each of
``batch`` candidates, e.g. the 5 candidates generated together in the Triton
kernel-fusion post for Qwen3-TTS, section 1) runs, for each layer:

    add + RMSNorm  (attention input)      residual <- residual + x_attn
    M-RoPE on q, k at the step's position (all three rows t/h/w = step)
    add + RMSNorm  (MLP input)            residual <- residual + x_mlp
    SwiGLU         (MLP activation)

With ``norm="layer"`` both norms are add + LayerNorm (with a beta per norm),
the architecture that "Optimising autoregressive speech models" §09 swaps for
RMSNorm; timing both chains measures that swap.

The projections, attention and MLP GEMMs between these operators are not part
of this library; their outputs are stood in for by fixed per-layer buffers, so
a step is exactly the 4 * layers operator launches.  The residual stream is the
only state carried from layer to layer and from step to step.

``DecodeChain`` owns the device buffers and launches each operator through the
C ABI with pre-bound arguments (no per-call tensor checks), either eagerly on
the current stream or replayed from a CUDA graph of one step.  By default the
launches use programmatic dependent launch: each kernel is scheduled while its
predecessor drains and prefetches its first inputs into L2 before waiting for
it, which removes most of the per-launch gap of a 112-kernel step.
"""
from __future__ import annotations

import ctypes

import torch

from . import DTYPES, ArOpsError, lib
from .inputs import EPS, SECTIONS, THETA, ChainShape, decode_chain_inputs, normal


def _pack(tensors, device, fill: bool = True):
    """One flat device buffer holding a view shaped like each tensor (copied
    into it when ``fill``), every view starting on a 16-byte boundary."""
    dtype = tensors[0].dtype
    esize = tensors[0].element_size()
    align = max(1, 16 // esize)
    offs, total = [], 0
    for t in tensors:
        assert t.dtype == dtype
        offs.append(total)
        total += -(-t.numel() // align) * align
    flat = torch.empty(max(total, 1), dtype=dtype, device=device)
    views = []
    for t, o in zip(tensors, offs):
        v = flat[o:o + t.numel()].view(t.shape)
        if fill:
            v.copy_(t)
        views.append(v)
    return flat, views


class DecodeChain:
    def __init__(self, shape: ChainShape, dtype: str = "bf16", seed: int = 0,
                 device: str | torch.device = "cuda", eps: float = EPS, theta: float = THETA,
                 sections=SECTIONS, host_inputs: dict | None = None, pdl: bool = True,
                 norm: str = "rms"):
        self.shape = shape
        self.dtype = dtype
        self.eps = eps
        self.theta = theta
        self.sections = tuple(int(s) for s in sections)
        self.pdl = pdl
        if norm not in ("rms", "layer"):
            raise ValueError(norm)
        self.norm = norm
        self.device = torch.device(device)
        host = host_inputs if host_inputs is not None else decode_chain_inputs(shape, dtype, seed)
        if norm == "layer" and "beta_attn" not in host:
            host = dict(host)
            host["beta_attn"] = [normal((shape.hidden,), seed + 500_000 + 2 * l, std=0.1, dtype=dtype)
                                 for l in range(shape.layers)]
            host["beta_mlp"] = [normal((shape.hidden,), seed + 500_001 + 2 * l, std=0.1, dtype=dtype)
                                for l in range(shape.layers)]
        self.host_inputs = host
        d = self.device
        self.residual0 = host["residual"].to(d)
        self.residual = self.residual0.clone()
        # Every per-layer input lives in one flat device buffer (`flat_in`) and
        # every per-layer output in another (`flat_out`), as views: a step's
        # inputs or outputs then move to or from the host as one copy each.
        # Each view starts on a 16-byte boundary (all sizes are multiples of 16
        # bytes for these shapes; odd ones are padded).
        in_keys = [k for k in host if k != "residual"]
        self.flat_in, views = _pack([t for k in in_keys for t in host[k]], d)
        self.inp = {}
        for k in in_keys:
            self.inp[k], views = views[:len(host[k])], views[len(host[k]):]
        L, B = shape.layers, shape.batch
        outs = ([t for t in self.inp["x_attn"]] + [t for t in self.inp["x_mlp"]] +
                [t for t in self.inp["q"]] + [t for t in self.inp["k"]] +
                [t for t in self.inp["gate"]])
        self.flat_out, views = _pack(outs, d, fill=False)
        self.y_attn, self.y_mlp = views[:L], views[L:2 * L]
        self.q_out, self.k_out, self.act = views[2 * L:3 * L], views[3 * L:4 * L], views[4 * L:]
        self.pos = torch.zeros(3, B, dtype=torch.int32, device=d)  # the step's position ids
        self._graph: torch.cuda.CUDAGraph | None = None
        self._graph_stream: int | None = None
        self._bind()

    # -- pre-bound C calls ----------------------------------------------------
    def _bind(self) -> None:
        L = lib()
        sh = self.shape
        code = DTYPES[self.residual.dtype]
        eps = ctypes.c_float(self.eps)
        theta = ctypes.c_float(self.theta)
        self._sec = (ctypes.c_int32 * 3)(*self.sections)
        res = self.residual.data_ptr()
        B, H, I = sh.batch, sh.hidden, sh.inter
        calls = []
        def norm_call(x, gamma, beta, y):
            if self.norm == "layer":
                return (L.arops_add_layernorm, [x.data_ptr(), res, res, gamma.data_ptr(),
                                                beta.data_ptr(), y.data_ptr(), B, H, eps, code])
            return (L.arops_add_rmsnorm, [x.data_ptr(), res, res, gamma.data_ptr(),
                                          y.data_ptr(), B, H, eps, code])

        for l in range(sh.layers):
            ba = self.inp["beta_attn"][l] if self.norm == "layer" else None
            bm = self.inp["beta_mlp"][l] if self.norm == "layer" else None
            calls.append(norm_call(self.inp["x_attn"][l], self.inp["gamma_attn"][l], ba,
                                   self.y_attn[l]))
            calls.append((L.arops_mrope_qk, [self.inp["q"][l].data_ptr(), self.inp["k"][l].data_ptr(),
                                             self.q_out[l].data_ptr(), self.k_out[l].data_ptr(),
                                             self.pos.data_ptr(), B, sh.n_q_heads, sh.n_k_heads,
                                             sh.head_dim, self._sec, theta, code]))
            calls.append(norm_call(self.inp["x_mlp"][l], self.inp["gamma_mlp"][l], bm,
                                   self.y_mlp[l]))
            calls.append((L.arops_swiglu, [self.inp["gate"][l].data_ptr(), self.inp["up"][l].data_ptr(),
                                           self.act[l].data_ptr(), B, I, code]))
        self._calls = calls

    @property
    def launches_per_step(self) -> int:
        return len(self._calls)

    def bytes_per_step(self) -> int:
        """Algorithmic HBM bytes of one step: every operand read once, every
        output written once (positions 12 B per row, norm weights once per norm)."""
        sh = self.shape
        e = self.residual.element_size()
        B, H, I = sh.batch, sh.hidden, sh.inter
        weights = 2 if self.norm == "layer" else 1  # gamma (and beta) per norm
        per_layer = (2 * (4 * B * H + weights * H) * e  # two add+norms: x, res in; res', y out
                     + 2 * B * (sh.n_q_heads + sh.n_k_heads) * sh.head_dim * e + 3 * B * 4
                     + 3 * B * I * e)
        return sh.layers * per_layer

    # -- execution ---------------------------------------------------------------
    def reset(self) -> None:
        self.residual.copy_(self.residual0)

    def set_position(self, step: int) -> None:
        """Position ids of decode step ``step`` (all rows equal to the step)."""
        self.pos.fill_(step)

    def launch_step(self, stream: int | None = None) -> None:
        """Enqueue the 4 * layers operator launches of one step (positions as set)."""
        if stream is None:
            stream = torch.cuda.current_stream(self.device).cuda_stream
        L = lib()
        old = L.arops_set_pdl(1 if self.pdl else 0)
        try:
            for fn, args in self._calls:
                st = fn(*args, stream)
                if st != 0:
                    raise ArOpsError(st, f"{L.arops_status_string(st).decode()}: "
                                         f"{L.arops_last_error().decode()}")
        finally:
            L.arops_set_pdl(old)

    def step(self, step: int) -> None:
        self.set_position(step)
        self.launch_step()

    def capture(self) -> torch.cuda.CUDAGraph:
        """Capture one step (positions read from ``self.pos``) as a CUDA graph."""
        with torch.cuda.device(self.device):
            saved = self.residual.clone()
            s = torch.cuda.Stream(self.device)
            s.wait_stream(torch.cuda.current_stream(self.device))
            with torch.cuda.stream(s):  # warm-up outside capture
                self.launch_step()
            torch.cuda.current_stream(self.device).wait_stream(s)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.launch_step()
            self.residual.copy_(saved)
        self._graph = g
        return g

    def replay(self, step: int) -> None:
        if self._graph is None:
            self.capture()
        self.set_position(step)
        self._graph.replay()
