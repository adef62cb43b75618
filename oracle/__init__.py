"""fp64 CPU oracle for RMSNorm, residual-add + RMSNorm, M-RoPE and SwiGLU.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The GPU library never imports it and shares no code with it.

The arithmetic lives in ``arops_oracle.c`` (plain C loops in fp64, compiled
without fast-math or FMA contraction).  This module only compiles that file with
gcc, loads it with ctypes and moves numpy arrays in and out.

Sources, by page title and section:
  * "Optimising autoregressive speech models", §09 "LayerNorm -> RMSNorm":
    RMSNorm(x) = gamma * x / sqrt(mean(x^2) + eps), eps = 1e-6 by default.
  * "Open Source: Triton-Kernel-Fusion ..." (news.hada.io 27742), section 3: the
    operators RMSNorm, M-RoPE, Norm+Residual and SwiGLU.
  * forpes.ru post 233929, "Stage 2": RoPE rotates Q and K in the complex plane.

Every function here is pinned by ``tests/test_oracle_pins.py`` (closed forms,
invariants, textbook special cases) and the pins are shown to catch planted
mistakes by ``tests/test_oracle_mutants.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "arops_oracle.c")
_BUILD = os.path.join(_HERE, "_build")

_c_double_p = ctypes.POINTER(ctypes.c_double)
_c_u16_p = ctypes.POINTER(ctypes.c_uint16)
_c_i32_p = ctypes.POINTER(ctypes.c_int32)


def lib_path(mutant: int = 0, omp: bool = False) -> str:
    if omp:
        assert mutant == 0
        return os.path.join(_BUILD, "liboracle_omp.so")
    name = "liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so"
    return os.path.join(_BUILD, name)


def build(mutant: int = 0, force: bool = False, omp: bool = False) -> str:
    """Compile the oracle (optionally with planted mistake ``mutant``).  With
    ``omp`` the same source is compiled with -fopenmp into liboracle_omp.so,
    whose marked row loops run across the host cores (the multi-core CPU
    baseline); the plain build is the oracle the tests use."""
    out = lib_path(mutant, omp)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    os.makedirs(_BUILD, exist_ok=True)
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=_BUILD)
    os.close(fd)
    # the oracle itself builds free of warnings; a planted mistake may leave a
    # term unused, so mutants only report theirs
    warn = ["-Wall", "-Wextra", "-Wpedantic"] + (["-Werror"] if int(mutant) == 0 else [])
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", *warn,
           *(["-fopenmp"] if omp else []),
           "-shared", f"-DORACLE_MUTANT={int(mutant)}", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _f64(a) -> np.ndarray:
    """fp64, C-contiguous copy of a numpy array or a CPU torch tensor."""
    if hasattr(a, "detach"):  # torch tensor: widening bf16/fp32 to fp64 is exact
        import torch

        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctype)


class Oracle:
    """ctypes view of one build of the oracle library."""

    def __init__(self, mutant: int = 0, omp: bool = False):
        self.mutant = mutant
        self.omp = omp
        self._lib = ctypes.CDLL(build(mutant, omp=omp))
        L = self._lib
        L.oracle_round_bf16_array.argtypes = [_c_double_p, _c_u16_p, ctypes.c_int64]
        L.oracle_bf16_value_array.argtypes = [_c_u16_p, _c_double_p, ctypes.c_int64]
        L.oracle_rmsnorm.argtypes = [_c_double_p, _c_double_p, _c_double_p,
                                     ctypes.c_int64, ctypes.c_int64, ctypes.c_double]
        L.oracle_add_rmsnorm.argtypes = [_c_double_p, _c_double_p, _c_double_p, _c_double_p,
                                         _c_double_p, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_double, ctypes.c_int]
        L.oracle_mrope_qk.argtypes = [_c_double_p, _c_double_p, _c_double_p, _c_double_p,
                                      _c_i32_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, _c_i32_p, ctypes.c_double]
        L.oracle_swiglu.argtypes = [_c_double_p, _c_double_p, _c_double_p, ctypes.c_int64]
        L.oracle_layernorm.argtypes = [_c_double_p, _c_double_p, _c_double_p, _c_double_p,
                                       ctypes.c_int64, ctypes.c_int64, ctypes.c_double]
        L.oracle_add_layernorm.argtypes = [_c_double_p, _c_double_p, _c_double_p, _c_double_p,
                                           _c_double_p, _c_double_p, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_double, ctypes.c_int]
        L.oracle_topk_sample.argtypes = [_c_double_p, ctypes.POINTER(ctypes.c_float), _c_i32_p,
                                         _c_double_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_float, ctypes.c_void_p]
        L.oracle_mrope_kv_append.argtypes = [
            _c_double_p, _c_double_p, _c_double_p, _c_double_p, _c_double_p, _c_double_p,
            _c_i32_p, _c_i32_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int64, _c_i32_p, ctypes.c_double, _c_double_p]
        L.oracle_mutant.restype = ctypes.c_int
        L.oracle_threads.restype = ctypes.c_int
        assert L.oracle_mutant() == mutant

    def threads(self) -> int:
        """Host threads this build's row loops use (1 for the plain build)."""
        return int(self._lib.oracle_threads())

    # -- dtype rounding ------------------------------------------------------
    def round_bf16(self, v) -> np.ndarray:
        """fp64 -> bf16 bit patterns (uint16), round to nearest even, direct."""
        v = _f64(v)
        out = np.empty(v.shape, dtype=np.uint16)
        self._lib.oracle_round_bf16_array(_ptr(v, _c_double_p), _ptr(out, _c_u16_p), v.size)
        return out

    def bf16_value(self, bits) -> np.ndarray:
        """Exact fp64 value of bf16 bit patterns."""
        bits = np.ascontiguousarray(bits, dtype=np.uint16)
        out = np.empty(bits.shape, dtype=np.float64)
        self._lib.oracle_bf16_value_array(_ptr(bits, _c_u16_p), _ptr(out, _c_double_p), bits.size)
        return out

    def round_to(self, v, dtype: str) -> np.ndarray:
        """fp64 result rounded once to ``dtype`` ('bf16' or 'f32'), returned as
        fp64 values of the rounded numbers."""
        if dtype == "bf16":
            return self.bf16_value(self.round_bf16(v))
        if dtype == "f32":
            return _f64(v).astype(np.float32).astype(np.float64)
        raise ValueError(dtype)

    # -- operators (fp64 in, fp64 out) --------------------------------------
    def rmsnorm(self, x, gamma, eps: float = 1e-6) -> np.ndarray:
        x = _f64(x)
        gamma = _f64(gamma)
        hidden = x.shape[-1]
        rows = x.size // hidden if hidden else 0
        assert gamma.shape == (hidden,)
        y = np.empty_like(x)
        self._lib.oracle_rmsnorm(_ptr(x, _c_double_p), _ptr(gamma, _c_double_p),
                                 _ptr(y, _c_double_p), rows, hidden, float(eps))
        return y

    def add_rmsnorm(self, x, residual, gamma, eps: float = 1e-6, dtype: str = "bf16"):
        """Returns (y, residual_out); residual_out is already rounded to dtype,
        y is the unrounded fp64 norm of it."""
        x = _f64(x)
        residual = _f64(residual)
        gamma = _f64(gamma)
        assert x.shape == residual.shape
        hidden = x.shape[-1]
        rows = x.size // hidden if hidden else 0
        y = np.empty_like(x)
        res_out = np.empty_like(x)
        code = {"f32": 0, "bf16": 1}[dtype]
        self._lib.oracle_add_rmsnorm(_ptr(x, _c_double_p), _ptr(residual, _c_double_p),
                                     _ptr(gamma, _c_double_p), _ptr(y, _c_double_p),
                                     _ptr(res_out, _c_double_p), rows, hidden, float(eps), code)
        return y, res_out

    def mrope_qk(self, q, k, pos, sections=(24, 20, 20), theta: float = 1e6):
        """q: [T, Hq, D], k: [T, Hk, D], pos: [3, T] int32 -> (q_out, k_out)."""
        q = _f64(q)
        k = _f64(k)
        if hasattr(pos, "detach"):
            pos = pos.detach().cpu().numpy()
        pos = np.ascontiguousarray(pos, dtype=np.int32)
        sec = np.ascontiguousarray(sections, dtype=np.int32)
        tokens, hq, d = q.shape
        hk = k.shape[1]
        assert k.shape == (tokens, hk, d) and pos.shape == (3, tokens)
        q_out = np.empty_like(q)
        k_out = np.empty_like(k)
        self._lib.oracle_mrope_qk(_ptr(q, _c_double_p), _ptr(k, _c_double_p),
                                  _ptr(q_out, _c_double_p), _ptr(k_out, _c_double_p),
                                  _ptr(pos, _c_i32_p), tokens, hq, hk, d,
                                  _ptr(sec, _c_i32_p), float(theta))
        return q_out, k_out

    def layernorm(self, x, gamma, beta, eps: float = 1e-6) -> np.ndarray:
        """gamma * (x - mean) / sqrt(var + eps) + beta over the last dimension
        (population variance)."""
        x = _f64(x)
        gamma = _f64(gamma)
        beta = _f64(beta)
        hidden = x.shape[-1]
        rows = x.size // hidden if hidden else 0
        assert gamma.shape == (hidden,) and beta.shape == (hidden,)
        y = np.empty_like(x)
        self._lib.oracle_layernorm(_ptr(x, _c_double_p), _ptr(gamma, _c_double_p),
                                   _ptr(beta, _c_double_p), _ptr(y, _c_double_p), rows, hidden,
                                   float(eps))
        return y

    def add_layernorm(self, x, residual, gamma, beta, eps: float = 1e-6, dtype: str = "bf16"):
        """Returns (y, residual_out) with residual_out = round(x + residual)."""
        x = _f64(x)
        residual = _f64(residual)
        gamma = _f64(gamma)
        beta = _f64(beta)
        hidden = x.shape[-1]
        rows = x.size // hidden if hidden else 0
        y = np.empty_like(x)
        res_out = np.empty_like(x)
        code = {"f32": 0, "bf16": 1}[dtype]
        self._lib.oracle_add_layernorm(_ptr(x, _c_double_p), _ptr(residual, _c_double_p),
                                       _ptr(gamma, _c_double_p), _ptr(beta, _c_double_p),
                                       _ptr(y, _c_double_p), _ptr(res_out, _c_double_p), rows,
                                       hidden, float(eps), code)
        return y, res_out

    def mrope_kv_append(self, q, k, v, pos, cache_loc, k_cache, v_cache, sections=(24, 20, 20),
                        theta: float = 1e6):
        """q [T, Hq, D], k/v [T, Hkv, D], pos [3, T], cache_loc [2, T] int32
        (cache row, position); k_cache/v_cache [rows, Hkv, max_seq, D] (their
        current contents).  Returns (q_out, k_cache', v_cache') in fp64."""
        q = _f64(q)
        k = _f64(k)
        v = _f64(v)
        kc = _f64(k_cache).copy()
        vc = _f64(v_cache).copy()
        pos = np.ascontiguousarray(pos.detach().cpu().numpy() if hasattr(pos, "detach") else pos,
                                   dtype=np.int32)
        loc = np.ascontiguousarray(cache_loc.detach().cpu().numpy()
                                   if hasattr(cache_loc, "detach") else cache_loc, dtype=np.int32)
        sec = np.ascontiguousarray(sections, dtype=np.int32)
        tokens, hq, d = q.shape
        hk = k.shape[1]
        rows, hk2, max_seq, d2 = kc.shape
        assert hk2 == hk and d2 == d and v.shape == k.shape and vc.shape == kc.shape
        assert pos.shape == (3, tokens) and loc.shape == (2, tokens)
        q_out = np.empty_like(q)
        k_rot = np.empty_like(k)
        self._lib.oracle_mrope_kv_append(
            _ptr(q, _c_double_p), _ptr(k, _c_double_p), _ptr(v, _c_double_p),
            _ptr(q_out, _c_double_p), _ptr(kc, _c_double_p), _ptr(vc, _c_double_p),
            _ptr(pos, _c_i32_p), _ptr(loc, _c_i32_p), tokens, hq, hk, d, rows, max_seq,
            _ptr(sec, _c_i32_p), float(theta), _ptr(k_rot, _c_double_p))
        return q_out, kc, vc

    def swiglu(self, gate, up) -> np.ndarray:
        gate = _f64(gate)
        up = _f64(up)
        assert gate.shape == up.shape
        out = np.empty_like(gate)
        self._lib.oracle_swiglu(_ptr(gate, _c_double_p), _ptr(up, _c_double_p),
                                _ptr(out, _c_double_p), gate.size)
        return out

    def topk_sample(self, logits, gumbel, top_k: int, temperature: float):
        """Gumbel-max sample from softmax(logits / T) restricted to the top_k
        logits.  logits [B, V]; gumbel [B, top_k] fp32 (draw j goes to the j-th
        largest logit).  Returns (token int32 [B], probability fp64 [B])."""
        logits = _f64(logits)
        g = np.ascontiguousarray(gumbel.detach().cpu().numpy() if hasattr(gumbel, "detach")
                                 else gumbel, dtype=np.float32)
        rows, vocab = logits.shape
        k = int(top_k)
        assert g.shape == (rows, k) and 1 <= k <= vocab
        tok = np.empty(rows, dtype=np.int32)
        prob = np.empty(rows, dtype=np.float64)
        scratch = ctypes.create_string_buffer(16 * k)
        self._lib.oracle_topk_sample(_ptr(logits, _c_double_p),
                                     g.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                     _ptr(tok, _c_i32_p), _ptr(prob, _c_double_p), rows, vocab, k,
                                     float(temperature), ctypes.cast(scratch, ctypes.c_void_p))
        return tok, prob

    # -- decode-step chain ---------------------------------------------------
    def decode_step(self, residual, layer_inputs: dict, step: int, eps: float = 1e-6,
                    theta: float = 1e6, sections=(24, 20, 20), dtype: str = "bf16",
                    outputs: bool = True, norm: str = "rms"):
        """One decode step over every layer, in the order add+RMSNorm, M-RoPE on
        q/k at position ``step`` in all three rows, add+RMSNorm, SwiGLU.

        ``residual`` is [B, H]; ``layer_inputs`` holds per-layer lists under the
        keys x_attn, gamma_attn, q, k, x_mlp, gamma_mlp, gate, up.  Every output
        is rounded to ``dtype`` at the operator boundary, as the GPU writes it.
        Returns (residual after the step, dict of per-layer outputs y_attn, q, k,
        y_mlp, act).  With ``outputs=False`` only the residual stream is
        computed and the dict is empty.  ``norm="layer"`` uses add + LayerNorm
        with betas from layer_inputs["beta_attn"] / ["beta_mlp"]."""
        res = _f64(residual)
        batch = res.shape[0]
        pos = np.full((3, batch), step, dtype=np.int32)
        outs = {"y_attn": [], "q": [], "k": [], "y_mlp": [], "act": []}
        def add_norm(x, r, key, layer):
            if norm == "layer":
                return self.add_layernorm(x, r, layer_inputs["gamma_" + key][layer],
                                          layer_inputs["beta_" + key][layer], eps, dtype)
            return self.add_rmsnorm(x, r, layer_inputs["gamma_" + key][layer], eps, dtype)

        m = self.mutant  # planted plumbing mistakes 19-22 (0: none)
        if m == 22:
            pos = pos + 1  # planted: positions one step ahead
        for layer in range(len(layer_inputs["x_attn"])):
            y, res = add_norm(layer_inputs["x_attn"][layer], res, "attn", layer)
            mlp_key = "attn" if m == 21 else "mlp"  # 21 planted: the MLP norm takes the attention weights
            if not outputs:
                _, res = add_norm(layer_inputs["x_mlp"][layer], res, mlp_key, layer)
                continue
            outs["y_attn"].append(self.round_to(y, dtype))
            qo, ko = self.mrope_qk(layer_inputs["q"][layer], layer_inputs["k"][layer], pos,
                                   sections, theta)
            outs["q"].append(self.round_to(qo, dtype))
            outs["k"].append(self.round_to(qo if m == 20 else ko, dtype))  # 20 planted: q for k
            y, res = add_norm(layer_inputs["x_mlp"][layer], res, mlp_key, layer)
            outs["y_mlp"].append(self.round_to(y, dtype))
            g, u = layer_inputs["gate"][layer], layer_inputs["up"][layer]
            if m == 19:
                g, u = u, g  # planted: gate and up swapped
            act = self.swiglu(g, u)
            outs["act"].append(self.round_to(act, dtype))
        if not outputs:
            outs = {}
        return res, outs


_default: Oracle | None = None
_omp: Oracle | None = None


def get() -> Oracle:
    """The oracle without planted mistakes (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle(0)
    return _default


def get_omp() -> Oracle:
    """The row-parallel (OpenMP) build of the same oracle, for timing on all
    host cores; its results equal the plain build's bit for bit."""
    global _omp
    if _omp is None:
        _omp = Oracle(0, omp=True)
    return _omp
