"""Python binding of libarops.so: per-token decode operators for B200 (sm_100a).

Thin ctypes wrappers with the names of the C entry points in ``include/arops.h``
(``arops_rmsnorm`` -> ``rmsnorm`` and so on).  They check that the tensors are
CUDA, contiguous and of one dtype, then pass ``data_ptr()`` values, sizes and
torch's current CUDA stream to the library.  Every step of every operator runs
in the library's CUDA kernels; there is no fallback of any kind.  If the shared
library has not been built, every call raises.

Build the library with ``python -m swiglu_ar_tts_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "rmsnorm", "add_rmsnorm", "layernorm", "add_layernorm", "mrope_qk", "mrope_kv_append",
    "swiglu", "set_pdl",
    "set_streaming", "set_topk_cluster", "topk_sample", "topk_sample_workspace", "topk_sample_prepare",
    "device_errors", "launch_count",
    "lib", "lib_path", "ArOpsError", "DTYPES",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libarops.so")

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA = 0, 1, 2, 3
DTYPES = {torch.float32: 0, torch.bfloat16: 1}

_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32


class ArOpsError(RuntimeError):
    """A non-OK status from libarops; ``status`` holds the code."""

    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


def lib_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded libarops.so (loaded on first use; raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m swiglu_ar_tts_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        L.arops_rmsnorm.argtypes = [_vp, _vp, _vp, _i64, _i64, ctypes.c_float, ctypes.c_int, _vp]
        L.arops_add_rmsnorm.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, ctypes.c_float,
                                        ctypes.c_int, _vp]
        L.arops_mrope_qk.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32,
                                     ctypes.POINTER(_i32), ctypes.c_float, ctypes.c_int, _vp]
        L.arops_swiglu.argtypes = [_vp, _vp, _vp, _i64, _i64, ctypes.c_int, _vp]
        L.arops_mrope_kv_append.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32,
                                            _i32, _i32, _i64, _i64, ctypes.POINTER(_i32),
                                            ctypes.c_float, ctypes.c_int, _vp]
        L.arops_mrope_kv_append.restype = ctypes.c_int
        L.arops_layernorm.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, ctypes.c_float,
                                      ctypes.c_int, _vp]
        L.arops_add_layernorm.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                          ctypes.c_float, ctypes.c_int, _vp]
        for fn in ("arops_rmsnorm", "arops_add_rmsnorm", "arops_mrope_qk", "arops_swiglu",
                   "arops_layernorm", "arops_add_layernorm"):
            getattr(L, fn).restype = ctypes.c_int
        L.arops_topk_sample_workspace.argtypes = [_i64, _i64, _i32, ctypes.POINTER(ctypes.c_size_t)]
        L.arops_topk_sample_workspace.restype = ctypes.c_int
        L.arops_topk_sample_prepare.argtypes = [_vp, ctypes.c_size_t, _vp]
        L.arops_topk_sample_prepare.restype = ctypes.c_int
        L.arops_topk_sample.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i32, ctypes.c_float,
                                        ctypes.c_int, _vp, ctypes.c_size_t, _vp]
        L.arops_topk_sample.restype = ctypes.c_int
        L.arops_set_pdl.argtypes = [ctypes.c_int]
        L.arops_set_pdl.restype = ctypes.c_int
        L.arops_set_streaming.argtypes = [ctypes.c_int]
        L.arops_set_streaming.restype = ctypes.c_int
        L.arops_set_topk_cluster.argtypes = [ctypes.c_int]
        L.arops_set_topk_cluster.restype = ctypes.c_int
        L.arops_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
        L.arops_device_errors.restype = ctypes.c_int
        L.arops_launch_count.restype = ctypes.c_uint64
        L.arops_status_string.argtypes = [ctypes.c_int]
        L.arops_status_string.restype = ctypes.c_char_p
        L.arops_last_error.restype = ctypes.c_char_p
        L.arops_version.restype = ctypes.c_int
        _lib = L
        return L


def _check(status: int) -> None:
    if status != OK:
        L = lib()
        raise ArOpsError(status, f"{L.arops_status_string(status).decode()}: "
                                 f"{L.arops_last_error().decode()}")


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _dtype_code(*ts: torch.Tensor) -> int:
    dt = ts[0].dtype
    if dt not in DTYPES:
        raise TypeError(f"unsupported dtype {dt}; use torch.float32 or torch.bfloat16")
    for t in ts:
        if t.dtype != dt:
            raise TypeError(f"dtype mismatch: {t.dtype} vs {dt}")
    return DTYPES[dt]


def _check_tensors(named) -> None:
    """Every (name, tensor) is a contiguous CUDA tensor on the first one's device:
    the kernels receive raw pointers and run on that device."""
    dev = None
    for name, t in named:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other tensors on {dev}")


def rmsnorm(x: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
            out: torch.Tensor | None = None) -> torch.Tensor:
    """y = gamma * x / sqrt(mean(x^2, -1) + eps); ``out`` may be ``x``."""
    hidden = x.shape[-1]
    if out is None:
        out = torch.empty_like(x)
    _check_tensors((("x", x), ("gamma", gamma), ("out", out)))
    if gamma.shape != (hidden,) or out.shape != x.shape:
        raise ValueError("shape mismatch")
    code = _dtype_code(x, gamma, out)
    rows = x.numel() // hidden if hidden else 0
    with torch.cuda.device(x.device):
        _check(lib().arops_rmsnorm(x.data_ptr(), gamma.data_ptr(), out.data_ptr(), rows, hidden,
                                   float(eps), code, _stream(x)))
    return out


def add_rmsnorm(x: torch.Tensor, residual: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                y: torch.Tensor | None = None, residual_out: torch.Tensor | None = None):
    """residual_out = x + residual (rounded to the dtype); y = RMSNorm(residual_out).

    ``residual_out`` defaults to ``residual`` (updated in place); ``y`` defaults to
    a new tensor.  Returns ``(y, residual_out)``."""
    hidden = x.shape[-1]
    if y is None:
        y = torch.empty_like(x)
    if residual_out is None:
        residual_out = residual
    _check_tensors((("x", x), ("residual", residual), ("gamma", gamma), ("y", y),
                    ("residual_out", residual_out)))
    if (residual.shape != x.shape or y.shape != x.shape or residual_out.shape != x.shape
            or gamma.shape != (hidden,)):
        raise ValueError("shape mismatch")
    code = _dtype_code(x, residual, gamma, y, residual_out)
    rows = x.numel() // hidden if hidden else 0
    with torch.cuda.device(x.device):
        _check(lib().arops_add_rmsnorm(x.data_ptr(), residual.data_ptr(), residual_out.data_ptr(),
                                       gamma.data_ptr(), y.data_ptr(), rows, hidden, float(eps),
                                       code, _stream(x)))
    return y, residual_out


def layernorm(x: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor, eps: float = 1e-6,
              out: torch.Tensor | None = None) -> torch.Tensor:
    """y = gamma * (x - mean) / sqrt(var + eps) + beta over the last dimension."""
    hidden = x.shape[-1]
    if out is None:
        out = torch.empty_like(x)
    _check_tensors((("x", x), ("gamma", gamma), ("beta", beta), ("out", out)))
    if gamma.shape != (hidden,) or beta.shape != (hidden,) or out.shape != x.shape:
        raise ValueError("shape mismatch")
    code = _dtype_code(x, gamma, beta, out)
    rows = x.numel() // hidden if hidden else 0
    with torch.cuda.device(x.device):
        _check(lib().arops_layernorm(x.data_ptr(), gamma.data_ptr(), beta.data_ptr(),
                                     out.data_ptr(), rows, hidden, float(eps), code, _stream(x)))
    return out


def add_layernorm(x: torch.Tensor, residual: torch.Tensor, gamma: torch.Tensor,
                  beta: torch.Tensor, eps: float = 1e-6, y: torch.Tensor | None = None,
                  residual_out: torch.Tensor | None = None):
    """residual_out = x + residual (rounded); y = LayerNorm(residual_out).
    ``residual_out`` defaults to ``residual`` (in place).  Returns ``(y, residual_out)``."""
    hidden = x.shape[-1]
    if y is None:
        y = torch.empty_like(x)
    if residual_out is None:
        residual_out = residual
    _check_tensors((("x", x), ("residual", residual), ("gamma", gamma), ("beta", beta), ("y", y),
                    ("residual_out", residual_out)))
    if (residual.shape != x.shape or y.shape != x.shape or residual_out.shape != x.shape
            or gamma.shape != (hidden,) or beta.shape != (hidden,)):
        raise ValueError("shape mismatch")
    code = _dtype_code(x, residual, gamma, beta, y, residual_out)
    rows = x.numel() // hidden if hidden else 0
    with torch.cuda.device(x.device):
        _check(lib().arops_add_layernorm(x.data_ptr(), residual.data_ptr(),
                                         residual_out.data_ptr(), gamma.data_ptr(),
                                         beta.data_ptr(), y.data_ptr(), rows, hidden, float(eps),
                                         code, _stream(x)))
    return y, residual_out


def mrope_qk(q: torch.Tensor, k: torch.Tensor, pos: torch.Tensor, sections=(24, 20, 20),
             theta: float = 1e6, q_out: torch.Tensor | None = None,
             k_out: torch.Tensor | None = None):
    """Multi-section rotary embedding of q [T, Hq, D] and k [T, Hk, D] with int32
    position ids pos [3, T] (rows t, h, w).  Outputs default to the inputs
    (rotation in place).  Returns ``(q_out, k_out)``."""
    if q_out is None:
        q_out = q
    if k_out is None:
        k_out = k
    _check_tensors((("q", q), ("k", k), ("pos", pos), ("q_out", q_out), ("k_out", k_out)))
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q and k must be [tokens, heads, head_dim]")
    tokens, hq, d = q.shape
    if k.shape[0] != tokens or k.shape[2] != d or q_out.shape != q.shape or k_out.shape != k.shape:
        raise ValueError("shape mismatch")
    if pos.dtype != torch.int32 or tuple(pos.shape) != (3, tokens):
        raise ValueError("pos must be int32 [3, tokens]")
    code = _dtype_code(q, k, q_out, k_out)
    sec = (_i32 * 3)(*[int(s) for s in sections])
    with torch.cuda.device(q.device):
        _check(lib().arops_mrope_qk(q.data_ptr(), k.data_ptr(), q_out.data_ptr(), k_out.data_ptr(),
                                    pos.data_ptr(), tokens, hq, k.shape[1], d, sec, float(theta),
                                    code, _stream(q)))
    return q_out, k_out


def mrope_kv_append(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor,
                    cache_loc: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                    sections=(24, 20, 20), theta: float = 1e6,
                    q_out: torch.Tensor | None = None) -> torch.Tensor:
    """Rotate q (into ``q_out``, default in place) and k with M-RoPE and write
    the rotated k and the unrotated v of token t into slot
    (cache_loc[0, t], cache_loc[1, t]) of k_cache / v_cache
    [cache_rows, n_kv_heads, max_seq, head_dim].  Returns ``q_out``."""
    if q_out is None:
        q_out = q
    _check_tensors((("q", q), ("k", k), ("v", v), ("pos", pos), ("cache_loc", cache_loc),
                    ("k_cache", k_cache), ("v_cache", v_cache), ("q_out", q_out)))
    tokens, hq, d = q.shape
    hk = k.shape[1]
    if (k.shape != (tokens, hk, d) or v.shape != k.shape or q_out.shape != q.shape
            or k_cache.dim() != 4 or k_cache.shape[1] != hk or k_cache.shape[3] != d
            or v_cache.shape != k_cache.shape):
        raise ValueError("shape mismatch")
    if pos.dtype != torch.int32 or tuple(pos.shape) != (3, tokens):
        raise ValueError("pos must be int32 [3, tokens]")
    if cache_loc.dtype != torch.int32 or tuple(cache_loc.shape) != (2, tokens):
        raise ValueError("cache_loc must be int32 [2, tokens]")
    code = _dtype_code(q, k, v, q_out, k_cache, v_cache)
    sec = (_i32 * 3)(*[int(s) for s in sections])
    with torch.cuda.device(q.device):
        _check(lib().arops_mrope_kv_append(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), q_out.data_ptr(), k_cache.data_ptr(),
            v_cache.data_ptr(), pos.data_ptr(), cache_loc.data_ptr(), tokens, hq, hk, d,
            k_cache.shape[0], k_cache.shape[2], sec, float(theta), code, _stream(q)))
    return q_out


def swiglu(gate: torch.Tensor, up: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """out = silu(gate) * up (fp32 math); ``out`` may be ``gate`` or ``up``."""
    if out is None:
        out = torch.empty_like(gate)
    _check_tensors((("gate", gate), ("up", up), ("out", out)))
    if up.shape != gate.shape or out.shape != gate.shape:
        raise ValueError("shape mismatch")
    code = _dtype_code(gate, up, out)
    inter = gate.shape[-1] if gate.dim() else 1
    rows = gate.numel() // inter if inter else 0
    with torch.cuda.device(gate.device):
        _check(lib().arops_swiglu(gate.data_ptr(), up.data_ptr(), out.data_ptr(), rows, inter,
                                  code, _stream(gate)))
    return out


def topk_sample_workspace(rows: int, vocab: int, top_k: int) -> int:
    """Bytes of device workspace that topk_sample needs for this shape."""
    n = ctypes.c_size_t(0)
    _check(lib().arops_topk_sample_workspace(rows, vocab, top_k, ctypes.byref(n)))
    return int(n.value)


def topk_sample_prepare(workspace: torch.Tensor) -> torch.Tensor:
    """Clears the arrival counters of a new sampling workspace (a uint8 device
    tensor) on the current stream; needed once, before its first use."""
    _check_tensors((("workspace", workspace),))
    with torch.cuda.device(workspace.device):
        _check(lib().arops_topk_sample_prepare(workspace.data_ptr(),
                                               workspace.numel() * workspace.element_size(),
                                               _stream(workspace)))
    return workspace


def topk_sample(logits: torch.Tensor, gumbel: torch.Tensor, top_k: int, temperature: float = 1.0,
                workspace: torch.Tensor | None = None, token_out: torch.Tensor | None = None,
                prob_out: torch.Tensor | None = None):
    """Gumbel-max sample from softmax(logits / temperature) restricted to the
    top_k logits of each row.  logits [rows, vocab] (bf16/f32); gumbel
    [rows, top_k] float32 Gumbel(0,1) draws, draw j for the j-th largest logit.
    Returns (token int32 [rows], probability float32 [rows]).  ``workspace`` is
    a uint8 device tensor of at least topk_sample_workspace() bytes whose
    counters were cleared once (topk_sample_prepare); allocated and cleared
    here if omitted."""
    if logits.dim() != 2:
        raise ValueError("logits must be [rows, vocab]")
    rows, vocab = logits.shape
    if token_out is None:
        token_out = torch.empty(rows, dtype=torch.int32, device=logits.device)
    if prob_out is None:
        prob_out = torch.empty(rows, dtype=torch.float32, device=logits.device)
    need = topk_sample_workspace(rows, vocab, top_k) if rows else 0
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=logits.device)
        if rows:
            topk_sample_prepare(workspace)
    _check_tensors((("logits", logits), ("gumbel", gumbel), ("token_out", token_out),
                    ("prob_out", prob_out), ("workspace", workspace)))
    if gumbel.dtype != torch.float32 or tuple(gumbel.shape) != (rows, top_k):
        raise ValueError("gumbel must be float32 [rows, top_k]")
    if token_out.dtype != torch.int32 or prob_out.dtype != torch.float32:
        raise ValueError("token_out must be int32 and prob_out float32")
    code = _dtype_code(logits)
    with torch.cuda.device(logits.device):
        _check(lib().arops_topk_sample(logits.data_ptr(), gumbel.data_ptr(), token_out.data_ptr(),
                                       prob_out.data_ptr(), rows, vocab, int(top_k),
                                       float(temperature), code, workspace.data_ptr(),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(logits)))
    return token_out, prob_out


def set_pdl(enable: bool) -> bool:
    """Turn programmatic dependent launch on or off; returns the old setting."""
    return bool(lib().arops_set_pdl(1 if enable else 0))


def set_streaming(enable: bool) -> bool:
    """Choose the shared-memory streaming kernels or the register kernels (the
    default); returns the old setting.  Both give results within tolerance."""
    return bool(lib().arops_set_streaming(1 if enable else 0))


def set_topk_cluster(mode) -> int:
    """Which kernels top-k sampling may take: 0 (or False) the slice kernel
    only; 1 (or True, the default) the cluster kernels, registers for calls
    whose rows' 16-CTA clusters are all resident at once and shared memory for
    the rest; 2 the shared-memory cluster kernel for every call; 3 the
    streaming kernel (one CTA a row) for 16-byte-aligned rows.  Returns the
    old mode.  Every kernel gives identical results."""
    return int(lib().arops_set_topk_cluster(int(mode)))


def device_errors(clear: bool = True) -> int:
    """Device-side error bits (1: a bulk-copy wait timed out; 2: a KV-cache slot
    out of range was skipped; 4: a sampling workspace's counters were not
    cleared); synchronises the device."""
    v = ctypes.c_uint32(0)
    _check(lib().arops_device_errors(ctypes.byref(v), 1 if clear else 0))
    return int(v.value)


def launch_count() -> int:
    """Kernels launched by libarops in this process so far."""
    return int(lib().arops_launch_count())
