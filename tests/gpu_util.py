"""Helpers for the GPU tests: device copies, guarded and misaligned buffers."""
from __future__ import annotations

import torch

GUARD = 4096  # elements of canary on each side of a guarded buffer
_CANARY_BITS = {torch.bfloat16: 0x7FA5, torch.float32: 0x7FC0_5A5A}


def dev(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda").contiguous()


class Guarded:
    """A device tensor with canary regions before and after it; ``check()``
    asserts that a kernel wrote nothing outside the tensor."""

    def __init__(self, shape, dtype, fill: torch.Tensor | None = None, offset: int = 0):
        n = 1
        for s in shape:
            n *= s
        self.n = n
        self.offset = offset  # extra elements of misalignment
        itype = torch.int16 if dtype == torch.bfloat16 else torch.int32
        self.buf = torch.empty(n + 2 * GUARD + offset, dtype=dtype, device="cuda")
        self.buf.view(itype).fill_(_CANARY_BITS[dtype] if dtype == torch.float32 else
                                   _CANARY_BITS[dtype])
        self.itype = itype
        self.t = self.buf[GUARD + offset: GUARD + offset + n].view(*shape)
        if fill is not None:
            self.t.copy_(fill)
        self._canary = _CANARY_BITS[dtype]

    def check(self) -> None:
        raw = self.buf.view(self.itype)
        head = raw[: GUARD + self.offset]
        tail = raw[GUARD + self.offset + self.n:]
        c = torch.tensor(self._canary, dtype=self.itype, device="cuda")
        assert bool((head == c).all()), "write before the buffer"
        assert bool((tail == c).all()), "write after the buffer"


def misaligned(t: torch.Tensor, by: int = 1) -> torch.Tensor:
    """A contiguous device copy of ``t`` whose data pointer is ``by`` elements
    past a 16-byte boundary."""
    buf = torch.empty(t.numel() + 16, dtype=t.dtype, device="cuda")
    out = buf[by: by + t.numel()].view(t.shape)
    out.copy_(t)
    assert out.data_ptr() % 16 != 0
    return out


def resident_threads() -> int:
    """Threads the device holds at once (2048 per SM).  The launchers treat a
    problem of at most one vector (norm, SwiGLU) or one head pass (M-RoPE) per
    resident thread or warp as latency-bound and lay it out differently; tests
    size cases on both sides of that line."""
    return torch.cuda.get_device_properties(0).multi_processor_count * 2048
