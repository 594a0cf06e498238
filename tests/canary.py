"""Poisoned canaries around the buffers a library call writes.

`Guarded(shape, dtype, device)` allocates the tensor inside a larger byte
buffer: GUARD bytes before and after it, and the tensor itself, are filled
with a NaN pattern (fp32 0x7FC0DEAD for 4-byte elements, bf16 0x7FC1 for
2-byte ones; as int32 0x7FC0DEAD is just an unlikely value).  After a call,
`intact()` says whether both guard bands still hold the pattern bit for bit,
and `untouched()` counts the tensor's elements that still hold it, so a call
that must write every element can be checked to have done so.
"""
from __future__ import annotations

import torch

GUARD = 4096  # bytes on each side (keeps the tensor 256-byte aligned)
_PAT = {4: (torch.int32, 0x7FC0DEAD), 2: (torch.int16, 0x7FC1), 1: (torch.uint8, 0xA5)}


class Guarded:
    def __init__(self, shape, dtype, device, guard: int = GUARD):
        self.shape, self.dtype = tuple(shape), dtype
        es = torch.empty((), dtype=dtype).element_size()
        n = 1
        for x in self.shape:
            n *= x
        self.nbytes = n * es
        self.guard = guard
        total = guard + self.nbytes + guard
        itype, pat = _PAT[es]
        if total % es:
            raise ValueError("guard must be a multiple of the element size")
        self.buf = torch.empty(total // es, dtype=itype, device=device)
        self.buf.fill_(pat)
        self.pattern = self.buf[:1].clone()
        raw = self.buf.view(torch.uint8)
        self.t = raw[guard:guard + self.nbytes].view(dtype).view(self.shape)
        self._raw, self._itype = raw, itype

    def intact(self) -> bool:
        """Both guard bands still hold the pattern."""
        lo = self._raw[:self.guard].view(self._itype)
        hi = self._raw[self.guard + self.nbytes:].view(self._itype)
        p = self.pattern.to(lo.device)
        return bool((lo == p).all().item()) and bool((hi == p).all().item())

    def untouched(self) -> int:
        """Elements of the tensor that still hold the pattern."""
        body = self._raw[self.guard:self.guard + self.nbytes].view(self._itype)
        return int((body == self.pattern.to(body.device)).sum().item())


class GuardedWorkspace(Guarded):
    """A caller workspace of exactly `nbytes` (the size the library asked
    for) between two guard bands."""

    def __init__(self, nbytes: int, device, guard: int = GUARD):
        nbytes = max(1, int(nbytes))
        super().__init__((nbytes,), torch.uint8, device, guard)
