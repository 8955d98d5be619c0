"""Canary guard regions around the buffers a call writes.

Stands in for a memory checker that cannot run on the GPUs used here: an
output (or workspace) is placed inside a larger device buffer whose every
other byte holds a known byte, optionally with padding rows after each
leading index (between the layers of a batched output) as well as a guard
before and after the whole. After the call, ``intact()`` says whether any
byte outside the tensor changed, and ``written()`` whether every element of
the tensor was overwritten (no element still holds the canary pattern: for
types of four and two bytes, 0x5A5A... is about 1.5e16, a value no output
of these calls takes).
"""
import math

import torch

CANARY = 0x5A
GUARD_BYTES = 256          # keeps the tensor 256-byte aligned (workspace rule)


class Guarded:
    """A tensor of ``shape`` and ``dtype`` whose storage is padded with
    ``pad`` extra rows along dim -2 (for a 1-D shape: ``pad`` extra elements)
    and surrounded by ``GUARD_BYTES`` canary bytes on both sides."""

    def __init__(self, shape, dtype, pad=0, device="cuda"):
        shape = tuple(int(s) for s in shape)
        esize = torch.empty(0, dtype=dtype).element_size()
        if len(shape) == 1:
            padded = (shape[0] + pad,)
        else:
            padded = shape[:-2] + (shape[-2] + pad, shape[-1])
        self.n = math.prod(padded) * esize
        self.buf = torch.full((GUARD_BYTES + self.n + GUARD_BYTES,), CANARY, dtype=torch.uint8,
                              device=device)
        self.store = self.buf[GUARD_BYTES:GUARD_BYTES + self.n].view(dtype).view(padded)
        if len(shape) == 1:
            self.t = self.store[:shape[0]]
        else:
            self.t = self.store[..., :shape[-2], :]
        self.shape, self.pad, self.esize = shape, pad, esize

    def intact(self) -> bool:
        """No byte outside the tensor has changed."""
        b = self.buf
        if not bool((b[:GUARD_BYTES] == CANARY).all()) or \
                not bool((b[GUARD_BYTES + self.n:] == CANARY).all()):
            return False
        if self.pad == 0:
            return True
        raw = self.buf[GUARD_BYTES:GUARD_BYTES + self.n]
        if len(self.shape) == 1:
            return bool((raw[self.shape[0] * self.esize:] == CANARY).all())
        rows = raw.view(self.store.shape[:-1] + (self.store.shape[-1] * self.esize,))
        return bool((rows[..., self.shape[-2]:, :] == CANARY).all())

    def written(self) -> bool:
        """Every element of the tensor differs from the canary pattern."""
        if self.t.numel() == 0:
            return True
        raw = self.t.contiguous().view(torch.uint8).reshape(-1, self.esize)
        return not bool((raw == CANARY).all(dim=1).any())
