"""Guarded buffers: a tensor placed inside a larger byte buffer whose head and tail hold a fixed
byte pattern, so that a write beyond either end of the tensor shows up afterwards.

Test helper only (the library never sees the guards: it gets the inner tensor's pointer).
"""
from __future__ import annotations

import math

import torch

GUARD_BYTES = 4096          # keeps the inner tensor 4096-byte aligned within the buffer
PATTERN = 0xA5


class Guarded:
    def __init__(self, shape, dtype, device, init=None):
        esz = torch.empty((), dtype=dtype).element_size()
        self.nbytes = math.prod(shape) * esz
        self.buf = torch.full((self.nbytes + 2 * GUARD_BYTES,), PATTERN, dtype=torch.uint8, device=device)
        inner = self.buf[GUARD_BYTES:GUARD_BYTES + self.nbytes]
        self.tensor = inner.view(dtype).view(shape) if self.nbytes else torch.empty(shape, dtype=dtype, device=device)
        if init is not None:
            self.tensor.copy_(init)

    def intact(self) -> bool:
        head = self.buf[:GUARD_BYTES]
        tail = self.buf[GUARD_BYTES + self.nbytes:]
        return bool((head == PATTERN).all().item()) and bool((tail == PATTERN).all().item())


def guarded_like(t: torch.Tensor, device=None) -> Guarded:
    return Guarded(tuple(t.shape), t.dtype, device or t.device, init=t)
