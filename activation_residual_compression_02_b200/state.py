"""Device buffers of a quantised-codec run (torch allocations; plumbing only)."""
from __future__ import annotations

from typing import List, Sequence

import torch

from ._cf import Slot


class QuantState:
    """Sender state (base, err), receiver state (cache) and payload of each slot."""

    def __init__(self, shapes: Sequence[Sequence[int]], bits: int, group: int, device="cuda"):
        self.shapes = [tuple(s) for s in shapes]
        self.base: List[torch.Tensor] = []
        self.err: List[torch.Tensor] = []
        self.cache: List[torch.Tensor] = []
        self.codes: List[torch.Tensor] = []
        self.scales: List[torch.Tensor] = []
        for rows, cols in self.shapes:
            n = rows * cols
            self.base.append(torch.empty(n, dtype=torch.bfloat16, device=device))
            self.err.append(torch.empty(n, dtype=torch.float32, device=device))
            self.cache.append(torch.empty(n, dtype=torch.float32, device=device))
            self.codes.append(torch.empty(n * bits // 8, dtype=torch.uint8, device=device))
            self.scales.append(torch.empty(n // group, dtype=torch.float32, device=device))

    def slots(self, xs: Sequence[torch.Tensor]) -> List[Slot]:
        return [Slot(x=x.reshape(-1), base=b, err=e, cache=c, codes=k, scales=s)
                for x, b, e, c, k, s in zip(xs, self.base, self.err, self.cache, self.codes, self.scales)]


def alloc_quant_state(shapes, bits, group, device="cuda") -> QuantState:
    return QuantState(shapes, bits, group, device)
