"""Seeded synthetic inputs for the residual-compression codec.

This module is shared by the CPU oracle's tests and the CUDA path's tests and
benchmark. It holds no codec arithmetic: only the input recipe, i.e. the shapes
of the workloads and the value distributions of the activations that the codec
consumes. It stands in for real FLUX.1-dev / CogVideoX-2b activations, which
need model weights and prompt sets that are not available here.

Recipe (per communicated tensor, called a slot):

* per-channel scale ``s_c = exp(0.5 * N(0,1))`` (LogNormal(0, 0.5));
* a seeded fraction of "outlier" channels gets ``s_c * outlier_gain``;
* ``X_0 = N(0,1) * s_c`` (token-major, channels contiguous);
* ``X_t = X_{t-1} + delta_t * g_t * (N_t * s_c)`` where ``g_t = 1`` for an
  absolute drift and ``g_t = ||X_{t-1}|| / ||N_t * s_c||`` for a drift stated
  as a relative L2 change per step;
* the running state is kept in fp32 and every emitted ``X_t`` is rounded to
  bf16.

Every random draw comes from a torch ``Generator`` seeded by a splitmix64 mix
of ``(seed, slot, step, purpose)``; CUDA generators use torch's counter-based
Philox, so device-side generation is reproducible for a fixed seed.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

_M64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """One step of the splitmix64 mixer (Steele, Lea, Flood 2014)."""
    z = (x + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def mix_seed(*vals: int) -> int:
    """Fold a tuple of integers into one 63-bit generator seed."""
    h = 0x243F6A8885A308D3
    for v in vals:
        h = splitmix64(h ^ (int(v) & _M64))
    return h & ((1 << 63) - 1)


def generator(device, *stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(mix_seed(*stream))
    return g


# Purpose tags keep the streams of one slot independent.
_TAG_SCALE, _TAG_OUTLIER, _TAG_X0, _TAG_DRIFT, _TAG_Q0, _TAG_LR = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution of one synthetic codec workload."""

    name: str
    slots: int
    rows: int
    cols: int
    steps: int           # including the uncompressed warmup step 0
    bits: int
    group: int
    drift: str           # "abs" or "rel"
    delta0: float        # drift at step 1
    delta1: float        # drift at the last step (linear ramp)
    outlier_frac: float = 0.0
    outlier_gain: float = 20.0
    mode: int = 0        # 0 = quantised, 1 = low-rank
    rank: int = 16
    iters: int = 2

    @property
    def elems_per_slot(self) -> int:
        return self.rows * self.cols

    @property
    def elems(self) -> int:
        return self.slots * self.rows * self.cols

    def delta(self, t: int) -> float:
        if t <= 1 or self.steps <= 2:
            return self.delta0
        f = (t - 1) / (self.steps - 2)
        return self.delta0 + f * (self.delta1 - self.delta0)

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny parity case, a FLUX.1-dev-shaped patch-parallel
# shard (4608 tokens / 4 devices), a CogVideoX-2b-shaped shard (17776 / 4), the
# low-rank mode (A given directly) and a 1-bit stress case over K and V.
TINY = Workload("tiny", 1, 256, 512, 4, 2, 128, "abs", 0.1, 0.1)
FLUX = Workload("flux", 57, 1152, 3072, 28, 2, 128, "rel", 0.05, 0.2, outlier_frac=0.01)
COGVIDEOX = Workload("cogvideox", 30, 4444, 1920, 50, 4, 64, "rel", 0.1, 0.1)
STRESS = Workload("stress", 60, 17776, 1920, 50, 1, 128, "rel", 0.1, 0.1)
LOWRANK = Workload("lowrank", 57, 4608, 3072, 1, 0, 0, "abs", 0.0, 0.0, mode=1, rank=16, iters=2)

WORKLOADS = {w.name: w for w in (TINY, FLUX, COGVIDEOX, STRESS, LOWRANK)}


def channel_scales(w: Workload, slot: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """Per-channel scales s_c (fp32, [cols]) of one slot."""
    g = generator(device, seed, slot, _TAG_SCALE)
    s = torch.exp(0.5 * torch.randn(w.cols, generator=g, device=device, dtype=torch.float32))
    n_out = int(round(w.outlier_frac * w.cols))
    if n_out > 0:
        go = generator("cpu", seed, slot, _TAG_OUTLIER)
        idx = torch.randperm(w.cols, generator=go)[:n_out].to(device)
        s[idx] *= w.outlier_gain
    return s


class SlotStream:
    """Step-by-step activations X_t of one slot (bf16, [rows, cols])."""

    def __init__(self, w: Workload, slot: int, seed: int = 0, device="cpu", rows: Optional[int] = None):
        self.w, self.slot, self.seed, self.device = w, slot, seed, device
        self.rows = w.rows if rows is None else rows
        self.s = channel_scales(w, slot, seed, device)
        self.t = -1
        self.state: Optional[torch.Tensor] = None

    def _noise(self, tag: int, t: int) -> torch.Tensor:
        g = generator(self.device, self.seed, self.slot, t, tag)
        return torch.randn(self.rows, self.w.cols, generator=g, device=self.device, dtype=torch.float32) * self.s

    def next(self) -> torch.Tensor:
        self.t += 1
        t = self.t
        if t == 0:
            self.state = self._noise(_TAG_X0, 0)
        else:
            n = self._noise(_TAG_DRIFT, t)
            d = self.w.delta(t)
            if self.w.drift == "rel":
                gain = (torch.linalg.vector_norm(self.state) / torch.linalg.vector_norm(n)).item()
            else:
                gain = 1.0
            self.state.add_(n, alpha=d * gain)
        return self.state.to(torch.bfloat16)


def activations(w: Workload, slot: int, steps: int, seed: int = 0, device="cpu", rows: Optional[int] = None) -> List[torch.Tensor]:
    """The first ``steps`` activations of one slot."""
    st = SlotStream(w, slot, seed, device, rows)
    return [st.next() for _ in range(steps)]


def gaussian(shape, seed: int, *stream: int, device="cpu", dtype=torch.float32) -> torch.Tensor:
    """i.i.d. N(0,1) draws on a named stream (e.g. the subspace-iteration start)."""
    g = generator(device, seed, *stream)
    return torch.randn(*shape, generator=g, device=device, dtype=dtype)


def q0(n: int, r: int, seed: int, mat: int, call: int = 0, device="cpu") -> torch.Tensor:
    """Gaussian start block Q_0 (fp32, [n, r]) of the subspace iteration."""
    return gaussian((n, r), seed, mat, call, _TAG_Q0, device=device)


def lowrank_matrix(m: int, n: int, r: int, mat: int, seed: int = 0, noise: float = 0.01, device="cpu") -> torch.Tensor:
    """Residual matrix of the low-rank workload: rank-r signal plus noise.

    ``A = U diag(1/k) V^T + noise * N(0,1)`` with unnormalised Gaussian U (m x r)
    and V (n x r), k = 1..r, as fp32 [m, n] row-major.
    """
    g = generator(device, seed, mat, _TAG_LR)
    U = torch.randn(m, r, generator=g, device=device, dtype=torch.float32)
    V = torch.randn(n, r, generator=g, device=device, dtype=torch.float32)
    sv = 1.0 / torch.arange(1, r + 1, device=device, dtype=torch.float32)
    A = (U * sv) @ V.T
    if noise:
        A.add_(torch.randn(m, n, generator=g, device=device, dtype=torch.float32), alpha=noise)
    return A.contiguous()


def bf16_bits(x: torch.Tensor) -> torch.Tensor:
    """Raw bf16 bit patterns as int16 (a view; for handing data to C code)."""
    assert x.dtype == torch.bfloat16
    return x.view(torch.int16)


__all__ = [
    "Workload", "WORKLOADS", "TINY", "FLUX", "COGVIDEOX", "STRESS", "LOWRANK",
    "channel_scales", "SlotStream", "activations", "gaussian", "q0", "lowrank_matrix",
    "splitmix64", "mix_seed", "generator", "bf16_bits",
]
