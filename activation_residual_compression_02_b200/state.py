"""Device buffers of a quantised-codec run, and host-streaming orchestration.

Plumbing only: torch allocations, CUDA streams and events.  Every step of the
codec itself runs in libcf's kernels.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from ._cf import Context, Slot


def _split(buf: torch.Tensor, sizes: Sequence[int]) -> List[torch.Tensor]:
    out, off = [], 0
    for n in sizes:
        out.append(buf[off:off + n])
        off += n
    return out


def _aligned_sizes(sizes: Sequence[int], elem: int) -> List[int]:
    """Round each slot's element count up so every view starts 16-byte aligned."""
    q = max(1, 16 // elem)
    return [(n + q - 1) // q * q for n in sizes]


class QuantState:
    """Sender state (base, err), receiver state (cache) and payload of each slot.

    Each array family is one contiguous allocation with per-slot views, so the
    payload of a step can leave the device in one copy.  ``lean=True`` holds
    err and cache in bf16 (the context's state_bf16 option).
    """

    def __init__(self, shapes: Sequence[Sequence[int]], bits: int, group: int, device="cuda", lean: bool = False,
                 recon: bool = False):
        self.shapes = [tuple(s) for s in shapes]
        self.bits, self.group, self.lean = bits, group, lean
        n = [r * c for r, c in self.shapes]
        self.elems = n
        nb = _aligned_sizes(n, 2)
        sdt = torch.bfloat16 if lean else torch.float32
        nf = _aligned_sizes(n, 2 if lean else 4)
        self.base_all = torch.empty(sum(nb), dtype=torch.bfloat16, device=device)
        self.err_all = torch.empty(sum(nf), dtype=sdt, device=device)
        self.cache_all = torch.empty(sum(nf), dtype=sdt, device=device)
        self.base = [v[:k] for v, k in zip(_split(self.base_all, nb), n)]
        self.err = [v[:k] for v, k in zip(_split(self.err_all, nf), n)]
        self.cache = [v[:k] for v, k in zip(_split(self.cache_all, nf), n)]
        # optional bf16 copy of each cache, written by the receiver calls
        self.recon_all = torch.empty(sum(nb), dtype=torch.bfloat16, device=device) if recon else None
        self.recon = [v[:k] for v, k in zip(_split(self.recon_all, nb), n)] if recon else [None] * len(n)
        self.codes_all, self.codes, self.scales_all, self.scales = self.payload_buffers(device)

    def payload_buffers(self, device="cuda", pin: bool = False):
        """A contiguous (codes, scales) pair with per-slot views."""
        nc = [k * self.bits // 8 for k in self.elems]
        ns = [k // self.group for k in self.elems]
        ncb, nsb = _aligned_sizes(nc, 1), _aligned_sizes(ns, 4)
        kw = dict(pin_memory=True) if pin else dict(device=device)
        codes_all = torch.empty(sum(ncb), dtype=torch.uint8, **kw)
        scales_all = torch.empty(sum(nsb), dtype=torch.float32, **kw)
        codes = [v[:k] for v, k in zip(_split(codes_all, ncb), nc)]
        scales = [v[:k] for v, k in zip(_split(scales_all, nsb), ns)]
        return codes_all, codes, scales_all, scales

    def activation_buffer(self, device="cuda", pin: bool = False):
        """A contiguous bf16 buffer for one step's activations of every slot, with per-slot views."""
        nb = _aligned_sizes(self.elems, 2)
        kw = dict(pin_memory=True) if pin else dict(device=device)
        buf = torch.empty(sum(nb), dtype=torch.bfloat16, **kw)
        return buf, [v[:k] for v, k in zip(_split(buf, nb), self.elems)]

    def slots(self, xs: Sequence[torch.Tensor], codes: Optional[Sequence[torch.Tensor]] = None,
              scales: Optional[Sequence[torch.Tensor]] = None) -> List[Slot]:
        codes = self.codes if codes is None else codes
        scales = self.scales if scales is None else scales
        return [Slot(x=x.reshape(-1), base=b, err=e, cache=c, codes=k, scales=s, recon=rc)
                for x, b, e, c, k, s, rc in zip(xs, self.base, self.err, self.cache, codes, scales, self.recon)]


def alloc_quant_state(shapes, bits, group, device="cuda") -> QuantState:
    return QuantState(shapes, bits, group, device)


class HostStreamCodec:
    """The quantised codec fed from host memory, with copies overlapped.

    Activations arrive in pinned host buffers and the payload (codes and
    scales) goes back to pinned host buffers, as when the codec sits between
    a host-side producer and a network.  Three CUDA streams run the
    host-to-device copy of step t+1, the codec of step t and the device-to-
    host copy of step t-1 at the same time; the device keeps `depth` input and
    payload buffers in rotation, and events order the reuse of each.
    """

    def __init__(self, shapes, bits: int = 2, group: int = 128, sign_scale: int = 0, depth: int = 2,
                 device="cuda"):
        self.ctx = Context(shapes, bits=bits, group=group, sign_scale=sign_scale)
        self.st = QuantState(shapes, bits, group, device)
        self.depth = depth
        self.x_dev = [self.st.activation_buffer(device) for _ in range(depth)]
        self.pay_dev = [self.st.payload_buffers(device) for _ in range(depth)]
        self.s_h2d = torch.cuda.Stream(device)
        self.s_codec = torch.cuda.Stream(device)
        self.s_d2h = torch.cuda.Stream(device)
        self.ev_in = [torch.cuda.Event() for _ in range(depth)]      # input landed
        self.ev_done = [torch.cuda.Event() for _ in range(depth)]    # codec finished with the input / payload
        self.ev_out = [torch.cuda.Event() for _ in range(depth)]     # payload left the device
        self.n = 0
        self.slot_arrays = [self.ctx._slots(self.st.slots(self.x_dev[i][1], self.pay_dev[i][1], self.pay_dev[i][3]))
                            for i in range(depth)]

    def step(self, t: int, x_host: torch.Tensor, codes_host: Optional[torch.Tensor] = None,
             scales_host: Optional[torch.Tensor] = None) -> None:
        """Enqueue step t: x_host is a pinned buffer from ``activation_buffer(pin=True)``;
        codes_host / scales_host are pinned buffers from ``payload_buffers(pin=True)``
        (ignored at the warmup step 0)."""
        from . import _cf

        i = self.n % self.depth
        xd = self.x_dev[i][0]
        with torch.cuda.stream(self.s_h2d):
            if self.n >= self.depth:
                self.s_h2d.wait_event(self.ev_done[i])
            xd.copy_(x_host, non_blocking=True)
            self.ev_in[i].record(self.s_h2d)
        self.s_codec.wait_event(self.ev_in[i])
        if self.n >= self.depth:
            self.s_codec.wait_event(self.ev_out[i])
        L = _cf.lib()
        h, arr, sh = self.ctx.handle, self.slot_arrays[i], self.s_codec.cuda_stream
        for fn in (L.cf_compress, L.cf_decompress):
            st = fn(h, arr, t, sh)
            if st != _cf.CF_OK:
                raise _cf.CfError(st, L.cf_last_error(h).decode())
        self.ev_done[i].record(self.s_codec)
        with torch.cuda.stream(self.s_d2h):
            self.s_d2h.wait_event(self.ev_done[i])
            if t > 0 and codes_host is not None:
                codes_host.copy_(self.pay_dev[i][0], non_blocking=True)
                scales_host.copy_(self.pay_dev[i][2], non_blocking=True)
            self.ev_out[i].record(self.s_d2h)
        self.n += 1

    def synchronize(self):
        for s in (self.s_h2d, self.s_codec, self.s_d2h):
            s.synchronize()

    def check(self) -> int:
        self.synchronize()
        return self.ctx.check(self.s_codec)
