"""Algorithm 1's all-gather of K and V, moving compressed payloads.

"Accelerating Parallel Diffusion Model Serving with Residual Compression"
(arXiv 2507.17511), Algorithm 1 (patch parallelism): each device projects Q,
K and V for its own patch of tokens, all-gathers K and V, and attends over
the whole sequence.  With residual compression the all-gather carries each
device's payload (codes and group scales of its K/V shards) instead of the
bf16 tensors; every device then decompresses each peer's payload into the
receiver cache it keeps for that peer's shards.  The warmup step sends the
activation itself (reproducibility table, "Dataset Splits" row).

Plumbing only: the codec runs in libcf's kernels and the collective is
torch.distributed (NCCL between GPUs).  Slots are split into buckets so that
the all-gather of bucket b overlaps the compression of bucket b + 1 and the
decompression of bucket b - 1: the collective of a bucket is issued
asynchronously right after its compression is enqueued, and the receiver
waits on it only when it needs that bucket.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from ._cf import CF_OK, CfError, Context, Slot, lib
from .state import QuantState


def _up16(n: int) -> int:
    return (n + 15) // 16 * 16


def payload_layout(shapes: Sequence[Sequence[int]], bits: int, group: int) -> Tuple[List[Tuple[int, int, int, int]], int]:
    """Byte layout of one device's payload for the given slots, in one buffer.

    Slot i's codes (rows*cols*bits/8 bytes) and its fp32 scales (rows*cols/group
    values) each start on a 16-byte boundary.  Returns ([(codes_offset,
    codes_bytes, scales_offset, scales_count)] per slot, total bytes).
    """
    out, off = [], 0
    for r, c in shapes:
        n = int(r) * int(c)
        if c % group or n * bits % 8:
            raise ValueError("cols must be a multiple of the group size")
        cb, ns = n * bits // 8, n // group
        co = off
        off = _up16(off + cb)
        so = off
        off = _up16(off + 4 * ns)
        out.append((co, cb, so, ns))
    return out, max(off, 16)


class PayloadBuffer:
    """One device's payload for a set of slots: a flat uint8 tensor with per-slot views."""

    def __init__(self, shapes, bits: int, group: int, device="cuda", data: Optional[torch.Tensor] = None):
        self.layout, self.nbytes = payload_layout(shapes, bits, group)
        self.data = torch.zeros(self.nbytes, dtype=torch.uint8, device=device) if data is None else data
        assert self.data.numel() == self.nbytes and self.data.dtype == torch.uint8

    def codes(self, i: int) -> torch.Tensor:
        co, cb, _, _ = self.layout[i]
        return self.data[co:co + cb]

    def scales(self, i: int) -> torch.Tensor:
        _, _, so, ns = self.layout[i]
        return self.data[so:so + 4 * ns].view(torch.float32)


def gather_payloads(local: torch.Tensor, world: int, pg=None, async_op: bool = False,
                    out: Optional[torch.Tensor] = None):
    """All-gather one flat uint8 payload per rank into a [world, nbytes] tensor
    (``out`` if given).  Returns (gathered, work); ``work`` is None unless
    async_op."""
    if out is None:
        out = torch.empty(world, local.numel(), dtype=local.dtype, device=local.device)
    work = dist.all_gather_into_tensor(out.view(-1), local, group=pg, async_op=async_op)
    return out, work


class PatchAllGather:
    """Compressed K/V exchange of patch parallelism for one rank.

    ``shapes`` are this rank's slots (e.g. the K and V shard of every layer);
    every rank passes the same shapes (equal patches).  The receiver keeps one
    fp32 cache per (peer, slot), plus a bf16 copy of it when ``recon`` is set.
    With ``include_self`` the rank also decodes its own payload into a cache
    for its own shards, as a peer would.
    """

    def __init__(self, shapes: Sequence[Sequence[int]], bits: int = 2, group: int = 128, sign_scale: int = 0,
                 buckets: int = 1, pg=None, include_self: bool = False, recon: bool = False, device=None):
        self.pg = pg
        self.world = dist.get_world_size(pg)
        self.rank = dist.get_rank(pg)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.shapes = [tuple(int(v) for v in s) for s in shapes]
        self.bits, self.group = bits, group
        self.peers = [p for p in range(self.world) if include_self or p != self.rank]
        nb = max(1, min(buckets, len(self.shapes)))
        edges = [round(i * len(self.shapes) / nb) for i in range(nb + 1)]
        self.buckets = [list(range(edges[i], edges[i + 1])) for i in range(nb) if edges[i + 1] > edges[i]]
        self.send_ctx, self.send_state, self.send_buf = [], [], []
        self.recv_ctx, self.recv_state, self.gathered = [], [], []
        self._send_arr, self._recv_arr = [], []
        for b, idx in enumerate(self.buckets):
            sh = [self.shapes[i] for i in idx]
            self.send_ctx.append(Context(sh, bits=bits, group=group, sign_scale=sign_scale))
            self.send_state.append(QuantState(sh, bits, group, device=self.device))
            self.send_buf.append(PayloadBuffer(sh, bits, group, device=self.device))
            rsh = sh * len(self.peers)
            self.recv_ctx.append(Context(rsh, bits=bits, group=group, sign_scale=sign_scale))
            self.recv_state.append(QuantState(rsh, bits, group, device=self.device, recon=recon))
            self.gathered.append(torch.empty(self.world, self.send_buf[b].nbytes, dtype=torch.uint8,
                                             device=self.device))
            # slot tables of the compressed steps, built once (only x changes per step)
            sb = self.send_buf[b]
            send = self.send_state[b].slots([torch.empty(0, dtype=torch.bfloat16, device=self.device)] * len(idx),
                                            codes=[sb.codes(s) for s in range(len(idx))],
                                            scales=[sb.scales(s) for s in range(len(idx))])
            self._send_arr.append(self.send_ctx[b]._slots(send))
            self._recv_arr.append(self.recv_ctx[b]._slots(self._peer_slots(b, self.gathered[b])))

    def cache(self, peer: int, slot: int, bf16: bool = False) -> torch.Tensor:
        """The receiver's reconstruction of ``peer``'s shard of slot ``slot``."""
        j = self.peers.index(peer)
        for b, idx in enumerate(self.buckets):
            if slot in idx:
                k = j * len(idx) + idx.index(slot)
                st = self.recv_state[b]
                return st.recon[k] if bf16 else st.cache[k]
        raise IndexError(slot)

    @staticmethod
    def _call(fn, ctx: Context, slots, t: int):
        arr = slots if not isinstance(slots, list) else ctx._slots(slots)
        st = fn(ctx.handle, arr, t, torch.cuda.current_stream().cuda_stream)
        if st != CF_OK:
            raise CfError(st, lib().cf_last_error(ctx.handle).decode())

    def _peer_slots(self, b: int, gathered: torch.Tensor, xs_peer=None) -> List[Slot]:
        idx = self.buckets[b]
        st = self.recv_state[b]
        out = []
        for j, p in enumerate(self.peers):
            pb = None if xs_peer is not None else PayloadBuffer([self.shapes[i] for i in idx], self.bits,
                                                                self.group, data=gathered[p])
            for s in range(len(idx)):
                k = j * len(idx) + s
                if xs_peer is not None:
                    out.append(Slot(x=xs_peer[p][s], cache=st.cache[k], recon=st.recon[k]))
                else:
                    out.append(Slot(codes=pb.codes(s), scales=pb.scales(s), cache=st.cache[k], recon=st.recon[k]))
        return out

    def step(self, t: int, xs: Sequence[torch.Tensor]) -> None:
        """Exchange step t for this rank's activations ``xs`` (bf16, one per
        slot, on this rank's GPU).  Step 0 all-gathers the activations
        themselves and initialises every cache; later steps move payloads."""
        L = lib()
        xs = [x.reshape(-1) for x in xs]
        for x, (r, c) in zip(xs, self.shapes):
            if x.dtype != torch.bfloat16 or x.device != self.device or not x.is_contiguous() or x.numel() != r * c:
                raise ValueError("activations must be contiguous bf16 tensors of the slot shapes on this device")
        pending = []
        for b, idx in enumerate(self.buckets):
            xb = [xs[i] for i in idx]
            arr = self._send_arr[b]
            for s, x in enumerate(xb):
                arr[s].x = x.data_ptr() if x.numel() else None
            self._call(L.cf_compress, self.send_ctx[b], arr, t)
            if t == 0:
                flat = torch.cat([x.view(torch.uint8) for x in xb])
                gathered, work = gather_payloads(flat, self.world, self.pg, async_op=True)
            else:
                gathered, work = gather_payloads(self.send_buf[b].data, self.world, self.pg, async_op=True,
                                                 out=self.gathered[b])
            pending.append((b, gathered, work))
            # decode the previous bucket while this one is in flight
            if len(pending) == 2:
                self._receive(t, *pending.pop(0))
        while pending:
            self._receive(t, *pending.pop(0))

    def _receive(self, t: int, b: int, gathered: torch.Tensor, work) -> None:
        work.wait()
        if t == 0:
            idx = self.buckets[b]
            xs_peer = {}
            for p in self.peers:
                views, off = [], 0
                for i in idx:
                    n = self.shapes[i][0] * self.shapes[i][1]
                    views.append(gathered[p][off:off + 2 * n].view(torch.bfloat16))
                    off += 2 * n
                xs_peer[p] = views
            slots = self._peer_slots(b, gathered, xs_peer)
        else:
            slots = self._recv_arr[b]
        self._call(lib().cf_decompress, self.recv_ctx[b], slots, t)

    def check(self) -> int:
        worst = CF_OK
        for ctx in self.send_ctx + self.recv_ctx:
            st = ctx.check()
            if st != CF_OK:
                worst = st
        return worst


def ring_pass(local: torch.Tensor, world: int, rank: int, on_receive, pg=None,
              spares: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """Algorithm 2's ring schedule for one flat buffer per rank.

    In round s (s = 1 .. world - 1) every rank sends the buffer it holds to
    rank + 1 and receives rank - 1's, so that after round s it holds the buffer
    that started on rank - s; ``on_receive(src, buf)`` is called with it before
    the next round forwards it.  The received buffers alternate between the
    two ``spares`` (each the size of ``local``; allocated when not given), so
    ``local`` itself is only sent, in the first ring round, and not modified.
    """
    if world <= 1:
        return
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if spares is None:
        spares = (torch.empty_like(local), torch.empty_like(local))
    bufs = [local, spares[0], spares[1]]
    cur = 0
    for s in range(1, world):
        dst = 1 if cur != 1 else 2
        ops = [dist.P2POp(dist.isend, bufs[cur], nxt, group=pg), dist.P2POp(dist.irecv, bufs[dst], prv, group=pg)]
        for w in dist.batch_isend_irecv(ops):
            w.wait()
        on_receive((rank - s) % world, bufs[dst])
        cur = dst


class RingExchange:
    """Compressed K/V ring of ring attention (Algorithm 2) for one rank.

    Each step the rank compresses its own slots into one packed payload
    buffer, which then travels the ring: in round s the rank receives the
    payload that started on rank - s, decompresses it into the cache it keeps
    for that rank's shards (the attention over that K/V block would follow
    here), and forwards it.  Step 0 sends the bf16 activations themselves.
    With ``include_self`` the rank also decodes its own payload before the first ring round.
    """

    def __init__(self, shapes: Sequence[Sequence[int]], bits: int = 2, group: int = 128, sign_scale: int = 0,
                 pg=None, include_self: bool = False, recon: bool = False, device=None):
        self.pg = pg
        self.world = dist.get_world_size(pg)
        self.rank = dist.get_rank(pg)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.shapes = [tuple(int(v) for v in s) for s in shapes]
        self.bits, self.group = bits, group
        self.include_self = include_self
        self.send_ctx = Context(self.shapes, bits=bits, group=group, sign_scale=sign_scale)
        self.send_state = QuantState(self.shapes, bits, group, device=self.device)
        self.send_buf = PayloadBuffer(self.shapes, bits, group, device=self.device)
        self.spares = (torch.empty_like(self.send_buf.data), torch.empty_like(self.send_buf.data))
        self.peers = [p for p in range(self.world) if include_self or p != self.rank]
        self.recv_ctx = {p: Context(self.shapes, bits=bits, group=group, sign_scale=sign_scale) for p in self.peers}
        self.recv_state = {p: QuantState(self.shapes, bits, group, device=self.device, recon=recon)
                           for p in self.peers}
        ns = len(self.shapes)
        send = self.send_state.slots([torch.empty(0, dtype=torch.bfloat16, device=self.device)] * ns,
                                     codes=[self.send_buf.codes(s) for s in range(ns)],
                                     scales=[self.send_buf.scales(s) for s in range(ns)])
        self._send_arr = self.send_ctx._slots(send)

    def cache(self, peer: int, slot: int, bf16: bool = False) -> torch.Tensor:
        st = self.recv_state[peer]
        return st.recon[slot] if bf16 else st.cache[slot]

    def _decode(self, t: int, src: int, buf: torch.Tensor) -> None:
        st = self.recv_state[src]
        if t == 0:
            slots, off = [], 0
            for i, (r, c) in enumerate(self.shapes):
                n = r * c
                slots.append(Slot(x=buf[off:off + 2 * n].view(torch.bfloat16), cache=st.cache[i], recon=st.recon[i]))
                off += 2 * n
        else:
            pb = PayloadBuffer(self.shapes, self.bits, self.group, data=buf)
            slots = [Slot(codes=pb.codes(i), scales=pb.scales(i), cache=st.cache[i], recon=st.recon[i])
                     for i in range(len(self.shapes))]
        PatchAllGather._call(lib().cf_decompress, self.recv_ctx[src], slots, t)

    def step(self, t: int, xs: Sequence[torch.Tensor]) -> None:
        """Ring step t for this rank's activations ``xs`` (bf16, one per slot)."""
        xs = [x.reshape(-1) for x in xs]
        for x, (r, c) in zip(xs, self.shapes):
            if x.dtype != torch.bfloat16 or x.device != self.device or not x.is_contiguous() or x.numel() != r * c:
                raise ValueError("activations must be contiguous bf16 tensors of the slot shapes on this device")
        for s, x in enumerate(xs):
            self._send_arr[s].x = x.data_ptr() if x.numel() else None
        PatchAllGather._call(lib().cf_compress, self.send_ctx, self._send_arr, t)
        local = torch.cat([x.view(torch.uint8) for x in xs]) if t == 0 else self.send_buf.data
        if self.include_self:
            self._decode(t, self.rank, local)
        ring_pass(local, self.world, self.rank, lambda src, buf: self._decode(t, src, buf), self.pg,
                  spares=None if t == 0 else self.spares)

    def check(self) -> int:
        worst = CF_OK
        for ctx in [self.send_ctx, *self.recv_ctx.values()]:
            st = ctx.check()
            if st != CF_OK:
                worst = st
        return worst
