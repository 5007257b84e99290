"""The payload all-gather of patch parallelism (Algorithm 1) and the payload
ring of ring attention (Algorithm 2), host side, on CPU.

Two gloo ranks each own the K/V shards of their own patch.  Each packs the
oracle's payload of its shards into the exchange layout, the ranks all-gather
the flat buffers, and each rank checks every peer's part: the bytes equal the
payload it recomputes for that peer's seeded shard, and decoding them gives the
oracle's receiver cache for that shard.  The CUDA codec is not involved; its
side of the exchange is tested on the GPU.
"""
import os
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(37, 512), (1, 256), (0, 256), (64, 768)]
BITS, GROUP, STEPS = 2, 128, 3


def test_layout_is_aligned_and_disjoint():
    from activation_residual_compression_02_b200.exchange import payload_layout

    for bits, group in ((2, 128), (4, 64), (1, 256)):
        lay, total = payload_layout(SHAPES, bits, group)
        spans = []
        for (co, cb, so, ns), (r, c) in zip(lay, SHAPES):
            assert co % 16 == 0 and so % 16 == 0
            assert cb == r * c * bits // 8 and ns == r * c // group
            spans += [(co, co + cb), (so, so + 4 * ns)]
        spans = sorted(s for s in spans if s[1] > s[0])
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
        assert total >= spans[-1][1] and total % 16 == 0


def _shard(rank, slot, t, shape):
    import synth

    r, c = shape
    w = synth.FLUX.scaled(rows=r, cols=c)
    xs = synth.activations(w, 100 * rank + slot, t + 1)
    return [synth.bf16_bits(x).numpy().view(np.uint16).ravel().copy() for x in xs]


def _oracle_slots(oracle, rank, t):
    """Oracle sender+receiver of every slot of `rank`'s shard after step t."""
    out = []
    for s, shape in enumerate(SHAPES):
        o = oracle.QuantSlot(BITS, GROUP)
        for k, x in enumerate(_shard(rank, s, t, shape)):
            o.step(k, x)
        out.append(o)
    return out


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist

    import oracle
    from activation_residual_compression_02_b200.exchange import PayloadBuffer, gather_payloads

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ok = True
        for t in range(1, STEPS):
            mine = _oracle_slots(oracle, rank, t)
            buf = PayloadBuffer(SHAPES, BITS, GROUP, device="cpu")
            for s, o in enumerate(mine):
                buf.codes(s).copy_(torch.from_numpy(o.codes))
                buf.scales(s).copy_(torch.from_numpy(o.scales))
            gathered, work = gather_payloads(buf.data, world, async_op=True)
            work.wait()
            for p in range(world):
                want = _oracle_slots(oracle, p, t)
                got = PayloadBuffer(SHAPES, BITS, GROUP, data=gathered[p])
                prev = _oracle_slots(oracle, p, t - 1)
                for s, o in enumerate(want):
                    ok &= np.array_equal(got.codes(s).numpy(), o.codes)
                    ok &= np.array_equal(got.scales(s).numpy(), o.scales)
                    # decode the received payload into the receiver cache of step t - 1
                    cache = prev[s].cache.copy()
                    if cache.size:
                        oracle.decompress(got.codes(s).numpy(), got.scales(s).numpy(), cache, BITS, GROUP)
                    ok &= np.array_equal(cache, o.cache)
        out[rank] = bool(ok)
    finally:
        dist.destroy_process_group()


def test_payload_all_gather_gloo():
    port = 29700 + os.getpid() % 1000
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: True, 1: True}


def _ring_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist

    import oracle
    from activation_residual_compression_02_b200.exchange import PayloadBuffer, ring_pass

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ok = True
        t = 2
        mine = _oracle_slots(oracle, rank, t)
        buf = PayloadBuffer(SHAPES, BITS, GROUP, device="cpu")
        for s, o in enumerate(mine):
            buf.codes(s).copy_(torch.from_numpy(o.codes))
            buf.scales(s).copy_(torch.from_numpy(o.scales))
        before = buf.data.clone()
        order = []

        def on_receive(src, data):
            nonlocal ok
            order.append(src)
            got = PayloadBuffer(SHAPES, BITS, GROUP, data=data)
            want, prev = _oracle_slots(oracle, src, t), _oracle_slots(oracle, src, t - 1)
            for s, o in enumerate(want):
                ok &= np.array_equal(got.codes(s).numpy(), o.codes)
                ok &= np.array_equal(got.scales(s).numpy(), o.scales)
                cache = prev[s].cache.copy()
                if cache.size:
                    oracle.decompress(got.codes(s).numpy(), got.scales(s).numpy(), cache, BITS, GROUP)
                ok &= np.array_equal(cache, o.cache)

        ring_pass(buf.data, world, rank, on_receive)
        ok &= order == [(rank - s) % world for s in range(1, world)]
        ok &= torch.equal(buf.data, before)       # the rank's own payload is not overwritten
        out[rank] = bool(ok)
    finally:
        dist.destroy_process_group()


def test_payload_ring_gloo():
    """Algorithm 2's ring over three gloo ranks: each rank receives every other
    rank's payload once, in ring order, bit-exact and decodable by the oracle."""
    port = 29800 + os.getpid() % 1000
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_ring_worker, args=(3, port, out), nprocs=3, join=True)
        assert dict(out) == {0: True, 1: True, 2: True}
