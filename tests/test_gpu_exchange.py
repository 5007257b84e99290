"""The compressed K/V all-gather (Algorithm 1) through libcf and NCCL.

Every GPU call here has one GPU, so the process group has one rank and the
rank decodes its own payload as a peer would (include_self): the path is the
whole exchange -- compress into the packed payload buffer, NCCL all-gather,
grouped decompress of the gathered payload with the bf16 reconstruction -- in
several buckets.  The caches must equal the oracle's bit for bit.
"""
import os

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_residual_compression_02_b200 as m

    m.lib()
    return m


@pytest.fixture(scope="module")
def pg():
    import torch.distributed as dist

    port = 29900 + os.getpid() % 500
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    yield None
    dist.destroy_process_group()


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).ravel()


@pytest.mark.parametrize("bits,group,buckets", [(2, 128, 2), (4, 64, 3), (1, 128, 1)])
def test_patch_all_gather_matches_oracle(cf, oracle, pg, bits, group, buckets):
    from activation_residual_compression_02_b200.exchange import PatchAllGather

    shapes = [(37, 512), (1, 256), (0, 256), (129, 768), (64, 256)]
    shapes = [(r, c) for r, c in shapes if c % group == 0]
    ex = PatchAllGather(shapes, bits=bits, group=group, buckets=buckets, include_self=True, recon=True)
    streams = [synth.SlotStream(synth.FLUX.scaled(rows=r, cols=c), slot=i) for i, (r, c) in enumerate(shapes)]
    ors = [oracle.QuantSlot(bits, group) for _ in shapes]
    for t in range(4):
        xs = [s.next() for s in streams]
        ex.step(t, [x.cuda() for x in xs])
        for i, x in enumerate(xs):
            ors[i].step(t, u16(x))
        torch.cuda.synchronize()
        for i in range(len(shapes)):
            assert np.array_equal(ex.cache(0, i).cpu().numpy(), ors[i].cache), (t, i)
            assert np.array_equal(u16(ex.cache(0, i, bf16=True)), ors[i].recon), (t, i)
            if t > 0:
                b = next(k for k, idx in enumerate(ex.buckets) if i in idx)
                s = ex.buckets[b].index(i)
                assert np.array_equal(ex.send_buf[b].codes(s).cpu().numpy(), ors[i].codes), (t, i)
    assert ex.check() == cf.CF_OK


@pytest.mark.parametrize("bits,group", [(2, 128), (4, 64)])
def test_ring_exchange_matches_oracle(cf, oracle, pg, bits, group):
    """Algorithm 2's ring on a one-rank group: the rank decodes its own payload
    (include_self) through libcf; the ring itself has no rounds here."""
    from activation_residual_compression_02_b200.exchange import RingExchange

    shapes = [(37, 512), (129, 768), (64, 256)]
    shapes = [(r, c) for r, c in shapes if c % group == 0]
    ex = RingExchange(shapes, bits=bits, group=group, include_self=True, recon=True)
    streams = [synth.SlotStream(synth.FLUX.scaled(rows=r, cols=c), slot=i) for i, (r, c) in enumerate(shapes)]
    ors = [oracle.QuantSlot(bits, group) for _ in shapes]
    for t in range(4):
        xs = [s.next() for s in streams]
        ex.step(t, [x.cuda() for x in xs])
        for i, x in enumerate(xs):
            ors[i].step(t, u16(x))
        torch.cuda.synchronize()
        for i in range(len(shapes)):
            assert np.array_equal(ex.cache(0, i).cpu().numpy(), ors[i].cache), (t, i)
            assert np.array_equal(u16(ex.cache(0, i, bf16=True)), ors[i].recon), (t, i)
    assert ex.check() == cf.CF_OK
