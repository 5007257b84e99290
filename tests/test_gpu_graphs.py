"""The codec calls inside CUDA graphs.

Every call is stream-ordered and allocates nothing on the device, so a step
(or a whole low-rank call) can be captured once and replayed.  A replayed
quantised step must match the oracle bit for bit, and a replayed low-rank call
must equal the eagerly launched one bit for bit (the call is deterministic).
"""
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


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).ravel()


@pytest.mark.parametrize("bits,group,loopback", [(2, 128, False), (4, 64, True), (1, 128, False)])
def test_quant_step_replayed_from_a_graph(cf, oracle, bits, group, loopback):
    shapes = [(37, 512), (1, 256), (129, 768)]
    shapes = [(r, c) for r, c in shapes if c % group == 0]
    ctx = cf.Context(shapes, bits=bits, group=group)
    st = cf.QuantState(shapes, bits, group, recon=True)
    xbuf, xviews = st.activation_buffer()        # the graph reads X from here
    streams = [synth.SlotStream(synth.FLUX.scaled(rows=r, cols=c), slot=i) for i, (r, c) in enumerate(shapes)]
    ors = [oracle.QuantSlot(bits, group) for _ in shapes]
    slots = st.slots(xviews)

    def feed(t):
        xs = [s.next() for s in streams]
        for v, x in zip(xviews, xs):
            v.copy_(x.reshape(-1))
        for o, x in zip(ors, xs):
            o.step(t, u16(x))

    feed(0)
    ctx.compress(slots, 0)
    ctx.decompress(slots, 0)
    feed(1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                   # one eager compressed step: shapes and caches settle
        if loopback:
            ctx.loopback(slots, 1, stream=s)
        else:
            ctx.compress(slots, 1, stream=s)
            ctx.decompress(slots, 1, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cs = torch.cuda.current_stream()
        if loopback:
            ctx.loopback(slots, 2, stream=cs)
        else:
            ctx.compress(slots, 2, stream=cs)
            ctx.decompress(slots, 2, stream=cs)
    for t in range(2, 5):
        feed(t)
        g.replay()
        torch.cuda.synchronize()
        for i, o in enumerate(ors):
            assert np.array_equal(st.codes[i].cpu().numpy(), o.codes), (t, i)
            assert np.array_equal(st.scales[i].cpu().numpy(), o.scales), (t, i)
            assert np.array_equal(st.err[i].cpu().numpy(), o.err), (t, i)
            assert np.array_equal(st.cache[i].cpu().numpy(), o.cache), (t, i)
            assert np.array_equal(u16(st.recon[i]), o.recon), (t, i)
    assert ctx.check() == cf.CF_OK


def test_lowrank_call_replayed_from_a_graph(cf):
    m, n, r, T, k = 600, 1024, 16, 2, 3
    ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=T)
    ws = torch.empty(ctx.lowrank_workspace_bytes(k, m, n), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    A = [synth.lowrank_matrix(m, n, r, mat=i).cuda() for i in range(k)]
    Q0 = [synth.q0(n, r, seed=0, mat=i).cuda() for i in range(k)]

    def outs():
        return ([torch.empty(m, r, device="cuda") for _ in A], [torch.empty(r, r, device="cuda") for _ in A],
                [torch.empty(n, r, device="cuda") for _ in A], [torch.empty(m, n, device="cuda") for _ in A])

    U1, R1, V1, E1 = outs()
    ctx.lowrank(A, Q0, U1, R1, V1, E1)
    U2, R2, V2, E2 = outs()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ctx.lowrank(A, Q0, U2, R2, V2, E2, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for t in E2:
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ctx.lowrank(A, Q0, U2, R2, V2, E2, stream=torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    assert ctx.check() == cf.CF_OK
    for a, b in zip(U1 + R1 + V1 + E1, U2 + R2 + V2 + E2):
        assert torch.equal(a, b)
