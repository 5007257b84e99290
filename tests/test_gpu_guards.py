"""Out-of-bounds writes: every output buffer sits between 4 KiB guard bands.

compute-sanitizer is not available on the GPUs this library is tested on, so
out-of-bounds writes are caught the simple way: each buffer a kernel writes is
the middle of a larger allocation whose first and last 4 KiB hold a canary
pattern, and after the run every guard byte must be unchanged.  The shapes are
ragged (tails inside a tile, a warp and a group row; single rows; an empty
slot) so that the last tile of every slot is partial.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
GUARD = 4096   # bytes on each side
CANARY = 0xA5


@pytest.fixture(scope="module")
def cf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_residual_compression_02_b200 as m

    m.lib()
    return m


class Guarded:
    """A device buffer of n elements inside canary guard bands."""

    def __init__(self, n, dtype, shape=None):
        esz = torch.empty(0, dtype=dtype).element_size()
        self.g = GUARD // esz
        self.raw = torch.empty(n * esz + 2 * GUARD, dtype=torch.uint8, device="cuda")
        self.raw.fill_(CANARY)
        self.view = self.raw[GUARD:GUARD + n * esz].view(dtype)
        if shape is not None:
            self.view = self.view.view(*shape)

    def intact(self):
        return bool((self.raw[:GUARD] == CANARY).all()) and bool((self.raw[-GUARD:] == CANARY).all())


@pytest.mark.parametrize("bits,group,lean,loopback", [(2, 128, False, False), (4, 64, False, False),
                                                      (1, 128, False, False), (1, 256, True, False),
                                                      (2, 8, True, False), (2, 128, False, True),
                                                      (4, 64, True, True)])
def test_quantised_kernels_write_only_their_buffers(cf, bits, group, lean, loopback):
    shapes = [(37, 512), (1, 256), (0, 256), (300, 768), (5, 1024), (129, 256)]
    shapes = [(r, c) for r, c in shapes if c % group == 0]
    sdt = torch.bfloat16 if lean else torch.float32
    ctx = cf.Context(shapes, bits=bits, group=group, state_bf16=int(lean))
    bufs = []
    for r, c in shapes:
        n = r * c
        bufs.append(dict(base=Guarded(n, torch.bfloat16), err=Guarded(n, sdt), cache=Guarded(n, sdt),
                         codes=Guarded(n * bits // 8, torch.uint8), scales=Guarded(n // group, torch.float32),
                         recon=Guarded(n, torch.bfloat16)))
    streams = [synth.SlotStream(synth.FLUX.scaled(rows=r, cols=c), slot=i) for i, (r, c) in enumerate(shapes)]
    for t in range(3):
        xs = [s.next().cuda().reshape(-1) for s in streams]
        slots = [cf.Slot(x=x, **{k: v.view for k, v in b.items()}) for x, b in zip(xs, bufs)]
        if loopback and t > 0:
            ctx.loopback(slots, t)
        else:
            ctx.compress(slots, t)
            ctx.decompress(slots, t)
    assert ctx.check() == cf.CF_OK
    for i, b in enumerate(bufs):
        for k, v in b.items():
            assert v.intact(), (i, shapes[i], k)


@pytest.mark.parametrize("m,n,r,T", [(300, 200, 16, 2), (130, 64, 16, 0), (200, 72, 8, 1), (160, 96, 24, 1)])
def test_lowrank_kernels_write_only_their_buffers(cf, m, n, r, T):
    k = 3
    ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=T)
    ws = Guarded(ctx.lowrank_workspace_bytes(k, m, n), torch.uint8)
    ctx.set_workspace(ws.view)
    A = [synth.lowrank_matrix(m, n, r, mat=i, noise=0.01).cuda() for i in range(k)]
    Q0 = [synth.q0(n, r, seed=0, mat=i).cuda() for i in range(k)]
    U = [Guarded(m * r, torch.float32, (m, r)) for _ in range(k)]
    R = [Guarded(r * r, torch.float32, (r, r)) for _ in range(k)]
    V = [Guarded(n * r, torch.float32, (n, r)) for _ in range(k)]
    E = [Guarded(m * n, torch.float32, (m, n)) for _ in range(k)]
    C = [Guarded(m * n, torch.float32, (m, n)) for _ in range(k)]
    for c in C:
        c.view.zero_()
    ctx.lowrank(A, Q0, [u.view for u in U], [x.view for x in R], [v.view for v in V], [e.view for e in E],
                [c.view for c in C])
    assert ctx.check() == cf.CF_OK
    assert ws.intact()
    for name, group in (("U", U), ("R", R), ("V", V), ("E", E), ("C", C)):
        for i, g in enumerate(group):
            assert g.intact(), (name, i)
