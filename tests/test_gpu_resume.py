"""Checkpoint / resume, and the host-side launch log.

All codec state is caller memory (base, err, cache per slot; V for the
low-rank warm start), so a checkpoint is a copy of those buffers plus the
index of the last step done.  A run stopped after step t, saved to the host,
restored into fresh buffers and continued on a fresh context with
cf_resume(t) must end bit-identical to the uninterrupted run.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def cf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_residual_compression_02_b200 as m

    m.lib()
    return m


def quant_run(cf, shapes, xs, steps, bits, group, lean, st=None, ctx=None):
    ctx = ctx or cf.Context(shapes, bits=bits, group=group, state_bf16=int(lean))
    st = st or cf.QuantState(shapes, bits, group, lean=lean)
    for t in steps:
        sl = st.slots([x[t] for x in xs])
        ctx.compress(sl, t)
        ctx.decompress(sl, t)
    torch.cuda.synchronize()
    assert ctx.check() == cf.CF_OK
    return ctx, st


@pytest.mark.parametrize("bits,group,lean", [(2, 128, False), (4, 64, False), (1, 128, True)])
def test_quant_resume_is_bit_identical(cf, bits, group, lean):
    shapes = [(64, 512), (37, 1024)]
    xs = [[x.cuda() for x in synth.activations(synth.FLUX.scaled(rows=r, cols=c), i, 6)] for i, (r, c) in
          enumerate(shapes)]
    _, full = quant_run(cf, shapes, xs, range(6), bits, group, lean)

    ctx, part = quant_run(cf, shapes, xs, range(3), bits, group, lean)
    saved = {f: [t.cpu().clone() for t in getattr(part, f)] for f in ("base", "err", "cache")}
    ctx.close()
    del part

    fresh = cf.QuantState(shapes, bits, group, lean=lean)
    for f, ts in saved.items():
        for dst, src in zip(getattr(fresh, f), ts):
            dst.copy_(src)
    ctx2 = cf.Context(shapes, bits=bits, group=group, state_bf16=int(lean))
    with pytest.raises(cf.CfError) as e:          # a fresh context refuses step 3 ...
        ctx2.compress(fresh.slots([x[3] for x in xs]), 3)
    assert e.value.status == cf.CF_E_STATE
    ctx2.resume(2)                                # ... until told where the run stands
    quant_run(cf, shapes, xs, range(3, 6), bits, group, lean, st=fresh, ctx=ctx2)
    for f in ("base", "err", "cache", "codes", "scales"):
        for i in range(len(shapes)):
            assert torch.equal(getattr(fresh, f)[i], getattr(full, f)[i]), (f, i)


def test_lowrank_warm_start_resume_is_bit_identical(cf):
    rows, cols, r, T = 192, 256, 16, 1
    shapes = [(rows, cols)]
    x = synth.gaussian((rows, cols), 0, 3, 99)
    seq = [x.to(torch.bfloat16)]
    for t in range(1, 5):
        L = synth.lowrank_matrix(rows, cols, r, mat=50 + t, noise=0.0)
        seq.append((seq[-1].float() + 0.5 * L / L.pow(2).mean().sqrt()).to(torch.bfloat16))
    seq = [s.reshape(-1).cuda() for s in seq]
    q0 = synth.q0(cols, r, seed=0, mat=3).cuda()

    def make():
        ctx = cf.Context(shapes, mode=cf.CF_MODE_LOWRANK, rank=r, iters=T, warm_start=1)
        ws = torch.empty(max(ctx.workspace_bytes(), 16), dtype=torch.uint8, device="cuda")
        ctx.set_workspace(ws)
        bufs = dict(base=torch.empty(rows * cols, dtype=torch.bfloat16, device="cuda"),
                    err=torch.empty(rows * cols, device="cuda"), cache=torch.empty(rows * cols, device="cuda"),
                    U=torch.empty(rows, r, device="cuda"), R=torch.empty(r, r, device="cuda"),
                    V=torch.empty(cols, r, device="cuda"))
        return ctx, ws, bufs

    def run(ctx, bufs, steps):
        for t in steps:
            sl = cf.Slot(x=seq[t], q0=q0 if t <= 1 else None, **bufs)
            ctx.compress([sl], t)
            ctx.decompress([sl], t)
        assert ctx.check() == cf.CF_OK

    ctx_a, ws_a, a = make()
    run(ctx_a, a, range(5))
    ctx_b, ws_b, b = make()
    run(ctx_b, b, range(3))
    saved = {k: b[k].cpu().clone() for k in ("base", "err", "cache", "V")}
    ctx_b.close()
    ctx_c, ws_c, c = make()
    for k, v in saved.items():
        c[k].copy_(v)
    ctx_c.resume(2)
    run(ctx_c, c, range(3, 5))
    for k in ("base", "err", "cache", "U", "R", "V"):
        assert torch.equal(c[k], a[k]), k


def test_launch_log(cf):
    """CF_LOG=1: every kernel launch prints one line to stderr."""
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "import torch, activation_residual_compression_02_b200 as cf\n"
        "ctx = cf.Context([(8, 256)], bits=2, group=128)\n"
        "st = cf.QuantState([(8, 256)], 2, 128)\n"
        "x = torch.zeros(8 * 256, dtype=torch.bfloat16, device='cuda')\n"
        "for t in range(2):\n"
        "    sl = st.slots([x]); ctx.compress(sl, t); ctx.decompress(sl, t)\n"
        "assert ctx.check() == cf.CF_OK\n" % ROOT)
    env = dict(os.environ, CF_LOG="1")
    p = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    lines = [l for l in p.stderr.splitlines() if l.startswith("cf: launch ")]
    assert len(lines) == 4, p.stderr
    assert "k_quant<op 2, k 2, G 128" in lines[2] and "block (256, 1, 1)" in lines[2], lines
    assert "k_quant<op 3, k 2, G 128" in lines[3], lines
