"""GPU parity of the quantised codec against the CPU oracle (through the C ABI).

Codes and scales must be bit-exact; so must E, base and the receiver cache,
because every floating-point step on both sides is a single IEEE binary32
operation with round-to-nearest-even.
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


def run_case(cf, oracle, shapes, steps, bits, group, ss=0, seed=0, w=synth.TINY, check_every_step=True,
             loopback=False, recon=False):
    """Run the codec on the GPU and the oracle on the CPU for `steps` steps."""
    ctx = cf.Context(shapes, bits=bits, group=group, sign_scale=ss)
    st = cf.QuantState(shapes, bits, group, recon=recon)
    streams = [synth.SlotStream(w.scaled(rows=r, cols=c), slot=i, seed=seed) for i, (r, c) in enumerate(shapes)]
    ors = [oracle.QuantSlot(bits, group, ss) for _ in shapes]
    for t in range(steps):
        xs_cpu = [s.next() for s in streams]
        xs = [x.cuda() for x in xs_cpu]
        slots = st.slots(xs)
        if loopback:
            ctx.loopback(slots, t)
        else:
            ctx.compress(slots, t)
            ctx.decompress(slots, t)
        for i, x in enumerate(xs_cpu):
            ors[i].step(t, u16(x))
        if check_every_step or t == steps - 1:
            torch.cuda.synchronize()
            for i in range(len(shapes)):
                o = ors[i]
                assert np.array_equal(u16(st.base[i]), o.base), (t, i, "base")
                assert np.array_equal(st.err[i].cpu().numpy(), o.err), (t, i, "err")
                assert np.array_equal(st.cache[i].cpu().numpy(), o.cache), (t, i, "cache")
                if recon:
                    assert np.array_equal(u16(st.recon[i]), o.recon), (t, i, "recon")
                if t > 0:
                    assert np.array_equal(st.codes[i].cpu().numpy(), o.codes), (t, i, "codes")
                    assert np.array_equal(st.scales[i].cpu().numpy(), o.scales), (t, i, "scales")
    assert ctx.check() == cf.CF_OK
    ctx.close()


@pytest.mark.parametrize("bits,group,ss", [(2, 128, 0), (4, 64, 0), (1, 128, 0), (1, 128, 1), (2, 8, 0), (2, 16, 0),
                                           (4, 32, 0), (4, 256, 0), (1, 8, 0), (1, 256, 1), (2, 256, 0), (4, 8, 0)])
def test_tiny_workload_bit_exact(cf, oracle, bits, group, ss):
    run_case(cf, oracle, [(256, 512)], 4, bits, group, ss)


@pytest.mark.parametrize("bits,group", [(2, 128), (4, 64), (1, 128)])
def test_ragged_multi_slot_grouped_launch(cf, oracle, bits, group):
    """Several slots of different sizes in one grouped launch: tails that end
    inside a tile, inside a warp, single rows, and an empty slot."""
    shapes = [(37, 512), (1, 256), (0, 256), (300, 768), (5, 1024), (129, 256)]
    shapes = [(r, c) for r, c in shapes if c % group == 0]
    run_case(cf, oracle, shapes, 4, bits, group, w=synth.COGVIDEOX)


@pytest.mark.parametrize("bits,group,ss", [(2, 128, 0), (4, 64, 0), (1, 128, 0), (1, 256, 1), (2, 8, 0), (4, 256, 0)])
def test_loopback_bit_exact(cf, oracle, bits, group, ss):
    """cf_loopback (sender and receiver fused in one pass) equals the oracle's
    compress + decompress bit for bit, on ragged multi-slot launches."""
    shapes = [(37, 512), (1, 256), (0, 256), (300, 768), (129, 256)]
    shapes = [(r, c) for r, c in shapes if c % group == 0]
    run_case(cf, oracle, shapes, 4, bits, group, ss, w=synth.FLUX, loopback=True)


@pytest.mark.parametrize("bits,group", [(2, 128), (1, 128), (4, 64)])
def test_more_slots_than_one_launch(cf, oracle, bits, group):
    """A call with more slots than one grouped launch's table holds (128) is
    split into several launches; every slot still matches the oracle."""
    shapes = [(3 + i % 5, 256) for i in range(131)]
    run_case(cf, oracle, shapes, 3, bits, group, w=synth.FLUX, check_every_step=False)


def test_grouped_equals_per_slot(cf):
    """Launch-shape invariance: one grouped launch over all slots equals one
    context (and launch) per slot, bit for bit."""
    shapes = [(64, 512), (33, 1024), (128, 256)]
    bits, group = 2, 128
    xs_steps = [[x.cuda() for x in synth.activations(synth.FLUX.scaled(rows=r, cols=c), i, 3)] for i, (r, c) in
                enumerate(shapes)]
    ctx = cf.Context(shapes, bits=bits, group=group)
    st = cf.QuantState(shapes, bits, group)
    for t in range(3):
        slots = st.slots([xs_steps[i][t] for i in range(len(shapes))])
        ctx.compress(slots, t)
        ctx.decompress(slots, t)
    singles = []
    for i, sh in enumerate(shapes):
        c1 = cf.Context([sh], bits=bits, group=group)
        s1 = cf.QuantState([sh], bits, group)
        for t in range(3):
            sl = s1.slots([xs_steps[i][t]])
            c1.compress(sl, t)
            c1.decompress(sl, t)
        singles.append(s1)
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        for f in ("base", "err", "cache", "codes", "scales"):
            assert torch.equal(getattr(st, f)[i], getattr(singles[i], f)[0]), (i, f)


def test_constant_group_round_trip(cf):
    """A constant residual reconstructs exactly: E = 0 and C = X."""
    shapes = [(16, 256)]
    for bits in (1, 2, 4):
        ctx = cf.Context(shapes, bits=bits, group=64)
        st = cf.QuantState(shapes, bits, 64)
        x0 = torch.full((16 * 256,), 1.0, dtype=torch.bfloat16, device="cuda")
        x1 = torch.full((16 * 256,), 1.75, dtype=torch.bfloat16, device="cuda")
        for t, x in enumerate((x0, x1)):
            sl = st.slots([x])
            ctx.compress(sl, t)
            ctx.decompress(sl, t)
        torch.cuda.synchronize()
        assert torch.all(st.err[0] == 0)
        assert torch.equal(st.cache[0], x1.float())
        assert torch.all(st.scales[0] == 0.75)


def test_nonfinite_sets_status(cf):
    shapes = [(4, 128)]
    ctx = cf.Context(shapes, bits=2, group=64)
    st = cf.QuantState(shapes, 2, 64)
    x0 = torch.zeros(512, dtype=torch.bfloat16, device="cuda")
    x1 = x0.clone()
    x1[70] = float("inf")
    for t, x in enumerate((x0, x1)):
        sl = st.slots([x])
        ctx.compress(sl, t)
        ctx.decompress(sl, t)
    assert ctx.check() == cf.CF_E_NONFINITE
    # the flag was cleared by the read
    assert ctx.check() == cf.CF_OK
    torch.cuda.synchronize()
    assert st.scales[0][1].item() == 0.0       # the group holding the inf is sent as zero


def test_argument_errors_launch_nothing(cf):
    shapes = [(8, 128)]
    with pytest.raises(cf.CfError) as e:
        cf.Context(shapes, bits=3, group=128)
    assert e.value.status == cf.CF_E_ARG
    with pytest.raises(cf.CfError) as e:
        cf.Context([(8, 100)], bits=2, group=128)
    assert e.value.status == cf.CF_E_SHAPE
    ctx = cf.Context(shapes, bits=2, group=128)
    st = cf.QuantState(shapes, 2, 128)
    x = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cf.CfError) as e:          # compressed step before the warmup
        ctx.compress(st.slots([x]), 1)
    assert e.value.status == cf.CF_E_STATE
    raw = torch.zeros(1024 + 8, dtype=torch.bfloat16, device="cuda")
    bad = cf.Slot(x=raw[1:1025], base=st.base[0], err=st.err[0])  # 2-byte offset: misaligned
    with pytest.raises(cf.CfError) as e:
        ctx.compress([bad], 0)
    assert e.value.status == cf.CF_E_ALIGN
    with pytest.raises(cf.CfError) as e:
        ctx.compress([cf.Slot(x=x, base=None, err=st.err[0])], 0)
    assert e.value.status == cf.CF_E_ARG
    assert ctx.check() == cf.CF_OK
    assert ctx.payload_bytes(0) == 1024 * 2 // 8 + 4 * (1024 // 128)


# ------------------------------------------------ full-size parity, every row

FULL = [
    ("flux", synth.FLUX, None),
    ("cogvideox", synth.COGVIDEOX, None),
    ("stress", synth.STRESS, (0, 29, 59)),
]


def first_mismatch(got, want):
    bad = np.flatnonzero(got != want)
    return f"{bad.size} mismatches, first at {bad[0]}: {got[bad[0]]!r} vs {want[bad[0]]!r}" if bad.size else ""


@pytest.mark.parametrize("name,w,check_slots", FULL)
def test_full_size_every_row_bit_exact(cf, oracle, name, w, check_slots):
    """Full-size workload in the benchmark's launch configuration (one grouped
    launch per step over every slot, persistent CTAs walking many tiles): the
    warmup and two compressed steps, with base, E, C, codes and scales of
    every row compared with the oracle -- every slot of the FLUX- and
    CogVideoX-shaped workloads, three whole slots of the stress workload."""
    import concurrent.futures
    import os

    shapes = [(w.rows, w.cols)] * w.slots
    ctx = cf.Context(shapes, bits=w.bits, group=w.group)
    st = cf.QuantState(shapes, w.bits, w.group)
    streams = [synth.SlotStream(w, i, seed=0, device="cuda") for i in range(w.slots)]
    checked = list(range(w.slots)) if check_slots is None else list(check_slots)
    ors = {s: oracle.QuantSlot(w.bits, w.group) for s in checked}
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(len(checked), os.cpu_count() or 1))) as ex:
        for t in range(3):
            xs = [s.next() for s in streams]
            slots = st.slots(xs)
            ctx.compress(slots, t)
            ctx.decompress(slots, t)
            x_host = {s: u16(xs[s]) for s in checked}
            list(ex.map(lambda s: ors[s].step(t, x_host[s]), checked))
            torch.cuda.synchronize()
            for s in checked:
                o = ors[s]
                for what, got, want in (("base", u16(st.base[s]), o.base), ("err", st.err[s].cpu().numpy(), o.err),
                                        ("cache", st.cache[s].cpu().numpy(), o.cache)):
                    assert np.array_equal(got, want), (t, s, what, first_mismatch(got, want))
                if t > 0:
                    got = st.codes[s].cpu().numpy()
                    assert np.array_equal(got, o.codes), (t, s, "codes", first_mismatch(got, o.codes))
                    got = st.scales[s].cpu().numpy()
                    assert np.array_equal(got, o.scales), (t, s, "scales", first_mismatch(got, o.scales))
    # and over every slot: C + E = X (the EF identity), relative L2 <= 1e-6
    for s in range(w.slots):
        x = xs[s].float().reshape(-1)
        rel = torch.linalg.vector_norm(st.cache[s] + st.err[s] - x) / torch.linalg.vector_norm(x)
        assert rel.item() <= 1e-6, s
    assert ctx.check() == cf.CF_OK


# ------------------------------------------ hand-worked groups through libcf

from goldens import CASES as GOLDEN_CASES, bf16 as bf16_bits, floats, num  # noqa: E402


@pytest.mark.parametrize("name", sorted(GOLDEN_CASES))
def test_hand_worked_group_through_libcf(cf, name):
    """The groups worked by hand in tests/golden (codes, bytes, scale, d, E and
    C derived on paper) through cf_compress / cf_decompress on the GPU: the
    state of step 0 is written into the buffers and cf_resume(0) makes the
    next call step 1.  Includes the zero-group boundary at a scale of 2^-120."""
    c = GOLDEN_CASES[name]
    bits, group, ss = int(c["bits"]), int(c["group"]), int(c["sign_scale"])
    lean = c.get("state") == "bf16"
    ctx = cf.Context([(1, group)], bits=bits, group=group, sign_scale=ss, state_bf16=int(lean))
    st = cf.QuantState([(1, group)], bits, group, lean=lean)
    x = torch.from_numpy(bf16_bits([num(v) for v in c["x"].split(",")]).view(np.int16)).view(torch.bfloat16).cuda()
    st.base[0].copy_(torch.from_numpy(bf16_bits([num(v) for v in c["base"].split(",")]).view(np.int16))
                     .view(torch.bfloat16))
    if lean:
        def state(key):
            return torch.from_numpy(bf16_bits([num(v) for v in c[key].split(",")]).view(np.int16)).view(torch.bfloat16)
    else:
        def state(key):
            return torch.from_numpy(floats(c[key]))
    st.err[0].copy_(state("e"))
    st.cache[0].copy_(state("cache"))
    ctx.resume(0)
    sl = st.slots([x])
    ctx.compress(sl, 1)
    ctx.decompress(sl, 1)
    torch.cuda.synchronize()
    assert ctx.check() == cf.CF_OK
    assert bytes(st.codes[0].cpu().numpy()) == bytes(int(b, 16) for b in c["bytes"].split(","))
    assert st.scales[0].cpu().tolist() == [num(c["scale"])]
    assert torch.equal(st.base[0].cpu().view(torch.int16), x.cpu().view(torch.int16))
    if "e_new" in c:
        got = st.err[0].cpu()
        assert torch.equal(got.view(torch.int16) if lean else got.view(torch.int32),
                           state("e_new").view(torch.int16) if lean else state("e_new").view(torch.int32))
    if "d_exact_mask" in c:
        mask = torch.tensor([int(v) for v in c["d_exact_mask"].split(",")], dtype=torch.bool)
        d_got = st.cache[0].cpu().float() - state("cache").float()
        d_want = torch.from_numpy(floats(c["d"]))
        assert torch.equal(d_got[mask], d_want[mask])
        assert torch.all((d_got - d_want).abs() <= num(c["scale"]) * 2.0 ** -22)
    else:
        got = st.cache[0].cpu()
        assert torch.equal(got.view(torch.int16) if lean else got.view(torch.int32),
                           state("cache_new").view(torch.int16) if lean else state("cache_new").view(torch.int32))


def test_host_stream_codec_matches_oracle(cf, oracle):
    """Host-fed pipeline (copies on their own streams, double-buffered inputs
    and payloads): the payload that reaches the host each step is bit-exact."""
    shapes = [(64, 512), (37, 256), (128, 768)]
    bits, group = 2, 128
    hc = cf.HostStreamCodec(shapes, bits=bits, group=group)
    ors = [oracle.QuantSlot(bits, group) for _ in shapes]
    streams = [synth.SlotStream(synth.FLUX.scaled(rows=r, cols=c), slot=i) for i, (r, c) in enumerate(shapes)]
    steps = 6
    xs = [[s.next() for s in streams] for _ in range(steps)]
    host_x, host_pay = [], []
    for t in range(steps):
        buf, views = hc.st.activation_buffer(pin=True)
        for v, x in zip(views, xs[t]):
            v.copy_(x.reshape(-1))
        host_x.append(buf)
        host_pay.append(hc.st.payload_buffers(pin=True))
    for t in range(steps):
        hc.step(t, host_x[t], host_pay[t][0], host_pay[t][2])
    assert hc.check() == cf.CF_OK
    for t in range(steps):
        for i, x in enumerate(xs[t]):
            ors[i].step(t, u16(x))
            if t > 0:
                assert np.array_equal(host_pay[t][1][i].numpy(), ors[i].codes), (t, i)
                assert np.array_equal(host_pay[t][3][i].numpy(), ors[i].scales), (t, i)
    for i in range(len(shapes)):
        assert np.array_equal(hc.st.cache[i].cpu().numpy(), ors[i].cache)
        assert np.array_equal(hc.st.err[i].cpu().numpy(), ors[i].err)


def run_lean(cf, oracle, shapes, steps, bits, group, ss=0, loopback=False, w=synth.FLUX, recon=False):
    ctx = cf.Context(shapes, bits=bits, group=group, sign_scale=ss, state_bf16=1)
    st = cf.QuantState(shapes, bits, group, lean=True, recon=recon)
    streams = [synth.SlotStream(w.scaled(rows=r, cols=c), slot=i) for i, (r, c) in enumerate(shapes)]
    ors = [oracle.QuantSlot(bits, group, ss, lean=True) for _ in shapes]
    for t in range(steps):
        xs = [s.next() for s in streams]
        slots = st.slots([x.cuda() for x in xs])
        if loopback:
            ctx.loopback(slots, t)
        else:
            ctx.compress(slots, t)
            ctx.decompress(slots, t)
        for i, x in enumerate(xs):
            ors[i].step(t, u16(x))
        torch.cuda.synchronize()
        for i in range(len(shapes)):
            o = ors[i]
            assert np.array_equal(u16(st.err[i]), o.err), (t, i, "err")
            assert np.array_equal(u16(st.cache[i]), o.cache), (t, i, "cache")
            assert np.array_equal(u16(st.base[i]), o.base), (t, i, "base")
            if recon:
                assert np.array_equal(u16(st.recon[i]), o.recon), (t, i, "recon")
            if t > 0:
                assert np.array_equal(st.codes[i].cpu().numpy(), o.codes), (t, i, "codes")
                assert np.array_equal(st.scales[i].cpu().numpy(), o.scales), (t, i, "scales")
    assert ctx.check() == cf.CF_OK


@pytest.mark.parametrize("bits,group,ss", [(2, 128, 0), (4, 64, 0), (1, 128, 0), (1, 128, 1), (2, 8, 0), (4, 256, 0)])
@pytest.mark.parametrize("loopback", [False, True])
def test_lean_state_bit_exact(cf, oracle, bits, group, ss, loopback):
    """Lean state (E and C in bf16): codes, scales, E, C and base bit-exact to
    the oracle's lean codec, for the pair and for the fused loopback."""
    shapes = [(37, 512), (1, 256), (0, 256), (129, 768)]
    shapes = [(r, c) for r, c in shapes if c % group == 0]
    run_lean(cf, oracle, shapes, 4, bits, group, ss, loopback)


def test_lean_state_rejected_in_lowrank_mode(cf):
    with pytest.raises(cf.CfError) as e:
        cf.Context([(64, 64)], mode=cf.CF_MODE_LOWRANK, rank=4, iters=1, state_bf16=1)
    assert e.value.status == cf.CF_E_ARG


@pytest.mark.parametrize("bits,group", [(2, 128), (4, 64), (1, 128), (2, 8)])
@pytest.mark.parametrize("lean,loopback", [(False, False), (False, True), (True, False), (True, True)])
def test_bf16_reconstruction_bit_exact(cf, oracle, bits, group, lean, loopback):
    """With a recon buffer the receiver also writes bf16(C) (RNE) from the same
    pass: equal to the oracle's rounding of its own C at every step (X_0 at the
    warmup), and C, E, codes and scales unchanged by it."""
    shapes = [(37, 512), (1, 256), (0, 256), (129, 768)]
    shapes = [(r, c) for r, c in shapes if c % group == 0]
    if lean:
        run_lean(cf, oracle, shapes, 4, bits, group, loopback=loopback, recon=True)
    else:
        run_case(cf, oracle, shapes, 4, bits, group, w=synth.FLUX, loopback=loopback, recon=True)


def test_bf16_reconstruction_only_where_asked(cf, oracle):
    """recon is per slot and per call: slot 1 gets a recon buffer at steps 0
    and 1 only, so afterwards it holds the step-1 reconstruction while slot 0's
    follows every step; a misaligned recon is refused before any launch."""
    shapes = [(64, 512), (32, 256)]
    ctx = cf.Context(shapes, bits=2, group=128)
    st = cf.QuantState(shapes, 2, 128, recon=True)
    streams = [synth.SlotStream(synth.FLUX.scaled(rows=r, cols=c), slot=i) for i, (r, c) in enumerate(shapes)]
    ors = [oracle.QuantSlot(2, 128) for _ in shapes]
    side = torch.empty(32 * 256, dtype=torch.bfloat16, device="cuda")
    expect_side = None
    for t in range(3):
        xs = [s.next() for s in streams]
        slots = st.slots([x.cuda() for x in xs])
        slots[1].recon = side if t < 2 else None
        ctx.compress(slots, t)
        if t == 2:
            bad = torch.empty(64 * 512 + 8, dtype=torch.bfloat16, device="cuda")
            slots[0].recon = bad[1:1 + 64 * 512]
            with pytest.raises(cf.CfError) as e:
                ctx.decompress(slots, t)
            assert e.value.status == cf.CF_E_ALIGN
            slots[0].recon = st.recon[0]
        ctx.decompress(slots, t)
        for i, x in enumerate(xs):
            ors[i].step(t, u16(x))
        if t == 1:
            expect_side = ors[1].recon
    torch.cuda.synchronize()
    assert ctx.check() == cf.CF_OK
    assert np.array_equal(u16(st.recon[0]), ors[0].recon)
    assert np.array_equal(st.cache[1].cpu().numpy(), ors[1].cache)
    assert np.array_equal(u16(side), expect_side)


@pytest.mark.parametrize("bits,ss", [(2, 0), (4, 0), (1, 0), (1, 1)])
def test_narrowest_rows(cf, oracle, bits, ss):
    """Rows of a single vector (cols = G = 8) and of two or three groups, with
    one-row slots: every group is a whole row and lanes of a warp cover
    several rows."""
    run_case(cf, oracle, [(3, 8), (1, 16), (7, 24), (1, 8), (65, 8)], 4, bits, 8, ss, w=synth.FLUX)
