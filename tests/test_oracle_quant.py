"""Pins of the oracle's quantised path against what the definitions fix.

Nothing here re-types the oracle's formulas: the checks are hand-worked
groups (tests/golden), exact special cases, closed-form error bounds and
invariants, and an independent decode of the payload with numpy's bit
routines.  Source: "Accelerating Parallel Diffusion Model Serving with
Residual Compression" (arXiv 2507.17511), abstract (compressed residuals plus
error feedback) and reproducibility table, "Dataset Splits" row (warmup
initialises the base tensor); xDiT issue 573 (8-16x less communication).
"""
import math
import os

import numpy as np
import pytest
import torch

import synth

from goldens import CASES, bf16, floats, num  # noqa: E402


@pytest.mark.parametrize("name", sorted(CASES))
def test_hand_worked_group(oracle, name):
    c = CASES[name]
    bits, group, ss = int(c["bits"]), int(c["group"]), int(c["sign_scale"])
    x = bf16([num(v) for v in c["x"].split(",")])
    base = bf16([num(v) for v in c["base"].split(",")])
    if c.get("state") == "bf16":
        err = bf16([num(v) for v in c["e"].split(",")])
        cache = bf16([num(v) for v in c["cache"].split(",")])
        codes, scales, flags = oracle.compress_lean(x, base, err, bits, group, ss)
        assert flags == 0
        assert codes.tobytes() == bytes(int(b, 16) for b in c["bytes"].split(","))
        assert scales.tolist() == [num(c["scale"])]
        assert np.array_equal(err, bf16([num(v) for v in c["e_new"].split(",")]))
        oracle.decompress_lean(codes, scales, cache, bits, group)
        assert np.array_equal(cache, bf16([num(v) for v in c["cache_new"].split(",")]))
        return
    err = floats(c["e"])
    cache = floats(c["cache"])
    codes, scales, flags = oracle.compress(x, base, err, bits, group, ss)
    assert flags == 0
    want_bytes = bytes(int(b, 16) for b in c["bytes"].split(","))
    assert codes.tobytes() == want_bytes
    assert scales.tolist() == [num(c["scale"])]
    # the per-element codes, read back through numpy's own bit routine
    bitstream = np.unpackbits(codes, bitorder="little")
    got = [int(sum(int(bitstream[j * bits + b]) << b for b in range(bits))) for j in range(group)]
    assert got == [int(v) for v in c["codes"].split(",")]
    # base advanced to x
    assert np.array_equal(base, x)
    oracle.decompress(codes, scales, cache, bits, group)
    d_want = floats(c["d"])
    s = num(c["scale"])
    if "d_exact_mask" in c:
        mask = np.array([int(v) for v in c["d_exact_mask"].split(",")], bool)
        d_got = cache - floats(c["cache"])
        assert np.array_equal(d_got[mask], d_want[mask])
        assert np.all(np.abs(d_got - d_want) <= s * 2.0 ** -22)
    else:
        assert np.array_equal(cache, floats(c["cache_new"]))
    if "e_new" in c:
        assert np.array_equal(err, floats(c["e_new"]))


@pytest.mark.parametrize("bits", [1, 2, 4])
@pytest.mark.parametrize("group", [8, 64, 128, 256])
@pytest.mark.parametrize("value", [0.75, -3.0, 2.0 ** -100, -1.5e4])
def test_constant_residual_round_trips_exactly(oracle, bits, group, value):
    """A group of equal residuals has scale |v| and level +-1: d = v, E = 0."""
    n = group * 3
    base = bf16([1.0] * n)
    x = bf16([1.0] * n)
    err = np.full(n, value, np.float32)   # residual a = 0 + value, exactly
    cache = np.zeros(n, np.float32)
    codes, scales, flags = oracle.compress(x, base, err, bits, group, 0)
    assert flags == 0
    assert np.all(scales == abs(np.float32(value)))
    oracle.decompress(codes, scales, cache, bits, group)
    assert np.array_equal(cache, np.full(n, value, np.float32))
    assert np.all(err == 0.0)


def _run(oracle, w, steps, bits, group, ss=0, slot=0, rows=None):
    xs = synth.activations(w, slot, steps, rows=rows)
    st = oracle.QuantSlot(bits, group, ss)
    out = []
    for t, x in enumerate(xs):
        xb = synth.bf16_bits(x).numpy().view(np.uint16).ravel().copy()
        a = None
        if t > 0:
            b2 = st.base.copy()
            a = oracle.residual(xb, b2, st.err)
        st.step(t, xb)
        out.append((x.float().numpy().ravel(), a, st.codes, st.scales, st.err.copy(), st.cache.copy()))
    return st, out


@pytest.mark.parametrize("bits,group,ss", [(2, 128, 0), (4, 64, 0), (1, 128, 0), (1, 128, 1), (2, 8, 0), (4, 256, 0)])
def test_error_feedback_identity(oracle, bits, group, ss):
    """C_t + E_t equals X_t: the receiver plus the carried error is the truth."""
    w = synth.TINY
    st, out = _run(oracle, w, 6, bits, group, ss)
    for t, (x, a, codes, scales, err, cache) in enumerate(out):
        x64 = x.astype(np.float64)
        rec = cache.astype(np.float64) + err.astype(np.float64)
        rel = np.linalg.norm(rec - x64) / np.linalg.norm(x64)
        assert rel <= 1e-6, (t, rel)
    assert st.flags == 0


@pytest.mark.parametrize("bits,group", [(2, 128), (4, 64), (2, 32), (4, 8)])
def test_per_element_error_bound(oracle, bits, group):
    """|a - d| <= s (1/(2L) + 2^-22): rounding to the nearest of 2L+1 levels."""
    L = (1 << (bits - 1)) - 1
    st, out = _run(oracle, synth.FLUX.scaled(rows=64, cols=512, outlier_frac=0.01), 5, bits, group)
    for t, (x, a, codes, scales, err, cache) in enumerate(out[1:], 1):
        s = np.repeat(scales.astype(np.float64), group)
        d = a.astype(np.float64) - err.astype(np.float64)
        bound = s * (0.5 / L + 2.0 ** -22)
        assert np.all(np.abs(a.astype(np.float64) - d) <= bound)
        # scale is the exact group absmax
        assert np.array_equal(scales, np.abs(a).reshape(-1, group).max(axis=1))
        # codes stay in [0, 2L]
        bitstream = np.unpackbits(codes, bitorder="little").reshape(-1, bits)
        code = (bitstream.astype(np.int64) << np.arange(bits)).sum(axis=1)
        assert code.min() >= 0 and code.max() <= 2 * L


@pytest.mark.parametrize("bits,group", [(2, 128), (4, 64), (1, 128), (2, 16)])
def test_independent_numpy_decode(oracle, bits, group):
    """Decoding the payload with numpy (unpackbits, level table from fractions)
    reproduces the oracle's dequantised values d = a - E_new."""
    L = (1 << (bits - 1)) - 1
    st, out = _run(oracle, synth.COGVIDEOX.scaled(rows=48, cols=640), 4, bits, group)
    for t, (x, a, codes, scales, err, cache) in enumerate(out[1:], 1):
        bitstream = np.unpackbits(codes, bitorder="little").reshape(-1, bits)
        code = (bitstream.astype(np.int64) << np.arange(bits)).sum(axis=1)
        s = np.repeat(scales.astype(np.float64), group)
        if bits == 1:
            d_np = np.where(code == 1, s, -s)
        else:
            d_np = (code - L) / L * s
        d_or = a.astype(np.float64) - err.astype(np.float64)
        # E_new = fl(a - d) is one rounding of a value below |a| + s
        tol = (np.abs(a.astype(np.float64)) + s) * 2.0 ** -23
        assert np.all(np.abs(d_np - d_or) <= tol)


@pytest.mark.parametrize("group", [8, 32, 128, 256])
def test_one_bit_mean_scale(oracle, group):
    """k=1 (mean |a| scale): s is the group mean of |a| to within a binary-tree
    sum's rounding, the error energy obeys ||E||^2 = ||a||^2 - G s^2, and the
    compressor is contractive."""
    st, out = _run(oracle, synth.STRESS.scaled(rows=32, cols=1024), 4, 1, group)
    depth = int(math.log2(group))
    for t, (x, a, codes, scales, err, cache) in enumerate(out[1:], 1):
        ag = a.astype(np.float64).reshape(-1, group)
        eg = err.astype(np.float64).reshape(-1, group)
        mean = np.abs(ag).mean(axis=1)
        assert np.all(np.abs(scales - mean) <= (depth + 1) * 2.0 ** -24 * mean)
        lhs = (eg ** 2).sum(axis=1)
        rhs = (ag ** 2).sum(axis=1) - group * scales.astype(np.float64) ** 2
        assert np.allclose(lhs, rhs, rtol=1e-5, atol=1e-30)
        assert np.all(lhs <= (ag ** 2).sum(axis=1) * (1 + 1e-6))
        # sign codes: 1 exactly where a >= 0
        bitstream = np.unpackbits(codes, bitorder="little")
        assert np.array_equal(bitstream.astype(bool), a >= 0)


def test_zero_and_subnormal_groups(oracle):
    """A group whose scale is zero or below 2^-120 is sent as all-zero."""
    G = 8
    x = bf16([2.0] * (3 * G))
    base = x.copy()
    err = np.zeros(3 * G, np.float32)
    err[G:2 * G] = np.float32(1e-39)          # subnormal residual
    err[2 * G] = np.float32(2.0 ** -119)     # just above the threshold
    for bits, zc in [(2, 1), (4, 7), (1, 1)]:
        e = err.copy()
        codes, scales, flags = oracle.compress(x, base.copy(), e, bits, G, 0)
        assert flags == 0
        bitstream = np.unpackbits(codes, bitorder="little").reshape(-1, bits)
        code = (bitstream.astype(np.int64) << np.arange(bits)).sum(axis=1)
        assert np.all(code[:2 * G] == zc)
        assert scales[0] == 0.0 and scales[1] == 0.0
        assert np.array_equal(e[:2 * G], err[:2 * G])   # all of a stays in E
        if bits >= 2:
            assert scales[2] == np.float32(2.0 ** -119)


def test_nonfinite_is_flagged(oracle):
    G = 16
    x = bf16([0.5] * (2 * G))
    for bad in (np.inf, -np.inf, np.nan):
        for bits, ss in [(2, 0), (4, 0), (1, 0), (1, 1)]:
            err = np.zeros(2 * G, np.float32)
            err[3] = bad
            err[G + 1] = 0.25
            base = bf16([0.0] * (2 * G))
            codes, scales, flags = oracle.compress(x, base, err, bits, G, ss)
            assert flags & oracle.FLAG_NONFINITE
            assert scales[0] == 0.0
            assert scales[1] > 0.0


def test_warmup(oracle):
    x = synth.activations(synth.TINY, 0, 1)[0]
    xb = synth.bf16_bits(x).numpy().view(np.uint16).ravel().copy()
    base, err = oracle.warmup_sender(xb)
    cache = oracle.warmup_receiver(xb)
    assert np.array_equal(base, xb)
    assert np.all(err == 0) and not np.any(np.signbit(err))
    assert np.array_equal(cache, x.float().numpy().ravel())


@pytest.mark.parametrize("bits,group,ratio", [(2, 128, 128 / 18), (1, 128, 12.8), (4, 64, 64 / 18)])
def test_payload_bytes_and_ratio(oracle, bits, group, ratio):
    """Payload = n k/8 + 4 n/G bytes; versus bf16 that is 16G/(kG+32)x.
    Before the scale overhead the ratio is 16/k: 8x at k=2 and 16x at k=1,
    the 8-16x range quoted for the method."""
    n = 1152 * 3072
    pb = oracle.payload_bytes(n, bits, group)
    assert pb == n * bits // 8 + 4 * (n // group)
    assert abs(2 * n / pb - ratio) < 1e-9
    assert oracle.payload_bytes(n + 1, bits, group) == -1


def test_rows_are_independent(oracle):
    """Each token row quantises on its own (groups never straddle rows): a row
    compressed alone equals the same row compressed inside the full slot."""
    st, out = _run(oracle, synth.COGVIDEOX.scaled(rows=40, cols=320), 3, 4, 64)
    xs = synth.activations(synth.COGVIDEOX.scaled(rows=40, cols=320), 0, 3)
    row = 17
    sub = oracle.QuantSlot(4, 64)
    for t, x in enumerate(xs):
        xb = synth.bf16_bits(x[row]).numpy().view(np.uint16).copy()
        sub.step(t, xb)
    cols = 320
    full = out[-1]
    assert np.array_equal(sub.err, full[4][row * cols:(row + 1) * cols])
    assert np.array_equal(sub.cache, full[5][row * cols:(row + 1) * cols])
    assert np.array_equal(sub.scales, full[3][row * cols // 64:(row + 1) * cols // 64])
    assert np.array_equal(sub.codes, full[2][row * cols // 2:(row + 1) * cols // 2])


def test_bad_arguments_rejected(oracle):
    x = bf16([0.0] * 24)
    with pytest.raises(ValueError):
        oracle.compress(x, x.copy(), np.zeros(24, np.float32), 3, 8)
    with pytest.raises(ValueError):
        oracle.compress(x, x.copy(), np.zeros(24, np.float32), 2, 16)  # 24 % 16 != 0


def _bits_to_f32(b):
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).float().numpy()


def _f32_to_bf16_bits(f):
    return torch.from_numpy(np.ascontiguousarray(f, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


@pytest.mark.parametrize("bits,group", [(2, 128), (4, 64), (1, 128)])
def test_lean_state_is_the_fp32_step_rounded_to_bf16(oracle, bits, group):
    """From a common state (E, C exact in bf16), one lean step sends the same
    payload as the fp32-state step, and its new E and C are the fp32-state
    results rounded to bf16 by torch (an independent round-to-nearest-even)."""
    w = synth.FLUX.scaled(rows=24, cols=512, outlier_frac=0.01)
    xs = synth.activations(w, 0, 4)
    lean = oracle.QuantSlot(bits, group, lean=True)
    for t in range(3):
        lean.step(t, synth.bf16_bits(xs[t]).numpy().view(np.uint16).ravel().copy())
    x3 = synth.bf16_bits(xs[3]).numpy().view(np.uint16).ravel().copy()
    base32, err32, cache32 = lean.base.copy(), _bits_to_f32(lean.err), _bits_to_f32(lean.cache)
    codes32, scales32, _ = oracle.compress(x3, base32, err32, bits, group)
    oracle.decompress(codes32, scales32, cache32, bits, group)
    lean.step(3, x3)
    assert np.array_equal(lean.codes, codes32)
    assert np.array_equal(lean.scales, scales32)
    assert np.array_equal(lean.err, _f32_to_bf16_bits(err32))
    assert np.array_equal(lean.cache, _f32_to_bf16_bits(cache32))
    assert np.array_equal(lean.base, x3)


def test_lean_state_error_feedback_identity(oracle):
    """With bf16 E and C the identity C + E = X holds up to the bf16 rounding of
    E and C at each step (a few 2^-9 relative over a handful of steps)."""
    w = synth.COGVIDEOX.scaled(rows=32, cols=640)
    xs = synth.activations(w, 1, 6)
    st = oracle.QuantSlot(4, 64, lean=True)
    for t, x in enumerate(xs):
        st.step(t, synth.bf16_bits(x).numpy().view(np.uint16).ravel().copy())
        x64 = x.float().numpy().ravel().astype(np.float64)
        rec = _bits_to_f32(st.cache).astype(np.float64) + _bits_to_f32(st.err).astype(np.float64)
        rel = np.linalg.norm(rec - x64) / np.linalg.norm(x64)
        assert rel <= (t + 1) * 2.0 ** -9, (t, rel)


@pytest.mark.parametrize("bits_in,bits_out", [
    (0x3F800000, 0x3F80),   # 1.0
    (0x3F808000, 0x3F80),   # 1 + 2^-8: halfway, the even neighbour is 1.0
    (0x3F818000, 0x3F82),   # 1 + 3*2^-8: halfway, the even neighbour is above
    (0x3F808001, 0x3F81),   # just above halfway rounds up
    (0x3F80FFFF, 0x3F81),
    (0xC0200000, 0xC020),   # -2.5, exact
    (0x80000000, 0x8000),   # -0 keeps its sign
    (0x7F7FFFFF, 0x7F80),   # the largest float rounds to +inf
    (0x7F800000, 0x7F80),   # +inf
    (0xFF800000, 0xFF80),   # -inf
    (0x00008000, 0x0000),   # subnormal halfway, even neighbour 0
    (0x00018000, 0x0002),   # subnormal halfway, even neighbour above
    (0x7FC00000, 0x7FC0),   # quiet NaN
    (0x7F800001, 0x7FC0),   # signalling NaN comes out quiet
])
def test_bf16_rounding_hand_values(oracle, bits_in, bits_out):
    """The receiver's bf16 reconstruction rounds to nearest even: hand-checked
    bit patterns, ties both ways, overflow, signed zero, subnormals, NaN."""
    f = np.array([bits_in], np.uint32).view(np.float32)
    assert int(oracle.to_bf16(f)[0]) == bits_out


def test_bf16_rounding_matches_torch(oracle):
    """Against torch's own float -> bfloat16 conversion (round to nearest even)
    on 2^20 finite floats spread over every exponent."""
    rng = np.random.default_rng(5)
    u = rng.integers(0, 2 ** 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.to_bf16(f), want)


def test_bf16_reconstruction_of_a_slot(oracle):
    """QuantSlot.recon is the warmup activation itself at step 0 and the
    rounding of the fp32 cache afterwards; with the lean state it is the
    cache."""
    w = synth.FLUX.scaled(rows=8, cols=256)
    xs = synth.activations(w, 0, 3)
    s32 = oracle.QuantSlot(2, 128)
    s16 = oracle.QuantSlot(2, 128, lean=True)
    for t, x in enumerate(xs):
        xb = synth.bf16_bits(x).numpy().view(np.uint16).ravel().copy()
        s32.step(t, xb)
        s16.step(t, xb)
        if t == 0:
            assert np.array_equal(s32.recon, xb)
            assert np.array_equal(s16.recon, xb)
        assert np.array_equal(s32.recon, oracle.to_bf16(s32.cache))
        assert np.array_equal(s16.recon, s16.cache)
