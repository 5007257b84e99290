"""Pins of the oracle's attention (per head of 64 channels, fp64).

Source: "Accelerating Parallel Diffusion Model Serving with Residual
Compression" (arXiv 2507.17511), reproducibility table, "Pseudocode" row,
Algorithms 1 and 2 (each device attends over the key/value blocks it
receives).  The oracle writes scaled dot-product attention out directly; the
checks below pin it to special cases whose answer is fixed without it: a
single key, identical keys, a dominant key, two keys (a closed form), the
independence of heads and the order of keys, and the scale 1/sqrt(64).
"""
import math

import numpy as np
import torch

H = 64


def bits(a):
    """bf16 bit patterns of values exact in bf16."""
    t = torch.tensor(np.asarray(a, np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t), "fixture values must be exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16).copy()


def val(b):
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).double().numpy()


def rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    t = (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def test_single_key_returns_its_value(oracle):
    cols = 2 * H
    q, k, v = rand_bf16((5, cols), 1), rand_bf16((1, cols), 2), rand_bf16((1, cols), 3)
    out = oracle.attention(q, k, v, cols)
    assert np.array_equal(out, np.repeat(val(v), 5, axis=0))


def test_identical_keys_average_the_values(oracle):
    cols = H
    q = rand_bf16((4, cols), 4)
    k = np.repeat(rand_bf16((1, cols), 5), 7, axis=0)
    v = rand_bf16((7, cols), 6)
    out = oracle.attention(q, k, v, cols)
    want = np.repeat(val(v).mean(axis=0, keepdims=True), 4, axis=0)
    assert np.allclose(out, want, rtol=0, atol=1e-13)


def test_dominant_key_wins_without_overflow(oracle):
    """A score of 1000 against 0 elsewhere: the weight of that key is 1 to
    within e^-1000 (and exp(1000) itself would overflow, so the max must be
    taken out first)."""
    cols = H
    q = np.zeros((1, cols), np.float32)
    q[0, 0] = 80.0
    k = np.zeros((6, cols), np.float32)
    k[3, 0] = 100.0                      # score 80 * 100 / 8 = 1000
    v = rand_bf16((6, cols), 7)
    out = oracle.attention(bits(q), bits(k), v, cols)
    assert np.all(np.isfinite(out))
    assert np.array_equal(out[0], val(v)[3])


def test_two_keys_closed_form(oracle):
    """Scores s0 and s1 = s0 - d give weights 1 / (1 + e^-d) and e^-d / (1 + e^-d)."""
    cols = H
    q = np.zeros((1, cols), np.float32)
    q[0, 1] = 2.0
    k = np.zeros((2, cols), np.float32)
    k[0, 1] = 4.0                        # score 2 * 4 / 8 = 1
    k[1, 1] = -2.0                       # score -0.5: d = 1.5
    v = np.zeros((2, cols), np.float32)
    v[0, :] = 1.0
    v[1, :] = -3.0
    out = oracle.attention(bits(q), bits(k), bits(v), cols)
    e = np.exp(-1.5)
    want = (1.0 + e * -3.0) / (1.0 + e)
    assert np.allclose(out[0], want, rtol=1e-15, atol=0)


def test_scale_is_one_over_sqrt_head_dim(oracle):
    """Two keys whose raw dot products differ by dd (about 8 ln 3): after the
    1/8 scale the weights are 1 / (1 + e^(-dd/8)) and the rest, about 3/4 and
    1/4."""
    cols = H
    q = np.zeros((1, cols), np.float32)
    q[0, 0] = 1.0
    k = np.zeros((2, cols), np.float32)
    k[0, 0] = torch.tensor(8.0 * math.log(3.0)).to(torch.bfloat16).item()   # the nearest bf16, 8.8125
    dd = float(k[0, 0])
    v = np.zeros((2, cols), np.float32)
    v[0, :] = 1.0
    out = oracle.attention(bits(q), bits(k), bits(v), cols)
    w0 = 1.0 / (1.0 + math.exp(-dd / 8.0))
    assert np.allclose(out[0], w0, rtol=1e-15, atol=0)
    assert abs(w0 - 0.75) < 2e-3


def test_heads_are_independent(oracle):
    cols = 3 * H
    q, k, v = rand_bf16((6, cols), 8), rand_bf16((9, cols), 9), rand_bf16((9, cols), 10)
    out = oracle.attention(q, k, v, cols)
    k2, v2 = k.copy(), v.copy()
    k2[:, H:2 * H] = rand_bf16((9, H), 11)
    v2[:, H:2 * H] = rand_bf16((9, H), 12)
    out2 = oracle.attention(q, k2, v2, cols)
    for h in (0, 2):
        assert np.array_equal(out[:, h * H:(h + 1) * H], out2[:, h * H:(h + 1) * H])
    assert not np.allclose(out[:, H:2 * H], out2[:, H:2 * H])


def test_key_order_does_not_matter(oracle):
    cols = H
    q, k, v = rand_bf16((4, cols), 13), rand_bf16((11, cols), 14), rand_bf16((11, cols), 15)
    perm = np.random.default_rng(0).permutation(11)
    out = oracle.attention(q, k, v, cols)
    out2 = oracle.attention(q, k[perm], v[perm], cols)
    assert np.allclose(out, out2, rtol=0, atol=1e-12)


# ---- the log-sum-exp of a row: what merges partial results over K/V blocks --


def test_lse_of_a_single_key_is_its_score(oracle):
    """With one key the sum has one term: lse = score = (q . k) / 8, here with
    values chosen so that the dot product is exact (q . k = 2 * 3 + 0.5 * -4)."""
    cols = 2 * H
    q = np.zeros((1, cols), np.float32)
    k = np.zeros((1, cols), np.float32)
    q[0, 5], k[0, 5] = 2.0, 3.0
    q[0, H + 7], k[0, H + 7] = 0.5, -4.0
    _, lse = oracle.attention(bits(q), bits(k), rand_bf16((1, cols), 20), cols, lse=True)
    assert lse.shape == (1, 2)
    assert lse[0, 0] == 6.0 / 8.0
    assert lse[0, 1] == -2.0 / 8.0


def test_lse_of_identical_keys_adds_log_count(oracle):
    """n equal scores s: lse = s + ln n."""
    cols = H
    q = np.zeros((3, cols), np.float32)
    q[:, 2] = [1.0, -2.0, 0.25]
    k = np.zeros((13, cols), np.float32)
    k[:, 2] = 4.0
    _, lse = oracle.attention(bits(q), bits(k), rand_bf16((13, cols), 21), cols, lse=True)
    want = np.array([4.0, -8.0, 1.0]) / 8.0 + math.log(13.0)
    assert np.allclose(lse[:, 0], want, rtol=1e-15, atol=1e-15)


def test_lse_of_a_dominant_key_is_its_score(oracle):
    """Scores 1000 and 0 (five times): lse = 1000 + ln(1 + 5 e^-1000) = 1000
    in fp64, with no overflow on the way."""
    cols = H
    q = np.zeros((1, cols), np.float32)
    q[0, 0] = 80.0
    k = np.zeros((6, cols), np.float32)
    k[3, 0] = 100.0
    _, lse = oracle.attention(bits(q), bits(k), rand_bf16((6, cols), 22), cols, lse=True)
    assert lse[0, 0] == 1000.0


def test_two_blocks_merge_by_lse_into_the_whole(oracle):
    """Attention over the keys of two blocks equals the two blocks' outputs
    weighted by exp(lse_b - lse), lse = ln(e^lse_1 + e^lse_2): the merge a
    ring step does (Algorithm 2) with each block's partial result."""
    cols = 2 * H
    q, k, v = rand_bf16((7, cols), 23, 2.0), rand_bf16((50, cols), 24, 2.0), rand_bf16((50, cols), 25)
    whole, lse = oracle.attention(q, k, v, cols, lse=True)
    o1, l1 = oracle.attention(q, k[:19], v[:19], cols, lse=True)
    o2, l2 = oracle.attention(q, k[19:], v[19:], cols, lse=True)
    merged_lse = np.logaddexp(l1, l2)
    assert np.allclose(merged_lse, lse, rtol=0, atol=1e-12)
    w1 = np.repeat(np.exp(l1 - merged_lse), H, axis=1)
    w2 = np.repeat(np.exp(l2 - merged_lse), H, axis=1)
    assert np.allclose(w1 * o1 + w2 * o2, whole, rtol=0, atol=1e-12)
