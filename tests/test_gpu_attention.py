"""cf_attention on the GPU: attention over a received K/V shard, against the
CPU oracle.

Source: "Accelerating Parallel Diffusion Model Serving with Residual
Compression" (arXiv 2507.17511), reproducibility table, "Pseudocode" row,
Algorithms 1 and 2 (each device attends over the key/value blocks it receives)
and the abstract (the receiver accumulates the decompressed residuals).

* The bf16 form is compared with the oracle's fp64 attention on the same bf16
  inputs, per head, within 1e-2 relative L2: the kernel rounds P and the
  output to bf16 (2^-9 relative each) and accumulates in fp32.
* The dequantise-on-load form, fed the receiver's cache before a step and the
  step's payload, must write exactly the cache the oracle's decompress gives
  (bit for bit) and produce exactly the output of the bf16 form fed the
  receiver's recon after the same step.
* The log-sum-exp of every row is compared with the oracle's within 2e-4
  (the scores are exact products of bf16 values summed in fp32, the sum of
  the exponentials is fp32), and two shards merged by it must give the
  attention over their union (a ring step, Algorithm 2).
"""
import ctypes

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


def bf16_rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def rel_per_head(got, want, cols):
    worst = 0.0
    for h in range(cols // 64):
        g, w = got[:, 64 * h:64 * h + 64], want[:, 64 * h:64 * h + 64]
        worst = max(worst, float(np.linalg.norm(g - w) / np.linalg.norm(w)))
    return worst


@pytest.mark.parametrize("lq,lk,cols,scale", [(128, 128, 64, 1.0), (300, 260, 128, 1.0), (1, 1, 64, 1.0),
                                              (129, 1000, 192, 1.0), (200, 333, 128, 3.0), (77, 4444, 64, 1.0)])
def test_attention_bf16_matches_oracle(cf, oracle, lq, lk, cols, scale):
    """Ragged query and key counts (not multiples of the 128-row blocks), one
    to three heads, one key, many key blocks, and larger scores (scale 3:
    score spread about 9) that make the online softmax rescale."""
    q, k, v = bf16_rand((lq, cols), 1, scale), bf16_rand((lk, cols), 2, scale), bf16_rand((lk, cols), 3)
    ctx = cf.Context([], mode=cf.CF_MODE_QUANT)
    out = torch.empty(lq, cols, dtype=torch.bfloat16, device="cuda")
    ctx.attention(q.cuda(), cf.KV(bf16=k.cuda()), cf.KV(bf16=v.cuda()), out)
    assert ctx.check() == cf.CF_OK
    want = oracle.attention(u16(q), u16(k), u16(v), cols)
    assert rel_per_head(out.float().cpu().double().numpy(), want, cols) <= 1e-2


def codec_step(cf, bits, group, lk, cols, seed):
    """K and V slots through the warmup and one compressed step: returns the
    receiver's caches before the step, the step's payload and the receiver's
    cache and recon after it."""
    w = synth.COGVIDEOX.scaled(rows=lk, cols=cols, bits=bits, group=group)
    shapes = [(lk, cols)] * 2
    ctx = cf.Context(shapes, bits=bits, group=group)
    st = cf.QuantState(shapes, bits, group, recon=True)
    streams = [synth.SlotStream(w, i, seed=seed, device="cuda") for i in range(2)]
    xs = [s.next() for s in streams]
    sl = st.slots(xs)
    ctx.compress(sl, 0)
    ctx.decompress(sl, 0)
    before = [c.clone() for c in st.cache]
    xs = [s.next() for s in streams]
    sl = st.slots(xs)
    ctx.compress(sl, 1)
    ctx.decompress(sl, 1)
    torch.cuda.synchronize()
    assert ctx.check() == cf.CF_OK
    return ctx, before, st


@pytest.mark.parametrize("bits,group,lq,lk,cols", [(4, 64, 300, 333, 128), (2, 64, 128, 1111, 192),
                                                   (2, 128, 100, 700, 256), (1, 128, 65, 260, 256),
                                                   (2, 64, 129, 129, 64), (4, 8, 100, 300, 128),
                                                   (2, 16, 64, 200, 64), (1, 32, 130, 261, 192),
                                                   (4, 256, 40, 97, 256)])
def test_attention_dequantise_matches_decompress_path(cf, oracle, bits, group, lq, lk, cols):
    ctx, before, st = codec_step(cf, bits, group, lk, cols, seed=7)
    q = bf16_rand((lq, cols), 11).cuda()
    out_a = torch.empty(lq, cols, dtype=torch.bfloat16, device="cuda")
    ctx.attention(q, cf.KV(bf16=st.recon[0]), cf.KV(bf16=st.recon[1]), out_a)
    out_b = torch.empty_like(out_a)
    new = [torch.full((lk * cols,), 12345.0, device="cuda") for _ in range(2)]
    kv = [cf.KV(cache_in=before[i], cache_out=new[i], codes=st.codes[i], scales=st.scales[i]) for i in range(2)]
    lse_a = torch.empty(lq, cols // 64, device="cuda")
    lse_b = torch.full((lq, cols // 64), 7.0, device="cuda")
    ctx.attention(q, cf.KV(bf16=st.recon[0]), cf.KV(bf16=st.recon[1]), out_a, lse=lse_a)
    ctx.attention(q, kv[0], kv[1], out_b, lse=lse_b)
    torch.cuda.synchronize()
    assert ctx.check() == cf.CF_OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    assert torch.equal(lse_a, lse_b)
    for i in range(2):
        c = before[i].cpu().numpy().copy()
        oracle.decompress(st.codes[i].cpu().numpy(), st.scales[i].cpu().numpy(), c, bits, group)
        assert np.array_equal(new[i].cpu().numpy(), c), i
        assert torch.equal(new[i], st.cache[i]), i
    want = oracle.attention(u16(q), u16(st.recon[0]), u16(st.recon[1]), cols)
    assert rel_per_head(out_b.float().cpu().double().numpy(), want, cols) <= 1e-2


def test_attention_full_size_cogvideox_shard(cf, oracle):
    """The CogVideoX-shaped shard (4444 tokens x 1920 channels = 30 heads,
    k = 4, G = 64) in the launch configuration the bench times: the two forms
    agree bit for bit, the written cache equals the decompress's, and sampled
    query rows (all heads) match the oracle."""
    lq = lk = 4444
    cols, bits, group = 1920, 4, 64
    ctx, before, st = codec_step(cf, bits, group, lk, cols, seed=3)
    q = bf16_rand((lq, cols), 5).cuda()
    out_a = torch.empty(lq, cols, dtype=torch.bfloat16, device="cuda")
    ctx.attention(q, cf.KV(bf16=st.recon[0]), cf.KV(bf16=st.recon[1]), out_a)
    out_b = torch.empty_like(out_a)
    new = [torch.empty(lk * cols, device="cuda") for _ in range(2)]
    kv = [cf.KV(cache_in=before[i], cache_out=new[i], codes=st.codes[i], scales=st.scales[i]) for i in range(2)]
    ctx.attention(q, kv[0], kv[1], out_b)
    torch.cuda.synchronize()
    assert ctx.check() == cf.CF_OK
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    for i in range(2):
        assert torch.equal(new[i], st.cache[i]), i
    rows = [0, 1, 127, 128, 2000, 4351, 4443]
    qs = q[rows]
    want = oracle.attention(u16(qs), u16(st.recon[0]), u16(st.recon[1]), cols)
    assert rel_per_head(out_b[rows].float().cpu().double().numpy(), want, cols) <= 1e-2


@pytest.mark.parametrize("lq,lk,cols,scale", [(300, 260, 128, 1.0), (129, 1000, 192, 3.0), (1, 1, 64, 1.0),
                                              (256, 4444, 64, 1.0)])
def test_attention_lse_matches_oracle(cf, oracle, lq, lk, cols, scale):
    q, k, v = bf16_rand((lq, cols), 31, scale), bf16_rand((lk, cols), 32, scale), bf16_rand((lk, cols), 33)
    ctx = cf.Context([], mode=cf.CF_MODE_QUANT)
    out = torch.empty(lq, cols, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(lq, cols // 64, device="cuda")
    ctx.attention(q.cuda(), cf.KV(bf16=k.cuda()), cf.KV(bf16=v.cuda()), out, lse=lse)
    assert ctx.check() == cf.CF_OK
    want_out, want_lse = oracle.attention(u16(q), u16(k), u16(v), cols, lse=True)
    assert rel_per_head(out.float().cpu().double().numpy(), want_out, cols) <= 1e-2
    got = lse.cpu().double().numpy()
    assert np.max(np.abs(got - want_lse) / np.maximum(1.0, np.abs(want_lse))) <= 2e-4


def test_ring_step_merges_two_shards_by_lse(cf, oracle):
    """A device that receives K/V in two blocks (a ring, Algorithm 2) attends
    over each and merges the partial outputs by their log-sum-exp; the result
    is the attention over the union of the blocks."""
    lq, cols = 300, 128
    q = bf16_rand((lq, cols), 41, 2.0)
    ks = [bf16_rand((n, cols), 42 + i, 2.0) for i, n in enumerate((1000, 777))]
    vs = [bf16_rand((n, cols), 52 + i) for i, n in enumerate((1000, 777))]
    ctx = cf.Context([], mode=cf.CF_MODE_QUANT)
    outs, lses = [], []
    for kb, vb in zip(ks, vs):
        o = torch.empty(lq, cols, dtype=torch.bfloat16, device="cuda")
        ls = torch.empty(lq, cols // 64, device="cuda")
        ctx.attention(q.cuda(), cf.KV(bf16=kb.cuda()), cf.KV(bf16=vb.cuda()), o, lse=ls)
        outs.append(o.double().cpu())
        lses.append(ls.double().cpu())
    assert ctx.check() == cf.CF_OK
    lse = torch.logaddexp(lses[0], lses[1])
    merged = sum(torch.exp(l_ - lse).repeat_interleave(64, dim=1) * o for l_, o in zip(lses, outs))
    want_out, want_lse = oracle.attention(u16(q), u16(torch.cat(ks)), u16(torch.cat(vs)), cols, lse=True)
    assert rel_per_head(merged.numpy(), want_out, cols) <= 1e-2
    assert np.max(np.abs(lse.numpy() - want_lse)) <= 2e-4


def test_attention_large_shard_sampled_rows(cf, oracle):
    """100,003 keys (past 2^16, ragged against the 128-key blocks) and 70,000
    queries (274 query blocks): sampled rows of every head and their
    log-sum-exp against the oracle."""
    lq, lk, cols = 70000, 100003, 128
    q, k, v = bf16_rand((lq, cols), 61), bf16_rand((lk, cols), 62), bf16_rand((lk, cols), 63)
    ctx = cf.Context([], mode=cf.CF_MODE_QUANT)
    out = torch.empty(lq, cols, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(lq, cols // 64, device="cuda")
    ctx.attention(q.cuda(), cf.KV(bf16=k.cuda()), cf.KV(bf16=v.cuda()), out, lse=lse)
    assert ctx.check() == cf.CF_OK
    rows = [0, 255, 256, 34999, 69887, 69888, 69999]
    want_out, want_lse = oracle.attention(u16(q[rows]), u16(k), u16(v), cols, lse=True)
    assert rel_per_head(out[rows].float().cpu().double().numpy(), want_out, cols) <= 1e-2
    got = lse[rows].cpu().double().numpy()
    assert np.max(np.abs(got - want_lse) / np.maximum(1.0, np.abs(want_lse))) <= 2e-4


def test_attention_is_deterministic(cf):
    lq, lk, cols = 300, 700, 128
    q, k, v = bf16_rand((lq, cols), 21).cuda(), bf16_rand((lk, cols), 22).cuda(), bf16_rand((lk, cols), 23).cuda()
    ctx = cf.Context([], mode=cf.CF_MODE_QUANT)
    outs = []
    for _ in range(2):
        o = torch.empty(lq, cols, dtype=torch.bfloat16, device="cuda")
        ctx.attention(q, cf.KV(bf16=k), cf.KV(bf16=v), o)
        outs.append(o)
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


def test_attention_arguments_checked(cf):
    lk, cols = 64, 128
    ctx = cf.Context([(lk, cols)], bits=2, group=64)
    q = torch.zeros(8, cols, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    k = torch.zeros(lk * cols, dtype=torch.bfloat16, device="cuda")
    c_in = torch.zeros(lk * cols, device="cuda")
    codes = torch.zeros(lk * cols * 2 // 8, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(lk * cols // 64, device="cuda")
    with pytest.raises(cf.CfError) as e:        # mixed forms
        ctx.attention(q, cf.KV(bf16=k), cf.KV(cache_in=c_in, codes=codes, scales=scales), out)
    assert e.value.status == cf.CF_E_ARG
    with pytest.raises(cf.CfError) as e:        # the new cache overlaps a cache being read
        kv = cf.KV(cache_in=c_in, cache_out=c_in, codes=codes, scales=scales)
        ctx.attention(q, kv, kv, out)
    assert e.value.status == cf.CF_E_ARG
    with pytest.raises(cf.CfError) as e:        # out written over the keys other CTAs still read
        ctx.attention(q, cf.KV(bf16=k), cf.KV(bf16=k), k[:8 * cols].view(8, cols))
    assert e.value.status == cf.CF_E_ARG
    with pytest.raises(cf.CfError) as e:        # ... or over a cache being dequantised
        kv = cf.KV(cache_in=c_in, codes=codes, scales=scales)
        ctx.attention(q, kv, kv, c_in[:8 * cols // 2].view(torch.bfloat16).view(8, cols))
    assert e.value.status == cf.CF_E_ARG
    q96 = torch.zeros(8, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cf.CfError) as e:        # heads are 64 channels
        ctx.attention(q96, cf.KV(bf16=k[:lk * 96]), cf.KV(bf16=k[:lk * 96]), torch.empty_like(q96))
    assert e.value.status == cf.CF_E_SHAPE
    lean = cf.Context([(lk, cols)], bits=2, group=64, state_bf16=1)
    with pytest.raises(cf.CfError) as e:        # dequantise-on-load reads an fp32 cache
        kv = cf.KV(cache_in=c_in, codes=codes, scales=scales)
        lean.attention(q, kv, kv, out)
    assert e.value.status == cf.CF_E_ARG
    raw = torch.empty(8 * 2 + 1, device="cuda")
    with pytest.raises(cf.CfError) as e:        # lse must be 4-byte aligned
        L = cf.lib()
        st = L.cf_attention(ctx.handle, 8, lk, cols, q.data_ptr(), ctypes.byref(cf.KV(bf16=k).to_c()),
                            ctypes.byref(cf.KV(bf16=k).to_c()), out.data_ptr(), raw.data_ptr() + 2, None)
        ctx._raise(st, "cf_attention")
    assert e.value.status == cf.CF_E_ALIGN
    with pytest.raises(ValueError):             # lse of the wrong shape
        ctx.attention(q, cf.KV(bf16=k), cf.KV(bf16=k), out, lse=torch.empty(8, 3, device="cuda"))
    # no queries: nothing to do
    ctx.attention(q[:0], cf.KV(bf16=k), cf.KV(bf16=k), out[:0], lk=lk)
    assert ctx.check() == cf.CF_OK
