"""Failure detection on the GPU without a fault.

Every mbarrier wait in the tcgen05 GEMM is bounded.  The fault-injection hook
CF_TEST_STARVE_GEMM=1, read when a low-rank context is created, makes the TMA
producer of that context's first cf_lowrank call issue no loads, so the
consumers wait on barriers that nothing completes; the wait gives up after
20 ms, the kernel drains, frees its tensor memory and returns, and cf_check
reports CF_E_TIMEOUT.  The context and the device stay usable: the next call
on the same context succeeds and matches the oracle.  CF_TEST_STARVE_ATTENTION=1
does the same for the attention kernel (both forms).
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


def test_bounded_wait_times_out_and_context_survives(cf, oracle):
    m, n, r, T = 256, 192, 16, 2
    A = [synth.lowrank_matrix(m, n, r, mat=11, device="cuda")]
    Q0 = [synth.q0(n, r, seed=0, mat=11, device="cuda")]
    # the hook is read when the context is created and starves its first call only
    os.environ["CF_TEST_STARVE_GEMM"] = "1"
    try:
        ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=T)
    finally:
        del os.environ["CF_TEST_STARVE_GEMM"]
    ws = torch.empty(ctx.lowrank_workspace_bytes(1, m, n), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    U, R, V = [torch.empty(m, r, device="cuda")], [torch.empty(r, r, device="cuda")], [torch.empty(n, r, device="cuda")]
    ctx.lowrank(A, Q0, U, R, V)
    status = ctx.check()
    assert status == cf.CF_E_TIMEOUT
    # the status word was cleared by the read, and the context still works
    ctx.lowrank(A, Q0, U, R, V)
    assert ctx.check() == cf.CF_OK
    Uo, Ro, Vo = oracle.subspace_iteration(A[0].cpu().numpy(), Q0[0].cpu().numpy(), T)
    Do, _, _ = oracle.lowrank_apply(A[0].cpu().numpy(), Uo, Ro, Vo)
    Dg = U[0].cpu().double().numpy() @ R[0].cpu().double().numpy() @ V[0].cpu().double().numpy().T
    assert np.linalg.norm(Dg - Do) / np.linalg.norm(Do) <= 1e-3
    ctx.close()


def test_device_errors_are_reported_not_raised_later(cf):
    """A non-finite input in the quantised path is reported by cf_check, and
    the next step on the same context runs clean."""
    shapes = [(8, 256)]
    ctx = cf.Context(shapes, bits=4, group=64)
    st = cf.QuantState(shapes, 4, 64)
    x0 = torch.zeros(2048, dtype=torch.bfloat16, device="cuda")
    x1 = x0.clone()
    x1[5] = float("nan")
    x2 = x0.clone()
    for t, x in enumerate((x0, x1)):
        sl = st.slots([x])
        ctx.compress(sl, t)
        ctx.decompress(sl, t)
    assert ctx.check() == cf.CF_E_NONFINITE
    # the NaN stays in the error buffer of its group (that group is sent as
    # zero); resetting the slot with a new warmup clears it
    for t, x in enumerate((x2, x2)):
        sl = st.slots([x])
        ctx.compress(sl, t)
        ctx.decompress(sl, t)
    assert ctx.check() == cf.CF_OK


def test_attention_waits_time_out_and_context_survives(cf, oracle):
    """CF_TEST_STARVE_ATTENTION=1 when a context is created: that context's
    first cf_attention call loads nothing, its bounded waits run out after
    20 ms and cf_check reports CF_E_TIMEOUT; the next call on the same context
    is correct.  Both forms (bf16 K/V, and dequantise-on-load writing the new
    cache)."""
    lq, lk, cols, bits, group = 200, 300, 128, 2, 64
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn(n, cols, generator=g).to(torch.bfloat16).cuda() for n in (lq, lk, lk))

    def u16(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    want = oracle.attention(u16(q), u16(k), u16(v), cols)
    codes = [torch.randint(0, 256, (lk * cols * bits // 8,), dtype=torch.uint8, generator=g).cuda() for _ in range(2)]
    scales = [(torch.rand(lk * cols // group, generator=g) * 0.1).cuda() for _ in range(2)]
    caches = [t.float().reshape(-1).contiguous() for t in (k, v)]
    for form in ("bf16", "dequantise"):
        os.environ["CF_TEST_STARVE_ATTENTION"] = "1"
        try:
            ctx = cf.Context([(lk, cols)], bits=bits, group=group)
        finally:
            del os.environ["CF_TEST_STARVE_ATTENTION"]
        out = torch.empty(lq, cols, dtype=torch.bfloat16, device="cuda")
        if form == "bf16":
            kv = (cf.KV(bf16=k), cf.KV(bf16=v))
        else:
            new = [torch.empty(lk * cols, device="cuda") for _ in range(2)]
            kv = tuple(cf.KV(cache_in=caches[i], cache_out=new[i], codes=codes[i], scales=scales[i]) for i in range(2))
        ctx.attention(q, kv[0], kv[1], out)
        assert ctx.check() == cf.CF_E_TIMEOUT, form
        ctx.attention(q, kv[0], kv[1], out)
        assert ctx.check() == cf.CF_OK, form
        if form == "bf16":
            got = out.double().cpu().numpy()
            for h in range(cols // 64):
                sl = slice(64 * h, 64 * h + 64)
                assert np.linalg.norm(got[:, sl] - want[:, sl]) / np.linalg.norm(want[:, sl]) <= 1e-2
        else:
            for i in range(2):
                c = caches[i].cpu().numpy().copy()
                oracle.decompress(codes[i].cpu().numpy(), scales[i].cpu().numpy(), c, bits, group)
                assert np.array_equal(new[i].cpu().numpy(), c), i
        ctx.close()
