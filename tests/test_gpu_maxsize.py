"""Slots and matrices past 2^31 elements: 64-bit indexing in every kernel.

Element 2^31 is where a 32-bit element index (or a 32-bit byte offset into a
quarter of the slot) would wrap, so the sampled rows straddle it.  Each test
needs tens of GB of device memory (a B200 has 180 GB) and is skipped when the
device has less free.
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


def need_free(gb):
    free = torch.cuda.mem_get_info()[0]
    if free < gb * 2 ** 30:
        pytest.skip(f"needs {gb} GB of free device memory, {free / 2 ** 30:.0f} GB free")


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).ravel()


def test_quant_slot_past_2_31_elements(cf, oracle):
    """One k = 2, G = 128 slot of (2^20 + 512) x 2048 = 2^31 + 2^20 elements,
    with the bf16 reconstruction: sampled rows on both sides of element 2^31
    bit-exact to the oracle for the warmup and two compressed steps."""
    need_free(80)
    rows, cols, bits, group = (1 << 20) + 512, 2048, 2, 128
    assert rows * cols > 2 ** 31
    w = synth.FLUX.scaled(slots=1, rows=rows, cols=cols, bits=bits, group=group)
    ctx = cf.Context([(rows, cols)], bits=bits, group=group)
    st = cf.QuantState([(rows, cols)], bits, group, recon=True)
    stream = synth.SlotStream(w, 0, seed=3, device="cuda")
    boundary = (1 << 31) // cols
    sample_rows = [0, boundary - 1, boundary, boundary + 1, rows - 1]
    ors = {r: oracle.QuantSlot(bits, group) for r in sample_rows}
    cb, gs = cols * bits // 8, cols // group
    for t in range(3):
        x = stream.next().reshape(-1)
        slots = st.slots([x])
        ctx.compress(slots, t)
        ctx.decompress(slots, t)
        torch.cuda.synchronize()
        for r in sample_rows:
            o = ors[r]
            sl = slice(r * cols, (r + 1) * cols)
            o.step(t, u16(x[sl]))
            assert np.array_equal(u16(st.base[0][sl]), o.base), (t, r)
            assert np.array_equal(st.err[0][sl].cpu().numpy(), o.err), (t, r)
            assert np.array_equal(st.cache[0][sl].cpu().numpy(), o.cache), (t, r)
            assert np.array_equal(u16(st.recon[0][sl]), o.recon), (t, r)
            if t > 0:
                assert np.array_equal(st.codes[0][r * cb:(r + 1) * cb].cpu().numpy(), o.codes), (t, r)
                assert np.array_equal(st.scales[0][r * gs:(r + 1) * gs].cpu().numpy(), o.scales), (t, r)
        del x, slots
    assert ctx.check() == cf.CF_OK
    ctx.close()


def test_lowrank_matrix_past_2_31_elements(cf):
    """Algorithm 3 on one exactly rank-16 fp32 matrix of (2^16 + 128) x 32768
    elements (2^31 + 2^22), with E written.  The oracle cannot run at this size,
    so the checks are properties that hold at any size: U and V orthonormal, R
    upper triangular, E small against A (exact rank), and on sampled rows on
    both sides of element 2^31, E = A - U R V^T for the returned factors."""
    need_free(40)
    m, n, r, T = (1 << 16) + 128, 32768, 16, 2
    assert m * n > 2 ** 31
    ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=T)
    ws = torch.empty(ctx.lowrank_workspace_bytes(1, m, n), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    A = synth.lowrank_matrix(m, n, r, mat=11, noise=0.0, device="cuda")
    Q0 = synth.q0(n, r, seed=0, mat=11, device="cuda")
    U = torch.empty(m, r, device="cuda")
    R = torch.empty(r, r, device="cuda")
    V = torch.empty(n, r, device="cuda")
    E = torch.empty(m, n, device="cuda")
    ctx.lowrank([A], [Q0], [U], [R], [V], [E])
    assert ctx.check() == cf.CF_OK
    Uh, Rh, Vh = (t.cpu().double().numpy() for t in (U, R, V))
    assert np.abs(Uh.T @ Uh - np.eye(r)).max() < 1e-4
    assert np.abs(Vh.T @ Vh - np.eye(r)).max() < 1e-4
    assert np.allclose(Rh, np.triu(Rh))
    rel = (torch.linalg.vector_norm(E) / torch.linalg.vector_norm(A)).item()
    assert rel < 1e-4, rel
    boundary = (1 << 31) // n
    W = Rh @ Vh.T
    for i in (0, boundary - 1, boundary, boundary + 1, m - 1):
        a = A[i].cpu().double().numpy()
        e = E[i].cpu().double().numpy()
        want = a - Uh[i] @ W
        assert np.abs(e - want).max() <= 1e-5 * np.abs(a).max() + 1e-6, i
    ctx.close()
