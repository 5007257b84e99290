"""GPU parity of the low-rank path (Algorithm 3) against the fp64 CPU oracle.

The factors (U, R, V) are unique only up to rotations within the subspace, so
the comparison is on what is unique: the reconstruction D = U R V^T, the new
error E = A - D and the updated cache C + D, each within 1e-3 relative
Frobenius of the oracle's (the tolerance of the low-rank path; TF32 operands
rounded to nearest give about 3e-5 on the low-rank workload).  U and V must
also be orthonormal.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
TOL = 1e-3


@pytest.fixture(scope="module")
def cf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_residual_compression_02_b200 as m

    m.lib()
    return m


def run_gpu(cf, As, Q0s, r, T, with_e=True, with_c=True, precision=0):
    m, n = As[0].shape
    ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=T, precision=precision)
    ws = torch.empty(ctx.lowrank_workspace_bytes(len(As), m, n), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    A = [a.cuda() for a in As]
    Q0 = [q.cuda() for q in Q0s]
    U = [torch.empty(m, r, device="cuda") for _ in As]
    R = [torch.empty(r, r, device="cuda") for _ in As]
    V = [torch.empty(n, r, device="cuda") for _ in As]
    E = [torch.empty(m, n, device="cuda") for _ in As] if with_e else None
    C0 = [torch.randn(m, n, generator=torch.Generator().manual_seed(i)) for i in range(len(As))] if with_c else None
    C = [c.cuda() for c in C0] if with_c else None
    ctx.lowrank(A, Q0, U, R, V, E, C)
    st = ctx.check()
    assert st == cf.CF_OK, st
    out = dict(U=[u.cpu().double().numpy() for u in U], R=[x.cpu().double().numpy() for x in R],
               V=[v.cpu().double().numpy() for v in V])
    if with_e:
        out["E"] = [e.cpu().double().numpy() for e in E]
    if with_c:
        out["C"] = [c.cpu().double().numpy() for c in C]
        out["C0"] = [c.numpy() for c in C0]
    ctx.close()
    return out


def rel(a, b, ref):
    return np.linalg.norm(a - b) / np.linalg.norm(ref)


def check(oracle, As, Q0s, out, T, idx=None):
    idx = range(len(As)) if idx is None else idx
    for i in idx:
        A = As[i].numpy()
        Uo, Ro, Vo = oracle.subspace_iteration(A, Q0s[i].numpy(), T)
        C0 = out["C0"][i] if "C0" in out else None
        Do, Eo, Co = oracle.lowrank_apply(A, Uo, Ro, Vo, C0)
        U, R, V = out["U"][i], out["R"][i], out["V"][i]
        r = U.shape[1]
        Dg = U @ R @ V.T
        assert rel(Dg, Do, Do) <= TOL, (i, rel(Dg, Do, Do))
        assert np.abs(U.T @ U - np.eye(r)).max() < 1e-4
        assert np.abs(V.T @ V - np.eye(r)).max() < 1e-4
        assert np.allclose(R, np.triu(R))
        if "E" in out:
            assert rel(out["E"][i], Eo, Do) <= TOL, i
        if "C" in out:
            assert rel(out["C"][i], Co, Do) <= TOL, i


# Ragged shapes in both dimensions (m and n not multiples of the 128-row
# tile or the 32-column box), full-width rows (n = 3072) and wider (3200),
# r from 1 to 32 (padded to 16 or 32 columns), T from 0 to 4, all within the
# 1e-3 bar.  Tall blocks (m = 8320, 8200) give the CholeskyQR of P 33 Gram
# chunks per matrix.  Where Algorithm 3 is still far from converged (r a large
# fraction of the smaller dimension with few iterations, e.g. 192 x 128 at
# r = 32, T = 2) the result follows every rounding of the products: TF32
# operands gave 1.6e-3 there in a CPU simulation of the kernels, so the
# automatic precision runs such calls with split (3xTF32) products.
@pytest.mark.parametrize("m,n,r,T", [(256, 256, 16, 2), (300, 200, 16, 2), (4444 // 4, 1920 // 4, 16, 2),
                                     (200, 72, 8, 2), (160, 96, 24, 1), (320, 256, 32, 2), (192, 128, 32, 4),
                                     (192, 128, 32, 2), (130, 64, 16, 0), (128, 128, 1, 3), (700, 1000, 16, 2),
                                     (300, 3072, 16, 2), (256, 3200, 8, 1), (8320, 256, 16, 1), (8200, 96, 24, 1)])
def test_lowrank_matches_oracle(cf, oracle, m, n, r, T):
    k = 3
    As = [synth.lowrank_matrix(m, n, r, mat=i, noise=0.01) for i in range(k)]
    Q0s = [synth.q0(n, r, seed=0, mat=i) for i in range(k)]
    out = run_gpu(cf, As, Q0s, r, T)
    check(oracle, As, Q0s, out, T)


# Shapes smaller than one tile or one TMA box in one or both dimensions, and
# the degenerate ranks: r == n (Q spans every column: D = A) and r == m (U is
# square).
@pytest.mark.parametrize("m,n,r,T", [(17, 20, 4, 2), (33, 36, 16, 1), (1000, 16, 16, 1), (16, 1000, 16, 2),
                                     (129, 8, 8, 1)])
def test_lowrank_small_and_degenerate_shapes(cf, oracle, m, n, r, T):
    k = 3
    As = [synth.lowrank_matrix(m, n, r, mat=i, noise=0.01) for i in range(k)]
    Q0s = [synth.q0(n, r, seed=0, mat=i) for i in range(k)]
    out = run_gpu(cf, As, Q0s, r, T)
    check(oracle, As, Q0s, out, T)


@pytest.mark.parametrize("k,m,n,r,T", [(8, 1024, 3072, 16, 2), (80, 1000, 128, 8, 1)])
def test_lowrank_many_tiles_and_matrices(cf, oracle, k, m, n, r, T):
    """Many matrices of many 128-row tiles in one call: the persistent GEMM
    walks tiles across matrix boundaries and its pipeline wraps around many
    times (8 x 1024 x 3072), and 80 matrices of ragged 1000-row tiles."""
    As = [synth.lowrank_matrix(m, n, r, mat=40 + i, noise=0.01) for i in range(k)]
    Q0s = [synth.q0(n, r, seed=0, mat=40 + i) for i in range(k)]
    out = run_gpu(cf, As, Q0s, r, T)
    check(oracle, As, Q0s, out, T, idx=[0, k // 2 + 1, k - 1])


def test_lowrank_is_deterministic(cf):
    """Every sum of the path runs in a fixed order (the GEMM's K loop, the
    CholeskyQR Gram chunks summed in chunk order, no atomics): two calls on
    the same inputs give bit-identical factors and error buffers."""
    m, n, r, T, k = 1152, 3072, 16, 2, 5
    As = [synth.lowrank_matrix(m, n, r, mat=30 + i, noise=0.01) for i in range(k)]
    Q0s = [synth.q0(n, r, seed=0, mat=30 + i) for i in range(k)]
    a = run_gpu(cf, As, Q0s, r, T, with_c=False)
    b = run_gpu(cf, As, Q0s, r, T, with_c=False)
    for key in ("U", "R", "V", "E"):
        for i in range(k):
            assert np.array_equal(a[key][i], b[key][i]), (key, i)


def test_lowrank_many_matrices_chunked(cf, oracle):
    """More matrices than one launch's parameter table holds (160 for the
    GEMM, 192 for CholeskyQR and the apply)."""
    m, n, r, T = 128, 96, 8, 2
    k = 200
    As = [synth.lowrank_matrix(m, n, r, mat=i, noise=0.01) for i in range(k)]
    Q0s = [synth.q0(n, r, seed=0, mat=i) for i in range(k)]
    out = run_gpu(cf, As, Q0s, r, T, with_c=False)
    check(oracle, As, Q0s, out, T, idx=[0, 159, 160, 191, 192, 199])


def test_lowrank_exact_rank_recovered(cf):
    """An exactly rank-r matrix is reconstructed to TF32 accuracy."""
    m, n, r = 512, 384, 16
    As = [synth.lowrank_matrix(m, n, r, mat=7, noise=0.0)]
    Q0s = [synth.q0(n, r, seed=0, mat=7)]
    out = run_gpu(cf, As, Q0s, r, 2, with_c=False)
    D = out["U"][0] @ out["R"][0] @ out["V"][0].T
    A = As[0].double().numpy()
    assert np.linalg.norm(D - A) / np.linalg.norm(A) < 1e-4


def test_lowrank_full_size_sampled(cf, oracle):
    """The low-rank workload at full size (57 x 4608 x 3072, r = 16, T = 2) in
    one call; the oracle re-runs three of the matrices."""
    w = synth.LOWRANK
    m, n, r = w.rows, w.cols, w.rank
    ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=w.iters)
    ws = torch.empty(ctx.lowrank_workspace_bytes(w.slots, m, n), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    A = [synth.lowrank_matrix(m, n, r, mat=i, device="cuda") for i in range(w.slots)]
    Q0 = [synth.q0(n, r, seed=0, mat=i, device="cuda") for i in range(w.slots)]
    U = [torch.empty(m, r, device="cuda") for _ in A]
    R = [torch.empty(r, r, device="cuda") for _ in A]
    V = [torch.empty(n, r, device="cuda") for _ in A]
    E = [torch.empty(m, n, device="cuda") for _ in A]
    ctx.lowrank(A, Q0, U, R, V, E)
    assert ctx.check() == cf.CF_OK
    for i in (0, w.slots // 2, w.slots - 1):
        Ah = A[i].cpu().numpy()
        Uo, Ro, Vo = oracle.subspace_iteration(Ah, Q0[i].cpu().numpy(), w.iters)
        Do, Eo, _ = oracle.lowrank_apply(Ah, Uo, Ro, Vo)
        Dg = U[i].cpu().double().numpy() @ R[i].cpu().double().numpy() @ V[i].cpu().double().numpy().T
        assert rel(Dg, Do, Do) <= TOL
        assert rel(E[i].cpu().double().numpy(), Eo, Do) <= TOL
    ctx.close()


def test_lowrank_mode_through_slots(cf, oracle):
    """cf_compress / cf_decompress in low-rank mode: residual + error feedback
    into Algorithm 3, E and the receiver cache updated, base advanced.  The
    oracle runs its own chain (its own fp32 E carried between steps); the two
    chains agree within the low-rank tolerance at every step.  The receiver
    also writes the bf16 reconstruction: torch's round-to-nearest-even cast of
    the cache it wrote, and within the tolerance plus one bf16 rounding
    (2^-8 relative) of the oracle's cache."""
    rows, cols, r, T = 192, 256, 16, 2
    shapes = [(rows, cols), (rows, cols)]
    ctx = cf.Context(shapes, mode=cf.CF_MODE_LOWRANK, rank=r, iters=T)
    ws = torch.empty(max(ctx.workspace_bytes(), 16), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    # activations whose step-wise change is (nearly) rank r, so that the
    # rank-r payload captures the residual and the comparison is well posed
    xs = []
    for i in range(2):
        x = synth.gaussian((rows, cols), 0, i, 99)
        seq = [x.to(torch.bfloat16)]
        for t in range(1, 3):
            L = synth.lowrank_matrix(rows, cols, r, mat=100 * i + t, noise=0.0)
            x = seq[-1].float() + 0.5 * L / L.pow(2).mean().sqrt()
            seq.append(x.to(torch.bfloat16))
        xs.append(seq)
    base = [torch.empty(rows * cols, dtype=torch.bfloat16, device="cuda") for _ in shapes]
    err = [torch.empty(rows * cols, device="cuda") for _ in shapes]
    cache = [torch.empty(rows * cols, device="cuda") for _ in shapes]
    U = [torch.empty(rows, r, device="cuda") for _ in shapes]
    R = [torch.empty(r, r, device="cuda") for _ in shapes]
    V = [torch.empty(cols, r, device="cuda") for _ in shapes]
    recon = [torch.empty(rows * cols, dtype=torch.bfloat16, device="cuda") for _ in shapes]
    ob = [None, None]
    oe = [None, None]
    oc = [None, None]
    for t in range(3):
        q0 = [synth.q0(cols, r, seed=0, mat=i, call=t) for i in range(2)]
        slots = [cf.Slot(x=xs[i][t].reshape(-1).cuda(), base=base[i], err=err[i], cache=cache[i], q0=q0[i].cuda(),
                         U=U[i], R=R[i], V=V[i], recon=recon[i]) for i in range(2)]
        ctx.compress(slots, t)
        ctx.decompress(slots, t)
        for i in range(2):
            xb = xs[i][t].view(torch.int16).numpy().view(np.uint16).ravel().copy()
            if t == 0:
                ob[i], oe[i] = oracle.warmup_sender(xb)
                oc[i] = oracle.warmup_receiver(xb).astype(np.float64)
                continue
            a = oracle.residual(xb, ob[i], oe[i]).reshape(rows, cols)
            Uo, Ro, Vo = oracle.subspace_iteration(a, q0[i].numpy(), T)
            Do, Eo, _ = oracle.lowrank_apply(a, Uo, Ro, Vo)
            torch.cuda.synchronize()
            eg = err[i].cpu().double().numpy().reshape(rows, cols)
            assert rel(eg, Eo, Do) <= TOL, (t, i)
            oc[i] = oc[i] + Do.ravel()
            assert rel(cache[i].cpu().double().numpy(), oc[i], Do) <= TOL, (t, i)
            assert np.array_equal(base[i].view(torch.int16).cpu().numpy().view(np.uint16), xb)
            cg = cache[i].cpu()
            assert torch.equal(recon[i].cpu(), cg.to(torch.bfloat16)), (t, i)
            assert rel(recon[i].cpu().double().numpy(), oc[i], oc[i]) <= TOL + 2.0 ** -8, (t, i)
            oe[i] = Eo.ravel().astype(np.float32)     # the oracle's E buffer is fp32, as the codec's
    assert ctx.check() == cf.CF_OK
    for i in range(2):
        x = xs[i][2].float().reshape(-1).cuda()
        assert (torch.linalg.vector_norm(cache[i] + err[i] - x) / torch.linalg.vector_norm(x)).item() < 1e-5


def test_lowrank_warm_start_through_slots(cf, oracle):
    """warm_start: from the second compressed step on, Algorithm 3 starts from
    the previous step's V (T = 1 here).  The oracle runs the same warm-started
    chain from its own V and E (both kept in fp32, as the codec keeps them);
    every step agrees within the tolerance, and the error feedback keeps
    C + E = X."""
    rows, cols, r, T = 192, 256, 16, 1
    shapes = [(rows, cols)]
    ctx = cf.Context(shapes, mode=cf.CF_MODE_LOWRANK, rank=r, iters=T, warm_start=1)
    ws = torch.empty(max(ctx.workspace_bytes(), 16), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    x = synth.gaussian((rows, cols), 0, 7, 99)
    # a slowly rotating rank-r increment: the subspace moves a little per step
    Ub = synth.gaussian((rows, r), 0, 7, 98)
    Vb = synth.gaussian((cols, r), 0, 7, 97)
    seq = [x.to(torch.bfloat16)]
    for t in range(1, 6):
        Ut = Ub + 0.05 * t * synth.gaussian((rows, r), 0, 7, t)
        Vt = Vb + 0.05 * t * synth.gaussian((cols, r), 0, 7, 100 + t)
        L = (Ut * (1.0 / torch.arange(1, r + 1))) @ Vt.T
        seq.append((seq[-1].float() + 0.5 * L / L.pow(2).mean().sqrt()).to(torch.bfloat16))
    base = torch.empty(rows * cols, dtype=torch.bfloat16, device="cuda")
    err = torch.empty(rows * cols, device="cuda")
    cache = torch.empty(rows * cols, device="cuda")
    U, R, V = torch.empty(rows, r, device="cuda"), torch.empty(r, r, device="cuda"), torch.empty(cols, r, device="cuda")
    q0 = synth.q0(cols, r, seed=0, mat=7).cuda()
    ob = oe = ov = None
    for t, xt in enumerate(seq):
        start = q0.cpu().numpy() if t <= 1 else ov
        slot = cf.Slot(x=xt.reshape(-1).cuda(), base=base, err=err, cache=cache, q0=q0 if t <= 1 else None,
                       U=U, R=R, V=V)
        ctx.compress([slot], t)
        ctx.decompress([slot], t)
        xb = xt.view(torch.int16).numpy().view(np.uint16).ravel().copy()
        if t == 0:
            ob, oe = oracle.warmup_sender(xb)
            continue
        a = oracle.residual(xb, ob, oe).reshape(rows, cols)
        Uo, Ro, Vo = oracle.subspace_iteration(a, start, T)
        Do, Eo, _ = oracle.lowrank_apply(a, Uo, Ro, Vo)
        torch.cuda.synchronize()
        eg = err.cpu().double().numpy().reshape(rows, cols)
        assert rel(eg, Eo, Do) <= TOL, t
        oe = Eo.ravel().astype(np.float32)
        ov = Vo.astype(np.float32)
    assert ctx.check() == cf.CF_OK
    xl = seq[-1].float().reshape(-1).cuda()
    assert (torch.linalg.vector_norm(cache + err - xl) / torch.linalg.vector_norm(xl)).item() < 1e-5


def test_lowrank_mode_without_workspace_is_refused(cf):
    """Low-rank mode cf_compress needs the caller's workspace for the fp32
    residuals and the Algorithm 3 blocks: without one, or with one that is too
    small, the call returns CF_E_NOMEM before anything is launched (the
    warmup step needs none), and the slot buffers keep their contents."""
    rows, cols, r = 128, 64, 8
    ctx = cf.Context([(rows, cols)], mode=cf.CF_MODE_LOWRANK, rank=r, iters=1)
    x = synth.gaussian((rows, cols), 0, 0, 5).to(torch.bfloat16).reshape(-1).cuda()
    base = torch.empty(rows * cols, dtype=torch.bfloat16, device="cuda")
    err = torch.empty(rows * cols, device="cuda")
    cache = torch.empty(rows * cols, device="cuda")
    U, R, V = torch.full((rows, r), 3.0, device="cuda"), torch.full((r, r), 3.0, device="cuda"), \
        torch.full((cols, r), 3.0, device="cuda")
    q0 = synth.q0(cols, r, seed=0, mat=0).cuda()
    slots = [cf.Slot(x=x, base=base, err=err, cache=cache, q0=q0, U=U, R=R, V=V)]
    ctx.compress(slots, 0)
    ctx.decompress(slots, 0)
    torch.cuda.synchronize()
    e0 = err.clone()
    with pytest.raises(cf.CfError) as e:
        ctx.compress(slots, 1)
    assert e.value.status == cf.CF_E_NOMEM
    small = torch.empty(ctx.workspace_bytes() - 256, dtype=torch.uint8, device="cuda")
    ctx.set_workspace(small)
    with pytest.raises(cf.CfError) as e:
        ctx.compress(slots, 1)
    assert e.value.status == cf.CF_E_NOMEM
    torch.cuda.synchronize()
    assert torch.equal(err, e0)
    for t in (U, R, V):
        assert bool(torch.all(t == 3.0))
    assert ctx.check() == cf.CF_OK


@pytest.mark.parametrize("m,n,r,T", [(192, 128, 32, 2), (300, 200, 16, 2), (700, 1000, 16, 2), (1152, 3072, 16, 2),
                                     (160, 96, 24, 1), (17, 20, 4, 2)])
def test_lowrank_split_products_near_fp32(cf, oracle, m, n, r, T):
    """The split (3xTF32) products, forced: D, E and C within 5e-5 of the
    fp64 oracle -- the ill-conditioned 192 x 128, r = 32, T = 2 case
    included -- where TF32 operands alone are held to 1e-3; both pipeline
    shapes (r <= 16 and r <= 32), ragged tiles and a sub-tile matrix."""
    k = 3
    As = [synth.lowrank_matrix(m, n, r, mat=i, noise=0.01) for i in range(k)]
    Q0s = [synth.q0(n, r, seed=0, mat=i) for i in range(k)]
    out = run_gpu(cf, As, Q0s, r, T, precision=cf.CF_PRECISION_SPLIT)
    for i in range(k):
        A = As[i].numpy()
        Uo, Ro, Vo = oracle.subspace_iteration(A, Q0s[i].numpy(), T)
        Do, Eo, Co = oracle.lowrank_apply(A, Uo, Ro, Vo, out["C0"][i])
        Dg = out["U"][i] @ out["R"][i] @ out["V"][i].T
        assert rel(Dg, Do, Do) <= 5e-5, (i, rel(Dg, Do, Do))
        assert rel(out["E"][i], Eo, Do) <= 5e-5, i
        assert rel(out["C"][i], Co, Do) <= 5e-5, i


def test_lowrank_precision_is_validated(cf):
    with pytest.raises(cf.CfError) as e:
        cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=16, iters=2, precision=3)
    assert e.value.status == cf.CF_E_ARG
    with pytest.raises(cf.CfError) as e:
        cf.Context([(8, 128)], bits=2, group=128, precision=cf.CF_PRECISION_SPLIT)
    assert e.value.status == cf.CF_E_ARG
    # the split form needs the lo blocks of Q^T and P^T as well
    a = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=16, iters=2, precision=cf.CF_PRECISION_TF32)
    b = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=16, iters=2, precision=cf.CF_PRECISION_SPLIT)
    assert b.lowrank_workspace_bytes(3, 1000, 512) > a.lowrank_workspace_bytes(3, 1000, 512)
