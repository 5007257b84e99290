"""cf_lowrank_noalloc: the low-rank call for callers that cannot allocate.

Callers that must not call cudaMalloc (or any allocating routine, torch's
included) where they compress -- inside a pre-reserved pool, a plug-in that
only gets its tensors, a step that must not change the device's allocation
state -- use this entry point: no context, no workspace, its scratch is a
fixed 8 MiB device array in libcf.  Its results must match the CPU oracle's
Algorithm 3 (D = U R V^T, E = A - D and C + D within the low-rank tolerance)
on two calls in a row, since the shared scratch keeps the previous call's
contents; a call after a larger one must not see that call's leftovers; and
calls that do not fit the scratch, or hand over memory the GPU cannot use,
are refused before anything is launched.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

TOL = 1e-3


@pytest.fixture(scope="module")
def cf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_residual_compression_02_b200 as m

    m.lib()
    return m


def outputs(m, n, r, k):
    return ([torch.empty(m, r, device="cuda") for _ in range(k)], [torch.empty(r, r, device="cuda") for _ in range(k)],
            [torch.empty(n, r, device="cuda") for _ in range(k)], [torch.empty(m, n, device="cuda") for _ in range(k)])


def rel(a, b, ref):
    return float(np.linalg.norm(a - b) / np.linalg.norm(ref))


def oracle_results(oracle, A, Q0, C0, T):
    """The oracle's D, E and C (fp64) for each matrix."""
    out = []
    for a, q, c in zip(A, Q0, C0):
        an = a.cpu().numpy()
        Uo, Ro, Vo = oracle.subspace_iteration(an, q.cpu().numpy(), T)
        out.append(oracle.lowrank_apply(an, Uo, Ro, Vo, c.cpu().numpy()))
    return out


def check_against_oracle(U, R, V, E, C, ref, tag):
    for i, (Do, Eo, Co) in enumerate(ref):
        u, rr, v = (t.cpu().double().numpy() for t in (U[i], R[i], V[i]))
        D = u @ rr @ v.T
        assert rel(D, Do, Do) <= TOL, (tag, i, rel(D, Do, Do))
        assert rel(E[i].cpu().double().numpy(), Eo, Do) <= TOL, (tag, i, "E")
        assert rel(C[i].cpu().double().numpy(), Co, Do) <= TOL, (tag, i, "C")
        r = u.shape[1]
        assert np.abs(u.T @ u - np.eye(r)).max() < 1e-4, (tag, i, "U orthonormal")
        assert np.abs(v.T @ v - np.eye(r)).max() < 1e-4, (tag, i, "V orthonormal")


def case(m, n, r, k, seed):
    A = [synth.lowrank_matrix(m, n, r, mat=i, seed=seed, device="cuda") for i in range(k)]
    Q0 = [synth.q0(n, r, seed=seed, mat=i, device="cuda") for i in range(k)]
    C0 = [torch.randn(m, n, generator=torch.Generator().manual_seed(100 + i)).cuda() for i in range(k)]
    return A, Q0, C0


@pytest.mark.gpu
@pytest.mark.parametrize("m,n,r,T,k", [(4608, 3072, 16, 2, 2), (300, 200, 16, 2, 3), (320, 256, 32, 2, 2),
                                       (130, 64, 8, 1, 2)])
def test_noalloc_matches_the_oracle_twice(cf, oracle, m, n, r, T, k):
    A, Q0, C0 = case(m, n, r, k, seed=0)
    ref = oracle_results(oracle, A, Q0, C0, T)
    for call in range(2):
        U, R, V, E = outputs(m, n, r, k)
        C = [c.clone() for c in C0]
        st = cf.cf_lowrank_noalloc(A, Q0, U, R, V, E, C, rank=r, iters=T)
        assert st == cf.CF_OK, (call, st)
        check_against_oracle(U, R, V, E, C, ref, call)


@pytest.mark.gpu
def test_noalloc_after_a_larger_call(cf, oracle):
    """The scratch keeps a larger call's buffers; a smaller call after it
    (another rank, shape and count) must still match the oracle."""
    A, Q0, C0 = case(4608, 3072, 16, 4, seed=3)
    U, R, V, E = outputs(4608, 3072, 16, 4)
    assert cf.cf_lowrank_noalloc(A, Q0, U, R, V, E, [c.clone() for c in C0], rank=16, iters=2) == cf.CF_OK
    m, n, r, T, k = 200, 96, 24, 1, 3
    A, Q0, C0 = case(m, n, r, k, seed=4)
    ref = oracle_results(oracle, A, Q0, C0, T)
    U, R, V, E = outputs(m, n, r, k)
    C = [c.clone() for c in C0]
    assert cf.cf_lowrank_noalloc(A, Q0, U, R, V, E, C, rank=r, iters=T) == cf.CF_OK
    check_against_oracle(U, R, V, E, C, ref, "after a larger call")


@pytest.mark.gpu
def test_noalloc_refuses_calls_beyond_its_scratch(cf):
    m, n, r = 4608, 3072, 16
    k = 9                       # nine 4608 x 3072 matrices need more than 8 MiB
    A = [torch.zeros(m, n, device="cuda") for _ in range(k)]
    Q0 = [torch.zeros(n, r, device="cuda") for _ in range(k)]
    U, R, V, E = outputs(m, n, r, k)
    C = [torch.empty(m, n, device="cuda") for _ in range(k)]
    sentinel = 12345.0
    for t in U + R + V + E + C:
        t.fill_(sentinel)
    assert cf.cf_lowrank_noalloc(A, Q0, U, R, V, E, C, rank=r, iters=2) == cf.CF_E_NOMEM
    torch.cuda.synchronize()
    # the refused call launched nothing: every output still holds the sentinel
    for t in U + R + V + E + C:
        assert bool(torch.all(t == sentinel))
    # and the next call works
    A2 = [synth.lowrank_matrix(256, 256, r, mat=5, device="cuda")]
    Q2 = [synth.q0(256, r, seed=0, mat=5, device="cuda")]
    U2, R2, V2, _ = outputs(256, 256, r, 1)
    assert cf.cf_lowrank_noalloc(A2, Q2, U2, R2, V2, rank=r, iters=2) == cf.CF_OK
    D = U2[0].double() @ R2[0].double() @ V2[0].double().T
    assert (torch.linalg.vector_norm(D - A2[0].double()) / torch.linalg.vector_norm(A2[0].double())).item() < 1e-2


@pytest.mark.gpu
def test_noalloc_refuses_memory_the_gpu_cannot_use(cf):
    """A host pointer among the arguments is refused (CF_E_ARG) before any
    launch: the outputs that are device memory keep their contents."""
    m, n, r = 128, 64, 8
    A, Q0, _ = case(m, n, r, 1, seed=7)
    U, R, V, _ = outputs(m, n, r, 1)
    for t in U + R + V:
        t.fill_(7.0)
    host = np.zeros(n * r, np.float32)        # pageable host memory, 16-byte aligned by numpy
    assert host.ctypes.data % 16 == 0
    L = cf.lib()
    cfg = cf.cf_config(cf.CF_MODE_LOWRANK, 0, 0, 0, r, 1, 0, 0, 0)

    def arr(*ptrs):
        return (ctypes.c_void_p * len(ptrs))(*ptrs)

    st = L.cf_lowrank_noalloc(ctypes.byref(cfg), 1, m, n, arr(A[0].data_ptr()), arr(Q0[0].data_ptr()),
                              arr(U[0].data_ptr()), arr(R[0].data_ptr()), arr(host.ctypes.data), None, None,
                              torch.cuda.current_stream().cuda_stream)
    assert st == cf.CF_E_ARG
    torch.cuda.synchronize()
    assert np.all(host == 0.0)
    for t in U + R + V:
        assert bool(torch.all(t == 7.0))


@pytest.mark.gpu
def test_noalloc_repeated_call_reserves_no_device_memory(cf):
    """After a first call on the device (which may load libcf's device code,
    and the scratch with it), a repeated call leaves the device's free memory
    unchanged."""
    m, n, r, T, k = 640, 512, 16, 2, 2
    A, Q0, C0 = case(m, n, r, k, seed=9)
    U, R, V, E = outputs(m, n, r, k)
    C = [c.clone() for c in C0]
    assert cf.cf_lowrank_noalloc(A, Q0, U, R, V, E, C, rank=r, iters=T) == cf.CF_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert cf.cf_lowrank_noalloc(A, Q0, U, R, V, E, C, rank=r, iters=T) == cf.CF_OK
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_binding_checks_tensors_before_the_call():
    """dtype and shape errors are refused by the binding before anything
    reaches libcf (CPU tensors suffice: the check comes first)."""
    from activation_residual_compression_02_b200 import _cf

    m, n, r = 64, 32, 8
    A = [torch.zeros(m, n)]
    Q0 = [torch.zeros(n, r)]
    U, R, V = [torch.zeros(m, r)], [torch.zeros(r, r)], [torch.zeros(n, r)]
    with pytest.raises(ValueError, match="float32"):
        _cf.cf_lowrank_noalloc([A[0].double()], Q0, U, R, V, rank=r)
    with pytest.raises(ValueError, match="shape"):
        _cf.cf_lowrank_noalloc(A, Q0, [torch.zeros(m, r + 1)], R, V, rank=r)
    with pytest.raises(ValueError, match="shape"):
        _cf.cf_lowrank_noalloc(A, [torch.zeros(n, r)], U, R, V, rank=r + 8)
    with pytest.raises(ValueError, match="tensors"):
        _cf.cf_lowrank_noalloc(A, Q0 * 2, U, R, V, rank=r)
