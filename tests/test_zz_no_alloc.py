"""cf_lowrank_noalloc: the low-rank call for callers that cannot allocate.

Callers that must not call cudaMalloc (or any allocating routine, torch's
included) where they compress -- inside a pre-reserved pool, a plug-in that
only gets its tensors, a step that must not change the device's allocation
state -- use this entry point: no context, no workspace, its scratch is a
fixed 8 MiB device array in libcf.  Its results must equal those of the
regular cf_lowrank (the same kernels) within the low-rank tolerance, on two
calls in a row (the shared scratch keeps the previous call's contents), and
calls that do not fit the scratch are refused before anything is launched.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
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


def outputs(m, n, r, k):
    return ([torch.empty(m, r, device="cuda") for _ in range(k)], [torch.empty(r, r, device="cuda") for _ in range(k)],
            [torch.empty(n, r, device="cuda") for _ in range(k)], [torch.empty(m, n, device="cuda") for _ in range(k)])


def recon(U, R, V):
    return [(u.double() @ rr.double() @ v.double().T) for u, rr, v in zip(U, R, V)]


def rel(a, b):
    return (torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b)).item()


@pytest.mark.parametrize("m,n,r,T,k", [(4608, 3072, 16, 2, 2), (300, 200, 16, 2, 3), (320, 256, 32, 2, 2)])
def test_noalloc_matches_cf_lowrank_twice(cf, m, n, r, T, k):
    A = [synth.lowrank_matrix(m, n, r, mat=i, device="cuda") for i in range(k)]
    Q0 = [synth.q0(n, r, seed=0, mat=i, device="cuda") for i in range(k)]
    # the existing entry point, with a context and a caller workspace
    ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=T)
    ws = torch.empty(ctx.lowrank_workspace_bytes(k, m, n), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    U0, R0, V0, E0 = outputs(m, n, r, k)
    ctx.lowrank(A, Q0, U0, R0, V0, E0)
    assert ctx.check() == cf.CF_OK
    D0 = recon(U0, R0, V0)
    for call in range(2):
        U1, R1, V1, E1 = outputs(m, n, r, k)
        st = cf.cf_lowrank_noalloc(A, Q0, U1, R1, V1, E1, rank=r, iters=T)
        assert st == cf.CF_OK, (call, st)
        D1 = recon(U1, R1, V1)
        for i in range(k):
            assert rel(D1[i], D0[i]) <= TOL, (call, i)
            # E = A - D: same comparison, relative to the reconstruction
            dE = torch.linalg.vector_norm(E1[i].double() - E0[i].double()) / torch.linalg.vector_norm(D0[i])
            assert dE.item() <= TOL, (call, i)
    ctx.close()


def test_noalloc_refuses_calls_beyond_its_scratch(cf):
    m, n, r = 4608, 3072, 16
    k = 9                       # nine 4608 x 3072 matrices need more than 8 MiB
    A = [torch.zeros(m, n, device="cuda") for _ in range(k)]
    Q0 = [torch.zeros(n, r, device="cuda") for _ in range(k)]
    U, R, V, _ = outputs(m, n, r, k)
    assert cf.cf_lowrank_noalloc(A, Q0, U, R, V, rank=r, iters=2) == cf.CF_E_NOMEM
    # the refused call launched nothing: outputs untouched, and the next call works
    A2 = [synth.lowrank_matrix(256, 256, r, mat=5, device="cuda")]
    Q2 = [synth.q0(256, r, seed=0, mat=5, device="cuda")]
    U2, R2, V2, _ = outputs(256, 256, r, 1)
    assert cf.cf_lowrank_noalloc(A2, Q2, U2, R2, V2, rank=r, iters=2) == cf.CF_OK
    D = recon(U2, R2, V2)[0]
    assert rel(D, A2[0].double()) < 1e-2
