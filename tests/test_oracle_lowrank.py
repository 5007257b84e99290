"""Pins of the oracle's low-rank path (Algorithm 3, subspace iteration).

Source: "Accelerating Parallel Diffusion Model Serving with Residual
Compression" (arXiv 2507.17511), reproducibility table, "Pseudocode" row,
Algorithm 3: start from a random Q and orthonormalise it; T times form
Z = A^T A Q and orthonormalise; then U = A Q orthonormalised and V = Q.
The checks use closed forms (exact rank-r input), numpy's SVD and QR as
independent library routines, Eckart-Young, and orthogonality.
"""
import numpy as np
import pytest
import torch

import synth


def rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("rows,r", [(40, 1), (50, 4), (300, 16), (64, 32)])
def test_cholqr_matches_numpy_qr(oracle, rows, r):
    Z = rng(rows * 7 + r).standard_normal((rows, r))
    Q, R = oracle.cholqr(Z)
    assert np.allclose(np.triu(R), R)
    assert np.all(np.diag(R) > 0)
    assert np.allclose(Q @ R, Z, atol=1e-12 * np.abs(Z).max())
    assert np.abs(Q.T @ Q - np.eye(r)).max() < 1e-10
    Qn, Rn = np.linalg.qr(Z)
    sgn = np.sign(np.diag(Rn))
    assert np.allclose(Rn * sgn[:, None], R, rtol=1e-9, atol=1e-12)
    assert np.allclose(Qn * sgn[None, :], Q, rtol=1e-8, atol=1e-10)


def test_cholqr_rejects_rank_deficient(oracle):
    Z = np.zeros((10, 2))
    Z[:, 0] = 1.0   # second column is zero: the Gram matrix is singular
    with pytest.raises(ValueError):
        oracle.cholqr(Z)


@pytest.mark.parametrize("m,n,r,T", [(96, 64, 4, 1), (200, 120, 16, 2), (128, 256, 8, 1)])
def test_exact_rank_r_is_recovered(oracle, m, n, r, T):
    """A rank-r matrix is reproduced exactly (to 1e-5 relative Frobenius) by
    a rank-r subspace iteration once T >= 1: A^T A Q then spans A's row space."""
    A = synth.lowrank_matrix(m, n, r, mat=3, noise=0.0).numpy()
    Q0 = synth.q0(n, r, seed=0, mat=3).numpy()
    U, R, V = oracle.subspace_iteration(A, Q0, T)
    D, E, _ = oracle.lowrank_apply(A, U, R, V)
    rel = np.linalg.norm(D - A) / np.linalg.norm(A)
    assert rel <= 1e-5
    assert np.abs(U.T @ U - np.eye(r)).max() < 1e-6
    assert np.abs(V.T @ V - np.eye(r)).max() < 1e-6


@pytest.mark.parametrize("r", [1, 2, 3, 4])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_brute_force_8x8_converges_to_truncated_svd(oracle, r, seed):
    """With many iterations the reconstruction is the best rank-r
    approximation (Eckart-Young), computed here by numpy's SVD."""
    A = rng(seed).standard_normal((8, 8)).astype(np.float32)
    Ad = A.astype(np.float64)
    u, s, vt = np.linalg.svd(Ad)
    gap = s[r] / s[r - 1]
    T = int(np.ceil(np.log(1e-14) / (2 * np.log(gap)))) + 5 if gap < 1 else 50
    T = min(max(T, 5), 4000)
    Q0 = rng(seed + 100).standard_normal((8, r)).astype(np.float32)
    U, R, V = oracle.subspace_iteration(A, Q0, T)
    D, _, _ = oracle.lowrank_apply(A, U, R, V)
    Ar = (u[:, :r] * s[:r]) @ vt[:r]
    assert np.linalg.norm(D - Ar) <= 1e-9 * np.linalg.norm(Ar)
    # the retained energy equals the sum of the top r squared singular values
    assert abs(np.linalg.norm(D) ** 2 - (s[:r] ** 2).sum()) <= 1e-9 * (s ** 2).sum()


@pytest.mark.parametrize("T", [0, 1, 2, 3])
def test_eckart_young_lower_bound(oracle, T):
    """No rank-r reconstruction beats the truncated SVD; more iterations do
    not make the error larger on a matrix with a spectral gap."""
    m, n, r = 120, 80, 6
    A = synth.lowrank_matrix(m, n, r, mat=9, noise=0.05).numpy()
    u, s, vt = np.linalg.svd(A.astype(np.float64), full_matrices=False)
    best = np.sqrt((s[r:] ** 2).sum())
    Q0 = synth.q0(n, r, seed=0, mat=9).numpy()
    errs = []
    for t in range(T + 1):
        U, R, V = oracle.subspace_iteration(A, Q0, t)
        D, E, _ = oracle.lowrank_apply(A, U, R, V)
        errs.append(np.linalg.norm(E))
        assert errs[-1] >= best * (1 - 1e-12)
    assert errs[-1] <= errs[0] * (1 + 1e-12)


def test_zero_iterations_is_projection_on_start_block(oracle):
    """T = 0: V spans the start block and D = A V V^T (numpy QR of Q0)."""
    m, n, r = 60, 40, 5
    A = rng(4).standard_normal((m, n)).astype(np.float32)
    Q0 = rng(5).standard_normal((n, r)).astype(np.float32)
    U, R, V = oracle.subspace_iteration(A, Q0, 0)
    D, _, _ = oracle.lowrank_apply(A, U, R, V)
    Qn, _ = np.linalg.qr(Q0.astype(np.float64))
    Dn = A.astype(np.float64) @ Qn @ Qn.T
    assert np.allclose(D, Dn, rtol=1e-10, atol=1e-10)


def test_apply_outputs(oracle):
    m, n, r = 33, 21, 3
    A = rng(6).standard_normal((m, n)).astype(np.float32)
    Q0 = rng(7).standard_normal((n, r)).astype(np.float32)
    U, R, V = oracle.subspace_iteration(A, Q0, 2)
    C = rng(8).standard_normal((m, n)).astype(np.float32)
    D, E, Cout = oracle.lowrank_apply(A, U, R, V, C)
    Dn = U @ R @ V.T
    assert np.allclose(D, Dn, rtol=1e-12, atol=1e-12)
    assert np.allclose(E, A.astype(np.float64) - Dn, rtol=1e-12, atol=1e-12)
    assert np.allclose(Cout, C.astype(np.float64) + Dn, rtol=1e-12, atol=1e-12)
    # P = A Q = U R with V = Q
    assert np.allclose(U @ R, A.astype(np.float64) @ V, rtol=1e-10, atol=1e-10)


def test_lowrank_workload_recovers_signal(oracle):
    """On the low-rank workload's recipe (rank-16 signal with 1/k singular
    values plus 0.01 noise), r = 16, T = 2 leaves only about the noise."""
    m, n, r = 576, 384, 16
    A = synth.lowrank_matrix(m, n, r, mat=0, noise=0.01).numpy()
    Q0 = synth.q0(n, r, seed=0, mat=0).numpy()
    U, R, V = oracle.subspace_iteration(A, Q0, 2)
    D, E, _ = oracle.lowrank_apply(A, U, R, V)
    noise = 0.01 * np.sqrt(m * n)
    assert np.linalg.norm(E) <= 1.05 * noise
    S = synth.lowrank_matrix(m, n, r, mat=0, noise=0.0).numpy().astype(np.float64)
    assert np.linalg.norm(D - S) <= 1e-2 * np.linalg.norm(S)
