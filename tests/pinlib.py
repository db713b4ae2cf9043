"""Independent reference computations used only to pin the oracle.

None of these is the oracle's own code path: each one reaches the same
mathematical object by a different, textbook route.
"""
from __future__ import annotations

import numpy as np


def jacobi_eigh(A: np.ndarray, sweeps: int = 30, tol: float = 1e-15):
    """Cyclic Jacobi eigensolver for a symmetric matrix (Golub & Van Loan,
    Matrix Computations, the symmetric Schur 2x2 decomposition applied over
    all off-diagonal pairs).  Returns (eigenvalues descending, eigenvectors as
    columns)."""
    A = np.array(A, dtype=np.float64, copy=True)
    d = A.shape[0]
    V = np.eye(d)
    for _ in range(sweeps):
        off = np.sqrt(np.sum(A * A) - np.sum(np.diag(A) ** 2))
        if off <= tol * np.linalg.norm(A):
            break
        for p in range(d - 1):
            for q in range(p + 1, d):
                apq = A[p, q]
                if apq == 0.0:
                    continue
                with np.errstate(over="ignore"):          # a tiny apq: tau = inf, t = 0 below
                    tau = (A[q, q] - A[p, p]) / (2.0 * apq)
                if abs(tau) > 1e100:
                    t = 0.5 / tau
                else:
                    t = np.sign(tau) / (abs(tau) + np.sqrt(1.0 + tau * tau)) if tau != 0 else 1.0
                c = 1.0 / np.sqrt(1.0 + t * t)
                s = t * c
                # A <- J^T A J with J the rotation in the (p, q) plane
                ap = A[:, p].copy()
                aq = A[:, q].copy()
                A[:, p] = c * ap - s * aq
                A[:, q] = s * ap + c * aq
                ap = A[p, :].copy()
                aq = A[q, :].copy()
                A[p, :] = c * ap - s * aq
                A[q, :] = s * ap + c * aq
                vp = V[:, p].copy()
                vq = V[:, q].copy()
                V[:, p] = c * vp - s * vq
                V[:, q] = s * vp + c * vq
    lam = np.diag(A).copy()
    order = np.argsort(-lam)
    return lam[order], V[:, order]


def coupled_newton_inverse_root(A: np.ndarray, p: int, iters: int = 200,
                                tol: float = 1e-15) -> np.ndarray:
    """A^(-1/p) for symmetric positive definite A by the coupled Newton
    iteration that "Shampoo -- Second-Order Optimizer" describes in
    "Computing the inverse fourth root": scale so ||A|| <= 1, start from
    X = I, M = A, and repeat F = ((p+1) I - M)/p, X <- X F, M <- F^p M."""
    A = np.asarray(A, dtype=np.float64)
    d = A.shape[0]
    c = np.linalg.norm(A, 2)
    M = A / c
    X = np.eye(d)
    I = np.eye(d)
    for _ in range(iters):
        F = ((p + 1) * I - M) / p
        X = X @ F
        M = np.linalg.matrix_power(F, p) @ M
        if np.linalg.norm(M - I) < tol * np.sqrt(d):
            break
    return X * c ** (-1.0 / p)


def random_orthogonal(d: int, rng: np.random.Generator) -> np.ndarray:
    q, r = np.linalg.qr(rng.standard_normal((d, d)))
    return q * np.sign(np.diag(r))[None, :]


def spd_with_spectrum(lam, rng: np.random.Generator) -> np.ndarray:
    V = random_orthogonal(len(lam), rng)
    return (V * np.asarray(lam)[None, :]) @ V.T


def mgs_qr(Y: np.ndarray):
    """Q with orthonormal columns and R upper triangular with a positive
    diagonal such that Y = Q R, by modified Gram-Schmidt run twice over each
    column (Golub & Van Loan, Matrix Computations, "Modified Gram-Schmidt";
    the second sweep restores orthogonality lost to cancellation).  A route
    to the QR factor independent of LAPACK's Householder reflections."""
    Y = np.array(Y, dtype=np.float64, copy=True)
    d, k = Y.shape
    Q = np.zeros((d, k))
    R = np.zeros((k, k))
    for j in range(k):
        v = Y[:, j].copy()
        for _ in range(2):
            for i in range(j):
                c = Q[:, i] @ v
                R[i, j] += c
                v -= c * Q[:, i]
        R[j, j] = np.linalg.norm(v)
        Q[:, j] = v / R[j, j]
    return Q, R


def sylvester_hadamard(d: int) -> np.ndarray:
    """The d x d Sylvester-Hadamard matrix (d a power of two): entries +-1,
    H H^T = d I."""
    H = np.ones((1, 1))
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H
