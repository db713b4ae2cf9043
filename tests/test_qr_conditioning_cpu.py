"""Which refreshes the fp32-accurate Cholesky-QR can orthogonalize.

The library runs the QR of a refresh, Y = (S + eps I) U, as shifted
Cholesky-QR passes in fp32-accurate arithmetic on the tensor cores, and
redoes a factor in fp64 when a pass breaks down.  On the single 1024 x 1024
layer with a rank-16 term ("4-bit Shampoo for Memory-Efficient Network
Training", the eigenvector-refresh step of its algorithm), lambda_max / eps
is near 4e8.

This module emulates those passes on the oracle's own Y (the Gram of the
fp32 operands rounded once to fp32, an exact diagonal, the first pass's
shift of 1e-5 d in the column-equilibrated frame, Cholesky in fp64, L and
the solve in fp32).  It pins the reading recorded for the fallback:
- the cold first refresh (U = I, Y = S + eps I) breaks down in pass 2 and
  needs the fp64 passes;
- a warm refresh (U from the previous refresh's 4-bit codes, rectified by
  Bjorck) is far better conditioned in the equilibrated frame, and two
  passes reach the orthogonality floor.

The emulation is optimistic about the Gram (exact products, rounded once),
so a breakdown here is a breakdown on the device too.
"""
import numpy as np
import pytest

from bit_quantized_shampoo_b200 import workloads as W
from oracle import shampoo4_oracle as O


def _r32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def _orth(Q):
    d = Q.shape[1]
    return np.linalg.norm(Q.T @ Q - np.eye(d)) / np.sqrt(d)


def _pass(X, shift):
    """One Cholesky-QR pass in the emulated arithmetic; None on a breakdown."""
    d = X.shape[1]
    Wm = _r32(X.T @ X)
    np.fill_diagonal(Wm, _r32((X * X).sum(0)))
    if shift:
        Wm[np.diag_indices(d)] *= 1.0 + shift
    try:
        L = np.linalg.cholesky(Wm)
    except np.linalg.LinAlgError:
        return None
    return _r32(np.linalg.solve(_r32(L), X.T).T)


def _two_passes(Y):
    d = Y.shape[1]
    X = _r32(Y)
    out = []
    for shift in (1e-5 * d, 0.0):
        X = _pass(X, shift)
        if X is None:
            out.append(None)
            break
        out.append(_orth(X))
    return out


@pytest.fixture(scope="module")
def lowrank_layer():
    w = W.WORKLOADS[2]
    orc = O.Shampoo4Oracle(list(w.shapes), beta=w.beta, eps=w.eps, bjorck_iters=w.bjorck_iters)
    orc.update_stats(W.gradients(w, 1))
    f = orc.factors[0]
    cold_Y = f.S.astype(np.float64) + w.eps * np.eye(f.d)
    lam_ratio = np.linalg.eigvalsh(f.S.astype(np.float64))[-1] / w.eps
    orc.refresh_roots()                                   # the cold refresh, in fp64
    for step in range(2, 12):
        orc.update_stats(W.gradients(w, step))
    U = O.dequantize(f.codes, f.scales, f.d * f.d).reshape(f.d, f.d).astype(np.float64)
    U = O.bjorck(U, w.bjorck_iters)
    warm_Y = f.S.astype(np.float64) @ U + w.eps * U
    return lam_ratio, cold_Y, warm_Y


def test_cold_refresh_of_the_lowrank_layer_breaks_down_in_fp32(lowrank_layer):
    lam_ratio, cold_Y, _ = lowrank_layer
    assert lam_ratio > 1e7
    res = _two_passes(cold_Y)
    assert res[-1] is None, res                           # pass 2 breaks down: fp64 redo


def test_warm_refresh_of_the_lowrank_layer_needs_no_fp64(lowrank_layer):
    _, _, warm_Y = lowrank_layer
    d = warm_Y.shape[1]
    Xe = warm_Y / np.linalg.norm(warm_Y, axis=0)
    s = np.linalg.svd(Xe, compute_uv=False)
    assert s[0] / s[-1] < 1e5                             # equilibrated: far from 4e8
    res = _two_passes(warm_Y)
    assert None not in res, res
    assert res[-1] <= 2e-7 * np.sqrt(d)                   # the last pass's gate lets it through
