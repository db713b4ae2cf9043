"""Pins for the CPU oracle: each test checks it against something other than
itself -- a closed form, a brute-force construction, a textbook routine or a
figure printed on the pages.  No GPU needed."""
import math

import numpy as np
import pytest

from oracle import shampoo4_oracle as O
from pinlib import (coupled_newton_inverse_root, jacobi_eigh, mgs_qr, random_orthogonal,
                    spd_with_spectrum, sylvester_hadamard)

EPS0 = 1e-300   # "eps -> 0" for the fp64 limits


def _converged_state(S: np.ndarray, eps: float, iters: int = 400):
    """Run quant-off refreshes with S fixed until the subspace iteration has
    converged; returns (U, lam)."""
    f = O.Factor(S.shape[0], S.astype(np.float32))
    for _ in range(iters):
        O.refresh_factor(f, eps, 0, quant=False)
    return f.U64, f.lam


# ---------------------------------------------------------------- codec (P7)

def test_codebook_is_signed_square_of_linear_grid():
    cb = O.codebook_f64()
    y = np.linspace(-1.0, 1.0, 16)           # the linear grid, independently
    assert np.allclose(cb, np.sign(y) * y * y, rtol=0, atol=1e-15)
    assert cb[0] == -1.0 and cb[-1] == 1.0
    assert np.all(np.diff(cb) > 0)
    assert not np.any(cb == 0.0)             # 16 levels, no exact zero
    t = O.thresholds_f32()
    assert t[7] == 0.0 and np.all(np.diff(t) > 0)


def test_codebook_points_roundtrip_exactly():
    rng = np.random.default_rng(1)
    cb32 = O.codebook_f32()
    for k in (-20, -3, 0, 5):
        j = rng.integers(0, 16, size=640)
        j[::64] = 15                         # absmax element = +2^k in every block
        x = (cb32[j] * np.float32(2.0 ** k)).astype(np.float32)
        codes, scales = O.quantize(x)
        assert np.all(scales == np.float32(2.0 ** k))
        assert np.array_equal(O.unpack_nibbles(codes, x.size), j.astype(np.uint8))
        assert np.array_equal(O.dequantize(codes, scales, x.size), x)


def test_quantizer_is_nearest_level_rounding_near_every_threshold():
    # Brute force: 2^16 consecutive fp32 bit patterns around each threshold.
    # The count rule must agree with nearest-codebook-level rounding (fp64
    # distances) except exactly on a threshold, where it takes the lower code.
    t = O.thresholds_f32()
    cb = O.codebook_f64()
    vals = []
    for tk in t:
        if tk == 0.0:
            base = np.arange(-32768, 32768, dtype=np.int64)
            pos = base[base >= 0].astype(np.uint32).view(np.float32)
            neg = (-base[base > 0]).astype(np.uint32).view(np.float32) * np.float32(-1)
            vals.append(pos); vals.append(neg)
        else:
            b = np.array([tk], np.float32).view(np.uint32)[0].astype(np.int64)
            vals.append((b + np.arange(-32768, 32768)).astype(np.uint32).view(np.float32))
    v = np.concatenate(vals).astype(np.float32)
    v = v[np.abs(v) <= 1.0]
    nblk = (v.size + 62) // 63
    x = np.zeros(nblk * 64, np.float32)
    x.reshape(nblk, 64)[:, 0] = 1.0          # absmax 1 -> v = x exactly
    flat = x.reshape(nblk, 64)[:, 1:].ravel()
    flat[:v.size] = v
    x.reshape(nblk, 64)[:, 1:] = flat.reshape(nblk, 63)
    codes, scales = O.quantize(x)
    assert np.all(scales == 1.0)
    got = O.unpack_nibbles(codes, x.size).reshape(nblk, 64)[:, 1:].ravel()[:v.size]
    # Nearest level, computed exactly: level j is nearest iff v lies between
    # the exact midpoints (a_{j-1}+a_j)/450 and (a_j+a_{j+1})/450 with
    # a_j = (2j-15)|2j-15| integers; 450 v is exact in fp64.
    a = np.array([(2 * j - 15) * abs(2 * j - 15) for j in range(16)], np.float64)
    assert np.array_equal(a / 225, cb)
    w = 450.0 * v.astype(np.float64)
    nearest = np.sum(w[:, None] > (a[:-1] + a[1:])[None, :], axis=1)
    on_thr = np.isin(v, t)
    assert np.array_equal(got[~on_thr], nearest[~on_thr])
    for k, tk in enumerate(t):
        assert np.all(got[v == tk] == k)


def test_quantizer_error_bound_and_absmax_exact():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(64 * 257 + 13).astype(np.float32)
    codes, scales = O.quantize(x)
    xr = O.dequantize(codes, scales, x.size)
    cb = O.codebook_f64()
    half_gap = np.max(np.diff(cb)) / 2          # 28/225
    assert abs(half_gap - 28 / 225) < 1e-15
    s = np.repeat(scales, 64)[:x.size].astype(np.float64)
    err = np.abs(x.astype(np.float64) - xr.astype(np.float64))
    assert np.all(err <= half_gap * s * (1 + 1e-6) + 1e-30)
    c = O.unpack_nibbles(codes, x.size)
    for b in range(scales.size):
        blk = slice(64 * b, min(64 * b + 64, x.size))
        i = np.argmax(np.abs(x[blk]))
        assert c[blk][i] in (0, 15)
        assert abs(xr[blk][i]) == scales[b]


def test_quantizer_zero_block_ragged_tail_and_packing():
    x = np.zeros(64 + 65, np.float32)
    x[64:] = np.linspace(-1, 1, 65, dtype=np.float32)
    codes, scales = O.quantize(x)
    assert codes.size == (x.size + 1) // 2 and scales.size == 3
    assert scales[0] == 0.0 and scales[2] == 1.0       # ragged last block of 1
    assert np.all(O.dequantize(codes, scales, x.size)[:64] == 0.0)
    # one element per 2 nibbles, even index low; padded high nibble is 0
    c = O.unpack_nibbles(codes, x.size)
    assert codes[-1] >> 4 == 0
    assert np.array_equal(codes[:-1], c[0:-1:2] | (c[1::2] << 4))


def test_quantizer_nonfinite_rule():
    x = np.ones(192, np.float32)
    x[3] = np.nan
    x[64 + 5] = np.inf
    codes, scales = O.quantize(x)
    assert np.isnan(scales[0]) and scales[1] == np.inf and scales[2] == 1.0
    c = O.unpack_nibbles(codes, x.size)
    assert np.all(c[:64] == 0)                 # NaN scale: every comparison fails
    assert c[64 + 5] == 0                      # inf / inf = NaN
    assert np.all(np.delete(c[64:128], 5) == 7)   # 1 / inf = +0 -> code 7


# ------------------------------------------------------------ stats (EMA)

def test_ema_stats_closed_form_and_sides():
    G = np.zeros((3, 5), np.float32)
    G[0, 1] = 2.0
    G[2, 4] = -1.0
    beta = float(np.float32(0.95))
    SL = np.zeros((3, 3), np.float32)
    SR = np.zeros((5, 5), np.float32)
    for _ in range(7):
        SL = O.ema_stats(SL, G, beta, "L")
        SR = O.ema_stats(SR, G, beta, "R")
    w = 1 - beta ** 7                          # geometric series sum (1-b) b^i
    eL = np.zeros((3, 3)); eL[0, 0] = 4 * w; eL[2, 2] = w
    eR = np.zeros((5, 5)); eR[1, 1] = 4 * w; eR[4, 4] = w
    assert np.allclose(SL, eL, rtol=1e-6, atol=0)
    assert np.allclose(SR, eR, rtol=1e-6, atol=0)


# ------------------------------------------- compressed statistics (f1)

def _signed_hadamard(d, rng):
    """A non-symmetric orthogonal matrix whose entries are all +-1/sqrt(d):
    Sylvester's Hadamard matrix with its columns permuted and sign-flipped.
    For d = 64 every entry is +-1/8, so each 64-block's absmax is 1/8 and
    every entry sits exactly on a codebook end level: the 4-bit codes hold
    it without error."""
    H = np.array([[1.0]])
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    H = H[:, rng.permutation(d)] * rng.choice([-1.0, 1.0], d)[None, :]
    return H / np.sqrt(d)


def test_compressed_update_equals_the_ema_when_the_codes_are_exact():
    # With a basis the codec stores exactly, U diag(lambda) U^T is the stored
    # statistic itself, so the compressed update is the plain EMA of it.
    rng = np.random.default_rng(21)
    d = 64
    U = _signed_hadamard(d, rng)
    assert np.allclose(U.T @ U, np.eye(d), atol=1e-15) and not np.allclose(U, U.T)
    lam = np.sort(rng.uniform(0.0, 3.0, d))[::-1].astype(np.float32)
    f = O.Factor(d, np.zeros((d, d), np.float32))
    f.codes, f.scales = O.quantize(U.astype(np.float32).ravel())
    assert np.array_equal(O.dequantize(f.codes, f.scales, d * d).reshape(d, d), U.astype(np.float32))
    f.lam = lam
    f.has_basis = True
    S_prev = (U * lam.astype(np.float64)[None, :]) @ U.T           # exact fp64 statistic
    beta = float(np.float32(0.9))
    for side, shape in (("L", (d, 40)), ("R", (40, d))):
        G = rng.standard_normal(shape).astype(np.float32)
        got = O.compressed_stats(f, G, beta, side)
        g = G.astype(np.float64)
        want = beta * S_prev + (1 - beta) * (g @ g.T if side == "L" else g.T @ g)
        assert np.allclose(got, want, rtol=0, atol=2e-6 * np.abs(want).max()), side
        # a transposed basis would rebuild a different matrix
        wrong = (U.T * lam.astype(np.float64)[None, :]) @ U
        assert not np.allclose(S_prev, wrong, atol=1e-3)


def test_compressed_update_first_step_and_nonfinite():
    rng = np.random.default_rng(22)
    d = 16
    f = O.Factor(d, np.zeros((d, d), np.float32))
    G = rng.standard_normal((d, 24)).astype(np.float32)
    beta = 0.8
    # nothing stored yet: the EMA from zero
    assert np.array_equal(O.compressed_stats(f, G, beta, "L"), O.ema_stats(f.S, G, beta, "L"))
    # a non-finite gradient leaves the stored statistic: zero before any refresh ...
    Gn = G.copy()
    Gn[3, 5] = np.inf
    assert np.array_equal(O.compressed_stats(f, Gn, beta, "L"), f.S)
    # ... and the rebuilt U diag(lambda) U^T after one
    f.S = O.compressed_stats(f, G, beta, "L")
    O.refresh_factor(f, 1e-6, 5)
    assert f.has_basis and f.lam.max() > 1.0
    U = O.dequantize(f.codes, f.scales, d * d).reshape(d, d).astype(np.float64)
    stored = (U * f.lam.astype(np.float64)[None, :]) @ U.T
    assert np.allclose(O.compressed_stats(f, Gn, beta, "L"), stored, rtol=0, atol=1e-6 * np.abs(stored).max())


# ------------------------------------------------ coupled Newton root (f4)

def test_newton_root_of_a_diagonal_is_the_elementwise_root():
    lam = np.array([1.0, 0.3, 2e-3, 7.5, 1e-4])
    R = O.newton_inverse_root(np.diag(lam), p=4, iters=40)
    assert np.allclose(R, np.diag(lam ** -0.25), rtol=1e-12, atol=0)


def test_newton_root_matches_the_eigen_form_on_a_known_spectrum():
    rng = np.random.default_rng(31)
    d = 24
    V = random_orthogonal(d, rng)
    lam = np.geomspace(1.0, 1e-4, d)                      # kappa = 1e4
    A = (V * lam[None, :]) @ V.T
    want = (V * (lam ** -0.25)[None, :]) @ V.T
    got = O.newton_inverse_root(A, p=4, iters=40)
    assert np.linalg.norm(got - want) <= 1e-10 * np.linalg.norm(want)
    # p = 2: the inverse square root of the same matrix
    got2 = O.newton_inverse_root(A, p=2, iters=60)
    assert np.allclose(got2, (V * (lam ** -0.5)[None, :]) @ V.T, rtol=0, atol=1e-9 * lam.min() ** -0.5)


def test_newton_root_coupling_invariant_and_homogeneity():
    # M_k = X_k^p A / c at every iteration (the coupling the iteration keeps),
    # and (s A)^(-1/p) = s^(-1/p) A^(-1/p)
    rng = np.random.default_rng(32)
    d = 10
    V = random_orthogonal(d, rng)
    A = (V * rng.uniform(0.05, 3.0, d)[None, :]) @ V.T
    c = np.linalg.norm(A)
    hist = []
    O.newton_inverse_root(A, p=4, iters=12, history=hist)
    for X, M in hist:
        assert np.allclose(M, np.linalg.matrix_power(X, 4) @ A / c, rtol=0, atol=1e-11)
    R = O.newton_inverse_root(A, p=4, iters=40)
    assert np.allclose(O.newton_inverse_root(16.0 * A, p=4, iters=40), R / 2.0, rtol=1e-12, atol=1e-14)


# ------------------------------- the abstract's comparisons, on the oracle

def test_quantizing_the_eigenvectors_beats_quantizing_the_statistic():
    # "4-bit Shampoo ...", abstract: keeping the eigenvector matrix in 4 bits
    # approximates the preconditioner far better than keeping the statistic
    # itself in 4 bits, and rectifying the dequantized eigenvectors' orthogonality
    # improves the inverse fourth root further.  Checked on statistics with a
    # decaying spectrum (kappa = 1e4), with the same codec for both.
    rng = np.random.default_rng(41)
    d, eps = 64, 1e-6
    for trial in range(3):
        V = random_orthogonal(d, rng)
        lam = np.geomspace(1.0, 1e-4, d) * rng.uniform(0.5, 2.0)
        S = (V * lam[None, :]) @ V.T
        P = (V * (lam + eps)[None, :] ** -0.25) @ V.T
        rel = lambda X: np.linalg.norm(X - P) / np.linalg.norm(P)
        # eigenvectors in 4 bits (eigenvalues exact), with and without Bjorck
        c, sc = O.quantize(V.astype(np.float32).ravel())
        Uq = O.dequantize(c, sc, d * d).reshape(d, d).astype(np.float64)
        err_u = rel(O.root_from_basis(Uq, lam, eps))
        err_ub = rel(O.root_from_basis(O.bjorck(Uq, 5), lam, eps))
        # the statistic itself in 4 bits, then its exact root (negative
        # eigenvalues of the dequantized matrix clamped at 0)
        c2, sc2 = O.quantize(S.astype(np.float32).ravel())
        Sq = O.dequantize(c2, sc2, d * d).reshape(d, d).astype(np.float64)
        Sq = 0.5 * (Sq + Sq.T)
        w, W = jacobi_eigh(Sq)
        err_s = rel((W * (np.maximum(w, 0.0) + eps)[None, :] ** -0.25) @ W.T)
        assert err_ub < err_u < err_s, (trial, err_ub, err_u, err_s)
        assert err_s > 10 * err_u


# ------------------------------------------------------------ Bjorck (P4)

def test_bjorck_closed_form_on_svd():
    rng = np.random.default_rng(3)
    d = 12
    Q1, Q2 = random_orthogonal(d, rng), random_orthogonal(d, rng)
    s = rng.uniform(0.2, 2.0, d)
    U = (Q1 * s) @ Q2.T
    got = O.bjorck(U, 1)
    want = (Q1 * (s * (1.5 - 0.5 * s * s))) @ Q2.T
    assert np.allclose(got, want, rtol=0, atol=1e-13)


def test_bjorck_orthogonality_residual_decreases_on_dequantized_basis():
    rng = np.random.default_rng(4)
    d = 96
    Q = random_orthogonal(d, rng).astype(np.float32)
    codes, scales = O.quantize(Q.ravel())
    U = O.dequantize(codes, scales, d * d).reshape(d, d).astype(np.float64)
    res = [np.linalg.norm(U.T @ U - np.eye(d))]
    for _ in range(5):
        U = O.bjorck(U, 1)
        res.append(np.linalg.norm(U.T @ U - np.eye(d)))
    assert res[0] > 1e-2
    assert all(b < a for a, b in zip(res[:3], res[1:4]))
    assert res[-1] < 1e-12


# ------------------------------------------- warm 4-bit refresh (a3-a8)

def _row_scaled_exact_basis(rng, d, r):
    """Codes and scales whose dequantization is exactly diag(r) V, with V a
    signed, row-permuted Sylvester-Hadamard basis H / sqrt(d) (not
    symmetric).  For d = 64 a quantization block is one row; every entry of
    a row of H is +-1, so the absmax-normalized values sit exactly on the
    codebook's end levels and the row's scale carries r_i / sqrt(d)."""
    H = sylvester_hadamard(d)[rng.permutation(d)] * rng.choice([-1.0, 1.0], d)[None, :]
    V = H / np.sqrt(d)
    codes, _ = O.quantize(H.astype(np.float32).ravel())
    scales = (np.asarray(r, np.float64) / np.sqrt(d)).astype(np.float32)
    return V, codes, scales


def _bjorck_scalar(s, t):
    """t steps of the scalar map s -> s (1.5 - 0.5 s^2): Bjorck's action on
    the singular values (one step: U = A diag(s) B^T -> A diag(s (1.5 -
    0.5 s^2)) B^T)."""
    for _ in range(t):
        s = s * (1.5 - 0.5 * s * s)
    return s


def test_warm_refresh_rectifies_the_dequantized_basis_before_the_subspace_step():
    """"4-bit Shampoo ...", abstract: the dequantized eigenvector matrix has
    its orthogonality rectified, which is what the inverse fourth root is
    then built from.  For a stored basis that dequantizes exactly to
    diag(r) V (V orthogonal), U U^T = diag(r^2), so every Bjorck step only
    rescales rows: U_t = diag(phi_t(r)) V with phi the scalar map above.
    The warm refresh must then equal one subspace step from that closed
    form, Q R = (S + eps I) diag(phi_t(r)) V, taken here by Gram-Schmidt.
    A refresh that skipped Bjorck, ran a different number of steps, ran it
    after the QR, transposed the dequantized matrix or dropped the eps shift
    lands measurably away (checked below, so the pin has teeth)."""
    rng = np.random.default_rng(21)
    d, t, eps = 64, 5, 1e-3
    r = rng.integers(16, 103, d) / 64.0              # row scales in [0.25, 1.6], exact in fp32
    V, codes, scales = _row_scaled_exact_basis(rng, d, r)
    lam_s = np.concatenate([rng.uniform(0.05, 1.0, d - 2), [0.0, 0.0]])    # two null directions
    S = spd_with_spectrum(lam_s, rng).astype(np.float32)
    S64 = S.astype(np.float64)
    f = O.Factor(d, S.copy(), codes=codes.copy(), scales=scales.copy(),
                 lam=np.zeros(d, np.float32), has_basis=True)
    U0 = O.dequantize(codes, scales, d * d).reshape(d, d).astype(np.float64)
    assert np.array_equal(U0, r[:, None] / np.sqrt(d) * np.sqrt(d) * V)      # exact diag(r) V
    O.refresh_factor(f, eps, t)

    def expected(rows, M=V, shift=eps):
        Q, R = mgs_qr((S64 + shift * np.eye(d)) @ (rows[:, None] * M))
        return Q
    Qw = expected(_bjorck_scalar(r, t))
    assert np.linalg.norm(f.q_last - Qw) <= 1e-9 * np.sqrt(d)
    lam_w = np.maximum(np.einsum("ij,ij->j", Qw, S64 @ Qw), 0.0)
    assert np.allclose(f.lam.astype(np.float64), lam_w, rtol=1e-6, atol=1e-9)
    # the requantized state is the codec applied to that Q
    c2, s2 = O.quantize(f.q_last.astype(np.float32).ravel())
    assert np.array_equal(f.codes, c2) and np.array_equal(f.scales, s2)
    # teeth: each plausible mistake moves Q far beyond the tolerance above
    wrong = {
        "no Bjorck": expected(r),
        "t - 1 steps": expected(_bjorck_scalar(r, t - 1)),
        "Bjorck after the QR": mgs_qr(expected(r))[0],
        # dequantized matrix read transposed: U = V^T diag(r), whose Bjorck
        # steps scale its columns the same way
        "transposed basis": expected(np.ones(d), M=V.T * _bjorck_scalar(r, t)[None, :]),
        "no eps shift": expected(_bjorck_scalar(r, t), shift=0.0),
    }
    for name, Qx in wrong.items():
        assert np.linalg.norm(f.q_last - Qx) > 1e-4 * np.sqrt(d), name


def test_exactly_stored_orthogonal_basis_passes_the_warm_refresh_unchanged():
    """An orthogonal basis the codes hold exactly (r = 1 above) is a fixed
    point of Bjorck; if it is also S's eigenbasis, the subspace step
    returns it exactly (up to rounding), with the eigenvalues as Rayleigh
    quotients, and requantization gives back the same codes."""
    rng = np.random.default_rng(22)
    d, eps = 64, 1e-6
    V, codes, scales = _row_scaled_exact_basis(rng, d, np.ones(d))
    assert np.array_equal(O.bjorck(O.dequantize(codes, scales, d * d).reshape(d, d), 5), V)
    lam_s = np.geomspace(1.0, 1e-3, d)
    S = ((V * lam_s[None, :]) @ V.T).astype(np.float32)
    f = O.Factor(d, S.copy(), codes=codes.copy(), scales=scales.copy(), lam=np.zeros(d, np.float32),
                 has_basis=True)
    O.refresh_factor(f, eps, 5)
    assert np.allclose(f.q_last, V, rtol=0, atol=1e-7)     # S holds fp32-rounded entries
    assert np.allclose(f.lam, lam_s, rtol=1e-6, atol=1e-7)   # fp32 rounding of S: about 1e-8 absolute
    assert np.array_equal(f.codes, codes) and np.array_equal(f.scales, scales)


def test_warm_refresh_is_homogeneous_with_the_quantizer_on():
    """[tut] "Where the fourth root comes from": the step is homogeneous of
    degree 0 in G.  Through a warm 4-bit refresh (eps -> 0) that means the
    same codes and scales, and eigenvalues scaled by exactly 4 for G -> 2G:
    every fp64 product scales by a power of two, the quantizer is scale
    invariant, and Bjorck acts on the same dequantized codes."""
    rng = np.random.default_rng(23)
    gs = [rng.standard_normal((12, 20)).astype(np.float32) for _ in range(3)]
    runs = []
    for scale in (1, 2):
        orc = O.Shampoo4Oracle([(12, 20)], eps=EPS0)
        for t, g in enumerate(gs, 1):
            orc.step(t, [g * np.float32(scale)], refresh_every=1)
        runs.append(orc)
    for fa, fb in zip(runs[0].factors, runs[1].factors):
        assert np.array_equal(fa.codes, fb.codes) and np.array_equal(fa.scales, fb.scales)
        assert np.array_equal(fb.lam, np.float32(4) * fa.lam)


# ----------------------------------------------------- eigenpairs (P5, P8)

def test_subspace_iteration_converges_to_jacobi_eigenpairs():
    rng = np.random.default_rng(5)
    d = 20
    lam_true = 0.7 ** np.arange(d)              # distinct, ratio 0.7
    S = spd_with_spectrum(lam_true, rng).astype(np.float32)
    U, lam = _converged_state(S, EPS0, iters=300)
    S64 = S.astype(np.float64)
    lj, Vj = jacobi_eigh(S64)
    assert np.allclose(lam, lj, rtol=1e-10, atol=1e-14)
    assert np.linalg.norm(S64 @ U - U * lam[None, :]) <= 1e-10 * np.linalg.norm(S64)
    # columns equal Jacobi's eigenvectors up to sign
    cos = np.abs(np.sum(U * Vj, axis=0))
    assert np.all(np.abs(cos - 1) < 1e-9)
    # third opinion: LAPACK eigh
    le = np.linalg.eigvalsh(S64)[::-1]
    assert np.allclose(lam, le, rtol=1e-10, atol=1e-14)


def test_subspace_step_is_the_qr_factor_with_positive_diagonal():
    rng = np.random.default_rng(8)
    d = 9
    G = rng.standard_normal((d, 4))
    S = (G @ G.T).astype(np.float32)             # rank 4: zero eigenvalues
    U = random_orthogonal(d, rng)
    eps = 1e-3
    Q, lam = O.subspace_step(S, U, eps)
    Y = (S.astype(np.float64) + eps * np.eye(d)) @ U
    R = Q.T @ Y                                  # Y = Q R  =>  R = Q^T Y
    assert np.allclose(Q.T @ Q, np.eye(d), atol=1e-13)
    assert np.allclose(np.tril(R, -1), 0, atol=1e-12)
    assert np.all(np.diag(R) > 0)
    assert np.all(lam >= 0)
    assert np.allclose(lam, np.maximum(np.diag(Q.T @ S.astype(np.float64) @ Q), 0), atol=1e-14)


def test_diagonal_statistic_with_identity_start_is_exact():
    lam_star = np.array([3.0, 0.5, 0.25, 2.0, 1e-3], np.float32)
    S = np.diag(lam_star).astype(np.float32)
    Q, lam = O.subspace_step(S, np.eye(5), 1e-6)
    assert np.array_equal(Q, np.eye(5))
    assert np.array_equal(lam, lam_star.astype(np.float64))
    # and the step D = diag(mu_L) G diag(mu_R) exactly (quant off)
    orc = O.Shampoo4Oracle([(5, 3)], quant=False)
    for f, d in zip(orc.factors, (5, 3)):
        f.S = np.diag(lam_star[:d]).astype(np.float32)
    orc.refresh_roots()
    G = np.arange(15, dtype=np.float32).reshape(5, 3) - 7
    D = orc.precondition([G])[0]
    muL = (lam_star[:5].astype(np.float64) + orc.eps) ** -0.25
    muR = (lam_star[:3].astype(np.float64) + orc.eps) ** -0.25
    want = (muL[:, None] * G.astype(np.float64) * muR[None, :]).astype(np.float32)
    assert np.array_equal(D, want)


# ----------------------------------------------------------- root (P6)

def test_root_matches_coupled_newton_and_fourth_power():
    rng = np.random.default_rng(6)
    d = 16
    lam_true = np.geomspace(2.0, 1e-4, d)
    S = spd_with_spectrum(lam_true, rng).astype(np.float32)
    eps = 1e-6
    U, lam = _converged_state(S, eps, iters=600)
    P = O.root_from_basis(U, lam, eps)
    A = S.astype(np.float64) + eps * np.eye(d)
    X = coupled_newton_inverse_root(A, 4)
    assert np.linalg.norm(P - X) <= 1e-10 * np.linalg.norm(X)
    P4 = np.linalg.matrix_power(P, 4)
    assert np.linalg.norm(P4 @ A - np.eye(d)) < 1e-9


# -------------------------------------- Kronecker identity and bound (P1)

@pytest.mark.parametrize("m,n", [(2, 3), (3, 2), (4, 4), (2, 2)])
def test_update_equals_kronecker_preconditioner_on_vec(m, n):
    rng = np.random.default_rng(10 * m + n)
    orc = O.Shampoo4Oracle([(m, n)], eps=1e-6, quant=False)
    for _ in range(6):
        orc.update_stats([rng.standard_normal((m, n)).astype(np.float32)])
    for _ in range(300):
        orc.refresh_roots()
    G = rng.standard_normal((m, n)).astype(np.float32)
    D = orc.precondition([G])[0].astype(np.float64)
    PL = O.factor_root(orc.factors[0], orc.eps, False)
    PR = O.factor_root(orc.factors[1], orc.eps, False)
    vec = lambda X: X.reshape(-1, order="F")           # column-major vec
    assert np.allclose(vec(D), np.kron(PR, PL) @ vec(G.astype(np.float64)),
                       rtol=1e-6, atol=1e-7)           # D is stored fp32
    # The page's route: (R^(1/2) kron L^(1/2))^(-1/2) acting on vec(G), with
    # the eps-shifted factors, built from LAPACK eigh on the full mn x mn
    # matrix -- no use of the oracle's own eigen machinery.
    def sqrtm(A):
        w, V = np.linalg.eigh(A)
        return (V * np.sqrt(w)) @ V.T
    Le = orc.factors[0].S.astype(np.float64) + orc.eps * np.eye(m)
    Re = orc.factors[1].S.astype(np.float64) + orc.eps * np.eye(n)
    K = np.kron(sqrtm(Re), sqrtm(Le))
    w, V = np.linalg.eigh(K)
    Kmh = (V * w ** -0.5) @ V.T
    assert np.allclose(vec(D), Kmh @ vec(G.astype(np.float64)), rtol=2e-6, atol=1e-6)


# ------------------------------------------------------ homogeneity (P2)

def test_step_is_homogeneous_of_degree_zero():
    rng = np.random.default_rng(7)
    G = rng.standard_normal((6, 6)).astype(np.float32)
    outs, codes = [], []
    for scale, quant in ((1, False), (2, False), (1, True), (2, True)):
        orc = O.Shampoo4Oracle([(6, 6)], eps=EPS0, quant=quant)
        D = orc.step(1, [G * np.float32(scale)], refresh_every=1)[0]
        outs.append(D.astype(np.float64))
        codes.append([f.codes for f in orc.factors] if quant else None)
    assert np.linalg.norm(outs[0] - outs[1]) <= 1e-12 * np.linalg.norm(outs[0])
    for a, b in zip(codes[2], codes[3]):
        assert np.array_equal(a, b)
    assert np.linalg.norm(outs[2] - outs[3]) <= 1e-6 * np.linalg.norm(outs[2])


# ------------------------------------------------------ partition (a1)

def test_partition_counts_for_the_workload_shapes():
    from bit_quantized_shampoo_b200.workloads import WORKLOADS
    b5 = O.partition(WORKLOADS[5].shapes, 1024)
    # 4096 x 11008 -> 4 row chunks x (10 full + one 768) = 44 blocks, x8;
    # 4096 x 4096 -> 16 blocks, x8.
    assert len(b5) == 4 * 11 * 8 + 16 * 8 == 480
    dims = [d for b in b5 for d in (b.m, b.n)]
    assert dims.count(1024) == 928 and dims.count(768) == 32
    b4 = O.partition(WORKLOADS[4].shapes, 1024)
    # per layer: 768x2304 -> 1024+1024+256; 768x768 -> 1; 768x3072 -> 3;
    # 3072x768 -> 3 row chunks.
    assert len(b4) == 12 * (3 + 1 + 3 + 3)
    assert sorted({(b.m, b.n) for b in b4}) == [(768, 256), (768, 768), (768, 1024), (1024, 768)]
    b1 = O.partition(WORKLOADS[1].shapes, 1024)
    assert [(b.m, b.n) for b in b1] == [(128, 128)]
    # a ragged tail is kept, not rebalanced
    assert [(b.r0, b.m) for b in O.partition([(2500, 10)], 1024)] == [(0, 1024), (1024, 1024), (2048, 452)]


# ------------------------------------------------------ cost model (P9)

def _golden_costs():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "shampoo_cost_model.txt")
    out = {}
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        k, v, tol, _ = [p.strip() for p in line.split("|")]
        out[k] = (float(v), float(tol))
    return out


def test_cost_model_reproduces_the_pages_figures():
    from bit_quantized_shampoo_b200 import costmodel as C
    g = _golden_costs()
    got = {
        "full_matrix_entries_1024x1024": C.full_matrix_entries(1024, 1024),
        "full_matrix_bytes_fp32_1024x1024": 4 * C.full_matrix_entries(1024, 1024),
        "full_matrix_root_flops_1024x1024": C.full_matrix_root_flops(1024, 1024),
        "kron_floats_1024x1024": C.kronecker_floats(1024, 1024),
        "kron_bytes_fp32_1024x1024": 4 * C.kronecker_floats(1024, 1024),
        "kron_root_flops_1024x1024": C.kronecker_root_flops(1024, 1024),
        "overhead_4096x4096_B1e6": C.overhead_ratio(4096, 4096, 1e6),
        "overhead_2048x2048_B4096": C.overhead_ratio(2048, 2048, 4096),
        "accumulator_floats_4096x11008": C.kronecker_floats(4096, 11008),
        "adam_floats_4096x11008": C.adam_floats(4096, 11008),
        "blocked_floats_per_param": C.kronecker_floats(1024, 1024) / (1024 * 1024),
        "cached_roots_floats_per_param": 2 * C.kronecker_floats(512, 512) / (512 * 512),
    }
    assert set(got) == set(g)
    for k, (v, tol) in g.items():
        assert abs(got[k] - v) <= tol * abs(v) + 1e-12, (k, got[k], v)
    # the per-step term is the sum of its four parts
    assert C.step_flops(300, 70) == C.stats_flops(300, 70) + C.apply_flops(300, 70)


# ------------------------------------------- dynamic tree codebook (f3)

def test_dynamic_tree_codebook_follows_its_bit_layout():
    """The 4-bit dynamic tree map: symmetric, both middle levels zero, and
    for each decimal exponent E (zeros before the indicator bit) the 2^(2-E)
    magnitudes lie in (0.1, 1] x 10^-E on an equally spaced grid of step
    0.9 x 10^-E / 2^(2-E) ending at 10^-E.  Every pattern is decoded here
    from its bits as a string, independently of the oracle's arithmetic."""
    cb = O.codebook_f64(O.DYNAMIC_TREE)
    assert cb.size == 16 and np.all(np.diff(cb) >= 0)
    assert np.array_equal(cb, -cb[::-1])
    assert cb[7] == 0.0 and cb[8] == 0.0 and cb[15] == 1.0
    pos = cb[8:]
    for p in range(8):
        bits = format(p, "03b")
        if "1" not in bits:
            assert pos[p] == 0.0
            continue
        e = bits.index("1")
        frac = bits[e + 1:]
        k = len(frac)
        i = int(frac, 2) if frac else 0
        lo, hi = 0.1 * 10.0 ** -e, 10.0 ** -e
        assert lo < pos[p] <= hi * (1 + 1e-15)
        step = 0.9 * 10.0 ** -e / 2 ** k
        assert abs(pos[p] - (hi - (2 ** k - 1 - i) * step)) <= 1e-15
    t = O.thresholds_f32(O.DYNAMIC_TREE)
    assert t[7] == 0.0 and np.all(np.diff(t) >= 0)


def test_dynamic_tree_count_rule_is_nearest_level():
    """Brute force around every threshold of the dynamic tree map (2^10 fp32
    neighbours each): the count rule picks the nearest level, measured with
    exact rational distances to the levels of the bit-layout definition,
    the lower one on an exact tie -- except between an fp32 threshold and
    the exact midpoint it rounds (inclusive of the threshold), where the
    fp32 threshold decides by definition.  Every level also round-trips
    exactly at absmax 2^k.  (The linear square map has its own exact test
    above.)"""
    from fractions import Fraction
    cbk = O.DYNAMIC_TREE
    cb = O.codebook_f64(cbk)
    t = O.thresholds_f32(cbk)

    def level(j):                       # exact rational from the bit layout
        p = j - 8 if j >= 8 else 7 - j
        bits = format(p, "03b")
        if "1" not in bits:
            return Fraction(0)
        e = bits.index("1")
        k = 2 - e
        i = int(bits[e + 1:], 2) if k else 0
        m = Fraction(1, 10 ** e) * (Fraction(1, 10) + Fraction(9, 10) * Fraction(i + 1, 2 ** k))
        return m if j >= 8 else -m
    lv = [level(j) for j in range(16)]
    assert np.array_equal(np.array([float(x) for x in lv]), cb)
    vals = []
    for tk in t:
        b = np.array([tk], np.float32).view(np.uint32)[0].astype(np.int64)
        if tk == 0.0:
            mag = np.arange(0, 512).astype(np.uint32).view(np.float32)
            vals += [mag, -mag]
        else:
            vals.append((b + np.arange(-512, 512)).astype(np.uint32).view(np.float32))
    v = np.unique(np.concatenate(vals).astype(np.float32))
    v = v[np.abs(v) <= 1.0]
    nblk = (v.size + 62) // 63
    x = np.zeros(nblk * 64, np.float32)
    x.reshape(nblk, 64)[:, 0] = 1.0
    flat = x.reshape(nblk, 64)[:, 1:].ravel()
    flat[:v.size] = v
    x.reshape(nblk, 64)[:, 1:] = flat.reshape(nblk, 63)
    codes, scales = O.quantize(x, codebook=cbk)
    got = O.unpack_nibbles(codes, x.size).reshape(nblk, 64)[:, 1:].ravel()[:v.size]
    mids = [(lv[k] + lv[k + 1]) / 2 for k in range(15)]
    checked = 0
    for vi, ci in zip(v.tolist(), got.tolist()):
        fv = Fraction(vi)
        if any(Fraction(float(tk)) != mk and min(Fraction(float(tk)), mk) <= fv <= max(Fraction(float(tk)), mk)
               for tk, mk in zip(t, mids)):
            continue
        dist = [abs(fv - L) for L in lv]
        nearest = dist.index(min(dist))                  # first = lower on ties
        assert lv[ci] == lv[nearest], (vi, ci, nearest)
        checked += 1
    assert checked > 0.9 * v.size
    for k in (-7, 0, 3):
        j = np.tile(np.arange(16), 8)
        j[::64] = 15
        xs = (O.codebook_f32(cbk)[j] * np.float32(2.0 ** k)).astype(np.float32)
        c2, s2 = O.quantize(xs, codebook=cbk)
        assert np.array_equal(O.dequantize(c2, s2, xs.size, codebook=cbk), xs)


def test_dynamic_tree_error_bound():
    rng = np.random.default_rng(12)
    x = rng.standard_normal(64 * 101 + 7).astype(np.float32)
    codes, scales = O.quantize(x, codebook=O.DYNAMIC_TREE)
    xr = O.dequantize(codes, scales, x.size, codebook=O.DYNAMIC_TREE)
    half_gap = np.max(np.diff(O.codebook_f64(O.DYNAMIC_TREE))) / 2     # (0.325 - 0.1) / 2
    assert abs(half_gap - 0.1125) < 1e-15
    s = np.repeat(scales, 64)[:x.size].astype(np.float64)
    assert np.all(np.abs(x.astype(np.float64) - xr) <= half_gap * s * (1 + 1e-6) + 1e-30)


# --------------------------------------------- Newton root method (f4)

def test_newton_root_method_matches_the_lapack_root_through_the_step():
    """Root method NEWTON: the refresh's P is (S + eps I)^(-1/4) and the
    update is P_L G P_R -- checked against roots built from LAPACK eigh of
    S + eps I (an independent route), through the oracle's whole step."""
    rng = np.random.default_rng(31)
    shapes = [(24, 40)]
    orc = O.Shampoo4Oracle(shapes, eps=1e-4, root_method=O.ROOT_NEWTON, newton_iters=40)
    gs = [rng.standard_normal(shapes[0]).astype(np.float32) for _ in range(3)]
    for t, g in enumerate(gs, 1):
        D = orc.step(t, [g], refresh_every=1)[0]

    def eig_root(S, eps):
        w, V = np.linalg.eigh(np.asarray(S, np.float64) + eps * np.eye(S.shape[0]))
        return (V * w ** -0.25) @ V.T
    PL, PR = (eig_root(f.S, orc.eps) for f in orc.factors)
    for f, P in zip(orc.factors, (PL, PR)):
        assert np.linalg.norm(f.P - P) <= 1e-6 * np.linalg.norm(P)        # P stored in fp32
    want = PL @ gs[-1].astype(np.float64) @ PR
    assert np.linalg.norm(D - want) <= 2e-6 * np.linalg.norm(want)


def test_newton_root_of_a_diagonal_statistic_and_the_quantized_root():
    """A diagonal S gives P = diag((s + eps)^-1/4) (Newton keeps diagonal
    iterates diagonal).  With NEWTON_Q4 each 64-element quantization block is
    one row of P: its absmax is the diagonal entry, which takes the top
    level and decodes exactly to the fp32 scale, and every other entry is
    an exact zero, which the count rule sends to code 7 -- level -1/225 of
    the linear square map (it has no zero), so it decodes to -scale/225."""
    d, eps = 64, 1e-6
    s = np.geomspace(1.0, 1e-3, d).astype(np.float32)
    want = (s.astype(np.float64) + eps) ** -0.25
    orc = O.Shampoo4Oracle([(d, d)], eps=eps, root_method=O.ROOT_NEWTON, newton_iters=40)
    f = orc.factors[0]
    f.S = np.diag(s).astype(np.float32)
    O.refresh_factor_newton(f, eps, 40, False)
    P = O.factor_root(f, eps, root_method=O.ROOT_NEWTON)
    assert np.count_nonzero(P - np.diag(np.diag(P))) == 0
    assert np.allclose(np.diag(P), want, rtol=1e-6, atol=0)
    fq = O.Factor(d, f.S.copy())
    O.refresh_factor_newton(fq, eps, 40, True)
    Pq = O.factor_root(fq, eps, root_method=O.ROOT_NEWTON_Q4)
    sc = fq.scales.astype(np.float64)
    assert np.array_equal(np.diag(Pq), sc)
    off = Pq - np.diag(np.diag(Pq))
    expect_off = (np.float32(-1.0 / 225.0) * fq.scales.astype(np.float32))[:, None] * (1 - np.eye(d))
    assert np.array_equal(off, expect_off.astype(np.float32).astype(np.float64))
    assert np.allclose(sc, want, rtol=1e-6, atol=0)


def test_the_abstracts_two_comparisons_on_both_codebooks():
    """"4-bit Shampoo ...", abstract: quantizing the eigenvector matrix beats
    quantizing the preconditioner itself, and linear square quantization is
    (slightly) better than dynamic tree quantization.  On statistics with a
    decaying spectrum (kappa = 1e4), the inverse-root error (relative
    Frobenius) of: eigenvectors in 4 bits + Bjorck, for each codebook, and
    the root itself in 4 bits, for each codebook.  The first comparison is
    asserted; the codebook comparison is reported (the dynamic tree map is
    a reading of a method the pages only name)."""
    rng = np.random.default_rng(43)
    d, eps = 64, 1e-6
    errs = {k: [] for k in ("U_ls", "U_dt", "P_ls", "P_dt")}
    for trial in range(4):
        V = random_orthogonal(d, rng)
        lam = np.geomspace(1.0, 1e-4, d) * rng.uniform(0.5, 2.0)
        P = (V * (lam + eps)[None, :] ** -0.25) @ V.T
        rel = lambda X: np.linalg.norm(X - P) / np.linalg.norm(P)
        for cbk, tag in ((O.LINEAR_SQUARE, "ls"), (O.DYNAMIC_TREE, "dt")):
            c, sc = O.quantize(V.astype(np.float32).ravel(), codebook=cbk)
            Uq = O.dequantize(c, sc, d * d, codebook=cbk).reshape(d, d).astype(np.float64)
            errs["U_" + tag].append(rel(O.root_from_basis(O.bjorck(Uq, 5), lam, eps)))
            c2, sc2 = O.quantize(P.astype(np.float32).ravel(), codebook=cbk)
            errs["P_" + tag].append(rel(O.dequantize(c2, sc2, d * d, codebook=cbk).reshape(d, d)))
    mean = {k: float(np.mean(v)) for k, v in errs.items()}
    print("inverse-root error, mean of 4:", {k: f"{v:.3e}" for k, v in mean.items()})
    assert max(mean["U_ls"], mean["U_dt"]) < min(mean["P_ls"], mean["P_dt"])
