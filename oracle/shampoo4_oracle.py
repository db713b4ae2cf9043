"""CPU oracle for the 4-bit Shampoo preconditioner step (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
the benchmark's CPU-baseline leg may import this module.  The product path
(the CUDA library and its Python binding) never calls it, and it shares no
code, table or constant generator with that path.

What it computes, and where that is stated:

* "Shampoo -- Second-Order Optimizer", section "Kronecker factorization":
  the two Kronecker factors L (m x m, from G G^T) and R (n x n, from G^T G)
  and the update direction L^(-1/4) G R^(-1/4).
* same page, section "Pitfalls, and the small-model view": the factors are
  exponential moving averages with decay beta, not plain sums.
* same page, section "Computing the inverse fourth root": the root from an
  eigendecomposition, U (Lambda + eps I)^(-1/4) U^T.
* same page, section "Blocked and distributed variants": every weight is cut
  into tiles of at most b x b that are preconditioned independently.
* "4-bit Shampoo for Memory-Efficient Network Training", abstract: the state
  kept in 4 bits is the preconditioner's *eigenvector matrix* U, its
  orthogonality is rectified after dequantization (Bjorck orthonormalization,
  first-order form U <- 1.5 U - 0.5 U U^T U), and the 4-bit code is a linear
  square quantizer applied block-wise.
* the eigenvector refresh is one step of warm-started orthogonal (subspace)
  iteration, Y = (S + eps I) U then Y = QR, with Rayleigh quotients as the
  eigenvalues -- the power-iteration reading of the same abstract.

The quantizer runs in fp32 exactly as defined below so that its 4-bit codes
can be compared bit for bit; everything else runs in fp64 and is rounded to
fp32 only where the state is stored in fp32.

Readings where the pages are silent (all repeated in the design notes):
  codebook    cb_j = sgn(y_j) y_j^2, y_j = -1 + 2j/15, j = 0..15 (16 levels,
              no exact zero); thresholds are the fp32-rounded midpoints.
              The dynamic tree alternative the abstract names: Dettmers'
              dynamic tree data type restricted to 4 bits (sign, decimal
              exponent as a run of zeros, indicator bit, linear fraction
              over [0.1, 1] at the upper bin edges; 000 is zero).
  Newton root the coupled Newton iteration of "Computing the inverse fourth
              root" with c = ||A||_F and a fixed iteration count, as a root
              method in place of the eigen form; its root is kept in fp32, or
              quantized block-wise (quantizing the preconditioner itself).
  scale       per 64-element block of the row-major flattening, fp32 absmax.
  code        number of thresholds strictly below v = fp32(x / absmax); a
              zero block gets code 7 everywhere; NaN in a block gives a NaN
              scale, +-Inf gives +Inf, and codes follow the same count rule.
  packing     element 2i in the low nibble of byte i, 2i+1 in the high one.
  eps         added to eigenvalues inside the root and used as the shift of
              the subspace step (S + eps I) U.
  order       stats -> refresh when (t-1) mod T == 0 -> precondition; the
              first refresh starts from U = I.
"""
from __future__ import annotations

import dataclasses
import math
import numpy as np

QUANT_BLOCK = 64
LINEAR_SQUARE = 0
DYNAMIC_TREE = 1


# --------------------------------------------------------------------------
# Block-wise 4-bit codec ("4-bit Shampoo ...", abstract: linear square
# quantization of the eigenvector matrix, block-wise, which it finds
# slightly better than dynamic tree quantization).
# --------------------------------------------------------------------------

def _dynamic_tree_magnitude(bits: int) -> float:
    """The 4-bit reading of the dynamic tree data type (Dettmers, "8-bit
    approximations for parallelism in deep learning", 2016): after the sign,
    the three bits hold a run of E zeros (the decimal exponent), an
    indicator 1, and the k = 2 - E bits left over as a linear fraction i;
    the value is 10^-E (0.1 + 0.9 (i + 1) / 2^k), and 000 (no indicator) is
    zero.  The fraction takes the upper edge of each of the 2^k equal bins
    of [0.1, 1], so the largest magnitude is 1 (absmax-normalized blocks
    keep their absmax exactly, as the linear square map's end levels do).
    Returns the magnitude as the fp64 rounding of the exact rational."""
    from fractions import Fraction
    b = [(bits >> 2) & 1, (bits >> 1) & 1, bits & 1]
    if 1 not in b:
        return 0.0
    e = b.index(1)                     # zeros before the indicator
    k = 2 - e                          # fraction bits after it
    i = bits & ((1 << k) - 1)
    return float(Fraction(10) ** -e * (Fraction(1, 10) + Fraction(9, 10) * Fraction(i + 1, 2 ** k)))


def codebook_f64(codebook: int = LINEAR_SQUARE) -> np.ndarray:
    """The 16 levels in ascending order, fp64.
    LINEAR_SQUARE: cb_j = sgn(y_j) * y_j^2 with y_j = (2j - 15)/15.
    DYNAMIC_TREE: level 8 + p is +magnitude(p), level 7 - p is
    -magnitude(p), for the 3-bit patterns p (so levels 7 and 8 are zero)."""
    if codebook == LINEAR_SQUARE:
        j = np.arange(16, dtype=np.float64)
        y = 2.0 * j - 15.0
        return (y * np.abs(y)) / 225.0
    if codebook == DYNAMIC_TREE:
        mag = [_dynamic_tree_magnitude(p) for p in range(8)]
        return np.array([-mag[7 - j] for j in range(8)] + [mag[p] for p in range(8)], np.float64)
    raise ValueError(f"unknown codebook {codebook}")


def codebook_f32(codebook: int = LINEAR_SQUARE) -> np.ndarray:
    return codebook_f64(codebook).astype(np.float32)


def thresholds_f32(codebook: int = LINEAR_SQUARE) -> np.ndarray:
    """t_k = fp32(midpoint of cb_k and cb_{k+1}) for k = 0..14."""
    cb = codebook_f64(codebook)
    return ((cb[:-1] + cb[1:]) / 2.0).astype(np.float32)


def quantize(x: np.ndarray, block: int = QUANT_BLOCK, codebook: int = LINEAR_SQUARE):
    """Quantize a flat fp32 vector to (packed codes uint8, scales fp32).

    Returns ceil(n/2) code bytes and ceil(n/block) scales.
    """
    x = np.asarray(x, dtype=np.float32).ravel()
    n = x.size
    nb = (n + block - 1) // block
    padded = np.zeros(nb * block, dtype=np.float32)   # zeros never raise an absmax
    padded[:n] = x
    xb = padded.reshape(nb, block)
    scales = np.abs(xb).max(axis=1) if nb else np.zeros(0, np.float32)
    # numpy's max already returns NaN for a block holding a NaN and +Inf for
    # one holding +-Inf (and no NaN).
    thr = thresholds_f32(codebook)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (xb / scales[:, None]).astype(np.float32)    # one IEEE fp32 division
    codes = np.zeros(xb.shape, dtype=np.uint8)
    for k in range(thr.size):                 # code = #{k : v > t_k}
        codes += (v > thr[k]).astype(np.uint8)
    codes[scales == 0, :] = 7
    codes = codes.ravel()
    return pack_nibbles(codes[:n]), scales


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    n = codes.size
    padded = np.zeros(2 * ((n + 1) // 2), dtype=np.uint8)
    padded[:n] = codes
    return (padded[0::2] | (padded[1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray, n: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(2 * packed.size, dtype=np.uint8)
    out[0::2] = packed & 0xF
    out[1::2] = packed >> 4
    return out[:n]


def dequantize(packed: np.ndarray, scales: np.ndarray, n: int,
               block: int = QUANT_BLOCK, codebook: int = LINEAR_SQUARE) -> np.ndarray:
    """x_i = fp32(cb_code(i)) * scale(i // block), one fp32 multiply."""
    codes = unpack_nibbles(packed, n)
    cb = codebook_f32(codebook)
    s = np.repeat(np.asarray(scales, dtype=np.float32), block)[:n]
    return (cb[codes] * s).astype(np.float32)


# --------------------------------------------------------------------------
# Blocking ("Shampoo -- Second-Order Optimizer", "Blocked and distributed
# variants"): greedy chunks of at most max_block from index 0.
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Block:
    param: int
    r0: int
    c0: int
    m: int
    n: int


def chunks(extent: int, b: int):
    out, s = [], 0
    while s < extent:
        out.append((s, min(b, extent - s)))
        s += b
    return out


def partition(shapes, max_block: int = 1024) -> list[Block]:
    """Blocks in order: parameter, then row chunk, then column chunk.
    Block k owns factor 2k (L, dimension m) and 2k+1 (R, dimension n)."""
    blocks = []
    for p, (rows, cols) in enumerate(shapes):
        for r0, m in chunks(rows, max_block):
            for c0, n in chunks(cols, max_block):
                blocks.append(Block(p, r0, c0, m, n))
    return blocks


# --------------------------------------------------------------------------
# The per-factor steps.
# --------------------------------------------------------------------------

def ema_stats(S: np.ndarray, Gb: np.ndarray, beta: float, side: str) -> np.ndarray:
    """S <- beta S + (1 - beta) G G^T (side 'L') or G^T G (side 'R').
    Accumulated in fp64, stored fp32 ("Kronecker factorization";
    EMA per "Pitfalls")."""
    g = np.asarray(Gb, dtype=np.float64)
    outer = g @ g.T if side == "L" else g.T @ g
    s = beta * np.asarray(S, dtype=np.float64) + (1.0 - beta) * outer
    return s.astype(np.float32)


def compressed_stats(f: "Factor", Gb: np.ndarray, beta: float, side: str,
                     codebook: int = LINEAR_SQUARE) -> np.ndarray:
    """The statistic update when S is kept only as its 4-bit eigenbasis and
    eigenvalues ("4-bit Shampoo ...", abstract: the preconditioner is stored
    through its quantized eigenvector matrix): the previous statistic is
    rebuilt as U diag(lambda) U^T from the dequantized codes (no Bjorck, as
    for the roots), then S = beta U diag(lambda) U^T + (1 - beta) G G^T.
    Before the first refresh there is nothing stored: S = (1 - beta) G G^T,
    the EMA from zero.  fp64, stored fp32.  A gradient holding NaN/Inf
    leaves the statistic as stored (the rebuilt U diag(lambda) U^T; zero
    before the first refresh)."""
    g = np.asarray(Gb, dtype=np.float64)
    stored = np.zeros((f.d, f.d))
    if f.has_basis:
        U = dequantize(f.codes, f.scales, f.d * f.d, codebook=codebook).reshape(f.d, f.d).astype(np.float64)
        lam = np.asarray(f.lam, np.float64)
        stored = (U * lam[None, :]) @ U.T
    if not np.all(np.isfinite(g)):
        # a non-finite gradient leaves the statistic as stored
        return stored.astype(np.float32) if f.has_basis else np.asarray(f.S, np.float32)
    outer = g @ g.T if side == "L" else g.T @ g
    return (beta * stored + (1.0 - beta) * outer).astype(np.float32)


def bjorck(U: np.ndarray, iters: int) -> np.ndarray:
    """Orthogonality rectification U <- 1.5 U - 0.5 U (U^T U), ``iters`` times."""
    U = np.asarray(U, dtype=np.float64)
    for _ in range(iters):
        U = 1.5 * U - 0.5 * (U @ (U.T @ U))
    return U


def subspace_step(S: np.ndarray, U: np.ndarray, eps: float):
    """One orthogonal-iteration step: Y = (S + eps I) U, Y = QR with
    diag(R) >= 0; eigenvalues are the Rayleigh quotients max(q_i^T S q_i, 0).
    Returns (Q fp64, lambda fp64)."""
    S64 = np.asarray(S, dtype=np.float64)
    d = S64.shape[0]
    Y = (S64 + eps * np.eye(d)) @ np.asarray(U, dtype=np.float64)
    Q, R = np.linalg.qr(Y)
    sgn = np.where(np.diag(R) < 0, -1.0, 1.0)
    Q = Q * sgn[None, :]
    lam = np.maximum(np.sum(Q * (S64 @ Q), axis=0), 0.0)
    return Q, lam


def root_from_basis(U: np.ndarray, lam: np.ndarray, eps: float) -> np.ndarray:
    """P = U diag((lambda + eps)^(-1/4)) U^T ("Computing the inverse fourth
    root"; "Rotation, not just rescaling")."""
    U = np.asarray(U, dtype=np.float64)
    mu = (np.asarray(lam, dtype=np.float64) + eps) ** -0.25
    return (U * mu[None, :]) @ U.T


def newton_inverse_root(A: np.ndarray, p: int = 4, iters: int = 40, history=None) -> np.ndarray:
    """A^(-1/p) for a symmetric positive definite A by the coupled Newton
    iteration of "Shampoo -- Second-Order Optimizer", section "Computing the
    inverse fourth root": scale A by c = ||A||_F (an upper bound of the
    spectral norm, so the spectrum of M lies in (0, 1]), start from X = I and
    M = A / c, and repeat F = ((p + 1) I - M) / p, X <- X F, M <- F^p M.
    Then A^(-1/p) = X c^(-1/p).  A fixed number of iterations (a device path
    has no host test to stop on).  ``history``, if a list, receives (X, M)
    after every iteration.  fp64."""
    A = np.asarray(A, dtype=np.float64)
    d = A.shape[0]
    c = float(np.linalg.norm(A))
    I = np.eye(d)
    X, M = I.copy(), A / c
    for _ in range(iters):
        F = ((p + 1) * I - M) / p
        X = X @ F
        M = np.linalg.matrix_power(F, p) @ M
        if history is not None:
            history.append((X, M))
    return X * c ** (-1.0 / p)


def apply_roots(PL: np.ndarray, Gb: np.ndarray, PR: np.ndarray) -> np.ndarray:
    """D = L^(-1/4) G R^(-1/4) ("Kronecker factorization")."""
    return (np.asarray(PL, np.float64) @ np.asarray(Gb, np.float64)
            @ np.asarray(PR, np.float64))


# --------------------------------------------------------------------------
# State and the step driver.
# --------------------------------------------------------------------------

@dataclasses.dataclass
class Factor:
    d: int
    S: np.ndarray                         # fp32 d x d
    codes: np.ndarray | None = None       # uint8 ceil(d*d/2)
    scales: np.ndarray | None = None      # fp32 ceil(d*d/64)
    lam: np.ndarray | None = None         # fp32 d
    U64: np.ndarray | None = None         # quant=off: fp64 basis
    has_basis: bool = False
    q_last: np.ndarray | None = None      # pre-quantization Q of last refresh
    P: np.ndarray | None = None           # NEWTON: the fp32 root


ROOT_EIGEN = 0
ROOT_NEWTON = 1
ROOT_NEWTON_Q4 = 2


def refresh_factor(f: Factor, eps: float, bjorck_iters: int, quant: bool = True,
                   codebook: int = LINEAR_SQUARE) -> None:
    d = f.d
    if not f.has_basis:
        U = np.eye(d)
    elif quant:
        U = dequantize(f.codes, f.scales, d * d, codebook=codebook).reshape(d, d).astype(np.float64)
        U = bjorck(U, bjorck_iters)
    else:
        U = f.U64
    Q, lam = subspace_step(f.S, U, eps)
    f.q_last = Q
    if quant:
        f.codes, f.scales = quantize(Q.astype(np.float32).ravel(), codebook=codebook)
        f.lam = lam.astype(np.float32)
    else:
        f.U64 = Q
        f.lam = lam
    f.has_basis = True


def refresh_factor_newton(f: Factor, eps: float, iters: int, quantize_root: bool,
                          codebook: int = LINEAR_SQUARE) -> None:
    """The root by the coupled Newton iteration ("Computing the inverse
    fourth root"), P = (S + eps I)^(-1/4), kept in fp32 -- or, with
    quantize_root, quantized block-wise to 4 bits: quantizing the
    preconditioner itself, the alternative the 4-bit Shampoo abstract argues
    against."""
    A = np.asarray(f.S, np.float64) + eps * np.eye(f.d)
    P = newton_inverse_root(A, 4, iters)
    f.q_last = P
    if quantize_root:
        f.codes, f.scales = quantize(P.astype(np.float32).ravel(), codebook=codebook)
    else:
        f.P = P.astype(np.float32)
    f.has_basis = True


def factor_root(f: Factor, eps: float, quant: bool = True, codebook: int = LINEAR_SQUARE,
                root_method: int = ROOT_EIGEN) -> np.ndarray:
    if root_method == ROOT_NEWTON:
        return np.asarray(f.P, np.float64)
    if root_method == ROOT_NEWTON_Q4:
        return dequantize(f.codes, f.scales, f.d * f.d, codebook=codebook).reshape(f.d, f.d).astype(np.float64)
    if quant:
        U = dequantize(f.codes, f.scales, f.d * f.d, codebook=codebook).reshape(f.d, f.d)
        return root_from_basis(U, f.lam, eps)
    return root_from_basis(f.U64, f.lam, eps)


class Shampoo4Oracle:
    """The whole preconditioner step over a list of 2-D parameters."""

    def __init__(self, shapes, beta=0.95, eps=1e-6, bjorck_iters=5,
                 max_block=1024, quant=True, compressed=False, codebook=LINEAR_SQUARE,
                 root_method=ROOT_EIGEN, newton_iters=32):
        self.shapes = [tuple(s) for s in shapes]
        self.beta = float(beta)
        self.eps = float(eps)
        self.bjorck_iters = int(bjorck_iters)
        self.quant = bool(quant)
        self.compressed = bool(compressed)
        self.codebook = int(codebook)
        self.root_method = int(root_method)
        self.newton_iters = int(newton_iters)
        if self.compressed and not self.quant:
            raise ValueError("compressed statistics need the 4-bit basis")
        if self.root_method != ROOT_EIGEN and self.compressed:
            raise ValueError("the Newton root needs the fp32 statistic")
        self.blocks = partition(self.shapes, max_block)
        self.factors: list[Factor] = []
        for b in self.blocks:
            self.factors.append(Factor(b.m, np.zeros((b.m, b.m), np.float32)))
            self.factors.append(Factor(b.n, np.zeros((b.n, b.n), np.float32)))

    def block_view(self, grads, k: int) -> np.ndarray:
        b = self.blocks[k]
        return np.asarray(grads[b.param])[b.r0:b.r0 + b.m, b.c0:b.c0 + b.n]

    def update_stats(self, grads) -> None:
        for k in range(len(self.blocks)):
            g = self.block_view(grads, k)
            fl, fr = self.factors[2 * k], self.factors[2 * k + 1]
            if self.compressed:
                fl.S = compressed_stats(fl, g, self.beta, "L", self.codebook)
                fr.S = compressed_stats(fr, g, self.beta, "R", self.codebook)
            else:
                fl.S = ema_stats(fl.S, g, self.beta, "L")
                fr.S = ema_stats(fr.S, g, self.beta, "R")

    def refresh_roots(self) -> None:
        for f in self.factors:
            if self.root_method == ROOT_EIGEN:
                refresh_factor(f, self.eps, self.bjorck_iters, self.quant, self.codebook)
            else:
                refresh_factor_newton(f, self.eps, self.newton_iters, self.root_method == ROOT_NEWTON_Q4,
                                      self.codebook)

    def precondition(self, grads) -> list[np.ndarray]:
        if not all(f.has_basis for f in self.factors):
            raise RuntimeError("precondition before the first refresh")
        out = [np.zeros(s, np.float32) for s in self.shapes]
        for k, b in enumerate(self.blocks):
            PL = factor_root(self.factors[2 * k], self.eps, self.quant, self.codebook, self.root_method)
            PR = factor_root(self.factors[2 * k + 1], self.eps, self.quant, self.codebook, self.root_method)
            d = apply_roots(PL, self.block_view(grads, k), PR)
            out[b.param][b.r0:b.r0 + b.m, b.c0:b.c0 + b.n] = d.astype(np.float32)
        return out

    def step(self, t: int, grads, refresh_every: int) -> list[np.ndarray]:
        """Optimizer step t (1-based): stats, refresh on (t-1) % T == 0,
        then precondition."""
        self.update_stats(grads)
        if (t - 1) % refresh_every == 0:
            self.refresh_roots()
        return self.precondition(grads)
