"""Work and memory formulas for the preconditioner step.

These give the algorithmic FLOPs and bytes that the throughput figures are
divided by.  The per-step and memory terms restate "Shampoo -- Second-Order
Optimizer", sections "The full-matrix ideal", "Kronecker factorization" and
"The cost dial"; the refresh count follows the steps of the 4-bit refresh.
"""
from __future__ import annotations

# ---- page formulas ---------------------------------------------------------

def full_matrix_entries(m: int, n: int) -> int:
    """Full-matrix AdaGrad statistic H: (m n)^2 entries."""
    return (m * n) ** 2


def full_matrix_root_flops(m: int, n: int) -> float:
    """Inverse square root of H taken as (m n)^3 operations."""
    return float(m * n) ** 3


def kronecker_floats(m: int, n: int) -> int:
    """The two factors L (m^2) and R (n^2)."""
    return m * m + n * n


def kronecker_root_flops(m: int, n: int) -> float:
    """Two roots at about d^3 each."""
    return float(m) ** 3 + float(n) ** 3


def step_flops(m: int, n: int) -> float:
    """Statistics 2 m^2 n + 2 m n^2 plus applying both roots, the same again:
    4 m n (m + n)."""
    return 4.0 * m * n * (m + n)


def overhead_ratio(m: int, n: int, tokens: float) -> float:
    """Per-step Shampoo work over a layer's forward+backward (6 B m n)."""
    return step_flops(m, n) / (6.0 * tokens * m * n)


def adam_floats(m: int, n: int) -> int:
    return 2 * m * n


# ---- work of the implemented stages, per block or per factor ----------------

def stats_flops(m: int, n: int) -> float:
    """S_L += G G^T and S_R += G^T G for one m x n block."""
    return 2.0 * m * m * n + 2.0 * m * n * n


def stats_bytes(m: int, n: int) -> float:
    """Read G once, read and write both fp32 statistics."""
    return 4.0 * m * n + 8.0 * (m * m + n * n)


def refresh_flops(d: int, bjorck_iters: int = 5) -> float:
    """Per factor: Bjorck 4 t d^3, subspace product 2 d^3, QR 8/3 d^3
    (Householder count), Rayleigh 2 d^3."""
    return (4.0 * bjorck_iters + 2.0 + 8.0 / 3.0 + 2.0) * float(d) ** 3


def root_flops(d: int) -> float:
    """P = U diag(mu) U^T."""
    return 2.0 * float(d) ** 3


def apply_flops(m: int, n: int) -> float:
    """D = P_L G P_R."""
    return 2.0 * m * m * n + 2.0 * m * n * n


def precondition_flops(m: int, n: int) -> float:
    return root_flops(m) + root_flops(n) + apply_flops(m, n)


def codec_bytes_per_element(block: int = 64) -> float:
    """fp32 value, half a byte of code, a 4-byte scale per block."""
    return 4.0 + 0.5 + 4.0 / block
