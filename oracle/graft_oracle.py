"""CPU oracle for grafting and the weight update (fp64, numpy).

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the test suite,
the package's smoke check and the benchmark's CPU-baseline leg may import it.

What it computes ("Shampoo -- Second-Order Optimizer", section "Grafting:
borrow a step size that already works"): Shampoo supplies the direction D of
each block, a method with a tuned step size supplies the per-block step
norm, and the weight moves by

    step_b = lr * ||d_graft_b||_F / (||D_b||_F + graft_eps) * D_b,
    W_b   <- W_b - step_b,

with the norms taken per tile of the blocked partition (the page lets the
norms be taken over a whole layer or over one block; the tiles are what is
preconditioned independently, section "Blocked and distributed variants").

d_graft is the step the grafted method would take, without its learning
rate:
  SGD   d_graft = G.
  Adam  the textbook method (Kingma and Ba, "Adam: A Method for Stochastic
        Optimization", ICLR 2015, Algorithm 1): m <- b1 m + (1-b1) G,
        v <- b2 v + (1-b2) G*G, m_hat = m / (1-b1^t), v_hat = v / (1-b2^t),
        d_graft = m_hat / (sqrt(v_hat) + adam_eps), t the 1-based step.

Readings where the page is silent (repeated in the design notes):
  norms     per tile, Frobenius, accumulated in fp64.
  ratio     lr * ||d_graft_b|| / (||D_b|| + graft_eps); a zero denominator
            gives a zero step (D_b is then zero as well).
  moments   stored fp32, updated in fp64 and rounded on storage (as the
            statistics are); d_graft is formed from the stored values.
  weights   stored fp32; W - step is formed in fp64 and rounded once.
  non-finite  a tile whose gradient holds NaN/Inf is skipped whole: its
            moments and weights stay unchanged (the statistics update leaves
            such a tile's statistics unchanged too).  A tile whose squared
            norms are not finite, or whose step factor lr * ratio is not
            finite in fp32, keeps its weights (its moments are updated).
"""
from __future__ import annotations

import numpy as np

from .shampoo4_oracle import partition

GRAFT_SGD = 0
GRAFT_ADAM = 1


def adam_moments(m: np.ndarray, v: np.ndarray, g: np.ndarray, beta1: float, beta2: float):
    """One moment update; fp32 in, fp64 arithmetic, fp32 out."""
    g = np.asarray(g, np.float64)
    m1 = (beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g).astype(np.float32)
    v1 = (beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g).astype(np.float32)
    return m1, v1


def adam_direction(m: np.ndarray, v: np.ndarray, t: int, beta1: float, beta2: float,
                   adam_eps: float) -> np.ndarray:
    """Bias-corrected Adam direction from the (already updated) moments."""
    mh = np.asarray(m, np.float64) / (1.0 - beta1 ** t)
    vh = np.asarray(v, np.float64) / (1.0 - beta2 ** t)
    return mh / (np.sqrt(vh) + adam_eps)


def graft_ratio(d_graft: np.ndarray, D: np.ndarray, graft_eps: float) -> float:
    """||d_graft||_F / (||D||_F + graft_eps), 0 when the denominator is 0."""
    ng = float(np.sqrt(np.sum(np.asarray(d_graft, np.float64) ** 2)))
    den = float(np.sqrt(np.sum(np.asarray(D, np.float64) ** 2))) + graft_eps
    return ng / den if den > 0.0 else 0.0


class GraftOracle:
    """Grafted weight update over the same blocked partition as the
    preconditioner."""

    def __init__(self, shapes, kind=GRAFT_ADAM, beta1=0.9, beta2=0.999, adam_eps=1e-8,
                 graft_eps=1e-16, max_block=1024):
        self.shapes = [tuple(s) for s in shapes]
        self.kind = int(kind)
        # the library takes these as fp32; use the same values here
        self.beta1 = float(np.float32(beta1))
        self.beta2 = float(np.float32(beta2))
        self.adam_eps = float(np.float32(adam_eps))
        self.graft_eps = float(np.float32(graft_eps))
        self.blocks = partition(self.shapes, max_block)
        self.m = [np.zeros(s, np.float32) for s in self.shapes]
        self.v = [np.zeros(s, np.float32) for s in self.shapes]

    def step(self, t: int, lr: float, grads, dirs, weights) -> list[np.ndarray]:
        """Returns the new weights; updates the moments in place."""
        lr = float(np.float32(lr))
        out = [np.array(w, np.float32, copy=True) for w in weights]
        for b in self.blocks:
            rs = slice(b.r0, b.r0 + b.m)
            cs = slice(b.c0, b.c0 + b.n)
            g = np.asarray(grads[b.param], np.float32)[rs, cs]
            if not np.all(np.isfinite(g)):
                continue
            if self.kind == GRAFT_ADAM:
                m1, v1 = adam_moments(self.m[b.param][rs, cs], self.v[b.param][rs, cs], g,
                                      self.beta1, self.beta2)
                self.m[b.param][rs, cs] = m1
                self.v[b.param][rs, cs] = v1
                dg = adam_direction(m1, v1, t, self.beta1, self.beta2, self.adam_eps)
            else:
                dg = np.asarray(g, np.float64)
            D = np.asarray(dirs[b.param], np.float32)[rs, cs]
            ng2 = float(np.sum(np.asarray(dg, np.float64) ** 2))
            nd2 = float(np.sum(np.asarray(D, np.float64) ** 2))
            if not (np.isfinite(ng2) and np.isfinite(nd2)):
                continue
            r = lr * graft_ratio(dg, D, self.graft_eps)
            if not abs(r) <= float(np.finfo(np.float32).max):
                continue
            w = np.asarray(weights[b.param], np.float64)[rs, cs]
            out[b.param][rs, cs] = (w - r * np.asarray(D, np.float64)).astype(np.float32)
        return out
