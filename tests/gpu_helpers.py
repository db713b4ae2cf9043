"""Helpers shared by the GPU parity tests: read the library's state back and
hand it to the oracle ("state injection"), so each stage is compared from the
same incoming state."""
from __future__ import annotations

import numpy as np
import torch

from oracle import shampoo4_oracle as O


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def cuda_f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def gpu_factor(sh, f: int) -> O.Factor:
    """The library's factor f as an oracle Factor (copies to host)."""
    S, codes, scales, lam = sh.factor_views(f)
    torch.cuda.synchronize()
    fac = O.Factor(S.shape[0], S.cpu().numpy().copy())
    fac.codes = codes.cpu().numpy().copy()
    fac.scales = scales.cpu().numpy().copy()
    fac.lam = lam.cpu().numpy().copy()
    return fac


def oracle_from_gpu(sh, shapes, has_basis: bool) -> O.Shampoo4Oracle:
    cfg = sh.config
    orc = O.Shampoo4Oracle(shapes, beta=float(np.float32(cfg.beta)), eps=float(np.float32(cfg.eps)),
                           bjorck_iters=cfg.bjorck_iters, max_block=cfg.max_block)
    for f in range(len(orc.factors)):
        g = gpu_factor(sh, f)
        g.has_basis = has_basis
        orc.factors[f] = g
    return orc


def basis_root(Q, lam, eps):
    Q = np.asarray(Q, np.float64)
    mu = (np.asarray(lam, np.float64) + eps) ** -0.25
    return (Q * mu[None, :]) @ Q.T


def refresh_errors(sh, orc, eps):
    """After sh.refresh_roots() and orc.refresh_roots() from the same incoming
    state: per factor (d, ||Q^T Q - I||_F/sqrt(d), lambda excess, root excess),
    with the requantized codes checked bit-exact against the oracle quantizer
    applied to the library's own Q.  The lambda and root excesses are taken
    over the fp32-accurate arithmetic's resolution, as in the stage tests:
    about 16 u lambda_max for lambda and u kappa for the basis-invariant root
    (u = 2^-21), nothing pinned beyond u32 kappa >= 1."""
    out = []
    for f in range(sh.nfactors):
        d = orc.factors[f].d
        Qg = sh.debug_q(f).cpu().numpy().astype(np.float64)
        g = gpu_factor(sh, f)
        oc, os_ = O.quantize(Qg.astype(np.float32).ravel())
        assert np.array_equal(g.codes, oc) and np.array_equal(g.scales, os_), f
        orth = float(np.linalg.norm(Qg.T @ Qg - np.eye(d)) / np.sqrt(d))
        Qo, lo = orc.factors[f].q_last, orc.factors[f].lam.astype(np.float64)
        lg = g.lam.astype(np.float64)
        big = lo > 1e3 * eps
        slack = 16 * 2.0 ** -21 * lo.max()
        excess = np.maximum(np.abs(lg - lo) - slack, 0.0)
        lam_err = float(np.max(excess[big] / lo[big])) if big.any() else 0.0
        kappa = (lo.max() + eps) / (lo.min() + eps)
        root_err = rel_fro(basis_root(Qg, lo, eps), basis_root(Qo, lo, eps))
        root_err = max(root_err - 2.0 ** -21 * kappa, 0.0)
        if 6e-8 * kappa >= 1.0:
            root_err = 0.0
        out.append((d, orth, lam_err, root_err))
    return out
