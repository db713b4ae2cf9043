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
