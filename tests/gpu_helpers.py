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
                           bjorck_iters=cfg.bjorck_iters, max_block=cfg.max_block, codebook=cfg.codebook,
                           root_method=cfg.root_method, newton_iters=cfg.newton_iters or 32)
    for f in range(len(orc.factors)):
        g = gpu_factor(sh, f)
        g.has_basis = has_basis
        orc.factors[f] = g
    return orc


def basis_root(Q, lam, eps):
    Q = np.asarray(Q, np.float64)
    mu = (np.asarray(lam, np.float64) + eps) ** -0.25
    return (Q * mu[None, :]) @ Q.T


# Unit roundoff of the fp32-accurate (3xTF32) products that the subspace
# step, the QR and the Rayleigh quotients run on.
U21 = 2.0 ** -21
# The refresh gates allow the stage tolerance plus this multiple of the
# oracle's own spread (the "band" below).
BAND_FACTOR = 4.0


def _oracle_spread(S, U, eps, Qo, lo, big, seeds=3):
    """The oracle's own sensitivity at this input: the largest change of
    lambda_i (relative, over lambda_i > 1e3 eps) and of the basis-invariant
    root when S and U carry independent relative perturbations of 2^-21 --
    the rounding any fp32-accurate arithmetic leaves in the subspace
    product, the QR and the Rayleigh product.  Rank-deficient or
    ill-conditioned statistics make the last columns of the QR inside S's
    range, and the eigen-directions next to eps, sensitive far beyond 2^-21;
    this measures by how much, for this very factor."""
    S = np.asarray(S, np.float64)
    U = np.asarray(U, np.float64)
    band_lam = band_root = 0.0
    ref = basis_root(Qo, lo, eps)
    for seed in range(seeds):
        rng = np.random.default_rng(9000 + seed)
        E = rng.standard_normal(S.shape)
        Sp = S * (1.0 + U21 * (E + E.T) / np.sqrt(2.0))
        Up = U * (1.0 + U21 * rng.standard_normal(U.shape))
        Qp, lp = O.subspace_step(Sp, Up, eps)
        if big.any():
            band_lam = max(band_lam, float(np.max(np.abs(lp - lo)[big] / lo[big])))
        band_root = max(band_root, rel_fro(basis_root(Qp, lo, eps), ref))
    return band_lam, band_root


def staged_refresh_check(sh, f, incoming, eps, bjorck_iters, tol, end_to_end=True, codebook=O.LINEAR_SQUARE):
    """Factor f's last refresh against the oracle, stage by stage, from the
    library's own incoming state (``incoming``: the factor as read before the
    refresh, has_basis set as the library had it).  Needs a handle made with
    debug=True (the capture of the rectified basis and of Q).

    Stage 1, dequantize + Bjorck: the library's rectified basis against
    oracle.bjorck(oracle.dequantize(codes)) -- relative Frobenius <= tol
    (the identity, exactly, on a first refresh).
    Stage 2, subspace step + QR + Rayleigh quotients, fed the library's own
    rectified basis: lambda_i (relative, lambda_i > 1e3 eps) and the
    basis-invariant root Q diag((lambda_o + eps)^-1/4) Q^T (relative
    Frobenius) each within tol + BAND_FACTOR x the oracle's own spread.
    Stage 3, requantization: codes and scales bit-exact with the oracle's
    quantizer applied to the library's Q.
    Also, not gated: the same lambda and root errors against the oracle's
    whole fp64 refresh from the incoming codes (fp64 Bjorck), which adds the
    sensitivity of stage 2 to the TF32 Bjorck's rounding.

    Returns a dict of the raw errors, the bands and the verdicts."""
    d = incoming.d
    Ug = sh.debug_rectified(f).cpu().numpy().astype(np.float64)
    Qg = sh.debug_q(f).cpu().numpy().astype(np.float64)
    g = gpu_factor(sh, f)
    rec = {"factor": f, "d": d}
    # stage 1
    if incoming.has_basis:
        U0 = O.dequantize(incoming.codes, incoming.scales, d * d, codebook=codebook).reshape(d, d).astype(np.float64)
        Uo = O.bjorck(U0, bjorck_iters)
        rec["bjorck"] = rel_fro(Ug, Uo)
        rec["bjorck_ok"] = rec["bjorck"] <= tol
    else:
        rec["bjorck"] = float(np.max(np.abs(Ug - np.eye(d))))
        rec["bjorck_ok"] = rec["bjorck"] == 0.0
    # stage 2, from the library's rectified basis
    Qo, lo = O.subspace_step(incoming.S, Ug, eps)
    lg = g.lam.astype(np.float64)
    big = lo > 1e3 * eps
    rec["lam"] = float(np.max(np.abs(lg - lo)[big] / lo[big])) if big.any() else 0.0
    rec["root"] = rel_fro(basis_root(Qg, lo, eps), basis_root(Qo, lo, eps))
    rec["band_lam"], rec["band_root"] = _oracle_spread(incoming.S, Ug, eps, Qo, lo, big)
    rec["lam_ok"] = rec["lam"] <= tol + BAND_FACTOR * rec["band_lam"]
    rec["root_ok"] = rec["root"] <= tol + BAND_FACTOR * rec["band_root"]
    rec["banded"] = bool(BAND_FACTOR * max(rec["band_lam"], rec["band_root"]) > tol)
    rec["orth"] = float(np.linalg.norm(Qg.T @ Qg - np.eye(d)) / np.sqrt(d))
    # stage 3
    oc, os_ = O.quantize(Qg.astype(np.float32).ravel(), codebook=codebook)
    rec["codes_ok"] = bool(np.array_equal(g.codes, oc) and np.array_equal(g.scales, os_))
    if end_to_end:
        e = O.Factor(d, incoming.S, codes=incoming.codes, scales=incoming.scales, lam=incoming.lam,
                     has_basis=incoming.has_basis)
        O.refresh_factor(e, eps, bjorck_iters, codebook=codebook)
        le = e.lam.astype(np.float64)
        bige = le > 1e3 * eps
        rec["e2e_lam"] = float(np.max(np.abs(lg - le)[bige] / le[bige])) if bige.any() else 0.0
        rec["e2e_root"] = rel_fro(basis_root(Qg, le, eps), basis_root(e.q_last, le, eps))
    rec["ok"] = bool(rec["bjorck_ok"] and rec["lam_ok"] and rec["root_ok"] and rec["codes_ok"])
    return rec


def format_record(tag, r):
    s = (f"{tag} factor {r['factor']} d={r['d']}: bjorck {r['bjorck']:.2e} lambda {r['lam']:.2e} "
         f"(band {r['band_lam']:.2e}) root {r['root']:.2e} (band {r['band_root']:.2e}) orth {r['orth']:.2e}")
    if "e2e_lam" in r:
        s += f" | whole fp64 refresh: lambda {r['e2e_lam']:.2e} root {r['e2e_root']:.2e}"
    return s + ("" if r["ok"] else "  FAIL")


def staged_refresh_all(sh, incoming, eps, bjorck_iters, tol, tag, end_to_end=True, codebook=O.LINEAR_SQUARE):
    """staged_refresh_check over the factors in ``incoming`` (factor index ->
    incoming Factor, has_basis set); prints one line per factor and how many
    needed the band, and asserts every verdict.  Returns the records."""
    recs = []
    for f in sorted(incoming):
        r = staged_refresh_check(sh, f, incoming[f], eps, bjorck_iters, tol, end_to_end, codebook)
        print(format_record(tag, r))
        recs.append(r)
    nb = sum(r["banded"] for r in recs)
    print(f"{tag}: {len(recs)} factors checked, {nb} with BAND_FACTOR x band above the tolerance; "
          f"worst bjorck {max(r['bjorck'] for r in recs):.2e} lambda {max(r['lam'] for r in recs):.2e} "
          f"root {max(r['root'] for r in recs):.2e}")
    bad = [r["factor"] for r in recs if not r["ok"]]
    assert not bad, f"{tag}: factors {bad} outside the staged refresh gates"
    return recs


def update_band(fl, fr, G, eps, seeds=2):
    """The oracle's own spread of the preconditioned update D = P_L G P_R
    (roots from the factors' codes and eigenvalues) when every operand of
    the TF32 products -- U diag(mu), U, G and the intermediate P_L G --
    carries an independent relative perturbation of the size of TF32
    round-to-nearest (uniform in +-2^-11).  A root that leans on the
    eigen-directions next to eps (the first refresh of a statistic, or a
    rank-deficient one) amplifies that rounding through cancellation in
    P_L G P_R."""
    def root(f, rng):
        U = O.dequantize(f.codes, f.scales, f.d * f.d).reshape(f.d, f.d).astype(np.float64)
        mu = (np.asarray(f.lam, np.float64) + eps) ** -0.25
        jit = lambda X: X * (1.0 + 2.0 ** -11 * rng.uniform(-1, 1, X.shape))
        return jit(U * mu[None, :]) @ jit(U).T
    ref = O.apply_roots(O.factor_root(fl, eps), G, O.factor_root(fr, eps))
    band = 0.0
    for seed in range(seeds):
        rng = np.random.default_rng(7000 + seed)
        PL, PR = root(fl, rng), root(fr, rng)
        jit = lambda X: X * (1.0 + 2.0 ** -11 * rng.uniform(-1, 1, X.shape))
        B = jit(jit(PL) @ jit(np.asarray(G, np.float64)))
        band = max(band, rel_fro(B @ jit(PR), ref))
    return band
