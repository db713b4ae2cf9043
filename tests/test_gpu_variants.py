"""The alternatives the 4-bit Shampoo abstract weighs the method against,
on the GPU against the oracle:
- the dynamic tree codebook in place of the linear square one (the
  refresh stage by stage from the library's incoming state, then the
  preconditioned update from its refreshed state);
- the inverse fourth root by the coupled Newton iteration ("Shampoo --
  Second-Order Optimizer", "Computing the inverse fourth root"), kept in
  fp32 (root method NEWTON) or quantized itself to 4 bits (NEWTON_Q4):
  the root against the oracle's fp64 Newton root of the library's own
  statistic, the stored codes bit-exact on the library's root, and the
  preconditioned update from the library's stored root."""
import numpy as np
import pytest
import torch

from oracle import shampoo4_oracle as O
from gpu_helpers import cuda_f32, gpu_factor, oracle_from_gpu, rel_fro, staged_refresh_all

pytestmark = pytest.mark.gpu

TOL = {"tf32": 2e-3, "fp32": 1e-5}
# fp32-accurate Newton products: measured about 4e-6 on condition numbers
# near 1e4 (the fp32 iteration's own drift, not the statistic's), so the
# root is held well inside the TF32 update tolerance
TOL_NEWTON_ROOT = 1e-4


def _grads(shapes, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal(s).astype(np.float32) for s in shapes]


@pytest.mark.parametrize("precision", ["tf32", "fp32"])
def test_dynamic_tree_codebook_refresh_and_precondition(precision):
    from bit_quantized_shampoo_b200 import api
    shapes = [(200, 130), (256, 512)]
    sh = api.Shampoo4(shapes, precision=precision, debug=True, codebook="dynamic_tree")
    eps = float(np.float32(1e-6))
    for rnd in range(2):
        for step in range(2):
            sh.update_stats([cuda_f32(g) for g in _grads(shapes, 700 + 10 * rnd + step)])
        torch.cuda.synchronize()
        incoming = {}
        for f in range(sh.nfactors):
            incoming[f] = gpu_factor(sh, f)
            incoming[f].has_basis = rnd > 0
        sh.refresh_roots()
        torch.cuda.synchronize()
        assert sh.status_flags() & ~0x10 == 0
        staged_refresh_all(sh, incoming, eps, 5, TOL[precision], f"dynamic tree {precision} round {rnd}",
                           codebook=O.DYNAMIC_TREE)
        orc = oracle_from_gpu(sh, shapes, has_basis=True)
        gs = _grads(shapes, 800 + rnd)
        out = sh.precondition([cuda_f32(g) for g in gs])
        torch.cuda.synchronize()
        for o, w in zip(out, orc.precondition(gs)):
            e = rel_fro(o.cpu().numpy(), w)
            print(f"dynamic tree {precision} round {rnd}: update {w.shape} {e:.2e}")
            assert e <= TOL[precision]


@pytest.mark.parametrize("precision", ["tf32", "fp32"])
@pytest.mark.parametrize("root", ["newton", "newton_q4"])
def test_newton_root(root, precision):
    from bit_quantized_shampoo_b200 import api
    shapes = [(200, 130), (512, 256), (1024, 1024)]
    iters = 32
    sh = api.Shampoo4(shapes, precision=precision, debug=True, root=root, newton_iters=iters)
    eps = float(np.float32(1e-6))
    for rnd in range(2):
        for step in range(3):
            sh.update_stats([cuda_f32(g) for g in _grads(shapes, 900 + 10 * rnd + step)])
        torch.cuda.synchronize()
        S = {f: gpu_factor(sh, f).S.astype(np.float64) for f in range(sh.nfactors)}
        sh.refresh_roots()
        torch.cuda.synchronize()
        assert sh.status_flags() == 0
        worst = 0.0
        for f in range(sh.nfactors):
            d = S[f].shape[0]
            A = S[f] + eps * np.eye(d)
            Pg = sh.debug_q(f).cpu().numpy().astype(np.float64)
            Po = O.newton_inverse_root(A, 4, iters)
            w, V = np.linalg.eigh(A)
            Pe = (V * w ** -0.25) @ V.T
            e, e_eig = rel_fro(Pg, Po), rel_fro(Pg, Pe)
            print(f"{root} {precision} round {rnd} factor {f} d={d}: root vs fp64 Newton {e:.2e}, "
                  f"vs eigh {e_eig:.2e}, kappa {w.max() / w.min():.2e}")
            worst = max(worst, e)
            if root == "newton":
                assert np.array_equal(sh.root_view(f).cpu().numpy(), Pg.astype(np.float32))
            else:
                g = gpu_factor(sh, f)
                oc, os_ = O.quantize(Pg.astype(np.float32).ravel())
                assert np.array_equal(g.codes, oc) and np.array_equal(g.scales, os_), f
        assert worst <= TOL_NEWTON_ROOT
        # the preconditioned update from the library's stored root
        orc = oracle_from_gpu(sh, shapes, has_basis=True)
        if root == "newton":
            for f in range(sh.nfactors):
                orc.factors[f].P = sh.root_view(f).cpu().numpy().copy()
        gs = _grads(shapes, 1000 + rnd)
        out = sh.precondition([cuda_f32(g) for g in gs])
        torch.cuda.synchronize()
        for o, wnt in zip(out, orc.precondition(gs)):
            e = rel_fro(o.cpu().numpy(), wnt)
            print(f"{root} {precision} round {rnd}: update {wnt.shape} {e:.2e}")
            assert e <= TOL[precision]
