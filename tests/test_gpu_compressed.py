"""Compressed statistics on the GPU ("4-bit Shampoo for Memory-Efficient
Network Training", abstract: the preconditioner is kept through its 4-bit
eigenvector matrix): each update_stats rebuilds S = beta U diag(lambda) U^T +
(1 - beta) G G^T from the stored codes and eigenvalues, and the refresh that
follows stores the new statistic.  Each stage is compared with the oracle
fed the library's incoming state."""
import numpy as np
import pytest
import torch

from oracle import shampoo4_oracle as O
from gpu_helpers import cuda_f32, gpu_factor, oracle_from_gpu, rel_fro, staged_refresh_all

pytestmark = pytest.mark.gpu

TOL = {"tf32": 2e-3, "fp32": 1e-5}
SHAPE_SETS = {
    # tensor-core tiles, a ragged one and a CUDA-core factor (d = 130)
    "ragged": [(64, 147), (200, 130), (96, 576)],
    # the factor sizes of the Llama-style layer set
    "full_1024": [(1024, 768)],
}
CASES = [("ragged", "tf32"), ("ragged", "fp32"), ("full_1024", "tf32")]


def _grads(shapes, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return [(rng.standard_normal(s) * scale).astype(np.float32) for s in shapes]


def _incoming(sh, has_basis):
    facs = []
    for f in range(sh.nfactors):
        g = gpu_factor(sh, f)
        g.has_basis = has_basis
        facs.append(g)
    return facs


@pytest.mark.parametrize("which,precision", CASES)
def test_compressed_steps_match_oracle(which, precision):
    from bit_quantized_shampoo_b200 import api
    shapes = SHAPE_SETS[which]
    sh = api.Shampoo4(shapes, precision=precision, compressed=True, debug=True)
    beta = float(np.float32(sh.config.beta))
    eps = float(np.float32(sh.config.eps))
    blocks = O.partition(shapes, 1024)
    for rnd in range(3):                       # cold refresh, then two warm ones
        incoming = _incoming(sh, has_basis=rnd > 0)
        gs = _grads(shapes, 500 + rnd)
        sh.update_stats([cuda_f32(g) for g in gs])
        torch.cuda.synchronize()
        # (i) the rebuilt-and-updated statistic
        worst = 0.0
        for k, b in enumerate(blocks):
            G = gs[b.param][b.r0:b.r0 + b.m, b.c0:b.c0 + b.n]
            for side, f in (("L", 2 * k), ("R", 2 * k + 1)):
                want = O.compressed_stats(incoming[f], G, beta, side)
                S = sh.factor_views(f)[0].cpu().numpy()
                assert np.array_equal(S, S.T), f
                worst = max(worst, rel_fro(S, want))
        print(f"compressed {which} {precision} round {rnd}: stats {worst:.2e}")
        assert worst <= TOL[precision]
        # (ii) the refresh from the rebuilt statistic, stage by stage
        before = {}
        for f in range(sh.nfactors):
            before[f] = gpu_factor(sh, f)
            before[f].has_basis = rnd > 0
        sh.refresh_roots()
        torch.cuda.synchronize()
        flags = sh.status_flags()
        assert flags & ~0x10 == 0, flags
        recs = staged_refresh_all(sh, before, eps, 5, TOL[precision], f"compressed {which} {precision} round {rnd}")
        assert max(r["orth"] for r in recs) <= 1e-5
    # (iii) precondition from the stored codes
    orc2 = oracle_from_gpu(sh, shapes, has_basis=True)
    gs = _grads(shapes, 600)
    out = sh.precondition([cuda_f32(g) for g in gs])
    torch.cuda.synchronize()
    for o, w in zip(out, orc2.precondition(gs)):
        assert rel_fro(o.cpu().numpy(), w) <= TOL[precision]


def test_compressed_call_order():
    from bit_quantized_shampoo_b200 import api
    from bit_quantized_shampoo_b200._lib import Shampoo4Error
    shapes = [(64, 96)]
    sh = api.Shampoo4(shapes, compressed=True)
    G = [cuda_f32(g) for g in _grads(shapes, 1)]
    with pytest.raises(Shampoo4Error) as e:          # nothing to store yet
        sh.refresh_roots()
    assert e.value.status == 3
    sh.update_stats(G)
    with pytest.raises(Shampoo4Error) as e:          # the first update is not stored yet
        sh.update_stats(G)
    assert e.value.status == 3
    sh.refresh_roots()
    sh.update_stats(G)                               # stored: the next update may run
    sh.refresh_roots()
    torch.cuda.synchronize()
    # a 64-row tile's 96 x 96 statistic is rank-deficient: its QR may be
    # redone in fp64 (an informational flag); nothing else may be raised
    assert sh.status_flags() & ~0x10 == 0


def test_compressed_nonfinite_gradient_keeps_the_stored_statistic():
    from bit_quantized_shampoo_b200 import api
    from bit_quantized_shampoo_b200._lib import FLAG_NONFINITE_GRAD
    shapes = [(128, 96), (64, 64)]
    sh = api.Shampoo4(shapes, compressed=True, precision="fp32")
    beta = float(np.float32(sh.config.beta))
    sh.update_stats([cuda_f32(g) for g in _grads(shapes, 2)])
    sh.refresh_roots()
    torch.cuda.synchronize()
    incoming = _incoming(sh, has_basis=True)
    gs = _grads(shapes, 3)
    gs[0][10, 20] = np.nan
    sh.update_stats([cuda_f32(g) for g in gs])
    assert sh.status_flags() & FLAG_NONFINITE_GRAD
    blocks = O.partition(shapes, 1024)
    for k, b in enumerate(blocks):
        G = gs[b.param][b.r0:b.r0 + b.m, b.c0:b.c0 + b.n]
        for side, f in (("L", 2 * k), ("R", 2 * k + 1)):
            want = O.compressed_stats(incoming[f], G, beta, side)
            S = sh.factor_views(f)[0].cpu().numpy()
            assert rel_fro(S, want) <= TOL["fp32"], f
