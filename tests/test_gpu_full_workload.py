"""Parity at the full size of the Llama-style layer set (8 x 4096x11008 +
8 x 4096x4096 gradients, 480 tiles, 960 factors), in the launch
configuration bench.py times, on sampled outputs the oracle computes one by
one, and on properties checked for every factor."""
import numpy as np
import pytest
import torch

from oracle import shampoo4_oracle as O
from gpu_helpers import gpu_factor, rel_fro, staged_refresh_all

pytestmark = pytest.mark.gpu

TOL_TF32 = 2e-3


def _sample_factors(sh):
    """Factor indices: both sides of the first tile, of a tile of the last
    4096x11008 matrix's ragged column block (n = 768) and of the last tile."""
    picks = {0, 1, sh.nfactors - 2, sh.nfactors - 1}
    for k in range(sh.nblocks):
        p, r0, c0, m, n = sh.block_info(k)
        if n == 768:
            last768 = k
    picks |= {2 * last768, 2 * last768 + 1}
    return sorted(picks)


def test_llama_layer_set_sampled():
    from bit_quantized_shampoo_b200 import api
    from bit_quantized_shampoo_b200.workloads import WORKLOADS, gradient

    w = WORKLOADS[5]
    shapes = list(w.shapes)
    sh = api.Shampoo4(shapes, beta=w.beta, eps=w.eps, max_block=w.max_block, bjorck_iters=w.bjorck_iters,
                      precision="tf32", debug=True)
    eps = float(np.float32(w.eps))
    g_host = {s: [gradient(w, i, s) for i in range(len(shapes))] for s in (1, 2, 3)}
    dev = lambda s: [torch.from_numpy(g).cuda() for g in g_host[s]]

    sh.update_stats(dev(1))
    sh.refresh_roots()                                   # cold: U = I
    sh.update_stats(dev(2))
    torch.cuda.synchronize()
    picks = _sample_factors(sh)
    before = {f: gpu_factor(sh, f) for f in picks}       # incoming state of the warm refresh
    sh.refresh_roots()
    torch.cuda.synchronize()
    assert sh.status_flags() == 0

    # every factor: orthonormal Q (fp64 Gram on the GPU)
    worst = 0.0
    for f in range(sh.nfactors):
        Q = sh.debug_q(f).double()
        d = Q.shape[0]
        e = float(torch.linalg.norm(Q.T @ Q - torch.eye(d, dtype=torch.float64, device=Q.device)) / d ** 0.5)
        worst = max(worst, e)
    print(f"full workload: worst ||Q^T Q - I||_F / sqrt(d) over {sh.nfactors} factors: {worst:.3e}")
    assert worst <= 1e-5

    # sampled factors, stage by stage against the oracle from the same state
    for f in picks:
        before[f].has_basis = True
    staged_refresh_all(sh, before, eps, w.bjorck_iters, TOL_TF32, "full workload")

    # sampled tiles of the preconditioned update, from the library's state
    out = sh.precondition(dev(3))
    torch.cuda.synchronize()
    for k in sorted({f // 2 for f in picks}):
        p, r0, c0, m, n = sh.block_info(k)
        G = g_host[3][p][r0:r0 + m, c0:c0 + n]
        want = O.apply_roots(O.factor_root(gpu_factor(sh, 2 * k), eps), G,
                             O.factor_root(gpu_factor(sh, 2 * k + 1), eps))
        got = out[p][r0:r0 + m, c0:c0 + n].cpu().numpy()
        e = rel_fro(got, want)
        print(f"tile {k} ({m}x{n}): update {e:.2e}")
        assert e <= TOL_TF32, k
