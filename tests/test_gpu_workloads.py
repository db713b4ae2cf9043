"""Parity on the four smaller workloads, with their own shapes and gradient
distributions: one 128x128 weight; one 1024x1024 layer with a fixed rank-16
term; the 53 ResNet-50 convolutions with Student-t gradients; a 12-block
d = 768 transformer stack.  Two steps (a cold refresh, then a warm one):
every factor's Q is checked for orthonormality on the GPU, sampled factors'
refreshes stage by stage against the oracle from the same incoming state
(gpu_helpers.staged_refresh_check), sampled tiles of the preconditioned
update against the oracle from the library's state.
Collected last: the longest GPU tests."""
import numpy as np
import pytest
import torch

from oracle import shampoo4_oracle as O
from gpu_helpers import gpu_factor, rel_fro, staged_refresh_all

pytestmark = pytest.mark.gpu

TOL_TF32 = 2e-3


def _sample_factors(sh, limit=8):
    """Both factors of the first and last tiles, of the tile with the
    largest and the smallest factor, and of a tile with a factor whose edge
    is not a multiple of 4 (the CUDA-core path), when there is one."""
    dims = []
    for k in range(sh.nblocks):
        _, _, _, m, n = sh.block_info(k)
        dims.append((m, n))
    tiles = {0, sh.nblocks - 1,
             max(range(sh.nblocks), key=lambda k: max(dims[k])),
             min(range(sh.nblocks), key=lambda k: min(dims[k]))}
    odd = [k for k in range(sh.nblocks) if dims[k][0] % 4 or dims[k][1] % 4]
    if odd:
        tiles.add(odd[0])
    picks = sorted({f for k in tiles for f in (2 * k, 2 * k + 1)})
    return picks[:limit] if len(picks) > limit else picks


@pytest.mark.parametrize("wid", [1, 2, 3, 4])
def test_workload_sampled(wid):
    from bit_quantized_shampoo_b200 import api, _lib
    from bit_quantized_shampoo_b200.workloads import WORKLOADS, gradient

    w = WORKLOADS[wid]
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
    # rank-deficient or very ill-conditioned statistics may be redone in
    # fp64 (an informational flag); nothing else may be raised
    assert sh.status_flags() & ~_lib.FLAG_QR_FALLBACK == 0

    worst = 0.0
    for f in range(sh.nfactors):
        Q = sh.debug_q(f).double()
        d = Q.shape[0]
        e = float(torch.linalg.norm(Q.T @ Q - torch.eye(d, dtype=torch.float64, device=Q.device)) / d ** 0.5)
        worst = max(worst, e)
    print(f"workload {wid}: worst ||Q^T Q - I||_F / sqrt(d) over {sh.nfactors} factors: {worst:.3e}")
    assert worst <= 1e-5

    for f in picks:
        before[f].has_basis = True
    staged_refresh_all(sh, before, eps, w.bjorck_iters, TOL_TF32, f"workload {wid}")

    out = sh.precondition(dev(3))
    torch.cuda.synchronize()
    for k in sorted({f // 2 for f in picks}):
        p, r0, c0, m, n = sh.block_info(k)
        G = g_host[3][p][r0:r0 + m, c0:c0 + n]
        want = O.apply_roots(O.factor_root(gpu_factor(sh, 2 * k), eps), G,
                             O.factor_root(gpu_factor(sh, 2 * k + 1), eps))
        got = out[p][r0:r0 + m, c0:c0 + n].cpu().numpy()
        e = rel_fro(got, want)
        print(f"workload {wid} tile {k} ({m}x{n}): update {e:.2e}")
        assert e <= TOL_TF32, k
