"""Parity of the grafted weight update on the GPU against the grafting
oracle ("Shampoo -- Second-Order Optimizer", section "Grafting: borrow a
step size that already works"), three optimizer steps in a row, each fed the
library's own direction D of that step."""
import numpy as np
import pytest
import torch

from oracle import graft_oracle as GO
from gpu_helpers import cuda_f32, rel_fro

pytestmark = pytest.mark.gpu

# the graft stage is fp32 elementwise plus fp64 norms: an fp32-level bound on
# each parameter's step, and a few ulp on the moments
TOL_STEP = 1e-5
TOL_MOMENT = 1e-6

CASES = {
    # tensor-core tiles, a ragged tile of 76 rows, and a parameter whose
    # column count is not a multiple of 4 (scalar path)
    "mixed": ([(1100, 704), (64, 48), (33, 30)], 512),
    # one square tile at the factor size of the Llama-style layer set
    "square1024": ([(1024, 1024)], 1024),
    # many small tiles, ragged in both directions
    "small_tiles": ([(37, 29)], 16),
}


def _rng_list(shapes, seed, scale):
    r = np.random.default_rng(seed)
    return [(r.standard_normal(s) * scale).astype(np.float32) for s in shapes]


def _run(kind, shapes, max_block, steps=3, lr=1e-2, nan_tile=None, dir_norms=False, precision="tf32"):
    from bit_quantized_shampoo_b200 import api
    sh = api.Shampoo4(shapes, max_block=max_block, precision=precision)
    go = GO.GraftOracle(shapes, kind=GO.GRAFT_ADAM if kind == "adam" else GO.GRAFT_SGD,
                        max_block=max_block)
    state = sh.graft_state(kind)
    W = [cuda_f32(w) for w in _rng_list(shapes, 90, 0.02)]
    results = []
    for t in range(1, steps + 1):
        g_host = _rng_list(shapes, 100 + t, 1.0)
        if nan_tile is not None and t == steps:
            p, r, c = nan_tile
            g_host[p][r, c] = np.nan
        G = [cuda_f32(g) for g in g_host]
        sh.update_stats(G)
        if t == 1:
            sh.refresh_roots()
        D = sh.precondition(G)
        torch.cuda.synchronize()
        w_before = [w.cpu().numpy() for w in W]
        d_host = [d.cpu().numpy() for d in D]
        sh.graft_update(state, t, lr, G, D, W, kind=kind, dir_norms=dir_norms)
        torch.cuda.synchronize()
        want = go.step(t, lr, g_host, d_host, w_before)
        got = [w.cpu().numpy() for w in W]
        results.append((w_before, want, got))
        if kind == "adam":
            for p in range(len(shapes)):
                m, v = (x.cpu().numpy() for x in sh.graft_moments(state, p))
                assert rel_fro(m, go.m[p]) <= TOL_MOMENT, (t, p)
                assert rel_fro(v, go.v[p]) <= TOL_MOMENT, (t, p)
    return sh, go, results


@pytest.mark.parametrize("dir_norms", [False, True])
@pytest.mark.parametrize("kind", ["sgd", "adam"])
@pytest.mark.parametrize("case", sorted(CASES))
def test_graft_update_matches_oracle(kind, case, dir_norms):
    # dir_norms: ||D_b|| as the apply recorded it while writing D (the
    # oracle still takes it from D itself)
    shapes, max_block = CASES[case]
    sh, go, results = _run(kind, shapes, max_block, dir_norms=dir_norms)
    for t, (before, want, got) in enumerate(results, 1):
        for p in range(len(shapes)):
            step_o = want[p].astype(np.float64) - before[p]
            step_g = got[p].astype(np.float64) - before[p]
            e = rel_fro(step_g, step_o)
            print(f"{case} {kind} t={t} param {p} {shapes[p]}: step {e:.2e}")
            assert e <= TOL_STEP, (t, p)
    # ragged tiles have rank-deficient statistics whose QR may be redone in
    # fp64 (an informational flag); nothing else may be raised
    from bit_quantized_shampoo_b200 import _lib
    assert sh.status_flags() & ~_lib.FLAG_QR_FALLBACK == 0


def test_graft_recorded_norms_fp32_path():
    # the fp32-accurate apply (persistent 3xTF32 kernel) records no ||D||^2:
    # with dir_norms the update reads D for every tile
    shapes, max_block = [(1100, 704), (64, 48)], 512
    sh, go, results = _run("adam", shapes, max_block, steps=2, dir_norms=True, precision="fp32")
    for t, (before, want, got) in enumerate(results, 1):
        for p in range(len(shapes)):
            e = rel_fro(got[p].astype(np.float64) - before[p], want[p].astype(np.float64) - before[p])
            print(f"fp32 recorded norms t={t} param {p}: step {e:.2e}")
            assert e <= TOL_STEP, (t, p)


def test_graft_recorded_norms_need_a_precondition():
    from bit_quantized_shampoo_b200 import api, _lib
    shapes = [(128, 96)]
    sh = api.Shampoo4(shapes, max_block=128, precision="tf32")
    G = [cuda_f32(x) for x in _rng_list(shapes, 3, 1.0)]
    W = [torch.zeros(shapes[0], dtype=torch.float32, device="cuda")]
    sh.update_stats(G)
    with pytest.raises(_lib.Shampoo4Error):
        sh.graft_update(None, 1, 0.1, G, G, W, kind="sgd", dir_norms=True)


def test_graft_step_norm_per_tile_on_the_gpu():
    # graft_eps = 0: each tile's step has norm lr * ||G_b|| (SGD graft),
    # whatever D's scale -- the invariant the page states, at the library's
    # own output.
    from bit_quantized_shampoo_b200 import api
    shapes, max_block = [(300, 260)], 128
    sh = api.Shampoo4(shapes, max_block=max_block, precision="tf32")
    g = _rng_list(shapes, 7, 1.0)
    G = [cuda_f32(x) for x in g]
    sh.update_stats(G)
    sh.refresh_roots()
    D = sh.precondition(G)
    W = [torch.zeros(shapes[0], dtype=torch.float32, device="cuda")]
    sh.graft_update(None, 1, 0.5, G, D, W, kind="sgd", graft_eps=0.0)
    step = -W[0].cpu().numpy().astype(np.float64)
    for k in range(sh.nblocks):
        _, r0, c0, m, n = sh.block_info(k)
        s = step[r0:r0 + m, c0:c0 + n]
        assert np.isclose(np.linalg.norm(s), 0.5 * np.linalg.norm(g[0][r0:r0 + m, c0:c0 + n]), rtol=1e-6)


def test_graft_skips_a_nonfinite_tile():
    # A NaN in the last step's gradient: that tile keeps its weights and
    # moments, every other tile is updated as the oracle says.
    from bit_quantized_shampoo_b200 import _lib
    shapes, max_block = [(256, 384)], 128
    sh, go, results = _run("adam", shapes, max_block, steps=2, nan_tile=(0, 130, 200))
    before, want, got = results[-1]
    assert np.array_equal(got[0][128:256, 128:256], before[0][128:256, 128:256])
    assert rel_fro(got[0] - before[0], want[0] - before[0].astype(np.float64)) <= TOL_STEP
    assert sh.status_flags() & _lib.FLAG_NONFINITE_GRAD


def test_graft_flags_a_nonfinite_direction():
    # A finite gradient with an infinite direction entry: the tile's weights
    # stay, the flag says why, the other tiles move.
    from bit_quantized_shampoo_b200 import api, _lib
    shapes, max_block = [(64, 128)], 64
    sh = api.Shampoo4(shapes, max_block=max_block, precision="tf32")
    g = _rng_list(shapes, 11, 1.0)
    G = [cuda_f32(x) for x in g]
    sh.update_stats(G)
    D = [cuda_f32(x) for x in _rng_list(shapes, 12, 1.0)]
    D[0][5, 70] = float("inf")
    W = [cuda_f32(x) for x in _rng_list(shapes, 13, 0.02)]
    w0 = W[0].cpu().numpy()
    sh.graft_update(None, 1, 0.1, G, D, W, kind="sgd")
    got = W[0].cpu().numpy()
    assert np.array_equal(got[:, 64:], w0[:, 64:])
    assert not np.array_equal(got[:, :64], w0[:, :64])
    assert sh.status_flags() == _lib.FLAG_GRAFT_SKIPPED


def test_graft_rejects_overlapping_weights():
    from bit_quantized_shampoo_b200 import api, _lib
    shapes = [(64, 64)]
    sh = api.Shampoo4(shapes, precision="tf32")
    G = [cuda_f32(x) for x in _rng_list(shapes, 3, 1.0)]
    with pytest.raises(_lib.Shampoo4Error):
        sh.graft_update(None, 1, 0.1, G, G, G, kind="sgd")
