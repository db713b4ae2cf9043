"""The seeded input recipe: every workload's gradients have the shapes and
the distribution the recipe states, are reproducible from their seed, and
change from step to step.  No GPU."""
import numpy as np
import pytest

from bit_quantized_shampoo_b200.workloads import WORKLOADS, gradient, resnet50_conv_shapes, u_like


def test_resnet50_has_53_convolutions_with_the_published_widths():
    s = resnet50_conv_shapes()
    assert len(s) == 53 and s[0] == (64, 147)
    assert max(r for r, _ in s) == 2048 and max(c for _, c in s) == 4608      # 512 * 9
    # every bottleneck's expand conv has 4x the width of its reduce conv
    assert sum(1 for r, c in s if r == 4 * c) >= 16


@pytest.mark.parametrize("wid,matrix", [(1, 0), (4, 2), (5, 9)])
def test_normal_gradients_have_the_stated_scale(wid, matrix):
    w = WORKLOADS[wid]
    g = gradient(w, matrix, 1)
    assert g.shape == w.shapes[matrix] and g.dtype == np.float32 and g.flags["C_CONTIGUOUS"]
    x = g.astype(np.float64).ravel()
    n = x.size
    assert abs(x.mean()) <= 5 * w.scale / np.sqrt(n)
    assert abs(x.std() / w.scale - 1.0) <= 5 * np.sqrt(2.0 / n) + 1e-3
    assert np.array_equal(g, gradient(w, matrix, 1))                         # reproducible
    assert not np.array_equal(g, gradient(w, matrix, 2))                     # a new draw per step


def test_lowrank_workload_carries_a_fixed_rank_16_term():
    w = WORKLOADS[2]
    g1, g2 = gradient(w, 0, 1).astype(np.float64), gradient(w, 0, 2).astype(np.float64)
    # the fixed term survives in the mean of two steps; its 16 singular
    # values stand far above the fresh noise's (about 0.02 * 2 sqrt(1024))
    s = np.linalg.svd(0.5 * (g1 + g2), compute_uv=False)
    noise_edge = 0.02 / np.sqrt(2.0) * 2.0 * np.sqrt(1024)
    assert s[15] > 5 * noise_edge and s[16] < 1.5 * noise_edge
    # the difference of two steps is pure noise of variance 2 * 0.02^2
    d = (g1 - g2).ravel()
    assert abs(d.std() / (0.02 * np.sqrt(2.0)) - 1.0) < 0.01


def test_student_t_workload_is_heavy_tailed_with_the_stated_scale():
    w = WORKLOADS[3]
    x = np.concatenate([gradient(w, i, 1).astype(np.float64).ravel() for i in range(w.nparams)])
    # t with 4 degrees of freedom: variance nu / (nu - 2) = 2 (times scale^2),
    # and far heavier tails than a normal of that variance
    assert abs(x.var() / (2.0 * w.scale ** 2) - 1.0) < 0.1
    sd = x.std()
    assert np.mean(np.abs(x) > 5 * sd) > 50 * 5.7e-7                          # normal: 5.7e-7


def test_u_like_matches_an_orthogonal_matrix_entry_scale():
    u = u_like(256, 3, count=2)
    assert u.shape == (2, 256, 256) and u.dtype == np.float32
    assert abs(np.mean(np.sum(u.astype(np.float64) ** 2, axis=1)) - 1.0) < 0.03   # unit columns on average
