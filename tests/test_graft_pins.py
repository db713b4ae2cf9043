"""Pins for the grafting oracle ("Shampoo -- Second-Order Optimizer", section
"Grafting: borrow a step size that already works"; Adam per Kingma and Ba,
ICLR 2015, Algorithm 1).  Each test checks the oracle against a closed form,
a special case that reduces to a textbook method, or an invariant the page
states; no GPU needed."""
import numpy as np
import pytest

from oracle import graft_oracle as GO


def _rng(seed):
    return np.random.default_rng(seed)


def test_adam_constant_gradient_closed_form():
    # For a gradient that never changes, bias correction makes m_hat = g and
    # v_hat = g^2 exactly at every step, so d = g / (|g| + eps).
    g = _rng(1).standard_normal((7, 5)).astype(np.float32)
    m = np.zeros_like(g)
    v = np.zeros_like(g)
    b1, b2, eps = 0.9, 0.999, 1e-3
    for t in range(1, 8):
        m, v = GO.adam_moments(m, v, g, b1, b2)
        d = GO.adam_direction(m, v, t, b1, b2, eps)
        want = g.astype(np.float64) / (np.abs(g.astype(np.float64)) + eps)
        # the moments are stored in fp32: a few ulp per step
        assert np.max(np.abs(d - want)) <= 2e-6, t


def test_adam_two_steps_unrolled():
    # m_2 = b1 (1-b1) g1 + (1-b1) g2 and v_2 = b2 (1-b2) g1^2 + (1-b2) g2^2,
    # divided by (1 - b^2): the recursion unrolled by hand.
    r = _rng(2)
    g1, g2 = (r.standard_normal(33).astype(np.float32) for _ in range(2))
    b1, b2, eps = 0.8, 0.95, 1e-8
    m, v = GO.adam_moments(np.zeros(33, np.float32), np.zeros(33, np.float32), g1, b1, b2)
    m, v = GO.adam_moments(m, v, g2, b1, b2)
    d = GO.adam_direction(m, v, 2, b1, b2, eps)
    a1, a2 = g1.astype(np.float64), g2.astype(np.float64)
    mh = (b1 * (1 - b1) * a1 + (1 - b1) * a2) / (1 - b1 * b1)
    vh = (b2 * (1 - b2) * a1 * a1 + (1 - b2) * a2 * a2) / (1 - b2 * b2)
    assert np.allclose(d, mh / (np.sqrt(vh) + eps), rtol=5e-6, atol=0)


def test_sgd_graft_on_the_gradient_itself_is_sgd():
    # D = G: the ratio is ||G|| / ||G|| = 1, so the grafted step is plain SGD.
    shapes = [(40, 70), (9, 9)]
    r = _rng(3)
    G = [r.standard_normal(s).astype(np.float32) for s in shapes]
    W = [r.standard_normal(s).astype(np.float32) for s in shapes]
    go = GO.GraftOracle(shapes, kind=GO.GRAFT_SGD, graft_eps=0.0, max_block=32)
    out = go.step(1, 0.05, G, G, W)
    lr = float(np.float32(0.05))
    for w, g, o in zip(W, G, out):
        assert np.array_equal(o, (w.astype(np.float64) - lr * g.astype(np.float64)).astype(np.float32))


def test_step_norm_is_the_graft_norm_and_direction_is_D():
    # With graft_eps = 0 and W = 0, each tile's step has norm lr * ||d_graft||
    # and points along D.  Adam's first step with adam_eps = 0 is sign(G), so
    # ||d_graft|| = sqrt(#tile elements) whatever G and D are.
    shapes = [(50, 37)]
    max_block = 16
    r = _rng(4)
    G = [r.standard_normal(shapes[0]).astype(np.float32)]
    D = [(r.standard_normal(shapes[0]) * 10.0 ** r.uniform(-3, 3)).astype(np.float32)]
    W = [np.zeros(shapes[0], np.float32)]
    lr = 0.25
    go = GO.GraftOracle(shapes, kind=GO.GRAFT_ADAM, adam_eps=0.0, graft_eps=0.0, max_block=max_block)
    out = go.step(1, lr, G, D, W)
    step = -out[0].astype(np.float64)
    for r0 in range(0, 50, max_block):
        for c0 in range(0, 37, max_block):
            s = step[r0:r0 + max_block, c0:c0 + max_block]
            d = D[0][r0:r0 + max_block, c0:c0 + max_block].astype(np.float64)
            assert np.isclose(np.linalg.norm(s), lr * np.sqrt(s.size), rtol=1e-6)
            cos = np.sum(s * d) / (np.linalg.norm(s) * np.linalg.norm(d))
            assert cos > 1 - 1e-12


def test_norms_are_per_tile():
    # Scaling D in one tile changes nothing anywhere (graft_eps = 0): the
    # ratio divides that tile's own norm back out, and no other tile sees it.
    shapes = [(12, 20)]
    r = _rng(5)
    G = [r.standard_normal(shapes[0]).astype(np.float32)]
    D = [r.standard_normal(shapes[0]).astype(np.float32)]
    W = [r.standard_normal(shapes[0]).astype(np.float32)]
    D2 = [D[0].copy()]
    D2[0][0:8, 8:16] *= 1024.0                      # exactly one 8 x 8 tile
    outs = []
    for dirs in (D, D2):
        go = GO.GraftOracle(shapes, kind=GO.GRAFT_SGD, graft_eps=0.0, max_block=8)
        outs.append(go.step(1, 0.1, G, dirs, W)[0])
    assert np.array_equal(outs[0], outs[1])
    # whereas one norm over the whole layer would move every tile
    go = GO.GraftOracle(shapes, kind=GO.GRAFT_SGD, graft_eps=0.0, max_block=1024)
    whole = [go.step(1, 0.1, G, dirs, W)[0] for dirs in (D, D2)]
    assert not np.array_equal(whole[0][0:8, 0:8], whole[1][0:8, 0:8])


def test_hand_worked_example():
    # G = diag(3, 4), D = all ones (2 x 2), W = all ones, lr = 0.1.
    # SGD: ||G|| = 5, ||D|| = 2 -> step = 0.1 * 5/2 * D = 0.25 -> W = 0.75.
    G = [np.array([[3.0, 0.0], [0.0, 4.0]], np.float32)]
    D = [np.ones((2, 2), np.float32)]
    W = [np.ones((2, 2), np.float32)]
    go = GO.GraftOracle([(2, 2)], kind=GO.GRAFT_SGD, graft_eps=0.0)
    assert np.array_equal(go.step(1, 0.1, G, D, W)[0], np.full((2, 2), np.float32(1.0 - np.float32(0.1) * 2.5)))
    # Adam with b1 = 1/2, b2 = 3/4 (exact in binary), t = 1, adam_eps = 1:
    # m = g/2, v = g^2/4, m_hat = g, v_hat = g^2, d = g / (|g| + 1) =
    # diag(3/4, 4/5), norm sqrt(0.5625 + 0.64) = sqrt(1.2025);
    # step = 0.1 * sqrt(1.2025) / 2.
    go = GO.GraftOracle([(2, 2)], kind=GO.GRAFT_ADAM, beta1=0.5, beta2=0.75, adam_eps=1.0, graft_eps=0.0)
    w = go.step(1, 0.1, G, D, W)[0]
    lr = float(np.float32(0.1))
    assert np.allclose(w, 1.0 - lr * np.sqrt(1.2025) / 2.0, rtol=0, atol=1e-7)
    assert np.array_equal(go.m[0], np.array([[1.5, 0.0], [0.0, 2.0]], np.float32))
    assert np.array_equal(go.v[0], np.array([[2.25, 0.0], [0.0, 4.0]], np.float32))


def test_zero_direction_and_nonfinite_tiles():
    shapes = [(8, 16)]
    r = _rng(6)
    G = [r.standard_normal(shapes[0]).astype(np.float32)]
    D = [r.standard_normal(shapes[0]).astype(np.float32)]
    W = [r.standard_normal(shapes[0]).astype(np.float32)]
    D[0][:, 0:8] = 0.0                               # tile 0: zero direction
    G[0][3, 12] = np.nan                             # tile 1: non-finite gradient
    go = GO.GraftOracle(shapes, kind=GO.GRAFT_ADAM, graft_eps=0.0, max_block=8)
    out = go.step(1, 0.1, G, D, W)[0]
    assert np.array_equal(out, W[0])                 # both tiles keep their weights
    assert np.all(go.m[0][:, 8:] == 0) and np.all(go.v[0][:, 8:] == 0)   # skipped tile
    assert np.any(go.m[0][:, :8] != 0)               # the zero-D tile still updates moments


@pytest.mark.parametrize("kind", [GO.GRAFT_SGD, GO.GRAFT_ADAM])
def test_ragged_partition_touches_every_element_once(kind):
    # Every element of a ragged parameter moves, by its own tile's ratio.
    shapes = [(37, 29)]
    r = _rng(7)
    G = [r.standard_normal(shapes[0]).astype(np.float32)]
    D = [r.standard_normal(shapes[0]).astype(np.float32)]
    W = [np.zeros(shapes[0], np.float32)]
    go = GO.GraftOracle(shapes, kind=kind, graft_eps=0.0, max_block=16)
    out = go.step(1, 1.0, G, D, W)[0].astype(np.float64)
    ratio = -out / D[0].astype(np.float64)
    for r0 in (0, 16, 32):
        for c0 in (0, 16):
            t = ratio[r0:r0 + 16, c0:c0 + 16]
            assert np.allclose(t, t.flat[0], rtol=1e-6)
