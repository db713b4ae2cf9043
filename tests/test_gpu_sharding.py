"""Refresh sharding on one GPU ("Shampoo -- Second-Order Optimizer",
"Blocked and distributed variants"): the ranks of a sharded refresh run one
after another on the same device (no rank waits on another), their spans are
copied across as the broadcast would, and every factor's codes, scales and
eigenvalues, and the preconditioned update, must equal bit for bit those of
one handle that refreshes every factor."""
import ctypes as C

import numpy as np
import pytest
import torch

from gpu_helpers import cuda_f32

pytestmark = pytest.mark.gpu

SHAPES = [(300, 260), (64, 147), (1024, 768)]


def _grads(seed):
    rng = np.random.default_rng(seed)
    return [cuda_f32((rng.standard_normal(s) * 0.1).astype(np.float32)) for s in SHAPES]


def _compressed_state(sh, f):
    from bit_quantized_shampoo_b200 import _lib as L
    o = [C.c_size_t() for _ in range(4)]
    d = C.c_int32()
    L.call("shampoo4_factor_layout", sh._h, f, *[C.byref(x) for x in o], C.byref(d))
    d2 = d.value ** 2
    st = sh.state
    return (st[o[1].value:o[1].value + (d2 + 1) // 2].cpu().numpy(),
            st[o[2].value:o[2].value + 4 * ((d2 + 63) // 64)].cpu().numpy(),
            st[o[3].value:o[3].value + 4 * d.value].cpu().numpy())


@pytest.mark.parametrize("world,compressed", [(2, False), (3, False), (2, True)])
def test_sharded_refresh_equals_single_rank(world, compressed):
    from bit_quantized_shampoo_b200 import api
    full = api.Shampoo4(SHAPES, precision="tf32", compressed=compressed)
    ranks = [api.Shampoo4(SHAPES, precision="tf32", compressed=compressed, refresh_rank=r, refresh_world=world)
             for r in range(world)]
    owners = [ranks[0].factor_owner(f) for f in range(full.nfactors)]
    assert set(owners) == set(range(world))
    spans = ranks[0].owner_spans()
    for rnd in range(3):
        G = _grads(40 + rnd)
        for sh in [full] + ranks:
            sh.update_stats(G)
            sh.refresh_roots()
        torch.cuda.synchronize()
        for r, (off, n) in enumerate(spans):               # the broadcast, on one device
            for q in range(world):
                if q != r:
                    ranks[q].state[off:off + n].copy_(ranks[r].state[off:off + n])
        torch.cuda.synchronize()
        for f in range(full.nfactors):
            want = _compressed_state(full, f)
            for q in range(world):
                got = _compressed_state(ranks[q], f)
                for a, b in zip(got, want):
                    assert np.array_equal(a, b), (rnd, f, q, owners[f])
        G2 = _grads(90 + rnd)
        D = full.precondition(G2)
        for q in range(world):
            Dq = ranks[q].precondition(G2)
            for a, b in zip(Dq, D):
                assert torch.equal(a, b), (rnd, q)
    for sh in [full] + ranks:
        assert sh.status_flags() & ~0x10 == 0
