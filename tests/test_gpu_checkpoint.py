"""Checkpoint and resume: all optimizer state lives in the caller's state
buffer, so a copy of it, bound to a fresh handle with reset = 0 and
has_basis declared, continues bit for bit as the original handle does."""
import numpy as np
import pytest
import torch

from gpu_helpers import cuda_f32

pytestmark = pytest.mark.gpu

SHAPES = [(300, 260), (64, 147)]


def _grads(seed):
    rng = np.random.default_rng(seed)
    return [cuda_f32((rng.standard_normal(s) * 0.1).astype(np.float32)) for s in SHAPES]


@pytest.mark.parametrize("compressed", [False, True])
def test_resume_from_a_copied_state_is_bit_identical(compressed):
    from bit_quantized_shampoo_b200 import api
    a = api.Shampoo4(SHAPES, precision="tf32", compressed=compressed)
    for t in (1, 2):
        G = _grads(t)
        a.update_stats(G)
        a.refresh_roots()
        a.precondition(G)
    torch.cuda.synchronize()
    ckpt = a.state.clone()                                   # what a checkpoint saves
    b = api.Shampoo4(SHAPES, precision="tf32", compressed=compressed, reset=False)
    b.state.copy_(ckpt)
    b.set_has_basis(True)
    for t in (3, 4):
        G = _grads(t)
        outs = []
        for sh in (a, b):
            sh.update_stats(G)
            sh.refresh_roots()
            outs.append(sh.precondition(G))
        torch.cuda.synchronize()
        assert torch.equal(a.state, b.state), t
        for x, y in zip(*outs):
            assert torch.equal(x, y), t
    assert a.status_flags() & ~0x10 == 0 and b.status_flags() & ~0x10 == 0
