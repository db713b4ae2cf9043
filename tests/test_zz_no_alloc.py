"""The allocation-free statistics update (shampoo4_update_stats_noalloc)
against the handle entry point shampoo4_update_stats on the same tile, two
calls in a row; its argument checks on the CPU.  Collected last on purpose:
it must pass both alone and after every other GPU test."""
import ctypes as C

import numpy as np
import pytest

from gpu_helpers import rel_fro

TOL_TF32 = 2e-3          # relative Frobenius, the TF32 bound of the statistics stage
STATUS_INVALID_ARG = 1
STATUS_WORKSPACE = 5


def _grads(shape, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal(shape).astype(np.float32) for _ in range(2)]


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(200, 130), (256, 512), (512, 512), (1024, 64)])
def test_noalloc_matches_handle_two_calls(shape):
    import torch
    from bit_quantized_shampoo_b200 import api

    m, n = shape
    beta = 0.95
    g1, g2 = _grads(shape, 7000 + m + n)
    G1, G2 = (torch.from_numpy(g).cuda() for g in (g1, g2))

    sh = api.Shampoo4([shape], beta=beta, precision="tf32")   # reset: statistics start at zero
    sh.update_stats([G1])
    sh.update_stats([G2])
    L_ref = sh.factor_views(0)[0].clone()
    R_ref = sh.factor_views(1)[0].clone()

    L = torch.zeros(m, m, dtype=torch.float32, device="cuda")
    R = torch.zeros(n, n, dtype=torch.float32, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.update_stats_noalloc(L, R, G1, beta, flags=flags)
    api.update_stats_noalloc(L, R, G2, beta, flags=flags)
    torch.cuda.synchronize()

    assert int(flags.item()) == 0
    assert rel_fro(L.cpu().numpy(), L_ref.cpu().numpy()) <= TOL_TF32
    assert rel_fro(R.cpu().numpy(), R_ref.cpu().numpy()) <= TOL_TF32
    # exact symmetry, as the handle path gives
    assert torch.equal(L, L.T) and torch.equal(R, R.T)
    # the fp64 definition of two EMA steps from zero
    for S, a, b in ((L, g1 @ g1.T, g2 @ g2.T), (R, g1.T @ g1, g2.T @ g2)):
        a = a.astype(np.float64)
        b = b.astype(np.float64)
        exact = beta * (1 - beta) * a + (1 - beta) * b
        assert rel_fro(S.cpu().numpy(), exact) <= TOL_TF32


@pytest.mark.gpu
def test_noalloc_nonfinite_gradient_leaves_state():
    import torch
    from bit_quantized_shampoo_b200 import api, _lib

    m, n = 96, 160
    g1, g2 = _grads((m, n), 71)
    g2[5, 7] = np.nan
    L = torch.zeros(m, m, dtype=torch.float32, device="cuda")
    R = torch.zeros(n, n, dtype=torch.float32, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.update_stats_noalloc(L, R, torch.from_numpy(g1).cuda(), 0.9, flags=flags)
    L1, R1 = L.clone(), R.clone()
    api.update_stats_noalloc(L, R, torch.from_numpy(g2).cuda(), 0.9, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == _lib.FLAG_NONFINITE_GRAD
    assert torch.equal(L, L1) and torch.equal(R, R1)
    # the next finite gradient updates again (the gate is reset per call)
    api.update_stats_noalloc(L, R, torch.from_numpy(g1).cuda(), 0.9)
    torch.cuda.synchronize()
    assert not torch.equal(L, L1)


@pytest.mark.gpu
def test_noalloc_calls_allocate_no_device_memory():
    """The point of the entry point: after a first call has loaded the
    module, further calls -- other shapes included -- leave the device's free
    memory and torch's allocator exactly where they were."""
    import torch
    from bit_quantized_shampoo_b200 import api

    bufs = {}
    for m, n in ((64, 96), (512, 512), (1024, 256), (300, 17)):
        g = torch.from_numpy(_grads((m, n), 90 + m)[0]).cuda()
        bufs[(m, n)] = (torch.zeros(m, m, device="cuda"), torch.zeros(n, n, device="cuda"), g)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    L, R, G = bufs[(64, 96)]
    api.update_stats_noalloc(L, R, G, 0.9, flags=flags)          # warm-up: module load
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    alloc0 = torch.cuda.memory_stats().get("allocated_bytes.all.current", 0)
    for _ in range(3):
        for L, R, G in bufs.values():
            api.update_stats_noalloc(L, R, G, 0.9, flags=flags)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_stats().get("allocated_bytes.all.current", 0) == alloc0
    assert int(flags.item()) == 0


def test_noalloc_rejects_before_touching_the_device():
    """Size and argument checks return before any CUDA call, so they run
    without a GPU; the pointers are never dereferenced."""
    from bit_quantized_shampoo_b200 import _lib as L

    f = L.lib().shampoo4_update_stats_noalloc
    fake = [C.c_void_p(256), C.c_void_p(512), C.c_void_p(1024)]
    # beyond the static scratch: m * n > 2^18, or an edge > 1024
    assert f(*fake, 1024, 512, 512, C.c_float(0.9), None, None) == STATUS_WORKSPACE
    assert f(*fake, 2048, 16, 16, C.c_float(0.9), None, None) == STATUS_WORKSPACE
    # bad arguments
    assert f(*fake, 64, 64, 32, C.c_float(0.9), None, None) == STATUS_INVALID_ARG      # ldg < n
    assert f(*fake, 64, 64, 64, C.c_float(1.0), None, None) == STATUS_INVALID_ARG      # beta = 1
    assert f(None, fake[1], fake[2], 64, 64, 64, C.c_float(0.9), None, None) == STATUS_INVALID_ARG
    assert f(*fake, 0, 64, 64, C.c_float(0.9), None, None) == STATUS_INVALID_ARG
