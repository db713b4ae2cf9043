"""The bounded waits of the tensor-core products return: with a pipeline
wait limit of 1 ns (shampoo4_debug_wait_limit) the CTAs of a statistics
update of a 1024 x 1024 tile give up waiting for their operands and
accumulator (a 1024-deep main loop takes microseconds), raise
SHAMPOO4_FLAG_TIMEOUT and exit after draining what they issued.  The call
returns, and the same handle and CUDA context then compute a correct update
with the default limit.  No kernel faults or hangs: the wait that runs out
is an ordinary bounded wait on work that does complete."""
import numpy as np
import pytest
import torch

from oracle import shampoo4_oracle as O
from gpu_helpers import cuda_f32, rel_fro

pytestmark = pytest.mark.gpu


def test_expired_pipeline_wait_returns_flags_and_leaves_the_handle_usable():
    from bit_quantized_shampoo_b200 import api, _lib as L
    shapes = [(1024, 1024)]
    sh = api.Shampoo4(shapes, precision="tf32")
    rng = np.random.default_rng(11)
    g = rng.standard_normal(shapes[0]).astype(np.float32)
    G = [cuda_f32(g)]
    L.call("shampoo4_debug_wait_limit", sh._h, 1)
    sh.update_stats(G)
    flags = sh.status_flags()                   # synchronizes the stream
    assert flags & L.FLAG_TIMEOUT, flags
    # the context is healthy: ordinary torch work and the library both run
    x = torch.ones(1 << 20, device="cuda")
    assert float(x.sum().item()) == float(1 << 20)
    L.call("shampoo4_debug_wait_limit", sh._h, 0)
    sh.bind(reset=True)                         # the timed-out call left S undefined
    sh.update_stats(G)
    torch.cuda.synchronize()
    assert sh.status_flags() == 0
    beta = float(np.float32(0.95))
    for f, side in ((0, "L"), (1, "R")):
        want = O.ema_stats(np.zeros((1024, 1024), np.float32), g, beta, side)
        got = sh.factor_views(f)[0].cpu().numpy()
        assert rel_fro(got, want) <= 2e-3
