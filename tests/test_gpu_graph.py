"""The step inside a CUDA graph: update_stats, refresh_roots and precondition
enqueue only stream work (pointer tables travel as kernel parameters), so a
graph captured around two steps with different gradient buffers replays
them exactly.  Replays are compared bit for bit with the same calls made
eagerly on a twin handle."""
import numpy as np
import pytest
import torch

from gpu_helpers import cuda_f32

pytestmark = pytest.mark.gpu

SHAPES = [(300, 260), (64, 147), (1024, 768)]


def _grads(seed):
    rng = np.random.default_rng(seed)
    return [cuda_f32((rng.standard_normal(s) * 0.1).astype(np.float32)) for s in SHAPES]


def _state(sh):
    return sh.state.clone()


@pytest.mark.parametrize("compressed", [False, True])
def test_graph_replay_equals_eager_steps(compressed):
    from bit_quantized_shampoo_b200 import api
    eager = api.Shampoo4(SHAPES, precision="tf32", compressed=compressed)
    graphed = api.Shampoo4(SHAPES, precision="tf32", compressed=compressed)
    G = [_grads(1), _grads(2)]
    outs = [[torch.empty(s, dtype=torch.float32, device="cuda") for s in SHAPES] for _ in range(2)]
    eouts = [[torch.empty(s, dtype=torch.float32, device="cuda") for s in SHAPES] for _ in range(2)]
    for sh, o in ((eager, eouts[0]), (graphed, outs[0])):        # warm: first refresh from U = I
        sh.update_stats(G[0])
        sh.refresh_roots()
        sh.precondition(G[0], out=o)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for i in (1, 0):                                     # two steps, alternating gradient buffers
                graphed.update_stats(G[i])
                graphed.refresh_roots()
                graphed.precondition(G[i], out=outs[i])
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for rep in range(2):
        g.replay()
        for i in (1, 0):
            eager.update_stats(G[i])
            eager.refresh_roots()
            eager.precondition(G[i], out=eouts[i])
        torch.cuda.synchronize()
        assert torch.equal(_state(graphed), _state(eager)), rep
        for i in range(2):
            for a, b in zip(outs[i], eouts[i]):
                assert torch.equal(a, b), (rep, i)
    del g
    assert eager.status_flags() & ~0x10 == 0 and graphed.status_flags() & ~0x10 == 0
