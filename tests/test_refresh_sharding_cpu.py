"""Refresh sharding on the host ("Shampoo -- Second-Order Optimizer",
"Blocked and distributed variants": the roots of different blocks are
computed on different workers, then shared): the cost-balanced owner
assignment, the per-rank state spans the exchange moves, and the exchange
itself between two gloo ranks on CPU tensors.  No GPU."""
import ctypes as C
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from bit_quantized_shampoo_b200 import _lib as L
from bit_quantized_shampoo_b200.workloads import WORKLOADS

SIZE_MAX = C.c_size_t(-1).value


def _init(shapes, rank, world, max_block=1024, compressed=0):
    cfg = L.Config(0.95, 1e-6, max_block, 64, 5, 0, compressed, rank, world)
    params = (L.Param * len(shapes))(*[L.Param(r, c) for r, c in shapes])
    h = C.c_void_p()
    L.call("shampoo4_init", C.byref(cfg), params, len(shapes), C.byref(h))
    return h


def _plan(h, world):
    nb, nf = C.c_int32(), C.c_int32()
    L.call("shampoo4_counts", h, C.byref(nb), C.byref(nf))
    owners, dims, lay = [], [], []
    for f in range(nf.value):
        r = C.c_int32()
        L.call("shampoo4_factor_owner", h, f, C.byref(r))
        o = [C.c_size_t() for _ in range(4)]
        d = C.c_int32()
        L.call("shampoo4_factor_layout", h, f, *[C.byref(x) for x in o], C.byref(d))
        owners.append(r.value)
        dims.append(d.value)
        lay.append(tuple(x.value for x in o))
    spans = []
    for r in range(world):
        off, n = C.c_size_t(), C.c_size_t()
        L.call("shampoo4_owner_span", h, r, C.byref(off), C.byref(n))
        spans.append((off.value, n.value))
    sb, wb = C.c_size_t(), C.c_size_t()
    L.call("shampoo4_sizes", h, C.byref(sb), C.byref(wb))
    return owners, dims, lay, spans, sb.value


@pytest.mark.parametrize("wid,world", [(3, 2), (3, 3), (5, 4), (4, 8), (1, 4)])
def test_owners_balance_and_spans(wid, world):
    w = WORKLOADS[wid]
    plans = []
    for rank in range(world):
        h = _init(w.shapes, rank, world, w.max_block)
        try:
            plans.append(_plan(h, world))
        finally:
            L.lib().shampoo4_destroy(h)
    owners, dims, lay, spans, _ = plans[0]
    cost = np.array(dims, np.float64) ** 3
    # every rank's handle plans the same owners, spans and compressed layout
    for o, d, l, sp, _ in plans[1:]:
        assert o == owners and sp == spans
        assert [x[1:] for x in l] == [x[1:] for x in lay]
    # a partition, balanced as longest-processing-time-first guarantees:
    # the heaviest rank exceeds the lightest by at most the largest cost
    loads = np.array([cost[np.array(owners) == r].sum() for r in range(world)])
    assert set(owners) <= set(range(world))
    assert loads.max() - loads.min() <= cost.max() + 1e-9
    # each rank's codes, scales and eigenvalues lie inside its span, spans
    # are disjoint and 256-byte aligned
    for f, (o_s, o_c, o_sc, o_l) in enumerate(lay):
        d2 = dims[f] ** 2
        off, n = spans[owners[f]]
        for a, size in ((o_c, (d2 + 1) // 2), (o_sc, 4 * ((d2 + 63) // 64)), (o_l, 4 * dims[f])):
            assert off <= a and a + size <= off + n
    live = sorted(s for s in spans if s[1])
    assert all(a[0] + a[1] <= b[0] for a, b in zip(live, live[1:]))
    assert all(off % 256 == 0 for off, _ in spans)
    # each handle keeps the statistics of its own factors only
    for rank, (o, d, l, sp, sb) in enumerate(plans):
        for f in range(len(o)):
            assert (l[f][0] != SIZE_MAX) == (o[f] == rank)
            if o[f] == rank:
                assert l[f][0] + 4 * d[f] ** 2 <= sb


def test_single_rank_owns_everything():
    shapes = [(300, 260)]
    h = _init(shapes, 0, 1)
    try:
        owners, dims, lay, spans, sb = _plan(h, 1)
        assert set(owners) == {0} and all(x[0] != SIZE_MAX for x in lay)
        assert lib_rejects_rank(shapes)
    finally:
        L.lib().shampoo4_destroy(h)


def lib_rejects_rank(shapes):
    params = (L.Param * len(shapes))(*[L.Param(r, c) for r, c in shapes])
    h = C.c_void_p()
    for rank, world in ((2, 2), (-1, 2), (0, -1)):
        cfg = L.Config(0.95, 1e-6, 1024, 64, 5, 0, 0, rank, world)
        if L.lib().shampoo4_init(C.byref(cfg), params, len(shapes), C.byref(h)) != 1:
            return False
    return True


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, shapes, out):
    import datetime
    import torch.distributed as dist
    from bit_quantized_shampoo_b200.api import exchange_spans
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        h = _init(shapes, rank, world, max_block=128)
        try:
            owners, dims, lay, spans, sb = _plan(h, world)
        finally:
            L.lib().shampoo4_destroy(h)
        # each rank writes its own span (its freshly refreshed factors) with a
        # rank-specific pattern and leaves the rest stale
        buf = torch.full((sb,), 255, dtype=torch.uint8)
        off, n = spans[rank]
        buf[off:off + n] = torch.arange(n, dtype=torch.int64).remainder(251).to(torch.uint8) + rank
        exchange_spans(buf, spans)
        out[rank] = [bytes(buf[o:o + k].numpy()) for o, k in spans]
    finally:
        dist.destroy_process_group()


def test_exchange_moves_every_span_from_its_owner_two_gloo_ranks():
    shapes = [(300, 260), (64, 147)]
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), shapes, out), nprocs=world, join=True)
    for r in range(world):
        for src, blob in enumerate(out[r]):
            n = len(blob)
            want = (np.arange(n) % 251 + src).astype(np.uint8).tobytes()
            assert blob == want, (r, src)
