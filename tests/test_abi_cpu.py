"""Host-side checks of the C ABI, no GPU: the library loads, exports every
entry point the header declares, plans tiles like the oracle, and rejects bad
arguments before touching a device."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from bit_quantized_shampoo_b200 import _lib as L
from bit_quantized_shampoo_b200.workloads import WORKLOADS
from oracle import shampoo4_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "shampoo4.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b((?:shampoo4|quant4)_[a-z_]+)\s*\(", txt)))


def test_library_exports_every_declared_entry_point():
    lib = L.lib()
    names = _declared()
    assert len(names) >= 17
    for n in names:
        assert hasattr(lib, n), n


def test_codec_tables_match_the_oracle_definition():
    cb = (C.c_float * 16)()
    th = (C.c_float * 15)()
    L.call("quant4_tables", cb, th)
    assert np.array_equal(np.array(cb, np.float32), O.codebook_f32())
    assert np.array_equal(np.array(th, np.float32), O.thresholds_f32())


def test_dynamic_tree_tables_match_the_oracle_definition():
    cb = (C.c_float * 16)()
    th = (C.c_float * 15)()
    L.call("quant4_tables_ex", L.CODEBOOK_DYNAMIC_TREE, cb, th)
    assert np.array_equal(np.array(cb, np.float32), O.codebook_f32(O.DYNAMIC_TREE))
    assert np.array_equal(np.array(th, np.float32), O.thresholds_f32(O.DYNAMIC_TREE))
    assert L.lib().quant4_tables_ex(7, cb, th) == 1


def test_codebook_and_root_method_configs():
    params = (L.Param * 1)(L.Param(64, 96))

    def init(**kw):
        cfg = L.Config(0.95, 1e-6, 1024, 64, 5, 0, kw.get("compressed", 0), 0, 1, kw.get("codebook", 0),
                       kw.get("root", 0), kw.get("iters", 0))
        h = C.c_void_p()
        st = L.lib().shampoo4_init(C.byref(cfg), params, 1, C.byref(h))
        return st, h
    for kw in ({"codebook": 2}, {"root": 3}, {"root": 1, "compressed": 1}, {"root": 2, "iters": 101},
               {"iters": -1}):
        st, h = init(**kw)
        assert st == 1 and not h.value, kw
    st, h = init(codebook=1, root=2, iters=20)
    assert st == 0
    off = C.c_size_t()
    assert L.lib().shampoo4_root_offset(h, 0, C.byref(off)) == 1          # no fp32 root kept
    L.lib().shampoo4_destroy(h)
    st, h = init(root=1)
    assert st == 0
    sizes = []
    for f in range(2):
        L.call("shampoo4_root_offset", h, f, C.byref(off))
        sizes.append(off.value)
    stb = C.c_size_t()
    L.call("shampoo4_sizes", h, C.byref(stb), None)
    assert sizes[0] % 256 == 0 and sizes[0] + 4 * 64 * 64 <= sizes[1] and sizes[1] + 4 * 96 * 96 <= stb.value
    L.lib().shampoo4_destroy(h)


def test_tile_groups_bound_the_workspace():
    """The calls' scratch is held for two groups of consecutive tiles, not
    for every tile: on the Llama layer set one group (what the automatic
    rule picks below 96 GiB) needs 81.9 GB, 48 tiles per group about a fifth
    of it, and 16 tiles per group less than one and a half times the 4.5 GB
    state; the Llama set twice over exceeds 96 GiB in one group, and the
    automatic rule groups it.  A negative group size is refused."""
    w = WORKLOADS[5]
    params = (L.Param * len(w.shapes))(*[L.Param(r, c) for r, c in w.shapes])
    sizes = {}
    for gt in (100000, 0, 48, 16, 1):
        cfg = L.Config(0.95, 1e-6, 1024, 64, 5, 0, 0, 0, 1, 0, 0, 0, gt)
        h = C.c_void_p()
        L.call("shampoo4_init", C.byref(cfg), params, len(w.shapes), C.byref(h))
        st, ws = C.c_size_t(), C.c_size_t()
        L.call("shampoo4_sizes", h, C.byref(st), C.byref(ws))
        sizes[gt] = (st.value, ws.value)
        L.lib().shampoo4_destroy(h)
    state = sizes[0][0]
    assert sizes[100000][1] > 80e9 and sizes[0][1] == sizes[100000][1]
    assert sizes[48][1] < 0.25 * sizes[100000][1]
    assert sizes[16][1] < 1.5 * state
    assert sizes[1][1] < sizes[16][1] < sizes[48][1]
    twice = list(w.shapes) * 2
    p2 = (L.Param * len(twice))(*[L.Param(r, c) for r, c in twice])
    cfg = L.Config(0.95, 1e-6, 1024, 64, 5, 0, 0, 0, 1, 0, 0, 0, 0)
    h = C.c_void_p()
    L.call("shampoo4_init", C.byref(cfg), p2, len(twice), C.byref(h))
    ws = C.c_size_t()
    L.call("shampoo4_sizes", h, None, C.byref(ws))
    assert ws.value < 20e9                      # grouped: two slots of at most 8 GiB
    L.lib().shampoo4_destroy(h)
    cfg = L.Config(0.95, 1e-6, 1024, 64, 5, 0, 0, 0, 1, 0, 0, 0, -1)
    h = C.c_void_p()
    assert L.lib().shampoo4_init(C.byref(cfg), params, len(w.shapes), C.byref(h)) == 1


def _init(shapes, **kw):
    cfg = L.Config(kw.get("beta", 0.95), kw.get("eps", 1e-6), kw.get("max_block", 1024), kw.get("qb", 64),
                   kw.get("bj", 5), kw.get("prec", 0), kw.get("compressed", 0))
    params = (L.Param * len(shapes))(*[L.Param(r, c) for r, c in shapes])
    h = C.c_void_p()
    st = L.lib().shampoo4_init(C.byref(cfg), params, len(shapes), C.byref(h))
    return st, h


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_plan_matches_oracle_partition(wid):
    w = WORKLOADS[wid]
    st, h = _init(w.shapes, max_block=w.max_block)
    assert st == 0
    try:
        nb, nf = C.c_int32(), C.c_int32()
        L.call("shampoo4_counts", h, C.byref(nb), C.byref(nf))
        blocks = O.partition(w.shapes, w.max_block)
        assert nb.value == len(blocks) and nf.value == 2 * len(blocks)
        p, m, n = C.c_int32(), C.c_int32(), C.c_int32()
        r0, c0 = C.c_int64(), C.c_int64()
        for k, b in enumerate(blocks):
            L.call("shampoo4_block_info", h, k, C.byref(p), C.byref(r0), C.byref(c0), C.byref(m), C.byref(n))
            assert (p.value, r0.value, c0.value, m.value, n.value) == (b.param, b.r0, b.c0, b.m, b.n)
        # state layout: every factor's pieces are disjoint, 256-aligned and inside the state
        sb, wb = C.c_size_t(), C.c_size_t()
        L.call("shampoo4_sizes", h, C.byref(sb), C.byref(wb))
        spans = []
        for f in range(nf.value):
            o = [C.c_size_t() for _ in range(4)]
            d = C.c_int32()
            L.call("shampoo4_factor_layout", h, f, *[C.byref(x) for x in o], C.byref(d))
            b = blocks[f // 2]
            assert d.value == (b.m if f % 2 == 0 else b.n)
            dd = d.value * d.value
            sizes = [4 * dd, (dd + 1) // 2, 4 * ((dd + 63) // 64), 4 * d.value]
            for off, sz in zip(o, sizes):
                assert off.value % 256 == 0
                spans.append((off.value, off.value + sz))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
        assert spans[-1][1] <= sb.value
        assert wb.value > 0
    finally:
        L.lib().shampoo4_destroy(h)


def test_init_rejects_bad_configs():
    bad = [dict(beta=1.0), dict(beta=-0.1), dict(eps=0.0), dict(max_block=0), dict(max_block=2048),
           dict(qb=32), dict(bj=-1), dict(bj=17), dict(prec=2), dict(compressed=2)]
    for kw in bad:
        st, h = _init([(8, 8)], **kw)
        assert st == 1, kw
    st, h = _init([(0, 8)])
    assert st == 1


def test_calls_before_bind_are_not_ready_and_null_handles_invalid():
    st, h = _init([(8, 8)])
    assert st == 0
    try:
        lib = L.lib()
        assert lib.shampoo4_refresh_roots(h, None) == 3
        g = L.ptr_array([0])
        assert lib.shampoo4_update_stats(h, g, L.i64_array([8]), None) == 3
        assert lib.shampoo4_refresh_roots(None, None) == 1
        assert lib.shampoo4_block_info(h, 5, None, None, None, None, None) == 1
        assert lib.quant4_pack(None, None, -1, None, None, None) == 1
        assert lib.quant4_pack(None, None, 0, None, None, None) == 0
        assert lib.shampoo4_status_string(3)
    finally:
        L.lib().shampoo4_destroy(h)


def test_graft_state_layout_and_argument_checks():
    shapes = [(37, 29), (1030, 8), (4, 4)]
    st, h = _init(shapes, max_block=16)
    assert st == 0
    try:
        lib = L.lib()
        n = C.c_size_t()
        L.call("shampoo4_graft_state_bytes", h, L.GRAFT_SGD, C.byref(n))
        assert n.value == 0
        L.call("shampoo4_graft_state_bytes", h, L.GRAFT_ADAM, C.byref(n))
        assert n.value >= sum(8 * r * c for r, c in shapes) and n.value % 256 == 0
        assert lib.shampoo4_graft_state_bytes(h, 2, C.byref(n)) == 1
        spans = []
        for p, (r, c) in enumerate(shapes):
            om, ov = C.c_size_t(), C.c_size_t()
            L.call("shampoo4_graft_layout", h, L.GRAFT_ADAM, p, C.byref(om), C.byref(ov))
            for o in (om.value, ov.value):
                assert o % 256 == 0
                spans.append((o, o + 4 * r * c))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:])) and spans[-1][1] <= n.value
        assert lib.shampoo4_graft_layout(h, L.GRAFT_ADAM, 3, None, None) == 1
        assert lib.shampoo4_graft_layout(h, L.GRAFT_SGD, 0, None, None) == 1
        cfg = L.GraftConfig(L.GRAFT_ADAM, 0.9, 0.999, 1e-8, 1e-16)
        ptrs = L.ptr_array([256, 512, 768])
        lds = L.i64_array([c for _, c in shapes])
        # unbound handle: not ready; null handle: invalid
        assert lib.shampoo4_graft_update(h, C.byref(cfg), C.c_void_p(256), 1, C.c_float(0.1), ptrs, lds, ptrs, lds,
                                         ptrs, lds, None) == 3
        assert lib.shampoo4_graft_update(None, C.byref(cfg), None, 1, C.c_float(0.1), ptrs, lds, ptrs, lds,
                                         ptrs, lds, None) == 1
    finally:
        L.lib().shampoo4_destroy(h)


def test_compressed_statistics_leave_the_state_and_move_to_the_workspace():
    shapes = [(300, 260), (64, 147)]
    sizes = {}
    for comp in (0, 1):
        st, h = _init(shapes, max_block=256, compressed=comp)
        assert st == 0
        try:
            sb, wb = C.c_size_t(), C.c_size_t()
            L.call("shampoo4_sizes", h, C.byref(sb), C.byref(wb))
            sizes[comp] = (sb.value, wb.value)
            nb, nf = C.c_int32(), C.c_int32()
            L.call("shampoo4_counts", h, C.byref(nb), C.byref(nf))
            dd = 0
            for f in range(nf.value):
                oS, d = C.c_size_t(), C.c_int32()
                L.call("shampoo4_factor_layout", h, f, C.byref(oS), None, None, None, C.byref(d))
                dd += d.value * d.value
                off = C.c_size_t()
                if comp:
                    assert oS.value == C.c_size_t(-1).value          # SIZE_MAX: not in the state
                    L.call("shampoo4_debug_s_offset", h, f, C.byref(off))
                    assert off.value % 256 == 0 and off.value + 4 * d.value ** 2 <= wb.value
                else:
                    assert L.lib().shampoo4_debug_s_offset(h, f, C.byref(off)) == 1
        finally:
            L.lib().shampoo4_destroy(h)
    # the state loses every statistic (4 d^2 bytes per factor); the workspace gains them
    assert sizes[0][0] - sizes[1][0] >= 4 * dd
    assert sizes[1][1] - sizes[0][1] >= 4 * dd


@pytest.mark.skipif(not (os.path.exists("/usr/bin/gcc") or os.path.exists("/usr/bin/cc")), reason="no C compiler")
def test_c_program_links_and_plans_through_the_header(tmp_path):
    """The header compiles as C11 with warnings as errors, the library links
    by its C names, and the host-only calls behave as documented, from C."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    libdir = os.path.dirname(L.library_path())
    exe = tmp_path / "abi_host_check"
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "native", "abi_host_check.c"), "-o", str(exe),
                    "-L", libdir, "-lshampoo4", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi ok" in r.stdout
