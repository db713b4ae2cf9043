"""Thin PyTorch-facing wrapper of the shampoo4 C ABI.

PyTorch provides the device memory (state, workspace, outputs) and the CUDA
stream; every arithmetic step runs in libshampoo4.so.  Tensors must be CUDA
float32 (gradients, outputs) or uint8 (codes).
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _lib as L


def _stream(stream=None) -> C.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need_cuda(t: torch.Tensor, dtype, name: str):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype):
        raise TypeError(f"{name} must be a CUDA {dtype} tensor")


def _row_major_2d(t: torch.Tensor, name: str) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit column stride")
    return t.stride(0)


class Shampoo4:
    """One handle: a fixed list of 2-D parameter shapes and their state."""

    def __init__(self, shapes, beta=0.95, eps=1e-6, max_block=1024, bjorck_iters=5,
                 precision="tf32", device=None, reset=True, compressed=False, refresh_rank=0, refresh_world=1,
                 debug=False, codebook="linear_square", root="eigen", newton_iters=0, group_tiles=0):
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.compressed = bool(compressed)
        self.refresh_rank, self.refresh_world = int(refresh_rank), int(refresh_world)
        self.codebook = _codebook(codebook)
        roots = {"eigen": L.ROOT_EIGEN, "newton": L.ROOT_NEWTON, "newton_q4": L.ROOT_NEWTON_Q4}
        if root not in roots:
            raise ValueError(f"root must be one of {sorted(roots)}")
        self.root_method = roots[root]
        cfg = L.Config(beta, eps, max_block, 64, bjorck_iters,
                       L.PREC_FP32 if precision == "fp32" else L.PREC_TF32, 1 if compressed else 0,
                       self.refresh_rank, self.refresh_world, self.codebook, self.root_method, int(newton_iters),
                       int(group_tiles))
        params = (L.Param * len(self.shapes))(*[L.Param(r, c) for r, c in self.shapes])
        h = C.c_void_p()
        L.call("shampoo4_init", C.byref(cfg), params, len(self.shapes), C.byref(h))
        self._h = h
        self.config = cfg
        st, ws = C.c_size_t(), C.c_size_t()
        L.call("shampoo4_sizes", h, C.byref(st), C.byref(ws))
        self.state_bytes, self.workspace_bytes = st.value, ws.value
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.state = torch.empty(max(self.state_bytes, 256), dtype=torch.uint8, device=self.device)
        self.workspace = torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8, device=self.device)
        nb, nf = C.c_int32(), C.c_int32()
        L.call("shampoo4_counts", h, C.byref(nb), C.byref(nf))
        self.nblocks, self.nfactors = nb.value, nf.value
        self.debug_buffer = None
        if debug:
            n = C.c_size_t()
            L.call("shampoo4_debug_capture_bytes", h, C.byref(n))
            self.debug_buffer = torch.zeros(max(n.value, 256), dtype=torch.uint8, device=self.device)
            L.call("shampoo4_debug_capture", h, C.c_void_p(self.debug_buffer.data_ptr()))
        self.bind(reset=reset)

    def bind(self, reset=True, stream=None):
        L.call("shampoo4_bind", self._h, C.c_void_p(self.state.data_ptr()),
               C.c_void_p(self.workspace.data_ptr()), 1 if reset else 0, _stream(stream))

    def set_has_basis(self, flag: bool):
        L.call("shampoo4_set_has_basis", self._h, 1 if flag else 0)

    def _ptrs(self, mats, name):
        if len(mats) != len(self.shapes):
            raise ValueError(f"expected {len(self.shapes)} {name}")
        lds = []
        for m, (r, c) in zip(mats, self.shapes):
            _need_cuda(m, torch.float32, name)
            if tuple(m.shape) != (r, c):
                raise ValueError(f"{name}: shape {tuple(m.shape)} != {(r, c)}")
            lds.append(_row_major_2d(m, name))
        return L.ptr_array([m.data_ptr() for m in mats]), L.i64_array(lds)

    def update_stats(self, grads, stream=None):
        p, ld = self._ptrs(grads, "grads")
        L.call("shampoo4_update_stats", self._h, p, ld, _stream(stream))

    def refresh_roots(self, stream=None):
        L.call("shampoo4_refresh_roots", self._h, _stream(stream))

    def precondition(self, grads, out=None, stream=None):
        if out is None:
            out = [torch.empty(s, dtype=torch.float32, device=self.device) for s in self.shapes]
        p, ld = self._ptrs(grads, "grads")
        q, ldo = self._ptrs(out, "out")
        L.call("shampoo4_precondition", self._h, p, ld, q, ldo, _stream(stream))
        return out

    # ---- grafting ("Shampoo -- Second-Order Optimizer", section "Grafting")

    def graft_state(self, kind="adam"):
        """A zero-filled device buffer for the grafting state (Adam's moments)."""
        n = C.c_size_t()
        L.call("shampoo4_graft_state_bytes", self._h, _graft_kind(kind), C.byref(n))
        return torch.zeros(max(n.value, 256), dtype=torch.uint8, device=self.device)

    def graft_moments(self, state, param):
        """(m, v) of parameter ``param`` as fp32 views into an Adam state buffer."""
        om, ov = C.c_size_t(), C.c_size_t()
        L.call("shampoo4_graft_layout", self._h, L.GRAFT_ADAM, param, C.byref(om), C.byref(ov))
        r, c = self.shapes[param]
        n = 4 * r * c
        return (state[om.value:om.value + n].view(torch.float32).view(r, c),
                state[ov.value:ov.value + n].view(torch.float32).view(r, c))

    def graft_update(self, state, step, lr, grads, dirs, weights, kind="adam", beta1=0.9, beta2=0.999,
                     adam_eps=1e-8, graft_eps=1e-16, dir_norms=False, stream=None):
        """W <- W - lr * ||d_graft|| / (||D|| + graft_eps) * D per tile, in place
        on ``weights``; ``dirs`` is this step's precondition output.
        dir_norms: take ||D|| as the last precondition recorded it (``dirs``
        must be that call's output, unmodified), so D is read once."""
        cfg = L.GraftConfig(_graft_kind(kind), beta1, beta2, adam_eps, graft_eps, 1 if dir_norms else 0)
        p, ld = self._ptrs(grads, "grads")
        q, ldq = self._ptrs(dirs, "dirs")
        w, ldw = self._ptrs(weights, "weights")
        sp = C.c_void_p(state.data_ptr()) if state is not None else C.c_void_p()
        L.call("shampoo4_graft_update", self._h, C.byref(cfg), sp, int(step), float(lr), p, ld, q, ldq, w, ldw,
               _stream(stream))

    # ---- refresh sharding ("Shampoo -- Second-Order Optimizer", "Blocked and
    # distributed variants")

    def owner_spans(self):
        """[(offset, bytes)] per rank: the state range holding the codes,
        scales and eigenvalues of the factors that rank refreshes."""
        out = []
        for r in range(max(1, self.refresh_world)):
            off, n = C.c_size_t(), C.c_size_t()
            L.call("shampoo4_owner_span", self._h, r, C.byref(off), C.byref(n))
            out.append((off.value, n.value))
        return out

    def factor_owner(self, f):
        r = C.c_int32()
        L.call("shampoo4_factor_owner", self._h, f, C.byref(r))
        return r.value

    def exchange_roots(self, group=None):
        """After refresh_roots on every rank: each rank's freshly refreshed
        span goes to all ranks (one torch.distributed broadcast per rank, on
        the state buffer in place).  Plumbing only."""
        exchange_spans(self.state, self.owner_spans(), group)

    def status_flags(self, stream=None) -> int:
        f = C.c_uint32()
        L.call("shampoo4_get_status_flags", self._h, C.byref(f), _stream(stream))
        return f.value

    def block_info(self, k):
        p, m, n = C.c_int32(), C.c_int32(), C.c_int32()
        r0, c0 = C.c_int64(), C.c_int64()
        L.call("shampoo4_block_info", self._h, k, C.byref(p), C.byref(r0), C.byref(c0), C.byref(m), C.byref(n))
        return p.value, r0.value, c0.value, m.value, n.value

    def factor_views(self, f):
        """(S, codes, scales, lambda) as tensor views into the state buffer
        (with compressed statistics, S is the workspace copy the last
        update_stats rebuilt; S is None for a factor another rank refreshes)."""
        oS, oc, os_, ol = C.c_size_t(), C.c_size_t(), C.c_size_t(), C.c_size_t()
        d = C.c_int32()
        L.call("shampoo4_factor_layout", self._h, f, C.byref(oS), C.byref(oc), C.byref(os_), C.byref(ol), C.byref(d))
        d = d.value
        n = d * d
        st = self.state
        if self.compressed:
            L.call("shampoo4_debug_s_offset", self._h, f, C.byref(oS))
            src = self.workspace
        else:
            src = st
        held = oS.value != C.c_size_t(-1).value
        S = src[oS.value:oS.value + 4 * n].view(torch.float32).view(d, d) if held else None
        codes = st[oc.value:oc.value + (n + 1) // 2]
        scales = st[os_.value:os_.value + 4 * ((n + 63) // 64)].view(torch.float32)
        lam = st[ol.value:ol.value + 4 * d].view(torch.float32)
        return S, codes, scales, lam

    def root_view(self, f):
        """Root method "newton": the factor's fp32 root P from the last
        refresh, as a view into the state buffer."""
        off = C.c_size_t()
        L.call("shampoo4_root_offset", self._h, f, C.byref(off))
        d = self._dim(f)
        return self.state[off.value:off.value + 4 * d * d].view(torch.float32).view(d, d)

    def _dim(self, f):
        d = C.c_int32()
        L.call("shampoo4_factor_layout", self._h, f, None, None, None, None, C.byref(d))
        return d.value

    def debug_q(self, f):
        """The pre-quantization Q of factor f from the last refresh: from the
        debug capture buffer when the handle has one, else from the workspace
        (valid until the next call)."""
        d = self._dim(f)
        if self.debug_buffer is not None:
            off = C.c_size_t()
            L.call("shampoo4_debug_capture_layout", self._h, f, None, C.byref(off))
            return self.debug_buffer[off.value:off.value + 4 * d * d].view(torch.float32).view(d, d)
        off = C.c_size_t()
        st = L.lib().shampoo4_debug_q_offset(self._h, f, C.byref(off))
        if st == 6:
            raise RuntimeError("debug_q: with several tile groups the workspace copy of Q does not survive the "
                               "refresh; make the handle with debug=True")
        L.check("shampoo4_debug_q_offset", st)
        return self.workspace[off.value:off.value + 4 * d * d].view(torch.float32).view(d, d)

    def debug_rectified(self, f):
        """The rectified basis (dequantized and Bjorck-rectified; the
        identity on a first refresh) that entered the last refresh's subspace
        step for factor f.  Needs a handle made with debug=True."""
        if self.debug_buffer is None:
            raise RuntimeError("debug_rectified needs a handle made with debug=True")
        d = self._dim(f)
        off = C.c_size_t()
        L.call("shampoo4_debug_capture_layout", self._h, f, C.byref(off), None)
        return self.debug_buffer[off.value:off.value + 4 * d * d].view(torch.float32).view(d, d)

    def close(self):
        if getattr(self, "_h", None):
            L.lib().shampoo4_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def exchange_spans(buf, spans, group=None):
    """Broadcast buf[off:off + n] from rank r to every rank, for each rank's
    (off, n) in ``spans`` (rank order).  ``buf`` is a 1-D uint8 tensor on the
    process group's device."""
    import torch.distributed as dist
    for r, (off, n) in enumerate(spans):
        if n:
            dist.broadcast(buf[off:off + n], src=r, group=group)


def _graft_kind(kind):
    kinds = {"sgd": L.GRAFT_SGD, "adam": L.GRAFT_ADAM}
    if kind not in kinds:
        raise ValueError(f"graft kind must be one of {sorted(kinds)}")
    return kinds[kind]


def _codebook(codebook):
    books = {"linear_square": L.CODEBOOK_LINEAR_SQUARE, "dynamic_tree": L.CODEBOOK_DYNAMIC_TREE}
    if codebook not in books:
        raise ValueError(f"codebook must be one of {sorted(books)}")
    return books[codebook]


def quant4_pack(xs, codes=None, scales=None, stream=None, codebook="linear_square"):
    """Quantize a list of fp32 CUDA tensors (flattened)."""
    xs = [x.contiguous() for x in xs]
    ns = [x.numel() for x in xs]
    for x in xs:
        _need_cuda(x, torch.float32, "x")
    if codes is None:
        codes = [torch.empty((n + 1) // 2, dtype=torch.uint8, device=x.device) for x, n in zip(xs, ns)]
    if scales is None:
        scales = [torch.empty((n + 63) // 64, dtype=torch.float32, device=x.device) for x, n in zip(xs, ns)]
    L.call("quant4_pack_ex", L.ptr_array([x.data_ptr() for x in xs]), L.i64_array(ns), len(xs),
           L.ptr_array([c.data_ptr() for c in codes]), L.ptr_array([s.data_ptr() for s in scales]),
           _codebook(codebook), _stream(stream))
    return codes, scales


def quant4_unpack(codes, scales, ns, out=None, stream=None, codebook="linear_square"):
    if out is None:
        out = [torch.empty(n, dtype=torch.float32, device=c.device) for c, n in zip(codes, ns)]
    L.call("quant4_unpack_ex", L.ptr_array([c.data_ptr() for c in codes]),
           L.ptr_array([s.data_ptr() for s in scales]), L.i64_array(ns), len(codes),
           L.ptr_array([o.data_ptr() for o in out]), _codebook(codebook), _stream(stream))
    return out


def update_stats_noalloc(L_, R_, G, beta, flags=None, stream=None):
    """shampoo4_update_stats_noalloc on caller-owned CUDA tensors: L_ (m x m)
    and R_ (n x n) fp32 contiguous, G (m x n) fp32 with unit column stride,
    flags an optional int32/uint32 device word.  Marshalling only; the
    library allocates nothing."""
    _need_cuda(G, torch.float32, "G")
    _need_cuda(L_, torch.float32, "L")
    _need_cuda(R_, torch.float32, "R")
    m, n = G.shape
    ldg = _row_major_2d(G, "G")
    if tuple(L_.shape) != (m, m) or not L_.is_contiguous():
        raise ValueError("L must be a contiguous m x m tensor")
    if tuple(R_.shape) != (n, n) or not R_.is_contiguous():
        raise ValueError("R must be a contiguous n x n tensor")
    fp = C.c_void_p(flags.data_ptr()) if flags is not None else C.c_void_p()
    L.call("shampoo4_update_stats_noalloc", C.c_void_p(L_.data_ptr()), C.c_void_p(R_.data_ptr()),
           C.c_void_p(G.data_ptr()), m, n, ldg, float(beta), fp, _stream(stream))


def quant4_tables(codebook="linear_square"):
    cb = (C.c_float * 16)()
    th = (C.c_float * 15)()
    L.call("quant4_tables_ex", _codebook(codebook), cb, th)
    return list(cb), list(th)
