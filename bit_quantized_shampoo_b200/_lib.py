"""ctypes binding of libshampoo4.so: argument marshalling only.

Every function here has the name and argument order of the C entry point in
include/shampoo4.h.  Nothing is computed in Python; a missing library raises.
"""
from __future__ import annotations

import ctypes as C
import os

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libshampoo4.so")
_lib = None

c_size_p = C.POINTER(C.c_size_t)
c_i32_p = C.POINTER(C.c_int32)
c_i64_p = C.POINTER(C.c_int64)
c_u32_p = C.POINTER(C.c_uint32)
c_f32_p = C.POINTER(C.c_float)

SHAMPOO4_OK = 0
STATUS_NAMES = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_CUDA", 3: "ERR_NOT_READY",
                4: "ERR_NONFINITE", 5: "ERR_WORKSPACE", 6: "ERR_UNSUPPORTED", 7: "ERR_TIMEOUT"}
FLAG_NONFINITE_GRAD = 0x1
FLAG_REFRESH_FAILED = 0x2
FLAG_NONFINITE_STATE = 0x4
FLAG_TIMEOUT = 0x8
FLAG_QR_FALLBACK = 0x10
FLAG_GRAFT_SKIPPED = 0x20
GRAFT_SGD = 0
GRAFT_ADAM = 1
PREC_TF32 = 0
PREC_FP32 = 1
CODEBOOK_LINEAR_SQUARE = 0
CODEBOOK_DYNAMIC_TREE = 1
ROOT_EIGEN = 0
ROOT_NEWTON = 1
ROOT_NEWTON_Q4 = 2


class Config(C.Structure):
    _fields_ = [("beta", C.c_float), ("eps", C.c_float), ("max_block", C.c_int32),
                ("quant_block", C.c_int32), ("bjorck_iters", C.c_int32), ("precision", C.c_int32),
                ("compressed_stats", C.c_int32), ("refresh_rank", C.c_int32), ("refresh_world", C.c_int32),
                ("codebook", C.c_int32), ("root_method", C.c_int32), ("newton_iters", C.c_int32),
                ("group_tiles", C.c_int32)]


class GraftConfig(C.Structure):
    _fields_ = [("kind", C.c_int32), ("beta1", C.c_float), ("beta2", C.c_float),
                ("adam_eps", C.c_float), ("graft_eps", C.c_float), ("dir_norms", C.c_int32)]


class Param(C.Structure):
    _fields_ = [("rows", C.c_int64), ("cols", C.c_int64)]


class Shampoo4Error(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")
        self.status = status


_SIGS = {
    "shampoo4_init": [C.POINTER(Config), C.POINTER(Param), C.c_int32, C.POINTER(C.c_void_p)],
    "shampoo4_sizes": [C.c_void_p, c_size_p, c_size_p],
    "shampoo4_bind": [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p],
    "shampoo4_set_has_basis": [C.c_void_p, C.c_int32],
    "shampoo4_update_stats": [C.c_void_p, C.POINTER(C.c_void_p), c_i64_p, C.c_void_p],
    "shampoo4_refresh_roots": [C.c_void_p, C.c_void_p],
    "shampoo4_precondition": [C.c_void_p, C.POINTER(C.c_void_p), c_i64_p, C.POINTER(C.c_void_p),
                              c_i64_p, C.c_void_p],
    "shampoo4_get_status_flags": [C.c_void_p, c_u32_p, C.c_void_p],
    "shampoo4_counts": [C.c_void_p, c_i32_p, c_i32_p],
    "shampoo4_block_info": [C.c_void_p, C.c_int32, c_i32_p, c_i64_p, c_i64_p, c_i32_p, c_i32_p],
    "shampoo4_factor_layout": [C.c_void_p, C.c_int32, c_size_p, c_size_p, c_size_p, c_size_p, c_i32_p],
    "shampoo4_debug_q_offset": [C.c_void_p, C.c_int32, c_size_p],
    "shampoo4_debug_s_offset": [C.c_void_p, C.c_int32, c_size_p],
    "shampoo4_debug_capture_bytes": [C.c_void_p, c_size_p],
    "shampoo4_debug_capture": [C.c_void_p, C.c_void_p],
    "shampoo4_debug_capture_layout": [C.c_void_p, C.c_int32, c_size_p, c_size_p],
    "shampoo4_debug_wait_limit": [C.c_void_p, C.c_uint64],
    "shampoo4_debug_refresh_parts": [C.c_void_p, C.c_int32],
    "shampoo4_factor_owner": [C.c_void_p, C.c_int32, c_i32_p],
    "shampoo4_owner_span": [C.c_void_p, C.c_int32, c_size_p, c_size_p],
    "quant4_pack": [C.POINTER(C.c_void_p), c_i64_p, C.c_int32, C.POINTER(C.c_void_p),
                    C.POINTER(C.c_void_p), C.c_void_p],
    "quant4_unpack": [C.POINTER(C.c_void_p), C.POINTER(C.c_void_p), c_i64_p, C.c_int32,
                      C.POINTER(C.c_void_p), C.c_void_p],
    "quant4_tables": [c_f32_p, c_f32_p],
    "quant4_pack_ex": [C.POINTER(C.c_void_p), c_i64_p, C.c_int32, C.POINTER(C.c_void_p),
                       C.POINTER(C.c_void_p), C.c_int32, C.c_void_p],
    "quant4_unpack_ex": [C.POINTER(C.c_void_p), C.POINTER(C.c_void_p), c_i64_p, C.c_int32,
                         C.POINTER(C.c_void_p), C.c_int32, C.c_void_p],
    "quant4_tables_ex": [C.c_int32, c_f32_p, c_f32_p],
    "shampoo4_root_offset": [C.c_void_p, C.c_int32, c_size_p],
    "shampoo4_update_stats_noalloc": [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_int64,
                                      C.c_float, C.c_void_p, C.c_void_p],
    "shampoo4_graft_state_bytes": [C.c_void_p, C.c_int32, c_size_p],
    "shampoo4_graft_layout": [C.c_void_p, C.c_int32, C.c_int32, c_size_p, c_size_p],
    "shampoo4_graft_update": [C.c_void_p, C.POINTER(GraftConfig), C.c_void_p, C.c_int64, C.c_float,
                              C.POINTER(C.c_void_p), c_i64_p, C.POINTER(C.c_void_p), c_i64_p,
                              C.POINTER(C.c_void_p), c_i64_p, C.c_void_p],
    "shampoo4_timing_enable": [C.c_void_p, C.c_int32],
    "shampoo4_timing_read": [C.c_void_p, C.c_int32, C.POINTER(C.c_double), c_i64_p, C.POINTER(C.c_double),
                             C.POINTER(C.c_double)],
}


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(_PATH):
            raise RuntimeError(f"{_PATH} is not built: run `python -m bit_quantized_shampoo_b200.build`")
        L = C.CDLL(_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = C.c_int
        L.shampoo4_destroy.argtypes = [C.c_void_p]
        L.shampoo4_destroy.restype = None
        L.shampoo4_stage_name.argtypes = [C.c_int32]
        L.shampoo4_stage_name.restype = C.c_char_p
        L.shampoo4_status_string.argtypes = [C.c_int]
        L.shampoo4_status_string.restype = C.c_char_p
        _lib = L
    return _lib


def library_path() -> str:
    return _PATH


def check(fn: str, status: int) -> None:
    if status != SHAMPOO4_OK:
        raise Shampoo4Error(fn, status)


def call(fn: str, *args) -> None:
    check(fn, getattr(lib(), fn)(*args))


def ptr_array(ptrs):
    return (C.c_void_p * max(1, len(ptrs)))(*[C.c_void_p(int(p)) for p in ptrs])


def i64_array(vals):
    return (C.c_int64 * max(1, len(vals)))(*[int(v) for v in vals])
