"""ctypes declarations of the libwal.so C ABI (include/wal.h), same names.

Every function takes plain integers for pointers (host pointers from numpy,
device pointers from torch ``data_ptr()``), raises ``WalError`` on a non-OK
status and otherwise returns what the C function returns.
"""
import ctypes
import os

from .build import LIB, build

WAL_OK = 0
WAL_ERR_ARG = -1
WAL_ERR_SHAPE = -2
WAL_ERR_FORMAT = -3
WAL_ERR_WORKSPACE = -4
WAL_ERR_CUDA = -5
WAL_ERR_UNSUPPORTED = -6
WAL_ERR_TIMEOUT = -7
WAL_MAX_RANK = 32
WAL_MAX_SMALL_M = 16
WAL_NOALLOC_SCRATCH_BYTES = 16 << 20

EXPORTED_SYMBOLS = [
    "wal_packed_sizes", "wal_pack_matrix", "wal_validate", "wal_unpack_matrix",
    "wal_workspace_bytes", "wal_gemv", "wal_gemm_small_m", "wal_gemm_tc_noalloc", "wal_noalloc_status", "wal_device_status",
    "wal_body_workspace_bytes", "wal_body_pass", "wal_body_plan_destroy", "wal_debug_barrier_fault",
    "wal_pq2_bytes", "wal_pq2_pack", "wal_pq2_workspace_bytes", "wal_pq2_gemm",
    "wal_pq2_body_workspace_bytes", "wal_pq2_body_pass",
    "wal_base3_bytes", "wal_base3_pack", "wal_base3_convert",
    "wal_rc1_sizes", "wal_rc1_prepare", "wal_rc1_workspace_bytes", "wal_rc1_gemm",
    "wal_rc1_body_workspace_bytes", "wal_rc1_body_pass",
    "wal_int4_sizes", "wal_int3_sizes", "wal_int4_pack", "wal_int3_pack", "wal_int4_workspace_bytes",
    "wal_int4_gemm", "wal_int3_embed",
    "wal_status_string", "wal_last_error",
]


class WalError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {wal_status_string(status)} ({wal_last_error()})")


class wal_matrix(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("k", ctypes.c_int32), ("r", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("sites", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("u_bits", ctypes.c_void_p), ("v_bits", ctypes.c_void_p), ("lr_scale", ctypes.c_void_p),
    ]


class wal_rc1_matrix(ctypes.Structure):
    _fields_ = wal_matrix._fields_


class wal_int4_matrix(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class wal_int3_table(ctypes.Structure):
    _fields_ = [("V", ctypes.c_int32), ("H", ctypes.c_int32), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class wal_pq2_matrix(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("blocks", ctypes.c_void_p)]


def _load():
    # built in-tree; rebuilt first when a source is newer than the library
    path = build()
    return ctypes.CDLL(path)


lib = _load()
lib_path = LIB

_vp, _sz, _i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
_MP = ctypes.POINTER(wal_matrix)

lib.wal_packed_sizes.argtypes = [_i, _i, _i, _i, ctypes.POINTER(_sz)]
lib.wal_pack_matrix.argtypes = [_vp] * 8 + [_i] * 4 + [ctypes.POINTER(_vp)]
lib.wal_validate.argtypes = [_MP, _vp, _sz, _vp]
lib.wal_unpack_matrix.argtypes = [_MP] + [_vp] * 7 + [_vp]
lib.wal_workspace_bytes.argtypes = [_MP, _i]
lib.wal_workspace_bytes.restype = _sz
lib.wal_gemv.argtypes = [_MP, _vp, _vp, _vp, _sz, _vp]
lib.wal_gemm_small_m.argtypes = [_MP, _vp, _i, _i, _vp, _i, _vp, _sz, _vp]
lib.wal_gemm_tc_noalloc.argtypes = [_MP, _vp, _i, _i, _vp, _i, _vp]
lib.wal_device_status.argtypes = [_vp, _vp]
lib.wal_noalloc_status.argtypes = [_vp]
lib.wal_body_workspace_bytes.argtypes = [_MP, _i, _i]
lib.wal_body_workspace_bytes.restype = _sz
lib.wal_body_pass.argtypes = [ctypes.POINTER(_vp), _MP, _i, ctypes.POINTER(ctypes.c_int32),
                              ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp, _sz, _vp]
lib.wal_body_plan_destroy.argtypes = [_vp]
lib.wal_body_plan_destroy.restype = None
lib.wal_debug_barrier_fault.argtypes = [_i]
_PP = ctypes.POINTER(wal_pq2_matrix)
lib.wal_pq2_bytes.argtypes = [_i, _i]
lib.wal_pq2_bytes.restype = _sz
lib.wal_pq2_pack.argtypes = [_vp, _vp, _i, _i, _vp]
lib.wal_pq2_workspace_bytes.argtypes = [_PP, _i]
lib.wal_pq2_workspace_bytes.restype = _sz
lib.wal_pq2_gemm.argtypes = [_PP, _vp, _i, _i, _vp, _i, _vp, _sz, _vp]
lib.wal_pq2_body_workspace_bytes.argtypes = [_PP, _i, _i]
lib.wal_pq2_body_workspace_bytes.restype = _sz
lib.wal_pq2_body_pass.argtypes = [ctypes.POINTER(_vp), _PP, _i, ctypes.POINTER(ctypes.c_int32),
                                  ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp, _sz, _vp]
lib.wal_base3_bytes.argtypes = [_i, _i]
lib.wal_base3_bytes.restype = _sz
lib.wal_base3_pack.argtypes = [_vp, _i, _i, _vp]
lib.wal_base3_convert.argtypes = [_vp, _vp, _i, _i, _vp, _vp, _vp, _sz, _vp]
_RP = ctypes.POINTER(wal_rc1_matrix)
lib.wal_rc1_sizes.argtypes = [_i, _i, _i, _i, _i, ctypes.POINTER(_sz), ctypes.POINTER(_sz)]
lib.wal_rc1_prepare.argtypes = [_i, _i, _i, _vp, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.wal_rc1_workspace_bytes.argtypes = [_RP, _i]
lib.wal_rc1_workspace_bytes.restype = _sz
lib.wal_rc1_gemm.argtypes = [_RP, _vp, _i, _i, _vp, _i, _vp, _sz, _vp]
lib.wal_rc1_body_workspace_bytes.argtypes = [_RP, _i, _i]
lib.wal_rc1_body_workspace_bytes.restype = _sz
lib.wal_rc1_body_pass.argtypes = [ctypes.POINTER(_vp), _RP, _i, ctypes.POINTER(ctypes.c_int32),
                                  ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp, _sz, _vp]
lib.wal_int4_sizes.argtypes = [_i, _i, ctypes.POINTER(_sz)]
lib.wal_int3_sizes.argtypes = [_i, _i, ctypes.POINTER(_sz)]
lib.wal_int4_pack.argtypes = [_vp, _vp, _i, _i, _vp, _vp]
lib.wal_int3_pack.argtypes = [_vp, _vp, _i, _i, _vp, _vp]
lib.wal_int4_workspace_bytes.argtypes = [ctypes.POINTER(wal_int4_matrix), _i]
lib.wal_int4_workspace_bytes.restype = _sz
lib.wal_int4_gemm.argtypes = [ctypes.POINTER(wal_int4_matrix), _vp, _i, _i, _vp, _i, _vp, _sz, _vp]
lib.wal_int3_embed.argtypes = [ctypes.POINTER(wal_int3_table), _vp, _i, _vp, _vp, _sz, _vp]
lib.wal_status_string.argtypes = [_i]
lib.wal_status_string.restype = ctypes.c_char_p
lib.wal_last_error.argtypes = []
lib.wal_last_error.restype = ctypes.c_char_p


def wal_status_string(status):
    return lib.wal_status_string(int(status)).decode()


def wal_last_error():
    return lib.wal_last_error().decode()


def _check(status, where):
    if status != WAL_OK:
        raise WalError(status, where)
    return status


def wal_packed_sizes(N, K, k, r):
    out = (_sz * 6)()
    _check(lib.wal_packed_sizes(N, K, k, r, out), "wal_packed_sizes")
    return [int(v) for v in out]


def wal_pack_matrix(T, site_pos, site_sign, alpha, beta, U, V, lr_scale, N, K, k, r, out):
    arr = (_vp * 6)(*[int(p) if p else None for p in out])
    return _check(lib.wal_pack_matrix(T, site_pos, site_sign, alpha, beta, U, V, lr_scale,
                                      N, K, k, r, arr), "wal_pack_matrix")


def wal_validate(m, ws, ws_bytes, stream):
    return _check(lib.wal_validate(ctypes.byref(m), ws, ws_bytes, stream), "wal_validate")


def wal_unpack_matrix(m, T, site_pos, site_sign, alpha, beta, U, V, stream):
    return _check(lib.wal_unpack_matrix(ctypes.byref(m), T, site_pos, site_sign, alpha, beta, U, V,
                                        stream), "wal_unpack_matrix")


def wal_workspace_bytes(m, M):
    return int(lib.wal_workspace_bytes(ctypes.byref(m), M))


def wal_gemv(m, x, y, ws, ws_bytes, stream):
    return _check(lib.wal_gemv(ctypes.byref(m), x, y, ws, ws_bytes, stream), "wal_gemv")


def wal_gemm_small_m(m, X, M, ldx, Y, ldy, ws, ws_bytes, stream):
    return _check(lib.wal_gemm_small_m(ctypes.byref(m), X, M, ldx, Y, ldy, ws, ws_bytes, stream),
                  "wal_gemm_small_m")


def wal_gemm_tc_noalloc(m, X, M, ldx, Y, ldy, stream):
    return _check(lib.wal_gemm_tc_noalloc(ctypes.byref(m), X, M, ldx, Y, ldy, stream), "wal_gemm_tc_noalloc")


def wal_noalloc_status(stream):
    return _check(lib.wal_noalloc_status(stream), "wal_noalloc_status")


def wal_device_status(ws, stream):
    return _check(lib.wal_device_status(ws, stream), "wal_device_status")


def wal_body_workspace_bytes(mats, M):
    arr = (wal_matrix * len(mats))(*mats)
    return int(lib.wal_body_workspace_bytes(arr, len(mats), M))


def wal_body_pass(plan, mats, stage_of, xs, ys, M, ws, ws_bytes, stream):
    """plan: a ctypes.c_void_p holding the plan handle (None on the first call)."""
    n = len(mats)
    marr = (wal_matrix * n)(*mats)
    sarr = (ctypes.c_int32 * n)(*stage_of)
    xarr = (_vp * n)(*xs)
    yarr = (_vp * n)(*ys)
    return _check(lib.wal_body_pass(ctypes.byref(plan), marr, n, sarr, xarr, yarr, M, ws, ws_bytes,
                                    stream), "wal_body_pass")


def wal_body_plan_destroy(plan):
    lib.wal_body_plan_destroy(plan)


def wal_debug_barrier_fault(on):
    """Fault injection for the timeout tests: body-pass plans built while it is
    set never pass their first grid barrier.  Returns the previous setting."""
    return int(lib.wal_debug_barrier_fault(1 if on else 0))


def wal_pq2_bytes(N, K):
    return int(lib.wal_pq2_bytes(N, K))


def wal_pq2_pack(T, d, N, K, out):
    return _check(lib.wal_pq2_pack(T, d, N, K, out), "wal_pq2_pack")


def wal_pq2_workspace_bytes(m, M):
    return int(lib.wal_pq2_workspace_bytes(ctypes.byref(m), M))


def wal_pq2_gemm(m, X, M, ldx, Y, ldy, ws, ws_bytes, stream):
    return _check(lib.wal_pq2_gemm(ctypes.byref(m), X, M, ldx, Y, ldy, ws, ws_bytes, stream), "wal_pq2_gemm")


def wal_pq2_body_workspace_bytes(mats, M):
    arr = (wal_pq2_matrix * len(mats))(*mats)
    return int(lib.wal_pq2_body_workspace_bytes(arr, len(mats), M))


def wal_pq2_body_pass(plan, mats, stage_of, xs, ys, M, ws, ws_bytes, stream):
    """plan: a ctypes.c_void_p holding the plan handle (None on the first call)."""
    n = len(mats)
    marr = (wal_pq2_matrix * n)(*mats)
    sarr = (ctypes.c_int32 * n)(*stage_of)
    xarr = (_vp * n)(*xs)
    yarr = (_vp * n)(*ys)
    return _check(lib.wal_pq2_body_pass(ctypes.byref(plan), marr, n, sarr, xarr, yarr, M, ws, ws_bytes,
                                        stream), "wal_pq2_body_pass")


def wal_base3_bytes(N, K):
    return int(lib.wal_base3_bytes(N, K))


def wal_base3_pack(T, N, K, out):
    return _check(lib.wal_base3_pack(T, N, K, out), "wal_base3_pack")


def wal_base3_convert(b3, scales_bf16, N, K, codes, alpha, ws, ws_bytes, stream):
    return _check(lib.wal_base3_convert(b3, scales_bf16, N, K, codes, alpha, ws, ws_bytes, stream),
                  "wal_base3_convert")


def wal_rc1_sizes(N, K, k, r1, r2):
    can, prep = (_sz * 7)(), (_sz * 4)()
    _check(lib.wal_rc1_sizes(N, K, k, r1, r2, can, prep), "wal_rc1_sizes")
    return [int(v) for v in can], [int(v) for v in prep]


def wal_rc1_prepare(N, K, k, scales24, r1, u1, v1, s1, r2, u2, v2, s2, scales32, u_bits, v_bits, lr32, stream):
    return _check(lib.wal_rc1_prepare(N, K, k, scales24, r1, u1, v1, s1, r2, u2, v2, s2, scales32, u_bits, v_bits,
                                      lr32, stream), "wal_rc1_prepare")


def wal_rc1_workspace_bytes(m, M):
    return int(lib.wal_rc1_workspace_bytes(ctypes.byref(m), M))


def wal_rc1_gemm(m, X, M, ldx, Y, ldy, ws, ws_bytes, stream):
    return _check(lib.wal_rc1_gemm(ctypes.byref(m), X, M, ldx, Y, ldy, ws, ws_bytes, stream), "wal_rc1_gemm")


def wal_rc1_body_workspace_bytes(mats, M):
    arr = (wal_rc1_matrix * len(mats))(*mats)
    return int(lib.wal_rc1_body_workspace_bytes(arr, len(mats), M))


def wal_rc1_body_pass(plan, mats, stage_of, xs, ys, M, ws, ws_bytes, stream):
    """plan: a ctypes.c_void_p holding the plan handle (None on the first call)."""
    n = len(mats)
    marr = (wal_rc1_matrix * n)(*mats)
    sarr = (ctypes.c_int32 * n)(*stage_of)
    xarr = (_vp * n)(*xs)
    yarr = (_vp * n)(*ys)
    return _check(lib.wal_rc1_body_pass(ctypes.byref(plan), marr, n, sarr, xarr, yarr, M, ws, ws_bytes,
                                        stream), "wal_rc1_body_pass")


def wal_int4_sizes(N, K):
    out = (_sz * 2)()
    _check(lib.wal_int4_sizes(N, K, out), "wal_int4_sizes")
    return [int(v) for v in out]


def wal_int3_sizes(V, H):
    out = (_sz * 2)()
    _check(lib.wal_int3_sizes(V, H, out), "wal_int3_sizes")
    return [int(v) for v in out]


def wal_int4_pack(q, d, N, K, codes, scales):
    return _check(lib.wal_int4_pack(q, d, N, K, codes, scales), "wal_int4_pack")


def wal_int3_pack(q, d, V, H, codes, scales):
    return _check(lib.wal_int3_pack(q, d, V, H, codes, scales), "wal_int3_pack")


def wal_int4_workspace_bytes(m, M):
    return int(lib.wal_int4_workspace_bytes(ctypes.byref(m), M))


def wal_int4_gemm(m, X, M, ldx, Y, ldy, ws, ws_bytes, stream):
    return _check(lib.wal_int4_gemm(ctypes.byref(m), X, M, ldx, Y, ldy, ws, ws_bytes, stream), "wal_int4_gemm")


def wal_int3_embed(t, ids, M, out, ws, ws_bytes, stream):
    return _check(lib.wal_int3_embed(ctypes.byref(t), ids, M, out, ws, ws_bytes, stream), "wal_int3_embed")
