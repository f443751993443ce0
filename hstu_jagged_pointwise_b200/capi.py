"""ctypes declarations of libhstu_b200 (the C ABI in include/hstu.h).

Importing this module loads the in-tree shared library and raises when it is
missing: there is no CPU fallback for any entry point.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhstu_b200.so")

HSTU_OK = 0
HSTU_ERR_INVALID_ARG = -1
HSTU_ERR_UNSUPPORTED = -2
HSTU_ERR_CUDA = -3
HSTU_ERR_DEVICE_TIMEOUT = -4
HSTU_ERR_DEVICE_BOUNDS = -5
HSTU_ERR_WORKSPACE = -6

HSTU_BF16 = 0
HSTU_F32 = 1
HSTU_MASK_CAUSAL = 0
HSTU_MASK_MTGR = 1
HSTU_MASK_MFALCON_SEQ = 2

# every symbol the header declares
EXPORTS = (
    "hstu_attn_workspace_bytes", "hstu_attn_fwd", "hstu_attn_bwd", "hstu_mfalcon_workspace_bytes",
    "hstu_mfalcon_score", "hstu_debug_indices", "hstu_check_device_error", "hstu_status_string",
    "hstu_version", "hstu_profile_enable", "hstu_profile_read", "hstu_profile_kind_name",
    "hstu_attn_fwd_noalloc", "hstu_mfalcon_cache_history", "hstu_attn_fwd_gln", "hstu_attn_bwd_gln",
    "hstu_attn_workspace_bytes_gln", "hstu_f1_fwd", "hstu_f2_fwd", "hstu_f1_bwd_workspace_bytes",
    "hstu_f2_bwd_workspace_bytes", "hstu_f1_bwd", "hstu_f2_bwd", "hstu_sl_sample", "hstu_gather_rows",
    "hstu_pack_balanced", "hstu_debug_set_wait_fault", "hstu_attn_bwd_dy",
)

NOALLOC_SCRATCH_BYTES = 4 << 20   # HSTU_NOALLOC_SCRATCH_BYTES


class HstuDims(C.Structure):
    _fields_ = [("B", C.c_int32), ("T", C.c_int32), ("H", C.c_int32), ("d_qk", C.c_int32),
                ("d_v", C.c_int32), ("dtype", C.c_int32), ("n_pos", C.c_int32),
                ("n_tbuckets", C.c_int32), ("max_seq_len", C.c_int32), ("alpha", C.c_float),
                ("ln_eps", C.c_float)]


class HstuMaskSpec(C.Structure):
    _fields_ = [("kind", C.c_int32), ("n_static", C.c_void_p), ("n_realtime", C.c_void_p)]


class HstuNormSpec(C.Structure):
    _fields_ = [("n_groups", C.c_int32), ("token_group", C.c_void_p)]


class HstuMfalconDims(C.Structure):
    _fields_ = [("B", C.c_int32), ("T_hist", C.c_int32), ("T_cand", C.c_int32), ("H", C.c_int32),
                ("d_qk", C.c_int32), ("d_v", C.c_int32), ("dtype", C.c_int32), ("n_pos", C.c_int32),
                ("n_tbuckets", C.c_int32), ("max_hist_len", C.c_int32), ("max_cand_len", C.c_int32),
                ("alpha", C.c_float), ("ln_eps", C.c_float)]


class HstuError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m hstu_jagged_pointwise_b200.build` "
            "(there is no CPU fallback)")
    lib = C.CDLL(LIB_PATH)
    P = C.c_void_p
    S = C.c_size_t
    i32 = C.c_int32
    lib.hstu_attn_workspace_bytes.argtypes = [C.POINTER(HstuDims), i32, i32]
    lib.hstu_attn_workspace_bytes.restype = S
    lib.hstu_attn_fwd.argtypes = [C.POINTER(HstuDims), C.POINTER(HstuMaskSpec)] + [P] * 15 + [S, P]
    lib.hstu_attn_fwd.restype = C.c_int
    lib.hstu_attn_fwd_noalloc.argtypes = [C.POINTER(HstuDims), C.POINTER(HstuMaskSpec)] + [P] * 15 + [P]
    lib.hstu_attn_fwd_noalloc.restype = C.c_int
    lib.hstu_attn_bwd.argtypes = [C.POINTER(HstuDims), C.POINTER(HstuMaskSpec)] + [P] * 23 + [S, P]
    lib.hstu_attn_bwd.restype = C.c_int
    lib.hstu_attn_bwd_dy.argtypes = [C.POINTER(HstuDims), C.POINTER(HstuMaskSpec)] + [P] * 14 + [S, P]
    lib.hstu_attn_bwd_dy.restype = C.c_int
    NS = C.POINTER(HstuNormSpec)
    lib.hstu_attn_workspace_bytes_gln.argtypes = [C.POINTER(HstuDims), i32, i32, i32]
    lib.hstu_attn_workspace_bytes_gln.restype = S
    lib.hstu_attn_fwd_gln.argtypes = [C.POINTER(HstuDims), C.POINTER(HstuMaskSpec), NS] + [P] * 15 + [S, P]
    lib.hstu_attn_fwd_gln.restype = C.c_int
    lib.hstu_attn_bwd_gln.argtypes = [C.POINTER(HstuDims), C.POINTER(HstuMaskSpec), NS] + [P] * 23 + [S, P]
    lib.hstu_attn_bwd_gln.restype = C.c_int
    lib.hstu_mfalcon_workspace_bytes.argtypes = [C.POINTER(HstuMfalconDims), i32]
    lib.hstu_mfalcon_workspace_bytes.restype = S
    lib.hstu_mfalcon_score.argtypes = [C.POINTER(HstuMfalconDims)] + [P] * 14 + [i32] + [P] * 3 + [S, P]
    lib.hstu_mfalcon_score.restype = C.c_int
    lib.hstu_mfalcon_cache_history.argtypes = [i32, i32, i32, i32, P, P, P, P, P, C.c_int64, P, P, P, P, P, P]
    lib.hstu_mfalcon_cache_history.restype = C.c_int
    lib.hstu_f1_fwd.argtypes = [i32, i32, i32] + [P] * 10
    lib.hstu_f1_fwd.restype = C.c_int
    lib.hstu_f2_fwd.argtypes = [i32, i32, i32] + [P] * 7
    lib.hstu_f2_fwd.restype = C.c_int
    lib.hstu_f1_bwd_workspace_bytes.argtypes = [i32, i32]
    lib.hstu_f1_bwd_workspace_bytes.restype = S
    lib.hstu_f2_bwd_workspace_bytes.argtypes = [i32, i32]
    lib.hstu_f2_bwd_workspace_bytes.restype = S
    lib.hstu_f1_bwd.argtypes = [i32, i32, i32] + [P] * 12 + [S, P, P]
    lib.hstu_f1_bwd.restype = C.c_int
    lib.hstu_f2_bwd.argtypes = [i32, i32, i32] + [P] * 7 + [S, P, P]
    lib.hstu_f2_bwd.restype = C.c_int
    lib.hstu_sl_sample.argtypes = [i32, i32, P, i32, C.c_uint64, C.c_int64, P, P, P, P]
    lib.hstu_sl_sample.restype = C.c_int
    lib.hstu_gather_rows.argtypes = [C.c_int64, i32, P, C.c_int64, P, P, P]
    lib.hstu_gather_rows.restype = C.c_int
    lib.hstu_pack_balanced.argtypes = [i32, P, i32, P, P, P, P]
    lib.hstu_pack_balanced.restype = C.c_int
    lib.hstu_debug_indices.argtypes = [i32, i32, P, P, P, P, i32, i32, P, P, P, P, P]
    lib.hstu_debug_indices.restype = C.c_int
    lib.hstu_check_device_error.argtypes = [P, P]
    lib.hstu_check_device_error.restype = C.c_int
    lib.hstu_status_string.argtypes = [C.c_int]
    lib.hstu_status_string.restype = C.c_char_p
    lib.hstu_version.argtypes = []
    lib.hstu_version.restype = C.c_char_p
    lib.hstu_debug_set_wait_fault.argtypes = [C.c_int64, i32]
    lib.hstu_debug_set_wait_fault.restype = C.c_int
    lib.hstu_profile_enable.argtypes = [i32]
    lib.hstu_profile_enable.restype = C.c_int
    lib.hstu_profile_read.argtypes = [i32, P, P]
    lib.hstu_profile_read.restype = C.c_int
    lib.hstu_profile_kind_name.argtypes = [i32]
    lib.hstu_profile_kind_name.restype = C.c_char_p
    return lib


LIB = load()


def status_string(status: int) -> str:
    return LIB.hstu_status_string(int(status)).decode()


def profile_enable(on: bool) -> None:
    check(LIB.hstu_profile_enable(1 if on else 0), "hstu_profile_enable")


def profile_read() -> dict:
    """{kernel name: (launches, total ms)} for kinds with at least one launch."""
    n = 32
    launches = (C.c_int32 * n)()
    ms = (C.c_double * n)()
    k = LIB.hstu_profile_read(n, launches, ms)
    if k < 0:
        raise HstuError(k, "hstu_profile_read")
    return {LIB.hstu_profile_kind_name(i).decode(): (int(launches[i]), float(ms[i]))
            for i in range(min(k, n)) if launches[i] > 0}


class wait_fault:
    """Context manager around hstu_debug_set_wait_fault (test hook): inside it, the
    pipelined kernels' main-loop waits give up after `limit_cycles` SM cycles and,
    with withhold=True, each CTA's producer withholds its first tile load so that
    those waits run out.  Normal operation is restored on exit."""

    def __init__(self, limit_cycles: int, withhold: bool = True):
        self.limit, self.withhold = int(limit_cycles), bool(withhold)

    def __enter__(self):
        check(LIB.hstu_debug_set_wait_fault(self.limit, 1 if self.withhold else 0), "hstu_debug_set_wait_fault")
        return self

    def __exit__(self, *exc):
        check(LIB.hstu_debug_set_wait_fault(0, 0), "hstu_debug_set_wait_fault")
        return False


def check(status: int, where: str) -> None:
    if status != HSTU_OK:
        raise HstuError(status, where)
