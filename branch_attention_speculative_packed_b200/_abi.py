"""ctypes view of the C ABI in include/ba.h (libba_b200.so).

Argument marshalling only: every step of branch attention runs in the CUDA
library.  Loading fails loudly when the library has not been built; there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libba_b200.so")

BA_OK = 0
BA_ERR_INVALID_ARG = -1
BA_ERR_UNSUPPORTED = -2
BA_ERR_CUDA = -3
BA_ERR_TIMEOUT = -4
BA_ERR_WORKSPACE = -5
BA_ERR_SCRATCH_LIMIT = -6

BA_MASK_CHAIN = 0
BA_MASK_BLOCK = 1
BA_MASK_BITMASK = 2

BA_WS_FWD = 0
BA_WS_BWD = 1

EXPORTED = (
    "ba_workspace_size", "ba_main_fwd", "ba_branch_fwd", "ba_lse_merge", "ba_fused_fwd",
    "ba_bwd", "ba_status_string", "ba_sync_status", "ba_plan_stats", "ba_profile_enable",
    "ba_profile_collect", "ba_last_error_word", "ba_fused_fwd_noalloc", "ba_plan_rank_work",
    "ba_plan_fwd_pairs", "ba_plan_prepare", "ba_clear_cache", "ba_plan_cache_stats",
    "ba_main_fwd_ring", "ba_set_wait_limit", "ba_check_bounded_wait",
)


class BaProblem(ctypes.Structure):
    _fields_ = [
        ("S", ctypes.c_int), ("ndoc", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("d", ctypes.c_int), ("Nb", ctypes.c_int), ("B", ctypes.c_int), ("mode", ctypes.c_int),
        ("R", ctypes.c_int), ("scale", ctypes.c_float),
        ("cu_seqlens_h", ctypes.c_void_p), ("cu_seqlens_d", ctypes.c_void_p),
        ("anchors_h", ctypes.c_void_p), ("anchors_d", ctypes.c_void_p),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("qb", ctypes.c_void_p), ("kb", ctypes.c_void_p), ("vb", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("window", ctypes.c_int),
        ("branch_mask_h", ctypes.c_void_p), ("branch_mask_d", ctypes.c_void_p),
        ("cp_select", ctypes.c_int), ("cp_rank", ctypes.c_int),
    ]


class BAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        extra = ""
        if status == BA_ERR_TIMEOUT:
            w = int(lib().ba_last_error_word())
            extra = (f" [kernel {(w >> 24) & 0x7f}, role {(w >> 16) & 0xff}, "
                     f"wait site {(w >> 8) & 0xff}, parity {w & 1}]")
        super().__init__(f"{where}: {status_string(status)} (status {status}){extra}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it is missing (build it first)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built; run `python -m branch_attention_speculative_packed_b200.build` "
                "(nvcc, sm_100a). There is no fallback path.")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(BaProblem)
        vp, i32, i64p = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)
        L.ba_workspace_size.argtypes = [P, i32]
        L.ba_workspace_size.restype = ctypes.c_size_t
        L.ba_main_fwd.argtypes = [P, vp, vp, vp]
        L.ba_main_fwd_ring.argtypes = [P, vp, vp, vp]
        L.ba_branch_fwd.argtypes = [P, vp, vp, vp]
        L.ba_fused_fwd.argtypes = [P, vp, vp, vp, vp]
        L.ba_fused_fwd_noalloc.argtypes = [P, vp, vp, vp, vp]
        L.ba_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.ba_lse_merge.argtypes = [i32, i32, i32, i32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                   i64p, vp, vp, ctypes.c_int64, vp]
        L.ba_status_string.argtypes = [i32]
        L.ba_status_string.restype = ctypes.c_char_p
        L.ba_sync_status.argtypes = [vp]
        L.ba_plan_stats.argtypes = [P, i64p, i64p, i64p]
        L.ba_plan_rank_work.argtypes = [P, i64p, i32]
        L.ba_plan_rank_work.restype = ctypes.c_int
        L.ba_plan_fwd_pairs.argtypes = [P, ctypes.POINTER(ctypes.c_int32), ctypes.c_int64]
        L.ba_plan_fwd_pairs.restype = ctypes.c_int64
        L.ba_plan_prepare.argtypes = [P, ctypes.POINTER(ctypes.c_double)]
        L.ba_plan_prepare.restype = ctypes.c_int
        L.ba_clear_cache.argtypes = []
        L.ba_clear_cache.restype = None
        L.ba_plan_cache_stats.argtypes = [i64p, i64p, i64p]
        L.ba_plan_cache_stats.restype = None
        L.ba_set_wait_limit.argtypes = [ctypes.c_longlong]
        L.ba_set_wait_limit.restype = None
        L.ba_check_bounded_wait.argtypes = [vp]
        L.ba_check_bounded_wait.restype = ctypes.c_int
        L.ba_last_error_word.argtypes = []
        L.ba_last_error_word.restype = ctypes.c_uint32
        L.ba_profile_enable.argtypes = [i32]
        L.ba_profile_enable.restype = None
        L.ba_profile_collect.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                         ctypes.POINTER(ctypes.c_int), i32]
        L.ba_profile_collect.restype = ctypes.c_int
        for name in ("ba_main_fwd", "ba_main_fwd_ring", "ba_branch_fwd", "ba_fused_fwd", "ba_fused_fwd_noalloc", "ba_bwd",
                     "ba_lse_merge",
                     "ba_sync_status", "ba_plan_stats"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def set_wait_limit(cycles: int) -> None:
    """Bound of every device-side wait of later launches, in SM cycles (<= 0:
    the default, about 2 s).  For testing the failure path."""
    lib().ba_set_wait_limit(int(cycles))


def error_word_fields(word: int) -> dict:
    """Decode a device error word (see ba_last_error_word in include/ba.h)."""
    return {"expired": bool(word >> 31), "kernel": (word >> 24) & 0x7f, "role": (word >> 16) & 0xff,
            "site": (word >> 8) & 0xff, "parity": word & 1}


def clear_cache() -> None:
    """Drop every cached host plan (ba_clear_cache)."""
    lib().ba_clear_cache()


def plan_cache_stats() -> dict:
    """{entries, hits, misses} of the library's host plan cache."""
    e, h, m = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    lib().ba_plan_cache_stats(ctypes.byref(e), ctypes.byref(h), ctypes.byref(m))
    return {"entries": e.value, "hits": h.value, "misses": m.value}


def status_string(status: int) -> str:
    return lib().ba_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != BA_OK:
        raise BAError(status, where)


def profile_enable(on: bool) -> None:
    """Bracket every kernel launch of the library with CUDA events (benchmarks)."""
    lib().ba_profile_enable(1 if on else 0)


def profile_collect() -> dict:
    """{kernel name: (total ms, launches)} of the launches recorded since the
    last collect (waits for their events)."""
    cap = 32
    names = (ctypes.c_char_p * cap)()
    ms = (ctypes.c_double * cap)()
    n = (ctypes.c_int * cap)()
    k = lib().ba_profile_collect(names, ms, n, cap)
    if k < 0:
        raise RuntimeError("ba_profile_collect: event query failed")
    return {names[i].decode(): (ms[i], n[i]) for i in range(min(k, cap))}
