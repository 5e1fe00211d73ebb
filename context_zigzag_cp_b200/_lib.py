"""ctypes view of libcpattn (include/cp_attn.h).  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcpattn.so")

CP_OK = 0
CP_ERR_INVALID_ARG = 1
CP_ERR_UNSUPPORTED = 2
CP_ERR_CUDA = 3
CP_ERR_TIMEOUT = 4
CP_ERR_WORKSPACE = 5
STATUS_NAMES = {0: "CP_OK", 1: "CP_ERR_INVALID_ARG", 2: "CP_ERR_UNSUPPORTED", 3: "CP_ERR_CUDA",
                4: "CP_ERR_TIMEOUT", 5: "CP_ERR_WORKSPACE"}

ROTATE = {"allgather": 0, "ring": 1}
MASK = {"causal": 0, "doc": 1, "full": 2}
MERGE = {"separate": 0, "fused": 1}

# Every function the header declares (checked against include/cp_attn.h by the tests).
EXPORTED = ("cp_plan_shards", "cp_unshard", "cp_attn_fwd", "cp_attn_bwd", "cp_lse_merge",
            "cp_get_device_status", "cp_set_wait_limit_ns", "cp_selftest_wait_timeout",
            "cp_launch_count", "cp_trace_begin", "cp_trace_end", "cp_selftest_exp2",
            "cp_attn_bwd_noalloc", "cp_selftest_stall", "cp_attn_fwd_rank", "cp_attn_fwd_step",
            "cp_attn_bwd_rank", "cp_attn_bwd_step", "cp_f32_to_bf16", "cp_version")

NOALLOC_MAX_ROWS = 4194304

SHARD = {"sequence": 0, "doc": 1}

KERNEL_NAMES = {1: "plan_meta", 2: "plan_index", 3: "gather", 4: "fwd", 5: "merge",
                6: "bwd_prep", 7: "bwd_dkdv", 8: "bwd_dq", 9: "selftest", 10: "selftest_exp2",
                11: "cast", 12: "bwd_fused", 13: "dq_convert"}
KERNEL_IDS = {name: i for i, name in KERNEL_NAMES.items()}


class CpProblem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("cp_size", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("rotate", ctypes.c_int32), ("mask", ctypes.c_int32), ("merge", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("num_docs", ctypes.c_int32),
                ("window", ctypes.c_int32), ("bwd_one_pass", ctypes.c_int32),
                ("shard", ctypes.c_int32), ("cu_seqlens", ctypes.c_void_p)]


class CpPlan(ctypes.Structure):
    _fields_ = [("perm", ctypes.c_void_p), ("inv_perm", ctypes.c_void_p),
                ("src", ctypes.c_void_p), ("doc_start", ctypes.c_void_p),
                ("rank_cu_off", ctypes.c_void_p), ("rank_cu", ctypes.c_void_p),
                ("pairs", ctypes.c_void_p), ("tile_orig", ctypes.c_void_p),
                ("tile_shard", ctypes.c_void_p)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libcpattn.so from the package directory.  There is no fallback: a
    missing or broken library is an error."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libcpattn.so not built at {LIB_PATH}; run "
                          "`python -m context_zigzag_cp_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz = ctypes.c_void_p, ctypes.POINTER(ctypes.c_size_t)
    P, PL = ctypes.POINTER(CpProblem), ctypes.POINTER(CpPlan)
    i64p = ctypes.POINTER(ctypes.c_int64)
    lib.cp_plan_shards.argtypes = [P, PL, ctypes.c_int32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                   i64p, i64p, vp, sz, vp]
    lib.cp_unshard.argtypes = [P, PL, ctypes.c_int32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                               i64p, i64p, vp]
    lib.cp_attn_fwd.argtypes = [P, PL, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cp_attn_bwd.argtypes = [P, PL, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cp_attn_bwd_noalloc.argtypes = [P, PL, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.cp_lse_merge.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, vp, vp, vp, vp, vp]
    lib.cp_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_int32), vp]
    lib.cp_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.cp_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.cp_version.argtypes = []
    lib.cp_launch_count.argtypes = []
    lib.cp_selftest_exp2.argtypes = [vp, vp, vp, ctypes.c_int64, vp]
    lib.cp_trace_begin.argtypes = [ctypes.POINTER(vp), ctypes.c_int32]
    lib.cp_trace_end.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
    lib.cp_selftest_stall.argtypes = [ctypes.c_int32, P, PL, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                      vp, sz, vp]
    i32 = ctypes.c_int32
    lib.cp_attn_fwd_rank.argtypes = [P, PL, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cp_attn_fwd_step.argtypes = [P, PL, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.cp_attn_bwd_rank.argtypes = [P, PL, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cp_attn_bwd_step.argtypes = [P, PL, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cp_f32_to_bf16.argtypes = [vp, vp, ctypes.c_int64, vp]
    for name in EXPORTED:
        getattr(lib, name).restype = ctypes.c_int32
    lib.cp_launch_count.restype = ctypes.c_int64
    _lib = lib
    return lib
