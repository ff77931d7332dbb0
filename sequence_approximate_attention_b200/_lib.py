"""ctypes view of ``libspava.so`` (the C ABI in include/spava.h)."""

import ctypes
import os

from . import build as _build

c_int32 = ctypes.c_int32
c_void_p = ctypes.c_void_p
c_size_t = ctypes.c_size_t

SPAVA_OK = 0
SPAVA_ERR_INVALID_ARG = 1
SPAVA_ERR_UNSUPPORTED = 2
SPAVA_ERR_CUDA = 3
SPAVA_ERR_TIMEOUT = 4
SPAVA_ERR_DEVICE_CHECK = 5
SPAVA_SCORES_GIVEN = 1

SPAVA_SHARD_CONTIGUOUS = 0
SPAVA_SHARD_ZIGZAG = 1
SPAVA_SHARD_LONGEST_FIRST = 2
SPAVA_SHARD_SELECT, SPAVA_SHARD_LOCAL, SPAVA_SHARD_REMOTE, SPAVA_SHARD_MERGE, SPAVA_SHARD_ATTEND = 0, 1, 2, 3, 4


class ShardLayout(ctypes.Structure):
    """spava_shard_layout (include/spava.h): byte offsets of the sharded prefill's
    exchange buffers in its workspace."""
    _fields_ = [("workspace_bytes", ctypes.c_uint64),
                ("pass_k_offset", ctypes.c_uint64), ("pass_v_offset", ctypes.c_uint64),
                ("pass_bytes_per_rank", ctypes.c_uint64),
                ("text_o_offset", ctypes.c_uint64), ("text_o_bytes_per_rank", ctypes.c_uint64),
                ("text_lse_offset", ctypes.c_uint64), ("text_lse_bytes_per_rank", ctypes.c_uint64),
                ("scores_offset", ctypes.c_uint64), ("idx_offset", ctypes.c_uint64),
                ("pass_slots", c_int32), ("text_slots", c_int32)]


# name -> (restype, argtypes); the names and order follow include/spava.h.
SIGNATURES = {
    "spava_plan_create": (c_int32, [ctypes.POINTER(c_void_p), c_int32, c_int32, c_int32,
                                    ctypes.POINTER(c_int32), c_int32, c_int32, c_int32,
                                    c_int32, c_int32, c_int32, ctypes.c_float]),
    "spava_plan_destroy": (c_int32, [c_void_p]),
    "spava_workspace_bytes": (c_size_t, [c_void_p]),
    "spava_plan_offsets": (c_int32, [c_void_p, ctypes.POINTER(c_int32)]),
    "spava_score_select": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     ctypes.c_uint32, c_void_p, c_void_p]),
    "spava_gather_passing": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p]),
    "spava_attn_prefill": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "spava_attn_prefill_noalloc": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                             c_void_p, c_void_p]),
    "spava_attn_prefill_two_stage": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                               c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "spava_two_stage_workspace_bytes": (c_size_t, [c_void_p]),
    "spava_dense_causal": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p]),
    "spava_shard_owners": (c_int32, [c_int32, c_int32, c_int32, ctypes.POINTER(c_int32)]),
    "spava_shard_owners_by_cost": (c_int32, [c_int32, c_int32, ctypes.POINTER(ctypes.c_int64),
                                             ctypes.POINTER(c_int32)]),
    "spava_plan_shard_owners": (c_int32, [c_void_p, c_int32, c_int32, ctypes.POINTER(c_int32)]),
    "spava_plan_set_shard": (c_int32, [c_void_p, c_int32, c_int32, ctypes.POINTER(c_int32)]),
    "spava_shard_query": (c_int32, [c_void_p, ctypes.POINTER(ShardLayout)]),
    "spava_shard_stage": (c_int32, [c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_void_p]),
    "spava_check_device_error": (c_int32, [c_void_p, c_void_p, c_void_p]),
    "spava_plan_set_debug": (c_int32, [c_void_p, ctypes.c_uint64, c_int32]),
    "spava_plan_set_score_reduce": (c_int32, [c_void_p, c_int32]),
    "spava_plan_set_score_kind": (c_int32, [c_void_p, c_int32]),
    "spava_plan_set_fused_select": (c_int32, [c_void_p, c_int32]),
    "spava_status_string": (ctypes.c_char_p, [c_int32]),
    "spava_last_error": (ctypes.c_char_p, []),
    "spava_last_launch_count": (c_int32, []),
    "spava_profile_begin": (c_int32, [c_void_p, c_int32]),
    "spava_profile_read": (c_int32, [c_void_p, ctypes.POINTER(c_int32), ctypes.POINTER(ctypes.c_float),
                                     c_int32]),
    "spava_profile_end": (c_int32, [c_void_p]),
    "spava_kernel_name": (ctypes.c_char_p, [c_int32]),
    "spava_layer_workspace_bytes": (c_size_t, [c_int32]),
    "spava_qkv_projection": (c_int32, [c_void_p, c_int32, c_int32, c_void_p, c_int32, c_int32, c_int32,
                                       ctypes.c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "spava_out_projection": (c_int32, [c_void_p, c_int32, c_int32, c_void_p, c_int32, c_void_p, c_void_p,
                                       c_void_p]),
    "spava_layer_check_error": (c_int32, [c_void_p, c_void_p]),
}

_LIB = None


class SpavaError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {_status_name(status)}: {detail}")


def _status_name(s: int) -> str:
    return {0: "SPAVA_OK", 1: "SPAVA_ERR_INVALID_ARG", 2: "SPAVA_ERR_UNSUPPORTED",
            3: "SPAVA_ERR_CUDA", 4: "SPAVA_ERR_TIMEOUT", 5: "SPAVA_ERR_DEVICE_CHECK"}.get(s, f"status {s}")


def load(build_if_missing: bool = True):
    """Load libspava.so (building it first if it is missing or older than its sources).
    SPAVA_LIB_PATH, if set, names another build of the same library to load instead."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = os.environ.get("SPAVA_LIB_PATH") or _build.LIB_PATH
    if path == _build.LIB_PATH and build_if_missing and _build.is_stale():
        _build.build()
    if not os.path.exists(path):
        raise ImportError(f"libspava.so is not built ({path}); run "
                          "python -m sequence_approximate_attention_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def launches_of_last_call() -> int:
    """spava_last_launch_count, or 0 where the library is not loaded (stand-in plans)."""
    return int(_LIB.spava_last_launch_count()) if _LIB is not None else 0


def check(status: int, where: str) -> None:
    if status != SPAVA_OK:
        detail = load().spava_last_error().decode(errors="replace")
        raise SpavaError(status, where, detail)
