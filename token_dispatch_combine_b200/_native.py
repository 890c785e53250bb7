"""ctypes binding of libmoe_b200.so (declared in include/moe_b200.h).

Argument marshalling only: every step of the round trip runs in the CUDA
library.  There is no fallback -- if the library cannot be built or loaded,
importing the package raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE, MOE_ERR_TIMEOUT = range(6)
MOE_F32, MOE_BF16 = 0, 1
FFN_TILING_AUTO, FFN_TILING_SINGLE, FFN_TILING_PAIR = 0, 1, 2
FFN_GATE_UP, FFN_DOWN = 0, 1

# error-word bits reported by moe_get_error
ERR_BAD_ID, ERR_BAD_OFFSETS, ERR_BAD_ROW, ERR_TIMEOUT = 1, 2, 4, 8

EXPORTS = (
    "moe_abi_version", "moe_status_string", "moe_last_error_message", "moe_route", "moe_dispatch_workspace_bytes",
    "moe_dispatch", "moe_expert_ffn", "moe_ffn_gate_up", "moe_ffn_down", "moe_combine", "moe_get_error", "moe_selftest_wait_timeout",
    "moe_dispatch_noalloc", "moe_set_ffn_tiling", "moe_get_ffn_tiling", "moe_ffn_tiling_for", "moe_router_topk",
    "moe_ffn_gate_up_gather", "moe_expert_ffn_gather", "moe_eplb_plan", "moe_eplb_remap", "moe_eplb_replicate",
    "moe_selftest_dispatch_timeout", "moe_combine_rank_partials", "moe_reduce_rank_partials",
    "moe_ep_plan_workspace_bytes", "moe_ep_plan", "moe_ep_plan_host", "moe_ep_exchange_offsets", "moe_ep_pack",
    "moe_enable_peer_access", "moe_ep_recv_index", "moe_route_count", "moe_dispatch_counted", "moe_ffn_down_combine", "moe_combine_finalize",
    "moe_route_count_workspace_bytes",
)

_lock = threading.Lock()
_lib = None


class MoeError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        self.status = status
        super().__init__(f"{fn} failed: status {status}: {msg}")


def _configure(lib):
    vp, i32, sz, u32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.POINTER(ctypes.c_uint32)
    sigs = {
        "moe_abi_version": ([], i32),
        "moe_status_string": ([i32], ctypes.c_char_p),
        "moe_last_error_message": ([], ctypes.c_char_p),
        "moe_route": ([vp, i32, i32, i32, vp, vp, vp], i32),
        "moe_dispatch_workspace_bytes": ([i32, i32, i32, i32], sz),
        "moe_dispatch": ([vp, i32, i32, i32, vp, i32, i32, i32] + [vp] * 8 + [vp, sz, vp], i32),
        "moe_expert_ffn": ([vp, i32, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp], i32),
        "moe_ffn_gate_up": ([vp, i32, vp, vp, vp, i32, i32, i32, i32, vp, vp], i32),
        "moe_ffn_down": ([vp, i32, vp, vp, i32, i32, i32, i32, vp, vp], i32),
        "moe_combine": ([vp, i32, vp, vp, i32, i32, i32, vp, vp], i32),
        "moe_get_error": ([vp, u32p], i32),
        "moe_selftest_wait_timeout": ([ctypes.c_uint, vp], i32),
        "moe_dispatch_noalloc": ([vp, i32, i32, i32, vp, i32, i32, i32] + [vp] * 8 + [vp], i32),
        "moe_router_topk": ([vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp], i32),
        "moe_set_ffn_tiling": ([i32], i32),
        "moe_get_ffn_tiling": ([], i32),
        "moe_ffn_tiling_for": ([i32, i32, i32], i32),
        "moe_ffn_gate_up_gather": ([vp, i32, i32, vp, i32, vp, vp, vp, i32, i32, i32, i32, vp, vp], i32),
        "moe_expert_ffn_gather": ([vp, i32, i32, vp, i32, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp], i32),
        "moe_eplb_plan": ([vp, i32, i32, i32, vp, vp, vp], i32),
        "moe_eplb_remap": ([vp, i32, i32, i32, vp, vp, i32, vp, vp], i32),
        "moe_eplb_replicate": ([vp, sz, i32, vp, i32, vp, vp], i32),
        "moe_combine_rank_partials": ([vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp], i32),
        "moe_reduce_rank_partials": ([vp, i32, i32, i32, i32, vp, vp], i32),
        "moe_ep_plan_workspace_bytes": ([i32, i32], sz),
        "moe_ep_plan": ([vp, vp, i32, i32, i32, i32] + [vp] * 7 + [vp, sz, vp], i32),
        "moe_ep_plan_host": ([vp, vp, i32, i32, i32, i32] + [vp] * 7, i32),
        "moe_ep_exchange_offsets": ([vp, i32, i32, vp, vp, vp], i32),
        "moe_enable_peer_access": ([i32], i32),
        "moe_ep_pack": ([vp, i32, i32, i32, i32, i32] + [vp] * 5 + [vp] * 4 + [vp], i32),
        "moe_ep_recv_index": ([vp, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp], i32),
        "moe_route_count_workspace_bytes": ([i32, i32, i32, i32], sz),
        "moe_route_count": ([vp, i32, i32, i32, i32, vp, vp, vp, sz, vp], i32),
        "moe_dispatch_counted": ([vp, i32, i32, i32, vp, i32, i32, i32] + [vp] * 8 + [vp, sz, vp], i32),
        "moe_ffn_down_combine": ([vp, i32, vp, vp, i32, i32, i32, i32, vp, vp, i32, i32, vp, vp], i32),
        "moe_combine_finalize": ([vp, i32, i32, i32, vp, vp], i32),
        "moe_selftest_dispatch_timeout": ([vp, i32, i32, i32, vp, i32, i32, i32] + [vp] * 8 + [vp, sz, ctypes.c_uint, vp],
                                          i32),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


def lib():
    """The loaded library: the file named by MOE_B200_LIBRARY if that is set
    (a prebuilt copy of this library), else the in-tree build (built first if
    missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            path = os.environ.get("MOE_B200_LIBRARY") or _build.build()
            _lib = _configure(ctypes.CDLL(path))
    return _lib


def check(status: int, fn: str):
    if status != MOE_OK:
        msg = lib().moe_last_error_message().decode(errors="replace")
        raise MoeError(status, fn, msg)


def library_path() -> str:
    return os.environ.get("MOE_B200_LIBRARY") or _build.LIB_PATH
