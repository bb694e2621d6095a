"""ctypes declarations of libiskv's C ABI (``include/iskv.h``). Marshalling only."""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libiskv.so")

c_i32, c_i64, c_sz, c_vp, c_f32, c_f64 = (ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                          ctypes.c_void_p, ctypes.c_float, ctypes.c_double)

ISKV_F32, ISKV_BF16, ISKV_F16 = 0, 1, 2
META_K, META_N, META_FOLDS, META_STATUS = 0, 1, 2, 3
STATUS = {0: "OK", 1: "ERR_ARG", 2: "ERR_SHAPE", 3: "ERR_CUDA", 4: "ERR_CAPACITY",
          5: "ERR_NONFINITE", 6: "ERR_NOT_CONVERGED", 7: "ERR_TIMEOUT", 8: "ERR_WORKSPACE"}


class IskvLowRank(ctypes.Structure):
    """Mirror of ``iskv_lowrank``."""

    _fields_ = [("d", c_i32), ("r_max", c_i32), ("n_cap", c_i64), ("storage", c_i32),
                ("reserved", c_i32), ("U", c_vp), ("sigma", c_vp), ("B", c_vp), ("pos", c_vp),
                ("meta", c_vp)]


class IskvExactTable(ctypes.Structure):
    """Mirror of ``iskv_exact_table``."""

    _fields_ = [("d", c_i32), ("window", c_i32), ("block", c_i32), ("reorth_rows", c_i32),
                ("dtype", c_i32), ("refit_rows", c_i32), ("cap_e", c_i64), ("rows", c_vp),
                ("pos", c_vp), ("live_host", ctypes.POINTER(c_i32)), ("live_cap", c_i64),
                ("n_prot", c_i64), ("n_live", c_i64), ("last", c_i64), ("fold_rows", c_i64),
                ("hist_rows", c_i64), ("refit_done", c_i64)]


# name -> (restype, argtypes)
SIGNATURES = {
    "iskv_abi_version": (c_i32, []),
    "iskv_status_string": (ctypes.c_char_p, [c_i32]),
    "iskv_last_error": (ctypes.c_char_p, []),
    "iskv_fold_workspace_size": (c_sz, [c_i32, c_i32, c_i32, c_i32]),
    "iskv_fold_block": (c_i32, [ctypes.POINTER(IskvLowRank), c_vp, c_i32, c_i32, c_vp, c_f32, c_vp,
                                c_sz, c_vp]),
    "iskv_fold_block_batched": (c_i32, [ctypes.POINTER(IskvLowRank), c_i32,
                                        ctypes.POINTER(c_vp), c_i32, c_i32, ctypes.POINTER(c_vp),
                                        c_f32, c_vp, c_sz, c_vp]),
    "iskv_fold_block_batched_after": (c_i32, [ctypes.POINTER(IskvLowRank), c_i32,
                                              ctypes.POINTER(c_vp), c_i32, c_i32,
                                              ctypes.POINTER(c_vp), c_f32, c_vp, c_sz, c_vp,
                                              c_vp]),
    "iskv_reorth_workspace_size": (c_sz, [c_i32, c_i32, c_i32, c_i64]),
    "iskv_reorth": (c_i32, [ctypes.POINTER(IskvLowRank), c_i32, c_vp, c_sz, c_vp]),
    "iskv_reconstruct_workspace_size": (c_sz, [c_i32, c_i32, c_i32]),
    "iskv_reconstruct": (c_i32, [ctypes.POINTER(IskvLowRank), c_vp, c_i32, c_vp, c_i64, c_i64,
                                 c_i32, c_i32, c_i32, c_f64, c_vp, c_i32, c_vp, c_sz, c_vp]),
    "iskv_reconstruct_batched": (c_i32, [ctypes.POINTER(IskvLowRank), c_i32, ctypes.POINTER(c_vp),
                                         c_i32, ctypes.POINTER(c_vp), ctypes.POINTER(c_i64),
                                         ctypes.POINTER(c_i64), c_i32, c_i32,
                                         ctypes.POINTER(c_i32), c_f64, ctypes.POINTER(c_vp), c_i32,
                                         c_vp, c_sz, c_vp]),
    "iskv_diagnostics_workspace_size": (c_sz, [c_i32, c_i32, c_i32, c_i64]),
    "iskv_diagnostics": (c_i32, [ctypes.POINTER(IskvLowRank), c_i32, ctypes.POINTER(c_i64), c_i32,
                                 c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "iskv_attention_workspace_size": (c_sz, [c_i32, c_i32, c_i32, c_i64, c_i64, c_i32]),
    "iskv_decode_attention": (c_i32, [ctypes.POINTER(IskvLowRank), ctypes.POINTER(IskvLowRank),
                                      c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_i32, c_i64, c_i32,
                                      c_i32, c_i32, c_f64, c_f32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "iskv_decode_attention_batched": (c_i32, [ctypes.POINTER(IskvLowRank),
                                              ctypes.POINTER(IskvLowRank), c_i32,
                                              ctypes.POINTER(c_vp), ctypes.POINTER(c_vp),
                                              ctypes.POINTER(c_i64), ctypes.POINTER(c_vp),
                                              ctypes.POINTER(c_vp), ctypes.POINTER(c_i64), c_i32,
                                              ctypes.POINTER(c_i64), c_i32, c_i32, c_i32, c_f64,
                                              c_f32, ctypes.POINTER(c_vp), ctypes.POINTER(c_vp),
                                              c_vp, c_sz, c_vp]),
    "iskv_select_workspace_size": (c_sz, [c_i64, c_i32, c_i32]),
    "iskv_select_prompt_blocks": (c_i32, [c_vp, c_i32, c_i64, c_i32, c_i32, c_i32, c_i32, c_i32,
                                          c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "iskv_select_prompt_blocks_noalloc": (c_i32, [c_vp, c_i32, c_i64, c_i32, c_i32, c_i32, c_i32,
                                                  c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "iskv_cache_prefill_workspace_size": (c_sz, [c_i32]),
    "iskv_cache_prefill": (c_i32, [ctypes.POINTER(IskvExactTable), c_vp, c_i32, c_i64, c_vp, c_i64,
                                   c_i32, c_vp, c_vp, ctypes.POINTER(c_i64), c_vp, c_sz, c_vp]),
    "iskv_cache_step_workspace_size": (c_sz, [c_i32, c_i32, c_i32, c_i32, c_i64, c_i32]),
    "iskv_cache_step": (c_i32, [ctypes.POINTER(ctypes.POINTER(IskvExactTable)),
                                ctypes.POINTER(ctypes.POINTER(IskvLowRank)), c_i32, c_vp, c_i32,
                                c_f32, ctypes.POINTER(c_i32), ctypes.POINTER(c_i32), c_vp, c_sz,
                                c_vp]),
    "iskv_cache_plan": (c_i32, [ctypes.POINTER(ctypes.POINTER(IskvExactTable)), c_i32, c_i32,
                                c_i64, c_i32, ctypes.POINTER(c_i32), ctypes.POINTER(c_i32)]),
    "iskv_reset": (c_i32, [ctypes.POINTER(IskvLowRank), c_vp]),
    "iskv_get_status": (c_i32, [ctypes.POINTER(IskvLowRank), ctypes.POINTER(c_i64),
                                ctypes.POINTER(c_i64), ctypes.POINTER(c_i64),
                                ctypes.POINTER(c_i64)]),
    "iskv_stage_timing": (c_i32, [c_i32]),
    "iskv_stage_count": (c_i32, []),
    "iskv_stage_name": (ctypes.c_char_p, [c_i32]),
    "iskv_stage_read": (c_i32, [ctypes.POINTER(c_f64), ctypes.POINTER(c_i64)]),
    "iskv_stage_reset": (None, []),
    "iskv_launch_count": (c_i64, []),
    "iskv_core_stats": (c_i32, [c_vp, c_i32]),
    "iskv_compress_prompt_workspace_size": (c_sz, [c_i32, c_i32, c_i32, c_i32]),
    "iskv_compress_prompt": (c_i32, [ctypes.POINTER(IskvLowRank), c_i32, ctypes.POINTER(c_vp),
                                     ctypes.POINTER(c_vp), ctypes.POINTER(c_i64), c_i32, c_i32,
                                     c_f32, c_vp, c_sz, c_vp]),
    "iskv_selftest_wait_timeout": (c_i32, [c_vp, c_i64, c_vp]),
}

_lib = None


def load(path: str | None = None):
    """Load libiskv.so (once). Raises if it has not been built: there is no fallback path."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libiskv.so not found at {p}; build it with "
                           "`python -m kv_cache_online_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


class IskvError(RuntimeError):
    """A non-OK status returned by a libiskv entry point."""

    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")
        self.status = status


def check(status: int, where: str):
    if status != 0:
        detail = load().iskv_last_error().decode(errors="replace")
        raise IskvError(status, where, detail)
