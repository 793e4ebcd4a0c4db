"""ctypes declarations of libcalibatt.so (the C ABI in include/calibatt.h)."""

from __future__ import annotations

import ctypes
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_int16, c_int32, c_int64, c_size_t, c_uint64, c_void_p
from pathlib import Path

LIB_PATH = Path(__file__).resolve().parent / "libcalibatt.so"

OK = 0
E_INVALID = -1
E_UNSUPPORTED = -2
E_CUDA = -3
E_TIMEOUT = -4
E_CORRUPT = -5
E_WORKSPACE = -6

BF16 = 0
FP32 = 1
SELECT_TOPK = 0
SELECT_ENERGY = 1
DEDUP_NONE = 0
DEDUP_HASH = 1
DEDUP_HASH_WEAK = 2

STATUS_NAMES = {
    OK: "CALIBATT_OK", E_INVALID: "CALIBATT_E_INVALID", E_UNSUPPORTED: "CALIBATT_E_UNSUPPORTED",
    E_CUDA: "CALIBATT_E_CUDA", E_TIMEOUT: "CALIBATT_E_TIMEOUT", E_CORRUPT: "CALIBATT_E_CORRUPT",
    E_WORKSPACE: "CALIBATT_E_WORKSPACE",
}

# Every function the header declares, with its ctypes signature.
EXPORTS = {
    "calibatt_last_error": (c_char_p, []),
    "calibatt_version": (c_int, []),
    "calibatt_launch_count": (c_uint64, []),
    "calibatt_set_spin_limit_ns": (None, [c_uint64]),
    "calibatt_get_spin_limit_ns": (c_uint64, []),
    "calibatt_sparse_attn_fwd": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                         c_int, c_int, c_int, c_float, c_void_p, c_int, c_void_p, c_void_p]),
    "calibatt_sparse_attn_fwd_streamed": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                  c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                                  c_int, c_int, c_int, c_float, c_void_p, c_int, c_int, c_void_p,
                                                  c_void_p]),
    "calibatt_timestep_clusters_workspace_size": (c_int, [c_int, c_int, c_int, POINTER(c_size_t)]),
    "calibatt_timestep_clusters": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_double, c_void_p,
                                           POINTER(c_int32), c_void_p, c_size_t, c_void_p]),
    "calibatt_share_masks": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p, c_int, c_void_p,
                                     c_void_p]),
    "calibatt_interval_counts": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p]),
    "calibatt_merge_intervals": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "calibatt_sparse_attn_fwd_qk": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                            c_int, c_int, c_int, c_int, c_int, c_float, c_void_p, c_int, c_void_p,
                                            c_void_p]),
    "calibatt_gather_rows": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p]),
    "calibatt_block_energy": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                                      c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "calibatt_block_energy_noalloc": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                              c_float, c_void_p, c_void_p, c_void_p]),
    "calibatt_calibrate_workspace_size": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, POINTER(c_size_t)]),
    "calibatt_select_vote": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_double, c_void_p, c_void_p, c_void_p]),
    "calibatt_finalize_mask": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p]),
    "calibatt_calibrate": (c_int, [POINTER(c_void_p), POINTER(c_void_p), c_int, c_int, c_int, c_int, c_int, c_int,
                                   c_int, c_int, c_float, c_int, c_double, c_void_p, c_void_p, c_int, c_void_p,
                                   c_void_p, c_size_t, c_void_p, c_void_p]),
    "calibatt_compile_workspace_size": (c_int, [c_int, c_int, c_int, POINTER(c_size_t)]),
    "calibatt_compile_size": (c_int, [c_void_p, c_int, c_int, c_int, c_int, POINTER(c_int64), POINTER(c_int32),
                                      POINTER(c_int32), c_void_p, c_size_t, c_void_p]),
    "calibatt_compile": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_size_t,
                                 c_void_p]),
    "calibatt_selftest_wait_timeout": (c_int, [c_uint64, c_void_p, c_void_p]),
    "calibatt_anchor_rows": (c_int, [c_int, c_int, c_void_p, c_void_p]),
    "calibatt_anchor_plan_size": (c_int, [c_int, c_int, c_int, c_int, POINTER(c_int), POINTER(c_int)]),
    "calibatt_anchor_plan": (c_int, [c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "calibatt_skiplist_sizes_workspace_size": (c_int, [c_int, c_int, c_int, POINTER(c_size_t)]),
    "calibatt_skiplist_sizes": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_int, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "calibatt_blocklist_bytes": (c_int, [c_int, c_int, c_int64, c_int32, c_int32, POINTER(c_int64),
                                         POINTER(c_int64)]),
    "calibatt_min_votes": (c_int, [c_double, c_int, POINTER(c_int32)]),
    "calibatt_topk_count": (c_int, [c_double, c_int, POINTER(c_int32)]),
    "calibatt_blocklist_kept": (c_int, [c_void_p, c_int, c_int, POINTER(c_int64), c_void_p, c_size_t, c_void_p]),
    "calibatt_spatial_similarity_workspace_size": (c_int, [c_int, c_int, POINTER(c_size_t)]),
    "calibatt_spatial_similarity": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                            c_int, c_float, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "calibatt_repetition_flags": (c_int, [c_void_p, c_int, c_int, c_float, c_void_p, c_void_p, c_void_p]),
}


class Blocklist(ctypes.Structure):
    """Mirror of ``calibatt_blocklist``."""

    _fields_ = [
        ("n_maps", c_int32), ("n_q_blocks", c_int32), ("n_k_blocks", c_int32),
        ("block_q", c_int32), ("block_k", c_int32),
        ("row_base", c_void_p), ("row_pat", c_void_p), ("pat_ptr", c_void_p), ("pat_off", c_void_p),
        ("csr_row_ptr", c_void_p), ("csr_col", c_void_p),
        ("n_pat", c_int32), ("nnz_pat", c_int32), ("nnz", c_int64),
    ]


_lib = None


def load(path: Path | None = None):
    """Loads libcalibatt.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    p = Path(path) if path else LIB_PATH
    if not p.exists():
        raise RuntimeError(f"{p} is missing: build the CUDA library first "
                           "(python -m block_sparse_attention_cross_b200.build)")
    lib = ctypes.CDLL(str(p))
    for name, (res, args) in EXPORTS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class CalibattError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def check(code):
    if code != OK:
        raise CalibattError(code, load().calibatt_last_error().decode(errors="replace"))
    return code
