"""ctypes loader for libbsa.so (the C ABI of include/bsa.h).

There is no fallback: if the in-tree library is missing or fails to load,
every call raises.  Build it with ``python -m block_sparse_attention_logits_b200.build``.
"""

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")

EXPORTS = (
    "bsa_strerror", "bsa_version", "bsa_score_blocks", "bsa_score_blocks_gather", "bsa_score_blocks_restricted",
    "bsa_block_drift",
    "bsa_select_topp_mask", "bsa_select_topp_mask_restricted",
    "bsa_interval_runs", "bsa_interval_width_for_merge", "bsa_kept_to_intervals", "bsa_intervals_to_kept",
    "bsa_tail_workspace_bytes", "bsa_tail_stats", "bsa_coarse_tail", "bsa_tail_refinement", "bsa_tail_reconstruct",
    "bsa_complement_lists", "bsa_quantize_fp8", "bsa_sparse_attn_fwd_fp8",
    "bsa_wait_selftest",
    "bsa_reorder_workspace_bytes", "bsa_reorder_tokens", "bsa_reorder_tokens_noalloc", "bsa_permute_tokens",
    "bsa_sparse_attn_fwd", "bsa_sparse_attn_fwd_scatter", "bsa_sparse_attn_fwd_gather", "bsa_sparse_attn_fwd_intervals", "bsa_sparse_attn_refresh", "bsa_refresh_refinement", "bsa_apply_correction",
)

BSA_OK, BSA_EINVAL, BSA_ESHAPE, BSA_ENODEV, BSA_ECUDA, BSA_EWORKSPACE = range(6)
BSA_DEV_TIMEOUT = 1
BSA_DEV_BAD_INDEX = 2
BSA_DEV_SCHED_CONFLICT = 4


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int),
                ("D", ctypes.c_int), ("blk", ctypes.c_int)]


class BsaError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t


def load():
    """Load libbsa.so once and declare every signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libbsa.so not found at {LIB_PATH}; build it with "
                           "`python -m block_sparse_attention_logits_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "bsa_strerror": (ctypes.c_char_p, [_I]),
        "bsa_version": (_I, []),
        "bsa_score_blocks": (_I, [Shape, _P, _P, _P, _P, _P, _P]),
        "bsa_score_blocks_gather": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_score_blocks_restricted": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_block_drift": (_I, [Shape, _P, _P, _P, _P, _P, _P]),
        "bsa_select_topp_mask": (_I, [Shape, _P, ctypes.POINTER(ctypes.c_float), _P, _P, _P, _P]),
        "bsa_select_topp_mask_restricted": (_I, [Shape, _P, ctypes.POINTER(ctypes.c_float), _P, _P, _P, _P, _P]),
        "bsa_interval_runs": (_I, [Shape, _P, _P, _P, _P, _P, _P]),
        "bsa_interval_width_for_merge": (_I, [ctypes.POINTER(ctypes.c_int32), _I, ctypes.c_double,
                                              ctypes.POINTER(ctypes.c_int)]),
        "bsa_kept_to_intervals": (_I, [Shape, _P, _P, _I, _P, _P, _P, _P, _P]),
        "bsa_intervals_to_kept": (_I, [Shape, _P, _P, _I, _P, _P, _P, _P, _P]),
        "bsa_wait_selftest": (_I, [_P, ctypes.c_ulonglong, _P]),
        "bsa_tail_workspace_bytes": (_SZ, [Shape]),
        "bsa_tail_stats": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
        "bsa_coarse_tail": (_I, [Shape, _P, _P, _P, _SZ, _P, _P, _P, _P]),
        "bsa_tail_refinement": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_tail_reconstruct": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_complement_lists": (_I, [Shape, _P, _P, _P, _P]),
        "bsa_quantize_fp8": (_I, [Shape, _P, _P, _P, _P]),
        "bsa_sparse_attn_fwd_fp8": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_reorder_workspace_bytes": (_SZ, [_I, _I, _I]),
        "bsa_reorder_tokens": (_I, [_I, _I, _I, _P, _P, _P, _SZ, _P]),
        "bsa_reorder_tokens_noalloc": (_I, [_I, _I, _I, _P, _P, _P]),
        "bsa_permute_tokens": (_I, [Shape, _P, _P, _P, _I, _P]),
        "bsa_sparse_attn_fwd": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_sparse_attn_fwd_scatter": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_sparse_attn_fwd_gather": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_sparse_attn_fwd_intervals": (_I, [Shape, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P]),
        "bsa_sparse_attn_refresh": (_I, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_refresh_refinement": (_I, [Shape, _P, _P, _P, _P]),
        "bsa_apply_correction": (_I, [Shape, _P, _P, _P, _P, _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def check(fn, code):
    if code != BSA_OK:
        msg = load().bsa_strerror(code).decode()
        raise BsaError(fn, code, msg)
