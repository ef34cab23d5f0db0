"""ctypes declarations of the libcsa C ABI (include/csa.h)."""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
# CSA_LIBRARY selects another build of the same ABI (e.g. libcsa_checked.so,
# whose kernels bounds-check their gathers); by default the library next to
# this file.
LIB_PATH = os.environ.get("CSA_LIBRARY") or os.path.join(_HERE, "libcsa.so")

c_i32, c_i64, c_f32, c_sz, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

CSA_OK, CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_WORKSPACE, CSA_ERR_CUDA, CSA_ERR_DEVICE_TIMEOUT = 0, 1, 2, 3, 4, 5
CSA_KV_BF16, CSA_KV_SPLIT_FP8 = 0, 1

# every symbol include/csa.h declares, with (restype, argtypes)
SIGNATURES = {
    "csa_version": (ctypes.c_char_p, []),
    "csa_status_string": (ctypes.c_char_p, [c_i32]),
    "csa_last_error": (ctypes.c_char_p, []),
    "csa_launch_count": (ctypes.c_uint64, []),
    "csa_profile_next_call": (c_i32, [c_vp, c_vp]),
    "csa_check_device_error": (c_i32, [c_vp]),
    "csa_debug_expire_wait": (c_i32, [c_vp]),
    "csa_compress": (c_i32, [c_vp, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "hca_compress": (c_i32, [c_vp, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "csa_compress_append": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp,
                                    c_vp, c_i64, c_vp]),
    "hca_compress_append": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp,
                                    c_vp, c_i64, c_vp]),
    "csa_compress_packed": (c_i32, [c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "hca_compress_packed": (c_i32, [c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "csa_indexer_topk_workspace_size": (c_sz, [c_i64, c_i64, c_i64, c_i32]),
    "csa_indexer_topk_coded_workspace_size": (c_sz, [c_i64, c_i64, c_i64, c_i32]),
    "csa_indexer_topk": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp, c_sz,
                                 c_vp]),
    "csa_indexer_topk_e4m3": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp,
                                      c_sz, c_vp]),
    "csa_indexer_topk_with_scores": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp,
                                             c_vp, c_sz, c_vp]),
    "csa_cp_topk_merge": (c_i32, [c_vp, c_vp, c_i64, c_i32, c_i32, c_vp, c_vp]),
    "csa_cp_attn_merge": (c_i32, [c_vp, c_vp, c_i32, c_i64, c_i32, c_vp, c_vp, c_vp]),
    "csa_indexer_topk_e2m1": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp,
                                      c_sz, c_vp]),
    "csa_indexer_topk_noalloc": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i32, c_i32, c_vp, c_vp]),
    "csa_sparse_mqa_workspace_size": (c_sz, [c_i64, c_i64, c_i32, c_i32, c_i32]),
    "csa_sparse_mqa": (c_i32, [c_vp, c_i64, c_i64, c_i32, c_i64, c_vp, c_i32, c_vp, c_i32, c_vp, c_f32, c_vp, c_vp,
                               c_vp, c_sz, c_vp]),
    "hca_dense_mqa_workspace_size": (c_sz, [c_i64, c_i64, c_i32, c_i64, c_i32]),
    "hca_dense_mqa": (c_i32, [c_vp, c_i64, c_i64, c_i32, c_i64, c_vp, c_i32, c_vp, c_f32, c_vp, c_vp, c_vp, c_sz,
                              c_vp]),
    "hca_dense_mqa_budget": (c_i32, [c_vp, c_i64, c_i64, c_i32, c_i64, c_vp, c_i32, c_vp, c_f32, c_vp, c_vp, c_i32,
                                     c_vp, c_sz, c_vp]),
    "csa_grouped_out_proj": (c_i32, [c_vp, c_i64, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp]),
    "csa_indexer_topk_packed_workspace_size": (c_sz, [c_vp, c_i32, c_i32]),
    "csa_indexer_topk_packed": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "csa_sparse_mqa_packed": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_i32, c_vp, c_i32, c_vp, c_f32, c_vp, c_vp, c_vp,
                                      c_sz, c_vp]),
    "hca_dense_mqa_packed": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_i32, c_vp, c_f32, c_vp, c_vp, c_vp, c_sz, c_vp]),
}


class KVCacheDesc(ctypes.Structure):
    """csa_kv_cache."""
    _fields_ = [("layout", c_i32), ("reserved", c_i32), ("n_entries", c_i64), ("k", c_vp), ("v", c_vp),
                ("nope", c_vp), ("rope", c_vp), ("scale", c_vp)]


class PackedDesc(ctypes.Structure):
    """csa_packed."""
    _fields_ = [("cu_tokens", c_vp), ("cu_entries", c_vp), ("n_seqs", c_i32), ("max_tokens", c_i32),
                ("total_tokens", c_i64), ("total_entries", c_i64)]


class WindowDesc(ctypes.Structure):
    """csa_window."""
    _fields_ = [("k", c_vp), ("v", c_vp), ("pos0", c_i64), ("rows", c_i64), ("len", c_i32), ("reserved", c_i32)]


_lib = None
_lock = threading.Lock()


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libcsa.so (once).  Raises if it has not been built: there is no fallback."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"libcsa.so not found at {path}; build it with "
                                   "`python -m long_context_sparse_10_b200.build` (nvcc, sm_100a)")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib
