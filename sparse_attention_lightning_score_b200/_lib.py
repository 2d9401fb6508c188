"""ctypes loader for ``libli.so`` (the C ABI declared in ``include/li.h``).

The library must have been built (``python -m sparse_attention_lightning_score_b200.build``);
there is no fallback: loading fails loudly when the shared object is missing.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libli.so")

LI_OK, LI_ERR_INVALID_ARG, LI_ERR_UNSUPPORTED, LI_ERR_CUDA, LI_ERR_TIMEOUT, LI_ERR_BOUNDS = range(6)
LI_DTYPE_F32, LI_DTYPE_BF16, LI_DTYPE_E4M3 = 0, 1, 2
LI_TOPK_MAX_LEN = 262144
LI_HS_NOALLOC_MAX_SCRATCH_FLOATS = 1048576
LI_OP_SCORE, LI_OP_TOPK, LI_OP_HS, LI_OP_DECODE_SELECT = range(4)

vp = ctypes.c_void_p
i32 = ctypes.c_int
i64 = ctypes.c_int64
sz = ctypes.c_size_t


class ScoreDesc(ctypes.Structure):
    _fields_ = [("rows", i32), ("heads", i32), ("dim", i32), ("max_len", i32), ("causal", i32),
                ("causal_offset", i32), ("q_dtype", i32), ("k_dtype", i32), ("tokens_per_request", i32)]


# name -> (restype, argtypes); every symbol declared in include/li.h
SIGNATURES = {
    "li_status_string": (ctypes.c_char_p, [i32]),
    "li_get_last_error": (i32, []),
    "li_quantize_query": (i32, [vp, vp, i32, i32, i32, vp, vp, vp, vp]),
    "li_index_score": (i32, [vp, vp, vp, vp, i64, vp, vp, i64, ctypes.POINTER(ScoreDesc), vp, sz, vp]),
    "li_index_score_workspace": (sz, [ctypes.POINTER(ScoreDesc)]),
    "li_workspace_size": (sz, [i32, i32, i32, i32]),
    "li_topk": (i32, [vp, i64, vp, i32, i32, i32, i32, i32, vp, vp, vp]),
    "li_decode_select": (i32, [vp, vp, vp, vp, i64, vp, vp, i64, ctypes.POINTER(ScoreDesc), i32, vp, vp, vp, sz,
                               vp]),
    "li_decode_select_workspace": (sz, [ctypes.POINTER(ScoreDesc)]),
    "li_decode_select_score": (i32, [vp, vp, vp, vp, i64, vp, vp, i64, ctypes.POINTER(ScoreDesc), vp, sz, vp]),
    "li_decode_select_finish": (i32, [vp, i64, vp, ctypes.POINTER(ScoreDesc), i32, vp, vp, vp, sz, vp]),
    "li_decode_score_hist": (i32, [vp, vp, vp, vp, i64, vp, vp, i64, ctypes.POINTER(ScoreDesc), vp, vp]),
    "li_topk_hist": (i32, [vp, i64, vp, i32, i32, i32, vp, vp, vp, i32, vp]),
    "li_absorb_query": (i32, [vp, vp, vp, i32, i32, i32, i32, vp]),
    "li_latent_score": (i32, [vp, vp, vp, i64, vp, vp, i64, i32, i32, i32, i32, vp]),
    "li_latent_score_hist": (i32, [vp, vp, vp, i64, vp, vp, i64, i32, i32, i32, i32, vp, vp]),
    "li_absorb_query_layers": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, vp]),
    "li_host_device_pointer": (i32, [vp, ctypes.POINTER(ctypes.c_void_p)]),
    "li_copy_from_host": (i32, [vp, vp, sz, vp]),
    "li_merge_shards": (i32, [vp, vp, i32, i32, i32, i64, i32, vp, vp, vp, sz, vp]),
    "li_merge_shards_workspace": (sz, [i32, i32, i32]),
    "li_latent_score_fp8": (i32, [vp, vp, vp, vp, i64, vp, vp, i64, i32, i32, i32, i32, vp, vp]),
    "li_hs_refine": (i32, [vp, i64, i64, vp, i32, i32, vp, vp, i32, i32, i32, i32, vp, vp, sz, vp]),
    "li_hs_refine_workspace": (sz, [i32, i32, i32]),
    "li_hs_refine_noalloc": (i32, [vp, i64, i64, vp, i32, i32, vp, vp, i32, i32, i32, i32, vp, vp]),
    "li_hs_refine_fp8": (i32, [vp, vp, i64, i64, vp, i32, i32, vp, vp, i32, i32, i32, i32, vp, vp, sz, vp]),
    "li_sparse_attention": (i32, [vp, vp, i64, i64, vp, i32, i32, i32, ctypes.c_float, vp, vp, sz, vp]),
    "li_sparse_attention_workspace": (sz, [i32, i32, i32]),
    "li_graph_instantiate": (i32, [vp, i32, ctypes.POINTER(ctypes.c_void_p)]),
    "li_graph_launch": (i32, [vp, vp]),
    "li_graph_destroy": (i32, [vp]),
    "li_selftest_wait_timeout": (i32, [ctypes.c_uint64, vp]),
}

_lib = None


class LiError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)}")


def load() -> ctypes.CDLL:
    """Load libli.so once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libli.so not found at {LIB_PATH}; build it with "
                              "`python -m sparse_attention_lightning_score_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().li_status_string(int(status)).decode()


def check(fn: str, status: int):
    if status != LI_OK:
        raise LiError(fn, status)
