"""ctypes binding of libspava.so (include/spava.h).  Argument marshalling only.

The library must exist: nothing here falls back to another implementation.
Build it with ``python -m sequence_sparse_attention_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspava.so")

SPAVA_OK = 0
STATUS_NAMES = {0: "SPAVA_OK", 1: "SPAVA_ERR_INVALID_ARG", 2: "SPAVA_ERR_UNSUPPORTED",
                3: "SPAVA_ERR_MISALIGNED", 4: "SPAVA_ERR_WORKSPACE", 5: "SPAVA_ERR_CUDA",
                6: "SPAVA_ERR_TIMEOUT"}

# Every symbol include/spava.h declares.
EXPORTS = ("spava_workspace_size", "spava_packed_len", "spava_score", "spava_topk_select",
           "spava_pack_passing", "spava_attn", "spava_prefill_attention",
           "spava_prefill_attention_host", "spava_device_status", "spava_attended_pairs",
           "spava_status_string", "spava_last_cuda_error", "spava_score_noalloc",
           "spava_selftest_wait_timeout", "spava_plan_chunks", "spava_score_noalloc_status",
           "spava_shard_layout", "spava_shard_sizes", "spava_shard_front", "spava_shard_local_attn",
           "spava_shard_context_attn", "spava_shard_merge")


class SpavaConfig(ctypes.Structure):
    """Mirror of ``spava_config``."""
    _fields_ = [
        ("H", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("n_tokens", ctypes.c_int64),
        ("anchor_len", ctypes.c_int64),
        ("query_len", ctypes.c_int64),
        ("chunk_offsets", ctypes.POINTER(ctypes.c_int64)),
        ("top_l", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("local_pair_full", ctypes.c_int32), ("score_norm", ctypes.c_int32),
        ("score_pool", ctypes.c_int32),
    ]


class SpavaError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        extra = f" (cuda error {cuda_error})" if status == 5 else ""
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}{extra}")


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sequence_sparse_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, cfgp = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(SpavaConfig)
    i64p = ctypes.POINTER(ctypes.c_int64)
    i32, szp = ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)
    sig = {
        "spava_workspace_size": [cfgp, ctypes.POINTER(ctypes.c_size_t)],
        "spava_packed_len": [cfgp, i64p],
        "spava_score": [cfgp, vp, vp, vp, vp, sz, vp],
        "spava_topk_select": [cfgp, vp, vp, vp],
        "spava_pack_passing": [cfgp, vp, vp, vp, vp, vp, vp],
        "spava_attn": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "spava_prefill_attention": [cfgp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "spava_prefill_attention_host": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp],
        "spava_device_status": [vp, sz, vp, ctypes.POINTER(ctypes.c_int32)],
        "spava_attended_pairs": [cfgp, i64p, i64p],
        "spava_score_noalloc": [cfgp, vp, vp, vp, vp],
        "spava_score_noalloc_status": [vp, ctypes.POINTER(ctypes.c_int32)],
        "spava_selftest_wait_timeout": [vp, sz, vp],
        "spava_plan_chunks": [ctypes.c_int32, i64p, ctypes.c_int64, ctypes.c_int64, i64p],
        "spava_shard_layout": [cfgp, i32, i32, i64p, i64p, ctypes.POINTER(ctypes.c_int32)],
        "spava_shard_sizes": [cfgp, i32, szp, szp, szp],
        "spava_shard_front": [cfgp, i32, i32, vp, vp, vp, vp, vp, sz, vp],
        "spava_shard_local_attn": [cfgp, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "spava_shard_context_attn": [cfgp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "spava_shard_merge": [cfgp, i32, i32, vp, vp, vp, vp, sz, vp],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.spava_status_string.argtypes = [ctypes.c_int]
    lib.spava_status_string.restype = ctypes.c_char_p
    lib.spava_last_cuda_error.argtypes = []
    lib.spava_last_cuda_error.restype = ctypes.c_int32
    _lib = lib
    return lib


def call(name: str, *args) -> None:
    lib = load()
    rc = getattr(lib, name)(*args)
    if rc != SPAVA_OK:
        raise SpavaError(name, rc, lib.spava_last_cuda_error() if rc == 5 else 0)
