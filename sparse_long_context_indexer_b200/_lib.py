"""ctypes binding of ``libdsa_b200.so`` (the C interface in ``include/dsa.h``).

Argument marshalling only.  The library is loaded from this package's
directory; if it is missing the import of the compute functions fails loudly
(there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdsa_b200.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, DSA_ERR_TIMEOUT, \
    DSA_ERR_INDEX_OOB, DSA_ERR_LENGTH = range(8)
DSA_F32, DSA_BF16, DSA_FP8_E4M3 = 0, 1, 2
DSA_OP_INDEXER, DSA_OP_TOPK, DSA_OP_SPARSE_MLA, DSA_OP_DECODE, DSA_OP_PREFILL, DSA_OP_DENSE_MLA = range(6)

# every symbol include/dsa.h declares
EXPORTS = (
    "dsa_workspace_size", "dsa_workspace_init", "dsa_indexer_scores", "dsa_prefill_indexer_scores", "dsa_topk",
    "dsa_sparse_mla_attn", "dsa_dense_mla_attn",
    "dsa_decode_step", "dsa_decode_step_paged", "dsa_append_tokens", "dsa_prefill", "dsa_get_device_status", "dsa_status_string", "dsa_last_cuda_error",
    "dsa_selftest_wait_timeout", "dsa_selftest_attention_stall", "dsa_version", "dsa_sparse_mla_attn_noalloc",
)


class DsaDims(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Nq", ctypes.c_int32), ("H_I", ctypes.c_int32), ("d_I", ctypes.c_int32),
        ("H", ctypes.c_int32), ("k", ctypes.c_int32), ("T_max", ctypes.c_int32), ("idx_dtype", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32), ("ld_scores", ctypes.c_int64),
    ]


class DsaStageEvents(ctypes.Structure):
    _fields_ = [("ev", ctypes.c_void_p * 5)]


class DsaPagedCache(ctypes.Structure):
    _fields_ = [("k_I", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("kv", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("max_blocks", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class DSAError(RuntimeError):
    def __init__(self, status, what, lib=None):
        msg = lib.dsa_status_string(status).decode() if lib is not None else str(status)
        extra = ""
        if lib is not None and status == DSA_ERR_CUDA:
            extra = f" (cudaError {lib.dsa_last_cuda_error()})"
        super().__init__(f"{what}: {msg}{extra}")
        self.status = status


_lock = threading.Lock()
_lib = None


def _declare(lib):
    P = ctypes.c_void_p
    S = ctypes.c_size_t
    I32 = ctypes.c_int32
    F = ctypes.c_float
    D = ctypes.POINTER(DsaDims)
    st = ctypes.c_int
    lib.dsa_workspace_size.argtypes = [D, I32, ctypes.POINTER(S)]
    lib.dsa_workspace_init.argtypes = [P, S, P]
    lib.dsa_indexer_scores.argtypes = [D, P, P, P, P, P, P, P, P, P, S, P]
    lib.dsa_prefill_indexer_scores.argtypes = [D, P, P, P, P, P, P, P, P, P, S, P]
    lib.dsa_topk.argtypes = [D, P, P, P, P, S, P]
    lib.dsa_sparse_mla_attn.argtypes = [D, P, P, P, P, P, F, P, P, P, S, P]
    lib.dsa_sparse_mla_attn_noalloc.argtypes = [D, P, P, P, P, P, F, P, P, P]
    lib.dsa_dense_mla_attn.argtypes = [D, P, P, P, P, F, P, P, P, S, P]
    lib.dsa_decode_step.argtypes = [D, P, P, P, P, P, P, P, P, P, F, P, P, P, P, P, S, P,
                                    ctypes.POINTER(DsaStageEvents)]
    lib.dsa_prefill.argtypes = [D, P, P, P, P, P, P, P, P, P, F, P, P, P, P, S, P]
    lib.dsa_append_tokens.argtypes = [D, ctypes.c_int32, P, P, P, P, P, P, P, ctypes.POINTER(DsaPagedCache), P,
                                       S, P]
    lib.dsa_decode_step_paged.argtypes = [D, P, P, P, ctypes.POINTER(DsaPagedCache), P, P, P, F, P, P, P, P, P, S,
                                          P, ctypes.POINTER(DsaStageEvents)]
    lib.dsa_get_device_status.argtypes = [P, P, ctypes.POINTER(I32)]
    lib.dsa_selftest_wait_timeout.argtypes = [P, S, I32, P]
    lib.dsa_selftest_attention_stall.argtypes = [D, P, P, P, P, P, F, P, P, P, S, I32, P]
    for name in ("dsa_workspace_size", "dsa_workspace_init", "dsa_indexer_scores", "dsa_prefill_indexer_scores",
                 "dsa_topk",
                 "dsa_sparse_mla_attn", "dsa_decode_step", "dsa_decode_step_paged", "dsa_append_tokens",
                 "dsa_prefill",
                 "dsa_get_device_status",
                 "dsa_selftest_wait_timeout", "dsa_selftest_attention_stall", "dsa_sparse_mla_attn_noalloc",
                 "dsa_dense_mla_attn"):
        getattr(lib, name).restype = st
    lib.dsa_status_string.argtypes = [I32]
    lib.dsa_status_string.restype = ctypes.c_char_p
    lib.dsa_last_cuda_error.restype = I32
    lib.dsa_version.restype = ctypes.c_char_p


def load(path: str = LIB_PATH):
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"CUDA library not built: {path} is missing "
                                   "(run python -m sparse_long_context_indexer_b200.build)")
            lib = ctypes.CDLL(path)
            _declare(lib)
            _lib = lib
    return _lib


def check(lib, status, what):
    if status != DSA_OK:
        raise DSAError(status, what, lib)
