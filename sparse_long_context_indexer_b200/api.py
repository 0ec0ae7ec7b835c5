"""Python entry points with the names of the C interface (``include/dsa.h``).

Marshalling only: each function checks the tensors' device, dtype and shape,
passes their device pointers and torch's current CUDA stream to the C library
and returns.  Every step of the hot path runs in the library's CUDA kernels;
nothing here computes on the host or falls back to torch operations.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

from . import _lib

D_K, D_V = 576, 512


@dataclass
class Dims:
    B: int
    Nq: int
    H_I: int
    d_I: int
    H: int
    k: int
    T_max: int
    idx_dtype: int
    kv_dtype: int
    ld_scores: int

    def c(self) -> _lib.DsaDims:
        return _lib.DsaDims(self.B, self.Nq, self.H_I, self.d_I, self.H, self.k, self.T_max, self.idx_dtype,
                            self.kv_dtype, 0, self.ld_scores)


def dims_of(inp, ld_scores: Optional[int] = None, Nq: Optional[int] = None) -> Dims:
    """Dims for an ``inputs.DSAInputs`` workload (ld_scores defaults to T_max rounded up to 4)."""
    ld = ld_scores if ld_scores is not None else (inp.T_max + 3) // 4 * 4
    return Dims(inp.B, inp.Nq if Nq is None else Nq, inp.H_I, inp.d_I, inp.H, inp.k, inp.T_max, inp.idx_dtype,
                inp.kv_dtype, ld)


def _stream_ptr(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def workspace_size(dims: Dims, op: int) -> int:
    lib = _lib.load()
    n = ctypes.c_size_t(0)
    d = dims.c()
    _lib.check(lib, lib.dsa_workspace_size(ctypes.byref(d), op, ctypes.byref(n)), "dsa_workspace_size")
    return int(n.value)


def make_workspace(dims: Dims, op: int, device=None) -> torch.Tensor:
    """A zero-initialised uint8 device buffer sized for `op` (torch allocates; the library never does)."""
    lib = _lib.load()
    nbytes = workspace_size(dims, op)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device or "cuda")
    _lib.check(lib, lib.dsa_workspace_init(ws.data_ptr(), ws.numel(), _stream_ptr()), "dsa_workspace_init")
    return ws


def get_device_status(ws: torch.Tensor) -> int:
    lib = _lib.load()
    v = ctypes.c_int32(0)
    _lib.check(lib, lib.dsa_get_device_status(ws.data_ptr(), _stream_ptr(), ctypes.byref(v)), "dsa_get_device_status")
    return int(v.value)


def status_string(code: int) -> str:
    return _lib.load().dsa_status_string(code).decode()


def indexer_scores(dims: Dims, q_I, q_scale, w, k_I, k_scale, q_seq, q_len, scores, ws=None):
    lib = _lib.load()
    d = dims.c()
    rc = lib.dsa_indexer_scores(ctypes.byref(d), _ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_I), _ptr(k_scale),
                                _ptr(q_seq), _ptr(q_len), _ptr(scores), _ptr(ws),
                                0 if ws is None else ws.numel(), _stream_ptr())
    _lib.check(lib, rc, "dsa_indexer_scores")
    return scores


def prefill_indexer_scores(dims: Dims, q_I, q_scale, w, k_I, k_scale, q_seq, q_len, scores, ws=None):
    """Indexer scores for rows of one prompt: four consecutive rows per tensor-core pass."""
    lib = _lib.load()
    d = dims.c()
    rc = lib.dsa_prefill_indexer_scores(ctypes.byref(d), _ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_I), _ptr(k_scale),
                                        _ptr(q_seq), _ptr(q_len), _ptr(scores), _ptr(ws),
                                        0 if ws is None else ws.numel(), _stream_ptr())
    _lib.check(lib, rc, "dsa_prefill_indexer_scores")
    return scores


def topk(dims: Dims, scores, q_len, idx, ws=None):
    lib = _lib.load()
    d = dims.c()
    rc = lib.dsa_topk(ctypes.byref(d), _ptr(scores), _ptr(q_len), _ptr(idx), _ptr(ws),
                      0 if ws is None else ws.numel(), _stream_ptr())
    _lib.check(lib, rc, "dsa_topk")
    return idx


def dense_mla_attn(dims: Dims, q, kv, q_seq, q_len, softmax_scale, out, lse, ws):
    """Attention over every position s < q_len[t] (the dense comparison of the sparse path)."""
    lib = _lib.load()
    d = dims.c()
    rc = lib.dsa_dense_mla_attn(ctypes.byref(d), _ptr(q), _ptr(kv), _ptr(q_seq), _ptr(q_len),
                                ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                _stream_ptr())
    _lib.check(lib, rc, "dsa_dense_mla_attn")
    return out


def sparse_mla_attn(dims: Dims, q, kv, idx, q_seq, q_len, softmax_scale, out, lse, ws):
    lib = _lib.load()
    d = dims.c()
    rc = lib.dsa_sparse_mla_attn(ctypes.byref(d), _ptr(q), _ptr(kv), _ptr(idx), _ptr(q_seq), _ptr(q_len),
                                 ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                 _stream_ptr())
    _lib.check(lib, rc, "dsa_sparse_mla_attn")
    return out, lse


@dataclass
class PagedCache:
    """Block pools and block table of a paged cache (device tensors)."""
    k_I: torch.Tensor          # [num_blocks, block_size, d_I] e4m3 (uint8)
    k_scale: torch.Tensor      # [num_blocks, block_size] fp32
    kv: torch.Tensor           # [num_blocks, block_size, 576] bf16
    block_table: torch.Tensor  # [B, max_blocks] int32
    block_size: int

    def c(self) -> _lib.DsaPagedCache:
        return _lib.DsaPagedCache(_ptr(self.k_I), _ptr(self.k_scale), _ptr(self.kv), _ptr(self.block_table),
                                  self.block_size, self.kv.shape[0], self.block_table.shape[1], 0)


def append_tokens(dims: Dims, seq, pos, kv_new, k_new, kv=None, k_I=None, k_scale=None,
                  cache: Optional["PagedCache"] = None, ws=None):
    """Write new tokens (bf16 latent rows, fp32 indexer keys) into the caches, quantising as
    the caches' types require; contiguous caches (kv, k_I, k_scale) or a paged cache."""
    lib = _lib.load()
    d = dims.c()
    pc = cache.c() if cache is not None else None
    rc = lib.dsa_append_tokens(ctypes.byref(d), int(seq.numel()), _ptr(seq), _ptr(pos), _ptr(kv_new), _ptr(k_new),
                               _ptr(kv), _ptr(k_I), _ptr(k_scale), ctypes.byref(pc) if pc is not None else None,
                               _ptr(ws), 0 if ws is None else ws.numel(), _stream_ptr())
    _lib.check(lib, rc, "dsa_append_tokens")


def decode_step_paged(dims: Dims, q_I, q_scale, w, cache: PagedCache, q, q_seq, q_len, softmax_scale, out, lse, ws,
                      scores_out=None, idx_out=None):
    """One decode step over a paged cache on torch's current stream."""
    lib = _lib.load()
    d = dims.c()
    pc = cache.c()
    rc = lib.dsa_decode_step_paged(ctypes.byref(d), _ptr(q_I), _ptr(q_scale), _ptr(w), ctypes.byref(pc), _ptr(q),
                                   _ptr(q_seq), _ptr(q_len), ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
                                   _ptr(scores_out), _ptr(idx_out), _ptr(ws), ws.numel(), _stream_ptr(), None)
    _lib.check(lib, rc, "dsa_decode_step_paged")
    return out, lse


def decode_step(dims: Dims, q_I, q_scale, w, k_I, k_scale, q, kv, q_seq, q_len, softmax_scale, out, lse, ws,
                scores_out=None, idx_out=None, events: Optional[Sequence] = None):
    """One decode step (indexer -> top-k -> sparse MLA) on torch's current stream.

    events: optional 5 ``torch.cuda.Event(enable_timing=True)`` recorded before
    the first stage and after each stage (indexer, top-k, attention, merge).
    """
    lib = _lib.load()
    d = dims.c()
    evp = None
    if events is not None:
        evs = _lib.DsaStageEvents()
        for i, e in enumerate(events):
            if e is not None and not e.cuda_event:
                e.record()  # torch creates the CUDA event lazily, on its first record
            evs.ev[i] = None if e is None else e.cuda_event
        evp = ctypes.byref(evs)
    rc = lib.dsa_decode_step(ctypes.byref(d), _ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_I), _ptr(k_scale), _ptr(q),
                             _ptr(kv), _ptr(q_seq), _ptr(q_len), ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
                             _ptr(scores_out), _ptr(idx_out), _ptr(ws), ws.numel(), _stream_ptr(), evp)
    _lib.check(lib, rc, "dsa_decode_step")
    return out, lse


def prefill(dims: Dims, q_I, q_scale, w, k_I, k_scale, q, kv, q_seq, q_len, softmax_scale, out, lse, ws,
            idx_out=None):
    lib = _lib.load()
    d = dims.c()
    rc = lib.dsa_prefill(ctypes.byref(d), _ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_I), _ptr(k_scale), _ptr(q),
                         _ptr(kv), _ptr(q_seq), _ptr(q_len), ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
                         _ptr(idx_out), _ptr(ws), ws.numel(), _stream_ptr())
    _lib.check(lib, rc, "dsa_prefill")
    return out, lse


def selftest_wait_timeout(ws: torch.Tensor, timeout_us: int = 200000):
    lib = _lib.load()
    rc = lib.dsa_selftest_wait_timeout(ws.data_ptr(), ws.numel(), int(timeout_us), _stream_ptr())
    _lib.check(lib, rc, "dsa_selftest_wait_timeout")


def selftest_attention_stall(dims: Dims, q, kv, idx, q_seq, q_len, softmax_scale, out, lse, ws,
                             timeout_us: int = 100000):
    """The attention kernel with its first tile never signalled: its bounded wait runs out."""
    lib = _lib.load()
    d = dims.c()
    rc = lib.dsa_selftest_attention_stall(ctypes.byref(d), _ptr(q), _ptr(kv), _ptr(idx), _ptr(q_seq), _ptr(q_len),
                                          ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                          int(timeout_us), _stream_ptr())
    _lib.check(lib, rc, "dsa_selftest_attention_stall")


# ---- conveniences over an inputs.DSAInputs workload --------------------------

def alloc_outputs(inp, device=None):
    dev = device or inp.device
    odt = torch.float32 if inp.kv_dtype == _lib.DSA_F32 else torch.bfloat16
    out = torch.empty((inp.Nq, inp.H, D_V), dtype=odt, device=dev)
    lse = torch.empty((inp.Nq, inp.H), dtype=torch.float32, device=dev)
    return out, lse


def run_decode(inp, ws=None, scores_out=None, idx_out=None, events=None, dims=None, out=None, lse=None):
    """decode_step over a device-resident ``DSAInputs``; returns (out, lse)."""
    dims = dims or dims_of(inp)
    if ws is None:
        ws = make_workspace(dims, _lib.DSA_OP_DECODE, inp.device)
    if out is None:
        out, lse = alloc_outputs(inp)
    return decode_step(dims, inp.q_I, inp.q_scale, inp.w, inp.k_I, inp.k_scale, inp.q, inp.kv, inp.q_seq, inp.q_len,
                       inp.softmax_scale, out, lse, ws, scores_out=scores_out, idx_out=idx_out, events=events)
