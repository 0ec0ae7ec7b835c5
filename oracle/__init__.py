"""CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

A thin ctypes wrapper around ``dsa_oracle.c`` (plain C, fp64 accumulation).
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package; the library's product path never does.

Functions take numpy arrays (or CPU torch tensors) holding the *stored* bytes
of the inputs (e4m3 codes as uint8, bf16 as uint16/int16 bit patterns, or
float32) and return float64 results.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdsa_oracle.so")
# A prebuilt oracle library to load instead.  Only the test that plants mistakes in a copy of
# the oracle source (and checks that the pins catch each one) uses it, in a child process that
# also sets DSA_ORACLE_MUTANT_RUN=1; anywhere else a stray DSA_ORACLE_LIB would swap the
# checker, so it is refused.
_LIB_OVERRIDE = os.environ.get("DSA_ORACLE_LIB")
if _LIB_OVERRIDE and os.environ.get("DSA_ORACLE_MUTANT_RUN") != "1":
    raise RuntimeError("DSA_ORACLE_LIB is honoured only inside the oracle mutation test's child process "
                       "(DSA_ORACLE_MUTANT_RUN=1); unset it")
_lock = threading.Lock()
_lib = None

F32, BF16, FP8 = 0, 1, 2


GCC_FLAGS = ["-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off"]


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c with gcc (-O2, OpenMP, IEEE arithmetic, no fast-math)."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc"] + GCC_FLAGS + [_SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            L = ctypes.c_int64
            D = ctypes.c_double
            lib.dsa_oracle_e4m3_decode.restype = D
            lib.dsa_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.dsa_oracle_bf16_decode.restype = D
            lib.dsa_oracle_bf16_decode.argtypes = [ctypes.c_uint16]
            lib.dsa_oracle_indexer.restype = I
            lib.dsa_oracle_indexer.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, P, P, L, I]
            lib.dsa_oracle_topk.restype = I
            lib.dsa_oracle_topk.argtypes = [I, L, P, P, I, P, I]
            for name in ("dsa_oracle_sparse_attn", "dsa_oracle_masked_dense_attn"):
                f = getattr(lib, name)
                f.restype = I
                f.argtypes = [I, I, I, I, I, I, P, P, P, P, P, D, P, P, I]
            lib.dsa_oracle_dense_attn.restype = I
            lib.dsa_oracle_dense_attn.argtypes = [I, I, I, I, I, P, P, P, P, D, P, P, I]
            lib.dsa_oracle_max_threads.restype = I
            _lib = lib
    return _lib


def _np(x, dtype=None):
    """Contiguous numpy view of a CPU array/tensor, reinterpreting 16-bit floats as bits."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                x = x.view(torch.int16)
            elif x.dtype == torch.float8_e4m3fn:
                x = x.view(torch.uint8)
            x = x.numpy()
    except ImportError:
        pass
    x = np.ascontiguousarray(x)
    if dtype is not None and x.dtype != dtype:
        x = x.astype(dtype)
    return x


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(_load().dsa_oracle_max_threads())


def e4m3_decode(code: int) -> float:
    return float(_load().dsa_oracle_e4m3_decode(int(code) & 0xFF))


def bf16_decode(bits: int) -> float:
    return float(_load().dsa_oracle_bf16_decode(int(bits) & 0xFFFF))


def indexer(inp, q_I=None, q_scale=None, w=None, k_I=None, k_scale=None, q_seq=None, q_len=None,
            ld=None, nthreads=0):
    """Scores [Nq, ld] float64 (NaN where s >= q_len[t]) for an ``inputs.DSAInputs``-like object."""
    q_I = _np(inp.q_I if q_I is None else q_I)
    w = _np(inp.w if w is None else w)
    k_I = _np(inp.k_I if k_I is None else k_I)
    qs = _np(inp.q_scale if q_scale is None else q_scale, np.float32)
    ks = _np(inp.k_scale if k_scale is None else k_scale, np.float32)
    q_seq = _np(inp.q_seq if q_seq is None else q_seq, np.int32)
    q_len = _np(inp.q_len if q_len is None else q_len, np.int32)
    Nq = q_seq.shape[0]
    if ld is None:
        ld = int(max(int(q_len.max()) if Nq else 1, 1))
    out = np.full((Nq, ld), np.nan, dtype=np.float64)
    rc = _load().dsa_oracle_indexer(Nq, inp.H_I, inp.d_I, inp.T_max, inp.B, inp.idx_dtype,
                                   _ptr(q_I), _ptr(qs), _ptr(w), _ptr(k_I), _ptr(ks),
                                   _ptr(q_seq), _ptr(q_len), _ptr(out), ld, nthreads)
    if rc != 0:
        raise ValueError(f"oracle indexer rejected its arguments (rc={rc})")
    return out


def topk(scores, q_len, k, nthreads=0):
    """Index lists [Nq, k] int32, ascending positions, -1 padded."""
    sc = _np(scores, np.float64)
    q_len = _np(q_len, np.int32)
    Nq, ld = sc.shape
    idx = np.empty((Nq, k), dtype=np.int32)
    rc = _load().dsa_oracle_topk(Nq, ld, _ptr(sc), _ptr(q_len), k, _ptr(idx), nthreads)
    if rc != 0:
        raise ValueError(f"oracle topk failed (rc={rc})")
    return idx


def _bf16_bits_to_f32(bits):
    """bf16 bit patterns -> float32: a bf16 value is the upper half of an IEEE binary32."""
    return (np.asarray(bits).astype(np.uint16).astype(np.uint32) << 16).view(np.float32)


def dequant_latent_fp8(entries):
    """656-byte FP8 latent entries (kgptalkie "What Does the GPU Actually Run?": 512 values
    in e4m3, 4 float32 scale factors, the 64 rope values in bf16) -> float32 [..., 576].

    Latent value i = e4m3(code_i) * scale[i // 128] (this oracle's own e4m3 decoding,
    products formed in float64 and stored as float32); rope values widened from bf16."""
    e = np.ascontiguousarray(_np(entries, np.uint8))
    lead = e.shape[:-1]
    e = e.reshape(-1, 656)
    table = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    scales = e[:, 512:528].copy().view(np.float32).astype(np.float64)  # [n, 4]
    lat = table[e[:, :512]].reshape(-1, 4, 128) * scales[:, :, None]
    rope = _bf16_bits_to_f32(e[:, 528:656].copy().view(np.uint16))
    out = np.concatenate([lat.reshape(-1, 512).astype(np.float32), rope.reshape(-1, 64)], axis=1)
    return out.reshape(*lead, 576)


def _attn_operands(inp, q, kv):
    """(q, kv, element type) for the C attention routines; an FP8 latent cache is dequantised
    here and the query widened to float32 with it (exact), so both go in as float32."""
    if inp.kv_dtype == FP8:
        return _bf16_bits_to_f32(_np(q)), dequant_latent_fp8(kv), F32
    return _np(q), _np(kv), inp.kv_dtype


def sparse_attn(inp, idx, q=None, kv=None, q_seq=None, q_len=None, scale=None, nthreads=0):
    """(out [Nq, H, 512] float64, lse [Nq, H] float64) over the positions in idx."""
    q, kv, kvdt = _attn_operands(inp, inp.q if q is None else q, inp.kv if kv is None else kv)
    idx = _np(idx, np.int32)
    q_seq = _np(inp.q_seq if q_seq is None else q_seq, np.int32)
    q_len = _np(inp.q_len if q_len is None else q_len, np.int32)
    Nq = q_seq.shape[0]
    k = idx.shape[1]
    out = np.zeros((Nq, inp.H, 512), dtype=np.float64)
    lse = np.zeros((Nq, inp.H), dtype=np.float64)
    sc = inp.softmax_scale if scale is None else scale
    rc = _load().dsa_oracle_sparse_attn(Nq, inp.H, inp.T_max, inp.B, k, kvdt, _ptr(q), _ptr(kv),
                                       _ptr(idx), _ptr(q_seq), _ptr(q_len), sc, _ptr(out), _ptr(lse),
                                       nthreads)
    if rc != 0:
        raise ValueError(f"oracle sparse attention failed (rc={rc})")
    return out, lse


def masked_dense_attn(inp, idx, scale=None, nthreads=0):
    q, kv, kvdt = _attn_operands(inp, inp.q, inp.kv)
    idx = _np(idx, np.int32)
    q_seq = _np(inp.q_seq, np.int32)
    q_len = _np(inp.q_len, np.int32)
    Nq = q_seq.shape[0]
    out = np.zeros((Nq, inp.H, 512), dtype=np.float64)
    lse = np.zeros((Nq, inp.H), dtype=np.float64)
    sc = inp.softmax_scale if scale is None else scale
    rc = _load().dsa_oracle_masked_dense_attn(Nq, inp.H, inp.T_max, inp.B, idx.shape[1], kvdt,
                                             _ptr(q), _ptr(kv), _ptr(idx), _ptr(q_seq), _ptr(q_len),
                                             sc, _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise ValueError(f"oracle masked attention failed (rc={rc})")
    return out, lse


def dense_attn(inp, scale=None, nthreads=0):
    q, kv, kvdt = _attn_operands(inp, inp.q, inp.kv)
    q_seq = _np(inp.q_seq, np.int32)
    q_len = _np(inp.q_len, np.int32)
    Nq = q_seq.shape[0]
    out = np.zeros((Nq, inp.H, 512), dtype=np.float64)
    lse = np.zeros((Nq, inp.H), dtype=np.float64)
    sc = inp.softmax_scale if scale is None else scale
    rc = _load().dsa_oracle_dense_attn(Nq, inp.H, inp.T_max, inp.B, kvdt, _ptr(q), _ptr(kv),
                                      _ptr(q_seq), _ptr(q_len), sc, _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise ValueError(f"oracle dense attention failed (rc={rc})")
    return out, lse


def decode(inp, nthreads=0):
    """The whole path: scores -> top-k -> sparse attention.  Returns (scores, idx, out, lse)."""
    sc = indexer(inp, nthreads=nthreads)
    idx = topk(sc, inp.q_len, inp.k, nthreads=nthreads)
    out, lse = sparse_attn(inp, idx, nthreads=nthreads)
    return sc, idx, out, lse
