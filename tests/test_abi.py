"""The C library: builds, loads, exports every symbol include/dsa.h declares,
plans workspaces and rejects bad arguments on the host (no GPU needed)."""
import ctypes
import os
import re

import pytest
import torch

from sparse_long_context_indexer_b200 import _lib, api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def header_functions():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = header_functions()
    for required in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn", "dsa_decode_step", "dsa_prefill"):
        assert required in names
    assert set(names) == set(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.dsa_version()
    for code in range(8):
        assert lib.dsa_status_string(code)


def decode_dims(**kw):
    d = dict(B=16, Nq=16, H_I=64, d_I=64, H=128, k=2048, T_max=131072, idx_dtype=_lib.DSA_FP8_E4M3,
             kv_dtype=_lib.DSA_BF16, ld_scores=131072)
    d.update(kw)
    return api.Dims(**d)


def test_workspace_sizes(lib):
    d = decode_dims()
    ws = api.workspace_size(d, _lib.DSA_OP_DECODE)
    assert ws >= 16 * 131072 * 4 + 16 * 2048 * 4
    assert api.workspace_size(d, _lib.DSA_OP_INDEXER) == 256
    assert api.workspace_size(d, _lib.DSA_OP_TOPK) == 256
    pre = api.workspace_size(decode_dims(B=1, Nq=65536, T_max=65536, ld_scores=65536), _lib.DSA_OP_PREFILL)
    assert pre <= (64 << 20) + (16 << 20), "prefill works in L2-sized row chunks"


def test_short_cache_decode_workspace_holds_the_dense_plan(lib):
    # a decode over a cache of at most k tokens runs the attention's dense form, whose splits are
    # planned over T_max rounded up to whole 64-row tiles: the decode workspace must hold those
    # partials beside its scores and index lists, for every batch size and width
    for k in (64, 100, 1000, 1100, 2048):
        for T_max in sorted({x // 4 * 4 for x in (k, k - 37, 64) if 4 <= x <= k}):  # FP8 keys: T_max % 4 == 0
            for nq in range(1, 41):
                ld = (T_max + 3) // 4 * 4
                d = decode_dims(B=nq, Nq=nq, k=k, T_max=T_max, ld_scores=ld)
                dec = api.workspace_size(d, _lib.DSA_OP_DECODE)
                dense = api.workspace_size(d, _lib.DSA_OP_DENSE_MLA)
                assert dec >= dense + nq * ld * 4 + nq * k * 4, (k, T_max, nq)


@pytest.mark.parametrize("bad,code", [
    (dict(d_I=96), _lib.DSA_ERR_UNSUPPORTED),
    (dict(H_I=32), _lib.DSA_ERR_UNSUPPORTED),
    (dict(H=64), _lib.DSA_ERR_UNSUPPORTED),
    (dict(k=4096), _lib.DSA_ERR_UNSUPPORTED),
    (dict(k=0), _lib.DSA_ERR_INVALID_ARG),
    (dict(ld_scores=131071), _lib.DSA_ERR_INVALID_ARG),
    (dict(idx_dtype=7), _lib.DSA_ERR_INVALID_ARG),
])
def test_bad_dims_rejected(lib, bad, code):
    d = decode_dims(**bad).c()
    n = ctypes.c_size_t(0)
    assert lib.dsa_workspace_size(ctypes.byref(d), _lib.DSA_OP_DECODE, ctypes.byref(n)) == code


def test_null_and_misaligned_pointers_rejected_before_launch(lib):
    d = decode_dims().c()
    P = 1 << 20
    args = [P] * 9
    # NULL q_I
    rc = lib.dsa_decode_step(ctypes.byref(d), None, *args[1:], ctypes.c_float(0.07), P, P, None, None, P, 1 << 30,
                             None, None)
    assert rc == _lib.DSA_ERR_INVALID_ARG
    # misaligned kv
    bad = list(args)
    bad[6] = P + 8  # kv
    rc = lib.dsa_decode_step(ctypes.byref(d), *bad, ctypes.c_float(0.07), P, P, None, None, P, 1 << 30, None, None)
    assert rc == _lib.DSA_ERR_INVALID_ARG
    # misaligned q_scale (every tensor base must be 16-byte aligned)
    bad = list(args)
    bad[1] = P + 4  # q_scale
    rc = lib.dsa_decode_step(ctypes.byref(d), *bad, ctypes.c_float(0.07), P, P, None, None, P, 1 << 30, None, None)
    assert rc == _lib.DSA_ERR_INVALID_ARG
    # workspace too small
    rc = lib.dsa_decode_step(ctypes.byref(d), *args, ctypes.c_float(0.07), P, P, None, None, P, 1024, None, None)
    assert rc == _lib.DSA_ERR_WORKSPACE
    # non-finite softmax scale
    rc = lib.dsa_decode_step(ctypes.byref(d), *args, ctypes.c_float(float("nan")), P, P, None, None, P, 1 << 30,
                             None, None)
    assert rc == _lib.DSA_ERR_INVALID_ARG


def test_python_layer_has_no_compute_fallback():
    """The binding marshals pointers only: no torch math on tensors in api.py."""
    src = open(os.path.join(ROOT, "sparse_long_context_indexer_b200", "api.py")).read()
    for forbidden in ("torch.topk", "torch.softmax", "torch.einsum", "torch.matmul", "@ ", "relu", "oracle"):
        assert forbidden not in src, forbidden


def _paged(block_size=64, max_blocks=2048, num_blocks=4096, k_scale=1 << 20, table=1 << 21, reserved=0):
    return _lib.DsaPagedCache(k_I=1 << 20, k_scale=k_scale, kv=1 << 22, block_table=table, block_size=block_size,
                              num_blocks=num_blocks, max_blocks=max_blocks, reserved=reserved)


@pytest.mark.parametrize("case,code", [
    (dict(n=-1), _lib.DSA_ERR_INVALID_ARG),
    (dict(n=70000), _lib.DSA_ERR_UNSUPPORTED),
    (dict(seq=None), _lib.DSA_ERR_INVALID_ARG),
    (dict(k_scale=None), _lib.DSA_ERR_INVALID_ARG),
    (dict(paged=_paged(block_size=48)), _lib.DSA_ERR_INVALID_ARG),
    (dict(paged=_paged(max_blocks=1000)), _lib.DSA_ERR_INVALID_ARG),
    (dict(paged=_paged(reserved=1)), _lib.DSA_ERR_INVALID_ARG),
    (dict(dims=dict(kv_dtype=_lib.DSA_F32)), _lib.DSA_ERR_UNSUPPORTED),
    (dict(ws_bytes=64), _lib.DSA_ERR_WORKSPACE),
    (dict(n=0), _lib.DSA_OK),
])
def test_append_tokens_host_checks(lib, case, code):
    P = 1 << 20
    d = decode_dims(**case.get("dims", {})).c()
    paged = case.get("paged")
    rc = lib.dsa_append_tokens(ctypes.byref(d), case.get("n", 4), case.get("seq", P), P, P, P, P, P,
                               case.get("k_scale", P), ctypes.byref(paged) if paged is not None else None, P,
                               case.get("ws_bytes", 256), None)
    assert rc == code


@pytest.mark.parametrize("case,code", [
    (dict(cache=None), _lib.DSA_ERR_INVALID_ARG),
    (dict(cache=_paged(table=None)), _lib.DSA_ERR_INVALID_ARG),
    (dict(cache=_paged(block_size=96)), _lib.DSA_ERR_INVALID_ARG),
    (dict(cache=_paged(block_size=32, max_blocks=4096)), _lib.DSA_ERR_INVALID_ARG),
    (dict(cache=_paged(max_blocks=1024)), _lib.DSA_ERR_INVALID_ARG),
    (dict(cache=_paged(k_scale=(1 << 20) + 4)), _lib.DSA_ERR_INVALID_ARG),
    (dict(cache=_paged(), dims=dict(idx_dtype=_lib.DSA_F32)), _lib.DSA_ERR_UNSUPPORTED),
    (dict(cache=_paged(), ws_bytes=1024), _lib.DSA_ERR_WORKSPACE),
])
def test_paged_decode_host_checks(lib, case, code):
    P = 1 << 20
    d = decode_dims(**case.get("dims", {})).c()
    cache = case["cache"]
    rc = lib.dsa_decode_step_paged(ctypes.byref(d), P, P, P, ctypes.byref(cache) if cache is not None else None, P,
                                   P, P, ctypes.c_float(0.07), P, P, None, None, P, case.get("ws_bytes", 1 << 30),
                                   None, None)
    assert rc == code


def test_dense_and_prefill_host_checks(lib):
    P = 1 << 20
    d = decode_dims().c()
    # dense attention: NULL query, then a workspace below its plan
    assert lib.dsa_dense_mla_attn(ctypes.byref(d), None, P, P, P, ctypes.c_float(0.07), P, P, P, 1 << 30,
                                  None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_dense_mla_attn(ctypes.byref(d), P, P, P, P, ctypes.c_float(0.07), P, P, P, 16,
                                  None) == _lib.DSA_ERR_WORKSPACE
    # prefill: misaligned w, non-finite scale, an empty batch (no launch)
    one = decode_dims(B=1, Nq=4096, T_max=4096, ld_scores=4096).c()
    args = [P, P, P, P, P, P, P, P, P]
    bad = list(args)
    bad[2] = P + 2
    assert lib.dsa_prefill(ctypes.byref(one), *bad, ctypes.c_float(0.07), P, P, None, P, 1 << 30,
                           None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_prefill(ctypes.byref(one), *args, ctypes.c_float(float("inf")), P, P, None, P, 1 << 30,
                           None) == _lib.DSA_ERR_INVALID_ARG
    empty = decode_dims(B=1, Nq=0, T_max=4096, ld_scores=4096).c()
    assert lib.dsa_prefill(ctypes.byref(empty), *args, ctypes.c_float(0.07), P, P, None, P, 1 << 30,
                           None) == _lib.DSA_OK


def planned_splits(nq, k=2048, sms=148):
    """The attention's split plan: SMs // (2 nq) clamped to [1, 16], rows per split rounded up to
    whole 64-row tiles, then the splits those rows need (a CPU without a GPU plans for 148 SMs)."""
    s = max(1, min(16, sms // (2 * nq)))
    rows = -(-(-(-k // s)) // 64) * 64
    return -(-k // rows)


@pytest.mark.skipif(torch.cuda.is_available(), reason="host-side refusal only: without a GPU no call can launch")
def test_noalloc_refuses_exactly_the_plans_beyond_its_scratch(lib):
    # more than 8 splits go through a static buffer of 64 (split, row) partials; at k = 2048 on
    # 148 SMs only Nq = 6 (11 splits x 6 rows = 66) exceeds it, which the entry refuses on the
    # host.  Only refused calls are made here (they return before any CUDA call).
    refused = [nq for nq in range(1, 80) if planned_splits(nq) > 8 and planned_splits(nq) * nq > 64]
    assert refused == [6]
    for nq in refused:
        d = decode_dims(B=nq, Nq=nq).c()
        P = ctypes.c_void_p(1 << 20)
        rc = lib.dsa_sparse_mla_attn_noalloc(ctypes.byref(d), P, P, P, P, P, ctypes.c_float(0.07), P, P,
                                             ctypes.c_void_p(0))
        assert rc == _lib.DSA_ERR_UNSUPPORTED
