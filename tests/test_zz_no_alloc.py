"""The no-allocation attention entry point, called through the C interface.

Some callers cannot allocate device memory at all: a host framework that owns
every device buffer and hands a kernel only its inputs and outputs, or a
serving loop whose memory budget is fixed at start-up.  For them
dsa_sparse_mla_attn_noalloc keeps the split partials of the attention in a
buffer the library holds statically on each GPU.

The buffer is only used when a row is split more than eight ways: up to eight
splits merge on chip.  With k = 2048 the library plans
min(16, SMs // (2 * Nq)) splits (rows per split rounded up to whole 64-row
tiles), so on a 148-SM B200 batches of 1 to 4 rows take 16 splits and go
through the static buffer.  These tests check, on two calls in a row with
different inputs (stale partials of the first call would show in the second),
that the entry point returns what the workspace-based dsa_sparse_mla_attn
returns and what the oracle computes; that the on-chip merge case agrees as
well; and that a request larger than the static buffer is refused before any
launch.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_indexer_b200 import _lib, api, inputs
from tests.tolerances import check_attention

pytestmark = pytest.mark.gpu

STATIC_PARTIAL_ROWS = 64   # (split, row) pairs the static buffer holds


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return _lib.load()


def planned_splits(nq, k=2048, tile=64):
    """The library's split plan: SMs // (2 nq) clamped to [1, 16], rows per split
    rounded up to whole 64-row tiles, then the splits those rows need."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    s = max(1, min(16, sms // (2 * nq)))
    rows = -(-(-(-k // s)) // tile) * tile
    return -(-k // rows)


def random_index_lists(nq, n, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.full((nq, k), -1, np.int32)
    for t in range(nq):
        m = k if t % 3 else k - 300          # every third row has a -1 tail
        idx[t, :m] = np.sort(rng.choice(n, m, replace=False))
    return torch.from_numpy(idx)


def call_noalloc(lib, dims, g, idx, out, lse):
    d = dims.c()
    return lib.dsa_sparse_mla_attn_noalloc(ctypes.byref(d), g.q.data_ptr(), g.kv.data_ptr(), idx.data_ptr(),
                                           g.q_seq.data_ptr(), g.q_len.data_ptr(), ctypes.c_float(g.softmax_scale),
                                           out.data_ptr(), lse.data_ptr(),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def two_calls_match(lib, nq, n, seeds):
    for call, seed in enumerate(seeds):
        inp = inputs.make_decode_inputs(f"noalloc_{nq}_{seed}", [n] * nq, T_max=n, seed=seed)
        idx = random_index_lists(nq, n, inp.k, seed)
        o_out, o_lse = oracle.sparse_attn(inp, idx)
        g = inp.to("cuda")
        idx_d = idx.cuda()
        dims = api.dims_of(g)
        ws = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
        ref_out, ref_lse = api.alloc_outputs(g)
        api.sparse_mla_attn(dims, g.q, g.kv, idx_d, g.q_seq, g.q_len, g.softmax_scale, ref_out, ref_lse, ws)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert call_noalloc(lib, dims, g, idx_d, out, lse) == _lib.DSA_OK
        torch.cuda.synchronize()
        assert api.get_device_status(ws) == 0
        assert torch.isfinite(out.float()).all(), f"nq={nq} call {call}: non-finite output"
        got_o, got_l = out.float().cpu().numpy(), lse.cpu().numpy()
        check_attention(got_o, ref_out.float().cpu().numpy(), got_l, ref_lse.cpu().numpy())
        check_attention(got_o, o_out, got_l, o_lse)


@pytest.mark.parametrize("nq", [1, 4])
def test_noalloc_partials_in_static_scratch_match_workspace_entry_and_oracle(lib, nq):
    # 16 splits per row on a 148-SM B200: the partials go through the static buffer
    # (4 rows x 16 splits = 64 partial rows, exactly what it holds)
    s = planned_splits(nq)
    assert s > 8 and s * nq <= STATIC_PARTIAL_ROWS, f"nq={nq} plans {s} splits: not the static-buffer path"
    two_calls_match(lib, nq, 4096, (100 + nq, 200 + nq))


def test_noalloc_on_chip_merge_matches_workspace_entry_and_oracle(lib):
    # 16 rows plan 4 splits: they merge on chip and the static buffer is not touched
    assert 2 <= planned_splits(16) <= 8
    two_calls_match(lib, 16, 4096, (301, 302))


def test_noalloc_refuses_requests_beyond_its_scratch(lib):
    nq = next(q for q in range(1, 75) if planned_splits(q) > 8 and planned_splits(q) * q > STATIC_PARTIAL_ROWS)
    g = inputs.make_decode_inputs("noalloc_big", [2048] * nq, T_max=2048, seed=7).to("cuda")
    idx = random_index_lists(nq, 2048, g.k, 7).cuda()
    out, lse = api.alloc_outputs(g)
    assert call_noalloc(lib, api.dims_of(g), g, idx, out, lse) == _lib.DSA_ERR_UNSUPPORTED
