"""The no-allocation attention entry point, called through the C interface.

Some callers cannot allocate device memory at all: a host framework that owns
every device buffer and hands a kernel only its inputs and outputs, or a
serving loop whose memory budget is fixed at start-up.  For them
dsa_sparse_mla_attn_noalloc keeps its split scratch in a buffer the library
holds statically on each GPU.  These tests check that it returns what the
workspace-based dsa_sparse_mla_attn returns, on two calls in a row (the second
call reuses the scratch the first one left behind), and that a request larger
than the static buffer is refused before any launch.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_long_context_indexer_b200 import _lib, api, inputs
from tests.tolerances import check_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return _lib.load()


def random_index_lists(nq, n, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.full((nq, k), -1, np.int32)
    for t in range(nq):
        m = k if t % 5 else k - 300          # one row in five has a -1 tail
        idx[t, :m] = np.sort(rng.choice(n, m, replace=False))
    return torch.from_numpy(idx)


def call_noalloc(lib, dims, g, idx, out, lse):
    d = dims.c()
    return lib.dsa_sparse_mla_attn_noalloc(ctypes.byref(d), g.q.data_ptr(), g.kv.data_ptr(), idx.data_ptr(),
                                           g.q_seq.data_ptr(), g.q_len.data_ptr(), ctypes.c_float(g.softmax_scale),
                                           out.data_ptr(), lse.data_ptr(),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_on_two_calls(lib):
    nq, n = 16, 4096   # 16 rows: several splits per row, so the static scratch is used
    for call, seed in enumerate((101, 102)):
        g = inputs.make_decode_inputs(f"noalloc_{seed}", [n] * nq, T_max=n, seed=seed).to("cuda")
        idx = random_index_lists(nq, n, g.k, seed).cuda()
        dims = api.dims_of(g)
        ws = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
        ref_out, ref_lse = api.alloc_outputs(g)
        api.sparse_mla_attn(dims, g.q, g.kv, idx, g.q_seq, g.q_len, g.softmax_scale, ref_out, ref_lse, ws)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert call_noalloc(lib, dims, g, idx, out, lse) == _lib.DSA_OK
        torch.cuda.synchronize()
        assert api.get_device_status(ws) == 0
        check_attention(out.float().cpu().numpy(), ref_out.float().cpu().numpy(), lse.cpu().numpy(),
                        ref_lse.cpu().numpy())
        assert torch.isfinite(out.float()).all(), f"call {call}: non-finite output"


def test_noalloc_refuses_requests_beyond_its_scratch(lib):
    sms = torch.cuda.get_device_properties(0).multi_processor_count

    def planned_splits(q, k=2048, tile=64):
        # the library's plan: sms // (2 nq) splits clamped to [1, 16], rows per
        # split rounded up to whole 64-row tiles, then the splits those rows need
        s = max(1, min(16, sms // (2 * q)))
        rows = -(-(-(-k // s)) // tile) * tile
        return -(-k // rows)

    # up to 8 splits run as a cluster and merge on chip; more write partials to the scratch
    nq = next(q for q in range(1, 75) if planned_splits(q) > 8 and planned_splits(q) * q > 64)
    g = inputs.make_decode_inputs("noalloc_big", [2048] * nq, T_max=2048, seed=7).to("cuda")
    idx = random_index_lists(nq, 2048, g.k, 7).cuda()
    out, lse = api.alloc_outputs(g)
    assert call_noalloc(lib, api.dims_of(g), g, idx, out, lse) == _lib.DSA_ERR_UNSUPPORTED
