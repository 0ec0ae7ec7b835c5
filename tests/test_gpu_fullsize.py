"""CUDA path vs the CPU oracle at the full workload sizes, on sampled outputs.

Each workload is generated on the GPU from its seed and run through the same
entry point, dimensions and workspace plan as bench.py (api.run_decode /
api.prefill).  The oracle cannot redo whole 128K-1M token batches in a test,
so it checks outputs it can compute one by one, from compact CPU copies of
exactly the data the GPU used:

* indexer scores: whole rows, or windows of a row (a score depends only on its
  own token), within the score tolerance;
* top-k: the oracle's selection on the GPU's own score rows, bit-exact, for
  every row of the batch (prefill: sampled rows);
* selected sets end to end: the GPU's selection against the oracle's selection
  on oracle scores, differing only within 1e-3 relative of the threshold;
* attention: the oracle on the rows the GPU selected (compact copies of those
  latent rows), within the bf16 attention tolerance.
"""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_indexer_b200 import _lib, api, inputs
from tests.tolerances import check_attention, check_scores, check_sets

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return _lib.load()


def _meta(g, B, T_max, Nq):
    return SimpleNamespace(B=B, Nq=Nq, H_I=g.H_I, d_I=g.d_I, H=g.H, k=g.k, T_max=T_max, idx_dtype=g.idx_dtype,
                           kv_dtype=g.kv_dtype, softmax_scale=g.softmax_scale)


def oracle_scores_window(g, t, s0, W):
    """Oracle indexer scores of query row t over cached positions [s0, s0 + W)."""
    b = int(g.q_seq[t])
    n = min(W, int(g.q_len[t]) - s0)
    m = _meta(g, 1, W, 1)
    sc = oracle.indexer(m, q_I=g.q_I[t:t + 1].cpu(), q_scale=None if g.q_scale is None else g.q_scale[t:t + 1].cpu(),
                        w=g.w[t:t + 1].cpu(), k_I=g.k_I[b:b + 1, s0:s0 + W].cpu(),
                        k_scale=None if g.k_scale is None else g.k_scale[b:b + 1, s0:s0 + W].cpu(),
                        q_seq=np.zeros(1, np.int32), q_len=np.array([n], np.int32), ld=W)
    return sc[0, :n]


def oracle_attention_on(g, t, idx_row):
    """Oracle attention of query row t over the positions idx_row (the GPU's selection)."""
    b = int(g.q_seq[t])
    sel = idx_row[idx_row >= 0]
    kv_c = g.kv[b][torch.from_numpy(sel.astype(np.int64)).to(g.kv.device)].cpu()[None]
    m = _meta(g, 1, max(1, len(sel)), 1)
    local = np.full((1, g.k), -1, np.int32)
    local[0, :len(sel)] = np.arange(len(sel), dtype=np.int32)
    out, lse = oracle.sparse_attn(m, local, q=g.q[t:t + 1].cpu(), kv=kv_c, q_seq=np.zeros(1, np.int32),
                                  q_len=np.array([len(sel)], np.int32))
    return out[0], lse[0]


def run_decode_like_bench(g):
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE)
    out, lse = api.alloc_outputs(g)
    scores = torch.empty((g.Nq, dims.ld_scores), dtype=torch.float32, device="cuda")
    idx = torch.empty((g.Nq, g.k), dtype=torch.int32, device="cuda")
    api.run_decode(g, ws=ws, out=out, lse=lse, dims=dims, scores_out=scores, idx_out=idx)
    torch.cuda.synchronize()
    return scores, idx, out, lse, api.get_device_status(ws)


def check_decode_workload(g, full_rows, window_rows, window=8192):
    scores, idx, out, lse, status = run_decode_like_bench(g)
    assert status == 0
    q_len = g.q_len.cpu().numpy()
    g_scores = scores.cpu().numpy()
    g_idx = idx.cpu().numpy()
    g_out = out.float().cpu().numpy()
    g_lse = lse.cpu().numpy()
    # top-k on the GPU's own score rows, every row, bit-exact
    o_idx = oracle.topk(g_scores.astype(np.float64), q_len, g.k)
    bad = [t for t in range(g.Nq) if not np.array_equal(o_idx[t], g_idx[t])]
    assert not bad, f"top-k differs from the oracle on identical scores in rows {bad}"
    # whole rows: scores, end-to-end sets, attention
    for t in full_rows:
        n = int(q_len[t])
        sc_o = oracle_scores_window(g, t, 0, n)
        check_scores(g_scores[t:t + 1, :n], sc_o[None], [n])
        o_sel = oracle.topk(sc_o[None], np.array([n], np.int32), g.k)
        check_sets(g_idx[t:t + 1], o_sel, sc_o[None], [n], g.k)
        o_out, o_lse = oracle_attention_on(g, t, g_idx[t])
        check_attention(g_out[t:t + 1], o_out[None], g_lse[t:t + 1], o_lse[None])
    # windows of long rows: scores at the start, middle and end of the row
    for t in window_rows:
        n = int(q_len[t])
        for s0 in (0, max(0, n // 2 - window // 2), max(0, n - window)):
            sc_o = oracle_scores_window(g, t, s0, window)
            w = len(sc_o)
            check_scores(g_scores[t:t + 1, s0:s0 + w], sc_o[None], [w])
        o_out, o_lse = oracle_attention_on(g, t, g_idx[t])
        check_attention(g_out[t:t + 1], o_out[None], g_lse[t:t + 1], o_lse[None])


def test_long_decode_16x128k_full_size(lib):
    g = inputs.long_decode(device="cuda")
    check_decode_workload(g, full_rows=[0, 11], window_rows=[5])


def test_long_decode_fp8_latent_full_size(lib):
    # the long decode with its latent cache in 656-byte FP8 entries
    g = inputs.with_fp8_latent(inputs.long_decode(device="cuda"))
    check_decode_workload(g, full_rows=[3], window_rows=[])


def test_decode_batch32_full_size(lib):
    g = inputs.decode32(device="cuda")
    check_decode_workload(g, full_rows=[0, 17, 31], window_rows=[])


def test_million_context_decode_full_size(lib):
    g = inputs.million(device="cuda")
    lens = g.q_len.cpu().numpy()
    ragged = int(np.argmin(lens))              # the shortest ragged row is redone whole
    check_decode_workload(g, full_rows=[ragged], window_rows=[0, 1], window=16384)


def test_prefill_64k_full_size(lib):
    g = inputs.prefill(device="cuda")
    L = g.Nq
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_PREFILL)
    out, lse = api.alloc_outputs(g)
    idx = torch.empty((L, g.k), dtype=torch.int32, device="cuda")
    api.prefill(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale,
                out, lse, ws, idx_out=idx)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    rows = [0, 1, 2046, 2047, 2048, 2049, 33333, L - 1]
    g_idx = idx[rows].cpu().numpy()
    g_out = out[rows].float().cpu().numpy()
    g_lse = lse[rows].cpu().numpy()
    for i, t in enumerate(rows):
        n = int(g.q_len[t])
        assert n == t + 1, "prefill rows are causal: row t sees positions 0..t"
        if n <= g.k:
            # every position <= t is selected
            assert np.array_equal(g_idx[i][:n], np.arange(n)) and np.all(g_idx[i][n:] == -1)
        else:
            sc_o = oracle_scores_window(g, t, 0, n)
            o_sel = oracle.topk(sc_o[None], np.array([n], np.int32), g.k)
            check_sets(g_idx[i:i + 1], o_sel, sc_o[None], [n], g.k)
        o_out, o_lse = oracle_attention_on(g, t, g_idx[i])
        check_attention(g_out[i:i + 1], o_out[None], g_lse[i:i + 1], o_lse[None])


def test_dense_attention_long_decode_sampled_rows(lib):
    # dense attention over all 131,072 cached tokens of the long decode, launched as bench.py's
    # dense line does; the oracle redoes two rows whole
    g = inputs.long_decode(device="cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_DENSE_MLA)
    out, lse = api.alloc_outputs(g)
    api.dense_mla_attn(dims, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale, out, lse, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    for t in (0, 9):
        n = int(g.q_len[t])
        b = int(g.q_seq[t])
        sub = SimpleNamespace(q=g.q[t:t + 1].cpu(), kv=g.kv[b:b + 1, :n].cpu(), q_seq=np.zeros(1, np.int32),
                              q_len=np.array([n], np.int32), H=g.H, T_max=n, B=1, kv_dtype=g.kv_dtype,
                              softmax_scale=g.softmax_scale)
        o_out, o_lse = oracle.dense_attn(sub)
        check_attention(out[t:t + 1].float().cpu().numpy(), o_out, lse[t:t + 1].cpu().numpy(), o_lse)
