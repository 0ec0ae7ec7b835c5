"""CUDA path vs the CPU oracle, stage by stage and end to end (needs a B200).

Inputs come from the seeded generator only; no oracle input is ever taken from
the CUDA path.  Top-k is checked bit-exact on identical score buffers drawn by
the generator; attention is checked on index lists chosen by the oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_indexer_b200 import _lib, api, inputs
from tests.tolerances import check_attention, check_scores, check_sets

pytestmark = pytest.mark.gpu

SMALL_LENS = [4097, 2500, 777, 2048, 2049, 129, 1]


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return _lib.load()


def small_decode(seed=11, lens=SMALL_LENS, k=2048, fp8=True, H_I=64, d_I=64, H=128):
    return inputs.make_decode_inputs(f"small_{seed}", lens, H_I=H_I, d_I=d_I, H=H, k=k, fp8=fp8,
                                     T_max=max(128, (max(lens) + 127) // 128 * 128), anchor_frac=0.01, seed=seed)


def np_scores(t):
    return t.detach().cpu().numpy()


# ------------------------------------------------------------------ top-k

def random_scores(rows, ld, seed, ties=True):
    g = torch.Generator().manual_seed(seed)
    sc = torch.randn((rows, ld), generator=g)
    if ties:
        sc = torch.round(sc * 16) / 16          # many exact ties
        z = torch.rand((rows, ld), generator=g) < 0.05
        sc[z] = 0.0
        negz = torch.rand((rows, ld), generator=g) < 0.5
        sc[z & negz] = -0.0
    return sc.float()


@pytest.mark.parametrize("lens,k", [
    ([0, 1, 100, 2047, 2048, 2049, 5000, 40000, 131072], 2048),
    ([131072] * 16, 2048),
    ([60000] * 64, 2048),
    ([30000] * 300, 2048),
    ([4096], 256),
    ([1048576, 300000], 2048),
    ([9000, 9001, 9002, 9003], 1),
    ([50000], 2000),
])
def test_topk_bit_exact_on_identical_scores(lib, lens, k):
    ld = (max(lens) + 3) // 4 * 4
    sc = random_scores(len(lens), ld, seed=len(lens) + k, ties=True)
    q_len = torch.tensor(lens, dtype=torch.int32)
    want = oracle.topk(sc.double().numpy(), q_len.numpy(), k)
    dims = api.Dims(B=1, Nq=len(lens), H_I=64, d_I=64, H=128, k=k, T_max=ld, idx_dtype=2, kv_dtype=1, ld_scores=ld)
    ws = api.make_workspace(dims, _lib.DSA_OP_TOPK)
    idx = torch.full((len(lens), k), -7, dtype=torch.int32, device="cuda")
    api.topk(dims, sc.cuda(), q_len.cuda(), idx, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    got = idx.cpu().numpy()
    for t in range(len(lens)):
        assert np.array_equal(got[t], want[t]), f"row {t} (n={lens[t]}): first diff at {np.argmax(got[t] != want[t])}"


def anchored_scores(seed):
    """Long rows for the first histogram's floor (2^-8 of the row's largest score) and its
    full-range rebuild: (scores [4, 131072], lengths).
      row 0 (131,072 keys) and row 1 (40,000 keys): N(0,1) scores plus a few anchors about
        1e4 times larger, so almost every key lies below the floor and the k-th largest too;
      row 2: exactly k-1 keys above the floor (the k-th largest sits just below it);
      row 3: exactly k keys above the floor (the k-th largest is the lowest of them)."""
    k, ld = 2048, 131072
    g = torch.Generator().manual_seed(seed)
    sc = torch.randn((4, ld), generator=g)
    for t, n_anchor in ((0, 24), (1, 7)):
        pos = torch.randperm(131072 if t == 0 else 40000, generator=g)[:n_anchor]
        sc[t, pos] = 1e4 * (1 + torch.rand(n_anchor, generator=g))
    for t, above in ((2, k - 1), (3, k)):
        row = torch.clamp(torch.randn(ld, generator=g), -3.5, 3.5)      # all below 1000 / 256
        pos = torch.randperm(ld, generator=g)[:above]
        row[pos] = 10 + 990 * torch.rand(above, generator=g)             # above the floor
        row[pos[0]] = 1000.0                                             # the row's largest
        row[pos[1:4]] = 500.0                                            # a few ties above it
        sc[t] = row
    sc[:, 5:9] = sc[:, 5:6]                                              # ties in the tail
    return sc.float(), [131072, 40000, 131072, 131072]


def test_topk_bit_exact_on_long_rows_with_anchors_and_floor_rebuild(lib):
    k = 2048
    sc, lens = anchored_scores(77)
    ld = sc.shape[1]
    q_len = torch.tensor(lens, dtype=torch.int32)
    want = oracle.topk(sc.double().numpy(), q_len.numpy(), k)
    # the rows really exercise the floor: their k-th largest score lies at or below max / 256
    for t in (0, 1, 2):
        row = np.sort(sc[t, :lens[t]].numpy())[::-1]
        assert row[k - 1] <= row[0] / 256
    dims = api.Dims(B=1, Nq=len(lens), H_I=64, d_I=64, H=128, k=k, T_max=ld, idx_dtype=2, kv_dtype=1, ld_scores=ld)
    ws = api.make_workspace(dims, _lib.DSA_OP_TOPK)
    idx = torch.full((len(lens), k), -7, dtype=torch.int32, device="cuda")
    api.topk(dims, sc.cuda(), q_len.cuda(), idx, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    got = idx.cpu().numpy()
    for t in range(len(lens)):
        assert np.array_equal(got[t], want[t]), f"row {t} (n={lens[t]}): first diff at {np.argmax(got[t] != want[t])}"


def test_topk_all_equal_scores_take_lowest_positions(lib):
    n, k = 70000, 2048
    sc = torch.full((2, n), 0.25)
    sc[1, ::3] = -0.0
    sc[1, 1::3] = 0.0
    sc[1, 2::3] = -1.0
    dims = api.Dims(B=1, Nq=2, H_I=64, d_I=64, H=128, k=k, T_max=n, idx_dtype=2, kv_dtype=1, ld_scores=n)
    ws = api.make_workspace(dims, _lib.DSA_OP_TOPK)
    idx = torch.empty((2, k), dtype=torch.int32, device="cuda")
    api.topk(dims, sc.cuda(), torch.tensor([n, n], dtype=torch.int32, device="cuda"), idx, ws)
    got = idx.cpu().numpy()
    assert np.array_equal(got[0], np.arange(k))
    want = oracle.topk(sc.double().numpy(), [n, n], k)
    assert np.array_equal(got[1], want[1])


# ------------------------------------------------------------------ indexer

@pytest.mark.parametrize("d_I", [64, 128])
def test_indexer_fp8_matches_oracle(lib, d_I):
    inp = small_decode(seed=5 + d_I, d_I=d_I)
    ora = oracle.indexer(inp, ld=inp.T_max)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_INDEXER)
    scores = torch.full((g.Nq, dims.ld_scores), float("nan"), device="cuda")
    api.indexer_scores(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q_seq, g.q_len, scores, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    got = np_scores(scores)
    check_scores(got, ora, inp.q_len.numpy())
    for t, n in enumerate(inp.q_len.tolist()):   # entries past q_len untouched
        assert np.all(np.isnan(got[t, n:]))


def test_indexer_f32_tiny_matches_oracle(lib):
    inp = inputs.tiny()
    ora = oracle.indexer(inp, ld=inp.T_max)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    scores = torch.empty((1, dims.ld_scores), device="cuda")
    api.indexer_scores(dims, g.q_I, None, g.w, g.k_I, None, g.q_seq, g.q_len, scores)
    check_scores(np_scores(scores), ora, inp.q_len.numpy())


# ------------------------------------------------------------------ sparse attention on oracle-chosen rows

@pytest.mark.parametrize("lens", [SMALL_LENS, [4096] * 16, [3000] * 40, [2100] * 3])
def test_sparse_mla_matches_oracle_on_same_indices(lib, lens):
    inp = small_decode(seed=21 + len(lens), lens=lens)
    sc = oracle.indexer(inp, ld=inp.T_max)
    idx = oracle.topk(sc, inp.q_len.numpy(), inp.k)
    o_out, o_lse = oracle.sparse_attn(inp, idx)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
    out, lse = api.alloc_outputs(g)
    api.sparse_mla_attn(dims, g.q, g.kv, torch.from_numpy(idx).cuda(), g.q_seq, g.q_len, g.softmax_scale, out, lse, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    check_attention(out.float().cpu().numpy(), o_out, lse.cpu().numpy(), o_lse)


def test_sparse_mla_random_index_sets_and_padding(lib):
    inp = small_decode(seed=31, lens=[5000, 5000, 300, 0], k=2048)
    rng = np.random.default_rng(0)
    idx = np.full((4, 2048), -1, np.int32)
    idx[0] = np.sort(rng.choice(5000, 2048, replace=False))
    idx[1, :1000] = np.sort(rng.choice(5000, 1000, replace=False))   # ragged tail of -1
    idx[2, :300] = np.arange(300)
    o_out, o_lse = oracle.sparse_attn(inp, idx)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
    out, lse = api.alloc_outputs(g)
    api.sparse_mla_attn(dims, g.q, g.kv, torch.from_numpy(idx).cuda(), g.q_seq, g.q_len, g.softmax_scale, out, lse, ws)
    torch.cuda.synchronize()
    check_attention(out.float().cpu().numpy(), o_out, lse.cpu().numpy(), o_lse)
    assert torch.all(out[3] == 0) and torch.all(torch.isneginf(lse[3]))


def test_sparse_mla_f32_tiny(lib):
    inp = inputs.tiny()
    sc = oracle.indexer(inp, ld=inp.T_max)
    idx = oracle.topk(sc, inp.q_len.numpy(), inp.k)
    o_out, o_lse = oracle.sparse_attn(inp, idx)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
    out, lse = api.alloc_outputs(g)
    api.sparse_mla_attn(dims, g.q, g.kv, torch.from_numpy(idx).cuda(), g.q_seq, g.q_len, g.softmax_scale, out, lse, ws)
    torch.cuda.synchronize()
    check_attention(out.cpu().numpy(), o_out, lse.cpu().numpy(), o_lse)


# ------------------------------------------------------------------ end to end

def run_decode_gpu(inp_gpu):
    dims = api.dims_of(inp_gpu)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE)
    scores = torch.empty((inp_gpu.Nq, dims.ld_scores), device="cuda")
    idx = torch.empty((inp_gpu.Nq, inp_gpu.k), dtype=torch.int32, device="cuda")
    out, lse = api.run_decode(inp_gpu, ws=ws, scores_out=scores, idx_out=idx, dims=dims)
    torch.cuda.synchronize()
    status = api.get_device_status(ws)
    return scores, idx, out, lse, status


@pytest.mark.parametrize("which", ["small", "tiny", "k512", "k1024", "dI128"])
def test_decode_step_end_to_end(lib, which):
    # budgets 512 / 1024 and d_I = 128 are the width variants of kgptalkie "How Does the Selector
    # Pick 1,024?" (V4 budgets) and its configuration table (d_I = 128)
    inp = {"small": lambda: small_decode(seed=41), "tiny": inputs.tiny,
           "k512": lambda: small_decode(seed=42, k=512), "k1024": lambda: small_decode(seed=43, k=1024),
           "dI128": lambda: small_decode(seed=44, d_I=128)}[which]()
    sc_o, idx_o, out_o, lse_o = oracle.decode(inp)
    scores, idx, out, lse, status = run_decode_gpu(inp.to("cuda"))
    assert status == 0
    check_scores(np_scores(scores), sc_o, inp.q_len.numpy())
    same, total = check_sets(idx.cpu().numpy(), idx_o, sc_o, inp.q_len.numpy(), inp.k)
    g_idx = idx.cpu().numpy()
    rows = [t for t in range(inp.Nq) if np.array_equal(g_idx[t], idx_o[t])]
    assert len(rows) >= max(1, total - 1), f"only {same}/{total} rows selected identical sets"
    check_attention(out.float().cpu().numpy(), out_o, lse.cpu().numpy(), lse_o, rows=rows)


def test_short_rows_skip_the_indexer_with_the_same_outputs(lib):
    # rows with q_len <= k: the decode step without scores_out skips their indexer work; the
    # selection (every position) and the attention must not change
    lens = [2048, 700, 1, 2049, 5000]
    inp = small_decode(seed=45, lens=lens)
    sc_o, idx_o, out_o, lse_o = oracle.decode(inp)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE)
    idx_a = torch.empty((len(lens), g.k), dtype=torch.int32, device="cuda")
    idx_b = torch.empty_like(idx_a)
    scores = torch.empty((len(lens), dims.ld_scores), device="cuda")
    out_a, lse_a = api.run_decode(g, ws=ws, idx_out=idx_a, dims=dims)                    # skips short rows
    out_b, lse_b = api.run_decode(g, ws=ws, idx_out=idx_b, scores_out=scores, dims=dims)  # scores every row
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    assert torch.equal(idx_a, idx_b)
    for t, n in enumerate(lens):
        if n <= g.k:
            assert torch.equal(idx_a[t, :n].cpu(), torch.arange(n, dtype=torch.int32))
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)
    # the dispatched step against the oracle (the short rows attend over every position)
    g_idx = idx_a.cpu().numpy()
    check_sets(g_idx, idx_o, sc_o, inp.q_len.numpy(), inp.k)
    rows = [t for t in range(len(lens)) if np.array_equal(g_idx[t], idx_o[t])]
    assert all(t in rows for t, n in enumerate(lens) if n <= g.k)
    assert len(rows) >= len(lens) - 1
    check_attention(out_a.float().cpu().numpy(), out_o, lse_a.cpu().numpy(), lse_o, rows=rows)


SHORT_CACHE_CASES = {
    # name: (row lengths, k, T_max, FP8 latent, paged block size)
    "partials": ([2048, 1500, 700, 64, 1, 0], 2048, 2048, False, 0),   # 11 splits: partials + merge kernel
    "cluster": ([(37 * t) % 2048 + 1 for t in range(20)], 2048, 2048, False, 0),  # 3 splits: on-chip merge
    "fp8_latent": ([2048, 999, 2, 0], 2048, 2048, True, 0),
    "paged": ([2048, 1300, 65, 1], 2048, 2048, False, 64),
    "k1000": ([1000, 999, 513, 1], 1000, 1000, False, 0),              # T_max not a whole 64-row tile
}


@pytest.mark.parametrize("case", list(SHORT_CACHE_CASES))
def test_short_cache_decode_is_dense_attention_and_matches_oracle(lib, case):
    # A cache of at most k positions: every row selects all of its positions (the smaller of the
    # budget and the number of tokens, kgptalkie "How Does the Selector Pick 1,024?"), and the
    # decode step runs the attention's dense form, with the indexer and the top-k only for the
    # outputs the caller asks for.  The outputs must equal the dense entry's bit for bit and the
    # oracle's decode within the attention tolerance; the positions asked for are 0..n-1.
    lens, k, T_max, fp8_latent, block = SHORT_CACHE_CASES[case]
    inp = inputs.make_decode_inputs(f"short_cache_{case}", lens, k=k, T_max=T_max, anchor_frac=0.01,
                                    seed=90 + len(case))
    if fp8_latent:
        inp = inputs.with_fp8_latent(inp)
    sc_o, idx_o, out_o, lse_o = oracle.decode(inp)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE)
    if block:
        k_pool, s_pool, kv_pool, table = inputs.paged_layout(g, block, seed=block)
        cache = api.PagedCache(k_pool, s_pool, kv_pool, table, block)

    def step(idx_out=None, scores_out=None):
        if not block:
            return api.run_decode(g, ws=ws, idx_out=idx_out, scores_out=scores_out, dims=dims)
        out, lse = api.alloc_outputs(g)
        api.decode_step_paged(dims, g.q_I, g.q_scale, g.w, cache, g.q, g.q_seq, g.q_len, g.softmax_scale, out, lse,
                              ws, scores_out=scores_out, idx_out=idx_out)
        return out, lse

    out_a, lse_a = step()                                                  # attention alone
    idx_b = torch.full((len(lens), k), 7, dtype=torch.int32, device="cuda")
    out_b, lse_b = step(idx_out=idx_b)                                     # + the top-k's positions
    idx_c = torch.full_like(idx_b, 7)
    sc_c = torch.empty((len(lens), dims.ld_scores), device="cuda")
    out_c, lse_c = step(idx_out=idx_c, scores_out=sc_c)                    # + the indexer's scores
    ws_d = api.make_workspace(dims, _lib.DSA_OP_DENSE_MLA)
    out_d, lse_d = api.alloc_outputs(g)
    if not block:
        api.dense_mla_attn(dims, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale, out_d, lse_d, ws_d)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0 and api.get_device_status(ws_d) == 0
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)
    assert torch.equal(out_a, out_c) and torch.equal(lse_a, lse_c)
    if not block:
        assert torch.equal(out_a, out_d) and torch.equal(lse_a, lse_d)
    want = np.full((len(lens), k), -1, np.int32)
    for t, n in enumerate(lens):
        want[t, :n] = np.arange(n)
    assert np.array_equal(idx_o, want)  # the oracle selects every position too
    assert np.array_equal(idx_b.cpu().numpy(), want) and np.array_equal(idx_c.cpu().numpy(), want)
    check_scores(np_scores(sc_c), sc_o, inp.q_len.numpy())
    check_attention(out_a.float().cpu().numpy(), out_o, lse_a.cpu().numpy(), lse_o)
    for t, n in enumerate(lens):
        if n == 0:
            assert torch.all(out_a[t] == 0) and torch.all(torch.isneginf(lse_a[t]))


@pytest.mark.parametrize("block_size", [64, 256])
def test_paged_decode_matches_oracle_and_contiguous(lib, block_size):
    # the same cache in blocks of a pool, in a random physical order, read through a block
    # table (kgptalkie "How Does the Selector Pick 1,024?": the selection is an address list
    # into the paged KV cache).  The paged outputs are checked against the oracle on the same
    # logical cache, and must equal the contiguous path's bit for bit.
    lens = [4097, 2500, 777, 2048, 2049, 129, 1]
    inp = inputs.make_decode_inputs("paged", lens, T_max=4352, anchor_frac=0.01, seed=71)
    sc_o, idx_o, out_o, lse_o = oracle.decode(inp)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE)
    idx_c = torch.empty((len(lens), g.k), dtype=torch.int32, device="cuda")
    sc_c = torch.empty((len(lens), dims.ld_scores), device="cuda")
    out_c, lse_c = api.run_decode(g, ws=ws, idx_out=idx_c, scores_out=sc_c, dims=dims)
    k_pool, s_pool, kv_pool, table = inputs.paged_layout(g, block_size, seed=block_size)
    cache = api.PagedCache(k_pool, s_pool, kv_pool, table, block_size)
    out_p, lse_p = api.alloc_outputs(g)
    idx_p = torch.empty_like(idx_c)
    sc_p = torch.full_like(sc_c, float("nan"))
    api.decode_step_paged(dims, g.q_I, g.q_scale, g.w, cache, g.q, g.q_seq, g.q_len, g.softmax_scale, out_p, lse_p, ws,
                          scores_out=sc_p, idx_out=idx_p)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    # against the oracle
    check_scores(np_scores(sc_p), sc_o, inp.q_len.numpy())
    g_idx = idx_p.cpu().numpy()
    same, total = check_sets(g_idx, idx_o, sc_o, inp.q_len.numpy(), inp.k)
    rows = [t for t in range(inp.Nq) if np.array_equal(g_idx[t], idx_o[t])]
    assert len(rows) >= max(1, total - 1), f"only {same}/{total} rows selected identical sets"
    check_attention(out_p.float().cpu().numpy(), out_o, lse_p.cpu().numpy(), lse_o, rows=rows)
    # and against the contiguous path
    for t, n in enumerate(lens):
        assert torch.equal(sc_p[t, :n], sc_c[t, :n]), f"row {t}: paged scores differ"
    assert torch.equal(idx_p, idx_c)
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)


def test_fp8_latent_attention_matches_oracle(lib):
    # the 656-byte FP8 latent entries, dequantised by the gather; random selections with -1
    # tails, an empty row
    inp = inputs.with_fp8_latent(small_decode(seed=81, lens=[5000, 5000, 300, 0], k=2048))
    rng = np.random.default_rng(3)
    idx = np.full((4, 2048), -1, np.int32)
    idx[0] = np.sort(rng.choice(5000, 2048, replace=False))
    idx[1, :1000] = np.sort(rng.choice(5000, 1000, replace=False))
    idx[2, :300] = np.arange(300)
    o_out, o_lse = oracle.sparse_attn(inp, idx)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
    out, lse = api.alloc_outputs(g)
    api.sparse_mla_attn(dims, g.q, g.kv, torch.from_numpy(idx).cuda(), g.q_seq, g.q_len, g.softmax_scale, out, lse, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    check_attention(out.float().cpu().numpy(), o_out, lse.cpu().numpy(), o_lse)
    assert torch.all(out[3] == 0) and torch.all(torch.isneginf(lse[3]))


def test_fp8_latent_decode_end_to_end(lib):
    inp = inputs.with_fp8_latent(small_decode(seed=82))
    sc_o, idx_o, out_o, lse_o = oracle.decode(inp)
    scores, idx, out, lse, status = run_decode_gpu(inp.to("cuda"))
    assert status == 0
    check_scores(np_scores(scores), sc_o, inp.q_len.numpy())
    same, total = check_sets(idx.cpu().numpy(), idx_o, sc_o, inp.q_len.numpy(), inp.k)
    g_idx = idx.cpu().numpy()
    rows = [t for t in range(inp.Nq) if np.array_equal(g_idx[t], idx_o[t])]
    assert len(rows) >= max(1, total - 1)
    check_attention(out.float().cpu().numpy(), out_o, lse.cpu().numpy(), lse_o, rows=rows)


def test_fp8_latent_dense_and_paged(lib):
    # the dense comparison and the paged cache read the same 656-byte entries
    lens = [3000, 2049, 64, 1]
    inp = inputs.with_fp8_latent(inputs.make_decode_inputs("fp8_paged", lens, T_max=3072, seed=83))
    out_o, lse_o = oracle.dense_attn(inp)
    sc_d, idx_d, out_dec, lse_dec = oracle.decode(inp)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws_d = api.make_workspace(dims, _lib.DSA_OP_DENSE_MLA)
    out, lse = api.alloc_outputs(g)
    api.dense_mla_attn(dims, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale, out, lse, ws_d)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE)
    idx_c = torch.empty((len(lens), g.k), dtype=torch.int32, device="cuda")
    out_c, lse_c = api.run_decode(g, ws=ws, idx_out=idx_c, dims=dims)
    k_pool, s_pool, kv_pool, table = inputs.paged_layout(g, 64, seed=5)
    cache = api.PagedCache(k_pool, s_pool, kv_pool, table, 64)
    out_p, lse_p = api.alloc_outputs(g)
    idx_p = torch.empty_like(idx_c)
    api.decode_step_paged(dims, g.q_I, g.q_scale, g.w, cache, g.q, g.q_seq, g.q_len, g.softmax_scale, out_p, lse_p,
                          ws, idx_out=idx_p)
    torch.cuda.synchronize()
    assert api.get_device_status(ws_d) == 0 and api.get_device_status(ws) == 0
    check_attention(out.float().cpu().numpy(), out_o, lse.cpu().numpy(), lse_o)
    # the paged decode against the oracle's decode of the same logical FP8 cache
    g_idx = idx_p.cpu().numpy()
    check_sets(g_idx, idx_d, sc_d, inp.q_len.numpy(), inp.k)
    rows = [t for t in range(len(lens)) if np.array_equal(g_idx[t], idx_d[t])]
    assert len(rows) >= len(lens) - 1
    check_attention(out_p.float().cpu().numpy(), out_dec, lse_p.cpu().numpy(), lse_dec, rows=rows)
    assert torch.equal(idx_p, idx_c) and torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)


@pytest.mark.parametrize("fp8_latent", [False, True])
def test_append_tokens_matches_the_input_quantisers(lib, fp8_latent):
    # kgptalkie "What Does the Whole Block Look Like?": the new token is compressed and written to
    # the cache.  The device's bytes must equal the input preparation's (torch's RNE e4m3 cast:
    # keys with one scale per token, the latent in four 128-value groups); a token at an
    # out-of-range position is skipped and reported.
    lens = [700, 300, 129]
    inp = inputs.make_decode_inputs("append", lens, T_max=768, seed=91)
    if fp8_latent:
        inp = inputs.with_fp8_latent(inp)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE)
    gen = torch.Generator().manual_seed(5)
    seq = torch.tensor([0, 1, 2, 1, 2], dtype=torch.int32)
    pos = torch.tensor([700, 10, 128, 767, 768], dtype=torch.int32)   # the last is out of range
    k_new = torch.randn((5, g.d_I), generator=gen) / 8
    k_new[2] = 0.0                                                   # all-zero key: scale 1
    kv_new = (torch.randn((5, 576), generator=gen) / 8).to(torch.bfloat16)
    # contiguous caches
    kv, k_I, k_scale = g.kv.clone(), g.k_I.clone(), g.k_scale.clone()
    api.append_tokens(dims, seq.cuda(), pos.cuda(), kv_new.cuda(), k_new.cuda(), kv, k_I, k_scale, ws=ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == _lib.DSA_ERR_LENGTH
    # the format definition, through the oracle's own e4m3 decoder: every written key value is
    # within half an e4m3 step of its fp32 input, and the scale is amax / 448 in fp32
    check_appended_against_format(k_I.cpu(), k_scale.cpu(), kv.cpu(), seq, pos, k_new, kv_new, fp8_latent)
    codes, scales = inputs.quantize_e4m3_per_row(k_new)
    want_kv = inputs.pack_fp8_latent(kv_new) if fp8_latent else kv_new
    for i in range(4):
        b, s_ = int(seq[i]), int(pos[i])
        assert torch.equal(k_I[b, s_].cpu(), codes[i]), f"token {i}: key codes"
        assert float(k_scale[b, s_]) == float(scales[i]), f"token {i}: key scale"
        assert torch.equal(kv[b, s_].cpu(), want_kv[i]), f"token {i}: latent entry"
    # everything else is untouched
    mask = torch.ones(kv.shape[:2], dtype=torch.bool)
    for i in range(4):
        mask[int(seq[i]), int(pos[i])] = False
    assert torch.equal(kv.cpu()[mask], g.kv.cpu()[mask]) and torch.equal(k_I.cpu()[mask], g.k_I.cpu()[mask])
    # the same appends into the paged form of the original cache
    k_pool, s_pool, kv_pool, table = inputs.paged_layout(g, 64, seed=2)
    full = table.clone()
    free = [p_ for p_ in range(kv_pool.shape[0]) if p_ not in set(table[table >= 0].tolist())]
    for b in range(3):                        # blocks for every position the appends may touch
        for j in range(full.shape[1]):
            if full[b, j] < 0:
                full[b, j] = free.pop()
    cache = api.PagedCache(k_pool, s_pool, kv_pool, full.cuda(), 64)
    api.append_tokens(dims, seq.cuda(), pos.cuda(), kv_new.cuda(), k_new.cuda(), cache=cache, ws=ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == _lib.DSA_ERR_LENGTH
    for i in range(4):
        b, s_ = int(seq[i]), int(pos[i])
        pr = int(full[b, s_ // 64]), s_ % 64
        assert torch.equal(k_pool[pr].cpu(), codes[i]) and float(s_pool[pr]) == float(scales[i])
        assert torch.equal(kv_pool[pr].cpu(), want_kv[i])


E4M3_MAX = 448.0


def e4m3_half_step_bound(ref, scale):
    """Largest error of one round-to-nearest e4m3 code times `scale` against `ref`: half a step,
    i.e. 2^-4 of |ref| in the normal range and 2^-10 of the scale in the subnormal range."""
    return np.maximum(2.0 ** -4 * np.abs(ref), 2.0 ** -10 * scale) * (1 + 1e-6)


def check_appended_against_format(k_I, k_scale, kv, seq, pos, k_new, kv_new, fp8_latent):
    """The appended token's stored bytes, decoded by the oracle, against the fp32/bf16 inputs."""
    table = np.array([oracle.e4m3_decode(c) for c in range(256)], dtype=np.float64)
    for i in range(4):
        b, s_ = int(seq[i]), int(pos[i])
        x = k_new[i].double().numpy()
        amax = np.float32(np.abs(k_new[i].numpy()).max())
        want_scale = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
        got_scale = np.float32(k_scale[b, s_])
        assert got_scale == want_scale, f"token {i}: key scale {got_scale} != amax/448 = {want_scale}"
        dec = table[k_I[b, s_].numpy()] * float(got_scale)
        assert np.all(np.abs(dec - x) <= e4m3_half_step_bound(x, float(got_scale))), f"token {i}: key codes"
        ref = kv_new[i].float().numpy().astype(np.float64)
        if fp8_latent:
            d = oracle.dequant_latent_fp8(kv[b, s_]).astype(np.float64)
            grp = np.abs(kv_new[i, :512].float().numpy()).reshape(4, 128).max(axis=1).astype(np.float32)
            want = np.where(grp > 0, grp / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
            got = kv[b, s_, 512:528].contiguous().view(torch.float32).numpy()
            assert np.array_equal(got, want), f"token {i}: latent group scales"
            bound = e4m3_half_step_bound(ref[:512], np.repeat(got.astype(np.float64), 128))
            assert np.all(np.abs(d[:512] - ref[:512]) <= bound), f"token {i}: latent codes"
            assert np.array_equal(d[512:], ref[512:]), f"token {i}: rope values"
        else:
            assert torch.equal(kv[b, s_], kv_new[i]), f"token {i}: latent row"


def test_prefill_matches_oracle(lib):
    L = 3000
    inp = inputs.make_prefill_inputs("prefill_small", L, seed=7)
    rows = np.r_[0:8, 1000:1004, 2040:2056, 2990:3000]
    sub = inputs.make_prefill_inputs("prefill_small", L, seed=7, rows=rows.tolist())
    sc_o, idx_o, out_o, lse_o = oracle.decode(sub)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_PREFILL)
    out, lse = api.alloc_outputs(g)
    idx = torch.empty((L, g.k), dtype=torch.int32, device="cuda")
    api.prefill(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale,
                out, lse, ws, idx_out=idx)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    g_idx = idx.cpu().numpy()[rows]
    check_sets(g_idx, idx_o, sc_o, sub.q_len.numpy(), sub.k)
    same = [i for i in range(len(rows)) if np.array_equal(g_idx[i], idx_o[i])]
    assert len(same) >= len(rows) - 2
    check_attention(out.float().cpu().numpy()[rows], out_o, lse.cpu().numpy()[rows], lse_o, rows=same)
    # rows t < k select every position <= t
    for i, t in enumerate(rows):
        if t + 1 <= g.k:
            assert np.array_equal(g_idx[i][: t + 1], np.arange(t + 1)) and np.all(g_idx[i][t + 1:] == -1)


def test_prefill_chunk_after_a_cached_context_matches_oracle(lib):
    # the last 1,200 rows of a 7,200-token prompt (a prefill chunk after 6,000 cached tokens):
    # rows hold 6,001..7,200 positions, far more than the chunk's own row count
    offset, L = 6000, 1200
    rows_all = list(range(offset, offset + L))
    inp = inputs.make_prefill_inputs("prefill_after_ctx", offset + L, seed=9, rows=rows_all)
    pick = np.r_[0:4, 597:601, 1196:1200]
    sub = inputs.make_prefill_inputs("prefill_after_ctx", offset + L, seed=9, rows=[rows_all[i] for i in pick])
    sc_o, idx_o, out_o, lse_o = oracle.decode(sub)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    assert dims.Nq == L and int(inp.q_len.min()) == offset + 1
    ws = api.make_workspace(dims, _lib.DSA_OP_PREFILL)
    out, lse = api.alloc_outputs(g)
    idx = torch.empty((L, g.k), dtype=torch.int32, device="cuda")
    api.prefill(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale,
                out, lse, ws, idx_out=idx)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    g_idx = idx.cpu().numpy()[pick]
    check_sets(g_idx, idx_o, sc_o, sub.q_len.numpy(), sub.k)
    same = [i for i in range(len(pick)) if np.array_equal(g_idx[i], idx_o[i])]
    assert len(same) >= len(pick) - 2
    check_attention(out.float().cpu().numpy()[pick], out_o, lse.cpu().numpy()[pick], lse_o, rows=same)


def oracle_scores_of_rows(inp, rows):
    """Oracle indexer scores of the given query rows (whole rows, ld = the longest)."""
    r = torch.as_tensor(list(rows), dtype=torch.long)
    return oracle.indexer(inp, q_I=inp.q_I[r], q_scale=inp.q_scale[r], w=inp.w[r], q_seq=inp.q_seq[r],
                          q_len=inp.q_len[r])


def test_prefill_indexer_scores_match_oracle(lib):
    # a prompt whose row count is not a multiple of four, several 128-token tiles and a ragged tail
    L = 1283
    inp = inputs.make_prefill_inputs("prefill_idx", L, seed=21)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_INDEXER)
    sc4 = torch.full((L, dims.ld_scores), float("nan"), dtype=torch.float32, device="cuda")
    sc1 = torch.full_like(sc4, float("nan"))
    api.prefill_indexer_scores(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q_seq, g.q_len, sc4, ws)
    api.indexer_scores(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q_seq, g.q_len, sc1, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    rows = np.r_[0:6, 127:131, 640:644, 1279:1283]
    sc_o = oracle_scores_of_rows(inp, rows)
    got4 = np_scores(sc4)[rows][:, :sc_o.shape[1]]
    q_len = inp.q_len.numpy()[rows]
    check_scores(got4, sc_o, q_len)
    got1 = np_scores(sc1)[rows][:, :sc_o.shape[1]]
    for i, n in enumerate(q_len):
        # the two entry points compute the same scores (the contraction and the epilogue are shared)
        np.testing.assert_allclose(got4[i, :n], got1[i, :n], rtol=1e-6, atol=1e-6 * np.abs(got1[i, :n]).max())


def test_prefill_indexer_flags_groups_that_mix_sequences(lib):
    # rows 0-2 belong to sequence 0 and rows 3-7 to sequence 1: the group of rows 0-3 mixes two
    # sequences (skipped and flagged), the group of rows 4-7 is computed
    lens = [300, 301, 302, 200, 201, 202, 203, 204]
    inp = inputs.make_decode_inputs("mixed", lens, T_max=384, seed=23)
    q_seq = torch.tensor([0, 0, 0, 1, 1, 1, 1, 1], dtype=torch.int32)
    inp.q_seq = q_seq
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_INDEXER)
    sc = torch.full((len(lens), dims.ld_scores), float("nan"), dtype=torch.float32, device="cuda")
    api.prefill_indexer_scores(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q_seq, g.q_len, sc, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == _lib.DSA_ERR_INVALID_ARG
    rows = [4, 5, 6, 7]
    sc_o = oracle_scores_of_rows(inp, rows)
    check_scores(np_scores(sc)[rows][:, :sc_o.shape[1]], sc_o, np.array(lens)[rows])
    assert torch.isnan(sc[:4]).all(), "the mixed group must be left untouched"


def test_dense_attention_matches_oracle(lib):
    # every position s < q_len[t]: ragged rows spanning several splits, a one-token row
    inp = small_decode(seed=61, lens=[4097, 2500, 777, 1, 2049, 129])
    out_o, lse_o = oracle.dense_attn(inp)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_DENSE_MLA)
    out, lse = api.alloc_outputs(g)
    api.dense_mla_attn(dims, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale, out, lse, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    check_attention(out.float().cpu().numpy(), out_o, lse.cpu().numpy(), lse_o)


def test_dense_equals_sparse_over_every_position(lib):
    # with a budget covering the whole row the sparse path selects every position: the two
    # entry points then compute the same attention
    lens = [2048, 1500, 64, 65]
    inp = small_decode(seed=62, lens=lens)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    idx = torch.full((len(lens), g.k), -1, dtype=torch.int32)
    for t, n in enumerate(lens):
        idx[t, :n] = torch.arange(n, dtype=torch.int32)
    ws_s = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
    ws_d = api.make_workspace(dims, _lib.DSA_OP_DENSE_MLA)
    out_s, lse_s = api.alloc_outputs(g)
    out_d, lse_d = api.alloc_outputs(g)
    api.sparse_mla_attn(dims, g.q, g.kv, idx.cuda(), g.q_seq, g.q_len, g.softmax_scale, out_s, lse_s, ws_s)
    api.dense_mla_attn(dims, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale, out_d, lse_d, ws_d)
    torch.cuda.synchronize()
    assert api.get_device_status(ws_s) == 0 and api.get_device_status(ws_d) == 0
    check_attention(out_d.float().cpu().numpy(), out_s.float().cpu().numpy(), lse_d.cpu().numpy(), lse_s.cpu().numpy())


# ------------------------------------------------------------------ device-side error reporting

def test_out_of_range_index_is_reported_and_masked(lib):
    inp = small_decode(seed=51, lens=[1000, 1000])
    idx = np.full((2, 2048), -1, np.int32)
    idx[0, :3] = [1, 5, 7]
    idx[1, :3] = [2, 999, 1000]        # 1000 >= q_len
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
    out, lse = api.alloc_outputs(g)
    api.sparse_mla_attn(dims, g.q, g.kv, torch.from_numpy(idx).cuda(), g.q_seq, g.q_len, g.softmax_scale, out, lse, ws)
    assert api.get_device_status(ws) == _lib.DSA_ERR_INDEX_OOB
    assert api.get_device_status(ws) == 0          # read clears it
    idx_ok = idx.copy()
    idx_ok[1, 2] = -1
    o_out, o_lse = oracle.sparse_attn(inp, idx_ok)
    check_attention(out.float().cpu().numpy(), o_out, lse.cpu().numpy(), o_lse)


def test_length_beyond_cache_is_reported(lib):
    inp = small_decode(seed=52, lens=[500, 600])
    g = inp.to("cuda")
    g.q_len = torch.tensor([500, g.T_max + 1], dtype=torch.int32, device="cuda")
    scores, idx, out, lse, status = run_decode_gpu(g)
    assert status == _lib.DSA_ERR_LENGTH


@pytest.mark.parametrize("lens", [[4096] * 16, [4096] * 2])
def test_production_attention_wait_times_out_and_context_survives(lib, lens):
    # the attention kernel itself (a cluster of 4 splits for 16 rows; 16 splits and the merge
    # kernel for 2 rows) with its first tile never signalled: the MMA warp's bounded wait runs
    # out after 50 ms, the kernel records DSA_ERR_TIMEOUT, drains and exits; afterwards the same
    # kernel on the same buffers matches the oracle
    inp = small_decode(seed=57, lens=lens)
    sc = oracle.indexer(inp, ld=inp.T_max)
    idx = oracle.topk(sc, inp.q_len.numpy(), inp.k)
    o_out, o_lse = oracle.sparse_attn(inp, idx)
    g = inp.to("cuda")
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_SPARSE_MLA)
    out, lse = api.alloc_outputs(g)
    idx_d = torch.from_numpy(idx).cuda()
    api.selftest_attention_stall(dims, g.q, g.kv, idx_d, g.q_seq, g.q_len, g.softmax_scale, out, lse, ws,
                                 timeout_us=50000)
    assert api.get_device_status(ws) == _lib.DSA_ERR_TIMEOUT
    out.zero_()
    api.sparse_mla_attn(dims, g.q, g.kv, idx_d, g.q_seq, g.q_len, g.softmax_scale, out, lse, ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == 0
    check_attention(out.float().cpu().numpy(), o_out, lse.cpu().numpy(), o_lse)


def test_bounded_wait_times_out_with_status(lib):
    dims = api.Dims(B=1, Nq=1, H_I=64, d_I=64, H=128, k=16, T_max=128, idx_dtype=2, kv_dtype=1, ld_scores=128)
    ws = api.make_workspace(dims, _lib.DSA_OP_TOPK)
    api.selftest_wait_timeout(ws, timeout_us=100000)
    assert api.get_device_status(ws) == _lib.DSA_ERR_TIMEOUT
    x = torch.ones(4, device="cuda") * 2       # the context is still usable
    assert float(x.sum()) == 8.0
