"""Host-side input preparation (no GPU): the paged layout is pure data movement,
row subsets of the prefill workload equal the same rows of the full draw, and
the seeded generators are reproducible."""
import torch

from sparse_long_context_indexer_b200 import inputs


def test_paged_layout_gathers_back_to_the_contiguous_cache():
    inp = inputs.make_decode_inputs("paged_cpu", [700, 129, 64, 1], T_max=768, seed=5)
    bs = 64
    k_pool, s_pool, kv_pool, table = inputs.paged_layout(inp, bs, seed=1, spare_blocks=3)
    B, mb = table.shape
    assert (B, mb) == (4, 768 // bs)
    used = table[table >= 0]
    assert used.unique().numel() == used.numel(), "a pool block serves one (sequence, block) pair"
    assert int(used.max()) < k_pool.shape[0]
    for b in range(B):
        n = int(inp.q_len[inp.q_seq == b].max())
        nblk = (n + bs - 1) // bs
        assert bool((table[b, :nblk] >= 0).all()) and bool((table[b, nblk:] == -1).all())
        for s in range(nblk * bs):
            pb, off = int(table[b, s // bs]), s % bs
            assert torch.equal(k_pool[pb, off], inp.k_I[b, s])
            assert torch.equal(kv_pool[pb, off], inp.kv[b, s])
            assert float(s_pool[pb, off]) == float(inp.k_scale[b, s])


def test_prefill_row_subsets_equal_the_full_draw():
    L = 300
    full = inputs.make_prefill_inputs("subset_cpu", L, seed=8)
    rows = [0, 1, 77, 150, 299]
    sub = inputs.make_prefill_inputs("subset_cpu", L, seed=8, rows=rows)
    r = torch.tensor(rows)
    for name in ("q_I", "q_scale", "w", "q", "q_len", "q_seq"):
        assert torch.equal(getattr(sub, name), getattr(full, name)[r]), name
    for name in ("k_I", "k_scale", "kv"):
        assert torch.equal(getattr(sub, name), getattr(full, name)), name
    assert full.q_len.tolist() == list(range(1, L + 1))


def test_decode_inputs_are_seeded():
    a = inputs.make_decode_inputs("seeded", [500, 300], T_max=512, seed=11)
    b = inputs.make_decode_inputs("seeded", [500, 300], T_max=512, seed=11)
    c = inputs.make_decode_inputs("seeded", [500, 300], T_max=512, seed=12)
    assert torch.equal(a.k_I, b.k_I) and torch.equal(a.kv, b.kv) and torch.equal(a.q, b.q)
    assert not torch.equal(a.kv, c.kv)
