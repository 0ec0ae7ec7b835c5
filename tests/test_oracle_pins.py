"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these retype the oracle's own formulas.  Each pins the oracle to a
closed form, a library routine, a hand-worked or page-printed example, an
invariant, or brute force on tiny inputs, chosen so that a dropped ReLU, a
wrong sign, a transposed head/key index, a missing or doubled scale, a wrong
tie rule or a softmax over the wrong set fails at least one of them.
"""
import itertools
import json
import math
import os
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def ns_indexer(q_I, w, k_I, q_len, *, fp8=False, q_scale=None, k_scale=None):
    """Wrap raw indexer arrays (one query row per sequence) for the oracle."""
    q_I = np.ascontiguousarray(q_I)
    k_I = np.ascontiguousarray(k_I)
    Nq, H_I, d_I = q_I.shape
    B, T_max, _ = k_I.shape
    return SimpleNamespace(H_I=H_I, d_I=d_I, T_max=T_max, B=B, idx_dtype=oracle.FP8 if fp8 else oracle.F32,
                           q_I=q_I, w=np.ascontiguousarray(w), k_I=k_I, q_scale=q_scale, k_scale=k_scale,
                           q_seq=np.arange(Nq, dtype=np.int32) % B,
                           q_len=np.asarray(q_len, dtype=np.int32))


def ns_attn(q, kv, q_len, scale, q_seq=None):
    q = np.ascontiguousarray(q, dtype=np.float32)
    kv = np.ascontiguousarray(kv, dtype=np.float32)
    Nq, H, _ = q.shape
    B, T_max, _ = kv.shape
    return SimpleNamespace(H=H, T_max=T_max, B=B, kv_dtype=oracle.F32, q=q, kv=kv,
                           q_seq=np.zeros(Nq, np.int32) if q_seq is None else np.asarray(q_seq, np.int32),
                           q_len=np.asarray(q_len, np.int32), softmax_scale=scale)


# ---------------------------------------------------------------- FP8 / bf16 decoding

def test_e4m3_decode_matches_format_definition_points():
    # OCP FP8 e4m3fn: bias 7, 3 mantissa bits, max 448, no inf, S.1111.111 = NaN
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9          # smallest subnormal
    assert oracle.e4m3_decode(0x07) == 7 / 8 * 2.0 ** -6  # largest subnormal
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6          # smallest normal
    assert oracle.e4m3_decode(0x38) == 1.0
    assert oracle.e4m3_decode(0x3C) == 1.5
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))
    assert oracle.e4m3_decode(0x00) == 0.0 and math.copysign(1, oracle.e4m3_decode(0x80)) == -1.0
    for c in range(128):
        a, b = oracle.e4m3_decode(c), oracle.e4m3_decode(c | 0x80)
        assert (math.isnan(a) and math.isnan(b)) or a == -b


def test_e4m3_decode_exhaustive_against_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_decode(c) for c in range(256)])
    both_nan = np.isnan(ref) & np.isnan(mine)
    assert np.all(both_nan | (ref == mine))
    pos = mine[:127]
    assert np.all(np.diff(pos) > 0), "positive codes must decode monotonically"


def test_bf16_decode_against_torch():
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(4096, generator=g) * 1000).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().astype(np.uint16)
    mine = np.array([oracle.bf16_decode(int(b)) for b in bits])
    assert np.array_equal(mine, x.double().numpy())


# ---------------------------------------------------------------- indexer

def test_indexer_hand_worked_example():
    g = json.load(open(os.path.join(GOLD, "indexer_hand_example.json")))
    q = np.array(g["q"], np.float32)[None]
    k = np.array(g["k"], np.float32)[None]
    w = np.array(g["w"], np.float32)[None]
    sc = oracle.indexer(ns_indexer(q, w, k, [k.shape[1]]))
    np.testing.assert_array_equal(sc[0], np.array(g["scores"]))


def test_indexer_single_head_reduces_to_scaled_dot_sketch():
    """lizeman 'DeepSeek Sparse Attention', section 3 (sketch): scores = k_I q_I / sqrt(d_I).

    With one head, w = 1/sqrt(d_I) and every dot positive, the multi-head ReLU
    form must equal the sketch's scaled dot product, and its top-k must equal
    the sketch's topk.
    """
    rng = np.random.default_rng(3)
    d_I, n, k = 64, 300, 17
    q = rng.uniform(0.1, 1.0, (1, 1, d_I)).astype(np.float32)
    keys = rng.uniform(0.0, 1.0, (1, n, d_I)).astype(np.float32)
    w = np.full((1, 1), 1 / math.sqrt(d_I), np.float32)
    sc = oracle.indexer(ns_indexer(q, w, keys, [n]))
    ref = (keys[0].astype(np.float64) @ q[0, 0].astype(np.float64)) * np.float64(np.float32(1 / math.sqrt(d_I)))
    np.testing.assert_allclose(sc[0], ref, rtol=1e-12)
    top = oracle.topk(sc, [n], k)[0]
    sketch = np.sort(torch.topk(torch.from_numpy(ref), k).indices.numpy())
    assert np.array_equal(top, sketch)


def test_indexer_relu_removes_negative_dots():
    rng = np.random.default_rng(4)
    d_I, H_I, n = 64, 8, 50
    q = rng.uniform(0.1, 1.0, (1, H_I, d_I)).astype(np.float32)
    keys = -rng.uniform(0.1, 1.0, (1, n, d_I)).astype(np.float32)   # every dot < 0
    w = rng.normal(size=(1, H_I)).astype(np.float32)
    sc = oracle.indexer(ns_indexer(q, w, keys, [n]))
    assert np.all(sc[0] == 0.0)


def test_indexer_negative_head_weight_votes_against():
    """kgptalkie: head weights have no sign constraint, so scores can be negative."""
    rng = np.random.default_rng(5)
    d_I, H_I, n = 64, 4, 40
    q = rng.normal(size=(1, H_I, d_I)).astype(np.float32)
    keys = rng.normal(size=(1, n, d_I)).astype(np.float32)
    for j in range(H_I):
        w = np.zeros((1, H_I), np.float32)
        w[0, j] = -1.0
        sc = oracle.indexer(ns_indexer(q, w, keys, [n]))[0]
        dots = keys[0].astype(np.float64) @ q[0, j].astype(np.float64)
        np.testing.assert_allclose(sc, -np.maximum(dots, 0), rtol=1e-12, atol=0)
        assert np.any(sc < 0)


def test_indexer_fp8_mode_equals_dequantised_f32_mode():
    """FP8 path = dequantise (code * per-token scale) then the fp32 definition.

    Scales are powers of two so the dequantised values are exact in float32;
    heads, weights and keys are all distinct so a transposed or dropped scale
    changes the result.
    """
    g = torch.Generator().manual_seed(7)
    Nq, H_I, d_I, T_max = 2, 5, 64, 96
    qc = torch.randint(0, 0x7E, (Nq, H_I, d_I), generator=g, dtype=torch.uint8)
    qc |= (torch.rand((Nq, H_I, d_I), generator=g) < 0.5).to(torch.uint8) << 7
    kc = torch.randint(0, 0x7E, (Nq, T_max, d_I), generator=g, dtype=torch.uint8)
    kc |= (torch.rand((Nq, T_max, d_I), generator=g) < 0.5).to(torch.uint8) << 7
    q_scale = (2.0 ** torch.randint(-9, -3, (Nq, H_I), generator=g)).float()
    k_scale = (2.0 ** torch.randint(-9, -3, (Nq, T_max), generator=g)).float()
    w = (torch.randn((Nq, H_I), generator=g)).to(torch.bfloat16)
    qv = qc.view(torch.float8_e4m3fn).float() * q_scale[:, :, None]
    kv = kc.view(torch.float8_e4m3fn).float() * k_scale[:, :, None]
    lens = [T_max, 61]
    a = oracle.indexer(ns_indexer(qc.numpy(), w.view(torch.int16).numpy(), kc.numpy(), lens, fp8=True,
                                  q_scale=q_scale.numpy(), k_scale=k_scale.numpy()))
    b = oracle.indexer(ns_indexer(qv.numpy(), w.float().numpy(), kv.numpy(), lens))
    np.testing.assert_array_equal(np.nan_to_num(a, nan=-7), np.nan_to_num(b, nan=-7))
    # scaling one token's key scale by 2 doubles exactly that token's score
    k2 = k_scale.clone()
    k2[1, 10] *= 2
    c = oracle.indexer(ns_indexer(qc.numpy(), w.view(torch.int16).numpy(), kc.numpy(), lens, fp8=True,
                                  q_scale=q_scale.numpy(), k_scale=k2.numpy()))
    assert c[1, 10] == 2 * a[1, 10]
    mask = np.ones_like(a, bool)
    mask[1, 10] = False
    np.testing.assert_array_equal(np.nan_to_num(c[mask], nan=-7), np.nan_to_num(a[mask], nan=-7))


def test_indexer_causal_entries_untouched_and_future_keys_ignored():
    rng = np.random.default_rng(9)
    q = rng.normal(size=(1, 3, 64)).astype(np.float32)
    keys = rng.normal(size=(1, 80, 64)).astype(np.float32)
    w = rng.normal(size=(1, 3)).astype(np.float32)
    a = oracle.indexer(ns_indexer(q, w, keys, [50]), ld=80)
    keys2 = keys.copy()
    keys2[0, 50:] = 1e6
    b = oracle.indexer(ns_indexer(q, w, keys2, [50]), ld=80)
    assert np.array_equal(a[0, :50], b[0, :50])
    assert np.all(np.isnan(a[0, 50:]))


# ---------------------------------------------------------------- top-k

def _brute_topk(scores, k):
    n = len(scores)
    m = min(k, n)
    found = []
    for S in itertools.combinations(range(n), m):
        rest = [b for b in range(n) if b not in S]
        if all((scores[a] > scores[b]) or (scores[a] == scores[b] and a < b) for a in S for b in rest):
            found.append(S)
    assert len(found) == 1
    return list(found[0])


def test_topk_brute_force_tiny_with_ties():
    rng = np.random.default_rng(11)
    for trial in range(300):
        n = int(rng.integers(1, 13))
        k = int(rng.integers(1, 4))
        sc = rng.integers(-3, 4, size=n).astype(np.float64)  # many ties
        if trial % 3 == 0:
            sc = rng.normal(size=n)
        got = oracle.topk(sc[None, :], [n], k)[0]
        want = _brute_topk(sc.tolist(), k)
        assert got[:len(want)].tolist() == want
        assert np.all(got[len(want):] == -1)


def test_topk_page_worked_example():
    g = json.load(open(os.path.join(GOLD, "p4_selector_example.json")))
    sc = np.zeros(g["n"])
    for d in (g["printed"], g["filler"]):
        for pos, v in d.items():
            sc[int(pos)] = v
    got = oracle.topk(sc[None], [g["n"]], g["budget"])[0]
    assert got.tolist() == g["selected_ascending"]


def test_topk_short_prompt_is_read_in_full():
    """kgptalkie: the selector asks for min(budget, tokens so far)."""
    sc = np.random.default_rng(1).normal(size=(1, 10))
    got = oracle.topk(sc, [10], 16)[0]
    assert got[:10].tolist() == list(range(10)) and np.all(got[10:] == -1)
    got0 = oracle.topk(sc, [0], 4)[0]
    assert np.all(got0 == -1)


def test_topk_signed_zero_and_tie_rule():
    sc = np.array([[-0.0, 0.0, -0.0, 0.0, -1.0, 5.0]])
    got = oracle.topk(sc, [6], 3)[0]
    assert got.tolist() == [0, 1, 5]


def test_topk_invariants_random():
    rng = np.random.default_rng(12)
    n, k = 5000, 300
    sc = np.round(rng.normal(size=(1, n)), 2)   # coarse rounding -> ties at the threshold
    got = oracle.topk(sc, [n], k)[0]
    assert len(set(got.tolist())) == k and np.all(np.diff(got) > 0)
    sel = np.zeros(n, bool)
    sel[got] = True
    tau = sc[0, sel].min()
    assert sc[0, ~sel].max() <= tau
    tied_out = np.where((~sel) & (sc[0] == tau))[0]
    tied_in = np.where(sel & (sc[0] == tau))[0]
    if len(tied_out) and len(tied_in):
        assert tied_in.max() < tied_out.min()


# ---------------------------------------------------------------- attention

def _rand_attn(seed, Nq=2, H=3, n=37, T_max=40):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(Nq, H, 576)).astype(np.float32) / 8
    kv = rng.normal(size=(1, T_max, 576)).astype(np.float32) / 8
    return q, kv


def test_dense_attention_matches_torch_sdpa():
    q, kv = _rand_attn(1)
    scale = 1 / math.sqrt(192)
    n = 37
    inp = ns_attn(q, kv, [n, n], scale)
    out, lse = oracle.dense_attn(inp)
    Q = torch.from_numpy(q).double()                       # [Nq, H, 576]
    K = torch.from_numpy(kv[0, :n]).double()               # [n, 576]
    V = K[:, :512]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K[None].expand(2, n, 576),
                                                           V[None].expand(2, n, 512), scale=scale)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-11, atol=1e-13)
    ref_lse = torch.logsumexp(scale * torch.einsum("thx,sx->ths", Q, K), dim=-1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=1e-12)


def test_sparse_equals_dense_when_budget_covers_all():
    q, kv = _rand_attn(2)
    inp = ns_attn(q, kv, [30, 37], 0.07)
    idx = np.array([list(range(30)) + [-1] * 20, list(range(37)) + [-1] * 13], np.int32)
    a, la = oracle.sparse_attn(inp, idx)
    b, lb = oracle.dense_attn(inp)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=1e-12)


def test_sparse_equals_mask_view():
    """kgptalkie: topk then a -inf mask on every other position gives the same output."""
    q, kv = _rand_attn(3)
    inp = ns_attn(q, kv, [37, 37], 0.05)
    rng = np.random.default_rng(0)
    idx = np.stack([np.sort(rng.choice(37, 9, replace=False)) for _ in range(2)]).astype(np.int32)
    a, la = oracle.sparse_attn(inp, idx)
    b, lb = oracle.masked_dense_attn(inp, idx)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=1e-12)
    d, _ = oracle.dense_attn(inp)
    assert np.abs(a - d).max() > 1e-4   # the selection really changes the result


def test_single_selected_row_returns_its_value():
    q, kv = _rand_attn(4)
    inp = ns_attn(q, kv, [37, 37], 0.1)
    idx = np.array([[5, -1, -1], [-1, 36, -1]], np.int32)
    out, lse = oracle.sparse_attn(inp, idx)
    np.testing.assert_array_equal(out[0], np.broadcast_to(kv[0, 5, :512].astype(np.float64), (3, 512)))
    np.testing.assert_array_equal(out[1], np.broadcast_to(kv[0, 36, :512].astype(np.float64), (3, 512)))
    z = 0.1 * (q[0].astype(np.float64) @ kv[0, 5].astype(np.float64))
    np.testing.assert_allclose(lse[0], z, rtol=1e-13)


def test_weights_sum_to_one_and_equal_logits_lse():
    rng = np.random.default_rng(5)
    kv = np.ones((1, 40, 576), np.float32)
    kv[0, :, 512:] = rng.normal(size=(40, 64))        # logits differ only through the rope part
    q = rng.normal(size=(1, 4, 576)).astype(np.float32)
    inp = ns_attn(q, kv, [40], 0.3)
    idx = np.array([[0, 3, 7, 8, 20, 39]], np.int32)
    out, _ = oracle.sparse_attn(inp, idx)
    np.testing.assert_allclose(out, 1.0, rtol=1e-13)
    q0 = np.zeros((1, 2, 576), np.float32)             # all logits 0 -> uniform weights
    kv2 = rng.normal(size=(1, 40, 576)).astype(np.float32)
    out2, lse2 = oracle.sparse_attn(ns_attn(q0, kv2, [40], 0.3), idx)
    np.testing.assert_allclose(lse2, math.log(6), rtol=1e-14)
    np.testing.assert_allclose(out2[0, 0], kv2[0, idx[0], :512].astype(np.float64).mean(0), rtol=1e-12)


def test_attention_empty_selection():
    q, kv = _rand_attn(6)
    inp = ns_attn(q, kv, [0, 37], 0.1)
    idx = np.array([[-1, -1], [-1, -1]], np.int32)
    out, lse = oracle.sparse_attn(inp, idx)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_attention_ignores_positions_outside_the_selection():
    q, kv = _rand_attn(7)
    inp = ns_attn(q, kv, [37, 37], 0.1)
    idx = np.array([[1, 4, 9, -1], [0, 2, 30, 36]], np.int32)
    a, _ = oracle.sparse_attn(inp, idx)
    kv2 = kv.copy()
    kv2[0, [3, 5, 10, 37, 38]] = 50.0
    b, _ = oracle.sparse_attn(ns_attn(q, kv2, [37, 37], 0.1), idx)
    assert np.array_equal(a, b)


def test_attention_rejects_index_beyond_causal_length():
    q, kv = _rand_attn(8)
    inp = ns_attn(q, kv, [10, 10], 0.1)
    with pytest.raises(ValueError):
        oracle.sparse_attn(inp, np.array([[10], [0]], np.int32))


# ------------------------------------------------------------------ FP8 latent cache entry

def _entry(codes, scales, rope_bits):
    e = np.zeros(656, np.uint8)
    e[:512] = codes
    e[512:528] = np.asarray(scales, np.float32).view(np.uint8)
    e[528:] = np.asarray(rope_bits, np.uint16).view(np.uint8)
    return e


def test_fp8_latent_entry_hand_decoded():
    # kgptalkie "What Does the GPU Actually Run?": 512 e4m3 values, 4 fp32 scales, 64 bf16 rope
    # values.  Codes by the format definition: 0x38 = 1.0, 0x40 = 2.0, 0xB8 = -1.0,
    # 0x01 = 2^-9 (smallest subnormal), 0x7E = 448; group g = values [128 g, 128 g + 128).
    codes = np.zeros(512, np.uint8)
    codes[0], codes[127] = 0x38, 0x40          # group 0, scale 0.5
    codes[128], codes[255] = 0xB8, 0x01        # group 1, scale 2.0
    codes[256] = 0x7E                          # group 2, scale 1.0
    codes[511] = 0x38                          # group 3, scale 0.25
    rope = np.zeros(64, np.uint16)
    rope[0], rope[63] = 0x3FC0, 0xC020         # bf16 1.5, -2.5
    d = oracle.dequant_latent_fp8(_entry(codes, [0.5, 2.0, 1.0, 0.25], rope)[None])[0]
    want = np.zeros(576)
    want[0], want[127] = 0.5, 1.0
    want[128], want[255] = -2.0, 2.0 * 2.0 ** -9
    want[256] = 448.0
    want[511] = 0.25
    want[512], want[575] = 1.5, -2.5
    assert np.array_equal(d.astype(np.float64), want)


def test_fp8_latent_round_trip_within_e4m3_half_ulp():
    # quantise a bf16 latent cache (input preparation) and decode it with the oracle: every
    # latent value is within half an e4m3 step of the original (relative 2^-4 for normals,
    # 2^-10 of the group scale in the subnormal range); rope values are untouched
    from sparse_long_context_indexer_b200 import inputs
    inp = inputs.make_decode_inputs("fp8_round_trip", [500, 130], T_max=512, seed=9)
    entries = inputs.pack_fp8_latent(inp.kv)
    d = oracle.dequant_latent_fp8(entries).astype(np.float64)
    ref = inp.kv.float().numpy().astype(np.float64)
    scales = entries[..., 512:528].contiguous().view(torch.float32).numpy().astype(np.float64)
    s_of = np.repeat(scales, 128, axis=-1)
    bound = np.maximum(2.0 ** -4 * np.abs(ref[..., :512]), 2.0 ** -10 * s_of)
    assert np.all(np.abs(d[..., :512] - ref[..., :512]) <= bound * (1 + 1e-6))
    assert np.array_equal(d[..., 512:], ref[..., 512:])
