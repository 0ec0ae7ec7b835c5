"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) hot path.

This module only draws random tensors with the shapes, value distributions and
planted structure of the workloads the DSA pages describe; it holds none of the
method's arithmetic (no scoring, selection or attention).  The same bytes feed
the CUDA path and the CPU oracle, so both sides see identical FP8/bf16 inputs.

Workloads (sizes from the pages):
  * "kgptalkie: DeepSeek Sparse Attention explained", section "What Does the GPU
    Actually Run?": FP8 indexer keys with one fp32 scale per token, a bf16
    576-value latent row per token (512 latent + 64 rope).
  * same page, "How Does the Lightning Indexer Score a Token?": H_I small heads
    of width d_I, a per-head weight, one shared key per cached token.
  * "lizeman: DeepSeek Sparse Attention", section 2: d_I = 64, K = 2048.

Layouts (row-major, contiguous):
  q_I     [Nq, H_I, d_I]   e4m3 bytes (uint8) or float32
  q_scale [Nq, H_I]        float32 (FP8 mode only; all heads of a token share it)
  w       [Nq, H_I]        bfloat16 (FP8 mode) or float32
  k_I     [B, T_max, d_I]  e4m3 bytes or float32
  k_scale [B, T_max]       float32 (FP8 mode only)
  q       [Nq, H, 576]     bfloat16 or float32 (absorbed MLA query)
  kv      [B, T_max, 576]  bfloat16 or float32 (latent cache rows)
  q_seq   [Nq] int32, q_len [Nq] int32 (causal candidate count of each row)
Rows of a sequence at positions >= its length are zero.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

D_K = 576   # latent key width: 512 latent + 64 rope
D_V = 512   # value width: the first 512 values of the same row
FP8_MAX = 448.0

F32, BF16, FP8 = 0, 1, 2   # element types, same codes as the C interface


@dataclass
class DSAInputs:
    name: str
    B: int
    Nq: int
    H_I: int
    d_I: int
    H: int
    k: int
    T_max: int
    idx_dtype: int
    kv_dtype: int
    softmax_scale: float
    q_I: torch.Tensor
    q_scale: Optional[torch.Tensor]
    w: torch.Tensor
    k_I: torch.Tensor
    k_scale: Optional[torch.Tensor]
    q: torch.Tensor
    kv: torch.Tensor
    q_seq: torch.Tensor
    q_len: torch.Tensor
    seq_lens: list = field(default_factory=list)
    seed: int = 0

    def to(self, device) -> "DSAInputs":
        out = DSAInputs(**{f: getattr(self, f) for f in self.__dataclass_fields__})
        for f in ("q_I", "q_scale", "w", "k_I", "k_scale", "q", "kv", "q_seq", "q_len"):
            t = getattr(self, f)
            if t is not None:
                setattr(out, f, t.to(device))
        return out

    @property
    def device(self):
        return self.kv.device


def _normal(shape, gen, device, std):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std


def quantize_e4m3_per_row(x: torch.Tensor):
    """Per-row FP8 e4m3 quantisation (scale = amax/448, round-to-nearest-even).

    Input generation only: the hot path receives the bytes and the scales.
    Rows that are all zero get scale 1.
    """
    flat = x.reshape(x.shape[0], -1)
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    q = (flat / scale[:, None]).clamp(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).reshape(x.shape), scale.float()


FP8_ENTRY_BYTES = 656      # 512 e4m3 latent values, 4 fp32 scales, 64 bf16 rope values
FP8_GROUP = 128            # latent values per scale


def pack_fp8_latent(kv: torch.Tensor) -> torch.Tensor:
    """The FP8 latent cache entry of kgptalkie "What Does the GPU Actually Run?": per token
    512 e4m3 codes (four groups of 128, each scaled by its amax / 448, round-to-nearest-even),
    the 4 fp32 scales, then the 64 rope values left in bf16.  kv: [..., 576] bf16 -> uint8
    [..., 656].  Input preparation only: the hot path and the oracle receive the bytes."""
    lead = kv.shape[:-1]
    x = kv.reshape(-1, 576)
    lat = x[:, :512].float().reshape(-1, 4, FP8_GROUP)
    amax = lat.abs().amax(dim=2)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax)).float()
    codes = (lat / scale[:, :, None]).clamp(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
    out = torch.empty((x.shape[0], FP8_ENTRY_BYTES), dtype=torch.uint8, device=kv.device)
    out[:, :512] = codes.reshape(-1, 512)
    out[:, 512:528] = scale.contiguous().view(torch.uint8).reshape(-1, 16)
    out[:, 528:] = x[:, 512:].contiguous().view(torch.uint8).reshape(-1, 128)
    return out.reshape(*lead, FP8_ENTRY_BYTES)


def with_fp8_latent(inp: "DSAInputs") -> "DSAInputs":
    """The same workload with its latent cache in 656-byte FP8 entries (kv_dtype FP8)."""
    out = DSAInputs(**{f: getattr(inp, f) for f in inp.__dataclass_fields__})
    out.kv = pack_fp8_latent(inp.kv)
    out.kv_dtype = FP8
    out.name = inp.name + "_fp8kv"
    return out


def _unit(v: torch.Tensor) -> torch.Tensor:
    n = v.norm()
    return v / n if float(n) > 0 else v


def make_decode_inputs(name: str, seq_lens: Sequence[int], *, H_I=64, d_I=64, H=128, k=2048,
                       fp8=True, T_max=None, w_std=None, n_anchors=0, anchor_frac=None,
                       anchor_region=1.0, recency=False, seed=0, device="cpu",
                       softmax_scale=1.0 / math.sqrt(192.0)) -> DSAInputs:
    """Decode workload: one query token per sequence, causal over its cached tokens.

    seq_lens[b] is the cached length of sequence b; query row b sees s < seq_lens[b].
    Anchors ("planted high-relevance positions"): the indexer key is set to
    4*|k|_typ * u/|u| with u = sum_{j: w_j>0} w_j q_I[j], and the latent row to
    4*|c|_typ * ubar/|ubar| with ubar = the head-mean of the MLA query.
    recency: k_I[s] += 2|k|_typ * exp(-(n-1-s)/4096) * u/|u|.
    """
    B = len(seq_lens)
    Nq = B
    if T_max is None:
        T_max = max(128, int(math.ceil(max(seq_lens) / 128.0)) * 128)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    std = 1.0 / 8.0
    if w_std is None:
        w_std = std if fp8 else 1.0 / math.sqrt(H_I)
    q_I = _normal((Nq, H_I, d_I), gen, device, std)
    w = _normal((Nq, H_I), gen, device, w_std)
    if fp8:
        w = w.to(torch.bfloat16)
    q = _normal((Nq, H, D_K), gen, device, std)
    if fp8:
        q = q.to(torch.bfloat16)
    k_I = torch.zeros((B, T_max, d_I), device=device, dtype=torch.float32)
    kv = torch.zeros((B, T_max, D_K), device=device,
                     dtype=torch.bfloat16 if fp8 else torch.float32)
    k_typ = math.sqrt(d_I) * std
    c_typ = math.sqrt(D_K) * std
    for b, n in enumerate(seq_lens):
        if n == 0:
            continue
        k_I[b, :n] = _normal((n, d_I), gen, device, std)
        # latent rows in chunks to bound the fp32 temporary
        step = 1 << 16
        for s0 in range(0, n, step):
            s1 = min(n, s0 + step)
            kv[b, s0:s1] = _normal((s1 - s0, D_K), gen, device, std).to(kv.dtype)
        wf = w[b].float()
        u = (wf.clamp(min=0)[:, None] * q_I[b]).sum(0)
        uh = _unit(u)
        if recency:
            s = torch.arange(n, device=device, dtype=torch.float32)
            bias = 2.0 * k_typ * torch.exp(-(n - 1 - s) / 4096.0)
            k_I[b, :n] += bias[:, None] * uh[None, :]
        na = n_anchors if anchor_frac is None else max(1, int(round(anchor_frac * n)))
        na = min(na, n)
        if na > 0:
            hi = max(1, int(n * anchor_region))
            pos = torch.randperm(hi, generator=gen, device=device)[:na]
            k_I[b, pos] = 4.0 * k_typ * uh
            ubar = _unit(q[b].float().mean(0))
            kv[b, pos] = (4.0 * c_typ * ubar).to(kv.dtype)
    if fp8:
        k8, ks = quantize_e4m3_per_row(k_I.reshape(B * T_max, d_I))
        k_I_out = k8.reshape(B, T_max, d_I)
        k_scale = ks.reshape(B, T_max)
        q8, qs = quantize_e4m3_per_row(q_I)
        q_I_out = q8
        q_scale = qs[:, None].expand(Nq, H_I).contiguous()
    else:
        k_I_out, k_scale, q_I_out, q_scale = k_I, None, q_I, None
    q_seq = torch.arange(Nq, device=device, dtype=torch.int32)
    q_len = torch.tensor(list(seq_lens), device=device, dtype=torch.int32)
    return DSAInputs(name=name, B=B, Nq=Nq, H_I=H_I, d_I=d_I, H=H, k=k, T_max=T_max,
                     idx_dtype=FP8 if fp8 else F32, kv_dtype=BF16 if fp8 else F32,
                     softmax_scale=softmax_scale, q_I=q_I_out, q_scale=q_scale, w=w,
                     k_I=k_I_out, k_scale=k_scale, q=q, kv=kv, q_seq=q_seq, q_len=q_len,
                     seq_lens=list(seq_lens), seed=seed)


def make_prefill_inputs(name: str, L: int, *, H_I=64, d_I=64, H=128, k=2048, seed=4,
                        device="cpu", rows: Optional[Sequence[int]] = None,
                        softmax_scale=1.0 / math.sqrt(192.0)) -> DSAInputs:
    """Prefill workload: one sequence of L tokens, every position a query.

    Row t sees s <= t (q_len[t] = t + 1).  N(0,1)/8 everywhere, FP8 indexer with
    per-token scales, bf16 latent.  `rows` restricts the query rows that are
    materialised (the key/latent cache is always the full sequence).
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    std = 1.0 / 8.0
    T_max = max(128, int(math.ceil(L / 128.0)) * 128)
    k_I = torch.zeros((1, T_max, d_I), device=device)
    k_I[0, :L] = _normal((L, d_I), gen, device, std)
    kv = torch.zeros((1, T_max, D_K), device=device, dtype=torch.bfloat16)
    step = 1 << 16
    for s0 in range(0, L, step):
        s1 = min(L, s0 + step)
        kv[0, s0:s1] = _normal((s1 - s0, D_K), gen, device, std).to(torch.bfloat16)
    # Query-side tensors are drawn for all L rows in one stream so that a row
    # subset is bit-identical to the same rows of the full draw.
    q_I_all = _normal((L, H_I, d_I), gen, device, std)
    w_all = _normal((L, H_I), gen, device, std).to(torch.bfloat16)
    sel = torch.arange(L, device=device) if rows is None else torch.as_tensor(list(rows), device=device, dtype=torch.long)
    q_I = q_I_all[sel]
    w = w_all[sel].contiguous()
    del q_I_all, w_all
    Nq = int(sel.numel())
    # MLA query drawn row by row from a per-row generator so subsets match the full draw
    q = torch.empty((Nq, H, D_K), device=device, dtype=torch.bfloat16)
    qgen = torch.Generator(device=device)
    chunk = 4096
    sel_cpu = sel.cpu().tolist()
    if rows is None:
        for r0 in range(0, L, chunk):
            r1 = min(L, r0 + chunk)
            qgen.manual_seed(seed * 1000003 + r0 // chunk)
            q[r0:r1] = _normal((r1 - r0, H, D_K), qgen, device, std).to(torch.bfloat16)
    else:
        by_chunk = {}
        for i, r in enumerate(sel_cpu):
            by_chunk.setdefault(r // chunk, []).append((i, r))
        for c, items in by_chunk.items():
            r0 = c * chunk
            r1 = min(L, r0 + chunk)
            qgen.manual_seed(seed * 1000003 + c)
            block = _normal((r1 - r0, H, D_K), qgen, device, std).to(torch.bfloat16)
            for i, r in items:
                q[i] = block[r - r0]
    k8, ks = quantize_e4m3_per_row(k_I.reshape(T_max, d_I))
    q8, qs = quantize_e4m3_per_row(q_I)
    q_scale = qs[:, None].expand(Nq, H_I).contiguous()
    q_seq = torch.zeros(Nq, device=device, dtype=torch.int32)
    q_len = (sel + 1).to(torch.int32)
    return DSAInputs(name=name, B=1, Nq=Nq, H_I=H_I, d_I=d_I, H=H, k=k, T_max=T_max,
                     idx_dtype=FP8, kv_dtype=BF16, softmax_scale=softmax_scale,
                     q_I=q8, q_scale=q_scale, w=w, k_I=k8.reshape(1, T_max, d_I),
                     k_scale=ks.reshape(1, T_max), q=q, kv=kv, q_seq=q_seq, q_len=q_len,
                     seq_lens=[L], seed=seed)


# ---- the five workloads ------------------------------------------------------

def paged_layout(inp: DSAInputs, block_size: int, seed: int = 0, spare_blocks: int = 3):
    """The same cache in paged form: pools of blocks in a seeded random physical order.

    Returns (k_I_pool, k_scale_pool, kv_pool, block_table) with block_table[b, j] the pool
    block holding tokens [j * block_size, (j + 1) * block_size) of sequence b; blocks past a
    sequence's longest query length get -1 (never read).  Pure data movement.
    """
    B, T_max = inp.kv.shape[0], inp.kv.shape[1]
    assert T_max % block_size == 0
    mb = T_max // block_size
    nb = B * mb + spare_blocks
    gen = torch.Generator().manual_seed(seed)
    perm = torch.randperm(nb, generator=gen)
    dev = inp.kv.device
    k_pool = torch.zeros((nb, block_size) + tuple(inp.k_I.shape[2:]), dtype=inp.k_I.dtype, device=dev)
    s_pool = torch.zeros((nb, block_size), dtype=torch.float32, device=dev)
    kv_pool = torch.zeros((nb, block_size, inp.kv.shape[2]), dtype=inp.kv.dtype, device=dev)
    table = torch.full((B, mb), -1, dtype=torch.int32)
    q_seq = inp.q_seq.cpu()
    q_len = inp.q_len.cpu()
    for b in range(B):
        rows = q_seq == b
        need = int(q_len[rows].max()) if bool(rows.any()) else 0
        for j in range((need + block_size - 1) // block_size):
            pb = int(perm[b * mb + j])
            table[b, j] = pb
            sl = slice(j * block_size, (j + 1) * block_size)
            k_pool[pb] = inp.k_I[b, sl]
            if inp.k_scale is not None:
                s_pool[pb] = inp.k_scale[b, sl]
            kv_pool[pb] = inp.kv[b, sl]
    return k_pool, s_pool, kv_pool, table.to(dev)


def tiny(device="cpu"):
    """Tiny decode: 1 query over 4096 cached tokens, fp32, H_I=4, top-256, 16 heads, 16 anchors."""
    return make_decode_inputs("tiny_decode_4k_fp32", [4096], H_I=4, d_I=64, H=16, k=256,
                              fp8=False, n_anchors=16, seed=0, device=device)


def decode_batch32_lengths(seed=2):
    g = torch.Generator()
    g.manual_seed(seed)
    return torch.randint(16384, 32769, (32,), generator=g).tolist()


def decode32(device="cpu"):
    """Decode batch 32, lengths uniform in [16384, 32768], FP8 indexer, 1% anchors."""
    return make_decode_inputs("decode_b32_16k_32k", decode_batch32_lengths(2), T_max=32768,
                              anchor_frac=0.01, seed=2, device=device)


def long_decode(device="cpu", batch=16):
    """Long decode: batch 16 at 131072 cached tokens, recency-biased keys, 32 anchors."""
    return make_decode_inputs("long_decode_b16_128k", [131072] * batch, T_max=131072,
                              n_anchors=32, recency=True, seed=3, device=device)


def million_lengths(seed=5):
    g = torch.Generator()
    g.manual_seed(seed)
    rag = torch.randint(65536, 524289, (6,), generator=g).tolist()
    return [1048576, 1048576] + rag


def million(device="cpu"):
    """1M-context decode: 2 x 1,048,576 plus 6 ragged lengths in [65536, 524288], 64 far-history anchors."""
    return make_decode_inputs("million_decode_b8", million_lengths(5), T_max=1048576,
                              n_anchors=64, anchor_region=0.1, seed=5, device=device)


def prefill(device="cpu", L=65536, rows=None):
    """Prefill: one sequence of L=65536 tokens, causal, every position a query."""
    return make_prefill_inputs("prefill_64k", L, seed=4, device=device, rows=rows)
