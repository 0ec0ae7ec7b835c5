"""Algorithmic work of the DSA hot path (bytes and FLOPs), used for rooflines.

Per query row with n causal candidates, d_I-wide FP8 indexer keys (+ one fp32
scale per token), H_I indexer heads, k selected rows of 576 bf16 values and H
query heads:
  indexer bytes   n * (d_I + 4) + H_I * (d_I + 4 + 2)      (keys + scales; q8, q_scale, w)
  indexer FLOPs   2 * H_I * d_I * n                       (FP8 MMA)
  gather bytes    min(k, n) * 576 * 2
  attention FLOPs 2 * H * min(k, n) * (576 + 512)          (Q K^T and P V)
  q / out bytes   H * 576 * 2 + H * 512 * 2 + H * 4        (query, output, lse)
Score rows and index lists are intermediate design traffic, not counted.

The page arithmetic these formulas must reproduce ("DeepSeek Sparse Attention
Explained", sections "Why Is Decoding Held Back by Memory?", "How Much
Arithmetic Does This Actually Save?" and "What Does the GPU Actually Run?";
"DeepSeek Sparse Attention Cuts Long-Context Cost", "What Does DSA Actually
Cost in Compute and Memory?"; "DeepSeek Sparse Attention" section 2) is
checked in tests/test_accounting.py.
"""
from __future__ import annotations

D_K, D_V = 576, 512


def latent_row_bytes(dtype_bytes: int = 2) -> int:
    return D_K * dtype_bytes


def fp8_latent_entry_bytes() -> int:
    """512 e4m3 values + 4 fp32 scales (one per 128 values) + 64 bf16 rope values."""
    return 512 * 1 + 4 * 4 + 64 * 2


def indexer_key_bytes(d_I: int) -> int:
    """d_I FP8 values plus one fp32 scale per cached token."""
    return d_I + 4


def pair_macs_attention(H: int = 128) -> int:
    """Multiply-adds of one (query, key) pair in MLA attention: H*(576 + 512)."""
    return H * (D_K + D_V)


def pair_macs_indexer(H_I: int, d_I: int) -> int:
    return H_I * d_I


def indexer_bytes_row(n: int, H_I: int, d_I: int) -> int:
    return n * indexer_key_bytes(d_I) + H_I * (d_I + 4 + 2)


def indexer_flops_row(n: int, H_I: int, d_I: int) -> int:
    return 2 * H_I * d_I * n


def attention_bytes_row(n: int, k: int, H: int) -> int:
    return min(k, n) * latent_row_bytes() + H * D_K * 2 + H * D_V * 2 + H * 4


def attention_flops_row(n: int, k: int, H: int) -> int:
    return 2 * H * min(k, n) * (D_K + D_V)


def decode_step_bytes(seq_lens, H_I=64, d_I=64, k=2048, H=128) -> dict:
    ib = sum(indexer_bytes_row(n, H_I, d_I) for n in seq_lens)
    ab = sum(attention_bytes_row(n, k, H) for n in seq_lens)
    return {"indexer": ib, "attention": ab, "total": ib + ab}


def decode_step_flops(seq_lens, H_I=64, d_I=64, k=2048, H=128) -> dict:
    fi = sum(indexer_flops_row(n, H_I, d_I) for n in seq_lens)
    fa = sum(attention_flops_row(n, k, H) for n in seq_lens)
    return {"indexer": fi, "attention": fa, "total": fi + fa}


def prefill_indexer_flops(L: int, H_I=64, d_I=64) -> int:
    """Causal pairs L(L+1)/2 times 2*H_I*d_I."""
    return 2 * H_I * d_I * L * (L + 1) // 2
