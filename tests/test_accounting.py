"""The roofline accounting reproduces the arithmetic the pages print."""
import math

from sparse_long_context_indexer_b200 import accounting as acc


def test_cache_entry_sizes():
    # kgptalkie "Why Is Decoding Held Back by Memory?": 576 values, 1,152 B in BF16,
    # 71,424 B across 62 layers, 8.72 GB (GiB) at 128K tokens
    assert acc.latent_row_bytes() == 1152
    assert acc.latent_row_bytes() * 62 == 71424
    assert round(131072 * 71424 / 2**30, 2) == 8.72
    # kgptalkie "What Does the GPU Actually Run?": 656-byte FP8 entry
    assert acc.fp8_latent_entry_bytes() == 656
    # milos-mitrovic "What Does DSA Actually Cost...": roughly 132 bytes per token (d_I = 128)
    assert acc.indexer_key_bytes(128) == 132


def test_per_pair_and_block_multiply_adds():
    # kgptalkie "How Much Arithmetic Does This Actually Save?"
    assert acc.pair_macs_attention(128) == 139264
    assert acc.pair_macs_indexer(64, 128) == 8192
    assert round(acc.pair_macs_attention() / acc.pair_macs_indexer(64, 128)) == 17
    T = 131072
    dense = acc.pair_macs_attention() * T * T
    scout = acc.pair_macs_indexer(64, 128) * T * T
    sparse = acc.pair_macs_attention() * T * 2048
    assert round(dense / 1e12) == 2393
    assert round(scout / 1e12) == 141
    assert round(sparse / 1e12) == 37
    assert round((scout + sparse) / 1e12) == 178
    assert round(dense / (scout + sparse), 1) == 13.4
    assert T // 2048 == 64
    assert round(scout / sparse, 1) == 3.8


def test_decode_read_footprint_at_131k():
    # milos-mitrovic: ~5.2 GB dense MLA vs ~1.1 GB DSA per decode step at 131K (61 layers, FP8 cache)
    T, layers = 131072, 61
    dense = T * acc.fp8_latent_entry_bytes() * layers
    dsa = (T * acc.indexer_key_bytes(128) + 2048 * acc.fp8_latent_entry_bytes()) * layers
    assert round(dense / 1e9, 1) == 5.2
    assert round(dsa / 1e9, 1) == 1.1


def test_lizeman_per_token_ops():
    # lizeman "DeepSeek Sparse Attention" section 2: 128,000*64 ~ 8.2e6, 2,000*512 ~ 1.0e6, 9.2e6 total,
    # 128,000*512 ~ 6.6e7 for full MLA, ~7x
    s1, s2 = 128000 * 64, 2000 * 512
    assert round(s1 / 1e6, 1) == 8.2 and round(s2 / 1e6, 1) == 1.0
    assert round((s1 + s2) / 1e6, 1) == 9.2
    full = 128000 * 512
    assert round(full / 1e7, 1) == 6.6 and round(full / (s1 + s2)) == 7


def test_long_decode_step_bytes():
    lens = [131072] * 16
    b = acc.decode_step_bytes(lens)
    assert b["indexer"] == 16 * (131072 * 68 + 64 * 70)
    assert b["attention"] == 16 * (2048 * 1152 + 128 * 576 * 2 + 128 * 512 * 2 + 128 * 4)
    assert math.isclose(b["total"] / 1e6, 184.9, rel_tol=2e-3)
    f = acc.decode_step_flops(lens)
    assert f["attention"] == 16 * 570425344
    assert acc.prefill_indexer_flops(65536) == 8192 * 65536 * 65537 // 2
