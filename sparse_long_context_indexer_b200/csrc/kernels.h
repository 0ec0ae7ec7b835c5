// kernels.h -- host-side launch interface between the C ABI (dsa_api.cu) and
// the kernel translation units.  Not installed; no torch types anywhere.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace dsa {

constexpr int kDK = 576;   // latent key width (512 latent + 64 rope)
constexpr int kDV = 512;   // value width
constexpr int kIdxTile = 128;  // indexer: cached tokens per tensor-core tile (MMA M)
constexpr int kIdxHeads = 64;  // indexer: heads per query (MMA N) for the FP8 kernel
constexpr int kMlaTile = 64;   // sparse MLA: gathered rows per tile (MMA N of Q K^T, K of P V)
constexpr int kMlaHeads = 128; // sparse MLA bf16 kernel: query heads (two CTAs of MMA M = 64)

struct IndexerArgs {
    const void* q_I;
    const float* q_scale;
    const void* w;
    const void* k_I;
    const float* k_scale;
    const int32_t* q_seq;
    const int32_t* q_len;
    float* scores;
    int64_t ld;
    int Nq, B, T_max, H_I, d_I;
    int* status;
    // rows (units) whose length is at most this get no scores: inside the library's pipelines,
    // where the scores are intermediate, the top-k selects every position of such a row
    // without reading them (0 = score every row)
    int skip_upto;
    // Paged cache (block_table != nullptr): token s of sequence b lives in pool row
    // block_table[b * max_blocks + s / block_size] * block_size + s % block_size of k_I
    // ([num_blocks * block_size, d_I]) and k_scale ([num_blocks, block_size]).
    const int32_t* block_table;
    int block_size, max_blocks, num_blocks;
    int page_box;  // key rows per TMA box in paged mode (set by the launcher)
};

struct TopkArgs {
    const float* scores;
    int64_t ld;
    const int32_t* q_len;
    int32_t* idx;
    int Nq, k, T_max;
    int* status;
    int pdl;  // launch as a programmatic dependent of the previous kernel (the library's own pipelines)
    // expected longest row (0: ld / T_max): sizes the cluster and each CTA's shared-memory slice;
    // a longer row stays correct (its slices beyond the cached size are read from global memory)
    int64_t row_len_hint;
};

struct MlaArgs {
    const void* q;
    const void* kv;
    const int32_t* idx;
    const int32_t* q_seq;
    const int32_t* q_len;
    void* out;
    float* lse;
    float* part_o;    // [splits, Nq, H, 512] when splits > 1
    float* part_lse;  // [splits, Nq, H]
    int Nq, B, T_max, k, H;
    int splits, rows_per_split;
    float softmax_scale;
    int* status;
    int pdl;  // launch as a programmatic dependent of the previous kernel (the library's own pipelines)
    // the index list is the library's own top-k output: entries past min(k, q_len[t]) are -1,
    // so the splits stop there
    int compact;
    // paged latent cache (block_table != nullptr): token s of sequence b is kv row
    // block_table[b * max_blocks + s / block_size] * block_size + s % block_size
    const int32_t* block_table;
    int block_size, max_blocks, num_blocks;
    // FP8 latent cache: 656-byte entries of 512 e4m3 values, 4 fp32 scales (one per 128
    // values) and the 64 rope values in bf16; dequantised to bf16 by the gather
    int kv_fp8;
    // Self-test of the bounded waits (0 in every production call): the gather never signals
    // the first tile, so the MMA warp's wait on it runs out after wait_budget_ns (0 = the
    // default budget) and the kernel records DSA_ERR_TIMEOUT and drains.
    int selftest_stall;
    uint64_t wait_budget_ns;
};
constexpr int kFp8EntryBytes = 656;  // 512 + 4 * 4 + 64 * 2
constexpr int kFp8ScaleOff = 512;
constexpr int kFp8RopeOff = 528;

// New tokens into the caches (contiguous when block_table is null, else pools of blocks).
struct AppendArgs {
    int n;                     // new tokens
    const int32_t* seq;        // [n] sequence of token i
    const int32_t* pos;        // [n] its position
    const void* kv_new;        // [n, 576] bf16 latent rows
    const float* k_new;        // [n, d_I] fp32 indexer keys
    void* kv;                  // latent cache: [.., 576] bf16 or [.., 656] FP8 entries
    void* k_I;                 // indexer keys: e4m3 codes (idx_fp8) or fp32
    float* k_scale;            // per-token key scales (idx_fp8)
    int B, T_max, d_I;
    int idx_fp8, kv_fp8;
    const int32_t* block_table;
    int block_size, max_blocks, num_blocks;
    int* status;
};
cudaError_t launch_append_tokens(const AppendArgs& a, cudaStream_t st);

cudaError_t launch_indexer_fp8(const IndexerArgs& a, int grid, cudaStream_t st);
// Same scores, four consecutive query rows per tensor-core pass: every group of four
// rows (row 4u .. 4u+3) must belong to one sequence (prefill).
cudaError_t launch_indexer_fp8_units4(const IndexerArgs& a, int grid, cudaStream_t st);
cudaError_t launch_indexer_f32(const IndexerArgs& a, cudaStream_t st);
cudaError_t launch_topk(const TopkArgs& a, int cluster, cudaStream_t st);
cudaError_t launch_sparse_mla_bf16(const MlaArgs& a, cudaStream_t st);
// Splits of one (row, head half) up to this count run as one thread-block cluster and
// merge through distributed shared memory inside the attention kernel; beyond it they
// write fp32 partials that launch_mla_combine merges (a no-op in the cluster case).
constexpr int kMlaClusterMaxSplits = 8;
inline bool mla_cluster_merge(int splits) { return splits >= 2 && splits <= kMlaClusterMaxSplits; }
cudaError_t launch_mla_combine(const MlaArgs& a, cudaStream_t st);
cudaError_t launch_sparse_mla_f32(const MlaArgs& a, cudaStream_t st);
cudaError_t launch_wait_timeout_selftest(int* status, int timeout_us, cudaStream_t st);

// Statically allocated split scratch of the attention kernel (no-allocation entry point):
// fp32 partial outputs for up to kStaticScratchPartials (split, row) pairs of 128 heads x 512,
// then their lse values.
constexpr int kMaxDevices = 64;
constexpr size_t kStaticScratchPartials = 64;
constexpr size_t kStaticScratchOBytes = kStaticScratchPartials * kMlaHeads * kDV * sizeof(float);  // 16 MiB
constexpr size_t kStaticScratchBytes = kStaticScratchOBytes + kStaticScratchPartials * kMlaHeads * sizeof(float);
// Device address of this device's static scratch (looked up on first use per device).
cudaError_t static_mla_scratch(void** ptr);

// Largest row chunk kept in shared memory by one top-k CTA (elements).
constexpr int kTopkSmemKeys = 45056;
// Most CTAs (one thread-block cluster, the portable size) sharing one top-k row; 16-CTA
// clusters were measured slower on the long decode (44 vs 32 us).
constexpr int kTopkMaxCluster = 8;

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
bool encode_tensor_map_2d(void* map, int dtype_bytes, const void* base, uint64_t inner, uint64_t outer,
                          uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_bytes);

}  // namespace dsa
