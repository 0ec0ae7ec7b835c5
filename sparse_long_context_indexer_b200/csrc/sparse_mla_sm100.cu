// sparse_mla_sm100.cu -- sparse MLA attention (MQA mode) over the selected
// latent rows, on the sm_100a tensor cores, plus the split merge.
//
// What it computes ("DeepSeek Sparse Attention Explained", sections "What Does
// the Whole Block Look Like?" -- softmax over the selected tokens only -- and
// "What Does the GPU Actually Run?" -- gather the selected rows, attend in BF16
// on chip; "DeepSeek V3.2-Exp Cuts Long-Context Costs", "Training and
// implementation details" -- MLA in MQA mode, every head shares each row):
//   out[t,h,:] = sum_{s in idx[t]} softmax_s(scale * q[t,h,:] . c[s,:]) c[s,0:512]
//   lse[t,h]   = ln sum_s exp(scale * q[t,h,:] . c[s,:])
//
// Design (one CTA per SM):
//   grid = (splits, 2 head halves, Nq).  Each CTA owns 64 of the 128 heads, so
//   every MMA is M = 64:
//     S = Q K^T   M = 64 heads, N = 64 rows, K = 576   (36 MMAs of K = 16, Q from TMEM)
//     O += P V    M = 64 heads, N = 2 x 256 values, K = 64 rows (P and V from shared memory)
//   The query block lives in tensor memory, which leaves shared memory to three
//   64-row gather stages (72 KB each).  The two CTAs of a (split, row) pair read
//   the same rows; the second read is an L2 hit.  TMEM (M = 64 layout: rows in
//   lanes 0..15 of each 32-lane subpartition, "low"; a second set at lane offset
//   16, "high"):
//     low   Q (two bf16 per column) at columns [0, 288); S buffers at [384, 448), [448, 512)
//     high  O[:, 0:256] at columns [0, 256), O[:, 256:512] at [256, 512)
//   warps 0..3  Q into TMEM at start; softmax with two threads per head (lanes r
//               and r+16 of warp w own head 16w+r: columns [0,32) and [32,64) of
//               S, alternate 32-column blocks of O); online softmax in the exp2
//               domain with lazy rescaling of O (only when the running maximum
//               grows by more than 8, i.e. a factor 256); P goes to a 128B-swizzled
//               K-major shared tile, the A operand of P V.
//   warp 4      TMEM allocator and the MMA issuer (converged warp, one elected
//               lane): QK^T(i+1) is issued before PV(i) so the softmax of tile i
//               overlaps the tensor core.
//   warps 5..12 row gather: 16-byte cp.async copies, eight threads per
//               128-byte piece of a row (a full line per eight lanes), straight
//               into the 128B-swizzled K-major tile the MMA reads; the same tile
//               serves as the MN-major V operand of P V.  Completion is tracked
//               by the stage's mbarrier (cp.async.mbarrier.arrive.noinc), so the
//               copiers never block on their own loads.  Skipped rows are
//               zero-filled without a read.  Rows a few tiles ahead are
//               prefetched to L2.  (Measured on B200: per-thread 16-byte copies
//               from 256 threads gather random 128-byte pieces at ~3.3 TB/s,
//               TMA tile::gather4 at ~1.4 TB/s.)
// Splits of a (row, head half) up to 8 run as one cluster: each CTA stages its
// normalised fp32 output and lse in shared memory and, after a cluster barrier,
// merges a slice of heads from all of them through distributed shared memory:
// O = sum_p exp(lse_p - L) O_p / sum_p exp(lse_p - L) with L = max_p lse_p.
// More splits write fp32 partials that mla_combine_kernel merges the same way.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <mutex>

#include <cuda_fp8.h>

#include "kernels.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kTileRows = kMlaTile;             // 64 gathered rows per tile
constexpr int kCtaHeads = kMlaHeads / 2;        // 64 heads per CTA (MMA M)
constexpr int kChunks = kDK / 64;               // 9 swizzle chunks of 64 bf16 (128 B)
constexpr int kChunkBytes = 64 * 128;           // one chunk of 64 rows (Q block or KV tile)
constexpr int kQBytes = kChunks * kChunkBytes;  // 73728
constexpr int kKvStageBytes = kChunks * kChunkBytes;  // 73728
constexpr int kPBytes = kCtaHeads * kTileRows * 2;    // 8192
constexpr int kStages = 3;
constexpr int kGatherWarp0 = 5;
constexpr int kGatherThreads = 256;
constexpr int kThreads = 32 * kGatherWarp0 + kGatherThreads;  // 416
constexpr int kOffKv = 0;
constexpr int kOffP = kOffKv + kStages * kKvStageBytes;
constexpr int kOffBar = kOffP + kPBytes;
// q_tma, q_full, kv_full[3], kv_empty[3], s_full[2], p_full, o_done
constexpr int kNumBar = 2 + 2 * kStages + 2 + 1 + 1;
constexpr int kOffMisc = kOffBar + kNumBar * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget of one CTA");
static_assert(kQBytes <= kKvStageBytes, "the query block is staged through the last gather stage");
constexpr int kQStage = kStages - 1;     // stage that holds the query block until it is in TMEM
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kLaneHi = 16u << 16;  // TMEM lane offset of the high M = 64 set
constexpr uint32_t kColQ = 0;            // Q: 288 columns (576 bf16), low lanes
constexpr uint32_t kColS = 384;          // S buffers: [384, 448), [448, 512), low lanes
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kPrefetchTiles = kStages + 1;  // L2 prefetch distance of the gather, in tiles
// split merge: received rows (at most 70 slots of (split, owned head), 1 KB each) and then their
// lse values, inside the idle gather stages
constexpr int kMergeLseOff = 72 * 1024;
static_assert(kMergeLseOff + 4 * 72 <= kStages * kKvStageBytes, "merge slots fit the gather stages");
constexpr uint32_t kIdescQK = make_idesc(kCtaHeads, kTileRows, 1 /*bf16*/, 1 /*bf16*/, 0, 0);
constexpr uint32_t kIdescPV = make_idesc(kCtaHeads, 256, 1 /*bf16*/, 1 /*bf16*/, 0 /*A K-major*/, 1 /*B MN-major*/);

struct MlaShared {
    int tmem_base;
    int abort_flag;
};

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Output modes: the final bf16 rows (one split), fp32 partials for the merge kernel,
// or a cluster of the splits that merges through distributed shared memory.
enum : int { kOutFinal = 0, kOutPartials = 1, kOutCluster = 2 };

template <int kOut>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_bf16_kernel(const MlaArgs a, const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_o) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sKv = sbase + kOffKv;
    const uint32_t sQs = sKv + kQStage * kKvStageBytes;  // query block staging (TMA -> TMEM)
    const uint32_t sP = sbase + kOffP;
    const uint32_t bar0 = sbase + kOffBar;
    const uint32_t bar_q_tma = bar0;
    const uint32_t bar_q = bar0 + 8u;
    auto bar_kv_full = [&](int s) { return bar0 + 8u * (2 + s); };
    auto bar_kv_empty = [&](int s) { return bar0 + 8u * (2 + kStages + s); };
    auto bar_s_full = [&](int s) { return bar0 + 8u * (2 + 2 * kStages + s); };
    const uint32_t bar_p_full = bar0 + 8u * (4 + 2 * kStages);
    const uint32_t bar_o = bar0 + 8u * (5 + 2 * kStages);
    MlaShared* sh = reinterpret_cast<MlaShared*>(smem + kOffMisc);
    volatile int* abort_flag = &sh->abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, half = blockIdx.y, t = blockIdx.z;

    int n_t = a.q_len[t];
    const int b = a.q_seq[t];
    const bool row_ok = n_t >= 0 && n_t <= a.T_max && b >= 0 && b < a.B;
    if (!row_ok) {
        if (split == 0 && half == 0 && tid == 0) record_status(a.status, DSA_STATUS_LENGTH);
        n_t = 0;
    }
    // Entries j of the row's selection handled by this split.  Dense mode (no index list):
    // entry j is position j itself and the row has n_t entries, so attention runs over every
    // position s < q_len[t].  A compact list (the library's top-k output) has min(k, n_t)
    // entries before its -1 padding.
    const bool dense = a.idx == nullptr;
    const int j_lo = split * a.rows_per_split;
    const int j_hi = min((dense || a.compact) ? min(a.k, n_t) : a.k, j_lo + a.rows_per_split);
    const int nrows = max(0, j_hi - j_lo);
    const int ntiles = (nrows + kTileRows - 1) / kTileRows;
    const int32_t* idx_row = dense ? nullptr : a.idx + (int64_t)t * a.k;
    const __nv_bfloat16* kv_base = reinterpret_cast<const __nv_bfloat16*>(a.kv);
    const __nv_bfloat16* kv_seq = kv_base + (int64_t)b * a.T_max * kDK;
    const int32_t* btab = a.block_table ? a.block_table + (int64_t)b * a.max_blocks : nullptr;
    // latent row of token s (contiguous cache, or through the block table of a paged one);
    // nullptr for a block id outside the pool
    auto kv_row = [&](int s) -> const __nv_bfloat16* {
        if (btab == nullptr) return kv_seq + (int64_t)s * kDK;
        const int pb = __ldg(btab + s / a.block_size);
        if (pb < 0 || pb >= a.num_blocks) return nullptr;
        return kv_base + ((int64_t)pb * a.block_size + s % a.block_size) * kDK;
    };
    // the same for the 656-byte FP8 entries
    const uint8_t* kv8_base = reinterpret_cast<const uint8_t*>(a.kv);
    auto kv8_row = [&](int s) -> const uint8_t* {
        int64_t row;
        if (btab == nullptr) {
            row = (int64_t)b * a.T_max + s;
        } else {
            const int pb = __ldg(btab + s / a.block_size);
            if (pb < 0 || pb >= a.num_blocks) return nullptr;
            row = (int64_t)pb * a.block_size + s % a.block_size;
        }
        return kv8_base + row * kFp8EntryBytes;
    };
    // entry r of tile i -> selected token, -1 past the end of the split
    auto load_pos = [&](int i, int r) -> int {
        const int j = j_lo + i * kTileRows + r;
        return j < j_hi ? (dense ? j : __ldg(idx_row + j)) : -1;
    };
    auto valid = [&](int s) { return s >= 0 && s < n_t; };

    if (tid == 0) {
        mbar_init(bar_q_tma, 1);
        mbar_init(bar_q, 128);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_kv_full(s), kGatherThreads);
            mbar_init(bar_kv_empty(s), 1);
        }
        for (int s = 0; s < 2; ++s) mbar_init(bar_s_full(s), 1);
        mbar_init(bar_p_full, 128);
        mbar_init(bar_o, 1);
        sh->abort_flag = 0;
        fence_barrier_init();
        if (ntiles > 0) {
            // the query block lands in the last gather stage and moves to TMEM from there
            mbar_arrive_expect_tx(bar_q_tma, kQBytes);
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c)
                tma_load_2d(sQs + c * kChunkBytes, &tmap_q, c * 64, t * kMlaHeads + half * kCtaHeads, bar_q_tma);
        }
    }
    if (warp == 4) {
        tmem_alloc(smem_u32(&sh->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    // Everything above (barriers, TMEM, the query block) may overlap the previous kernel;
    // the index lists come from it (programmatic dependent launch).  The first index
    // loads of each role go out before the setup barrier.
    griddep_wait();
    griddep_launch_dependents();
    const int p = tid - 32 * kGatherWarp0;  // gather thread (warps >= kGatherWarp0)
    const int rr = (p >> 3) & 31, gl = p & 7;
    const bool pf_lane = warp >= kGatherWarp0 && gl == 0;  // 32 threads issue the L2 prefetches
    int cur0 = -1, cur1 = -1, pf = -1, pf_first = -1, v0 = -1, v1 = -1;
    if (ntiles > 0) {
        if (warp >= kGatherWarp0) {
            cur0 = load_pos(0, rr);
            cur1 = load_pos(0, rr + 32);
            // each CTA of the head pair prefetches one half of the rows
            if (pf_lane && kStages < ntiles) pf_first = load_pos(kStages, rr + 32 * half);
            if (pf_lane && kPrefetchTiles < ntiles) pf = load_pos(kPrefetchTiles, rr + 32 * half);
        } else if (warp < 4) {
            v0 = load_pos(0, lane);
            v1 = load_pos(0, lane + 32);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)sh->tmem_base;

    if (warp >= kGatherWarp0) {
        // ------------------------------------------------ row gather (8 warps)
        // thread p copies 16-byte granule (p & 7) of every 128-byte piece of rows
        // (p >> 3) and (p >> 3) + 32 of each tile.
        auto prefetch_row = [&](int s) {
            if (valid(s)) {
                if (a.kv_fp8) {
                    const uint8_t* r = kv8_row(s);
                    if (r) l2_prefetch_bulk(r, kFp8EntryBytes);
                } else {
                    const __nv_bfloat16* r = kv_row(s);
                    if (r) l2_prefetch_bulk(r, kDK * 2);
                }
            }
        };
        if (pf_lane) prefetch_row(pf_first);
        if (a.kv_fp8) {
            // FP8 entries: thread p owns row p / 4 of each tile and its 128-value group p % 4:
            // eight 16-byte loads of e4m3 codes and one scale into registers a tile ahead,
            // dequantised to bf16 into the tile the MMAs read (chunks 2q and 2q + 1); the rope
            // values (chunk 8) go by asynchronous copies.
            const int r8 = p >> 2, q8 = p & 3;
            uint4 lat[8];
            float scl = 0.f;
            bool has = false;
            auto load_tile = [&](int i) {
                const int s = load_pos(i, r8);
                const uint8_t* row = valid(s) ? kv8_row(s) : nullptr;
                if (valid(s) && row == nullptr && q8 == 0) record_status(a.status, DSA_STATUS_INDEX_OOB);
                if (valid(s) == false && s != -1 && q8 == 0 && row_ok && half == 0)
                    record_status(a.status, DSA_STATUS_INDEX_OOB);
                has = row != nullptr;
                if (has) {
                    const uint4* src = reinterpret_cast<const uint4*>(row + q8 * 128);
#pragma unroll
                    for (int k = 0; k < 8; ++k) lat[k] = __ldg(src + k);
                    scl = __ldg(reinterpret_cast<const float*>(row + kFp8ScaleOff) + q8);
                }
                return row;
            };
            const uint8_t* row_cur = load_tile(0);
            for (int i = 0; i < ntiles; ++i) {
                const int st = i % kStages;
                const uint32_t stage = sKv + st * kKvStageBytes;
                // rope: granules 2 q8 and 2 q8 + 1 of the row's 128 bytes, chunk 8
#pragma unroll
                for (int g2 = 0; g2 < 2; ++g2) {
                    const int g = 2 * q8 + g2;
                    const uint8_t* src = row_cur ? row_cur + kFp8RopeOff + 16 * g : kv8_base;
                    cp_async16_zfill(stage + 8 * kChunkBytes + r8 * 128 + ((g ^ (r8 & 7)) << 4), src, row_cur ? 16u : 0u);
                }
                // dequantise this tile's codes (taken out of the registers before the next loads)
                uint4 cur[8];
                const float sc = scl;
                const bool cur_has = has;
#pragma unroll
                for (int k = 0; k < 8; ++k) cur[k] = lat[k];
                if (pf_lane && i + kPrefetchTiles < ntiles) prefetch_row(pf);
                if (i + 1 < ntiles) {
                    row_cur = load_tile(i + 1);
                    if (pf_lane && i + 1 + kPrefetchTiles < ntiles) pf = load_pos(i + 1 + kPrefetchTiles, rr + 32 * half);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    // 16 codes = values 128 q8 + 16 k .. + 15: chunk 2 q8 + k / 4, granules 2 (k % 4), + 1
                    const uint32_t w[4] = {cur[k].x, cur[k].y, cur[k].z, cur[k].w};
                    uint32_t o[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[e] & 0xFFFFu), __NV_E4M3);
                        const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[e] >> 16), __NV_E4M3);
                        const float2 flo = __half22float2(*reinterpret_cast<const __half2*>(&lo));
                        const float2 fhi = __half22float2(*reinterpret_cast<const __half2*>(&hi));
                        o[2 * e] = cur_has ? pack_bf16x2(flo.x * sc, flo.y * sc) : 0u;
                        o[2 * e + 1] = cur_has ? pack_bf16x2(fhi.x * sc, fhi.y * sc) : 0u;
                    }
                    const int c = 2 * q8 + (k >> 2);
#pragma unroll
                    for (int g2 = 0; g2 < 2; ++g2) {
                        const int g = 2 * (k & 3) + g2;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(stage + c * kChunkBytes + r8 * 128 +
                                                                                     ((g ^ (r8 & 7)) << 4)),
                                     "r"(o[4 * g2]), "r"(o[4 * g2 + 1]), "r"(o[4 * g2 + 2]), "r"(o[4 * g2 + 3])
                                     : "memory");
                    }
                }
                // the tile is complete for this thread: its rope copies have landed and its stores are
                // visible to the tensor cores
                cp_async_wait_all();
                fence_proxy_async_smem();
                mbar_arrive(bar_kv_full(st));
                if (i + 1 < ntiles) {
                    const int nx = i + 1;
                    bool ok = true;
                    if (lane == 0) {
                        if (nx == kQStage) {
                            ok = mbar_wait_spin(bar_q, 0, abort_flag, a.status);
                        } else if (nx >= kStages) {
                            ok = mbar_wait_spin(bar_kv_empty(nx % kStages), ((nx / kStages) - 1) & 1, abort_flag,
                                                a.status);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                }
            }
        } else
        for (int i = 0; i < ntiles; ++i) {
            const int st = i % kStages;
            if (gl == 0 && row_ok && half == 0 &&
                ((cur0 < -1 || cur0 >= n_t) || (cur1 < -1 || cur1 >= n_t)))
                record_status(a.status, DSA_STATUS_INDEX_OOB);
            const uint32_t stage = sKv + st * kKvStageBytes;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int s = h2 ? cur1 : cur0;
                const int r = rr + 32 * h2;
                const __nv_bfloat16* row = valid(s) ? kv_row(s) : nullptr;
                if (valid(s) && row == nullptr && gl == 0) record_status(a.status, DSA_STATUS_INDEX_OOB);
                const bool ok_row = row != nullptr;
                const __nv_bfloat16* src = ok_row ? row + gl * 8 : kv_base;
                const uint32_t dst = stage + r * 128 + ((gl ^ (r & 7)) << 4);
#pragma unroll
                for (int c = 0; c < kChunks; ++c) cp_async16_zfill(dst + c * kChunkBytes, src + c * 64, ok_row ? 16u : 0u);
            }
            if (!(a.selftest_stall && i == 0)) cp_async_arrive_noinc(bar_kv_full(st));
            if (pf_lane && i + kPrefetchTiles < ntiles) prefetch_row(pf);
            if (i + 1 < ntiles) {
                cur0 = load_pos(i + 1, rr);
                cur1 = load_pos(i + 1, rr + 32);
                if (pf_lane && i + 1 + kPrefetchTiles < ntiles) pf = load_pos(i + 1 + kPrefetchTiles, rr + 32 * half);
                const int nx = i + 1;
                bool ok = true;
                if (lane == 0) {
                    if (nx == kQStage) {
                        // the query block's staging must have moved to TMEM first
                        ok = mbar_wait_spin(bar_q, 0, abort_flag, a.status);
                    } else if (nx >= kStages) {
                        // the stage is free once PV(nx - kStages) has completed
                        ok = mbar_wait_spin(bar_kv_empty(nx % kStages), ((nx / kStages) - 1) & 1, abort_flag, a.status);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        // copies still in flight on an early exit land before the CTA's shared memory goes away
        cp_async_wait_all();
    } else if (warp == 4) {
        // ------------------------------------------------ MMA issue (converged warp, one elected lane)
        if (ntiles > 0) {
            // warp-uniform copies of the bases keep the per-MMA operands in uniform registers
            const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
            const uint32_t sb0 = __shfl_sync(0xffffffffu, sbase, 0);
            bool ok = mbar_wait(bar_q, 0, abort_flag, a.status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            const uint64_t dk = make_smem_desc(sb0 + kOffKv, 16, 1024, kSwizzle128B);
            const uint64_t dp = make_smem_desc(sb0 + kOffP, 16, 1024, kSwizzle128B);
            const uint64_t dv = make_smem_desc(sb0 + kOffKv, kChunkBytes, 1024, kSwizzle128B);
            // Issue in dependency order, whichever is ready first: QK^T(q) needs its
            // gathered tile and PV(q-2) already issued (S buffer reuse); PV(p) needs
            // the softmax of tile p.  PV is preferred: it frees a gather stage.
            int qk = 0, pv = 0;
            uint64_t t_last = globaltimer_ns();
            uint32_t spins = 0;
            while (ok && pv < ntiles) {
                const bool pv_ready = pv < qk && __shfl_sync(0xffffffffu, mbar_test(bar_p_full, pv & 1), 0);
                const bool qk_ready =
                    !pv_ready && qk < ntiles && qk <= pv + 1 &&
                    __shfl_sync(0xffffffffu, mbar_test(bar_kv_full(qk % kStages), (qk / kStages) & 1), 0);
                if (pv_ready) {
                    tc_fence_after();
                    const uint32_t soff = (pv % kStages) * kKvStageBytes;
                    if (elect_one()) {
#pragma unroll
                        for (int vh = 0; vh < 2; ++vh) {
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks) {
                                const uint64_t ad = dp + ((ks * 32) >> 4);
                                const uint64_t bd = dv + ((soff + vh * 4 * kChunkBytes + ks * 2048) >> 4);
                                mma_f16_ss(tm + kLaneHi + 256u * vh, ad, bd, kIdescPV, (pv > 0 || ks > 0) ? 1u : 0u);
                            }
                        }
                        mma_commit(bar_kv_empty(pv % kStages));
                    }
                    __syncwarp();
                    ++pv;
                    t_last = globaltimer_ns();
                } else if (qk_ready) {
                    tc_fence_after();
                    const uint32_t d = tm + kColS + 64 * (qk & 1);
                    const uint32_t soff = (qk % kStages) * kKvStageBytes;
                    // one elected lane issues the whole pass (operands computed by the
                    // converged warp beforehand stay in uniform registers)
                    if (elect_one()) {
#pragma unroll
                        for (int c = 0; c < kChunks; ++c) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t off = c * kChunkBytes + kk * 32;
                                // K step 4c + kk: 16 bf16 of Q = 8 TMEM columns
                                mma_f16_ts(d, tm + kColQ + 8u * (4 * c + kk), dk + ((soff + off) >> 4), kIdescQK,
                                           (c | kk) ? 1u : 0u);
                            }
                        }
                        mma_commit(bar_s_full(qk & 1));
                    }
                    __syncwarp();
                    ++qk;
                    t_last = globaltimer_ns();
                } else if ((++spins & 255u) == 0) {
                    bool stop = false;
                    if (*abort_flag) {
                        stop = true;
                    } else if (globaltimer_ns() - t_last > (a.wait_budget_ns ? a.wait_budget_ns : kWaitBudgetNs)) {
                        if (lane == 0) {
                            record_status(a.status, DSA_STATUS_TIMEOUT);
                            *abort_flag = 1;
                        }
                        stop = true;
                    }
                    ok = !__shfl_sync(0xffffffffu, stop, 0);
                }
            }
            if (ok && elect_one()) mma_commit(bar_o);
            __syncwarp();
            if (!ok && pv > 0 && lane == 0)
                mbar_wait(bar_kv_empty((pv - 1) % kStages), ((pv - 1) / kStages) & 1, nullptr, nullptr, 50000000ull);
        }
    } else {
        // ------------------------------------------------ softmax, two threads per head
        const int r = lane & 15, hh = lane >> 4;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);  // low lanes of this subpartition
        const uint32_t o_base = lane_base + kLaneHi;                       // high lanes: O
        const float scale_log2 = a.softmax_scale * 1.4426950408889634f;
        const int prow = warp * 16 + r;  // head within this CTA = row of P
        const uint32_t prow_addr = sP + (prow >> 3) * 1024 + (prow & 7) * 128;
        float m_used = -CUDART_INF_F;
        float l = 0.f;
        bool ok = true;
        if (ntiles > 0) {
            // ---- the query block into TMEM: 32-column step c of row prow takes 16 columns
            // (32 bf16, four 16-byte granules of chunk c) per thread
            ok = mbar_wait(bar_q_tma, 0, abort_flag, a.status);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
#pragma unroll 1
                for (int c = 0; c < kChunks; ++c) {
                    const uint32_t src = sQs + c * kChunkBytes + prow * 128;
                    uint32_t w[16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(w[4 * q4]), "=r"(w[4 * q4 + 1]), "=r"(w[4 * q4 + 2]), "=r"(w[4 * q4 + 3])
                                     : "r"(src + (((4 * hh + q4) ^ (prow & 7)) << 4)));
                    tmem_st16x2_16(lane_base + kColQ + 32 * c, w);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_q);
        }
        for (int i = 0; i < ntiles && ok; ++i) {
            const int sb = i & 1;
            const unsigned b0 = __ballot_sync(0xffffffffu, valid(v0));
            const unsigned b1 = __ballot_sync(0xffffffffu, valid(v1));
            const unsigned vbits = hh ? b1 : b0;
            if (i + 1 < ntiles) {
                v0 = load_pos(i + 1, lane);
                v1 = load_pos(i + 1, lane + 32);
            }
            ok = mbar_wait_spin(bar_s_full(sb), (i >> 1) & 1, abort_flag, a.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[32];
            tmem_ld16x2_32(lane_base + kColS + 64 * sb, sv);
            tmem_wait_ld();
            float x[32];
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                x[c] = ((vbits >> c) & 1u) ? __uint_as_float(sv[c]) * scale_log2 : -CUDART_INF_F;
                mx = fmaxf(mx, x[c]);
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            // P's buffer and O are free once PV(i-1) has completed
            if (i > 0) {
                ok = mbar_wait_spin(bar_kv_empty((i - 1) % kStages), ((i - 1) / kStages) & 1, abort_flag, a.status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
            }
            if (mx > m_used + kRescaleThreshold) {
                if (m_used != -CUDART_INF_F) {
                    // this thread owns the 32-column blocks [c0 + 32 hh, c0 + 32 hh + 32) of its O row
                    const float alpha = fast_exp2(m_used - mx);
#pragma unroll 1
                    for (int c0 = 0; c0 < kDV; c0 += 64) {
                        uint32_t ov[32];
                        tmem_ld16x2_32(o_base + c0, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
                        tmem_st16x2_32(o_base + c0, ov);
                    }
                    tmem_wait_st();
                    l *= alpha;
                }
                m_used = mx;
            }
            const float msub = m_used == -CUDART_INF_F ? 0.f : m_used;
            uint32_t pk[16];
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float p0 = fast_exp2(x[2 * c] - msub);
                const float p1 = fast_exp2(x[2 * c + 1] - msub);
                rs += p0 + p1;
                pk[c] = pack_bf16x2(p0, p1);
            }
            l += rs;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const int g = 4 * hh + q4;  // 16-byte granule = 8 positions of the tile
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow_addr + ((g ^ (prow & 7)) << 4)),
                             "r"(pk[4 * q4]), "r"(pk[4 * q4 + 1]), "r"(pk[4 * q4 + 2]), "r"(pk[4 * q4 + 3])
                             : "memory");
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_p_full);
        }
        // ---- epilogue: the normalised row goes to shared memory (the gather stages are idle
        // now), 32 columns per step: this thread's blocks start at col = c0 + 32 hh
        const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
        const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
        const float lse_v = l_row > 0.f ? (m_used + __log2f(l_row)) * 0.6931471805599453f : -CUDART_INF_F;
        const bool have_o = ok && ntiles > 0;
        if (have_o) {
            ok = mbar_wait_spin(bar_o, 0, abort_flag, a.status);
            ok = __all_sync(0xffffffffu, ok);
        }
        const bool read_o = have_o && ok;
        if (read_o) tc_fence_after();
        const int64_t th = (int64_t)t * kMlaHeads + half * kCtaHeads + prow;
        if (kOut == kOutCluster) {
            // every warp of the CTA stages the rows after the role loops: publish this head's
            // normaliser and lse, and whether its O may be read (in P's idle tile)
            if (hh == 0) {
                float* pub = reinterpret_cast<float*>(smem + kOffP);
                pub[prow] = read_o ? inv_l : 0.f;
                pub[kCtaHeads + prow] = lse_v;
                if (r == 0) reinterpret_cast<int*>(pub)[2 * kCtaHeads + warp] = read_o ? 1 : 0;
            }
        } else if (hh == 0) {
            if (kOut == kOutFinal) {
                if (a.lse) a.lse[th] = lse_v;
            } else {
                a.part_lse[(int64_t)split * a.Nq * kMlaHeads + th] = lse_v;
            }
        }
#pragma unroll 1
        for (int c0 = 0; c0 < (kOut == kOutCluster ? 0 : kDV); c0 += 64) {
            uint32_t ov[32];
            if (read_o) {
                tmem_ld16x2_32(o_base + c0, ov);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) ov[c] = 0u;
            }
            const int col = c0 + 32 * hh;  // first output column of this piece
            if (kOut == kOutFinal) {
                // bf16 TMA-store boxes of 64 heads x 64 columns: box k holds columns [64k, 64k + 64)
                const uint32_t box = sKv + prow * 128 + (col >> 6) * kChunkBytes;
                const int g0 = (col & 63) >> 3;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(ov[8 * q4 + 2 * e]) * inv_l,
                                           __uint_as_float(ov[8 * q4 + 2 * e + 1]) * inv_l);
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(box + (((g0 + q4) ^ (prow & 7)) << 4)),
                                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
            } else {
                // fp32 TMA-store boxes of 64 heads x 32 columns: box k holds columns [32k, 32k + 32)
                const uint32_t box = sKv + prow * 128 + (col >> 5) * kChunkBytes;
#pragma unroll
                for (int g = 0; g < 8; ++g)
                    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(box + ((g ^ (prow & 7)) << 4)),
                                 "f"(__uint_as_float(ov[4 * g]) * inv_l), "f"(__uint_as_float(ov[4 * g + 1]) * inv_l),
                                 "f"(__uint_as_float(ov[4 * g + 2]) * inv_l), "f"(__uint_as_float(ov[4 * g + 3]) * inv_l)
                                 : "memory");
            }
        }
        if (kOut != kOutCluster) {
            constexpr bool final_out = kOut == kOutFinal;
            fence_proxy_async_smem();
            named_barrier_sync(1, 128);
            if (tid == 0) {
                const int nbox = final_out ? kDV / 64 : kDV / 32;
                const int y = final_out ? t * kMlaHeads + half * kCtaHeads
                                        : (split * a.Nq + t) * kMlaHeads + half * kCtaHeads;
                for (int k = 0; k < nbox; ++k)
                    tma_store_2d(&tmap_o, k * (final_out ? 64 : 32), y, sKv + k * kChunkBytes);
                bulk_commit_group();
                bulk_wait_group_read0();
            }
        }
    }
    if (kOut == kOutCluster) {
        // ---- merge of the splits.  CTA `rank` of the cluster owns heads [rank * hp, rank * hp + hp)
        // O = sum_s exp(lse_s - L) O_s / sum_s exp(lse_s - L),  lse = L + ln sum_s exp(lse_s - L)
        // Every CTA pushes its normalised bf16 rows (and lse values) straight into the shared
        // memory of the head's owner -- stores cross the cluster network without a round trip
        // each -- and every owner then merges from its own shared memory.  The first barrier
        // makes sure no peer still reads its gather stages (the push lands there).
        const int S = a.splits;
        const int rank = (int)cluster_ctarank();
        const int hp = (kCtaHeads + S - 1) / S;
        const float* pub = reinterpret_cast<const float*>(smem + kOffP);
        cluster_sync_all();  // (also the CTA's own barrier: every warp has left its role)
        tc_fence_after();
        {
            // receive slot of (split s, owned head hl): 1 KB row at sKv + (s * hp + hl) * 1024, its
            // 16-byte granule j (eight values) at (j & ~7) | ((j ^ row) & 7); its lse at
            // sKv + kMergeLseOff + 4 * (s * hp + hl)
            const int sub = warp & 3;                      // TMEM sub-partition this warp may read
            const int nw = sub == 0 ? 4 : 3;               // warps 0..12 per sub-partition
            const int iw = warp >> 2;
            const int r = lane & 15, hh = lane >> 4;
            const int prow = sub * 16 + r;                 // head within this CTA
            const int owner = prow / hp, hl = prow - owner * hp;
            const int slot = split * hp + hl;
            const uint32_t dst_row = mapa_shared(sKv + slot * (kDV * 2), (uint32_t)owner);
            const float inv_l = pub[prow];
            const bool sub_ok = reinterpret_cast<const int*>(pub)[2 * kCtaHeads + sub] != 0;
            const uint32_t o_sub = tmem + ((uint32_t)(sub * 32) << 16) + kLaneHi;
#pragma unroll 1
            for (int ck = iw; ck < kDV / 64; ck += nw) {
                const int c0 = ck * 64;
                uint32_t ov[32];
                if (sub_ok) {
                    tmem_ld16x2_32(o_sub + c0, ov);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) ov[c] = 0u;
                }
                const int jb = (c0 + 32 * hh) >> 3;  // first granule of this thread's 32 columns
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(ov[8 * q4 + 2 * e]) * inv_l,
                                           __uint_as_float(ov[8 * q4 + 2 * e + 1]) * inv_l);
                    const int j = jb + q4;
                    st_shared_cluster_v4_u32(dst_row + ((((j & ~7) | ((j ^ slot) & 7))) << 4), w[0], w[1], w[2], w[3]);
                }
            }
        }
        if (tid < kCtaHeads) {
            const int ow = tid / hp;
            st_shared_cluster_f32(mapa_shared(sKv + kMergeLseOff + 4 * (split * hp + tid - ow * hp), (uint32_t)ow),
                                  pub[kCtaHeads + tid]);
        }
        cluster_sync_all();  // every push has landed
        const int h0 = rank * hp;
        const int nh = max(0, min(kCtaHeads, h0 + hp) - h0);
        const int nunits = 2 * nh;  // (head, half row) units
        const float* lse_in = reinterpret_cast<const float*>(smem + kOffKv + kMergeLseOff);
        for (int u = warp; u < nunits; u += kThreads / 32) {
            const int hl = u >> 1;
            const int jh = (u & 1) * 32;  // first granule of the half row
            const int j = jh + lane;
            const float ls = lane < S ? lse_in[lane * hp + hl] : -CUDART_INF_F;
            float L = ls;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, o));
            const float e = (lane < S && L != -CUDART_INF_F) ? __expf(ls - L) : 0.f;
            float esum = e;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) esum += __shfl_xor_sync(0xffffffffu, esum, o);
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int sp = 0; sp < kMlaClusterMaxSplits; ++sp) {
                const float es = __shfl_sync(0xffffffffu, e, sp);  // 0 for absent or empty splits
                if (sp < S) {
                    const int slot = sp * hp + hl;
                    uint4 v;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                 : "r"(sKv + slot * (kDV * 2) + ((((j & ~7) | ((j ^ slot) & 7))) << 4)));
                    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[2 * q] = fmaf(es, __uint_as_float(vw[q] << 16), acc[2 * q]);
                        acc[2 * q + 1] = fmaf(es, __uint_as_float(vw[q] & 0xFFFF0000u), acc[2 * q + 1]);
                    }
                }
            }
            const float inv = esum > 0.f ? 1.f / esum : 0.f;
            const int64_t trow = (int64_t)t * kMlaHeads + half * kCtaHeads + h0 + hl;
            uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + trow * kDV);
            o[j] = make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                              pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
            if (lane == 0 && (u & 1) == 0 && a.lse) a.lse[trow] = esum > 0.f ? L + __logf(esum) : -CUDART_INF_F;
        }
        // no peer touches this CTA's shared memory after the last barrier: no exit barrier
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge of split partials: one CTA of 128 threads per (head, row); thread j
// owns values [4j, 4j+4) of the 512-wide output row.
__global__ void __launch_bounds__(128) mla_combine_kernel(const MlaArgs a) {
    const int h = blockIdx.x, t = blockIdx.y, j = threadIdx.x;
    const int64_t plane = (int64_t)a.Nq * kMlaHeads;
    const int64_t th = (int64_t)t * kMlaHeads + h;
    float lp[16];
    float L = -CUDART_INF_F;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        lp[p] = p < a.splits ? a.part_lse[p * plane + th] : -CUDART_INF_F;
        L = fmaxf(L, lp[p]);
    }
    float s = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        if (p < a.splits) {
            const float e = (L == -CUDART_INF_F) ? 0.f : __expf(lp[p] - L);
            s += e;
            const float4 v = reinterpret_cast<const float4*>(a.part_o + (p * plane + th) * kDV)[j];
            acc.x = fmaf(e, v.x, acc.x);
            acc.y = fmaf(e, v.y, acc.y);
            acc.z = fmaf(e, v.z, acc.z);
            acc.w = fmaf(e, v.w, acc.w);
        }
    }
    const float inv = s > 0.f ? 1.f / s : 0.f;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) + th * kDV)[j] = pk;
    if (j == 0 && a.lse) a.lse[th] = s > 0.f ? L + __logf(s) : -CUDART_INF_F;
}

}  // namespace

cudaError_t launch_sparse_mla_bf16(const MlaArgs& a, cudaStream_t st) {
    if (a.Nq == 0) return cudaSuccess;
    // q: [Nq * 128 heads, 576] bf16, 64 x 64 boxes, 128B-swizzled
    alignas(64) CUtensorMap tq;
    if (!encode_tensor_map_2d(&tq, 2, a.q, kDK, (uint64_t)a.Nq * kMlaHeads, kDK * 2, 64, kCtaHeads, 128))
        return cudaErrorInvalidValue;
    dim3 grid(a.splits, 2, a.Nq);
    if (mla_cluster_merge(a.splits)) {
        auto kern = sparse_mla_bf16_kernel<kOutCluster>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmemBytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)a.splits;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = a.pdl ? 2 : 1;
        e = cudaLaunchKernelEx(&cfg, kern, a, tq, tq);  // the output map is unused in this mode
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    // output: bf16 [Nq * 128, 512] (one split) or fp32 partials [splits * Nq * 128, 512];
    // boxes of 128 bytes x 64 heads, 128B-swizzled
    alignas(64) CUtensorMap to;
    const bool final_out = a.splits == 1;
    const uint64_t out_rows = (uint64_t)(final_out ? 1 : a.splits) * a.Nq * kMlaHeads;
    if (!encode_tensor_map_2d(&to, final_out ? 2 : 4, final_out ? a.out : static_cast<void*>(a.part_o), kDV, out_rows,
                              kDV * (final_out ? 2 : 4), final_out ? 64 : 32, kCtaHeads, 128))
        return cudaErrorInvalidValue;
    auto kern = final_out ? sparse_mla_bf16_kernel<kOutFinal> : sparse_mla_bf16_kernel<kOutPartials>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, a, tq, to);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Library-owned scratch for callers that cannot allocate device memory.
// One statically sized buffer per device holds the split partials of the
// attention kernel (normalised fp32 O and lse of every split).  Every call
// shares it: calls whose kernels overlap on the GPU race on it.  Nothing in
// it needs to start at zero (each call overwrites every partial it reads).
static __device__ __align__(256) unsigned char g_mla_static_scratch[kStaticScratchBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
}  // namespace

cudaError_t static_mla_scratch(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        // host code only sees a stand-in for the array: ask the runtime for the
        // device address, once per device, with that device current
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_mla_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *ptr = g_scratch_ptr[dev];
    return cudaSuccess;
}

cudaError_t launch_mla_combine(const MlaArgs& a, cudaStream_t st) {
    if (a.Nq == 0 || a.splits <= 1 || mla_cluster_merge(a.splits)) return cudaSuccess;
    if (a.splits > 16) return cudaErrorInvalidValue;
    mla_combine_kernel<<<dim3(kMlaHeads, a.Nq), 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
