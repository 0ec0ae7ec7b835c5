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
//   grid = (splits, 2 value halves, Nq).  TMEM holds 128 lanes x 512 fp32
//   columns; the 128-head x 512 output alone would fill it, so each CTA of a
//   pair owns one 256-wide half of the value dimension (256 columns) and both
//   recompute S = Q K^T (M = 128 heads, N = 32 rows, K = 576).  The second CTA's
//   gather of the same rows is served by L2.
//   warps 0..3  softmax: thread h owns head h (TMEM lane h); online softmax in
//               the exp2 domain with lazy rescaling of O (only when the running
//               maximum grows by more than 8, i.e. a factor 256); P is written
//               back into TMEM as bf16 over the S columns it came from.
//   warp 4      TMEM allocator, Q TMA (9 boxes of 128 x 64, 128B swizzle) and
//               the single-thread tcgen05.mma issuer: QK^T(i+1) is issued
//               before PV(i) so the softmax of tile i overlaps the tensor core.
//   warps 5..8  gather: each selected 1152-byte row is read with 16-byte vector
//               loads (consecutive lanes -> consecutive bytes of one row) and
//               stored into the 128B-swizzled K-major tile the MMA reads; the
//               same tile serves as the MN-major V operand of P V.
// Splits > 1 write normalised fp32 partials and their lse; mla_combine_kernel
// merges them: O = sum_p exp(lse_p - L) O_p with L = logsumexp_p lse_p.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <mutex>

#include "kernels.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kTileRows = kMlaTile;          // 32 gathered rows per tile
constexpr int kHeads = kMlaHeads;            // 128 (MMA M)
constexpr int kChunks = kDK / 64;            // 9 swizzle chunks of 64 bf16 (128 B)
constexpr int kQBytes = kHeads * kDK * 2;    // 147456
constexpr int kQChunkBytes = kHeads * 128;   // 16384
constexpr int kKvChunkBytes = kTileRows * 128;  // 4096
constexpr int kKvStageBytes = kChunks * kKvChunkBytes;  // 36864
constexpr int kStages = 2;
constexpr int kThreads = 288;
constexpr int kGatherThreads = 128;
constexpr int kGranules = kTileRows * (kDK * 2 / 16);  // 2304 16-byte granules per tile
constexpr int kOffQ = 0;
constexpr int kOffKv = kOffQ + kQBytes;
constexpr int kOffBar = kOffKv + kStages * kKvStageBytes;
constexpr int kNumBar = 1 + 2 * kStages + 2 + 2 + 1;  // q_full, kv_full[2], kv_empty[2], s_full[2], p_full[2], o_done
constexpr int kOffMisc = kOffBar + kNumBar * 8;
constexpr int kOffIdx = kOffMisc + 64;                   // up to 2048 staged positions
constexpr int kSmemBytes = kOffIdx + 2048 * 4 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;     // O half: columns [0, 256)
constexpr uint32_t kColS = 256;   // S/P buffers: [256, 288), [288, 320)
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kPrefetchTiles = 4;          // L2 prefetch distance of the gather, in tiles
constexpr uint32_t kIdescQK = make_idesc(kHeads, kTileRows, 1 /*bf16*/, 1 /*bf16*/, 0, 0);
constexpr uint32_t kIdescPV = make_idesc(kHeads, 256, 1 /*bf16*/, 1 /*bf16*/, 0 /*A K-major*/, 1 /*B MN-major*/);

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

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_bf16_kernel(const MlaArgs a, const __grid_constant__ CUtensorMap tmap_q) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + kOffQ;
    const uint32_t sKv = sbase + kOffKv;
    const uint32_t bar0 = sbase + kOffBar;
    const uint32_t bar_q = bar0;
    auto bar_kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto bar_kv_empty = [&](int s) { return bar0 + 8u * (1 + kStages + s); };
    auto bar_s_full = [&](int s) { return bar0 + 8u * (1 + 2 * kStages + s); };
    auto bar_p_full = [&](int s) { return bar0 + 8u * (3 + 2 * kStages + s); };
    const uint32_t bar_o = bar0 + 8u * (5 + 2 * kStages);
    MlaShared* sh = reinterpret_cast<MlaShared*>(smem + kOffMisc);
    int32_t* sidx = reinterpret_cast<int32_t*>(smem + kOffIdx);  // this split's positions, -1 = skip
    volatile int* abort_flag = &sh->abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, half = blockIdx.y, t = blockIdx.z;

    // rows of idx handled by this split
    const int j_lo = split * a.rows_per_split;
    const int j_hi = min(a.k, j_lo + a.rows_per_split);
    const int nrows = max(0, j_hi - j_lo);
    const int ntiles = (nrows + kTileRows - 1) / kTileRows;
    int n_t = a.q_len[t];
    const int b = a.q_seq[t];
    const bool row_ok = n_t >= 0 && n_t <= a.T_max && b >= 0 && b < a.B;
    if (!row_ok) {
        if (split == 0 && half == 0 && tid == 0) record_status(a.status, DSA_STATUS_LENGTH);
        n_t = 0;
    }
    const __nv_bfloat16* kv_seq = reinterpret_cast<const __nv_bfloat16*>(a.kv) + (int64_t)b * a.T_max * kDK;

    if (tid == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_kv_full(s), kGatherThreads);
            mbar_init(bar_kv_empty(s), 1);
            mbar_init(bar_s_full(s), 1);
            mbar_init(bar_p_full(s), 128);
        }
        mbar_init(bar_o, 1);
        sh->abort_flag = 0;
        fence_barrier_init();
        if (ntiles > 0) {
            // the query block is needed first and does not depend on the staging below
            mbar_arrive_expect_tx(bar_q, kQBytes);
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) tma_load_2d(sQ + c * kQChunkBytes, &tmap_q, c * 64, t * kHeads, bar_q);
        }
    }
    if (warp == 4) {
        tmem_alloc(smem_u32(&sh->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    // Stage this split's positions (sanitised: anything outside [0, n_t) becomes -1)
    // and start pulling the first tiles' rows into L2: each CTA of the value pair
    // prefetches one half of the rows, so every row leaves HBM once, early.
    for (int r = tid; r < ntiles * kTileRows; r += kThreads) {
        int s = r < nrows ? a.idx[(int64_t)t * a.k + j_lo + r] : -1;
        if (s < -1 || s >= n_t) {
            if (half == 0 && row_ok) record_status(a.status, DSA_STATUS_INDEX_OOB);
            s = -1;
        }
        sidx[r] = s;
        if (s >= 0 && (r & 1) == half && r < kPrefetchTiles * kTileRows)
            l2_prefetch_bulk(kv_seq + (int64_t)s * kDK, kDK * 2);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)sh->tmem_base;

    if (warp == 4) {
        // ------------------------------------------------ Q load + MMA issue
        if (lane == 0 && ntiles > 0) {
            bool ok = mbar_wait(bar_q, 0, abort_flag, a.status);
            // Issue in dependency order, whichever is ready first: QK^T(q) needs its
            // gathered tile and PV(q-2) already issued (S/P buffer reuse); PV(p) needs
            // the softmax of tile p.  PV is preferred: it frees a gather stage.
            int qk = 0, pv = 0;
            uint64_t t_last = globaltimer_ns();
            uint32_t spins = 0;
            while (ok && pv < ntiles) {
                if (pv < qk && mbar_test(bar_p_full(pv & 1), (pv >> 1) & 1)) {
                    tc_fence_after();
                    const int sb = pv & 1;
                    const uint32_t v_base = sKv + sb * kKvStageBytes + (4 * half) * kKvChunkBytes;
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const uint64_t bd = make_smem_desc(v_base + ks * 2048, kKvChunkBytes, 1024, kSwizzle128B);
                        mma_f16_ts(tmem + kColO, tmem + kColS + 32 * sb + 8 * ks, bd, kIdescPV,
                                   (pv > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(bar_kv_empty(sb));
                    ++pv;
                    t_last = globaltimer_ns();
                } else if (qk < ntiles && qk <= pv + 1 && mbar_test(bar_kv_full(qk & 1), (qk >> 1) & 1)) {
                    tc_fence_after();
                    const int st = qk & 1;
                    const uint32_t d = tmem + kColS + 32 * st;
                    const uint32_t k_base = sKv + st * kKvStageBytes;
#pragma unroll 1
                    for (int c = 0; c < kChunks; ++c) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = make_smem_desc(sQ + c * kQChunkBytes + kk * 32, 16, 1024, kSwizzle128B);
                            const uint64_t bd = make_smem_desc(k_base + c * kKvChunkBytes + kk * 32, 16, 1024, kSwizzle128B);
                            mma_f16_ss(d, ad, bd, kIdescQK, (c | kk) ? 1u : 0u);
                        }
                    }
                    mma_commit(bar_s_full(st));
                    ++qk;
                    t_last = globaltimer_ns();
                } else if ((++spins & 255u) == 0) {
                    if (*abort_flag) {
                        ok = false;
                    } else if (globaltimer_ns() - t_last > kWaitBudgetNs) {
                        record_status(a.status, DSA_STATUS_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                    }
                }
            }
            if (ok) mma_commit(bar_o);
            if (!ok && pv > 0)
                mbar_wait(bar_kv_empty((pv - 1) & 1), ((pv - 1) >> 1) & 1, nullptr, nullptr, 50000000ull);
        }
    } else if (warp >= 5) {
        // ------------------------------------------------ gather producers
        const int p = tid - 5 * 32;  // 0..127
        for (int i = 0; i < ntiles; ++i) {
            const int st = i & 1;
            if (i >= kStages && !mbar_wait(bar_kv_empty(st), ((i >> 1) - 1) & 1, abort_flag, a.status)) break;
            // keep the L2 prefetch kPrefetchTiles tiles ahead of the gather (each CTA of
            // the value pair takes every other row)
            if (p < kTileRows && i + kPrefetchTiles < ntiles && (p & 1) == half) {
                const int s = sidx[(i + kPrefetchTiles) * kTileRows + p];
                if (s >= 0) l2_prefetch_bulk(kv_seq + (int64_t)s * kDK, kDK * 2);
            }
            const uint32_t stage = sKv + st * kKvStageBytes;
            const int32_t* tile_idx = sidx + i * kTileRows;
            uint4 v[kGranules / kGatherThreads];
#pragma unroll
            for (int u = 0; u < kGranules / kGatherThreads; ++u) {
                const int G = p + u * kGatherThreads;
                const int r = G / 72, c = G % 72;
                const int s = tile_idx[r];
                if (s >= 0) {
                    v[u] = __ldg(reinterpret_cast<const uint4*>(kv_seq + (int64_t)s * kDK) + c);
                } else {
                    v[u] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int u = 0; u < kGranules / kGatherThreads; ++u) {
                const int G = p + u * kGatherThreads;
                const int r = G / 72, c = G % 72;
                const int chunk = c >> 3, g = c & 7;
                const uint32_t dst = stage + chunk * kKvChunkBytes + (r >> 3) * 1024 + (r & 7) * 128 + ((g ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[u].x), "r"(v[u].y),
                             "r"(v[u].z), "r"(v[u].w)
                             : "memory");
            }
            fence_proxy_async_smem();
            mbar_arrive(bar_kv_full(st));
        }
    } else {
        // ------------------------------------------------ softmax, one head per thread
        const int h = tid;  // warps 0..3 -> TMEM lanes 0..127
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        const float scale_log2 = a.softmax_scale * 1.4426950408889634f;
        float m_used = -CUDART_INF_F;
        float l = 0.f;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int sb = i & 1;
            const unsigned valid = __ballot_sync(0xffffffffu, sidx[i * kTileRows + lane] >= 0);
            ok = mbar_wait(bar_s_full(sb), (i >> 1) & 1, abort_flag, a.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[32];
            tmem_ld32(lane_addr + kColS + 32 * sb, sv);
            tmem_wait_ld();
            float x[32];
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                x[c] = ((valid >> c) & 1u) ? __uint_as_float(sv[c]) * scale_log2 : -CUDART_INF_F;
                mx = fmaxf(mx, x[c]);
            }
            if (mx > m_used + kRescaleThreshold) {
                if (m_used != -CUDART_INF_F) {
                    // O holds data scaled by 2^-m_used: wait until PV(i-1) landed, then rescale it
                    const float alpha = fast_exp2(m_used - mx);
                    ok = mbar_wait(bar_kv_empty((i - 1) & 1), ((i - 1) >> 1) & 1, abort_flag, a.status);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int c0 = 0; c0 < 256; c0 += 32) {
                        uint32_t ov[32];
                        tmem_ld32(lane_addr + kColO + c0, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
                        tmem_st32(lane_addr + kColO + c0, ov);
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
            tmem_st16(lane_addr + kColS + 32 * sb, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p_full(sb));
        }
        // ---- epilogue
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const float lse_v = l > 0.f ? (m_used + __log2f(l)) * 0.6931471805599453f : -CUDART_INF_F;
        const bool have_o = ok && ntiles > 0;
        if (have_o) {
            ok = mbar_wait(bar_o, 0, abort_flag, a.status);
            ok = __all_sync(0xffffffffu, ok);
        }
        const int64_t th = (int64_t)t * kHeads + h;
        if (a.splits == 1) {
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + th * kDV + half * 256;
            if (half == 0 && a.lse) a.lse[th] = lse_v;
            if (have_o && ok) tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < 256; c0 += 32) {
                uint32_t ov[32];
                if (have_o && ok) {
                    tmem_ld32(lane_addr + kColO + c0, ov);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) ov[c] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    pk[c] = pack_bf16x2(__uint_as_float(ov[2 * c]) * inv_l, __uint_as_float(ov[2 * c + 1]) * inv_l);
                uint4* dst = reinterpret_cast<uint4*>(o + c0);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
            }
        } else {
            float* o = a.part_o + ((int64_t)split * a.Nq * kHeads + th) * kDV + half * 256;
            if (half == 0) a.part_lse[(int64_t)split * a.Nq * kHeads + th] = lse_v;
            if (have_o && ok) tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < 256; c0 += 32) {
                uint32_t ov[32];
                if (have_o && ok) {
                    tmem_ld32(lane_addr + kColO + c0, ov);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) ov[c] = 0u;
                }
                float4* dst = reinterpret_cast<float4*>(o + c0);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                    dst[q4] = make_float4(__uint_as_float(ov[4 * q4]) * inv_l, __uint_as_float(ov[4 * q4 + 1]) * inv_l,
                                          __uint_as_float(ov[4 * q4 + 2]) * inv_l, __uint_as_float(ov[4 * q4 + 3]) * inv_l);
            }
        }
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
    const int64_t plane = (int64_t)a.Nq * kHeads;
    const int64_t th = (int64_t)t * kHeads + h;
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
    alignas(64) CUtensorMap tq;
    if (!encode_tensor_map_2d(&tq, 2, a.q, kDK, (uint64_t)a.Nq * kHeads, kDK * 2, 64, kHeads, 128))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(a.splits, 2, a.Nq);
    sparse_mla_bf16_kernel<<<grid, kThreads, kSmemBytes, st>>>(a, tq);
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
    if (a.Nq == 0 || a.splits <= 1) return cudaSuccess;
    if (a.splits > 16) return cudaErrorInvalidValue;
    mla_combine_kernel<<<dim3(kHeads, a.Nq), 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
