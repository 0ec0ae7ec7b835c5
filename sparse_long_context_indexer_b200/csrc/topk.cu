// topk.cu -- per-query causal top-k over indexer scores.
//
// What it computes ("DeepSeek Sparse Attention Explained", section "How Does
// the Selector Pick 1,024?"): for query row t with n = q_len[t] candidates,
// the min(k, n) positions with the highest scores, redone for every query.
// Order: score descending, ties to the lower position, -0.0 == +0.0.  The
// positions are written in ascending order and padded with -1.
//
// Method: each score becomes an order-preserving 32-bit key; a radix select
// over three digits (11, 11, 10 bits, most significant first) finds the
// k-th largest key tau and how many keys equal to tau must be taken.  A row is
// split across a thread-block cluster of C CTAs (C <= 8): every CTA keeps its
// slice of the row in shared memory, builds a digit histogram with warp-
// aggregated shared atomics (match_any + ballot), and the C histograms are
// merged through distributed shared memory.  A final pass compacts the
// selected positions in order with block-wide scans; CTA r learns from the
// lower-ranked CTAs how many ties and outputs precede it, which gives the
// deterministic lower-index tie rule across the whole row.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "status.cuh"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kBins = 2048;
constexpr int kOffHist = 0;              // 2 x kBins (ping-pong, read remotely)
constexpr int kOffTot = 2 * kBins;       // kBins merged histogram
constexpr int kOffMisc = 3 * kBins;      // 64 words: counts, scan scratch, results
constexpr int kOffKeys = 3 * kBins + 64; // cached keys
constexpr int kBaseWords = kOffKeys;

__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 ranks as +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one int per thread (kThreads threads).
// scratch: >= 33 ints of shared memory.  Returns the exclusive prefix; *total
// receives the block sum.  Must be called by every thread of the block.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wv = scratch[lane];
        int wi = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        scratch[lane] = wi - wv;
        if (lane == 31) scratch[32] = wi;
    }
    __syncthreads();
    const int r = scratch[warp] + incl - v;
    *total = scratch[32];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kThreads, 1) topk_radix_kernel(const TopkArgs a, int cached_cap) {
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    extern __shared__ uint32_t sm[];
    uint32_t* tot = sm + kOffTot;
    int* misc = reinterpret_cast<int*>(sm + kOffMisc);
    int* scan_scratch = misc + 16;
    uint32_t* keys = sm + kOffKeys;
    const int tid = threadIdx.x;
    const int lane = tid & 31;

    const int t = blockIdx.y;
    int n = a.q_len[t];
    if (n < 0 || n > a.T_max || (int64_t)n > a.ld) {
        if (rank == 0 && tid == 0) record_status(a.status, DSA_STATUS_LENGTH);
        n = 0;
    }
    int32_t* out = a.idx + (int64_t)t * a.k;
    if (n <= a.k) {
        // short prompt: everything is selected (same branch for the whole cluster)
        for (int i = rank * kThreads + tid; i < a.k; i += C * kThreads) out[i] = i < n ? i : -1;
        return;
    }

    const float* row = a.scores + (int64_t)t * a.ld;
    const int chunk = (((n + C - 1) / C) + 3) & ~3;
    const int lo = min(n, rank * chunk);
    const int hi = min(n, lo + chunk);
    const int len = hi - lo;
    const bool cached = len <= cached_cap;
    if (cached) {
        const int nv = len >> 2;
        const float4* r4 = reinterpret_cast<const float4*>(row + lo);
        for (int i = tid; i < nv; i += kThreads) {
            const float4 f = __ldg(r4 + i);
            keys[4 * i + 0] = score_key(f.x);
            keys[4 * i + 1] = score_key(f.y);
            keys[4 * i + 2] = score_key(f.z);
            keys[4 * i + 3] = score_key(f.w);
        }
        for (int i = 4 * nv + tid; i < len; i += kThreads) keys[i] = score_key(__ldg(row + lo + i));
    }
    __syncthreads();

    uint32_t prefix = 0, pmask = 0;
    int remaining = a.k;
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
        const int width = p == 2 ? 10 : 11;
        const int sh = p == 0 ? 21 : (p == 1 ? 10 : 0);
        uint32_t* h = sm + kOffHist + (p & 1) * kBins;
        for (int i = tid; i < kBins; i += kThreads) h[i] = 0u;
        __syncthreads();
        const uint32_t dmask = (1u << width) - 1u;
        for (int i0 = 0; i0 < len; i0 += kThreads) {
            const int i = i0 + tid;
            uint32_t kk = 0;
            bool take = false;
            if (i < len) {
                kk = cached ? keys[i] : score_key(__ldg(row + lo + i));
                take = (kk & pmask) == prefix;
            }
            const unsigned act = __ballot_sync(0xffffffffu, take);
            if (take) {
                const uint32_t bin = (kk >> sh) & dmask;
                const unsigned peers = __match_any_sync(act, bin);
                if (lane == __ffs(peers) - 1) atomicAdd(&h[bin], (uint32_t)__popc(peers));
            }
        }
        cluster.sync();
        for (int i = tid; i < kBins; i += kThreads) {
            uint32_t s = 0;
            for (int r = 0; r < C; ++r) s += cluster.map_shared_rank(h, r)[i];
            tot[i] = s;
        }
        __syncthreads();
        // locate the digit holding the remaining-th largest key (scan from the top digit down)
        const int nb = 1 << width;
        const int d1 = nb - 1 - 2 * tid, d0 = nb - 2 - 2 * tid;
        const int c1 = d1 >= 0 ? (int)tot[d1] : 0;
        const int c0 = d0 >= 0 ? (int)tot[d0] : 0;
        int tsum;
        const int before = block_exclusive_scan(c1 + c0, scan_scratch, &tsum);
        if (d1 >= 0 && before < remaining && remaining <= before + c1) {
            misc[0] = d1;
            misc[1] = before;
        } else if (d0 >= 0 && before + c1 < remaining && remaining <= before + c1 + c0) {
            misc[0] = d0;
            misc[1] = before + c1;
        }
        __syncthreads();
        prefix |= (uint32_t)misc[0] << sh;
        pmask |= dmask << sh;
        remaining -= misc[1];
        __syncthreads();
    }
    const uint32_t tau = prefix;
    const int take_eq_total = remaining;  // keys equal to tau that are selected, lowest positions first

    // per-CTA counts of keys above / equal to tau
    int my_gt = 0, my_eq = 0;
    for (int i = tid; i < len; i += kThreads) {
        const uint32_t kk = cached ? keys[i] : score_key(__ldg(row + lo + i));
        my_gt += kk > tau;
        my_eq += kk == tau;
    }
    int n_gt, n_eq;
    block_exclusive_scan(my_gt, scan_scratch, &n_gt);
    block_exclusive_scan(my_eq, scan_scratch, &n_eq);
    if (tid == 0) {
        misc[2] = n_gt;
        misc[3] = n_eq;
    }
    cluster.sync();
    int eq_before = 0, out_before = 0;
    for (int r = 0; r < rank; ++r) {
        const int* rm = cluster.map_shared_rank(misc, r);
        const int g = rm[2], e = rm[3];
        const int te = max(0, min(take_eq_total - eq_before, e));
        out_before += g + te;
        eq_before += e;
    }
    const int take_eq_local = max(0, min(take_eq_total - eq_before, n_eq));

    // ordered compaction, 4 consecutive elements per thread per round
    int eq_run = 0, sel_run = 0;
    for (int r0 = 0; r0 < len; r0 += 4 * kThreads) {
        const int e0 = r0 + 4 * tid;
        uint32_t kk[4];
        int ceq = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = e0 + u;
            kk[u] = i < len ? (cached ? keys[i] : score_key(__ldg(row + lo + i))) : 0u;
            ceq += (i < len) && kk[u] == tau;
        }
        int eq_tot;
        const int eqp = block_exclusive_scan(ceq, scan_scratch, &eq_tot);
        int eq_seen = eq_run + eqp;
        bool sel[4];
        int csel = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = e0 + u;
            bool s = false;
            if (i < len) {
                if (kk[u] > tau) {
                    s = true;
                } else if (kk[u] == tau) {
                    s = eq_seen < take_eq_local;
                    ++eq_seen;
                }
            }
            sel[u] = s;
            csel += s;
        }
        int sel_tot;
        const int selp = block_exclusive_scan(csel, scan_scratch, &sel_tot);
        int o = out_before + sel_run + selp;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (sel[u]) {
                if (o < a.k) out[o] = lo + e0 + u;
                ++o;
            }
        eq_run += eq_tot;
        sel_run += sel_tot;
    }
    cluster.sync();  // keep this CTA's shared memory alive until every peer has read it
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, int cluster, cudaStream_t st) {
    if (a.Nq == 0) return cudaSuccess;
    if (cluster < 1 || cluster > 8) return cudaErrorInvalidValue;
    const int64_t row_max = a.ld < (int64_t)a.T_max ? a.ld : (int64_t)a.T_max;
    int64_t chunk = (row_max + cluster - 1) / cluster;
    chunk = (chunk + 3) & ~int64_t(3);
    const int cap = (int)(chunk < kTopkSmemKeys ? chunk : kTopkSmemKeys);
    const size_t smem = (size_t)(kBaseWords + cap) * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster, a.Nq, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, topk_radix_kernel, a, cap);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace dsa
