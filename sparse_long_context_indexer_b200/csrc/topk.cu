// topk.cu -- per-query causal top-k over indexer scores.
//
// What it computes ("DeepSeek Sparse Attention Explained", section "How Does
// the Selector Pick 1,024?"): for query row t with n = q_len[t] candidates,
// the min(k, n) positions with the highest scores, redone for every query.
// Order: score descending, ties to the lower position, -0.0 == +0.0.  The
// positions are written in ascending order and padded with -1.
//
// Method: each score becomes an order-preserving 32-bit key; the selection is
// the k-th largest key tau plus how many keys equal to tau are taken.  A row is
// split across a thread-block cluster of C CTAs (C <= 8, or up to 16 one-SM CTAs
// for rows too long for shared memory at 8); every CTA keeps its slice of the
// row in shared memory as keys -- a slice too long for it keeps its first part
// there and reads the rest from global memory in every pass -- and tracks the
// keys' min and max.
//  1. One histogram of 2048 bins over (key - base) >> shift, the shift chosen
//     so that [base, max] fills the bins (the top digits of a float key --
//     sign and exponent -- put most scores of a row in a handful of bins, so
//     fixed digits would need several full passes).  base is the row's
//     minimum key, raised to 2^-8 of its largest score when that is positive
//     (keys below count in bin 0; if the threshold lands there the histogram
//     is rebuilt from the minimum).  Every CTA of the cluster then finds the
//     threshold bin b* itself: the 64 coarse totals (groups of 32 bins) of
//     all CTAs, read through distributed shared memory, give the group that
//     holds the k-th largest key, and that group's 32 bins of all CTAs give b*.
//  2. The keys of bin b* are collected (usually a few dozen); every CTA
//     gathers all of them from the cluster and finds tau itself: with at most
//     64 of them warp 0 ranks them directly (and also sets every rank's counts
//     and the compaction's slots), otherwise it refines with 2048-bin histograms
//     of the bits below the bin's base (at most two levels).  If bin b* holds
//     more than kCandMax keys (extremely
//     concentrated scores) the kernel falls back to a radix select over four
//     8-bit digits of all keys (warp-private histograms with match_any
//     aggregation, merged across the cluster).  Rows whose keys are all equal
//     take the first k positions directly.
//  3. A final pass compacts the selected positions in position order: each warp
//     owns a contiguous segment of the CTA's keys and writes its selected
//     positions, with ballots ranking the keys inside each step.  Its counts
//     come from the candidate pass of step 2, which reads the same segments
//     (keys above b*, and its own candidates against tau); the rare paths
//     without that pass (all-equal rows, the radix fallback) count first.
//     CTA r knows from the gathered threshold-bin keys how many ties and
//     outputs the lower-ranked CTAs hold, which gives the lower-index tie rule
//     across the whole row.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

// Cluster sizes up to 8 are planned for every launch; rows whose slices would not fit shared
// memory at that size may take up to 16 one-SM CTAs (a non-portable cluster size).
constexpr int kMaxCluster = 16;
static_assert(kMaxCluster >= kTopkMaxCluster && 26 + kMaxCluster < 64, "cluster offsets fit the misc words");
constexpr int kBins = 256;
constexpr int kLoadBatch = 8;  // 16-byte score loads in flight per thread
constexpr int kFineBits = 11;
constexpr int kFineBins = 1 << kFineBits;  // adaptive histogram bins
constexpr int kCandMax = 2048;             // threshold-bin keys resolved on chip by every CTA
constexpr int kRankMax = 64;               // up to this many, tau is found by direct ranking
constexpr uint32_t kFloorOctaves = 8;      // the first histogram's floor: 2^-8 of the row's largest score
constexpr int kMiscAbove = 48;             // misc words 48 .. 63: every rank's keys above b* (local copies)
static_assert(kMiscAbove >= 26 + 16 + 1 && kMiscAbove + 16 <= 64, "the copies fit beside the cluster offsets");

// Shared-memory map (32-bit words) of a CTA of T threads.  512-thread CTAs fit two per SM
// (launches with more rows than one wave holds); 1024-thread CTAs take a whole SM (launches
// whose clusters all fit one wave: decode).
template <int T>
struct TopkLayout {
    static constexpr int kWarps = T / 32;
    static constexpr int kOffPriv = 0;                          // kWarps x kBins warp-private histograms
    static constexpr int kOffHist = kOffPriv + kWarps * kBins;  // 2 x kBins per-CTA histogram (ping-pong, read remotely)
    static constexpr int kOffTot = kOffHist + 2 * kBins;        // kBins cluster-wide histogram
    static constexpr int kOffMisc = kOffTot + kBins;            // 64 words: results, counts (read remotely)
    static constexpr int kOffScan = kOffMisc + 64;              // block-scan and compaction scratch
    static constexpr int kScanWords = 4 * kWarps + 16;
    static constexpr int kOffFine = (kOffScan + kScanWords + 3) & ~3;  // kFineBins counts (read remotely)
    static constexpr int kOffRange = kOffFine + kFineBins;            // coarse totals (this CTA's, read remotely; the cluster's)
    static constexpr int kOffGather = kOffRange + kFineBins;          // all candidates of the row
    static constexpr int kOffKeys = (kOffGather + kCandMax + 3) & ~3;
    static constexpr int kBaseWords = kOffKeys;
    static_assert(kWarps * kBins >= 2 * kCandMax,
                  "the local candidate list and its warps live in the warp-private histograms");
};

__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 ranks as +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one int per thread.  scratch >= kWarps + 1 ints.
template <int T>
__device__ __forceinline__ int block_scan1(int v, int* scratch, int* total) {
    constexpr int kWarps = T / 32;
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
        const int wv = lane < kWarps ? scratch[lane] : 0;
        int wi = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < kWarps) scratch[lane] = wi - wv;
        if (lane == 31) scratch[kWarps] = wi;
    }
    __syncthreads();
    const int r = scratch[warp] + incl - v;
    *total = scratch[kWarps];
    __syncthreads();
    return r;
}

// BATCH: some rows' slices exceed the shared-memory cache, so their passes read the scores
// past the cached first part of the slice from global memory (L2); those reads go out 16 bytes
// and U steps at a time per thread (one CTA per SM then, for the registers).  Launches whose
// slices all fit compile without it.
template <int T, bool BATCH>
__global__ void __launch_bounds__(T, (T == 512 && !BATCH) ? 2 : 1) topk_radix_kernel(const TopkArgs a, int cached_cap) {
    using L = TopkLayout<T>;
    constexpr int U = BATCH ? 4 : 1;  // steps of every pass loaded before any is used
    constexpr int kMaxC = BATCH ? kMaxCluster : kTopkMaxCluster;  // cluster size bound of this variant
    constexpr int kThreads = T;
    constexpr int kWarps = L::kWarps;
    constexpr int kOffPriv = L::kOffPriv, kOffHist = L::kOffHist, kOffTot = L::kOffTot, kOffMisc = L::kOffMisc;
    constexpr int kOffScan = L::kOffScan, kOffFine = L::kOffFine, kOffRange = L::kOffRange;
    constexpr int kOffGather = L::kOffGather, kOffKeys = L::kOffKeys;
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    extern __shared__ uint32_t sm[];
    uint32_t* priv = sm + kOffPriv;
    uint32_t* tot = sm + kOffTot;
    int* misc = reinterpret_cast<int*>(sm + kOffMisc);
    int* scr = reinterpret_cast<int*>(sm + kOffScan);
    uint32_t* keys = sm + kOffKeys;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_launch_dependents();  // the attention kernel may start its setup on free SMs

    const int t = blockIdx.y;
    int n = a.q_len[t];
    if (n < 0 || n > a.T_max || (int64_t)n > a.ld) {
        if (rank == 0 && tid == 0) record_status(a.status, DSA_STATUS_LENGTH);
        n = 0;
    }
    int32_t* out = a.idx + (int64_t)t * a.k;
    if (n <= a.k) {
        // short prompt: everything is selected (same branch for the whole cluster); the
        // previous kernel may still be writing the workspace this output may live in
        griddep_wait();
        for (int i = rank * kThreads + tid; i < a.k; i += C * kThreads) out[i] = i < n ? i : -1;
        return;
    }

    // the score rows come from the previous kernel (programmatic dependent launch)
    griddep_wait();
    const float* row = a.scores + (int64_t)t * a.ld;
    const int chunk = (((n + C - 1) / C) + 3) & ~3;
    const int lo = min(n, rank * chunk);
    const int hi = min(n, lo + chunk);
    const int len = hi - lo;
    const bool cached = len <= cached_cap;
    // keys kept in shared memory: the whole slice when it fits; otherwise (the variant that
    // streams from global memory) its first cached_cap keys, so that every later pass reads
    // only the rest of the slice from L2
    const int ncache = cached ? len : (BATCH ? (cached_cap & ~3) : 0);
    if (tid == 0) {
        misc[4] = -1;  // key min (as uint32), max
        misc[5] = 0;
        misc[13] = 0;  // local candidate count
    }
    __syncthreads();
    uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
    if (cached) {
        // 16-byte loads, eight in flight per thread (a 16 K-key slice in one round trip), keys
        // written in place
        const int nv = len >> 2;
        const float4* r4 = reinterpret_cast<const float4*>(row + lo);
        uint4* k4 = reinterpret_cast<uint4*>(keys);
        for (int i0 = 0; i0 < nv; i0 += kLoadBatch * kThreads) {
            float4 f[kLoadBatch];
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) {
                const int i = i0 + u * kThreads + tid;
                f[u] = i < nv ? __ldg(r4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) {
                const int i = i0 + u * kThreads + tid;
                if (i < nv) {
                    const uint4 kk = make_uint4(score_key(f[u].x), score_key(f[u].y), score_key(f[u].z), score_key(f[u].w));
                    k4[i] = kk;
                    kmn = min(kmn, min(min(kk.x, kk.y), min(kk.z, kk.w)));
                    kmx = max(kmx, max(max(kk.x, kk.y), max(kk.z, kk.w)));
                }
            }
        }
        for (int i = 4 * nv + tid; i < len; i += kThreads) {
            const uint32_t kk = score_key(__ldg(row + lo + i));
            keys[i] = kk;
            kmn = min(kmn, kk);
            kmx = max(kmx, kk);
        }
    } else if constexpr (BATCH) {
        // the same 16-byte loads, eight in flight per thread, the first ncache keys kept
        const int nv = len >> 2;
        const int nc4 = ncache >> 2;
        const float4* r4 = reinterpret_cast<const float4*>(row + lo);
        uint4* k4 = reinterpret_cast<uint4*>(keys);
        for (int i0 = 0; i0 < nv; i0 += kLoadBatch * kThreads) {
            float4 f[kLoadBatch];
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) {
                const int i = i0 + u * kThreads + tid;
                f[u] = i < nv ? __ldg(r4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) {
                const int i = i0 + u * kThreads + tid;
                if (i < nv) {
                    const uint32_t k0 = score_key(f[u].x), k1 = score_key(f[u].y), k2 = score_key(f[u].z),
                                   k3 = score_key(f[u].w);
                    if (i < nc4) k4[i] = make_uint4(k0, k1, k2, k3);
                    kmn = min(kmn, min(min(k0, k1), min(k2, k3)));
                    kmx = max(kmx, max(max(k0, k1), max(k2, k3)));
                }
            }
        }
        for (int i = 4 * nv + tid; i < len; i += kThreads) {
            const uint32_t kk = score_key(__ldg(row + lo + i));
            kmn = min(kmn, kk);
            kmx = max(kmx, kk);
        }
    } else {
        for (int i = tid; i < len; i += kThreads) {
            const uint32_t kk = score_key(__ldg(row + lo + i));
            kmn = min(kmn, kk);
            kmx = max(kmx, kk);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmn = min(kmn, __shfl_xor_sync(0xffffffffu, kmn, o));
        kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, o));
    }
    if (lane == 0) {
        atomicMin(reinterpret_cast<unsigned*>(misc + 4), kmn);
        atomicMax(reinterpret_cast<unsigned*>(misc + 5), kmx);
    }
    auto key_at = [&](int i) -> uint32_t { return i < ncache ? keys[i] : score_key(__ldg(row + lo + i)); };
    // the 4 consecutive keys starting at i (a multiple of 4); out-of-range keys read as 0 (never selected:
    // the caller checks i < len)
    auto keys4_at = [&](int i) -> uint4 {
        if (i + 3 < ncache) return reinterpret_cast<const uint4*>(keys)[i >> 2];
        if (BATCH && i + 3 < len) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(row + lo + i));
            return make_uint4(score_key(f.x), score_key(f.y), score_key(f.z), score_key(f.w));
        }
        uint4 r;
        r.x = i < len ? key_at(i) : 0u;
        r.y = i + 1 < len ? key_at(i + 1) : 0u;
        r.z = i + 2 < len ? key_at(i + 2) : 0u;
        r.w = i + 3 < len ? key_at(i + 3) : 0u;
        return r;
    };
    cluster.sync();  // (a cluster barrier orders this CTA's own shared memory as well)
    // the row's key range: lane r of warp 0 reads CTA r's min and max (one remote read each,
    // instead of every thread reading every rank), shared through this CTA's memory
    if (warp == 0) {
        uint32_t mn = 0xFFFFFFFFu, mx = 0u;
        if (lane < C) {
            const int* rm = cluster.map_shared_rank(misc, lane);
            mn = (uint32_t)rm[4];
            mx = (uint32_t)rm[5];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (lane == 0) {
            misc[22] = (int)mn;
            misc[23] = (int)mx;
        }
    }
    __syncthreads();
    const uint32_t kmin = (uint32_t)misc[22], kmax = (uint32_t)misc[23];

    uint32_t tau;
    int take_eq_total;  // keys equal to tau that are selected, lowest positions first
    int local_gt = 0;   // keys of this CTA above tau
    int local_eq = 0;   // keys of this CTA equal to tau
    int eq_before = 0, out_before = 0;  // ties / outputs of the lower ranks
    bool counts_done = false;           // (cluster-uniform) the lower ranks' counts are known
    bool warp_counts = false;           // (block-uniform) scr holds every warp's counts for the compaction
    bool slots_done = false;            // (block-uniform) scr holds every warp's first tie rank and slot
    // Warp 0, lane w: from warp w's keys above tau (scr[w]) and equal to it (scr[kWarps + w]),
    // warp w's first tie rank (scr[2 kWarps + w]) and first output slot (scr[3 kWarps + w]).
    auto warp_slots = [&](int take_eq_local, int first_out) {
        const int g = lane < kWarps ? scr[lane] : 0;
        const int e = lane < kWarps ? scr[kWarps + lane] : 0;
        int e_incl = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, e_incl, o);
            if (lane >= o) e_incl += v;
        }
        const int e_excl = e_incl - e;
        const int taken = g + max(0, min(take_eq_local - e_excl, e));
        int t_incl = taken;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, t_incl, o);
            if (lane >= o) t_incl += v;
        }
        if (lane < kWarps) {
            scr[2 * kWarps + lane] = e_excl;
            scr[3 * kWarps + lane] = first_out + t_incl - taken;
        }
    };
    if (kmin == kmax) {
        // every key of the row is equal: the first k positions
        tau = kmin;
        take_eq_total = a.k;
        local_eq = len;
    } else {
        // ---- 1. adaptive histogram over the row's key range, its coarse and fine totals
        // over the cluster, threshold bin b*.  The bins cover [kbase, kmax]: kbase is the row's minimum,
        // raised to 2^-kFloorOctaves of the largest score when that is positive (the k-th
        // largest score of a row almost always lies within those octaves of the largest, and
        // the narrower range leaves a few keys in b* instead of hundreds); keys below kbase
        // count in bin 0.  Should b* be bin 0 all the same, the histogram is rebuilt over the
        // full range.
        constexpr uint32_t kFloorStep = kFloorOctaves << 23;  // the exponent field of a key
        uint32_t kbase = kmin;
        if (kmax > 0x80000000u + kFloorStep && kmax - kFloorStep > kmin) kbase = kmax - kFloorStep;
        int shift = 0;
        auto bin_of = [&](uint32_t kk) -> int {
            return kk <= kbase ? 0 : min(kFineBins - 1, (int)((kk - kbase) >> shift));
        };
        uint32_t* fine = sm + kOffFine;
        constexpr int kGroup = kFineBins / 64;  // bins per coarse group (one per lane)
        static_assert(kGroup == 32, "a coarse group is one warp's worth of bins");
        uint32_t* coarse = sm + kOffRange;       // this CTA's 64 coarse totals (read by every peer)
        uint32_t* ctot = coarse + 64;            // the cluster's coarse totals
        uint32_t* ftot = coarse + 128;           // the cluster's totals of one group's bins
#pragma unroll 1
        while (true) {
        shift = max(0, 32 - __clz((int)(kmax - kbase)) - kFineBits);
        for (int i = tid; i < kFineBins; i += kThreads) fine[i] = 0u;
        __syncthreads();
        // keys at or below the base (most of a row's keys once the base is raised) are counted
        // in registers: one shared-memory address taking every one of them serialises the atomics
        int below = 0;
        if constexpr (U == 1) {
            for (int i0 = 4 * tid; i0 < len; i0 += 4 * kThreads) {
                const uint4 k4 = keys4_at(i0);
                const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (i0 + u < len) {
                        if (kv[u] <= kbase)
                            ++below;
                        else
                            atomicAdd(&fine[bin_of(kv[u])], 1u);
                    }
                }
            }
        } else {
#pragma unroll 1
            for (int i00 = 4 * tid; i00 < len; i00 += 4 * kThreads * U) {
                uint4 kq[U];
#pragma unroll
                for (int uu = 0; uu < U; ++uu) kq[uu] = keys4_at(i00 + uu * 4 * kThreads);
#pragma unroll
                for (int uu = 0; uu < U; ++uu) {
                    const int i0 = i00 + uu * 4 * kThreads;
                    const uint32_t kv[4] = {kq[uu].x, kq[uu].y, kq[uu].z, kq[uu].w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (i0 + u < len) {
                            if (kv[u] <= kbase)
                                ++below;
                            else
                                atomicAdd(&fine[bin_of(kv[u])], 1u);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
        if (lane == 0 && below > 0) atomicAdd(&fine[0], (uint32_t)below);
        __syncthreads();
        // this CTA's coarse totals: 64 groups of kGroup consecutive bins (read by every peer)
        for (int g = warp; g < 64; g += kWarps) {
            const uint32_t v = __reduce_add_sync(0xffffffffu, fine[g * kGroup + lane]);
            if (lane == 0) coarse[g] = v;
        }
        cluster.sync();
        // Every CTA finds b* itself from the same totals: the coarse group holding the k-th
        // largest key (groups summed over the cluster), then that group's bins, summed over the
        // cluster the same way.  Peers read this CTA's coarse and fine totals until the next
        // cluster barrier, so neither is written before it.
        if (tid < 64) {
            uint32_t tot = 0u;
#pragma unroll
            for (int r = 0; r < kMaxC; ++r) tot += r < C ? cluster.map_shared_rank(coarse, r)[tid] : 0u;
            ctot[tid] = tot;
        }
        __syncthreads();
        if (warp == 0) {
            // lane l holds groups 63 - 2l and 62 - 2l: lanes in descending key order
            const int v_hi = (int)ctot[63 - 2 * lane], v_lo = (int)ctot[62 - 2 * lane];
            const int v = v_hi + v_lo;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            const int excl = incl - v;
            const unsigned m = __ballot_sync(0xffffffffu, excl < a.k && a.k <= incl);
            if (m != 0u && lane == __ffs(m) - 1) {
                const bool upper = a.k <= excl + v_hi;
                misc[24] = upper ? 63 - 2 * lane : 62 - 2 * lane;
                misc[25] = upper ? excl : excl + v_hi;
            }
        }
        __syncthreads();
        const int grp = misc[24], above_g = misc[25];
        if (tid < kGroup) {
            uint32_t tot = 0u;
#pragma unroll
            for (int r = 0; r < kMaxC; ++r) tot += r < C ? cluster.map_shared_rank(fine, r)[grp * kGroup + tid] : 0u;
            ftot[tid] = tot;
        }
        __syncthreads();
        if (warp == 0) {
            // lane j holds bin grp * kGroup + kGroup - 1 - j: descending again
            const int v = (int)ftot[kGroup - 1 - lane];
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            const int excl = incl - v;
            const int need = a.k - above_g;
            const unsigned m = __ballot_sync(0xffffffffu, excl < need && need <= incl);
            if (m != 0u && lane == __ffs(m) - 1) {
                misc[8] = grp * kGroup + kGroup - 1 - lane;
                misc[9] = above_g + excl;
                misc[10] = v;
            }
        }
        __syncthreads();
        // the same b* in every CTA of the cluster (read from the same totals): a uniform exit
        if (misc[8] != 0 || kbase == kmin) break;
        // b* fell to the floor bin: rebuild over the full range once every peer has read this
        // CTA's coarse and fine totals
        kbase = kmin;
        cluster.sync();
        }
        const int bstar = misc[8];
        const int above_total = misc[9];
        const int Tc = misc[10];
        // this CTA's keys in bins above b*
        int la = 0;
        for (int bb = bstar + 1 + tid; bb < kFineBins; bb += kThreads) la += (int)fine[bb];
        int latot;
        block_scan1<T>(la, scr, &latot);
        if (tid == 0) misc[7] = latot;  // read by the higher ranks after the candidate barrier
        if (Tc <= kCandMax) {
            // ---- 2. the keys of bin b*: every CTA gathers them all and finds tau itself.  Each
            // warp reads the segment of keys it compacts at the end (see below), counts its keys
            // above b* (all above tau) and records with each of its candidates its warp, so that
            // the compaction needs no counting pass of its own.
            uint32_t* cand = priv;
            uint32_t* cand_w = priv + kCandMax;
            {
                const int seg = ((len + kWarps - 1) / kWarps + 127) & ~127;
                const int w_lo = min(len, warp * seg), w_hi = min(len, w_lo + seg);
                int above = 0;
#pragma unroll 1
                for (int base0 = w_lo; base0 < w_hi; base0 += 128 * U) {
                    uint4 kq[U];
#pragma unroll
                    for (int uu = 0; uu < U; ++uu) kq[uu] = keys4_at(base0 + uu * 128 + 4 * lane);
#pragma unroll
                    for (int uu = 0; uu < U; ++uu) {
                        const int i0 = base0 + uu * 128 + 4 * lane;
                        const uint32_t kv[4] = {kq[uu].x, kq[uu].y, kq[uu].z, kq[uu].w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (i0 + u < w_hi) {
                                const int bb = bin_of(kv[u]);
                                if (bb > bstar) {
                                    ++above;
                                } else if (bb == bstar) {
                                    const int slot = atomicAdd(misc + 13, 1);
                                    cand[slot] = kv[u];
                                    cand_w[slot] = (uint32_t)warp;
                                }
                            }
                        }
                    }
                }
                above = __reduce_add_sync(0xffffffffu, above);
                if (lane == 0) scr[2 * kWarps + warp] = above;  // block_scan1 uses scr[0 .. kWarps] only
            }
            cluster.sync();
            uint32_t* gbuf = sm + kOffGather;
            // every CTA's candidate count (lane r of warp 0 reads CTA r's) and their offsets in
            // the gathered list, then all copies at once
            if (warp == 0) {
                const int* rm = cluster.map_shared_rank(misc, lane < C ? lane : 0);
                const int c = lane < C ? rm[13] : 0;
                // each rank's keys above b* come along (used for the counts once tau is known)
                if (lane < C) misc[kMiscAbove + lane] = rm[7];
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += u;
                }
                if (lane < kMaxC) misc[26 + lane] = incl - c;
                if (lane == 31) misc[26 + kMaxC] = incl;
            }
            __syncthreads();
            const int off = misc[26 + kMaxC];
            for (int i = tid; i < off; i += kThreads) {
                int r = 0, base = 0;
#pragma unroll
                for (int q = 1; q < kMaxC; ++q) {
                    const int oq = misc[26 + q];
                    if (q < C && i >= oq) {
                        r = q;
                        base = oq;
                    }
                }
                gbuf[i] = cluster.map_shared_rank(cand, r)[i - base];
            }
            __syncthreads();
            if (off <= kRankMax) {
                // A few candidates, two per lane of warp 0, which alone finds tau, every rank's
                // counts, this CTA's per-warp counts and the compaction's slots; the other warps
                // wait at one barrier.  tau is the candidate c with #{> c} < rem <= #{>= c}, found
                // by ranking every candidate against all others.
                if (warp == 0) {
                    const int rem = a.k - above_total;
                    const bool v0 = lane < off, v1 = lane + 32 < off;
                    const uint32_t c0 = v0 ? gbuf[lane] : 0u;
                    const uint32_t c1 = v1 ? gbuf[lane + 32] : 0u;
                    int gt0 = 0, ge0 = 0, gt1 = 0, ge1 = 0;
                    const int n0 = min(off, 32);
#pragma unroll 4
                    for (int j = 0; j < n0; ++j) {
                        const uint32_t o = __shfl_sync(0xffffffffu, c0, j);
                        gt0 += o > c0;
                        ge0 += o >= c0;
                        gt1 += o > c1;
                        ge1 += o >= c1;
                    }
#pragma unroll 4
                    for (int j = 0; j < off - 32; ++j) {
                        const uint32_t o = __shfl_sync(0xffffffffu, c1, j);
                        gt0 += o > c0;
                        ge0 += o >= c0;
                        gt1 += o > c1;
                        ge1 += o >= c1;
                    }
                    // every copy of tau has the same counts: take the first
                    const unsigned h0 = __ballot_sync(0xffffffffu, v0 && gt0 < rem && rem <= ge0);
                    const unsigned h1 = __ballot_sync(0xffffffffu, v1 && gt1 < rem && rem <= ge1);
                    const int src = h0 ? __ffs(h0) - 1 : __ffs(h1) - 1;
                    const uint32_t t = __shfl_sync(0xffffffffu, h0 ? c0 : c1, src);
                    const int take_eq = rem - __shfl_sync(0xffffffffu, h0 ? gt0 : gt1, src);
                    // bit i of mgt / meq: candidate gbuf[i] is above / equal to tau; rank r's
                    // candidates are gbuf[misc[26 + r], misc[27 + r]), lane r counts rank r
                    const uint64_t mgt = (uint64_t)__ballot_sync(0xffffffffu, v1 && c1 > t) << 32 |
                                         __ballot_sync(0xffffffffu, v0 && c0 > t);
                    const uint64_t meq = (uint64_t)__ballot_sync(0xffffffffu, v1 && c1 == t) << 32 |
                                         __ballot_sync(0xffffffffu, v0 && c0 == t);
                    int g = 0, e = 0;
                    if (lane < C) {
                        const int b0 = misc[26 + lane], b1 = misc[27 + lane];
                        const uint64_t below0 = b0 >= 64 ? ~0ull : (1ull << b0) - 1ull;
                        const uint64_t below1 = b1 >= 64 ? ~0ull : (1ull << b1) - 1ull;
                        g = misc[kMiscAbove + lane] + __popcll(mgt & below1 & ~below0);
                        e = __popcll(meq & below1 & ~below0);
                    }
                    int e_incl = e;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int u = __shfl_up_sync(0xffffffffu, e_incl, o);
                        if (lane >= o) e_incl += u;
                    }
                    const int e_excl = e_incl - e;
                    int ob = lane < rank ? g + max(0, min(take_eq - e_excl, e)) : 0;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) ob += __shfl_xor_sync(0xffffffffu, ob, o);
                    const int my_eq = __shfl_sync(0xffffffffu, e, rank);
                    const int my_eq_before = __shfl_sync(0xffffffffu, e_excl, rank);
                    // this CTA's per-warp counts: the warp's keys above b* plus its own candidates
                    // above and equal to tau (local candidate i is cand[i], found by warp cand_w[i])
                    if (lane < kWarps) {
                        scr[lane] = scr[2 * kWarps + lane];
                        scr[kWarps + lane] = 0;
                    }
                    __syncwarp();
                    const int nloc = misc[13];
#pragma unroll
                    for (int i = lane; i < 64; i += 32) {
                        if (i < nloc) {
                            const uint32_t kk = cand[i];
                            if (kk > t)
                                atomicAdd(&scr[cand_w[i]], 1);
                            else if (kk == t)
                                atomicAdd(&scr[kWarps + cand_w[i]], 1);
                        }
                    }
                    __syncwarp();
                    warp_slots(max(0, min(take_eq - my_eq_before, my_eq)), ob);
                    if (lane == 0) {
                        misc[11] = (int)t;
                        misc[12] = take_eq;
                        misc[17] = my_eq;
                        misc[20] = ob;
                        misc[21] = my_eq_before;
                    }
                }
                __syncthreads();
                slots_done = true;
            } else {
                // tau among the candidates (keys in [base, base + 2^shift)): refine by 2048-bin
                // histograms of the bits below the bin base, at most two levels for shift <= 22;
                // this CTA's own fine histogram is free now (peers read it only before the range merge)
                int rem = a.k - above_total;
                uint64_t base = (uint64_t)kbase + ((uint64_t)bstar << shift);
                int sh = shift;
#pragma unroll 1
                while (sh > 0) {
                    const int sh2 = max(0, sh - kFineBits);
                    const int nb = 1 << (sh - sh2);  // <= kFineBins
                    for (int i = tid; i < nb; i += kThreads) fine[i] = 0u;
                    __syncthreads();
                    for (int i = tid; i < off; i += kThreads) {
                        const uint64_t kk = gbuf[i];
                        if (kk >= base && kk < base + (1ull << sh)) atomicAdd(&fine[(uint32_t)((kk - base) >> sh2)], 1u);
                    }
                    __syncthreads();
                    int cb[4], c4 = 0;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int bb = nb - 1 - 4 * tid - u;
                        cb[u] = bb >= 0 ? (int)fine[bb] : 0;
                        c4 += cb[u];
                    }
                    int tsum;
                    const int before = block_scan1<T>(c4, scr, &tsum);
                    if (before < rem && rem <= before + c4) {
                        int run = before;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (run < rem && rem <= run + cb[u]) {
                                misc[14] = nb - 1 - 4 * tid - u;
                                misc[15] = run;
                            }
                            run += cb[u];
                        }
                    }
                    __syncthreads();
                    base += (uint64_t)misc[14] << sh2;
                    rem -= misc[15];
                    sh = sh2;
                    __syncthreads();
                }
                if (tid == 0) {
                    misc[11] = (int)(uint32_t)base;
                    misc[12] = rem;  // candidates equal to tau that are taken
                }
                __syncthreads();
            }
            tau = (uint32_t)misc[11];
            take_eq_total = misc[12];
            // Every rank's counts come from the gathered list (rank r's candidates are
            // gbuf[misc[26 + r], misc[27 + r])) and from its keys above b* (its misc[7]): lane r
            // of warp 0 counts rank r; ties are taken lowest rank first.  No further exchange.
            if (!slots_done && warp == 0) {
                int g = 0, e = 0;
                if (lane < C) {
                    g = misc[kMiscAbove + lane];
                    const int b0 = misc[26 + lane], b1 = misc[27 + lane];
                    for (int i = b0; i < b1; ++i) {
                        g += gbuf[i] > tau;
                        e += gbuf[i] == tau;
                    }
                }
                int e_incl = e;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, e_incl, o);
                    if (lane >= o) e_incl += u;
                }
                const int e_excl = e_incl - e;
                const int te = max(0, min(take_eq_total - e_excl, e));
                int ob = lane < rank ? g + te : 0;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ob += __shfl_xor_sync(0xffffffffu, ob, o);
                if (lane == rank) {
                    misc[16] = g;
                    misc[17] = e;
                    misc[20] = ob;
                    misc[21] = e_excl;
                }
            }
            // every warp's counts for the compaction: its keys above b* plus its own candidates
            // above and equal to tau
            if (!slots_done) {
                if (tid < kWarps) {
                    scr[tid] = scr[2 * kWarps + tid];
                    scr[kWarps + tid] = 0;
                }
                __syncthreads();
                for (int i = tid; i < misc[13]; i += kThreads) {
                    const uint32_t kk = cand[i];
                    if (kk > tau)
                        atomicAdd(&scr[cand_w[i]], 1);
                    else if (kk == tau)
                        atomicAdd(&scr[kWarps + cand_w[i]], 1);
                }
                local_gt = misc[16];
            }
            warp_counts = true;
            local_eq = misc[17];
            out_before = misc[20];
            eq_before = misc[21];
            counts_done = true;
        } else {
            // ---- fallback: radix select over four 8-bit digits of all keys
            uint32_t prefix = 0, pmask = 0;
            int remaining = a.k;
#pragma unroll 1
            for (int p = 0; p < 4; ++p) {
                const int sh = 24 - 8 * p;
                uint32_t* hist = sm + kOffHist + (p & 1) * kBins;
                for (int i = tid; i < kWarps * kBins; i += kThreads) priv[i] = 0u;
                __syncthreads();
                uint32_t* my = priv + warp * kBins;
                for (int i0 = 0; i0 < len; i0 += kThreads) {
                    const int i = i0 + tid;
                    uint32_t kk = 0;
                    bool take = false;
                    if (i < len) {
                        kk = key_at(i);
                        take = (kk & pmask) == prefix;
                    }
                    const unsigned act = __ballot_sync(0xffffffffu, take);
                    if (take) {
                        const uint32_t bin = (kk >> sh) & 0xFFu;
                        const unsigned peers = __match_any_sync(act, bin);
                        if (lane == __ffs(peers) - 1) atomicAdd(&my[bin], (uint32_t)__popc(peers));
                    }
                }
                __syncthreads();
                if (tid < kBins) {
                    uint32_t sum = 0;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) sum += priv[w * kBins + tid];
                    hist[tid] = sum;
                }
                cluster.sync();
                if (tid < kBins) {
                    uint32_t sum_r = 0u;
#pragma unroll
                    for (int r = 0; r < kMaxC; ++r) sum_r += r < C ? cluster.map_shared_rank(hist, r)[tid] : 0u;
                    tot[tid] = sum_r;
                }
                __syncthreads();
                // digit holding the remaining-th largest key: scan from the top digit down
                const int d = kBins - 1 - tid;
                const int c = tid < kBins ? (int)tot[d] : 0;
                int tsum;
                const int before = block_scan1<T>(c, scr, &tsum);
                if (tid < kBins && before < remaining && remaining <= before + c) {
                    misc[0] = d;
                    misc[1] = before;
                }
                __syncthreads();
                const int dsel = misc[0];
                const int above = misc[1];
                // this CTA's keys in digits above the chosen one (same prefix) are above tau
                int atot;
                block_scan1<T>((tid < kBins && d > dsel) ? (int)hist[d] : 0, scr, &atot);
                local_gt += atot;
                if (p == 3) local_eq = (int)hist[dsel];
                prefix |= (uint32_t)dsel << sh;
                pmask |= 0xFFu << sh;
                remaining -= above;
            }
            tau = prefix;
            take_eq_total = remaining;
        }
    }

    if (!counts_done) {
        // all-equal rows and the radix fallback: exchange the counts through the cluster
        if (tid == 0) {
            misc[2] = local_gt;
            misc[3] = local_eq;
        }
        cluster.sync();
        if (warp == 0) {
            // lane r < rank reads CTA r's counts; ties are taken lowest rank first
            int g = 0, e = 0;
            if (lane < rank) {
                const int* rm = cluster.map_shared_rank(misc, lane);
                g = rm[2];
                e = rm[3];
            }
            int e_incl = e;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, e_incl, o);
                if (lane >= o) e_incl += u;
            }
            const int te = max(0, min(take_eq_total - (e_incl - e), e));
            int ob = g + te;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ob += __shfl_xor_sync(0xffffffffu, ob, o);
            if (lane == 31) {
                misc[20] = ob;
                misc[21] = e_incl;  // the ties of all lower ranks
            }
        }
        __syncthreads();
        out_before = misc[20];
        eq_before = misc[21];
    }
    // This thread reads no peer's shared memory from here on: arrive now, wait before exiting
    // (peers may still be reading this CTA's candidates and counts until they arrive).  The
    // arrival is per thread, so no block barrier is needed in front of it.
    cluster_arrive_release();
    const int take_eq_local = max(0, min(take_eq_total - eq_before, local_eq));

    // ordered compaction: warp w owns the contiguous segment [w * seg, w * seg + seg) of this
    // CTA's keys, read four consecutive keys per lane (128 per warp step).  Pass 1 counts each
    // warp's keys above tau and equal to it; one warp turns the counts into the warp's first tie
    // rank and first output slot; pass 2 writes the selected positions in position order
    // (ballots give every key its rank inside the step).  A tie is selected while its rank
    // among this CTA's ties is below take_eq_local.
    {
        const int seg = ((len + kWarps - 1) / kWarps + 127) & ~127;
        const int w_lo = min(len, warp * seg), w_hi = min(len, w_lo + seg);
        if (!warp_counts) {
            int gt = 0, eq = 0;
#pragma unroll 1
            for (int base0 = w_lo; base0 < w_hi; base0 += 128 * U) {  // warp-uniform steps
                uint4 kq[U];
#pragma unroll
                for (int uu = 0; uu < U; ++uu) kq[uu] = keys4_at(base0 + uu * 128 + 4 * lane);
#pragma unroll
                for (int uu = 0; uu < U; ++uu) {
                    const int i0 = base0 + uu * 128 + 4 * lane;
                    const uint32_t kv[4] = {kq[uu].x, kq[uu].y, kq[uu].z, kq[uu].w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const bool in = i0 + u < w_hi;
                        gt += in && kv[u] > tau;
                        eq += in && kv[u] == tau;
                    }
                }
            }
            gt = __reduce_add_sync(0xffffffffu, gt);
            eq = __reduce_add_sync(0xffffffffu, eq);
            if (lane == 0) {
                scr[warp] = gt;
                scr[kWarps + warp] = eq;
            }
        }
        if (!slots_done) {
            __syncthreads();
            if (warp == 0) warp_slots(take_eq_local, out_before);
            __syncthreads();
        }
        int eq_run = scr[2 * kWarps + warp];
        int out_run = scr[3 * kWarps + warp];
        const unsigned lt = (1u << lane) - 1u;
        if (scr[kWarps + warp] == 0) {
            // no key of this warp equals tau: the keys above it, in position order
#pragma unroll 1
            for (int base0 = w_lo; base0 < w_hi; base0 += 128 * U) {  // warp-uniform steps (ballots below)
                uint4 kq[U];
#pragma unroll
                for (int uu = 0; uu < U; ++uu) kq[uu] = keys4_at(base0 + uu * 128 + 4 * lane);
#pragma unroll
                for (int uu = 0; uu < U; ++uu) {
                    const int i0 = base0 + uu * 128 + 4 * lane;
                    const uint32_t kv[4] = {kq[uu].x, kq[uu].y, kq[uu].z, kq[uu].w};
                    unsigned sb[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) sb[u] = __ballot_sync(0xffffffffu, i0 + u < w_hi && kv[u] > tau);
                    if ((sb[0] | sb[1] | sb[2] | sb[3]) == 0u) continue;
                    int o = out_run + __popc(sb[0] & lt) + __popc(sb[1] & lt) + __popc(sb[2] & lt) +
                            __popc(sb[3] & lt);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if ((sb[u] >> lane) & 1u) {
                            if (o < a.k) out[o] = lo + i0 + u;
                            ++o;
                        }
                    }
                    out_run += __popc(sb[0]) + __popc(sb[1]) + __popc(sb[2]) + __popc(sb[3]);
                }
            }
        } else {
#pragma unroll 1
            for (int base0 = w_lo; base0 < w_hi; base0 += 128 * U) {  // warp-uniform steps (ballots below)
                uint4 kq[U];
#pragma unroll
                for (int uu = 0; uu < U; ++uu) kq[uu] = keys4_at(base0 + uu * 128 + 4 * lane);
#pragma unroll
                for (int uu = 0; uu < U; ++uu) {
                    const int i0 = base0 + uu * 128 + 4 * lane;
                    const uint32_t kv[4] = {kq[uu].x, kq[uu].y, kq[uu].z, kq[uu].w};
                    unsigned eb[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) eb[u] = __ballot_sync(0xffffffffu, i0 + u < w_hi && kv[u] == tau);
                    // ties at lower positions in this step: lower lanes (all four keys), then this lane's
                    int eq_before = eq_run + __popc(eb[0] & lt) + __popc(eb[1] & lt) + __popc(eb[2] & lt) +
                                    __popc(eb[3] & lt);
                    bool sel[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const bool in = i0 + u < w_hi;
                        const bool is_eq = (eb[u] >> lane) & 1u;
                        sel[u] = in && (kv[u] > tau || (is_eq && eq_before < take_eq_local));
                        eq_before += is_eq;
                    }
                    eq_run += __popc(eb[0]) + __popc(eb[1]) + __popc(eb[2]) + __popc(eb[3]);
                    unsigned sb[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) sb[u] = __ballot_sync(0xffffffffu, sel[u]);
                    int o = out_run + __popc(sb[0] & lt) + __popc(sb[1] & lt) + __popc(sb[2] & lt) +
                            __popc(sb[3] & lt);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (sel[u]) {
                            if (o < a.k) out[o] = lo + i0 + u;
                            ++o;
                        }
                    }
                    out_run += __popc(sb[0]) + __popc(sb[1]) + __popc(sb[2]) + __popc(sb[3]);
                }
            }
        }
    }
    cluster_wait_acquire();  // keep this CTA's shared memory alive until every peer has read it
}

}  // namespace

namespace {

// Largest shared-memory slice (keys) of one CTA: what fits beside the CTA's own map.
template <int T>
constexpr int smem_keys_cap() {
    return T == 512 ? kTopkSmemKeys : 40960;
}

template <int T, bool BATCH>
cudaError_t launch_topk_variant(const TopkArgs& a, int cluster, int cap, cudaStream_t st) {
    const size_t smem = (size_t)(TopkLayout<T>::kBaseWords + cap) * sizeof(uint32_t);
    cudaError_t e =
        cudaFuncSetAttribute(topk_radix_kernel<T, BATCH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (cluster > 8) {
        e = cudaFuncSetAttribute(topk_radix_kernel<T, BATCH>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster, a.Nq, 1);
    cfg.blockDim = dim3(T, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, topk_radix_kernel<T, BATCH>, a, cap);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Slices of up to smem_keys_cap keys live in shared memory; a launch whose longest row's
// slices are longer takes the variant that streams the rest from global memory in batches.
template <int T>
cudaError_t launch_topk_impl(const TopkArgs& a, int cluster, int64_t row_max, cudaStream_t st) {
    int64_t chunk = (row_max + cluster - 1) / cluster;
    chunk = (chunk + 3) & ~int64_t(3);
    const int cap = (int)(chunk < smem_keys_cap<T>() ? chunk : smem_keys_cap<T>());
    return chunk > cap || cluster > kTopkMaxCluster ? launch_topk_variant<T, true>(a, cluster, cap, st)
                                                    : launch_topk_variant<T, false>(a, cluster, cap, st);
}

// How many clusters of c 1024-thread CTAs (one per SM) the device holds at once: cluster
// placement is per GPC, so this can be below SMs / c.  Asked once per device and size.
constexpr int kMaxTopkDevices = 64;
int g_wide_clusters[kMaxTopkDevices][kMaxCluster + 1];

int max_wide_clusters(int c) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxTopkDevices) return 0;
    int& slot = g_wide_clusters[dev][c];
    if (slot == 0) {
        constexpr int T = 1024;
        const size_t smem = (size_t)(TopkLayout<T>::kBaseWords + smem_keys_cap<T>()) * sizeof(uint32_t);
        int n = -1;
        // sizes above 8 exist only in the variant that streams from global memory
        auto kern = c <= kTopkMaxCluster ? topk_radix_kernel<T, false> : topk_radix_kernel<T, true>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess &&
            (c <= 8 || cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(c, 1, 1);
            cfg.blockDim = dim3(T, 1, 1);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = c;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int m = 0;
            if (cudaOccupancyMaxActiveClusters(&m, kern, &cfg) == cudaSuccess && m > 0) n = m;
        }
        (void)cudaGetLastError();  // a refused query only means: no wide launch
        slot = n;
    }
    return slot > 0 ? slot : 0;
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, int cluster, cudaStream_t st) {
    if (a.Nq == 0) return cudaSuccess;
    if (cluster < 1 || cluster > kMaxCluster) return cudaErrorInvalidValue;
    int64_t row_max = a.ld < (int64_t)a.T_max ? a.ld : (int64_t)a.T_max;
    if (a.row_len_hint > 0 && a.row_len_hint < row_max) row_max = a.row_len_hint;
    // When every row's cluster fits one wave at one CTA per SM, a 1024-thread CTA per SM runs
    // the same chain with twice the threads and no SM shared by two CTAs: the largest cluster
    // size up to the planned one whose Nq clusters the device holds at once, provided the
    // slices still fit shared memory wherever the planned launch's would.
    int sms = 0, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // Rows whose slices would not fit shared memory even as 1,024-thread slices of the planned
    // cluster: more, smaller slices -- up to 16 one-SM CTAs per row, when the device holds
    // every row's cluster in one wave (the passes over the scores in global memory then take
    // proportionally less per CTA).
    if (sms > 0 && (row_max + cluster - 1) / cluster > smem_keys_cap<1024>()) {
        for (int c = kMaxCluster; c > cluster; --c)
            if ((int64_t)a.Nq * c <= sms && a.Nq <= max_wide_clusters(c))
                return launch_topk_impl<1024>(a, c, row_max, st);
    }
    if (sms > 0 && (int64_t)a.Nq * cluster <= sms) {
        const bool planned_fits = (row_max + cluster - 1) / cluster <= smem_keys_cap<512>();
        for (int c = cluster; c >= 1; --c) {
            const bool fits = (row_max + c - 1) / c <= smem_keys_cap<1024>();
            if (planned_fits && !fits) break;
            if (a.Nq <= max_wide_clusters(c)) return launch_topk_impl<1024>(a, c, row_max, st);
        }
    }
    return launch_topk_impl<512>(a, cluster, row_max, st);
}

}  // namespace dsa
