// indexer_sm100.cu -- lightning-indexer scores on the sm_100a tensor cores.
//
// What it computes ("DeepSeek Sparse Attention Explained", section "How Does
// the Lightning Indexer Score a Token?"; "DeepSeek V3.2-Exp Cuts Long-Context
// Costs", "How DSA works": FP8, a few small heads, ReLU):
//   I[t,s] = k_scale[s] * sum_j (w[t,j] * q_scale[t,j]) * ReLU(sum_x q8[t,j,x] k8[s,x])
// which equals sum_j w[t,j] ReLU(q[t,j] . k[s]) with q = q8*q_scale, k = k8*k_scale
// because both scales are positive and ReLU(c x) = c ReLU(x) for c > 0.
//
// Shape of the work: for one query row, [H_I x d_I] . [d_I x n] is a dense
// FP8 contraction.  Decode (rows of different sequences): a stage is 512
// cached tokens, four MMA tiles of 128 tokens (MMA M = 128) against the 64
// heads of one query (MMA N = 64), K = d_I, accumulated in fp32 in tensor
// memory.  Prefill (consecutive rows of one sequence): a stage is one tile of
// 128 tokens against four query rows at once (MMA N = 4 x 64 = 256), so a key
// tile is read once per four rows.  Either way an accumulator is four blocks of
// 64 columns.  The epilogue reads one token row per thread from TMEM, applies
// ReLU, the weighted head sum and the key scale, and writes one fp32 score:
// per-head products never leave the chip.
//
// Every asynchronous hand-off (a TMA copy, an MMA, a commit) costs the
// per-SM pipeline time of its own (measured on B200: ~60 cycles per MMA and
// ~100 per commit on the critical path of a 128-token tile, which held the
// kernel at ~2.1 TB/s with 128-token stages), so a decode stage carries 512
// tokens with one commit, and the key stage and the accumulator are released
// by the epilogue warps (which have seen the MMA complete and hold its result
// in registers) rather than by a second commit.
//
// The epilogue is ALU bound in prefill: per (token, head) one ReLU (FMNMX, on
// the half-rate ALU pipe) and half a packed fp32 FMA.  Sixteen epilogue warps,
// four per TMEM sub-partition, give an accumulator back as soon as their loads
// have landed, so the tensor pipe never waits for the arithmetic.  Decode: each
// warp owns one 64-column block of every accumulator.  Prefill: two groups of
// eight warps take alternate stages (accumulators), each warp two blocks, so
// one group's arithmetic overlaps the other's TMEM loads and waits.
//
// Roles (one persistent CTA per SM, each owning a contiguous range of the
// flat list of (unit, stage) pairs; a unit is one query row in decode, four
// in prefill):
//   producer     decode: warps 0-1 copy each key stage and its fp32 scales with
//                16-byte cp.async into the swizzled stage ring; prefill: warp 0,
//                lane 0 issuing TMA boxes.  At a new unit warp 0 has lane 0
//                fetch the unit's q8 block by TMA and writes the folded weights
//                w*q_scale to shared memory
//   next warp    TMEM allocator and single-thread tcgen05.mma issuer
//   the rest     epilogue quads (one warp per TMEM sub-partition), each reading
//                one block of every accumulator (decode) or two blocks of every
//                other accumulator (prefill)
// Every wait is bounded; a timeout records DSA_ERR_TIMEOUT and the CTA drains
// and exits instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

#ifndef PREFILL_ROWS
#define PREFILL_ROWS 4
#endif

namespace dsa {
namespace {

// R = query rows per MMA: 1 for decode (rows of different sequences), 4 for prefill
// (consecutive rows of one sequence share every key tile, so one MMA of N = 4 x 64
// covers four rows and a key tile is read once per four rows).
template <int D_I, int R>
struct IdxCfg {
    static constexpr int TILE = kIdxTile;         // MMA M: tokens per MMA tile
    static constexpr int HEADS = kIdxHeads;       // heads per query row
    static constexpr int NCOL = R * HEADS;        // MMA N: R rows x HEADS heads
    static constexpr int SUB = R > 1 ? 1 : (D_I == 64 ? 4 : 2);  // MMA tiles per stage
    static constexpr int STOK = SUB * TILE;       // tokens per stage
    static constexpr int BOX = STOK < 256 ? STOK : 256;  // tokens per TMA box (the box limit is 256)
    static constexpr int NBOX = STOK / BOX;       // key and scale boxes per stage
    static constexpr int STAGES = R > 1 ? (D_I == 64 ? 12 : 6) : (D_I == 64 ? 4 : 5);
    static constexpr int KTILE_BYTES = STOK * D_I;
    static constexpr int Q_BYTES = NCOL * D_I;
    static constexpr uint32_t SWZ = D_I == 64 ? kSwizzle64B : kSwizzle128B;
    static constexpr uint32_t SBO = 8 * D_I;      // 8-row swizzle atom
    static constexpr int TMEM_COLS = 512;
    static constexpr int ACC = TMEM_COLS / (SUB * NCOL);  // TMEM accumulators of SUB x NCOL columns
    static_assert(ACC >= 2 && ACC * SUB * NCOL <= TMEM_COLS, "accumulators must fit TMEM twice");
    // 64-column blocks of one accumulator (one query row of one 128-token tile each).  An
    // epilogue quad (four warps, one per TMEM sub-partition) reads one block; a group of NB
    // quads covers an accumulator, and with QP groups group g takes the stages it % QP == g.
    static constexpr int NB = SUB * R;
    // Prefill splits its epilogue into QP = 2 groups on alternating stages (accumulators),
    // each warp reading BPQ = 2 blocks; decode keeps one group of one block per warp.
    static constexpr int QP = R == 1 ? 1 : 2;
    static constexpr int BPQ = R == 4 ? 2 : 1;
    // Decode streams its keys with 16-byte cp.async copies from two producer warps, which write
    // the swizzled tile themselves (measured on B200: the long decode's 142.7 MB of keys and
    // scales stream in 27.6 us with plain 16-byte loads against 33.6 us with 64-byte TMA box
    // rows); prefill, bound by its epilogue, keeps one TMA producer lane.
    static constexpr bool CPASYNC = R == 1;
    static constexpr int PROD_WARPS = CPASYNC ? 2 : 1;
    static constexpr int PROD_THREADS = 32 * PROD_WARPS;
    static constexpr int MMA_WARP = PROD_WARPS;
    static constexpr int EPI_WARP0 = PROD_WARPS + 1;
    static constexpr int KCHUNKS = STOK * D_I / 16;  // 16-byte pieces of a key stage
    static constexpr int SCHUNKS = STOK / 4;         // 16-byte pieces of its scales
    static_assert(!CPASYNC || (KCHUNKS % PROD_THREADS == 0 && SCHUNKS % PROD_THREADS == 0),
                  "every producer thread copies the same number of pieces per stage");
    static constexpr int EPI_QUADS = NB * QP / BPQ;  // epilogue quads
    static constexpr int GQ = EPI_QUADS / QP;          // quads per group
    static_assert(EPI_QUADS * BPQ == NB * QP && GQ * QP == EPI_QUADS && GQ * BPQ == NB,
                  "every block of an accumulator is read by one quad of its group");
    static constexpr int EPI_WARPS = 4 * EPI_QUADS;
    static constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;
    static constexpr int K_STEPS = D_I / 32;      // kind::f8f6f4 consumes 32 bytes of K per MMA
    // shared memory map (offsets from a 1024-byte aligned base)
    static constexpr int OFF_K = 0;
    static constexpr int OFF_Q = OFF_K + STAGES * KTILE_BYTES;
    static constexpr int OFF_SC = OFF_Q + 2 * Q_BYTES;     // per-stage key scales (STOK fp32)
    static constexpr int SC_BYTES = STOK * 4;
    static constexpr int OFF_WQ = OFF_SC + STAGES * SC_BYTES;  // 2 x NCOL folded weights
    static constexpr int OFF_BAR = OFF_WQ + 2 * NCOL * 4;
    static constexpr int NBAR = 2 * STAGES + 4 + 2 * ACC;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
    static constexpr uint32_t IDESC = make_idesc(TILE, NCOL, 0 /*e4m3*/, 0 /*e4m3*/, 0, 0);
};

struct IdxShared {
    int row0, j0, count;
    int n0, b0, nt0;  // the first unit's longest row, sequence and stage count
    int tmem_base;
    int abort_flag;
};

// Number of key stages (stok tokens each) of a query row with length n in sequence b (0 when the
// sizes are invalid).
__device__ __forceinline__ int tiles_of(const IndexerArgs& a, int n, int b, int stok) {
    if (n < 0 || n > a.T_max || (int64_t)n > a.ld || b < 0 || b >= a.B) return 0;
    return (n + stok - 1) / stok;
}
__device__ __forceinline__ int row_tiles(const IndexerArgs& a, int r, int stok) {
    return tiles_of(a, a.q_len[r], a.q_seq[r], stok);
}
// A unit is R consecutive query rows of one sequence; its key range is the longest of
// its rows.  -1 (unit skipped) for an invalid length or rows of different sequences.
__device__ __forceinline__ int unit_len(const IndexerArgs& a, int u, int R) {
    int n = 0;
    const int b = a.q_seq[u * R];
    for (int r = u * R; r < min(a.Nq, u * R + R); ++r) {
        const int nr = a.q_len[r];
        if (nr < 0 || nr > a.T_max || (int64_t)nr > a.ld || a.q_seq[r] != b) return -1;
        n = max(n, nr);
    }
    return n;
}
// Stages scheduled for a unit: none for an invalid unit, and none for a unit whose longest
// row is at most skip_upto (short rows: the top-k takes every position without scores).
__device__ __forceinline__ int unit_tiles(const IndexerArgs& a, int u, int R, int stok) {
    const int n = R == 1 ? a.q_len[u] : unit_len(a, u, R);
    if (n <= a.skip_upto) return 0;
    return R == 1 ? row_tiles(a, u, stok) : (n < 0 ? 0 : tiles_of(a, n, a.q_seq[u * R], stok));
}

// Walks the flat (unit, stage) list.  The unit's sequence and length are read
// once per unit, never per stage: every issuing loop depends on them.
template <int STOK, int R>
struct TileCursor {
    int row, j, nt, b, n;  // row = unit (R query rows), n = the unit's longest row
    __device__ void load_row(const IndexerArgs& a) {
        if (row * R < a.Nq) {
            n = R == 1 ? a.q_len[row] : max(0, unit_len(a, row, R));
            b = a.q_seq[row * R];
            nt = unit_tiles(a, row, R, STOK);
        } else {
            n = 0;
            b = 0;
            nt = 1;  // sentinel past the last row
        }
    }
    __device__ void start(const IndexerArgs& a, int r0, int j0) {
        row = r0;
        j = j0;
        load_row(a);
    }
    // the same start from values another warp loaded (no global reads on the way in)
    __device__ void start(int r0, int j0, int n0, int b0, int nt0) {
        row = r0;
        j = j0;
        n = n0;
        b = b0;
        nt = nt0;
    }
    __device__ void advance(const IndexerArgs& a) {
        if (++j >= nt) {
            j = 0;
            do {
                ++row;
                load_row(a);
            } while (nt == 0);
        }
    }
};

template <int D_I, int R>
__global__ void __launch_bounds__(IdxCfg<D_I, R>::THREADS, 1)
    indexer_fp8_kernel(const IndexerArgs a, const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_s) {
    using C = IdxCfg<D_I, R>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sK = sbase + C::OFF_K;
    const uint32_t sQ = sbase + C::OFF_Q;
    const uint32_t sS = sbase + C::OFF_SC;
    const float* scale_smem = reinterpret_cast<const float*>(smem + C::OFF_SC);
    float* wq_smem = reinterpret_cast<float*>(smem + C::OFF_WQ);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
    auto bar_qfull = [&](int q) { return bar0 + 8u * (2 * C::STAGES + q); };
    auto bar_qempty = [&](int q) { return bar0 + 8u * (2 * C::STAGES + 2 + q); };
    auto bar_tfull = [&](int c) { return bar0 + 8u * (2 * C::STAGES + 4 + c); };
    auto bar_tempty = [&](int c) { return bar0 + 8u * (2 * C::STAGES + 4 + C::ACC + c); };
    IdxShared* sh = reinterpret_cast<IdxShared*>(smem + C::OFF_MISC);
    volatile int* abort_flag = &sh->abort_flag;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            // TMA: one arrival with the stage's bytes; cp.async: one arrival per producer thread
            // once its copies of the stage have landed
            mbar_init(bar_full(s), C::CPASYNC ? C::PROD_THREADS : 1);
            mbar_init(bar_empty(s), 4 * C::NB);  // every warp of the stage's epilogue group, once it
                                                 // has its scales (the MMA that read the keys has
                                                 // completed before)
        }
        for (int q = 0; q < 2; ++q) {
            // producer arrivals: one with the q8 block's tx bytes (issued first), one once the
            // folded weights are in shared memory (written after the unit's first key copies)
            mbar_init(bar_qfull(q), 2);
            mbar_init(bar_qempty(q), 1 + C::EPI_WARPS);    // MMA commit + every epilogue warp
        }
        for (int c = 0; c < C::ACC; ++c) {
            mbar_init(bar_tfull(c), 1);
            mbar_init(bar_tempty(c), 4 * C::NB);  // every warp of the stage's group, once its loads landed
        }
        sh->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_s);
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(smem_u32(&sh->tmem_base), C::TMEM_COLS);
        tmem_relinquish();
    }
    // Work range: this CTA's slice of the flat (unit, stage) list (the first epilogue warp
    // scans the units).
    const int nunits = (a.Nq + R - 1) / R;
    if (warp == C::EPI_WARP0) {
        if (blockIdx.x == 0) {
            for (int r = lane; r < a.Nq; r += 32) {
                if (a.q_len[r] != 0 && row_tiles(a, r, C::STOK) == 0) record_status(a.status, DSA_STATUS_LENGTH);
                if (R > 1 && a.q_seq[r] != a.q_seq[r - r % R]) record_status(a.status, DSA_STATUS_INVALID_ARG);
            }
        }
        long long total = 0;
        for (int base = 0; base < nunits; base += 32) {
            const int r = base + lane;
            int v = r < nunits ? unit_tiles(a, r, R, C::STOK) : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            total += v;
        }
        const long long begin = total * blockIdx.x / gridDim.x;
        const long long end = total * (blockIdx.x + 1) / gridDim.x;
        int row0 = nunits, j0 = 0;
        long long run = 0;
        for (int base = 0; base < nunits && row0 == nunits; base += 32) {
            const int r = base + lane;
            const int v = r < nunits ? unit_tiles(a, r, R, C::STOK) : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            const long long excl = run + incl - v;
            const bool hit = v > 0 && excl <= begin && begin < excl + v;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            if (m) {
                const int src = __ffs(m) - 1;
                row0 = base + src;
                j0 = (int)(begin - __shfl_sync(0xffffffffu, excl, src));
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            sh->row0 = row0;
            sh->j0 = j0;
            sh->count = (int)(end - begin);
            TileCursor<C::STOK, R> first;
            first.start(a, row0, j0);
            sh->n0 = first.n;
            sh->b0 = first.b;
            sh->nt0 = first.nt;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)sh->tmem_base;
    const int count = sh->count;
    griddep_launch_dependents();  // the top-k may start its setup on SMs this grid leaves free

    if (warp < C::PROD_WARPS) {
        // ---------------- producer
        if (count > 0) {
            TileCursor<C::STOK, R> cur;
            cur.start(sh->row0, sh->j0, sh->n0, sh->b0, sh->nt0);
            int qi = -1;
            int issued = 0;
            const uint64_t stream_policy = l2_policy_evict_first();
            for (int it = 0; it < count; ++it) {
                const bool new_unit = it == 0 || cur.j == 0;
                int qb = 0;
                if (new_unit) {
                    ++qi;
                    qb = qi & 1;
                    if (warp == 0) {
                        if (qi >= 2) {
                            const bool okq = mbar_wait(bar_qempty(qb), ((qi - 2) >> 1) & 1, abort_flag, a.status);
                            if (!__all_sync(0xffffffffu, okq)) break;
                        }
                        // the unit's q8 block first: it depends on nothing the copies below need
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bar_qfull(qb), C::Q_BYTES);
                            tma_load_2d(sQ + qb * C::Q_BYTES, &tmap_q, 0, cur.row * C::NCOL, bar_qfull(qb));
                        }
                    }
                }
                const int st = it % C::STAGES;
                if (it >= C::STAGES) {
                    const bool oke = mbar_wait(bar_empty(st), ((it / C::STAGES) - 1) & 1, abort_flag, a.status);
                    if (!__all_sync(0xffffffffu, oke)) break;
                }
                if constexpr (C::CPASYNC) {
                    // Piece i of the stage = 16 bytes of token row r = i / (D_I / 16), chunk c; it goes
                    // to the K-major swizzled slot the MMA reads: 64B swizzle (d_I = 64) XORs the
                    // chunk with bits 1-2 of the row, 128B swizzle (d_I = 128) with bits 0-2.  Thread
                    // pt copies pieces pt + k * PROD_THREADS: its chunk c and its rows' swizzle are the
                    // same for every k (the row step is a multiple of 8), so each copy is a fixed offset
                    // from the first.  Rows at or past the unit's length are zero-filled without a read.
                    constexpr int CPR = D_I / 16;
                    constexpr int RSTEP = C::PROD_THREADS / CPR;        // rows between a thread's pieces
                    constexpr int NIT = C::KCHUNKS / C::PROD_THREADS;   // pieces per thread per stage
                    constexpr int STEP = RSTEP * D_I;                   // bytes between them (1024)
                    static_assert(RSTEP % 8 == 0, "the swizzle phase repeats every 8 rows");
                    const int tok0 = cur.j * C::STOK;
                    const int live = max(0, min(C::STOK, cur.n - tok0));
                    const int pt = tid;  // 0 .. PROD_THREADS - 1
                    const int c = pt % CPR, r0 = pt / CPR;
                    const int sw = D_I == 64 ? ((r0 >> 1) & 3) : (r0 & 7);
                    const uint32_t kd0 = sK + st * C::KTILE_BYTES + r0 * D_I + ((c ^ sw) << 4);
                    const uint32_t sd0 = sS + st * C::SC_BYTES + 16 * pt;
                    const uint8_t* kbase = reinterpret_cast<const uint8_t*>(a.k_I);
                    if (a.block_table == nullptr) {
                        const uint8_t* ks0 = kbase + ((int64_t)cur.b * a.T_max + tok0) * D_I + 16 * pt;
                        const float* ss0 = a.k_scale + (int64_t)cur.b * a.T_max + tok0 + 4 * pt;
                        if (live == C::STOK) {
#pragma unroll
                            for (int k = 0; k < NIT; ++k) cp_async16_hint(kd0 + k * STEP, ks0 + k * STEP, stream_policy);
#pragma unroll
                            for (int k = 0; k < C::SCHUNKS / C::PROD_THREADS; ++k)
                                cp_async16_hint(sd0 + k * 16 * C::PROD_THREADS, ss0 + k * 4 * C::PROD_THREADS,
                                                stream_policy);
                        } else {
#pragma unroll
                            for (int k = 0; k < NIT; ++k) {
                                const bool ok = r0 + k * RSTEP < live;
                                cp_async16_zfill_hint(kd0 + k * STEP, ok ? ks0 + k * STEP : kbase, ok ? 16u : 0u,
                                                      stream_policy);
                            }
#pragma unroll
                            for (int k = 0; k < C::SCHUNKS / C::PROD_THREADS; ++k) {
                                const bool ok = 4 * (pt + k * C::PROD_THREADS) < live;
                                cp_async16_zfill_hint(sd0 + k * 16 * C::PROD_THREADS,
                                                      ok ? ss0 + k * 4 * C::PROD_THREADS : a.k_scale, ok ? 16u : 0u,
                                                      stream_policy);
                            }
                        }
                    } else {
                        // paged cache: lane q holds the pool block of the stage's q-th block-sized piece
                        // (block_size >= 64 is a power of two; a thread's rows r0 + k * RSTEP with
                        // r0 < RSTEP never straddle a block, so piece k lies in block slot
                        // (k * RSTEP) / block_size)
                        const int bs = a.block_size;
                        const int nblk = bs >= C::STOK ? 1 : C::STOK / bs;
                        int pb_l = 0;
                        if (lane < nblk && tok0 + lane * bs < cur.n) {
                            pb_l = a.block_table[(int64_t)cur.b * a.max_blocks + (tok0 + lane * bs) / bs];
                            if (pb_l < 0 || pb_l >= a.num_blocks) {
                                if (warp == 0) record_status(a.status, DSA_STATUS_INDEX_OOB);
                                pb_l = 0;
                            }
                        }
                        const int lbs = 31 - __clz(bs);
                        const int off0 = tok0 & (bs - 1);  // the stage's offset inside its first block
#pragma unroll
                        for (int k = 0; k < NIT; ++k) {
                            const int r = r0 + k * RSTEP;
                            const bool ok = r < live;
                            const int pb = __shfl_sync(0xffffffffu, pb_l, (k * RSTEP) >> lbs);
                            const int64_t prow = ((int64_t)pb << lbs) + ((off0 + r) & (bs - 1));
                            cp_async16_zfill_hint(kd0 + k * STEP, ok ? kbase + prow * D_I + 16 * c : kbase,
                                                  ok ? 16u : 0u, stream_policy);
                        }
#pragma unroll
                        for (int k = 0; k < C::SCHUNKS / C::PROD_THREADS; ++k) {
                            const int r = 4 * (pt + k * C::PROD_THREADS);
                            const bool ok = r < live;
                            const int pb = __shfl_sync(0xffffffffu, pb_l, r >> lbs);
                            const int64_t prow = ((int64_t)pb << lbs) + ((off0 + r) & (bs - 1));
                            cp_async16_zfill_hint(sd0 + k * 16 * C::PROD_THREADS, ok ? a.k_scale + prow : a.k_scale,
                                                  ok ? 16u : 0u, stream_policy);
                        }
                    }
                    cp_async_arrive_noinc(bar_full(st));
                } else {
                    if (a.block_table == nullptr) {
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bar_full(st), C::KTILE_BYTES + C::SC_BYTES);
#pragma unroll
                            for (int q = 0; q < C::NBOX; ++q) {
                                const int tok = cur.j * C::STOK + q * C::BOX;
                                tma_load_2d(sK + st * C::KTILE_BYTES + q * (C::BOX * D_I), &tmap_k, 0,
                                            cur.b * a.T_max + tok, bar_full(st));
                                tma_load_2d(sS + st * C::SC_BYTES + q * (C::BOX * 4), &tmap_s, tok, cur.b,
                                            bar_full(st));
                            }
                        }
                    } else {
                        // paged cache: one key box and one scale box per block piece of the stage, for
                        // the pieces that hold tokens of the unit (later pieces may have no block; their
                        // stale rows only reach scores that are never stored).  Lane q reads piece q's
                        // block id, so the table reads overlap.
                        const int kb = a.page_box;
                        const int tok0 = cur.j * C::STOK;
                        const int live = min(C::STOK / kb, (cur.n - tok0 + kb - 1) / kb);
                        int pb_l = 0;
                        if (lane < live) {
                            pb_l = a.block_table[(int64_t)cur.b * a.max_blocks + (tok0 + lane * kb) / a.block_size];
                            if (pb_l < 0 || pb_l >= a.num_blocks) {
                                record_status(a.status, DSA_STATUS_INDEX_OOB);
                                pb_l = 0;
                            }
                        }
                        if (lane == 0) mbar_arrive_expect_tx(bar_full(st), (uint32_t)live * kb * (D_I + 4));
#pragma unroll
                        for (int q = 0; q < C::STOK / 64; ++q) {  // kb >= 64: at most STOK / 64 pieces
                            const int pb = __shfl_sync(0xffffffffu, pb_l, q);
                            if (lane == 0 && q < live) {
                                const int off = (tok0 + q * kb) % a.block_size;
                                tma_load_2d(sK + st * C::KTILE_BYTES + q * (kb * D_I), &tmap_k, 0,
                                            pb * a.block_size + off, bar_full(st));
                                tma_load_2d(sS + st * C::SC_BYTES + q * (kb * 4), &tmap_s, off, pb, bar_full(st));
                            }
                        }
                    }
                }
                if (new_unit && warp == 0) {
                    // folded weights w * q_scale of the unit's rows (0 past the last row), after the
                    // stage's copies so that their load latency does not delay the key stream
                    const int64_t o = (int64_t)cur.row * C::NCOL;
                    const __nv_bfloat16* wr = reinterpret_cast<const __nv_bfloat16*>(a.w) + o;
                    const int64_t lim = (int64_t)a.Nq * C::HEADS - o;
                    for (int i = lane; i < C::NCOL; i += 32)
                        wq_smem[qb * C::NCOL + i] = i < lim ? __bfloat162float(wr[i]) * a.q_scale[o + i] : 0.f;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_qfull(qb));
                }
                ++issued;
                cur.advance(a);
            }
            if constexpr (C::CPASYNC) {
                // copies still in flight land before the CTA's shared memory is released
                cp_async_wait_all();
            } else if (lane == 0 && *abort_flag) {
                // drain copies still in flight before the CTA's shared memory is released
                for (int it = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; it < issued; ++it)
                    mbar_wait(bar_full(it % C::STAGES), (it / C::STAGES) & 1, nullptr, nullptr, 50000000ull);
            }
        }
    } else if (warp == C::MMA_WARP) {
        if (lane == 0 && count > 0) {
            // ---------------- MMA issuer
            TileCursor<C::STOK, R> cur;
            cur.start(sh->row0, sh->j0, sh->n0, sh->b0, sh->nt0);
            int qi = -1, qb = 0;
            int last_acc = -1, last_it = -1;
            for (int it = 0; it < count; ++it) {
                if (it == 0 || cur.j == 0) {
                    ++qi;
                    qb = qi & 1;
                    if (!mbar_wait(bar_qfull(qb), (qi >> 1) & 1, abort_flag, a.status)) break;
                }
                const int st = it % C::STAGES;
                if (!mbar_wait(bar_full(st), (it / C::STAGES) & 1, abort_flag, a.status)) break;
                // keys written by cp.async (generic proxy) are read by the tensor core (async proxy)
                if constexpr (C::CPASYNC) fence_proxy_async_smem();
                const int acc = it % C::ACC;
                // polled: the accumulator comes back while the epilogue warps compute, and a
                // suspended wait would resume late on the tensor pipe's critical path
                if (it >= C::ACC && !mbar_wait_spin(bar_tempty(acc), ((it / C::ACC) - 1) & 1, abort_flag, a.status))
                    break;
                tc_fence_after();
                const uint32_t b_addr = sQ + qb * C::Q_BYTES;
#pragma unroll
                for (int h = 0; h < C::SUB; ++h) {
                    const uint32_t d = tmem + acc * (C::SUB * C::NCOL) + h * C::NCOL;
                    const uint32_t a_addr = sK + st * C::KTILE_BYTES + h * (C::TILE * D_I);
#pragma unroll
                    for (int ks = 0; ks < C::K_STEPS; ++ks) {
                        const uint64_t ad = make_smem_desc(a_addr + ks * 32, 16, C::SBO, C::SWZ);
                        const uint64_t bd = make_smem_desc(b_addr + ks * 32, 16, C::SBO, C::SWZ);
                        mma_f8f6f4_ss(d, ad, bd, C::IDESC, ks > 0 ? 1u : 0u);
                    }
                }
                mma_commit(bar_tfull(acc));
                last_acc = acc;
                last_it = it;
                if (cur.j == cur.nt - 1 || it == count - 1) mma_commit(bar_qempty(qb));
                cur.advance(a);
            }
            if (*abort_flag && last_it >= 0)
                mbar_wait(bar_tfull(last_acc), (last_it / C::ACC) & 1, nullptr, nullptr, 50000000ull);
        }
    } else {
        // ---------------- epilogue: BPQ 64-column blocks of its group's accumulators per warp
        // A warp reads a block (32 token lanes x 64 heads) in the 16x256b shape: thread t holds
        // tokens g, g+8, g+16, g+24 (g = t/4) at the 16 heads 8k + 2(t%4) + {0, 1}, so its 16
        // folded weights per block stay in registers for the whole unit; four threads then
        // combine their partial sums by shuffles.  With two groups (prefill) each group takes
        // every other stage, so one group's arithmetic overlaps the other's loads and waits;
        // its warps then read two blocks each, half a block (16 token lanes) at a time.
        const int q = (warp - C::EPI_WARP0) >> 2;  // quad
        const int grp = q / C::GQ;                 // group: stages it % QP == grp
        const int qq = q % C::GQ;                  // quad within the group: blocks qq + b GQ
        const int sub = warp & 3;                  // TMEM sub-partition this warp may access
        const int g = lane >> 2;
        const int i4 = lane & 3;
        // after the shuffles thread t owns token slot u = 2 (t%2) + (t%4)/2: token g + 8u of the
        // warp's 32 lanes, i.e. token `tok` of every stage (R = 1: of the block's tile)
        const int tok = (R == 1 ? qq : 0) * C::TILE + sub * 32 + g + 8 * (2 * (i4 & 1) + (i4 >> 1));
        TileCursor<C::STOK, R> cur;
        if (count > 0) cur.start(sh->row0, sh->j0, sh->n0, sh->b0, sh->nt0);
        int qi = -1;
        int nrow[C::BPQ];           // this thread's scores of block b exist for s < nrow[b] (s = stage base + tok)
        float* srow[C::BPQ];        // score row of block b's query row, offset by tok
        int acc = 0, accph = 0;     // accumulator of stage `it` and its phase parity
        uint64_t w2[C::BPQ][8];     // folded weights of heads 8k + 2(t%4) + {0, 1}, packed in pairs
#pragma unroll
        for (int b = 0; b < C::BPQ; ++b) {
            nrow[b] = 0;
            srow[b] = nullptr;
#pragma unroll
            for (int k = 0; k < 8; ++k) w2[b][k] = 0;
        }
        for (int it = 0; it < count; ++it) {
            if (it == 0 || cur.j == 0) {
                ++qi;
                const int qb = qi & 1;
                // folded weights of the unit: published by the producer with the q8 block
                const bool okq = mbar_wait(bar_qfull(qb), (qi >> 1) & 1, abort_flag, a.status);
                if (!__all_sync(0xffffffffu, okq)) break;
#pragma unroll
                for (int b = 0; b < C::BPQ; ++b) {
                    const int blk = qq + b * C::GQ;
                    const int r = R == 1 ? 0 : blk;  // the block's query row within the unit
                    const int64_t row = (int64_t)cur.row * R + r;
                    nrow[b] = (R == 1 ? cur.n : (row < a.Nq ? max(0, min(a.q_len[row], cur.n)) : 0)) - tok;
                    srow[b] = a.scores + row * a.ld + tok;
                    const float* wsrc = wq_smem + qb * C::NCOL + r * C::HEADS + 2 * i4;
#pragma unroll
                    for (int k = 0; k < 8; ++k) w2[b][k] = pack_f32x2(wsrc[8 * k], wsrc[8 * k + 1]);
                }
                // the weights are in registers: the producer may reuse the buffer
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_qempty(qb));
            }
            if (C::QP == 1 || it % C::QP == grp) {
                const int st = it % C::STAGES;
                bool ok = mbar_wait(bar_tfull(acc), accph, abort_flag, a.status);
                ok = ok && mbar_wait(bar_full(st), (it / C::STAGES) & 1, abort_flag, a.status);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                const int sb = cur.j * C::STOK;
#pragma unroll
                for (int b = 0; b < C::BPQ; ++b) {
                    const int blk = qq + b * C::GQ;
                    const uint32_t taddr =
                        tmem + ((uint32_t)(sub * 32) << 16) + acc * (C::SUB * C::NCOL) + blk * C::HEADS;
                    // p2[u]: this thread's 16 heads of token slot u (tokens g, g+8 from the first
                    // 16 lanes, g+16, g+24 from the second), two heads per packed FMA
                    uint64_t p2[4] = {0, 0, 0, 0};
                    auto accumulate = [&](const uint32_t (&v)[32], int u0) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
#pragma unroll
                            for (int uu = 0; uu < 2; ++uu) {
                                const uint32_t* x = &v[4 * k + 2 * uu];
                                p2[u0 + uu] = fma_f32x2(w2[b][k],
                                                        pack_f32x2(fmaxf(__uint_as_float(x[0]), 0.f),
                                                                   fmaxf(__uint_as_float(x[1]), 0.f)),
                                                        p2[u0 + uu]);
                            }
                        }
                    };
                    // the key scale (from the stage's shared copy); then the accumulator block and the
                    // key stage are released (the MMA that read the keys has completed)
                    auto release = [&]() {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive(bar_tempty(acc));
                            mbar_arrive(bar_empty(st));
                        }
                    };
                    float ks;
                    if constexpr (C::BPQ == 1) {
                        uint32_t v[2][32];
                        tmem_ld16x256b_x8(taddr, v[0]);
                        tmem_ld16x256b_x8(taddr + (16u << 16), v[1]);
                        tmem_wait_ld_regs(v[0]);
                        tmem_wait_ld_regs(v[1]);
                        ks = scale_smem[st * C::STOK + tok];
                        release();
                        accumulate(v[0], 0);
                        accumulate(v[1], 2);
                    } else {
                        uint32_t v[32];
                        tmem_ld16x256b_x8(taddr, v);
                        tmem_wait_ld_regs(v);
                        accumulate(v, 0);
                        tmem_ld16x256b_x8(taddr + (16u << 16), v);
                        tmem_wait_ld_regs(v);
                        ks = scale_smem[st * C::STOK + tok];
                        release();
                        accumulate(v, 2);
                    }
                    float s0, s1, s2, s3, t0, t1, t2, t3;
                    unpack_f32x2(p2[0], s0, t0);
                    unpack_f32x2(p2[1], s1, t1);
                    unpack_f32x2(p2[2], s2, t2);
                    unpack_f32x2(p2[3], s3, t3);
                    s0 += t0;
                    s1 += t1;
                    s2 += t2;
                    s3 += t3;
                    // sum over the four threads of a token group, leaving slot 2 (t%2) + (t%4)/2 here
                    const bool odd = i4 & 1;
                    const float qa = (odd ? s2 : s0) + __shfl_xor_sync(0xffffffffu, odd ? s0 : s2, 1);
                    const float qc = (odd ? s3 : s1) + __shfl_xor_sync(0xffffffffu, odd ? s1 : s3, 1);
                    const bool hi = i4 & 2;
                    const float sum = (hi ? qc : qa) + __shfl_xor_sync(0xffffffffu, hi ? qa : qc, 2);
                    if (sb < nrow[b]) srow[b][sb] = ks * sum;
                }
            }
            if (++acc == C::ACC) {
                acc = 0;
                accph ^= 1;
            }
            cur.advance(a);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D_I, int R>
cudaError_t launch_fp8_impl(const IndexerArgs& a, int grid, cudaStream_t st) {
    using C = IdxCfg<D_I, R>;
    alignas(64) CUtensorMap tk, tq, ts;
    const int swz = D_I;  // 64-byte rows -> 64B swizzle, 128-byte rows -> 128B swizzle
    IndexerArgs b = a;
    if (a.block_table == nullptr) {
        if (!encode_tensor_map_2d(&tk, 1, a.k_I, D_I, (uint64_t)a.B * a.T_max, D_I, D_I, C::BOX, swz))
            return cudaErrorInvalidValue;
        if (!encode_tensor_map_2d(&ts, 4, a.k_scale, a.T_max, (uint64_t)a.B, (uint64_t)a.T_max * 4, C::BOX, 1, 0))
            return cudaErrorInvalidValue;
    } else {
        // pools of num_blocks blocks: keys [num_blocks * block_size, d_I], scales [num_blocks, block_size]
        if (a.block_size < 64 || (a.block_size & (a.block_size - 1)) != 0 || a.num_blocks < 1)
            return cudaErrorInvalidValue;
        b.page_box = a.block_size < C::BOX ? a.block_size : C::BOX;
        if (C::STOK % b.page_box != 0) return cudaErrorInvalidValue;
        if (!encode_tensor_map_2d(&tk, 1, a.k_I, D_I, (uint64_t)a.num_blocks * a.block_size, D_I, D_I,
                                  (uint32_t)b.page_box, swz))
            return cudaErrorInvalidValue;
        if (!encode_tensor_map_2d(&ts, 4, a.k_scale, (uint64_t)a.block_size, (uint64_t)a.num_blocks,
                                  (uint64_t)a.block_size * 4, (uint32_t)b.page_box, 1, 0))
            return cudaErrorInvalidValue;
    }
    // q8 rows of a unit are consecutive: [Nq * HEADS, d_I], boxes of NCOL rows
    if (!encode_tensor_map_2d(&tq, 1, a.q_I, D_I, (uint64_t)a.Nq * C::HEADS, D_I, D_I, C::NCOL, swz))
        return cudaErrorInvalidValue;
    auto kern = indexer_fp8_kernel<D_I, R>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(b, tk, tq, ts);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer_fp8(const IndexerArgs& a, int grid, cudaStream_t st) {
    if (a.Nq == 0) return cudaSuccess;
    if (a.d_I == 64) return launch_fp8_impl<64, 1>(a, grid, st);
    if (a.d_I == 128) return launch_fp8_impl<128, 1>(a, grid, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_indexer_fp8_units4(const IndexerArgs& a, int grid, cudaStream_t st) {
    if (a.Nq == 0) return cudaSuccess;
    if (a.d_I == 64) return launch_fp8_impl<64, PREFILL_ROWS>(a, grid, st);
    if (a.d_I == 128) return launch_fp8_impl<128, PREFILL_ROWS>(a, grid, st);
    return cudaErrorInvalidValue;
}

}  // namespace dsa
