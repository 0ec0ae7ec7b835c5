// dsa_api.cu -- the extern "C" boundary declared in include/dsa.h.
// Host-side argument checks, launch planning (split counts, cluster sizes,
// prefill row chunks), workspace carving and the stage launches.  Nothing
// here allocates device memory or synchronises, except dsa_get_device_status.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/dsa.h"
#include "kernels.h"

namespace {

thread_local int32_t g_last_cuda_error = 0;

constexpr size_t kStatusBytes = 256;
constexpr size_t kAlign = 256;
constexpr size_t kPrefillChunkScoreBytes = size_t(64) << 20;  // score rows of one prefill chunk (L2-sized)

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsa_status_t cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int32_t)e;
    return DSA_ERR_CUDA;
}

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
    return sms;
}

dsa_status_t check_dims(const dsa_dims* d, bool need_indexer, bool need_mla, bool chunked = false) {
    if (d == nullptr) return DSA_ERR_INVALID_ARG;
    if (d->reserved != 0 || d->B < 1 || d->Nq < 0 || d->T_max < 1 || d->k < 1) return DSA_ERR_INVALID_ARG;
    if (d->ld_scores < 1 || (d->ld_scores & 3) != 0) return DSA_ERR_INVALID_ARG;
    if (d->k > 2048) return DSA_ERR_UNSUPPORTED;
    if ((int64_t)d->B * d->T_max > (int64_t)INT32_MAX / 2) return DSA_ERR_UNSUPPORTED;
    if (need_indexer) {
        if (d->d_I != 64 && d->d_I != 128) return DSA_ERR_UNSUPPORTED;
        if (d->idx_dtype == DSA_FP8_E4M3) {
            if (d->H_I != dsa::kIdxHeads) return DSA_ERR_UNSUPPORTED;
            if ((d->T_max & 3) != 0) return DSA_ERR_UNSUPPORTED;  // k_scale rows are fetched by TMA
        } else if (d->idx_dtype == DSA_F32) {
            if (d->H_I < 1 || d->H_I > 64) return DSA_ERR_UNSUPPORTED;
        } else {
            return DSA_ERR_INVALID_ARG;
        }
        if ((int64_t)d->Nq * d->H_I > INT32_MAX / 2) return DSA_ERR_UNSUPPORTED;
    }
    if (need_mla) {
        if (d->kv_dtype == DSA_BF16 || d->kv_dtype == DSA_FP8_E4M3) {  // FP8: the 656-byte latent entry
            if (d->H != dsa::kMlaHeads) return DSA_ERR_UNSUPPORTED;
        } else if (d->kv_dtype == DSA_F32) {
            if (d->H < 1 || d->H > 128) return DSA_ERR_UNSUPPORTED;
        } else {
            return DSA_ERR_INVALID_ARG;
        }
        if (!chunked && d->Nq > 65535) return DSA_ERR_UNSUPPORTED;  // grid extent of the row-parallel kernels
    }
    return DSA_OK;
}

struct MlaPlan {
    int splits = 1;
    int rows_per_split = 2048;
};

MlaPlan plan_mla(const dsa_dims* d, int nq) {
    MlaPlan p;
    if (d->kv_dtype == DSA_F32 || nq <= 0) {
        p.rows_per_split = d->k;
        return p;
    }
    const int sms = device_sms();
    int splits = sms / (2 * nq);
    if (splits < 1) splits = 1;
    if (splits > 16) splits = 16;
    int rows = (d->k + splits - 1) / splits;
    rows = (rows + dsa::kMlaTile - 1) / dsa::kMlaTile * dsa::kMlaTile;
    p.rows_per_split = rows;
    p.splits = (d->k + rows - 1) / rows;
    return p;
}

int plan_topk_cluster(const dsa_dims* d, int nq, int64_t row_len_hint = 0) {
    const int sms = device_sms();
    int64_t rowmax = d->ld_scores < d->T_max ? d->ld_scores : d->T_max;
    if (row_len_hint > 0 && row_len_hint < rowmax) rowmax = row_len_hint;
    int c = (int)((rowmax + dsa::kTopkSmemKeys - 1) / dsa::kTopkSmemKeys);
    const int fill = nq > 0 ? sms / nq : 8;
    if (fill > c) c = fill;
    if (c < 1) c = 1;
    if (c > dsa::kTopkMaxCluster) c = dsa::kTopkMaxCluster;
    return c;
}

int plan_prefill_chunk(const dsa_dims* d) {
    int64_t rows = (int64_t)(kPrefillChunkScoreBytes / ((size_t)d->ld_scores * sizeof(float)));
    if (rows < 1) rows = 1;
    // The attention of a chunk runs one CTA per (row, head half) on one SM each: a chunk of
    // whole waves (2 rows x SMs / 2 per wave) in multiples of four rows (the indexer's units)
    // keeps the last wave full.
    const int64_t per_wave = device_sms() / 2;
    if (rows >= per_wave) rows = rows / per_wave * per_wave / 4 * 4;
    if (rows < 1) rows = 1;
    if (rows > d->Nq) rows = d->Nq;
    if (rows > 65535) rows = 65535;
    return (int)(rows < 1 ? 1 : rows);
}

struct Layout {
    size_t scores = 0, idx = 0, part_o = 0, part_lse = 0, total = kStatusBytes;
};

void add_mla_partials(Layout& L, const dsa_dims* d, int nq, const MlaPlan& p) {
    if (p.splits > 1) {
        L.part_o = L.total;
        L.total = align_up(L.total + (size_t)p.splits * nq * d->H * dsa::kDV * sizeof(float));
        L.part_lse = L.total;
        L.total = align_up(L.total + (size_t)p.splits * nq * d->H * sizeof(float));
    }
}

// Dense attention plans its splits over every cached position: the selection length k is
// T_max (rounded up to whole 64-row tiles).
dsa_dims dense_dims(const dsa_dims* d) {
    dsa_dims e = *d;
    e.k = (d->T_max + dsa::kMlaTile - 1) / dsa::kMlaTile * dsa::kMlaTile;
    return e;
}

// A decode over a cache of at most k positions per sequence: every row selects all of its
// positions (min(k, n) = n), so the step is attention over every position s < q_len[t], which
// the attention kernel's dense form computes with no indexer and no top-k.  Rows can then exceed
// neither k nor the scores' row length without exceeding T_max, which the attention checks.
// The fp32 cache has no dense form.
bool short_cache_decode(const dsa_dims* d) {
    return d->T_max <= d->k && d->ld_scores >= d->T_max && d->kv_dtype != DSA_F32;
}

Layout layout_for(const dsa_dims* d, int op) {
    Layout L;
    if (op == DSA_OP_SPARSE_MLA) {
        add_mla_partials(L, d, d->Nq, plan_mla(d, d->Nq));
    } else if (op == DSA_OP_DENSE_MLA) {
        const dsa_dims e = dense_dims(d);
        add_mla_partials(L, &e, d->Nq, plan_mla(&e, d->Nq));
    } else if (op == DSA_OP_DECODE || op == DSA_OP_PREFILL) {
        const int rows = op == DSA_OP_PREFILL ? plan_prefill_chunk(d) : d->Nq;
        L.scores = L.total;
        L.total = align_up(L.total + (size_t)rows * d->ld_scores * sizeof(float));
        L.idx = L.total;
        L.total = align_up(L.total + (size_t)rows * d->k * sizeof(int32_t));
        MlaPlan p = plan_mla(d, rows);
        if (op == DSA_OP_DECODE && short_cache_decode(d)) {
            // the dense form plans its splits over T_max rounded up to whole tiles
            const dsa_dims e = dense_dims(d);
            const MlaPlan pe = plan_mla(&e, rows);
            if (pe.splits > p.splits) p = pe;
        }
        add_mla_partials(L, d, rows, p);
    }
    return L;
}

int* status_word(void* ws) { return reinterpret_cast<int*>(ws); }

void record_event(const dsa_stage_events* ev, int i, cudaStream_t st) {
    if (ev != nullptr && ev->ev[i] != nullptr) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev->ev[i]), st);
}

dsa_status_t run_indexer(const dsa_dims* d, int nq, const void* q_I, const float* q_scale, const void* w,
                         const void* k_I, const float* k_scale, const int32_t* q_seq, const int32_t* q_len,
                         float* scores, int* status, cudaStream_t st, bool rows_of_one_sequence = false,
                         int skip_upto = 0, const dsa_paged_cache* paged = nullptr) {
    dsa::IndexerArgs a{};
    a.q_I = q_I;
    a.q_scale = q_scale;
    a.w = w;
    a.k_I = k_I;
    a.k_scale = k_scale;
    a.q_seq = q_seq;
    a.q_len = q_len;
    a.scores = scores;
    a.ld = d->ld_scores;
    a.Nq = nq;
    a.B = d->B;
    a.T_max = d->T_max;
    a.H_I = d->H_I;
    a.d_I = d->d_I;
    a.status = status;
    a.skip_upto = skip_upto;
    if (paged != nullptr) {
        a.block_table = paged->block_table;
        a.block_size = paged->block_size;
        a.max_blocks = paged->max_blocks;
        a.num_blocks = paged->num_blocks;
    }
    cudaError_t e = d->idx_dtype != DSA_FP8_E4M3 ? dsa::launch_indexer_f32(a, st)
                    : rows_of_one_sequence      ? dsa::launch_indexer_fp8_units4(a, device_sms(), st)
                                                : dsa::launch_indexer_fp8(a, device_sms(), st);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e);
}

dsa_status_t run_topk(const dsa_dims* d, int nq, const float* scores, const int32_t* q_len, int32_t* idx, int* status,
                      cudaStream_t st, bool pdl = false, int64_t row_len_hint = 0) {
    dsa::TopkArgs a{};
    a.scores = scores;
    a.ld = d->ld_scores;
    a.q_len = q_len;
    a.idx = idx;
    a.Nq = nq;
    a.k = d->k;
    a.T_max = d->T_max;
    a.status = status;
    a.pdl = pdl ? 1 : 0;
    a.row_len_hint = row_len_hint;
    cudaError_t e = dsa::launch_topk(a, plan_topk_cluster(d, nq, row_len_hint), st);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e);
}

dsa_status_t run_mla(const dsa_dims* d, int nq, const void* q, const void* kv, const int32_t* idx, const int32_t* q_seq,
                     const int32_t* q_len, float scale, void* out, float* lse, void* ws, const Layout& L,
                     const dsa_stage_events* ev, cudaStream_t st, bool pdl = false, bool compact_idx = false,
                     const dsa_paged_cache* paged = nullptr) {
    const MlaPlan p = plan_mla(d, nq);
    dsa::MlaArgs a{};
    a.q = q;
    a.kv = kv;
    a.idx = idx;
    a.q_seq = q_seq;
    a.q_len = q_len;
    a.out = out;
    a.lse = lse;
    a.part_o = p.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + L.part_o) : nullptr;
    a.part_lse = p.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + L.part_lse) : nullptr;
    a.Nq = nq;
    a.B = d->B;
    a.T_max = d->T_max;
    a.k = d->k;
    a.H = d->H;
    a.splits = p.splits;
    a.rows_per_split = p.rows_per_split;
    a.softmax_scale = scale;
    a.status = ws ? status_word(ws) : nullptr;
    a.pdl = pdl ? 1 : 0;
    a.compact = compact_idx ? 1 : 0;
    if (paged != nullptr) {
        a.block_table = paged->block_table;
        a.block_size = paged->block_size;
        a.max_blocks = paged->max_blocks;
        a.num_blocks = paged->num_blocks;
    }
    a.kv_fp8 = d->kv_dtype == DSA_FP8_E4M3 ? 1 : 0;
    cudaError_t e;
    if (d->kv_dtype != DSA_F32) {
        e = dsa::launch_sparse_mla_bf16(a, st);
        record_event(ev, 3, st);
        if (e == cudaSuccess) e = dsa::launch_mla_combine(a, st);
    } else {
        e = dsa::launch_sparse_mla_f32(a, st);
        record_event(ev, 3, st);
    }
    return e == cudaSuccess ? DSA_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

const char* dsa_version(void) { return "dsa-b200 0.1.0 (sm_100a)"; }

int32_t dsa_last_cuda_error(void) { return g_last_cuda_error; }

const char* dsa_status_string(int32_t s) {
    switch (s) {
        case DSA_OK: return "ok";
        case DSA_ERR_INVALID_ARG: return "invalid argument";
        case DSA_ERR_UNSUPPORTED: return "unsupported size or type";
        case DSA_ERR_WORKSPACE: return "workspace missing or too small";
        case DSA_ERR_CUDA: return "CUDA runtime error";
        case DSA_ERR_TIMEOUT: return "device wait timed out";
        case DSA_ERR_INDEX_OOB: return "index outside [-1, q_len)";
        case DSA_ERR_LENGTH: return "q_len or q_seq out of range";
        default: return "unknown status";
    }
}

dsa_status_t dsa_workspace_size(const dsa_dims* dims, int32_t op, size_t* bytes) {
    if (bytes == nullptr || op < DSA_OP_INDEXER || op > DSA_OP_DENSE_MLA) return DSA_ERR_INVALID_ARG;
    const bool idx = op == DSA_OP_INDEXER || op == DSA_OP_DECODE || op == DSA_OP_PREFILL;
    const bool mla = op == DSA_OP_SPARSE_MLA || op == DSA_OP_DENSE_MLA || op == DSA_OP_DECODE || op == DSA_OP_PREFILL;
    dsa_status_t s = check_dims(dims, idx, mla, op == DSA_OP_PREFILL);
    if (s != DSA_OK) return s;
    *bytes = layout_for(dims, op).total;
    return DSA_OK;
}

dsa_status_t dsa_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
    if (workspace == nullptr || ws_bytes < kStatusBytes) return DSA_ERR_WORKSPACE;
    cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DSA_OK : cuda_fail(e);
}

dsa_status_t dsa_indexer_scores(const dsa_dims* dims, const void* q_I, const float* q_scale, const void* w,
                                const void* k_I, const float* k_scale, const int32_t* q_seq, const int32_t* q_len,
                                float* scores, void* workspace, size_t ws_bytes, void* stream) {
    dsa_status_t s = check_dims(dims, true, false);
    if (s != DSA_OK) return s;
    if (dims->Nq == 0) return DSA_OK;
    const bool fp8 = dims->idx_dtype == DSA_FP8_E4M3;
    if (!q_I || !w || !k_I || !q_seq || !q_len || !scores || (fp8 && (!q_scale || !k_scale)))
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_I) || !aligned16(k_I) || !aligned16(scores) || !aligned16(w) ||
        (fp8 && (!aligned16(k_scale) || !aligned16(q_scale))))
        return DSA_ERR_INVALID_ARG;
    if (workspace != nullptr && ws_bytes < kStatusBytes) return DSA_ERR_WORKSPACE;
    return run_indexer(dims, dims->Nq, q_I, q_scale, w, k_I, k_scale, q_seq, q_len, scores,
                       workspace ? status_word(workspace) : nullptr, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_prefill_indexer_scores(const dsa_dims* dims, const void* q_I, const float* q_scale, const void* w,
                                        const void* k_I, const float* k_scale, const int32_t* q_seq,
                                        const int32_t* q_len, float* scores, void* workspace, size_t ws_bytes,
                                        void* stream) {
    dsa_status_t s = check_dims(dims, true, false);
    if (s != DSA_OK) return s;
    if (dims->idx_dtype != DSA_FP8_E4M3 || dims->H_I != dsa::kIdxHeads || (dims->d_I != 64 && dims->d_I != 128))
        return DSA_ERR_UNSUPPORTED;
    if (dims->Nq == 0) return DSA_OK;
    if (!q_I || !q_scale || !w || !k_I || !k_scale || !q_seq || !q_len || !scores) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_I) || !aligned16(k_I) || !aligned16(scores) || !aligned16(w) || !aligned16(k_scale) ||
        !aligned16(q_scale))
        return DSA_ERR_INVALID_ARG;
    if (workspace != nullptr && ws_bytes < kStatusBytes) return DSA_ERR_WORKSPACE;
    return run_indexer(dims, dims->Nq, q_I, q_scale, w, k_I, k_scale, q_seq, q_len, scores,
                       workspace ? status_word(workspace) : nullptr, reinterpret_cast<cudaStream_t>(stream), true);
}

dsa_status_t dsa_topk(const dsa_dims* dims, const float* scores, const int32_t* q_len, int32_t* idx, void* workspace,
                      size_t ws_bytes, void* stream) {
    dsa_status_t s = check_dims(dims, false, false);
    if (s != DSA_OK) return s;
    if (dims->Nq == 0) return DSA_OK;
    if (!scores || !q_len || !idx) return DSA_ERR_INVALID_ARG;
    if (!aligned16(scores) || !aligned16(idx)) return DSA_ERR_INVALID_ARG;
    if (dims->Nq > 65535) return DSA_ERR_UNSUPPORTED;
    if (workspace != nullptr && ws_bytes < kStatusBytes) return DSA_ERR_WORKSPACE;
    return run_topk(dims, dims->Nq, scores, q_len, idx, workspace ? status_word(workspace) : nullptr,
                    reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_sparse_mla_attn(const dsa_dims* dims, const void* q, const void* kv, const int32_t* idx,
                                 const int32_t* q_seq, const int32_t* q_len, float softmax_scale, void* out,
                                 float* lse, void* workspace, size_t ws_bytes, void* stream) {
    dsa_status_t s = check_dims(dims, false, true);
    if (s != DSA_OK) return s;
    if (dims->Nq == 0) return DSA_OK;
    if (!q || !kv || !idx || !q_seq || !q_len || !out || !std::isfinite(softmax_scale)) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    const Layout L = layout_for(dims, DSA_OP_SPARSE_MLA);
    if (workspace == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    return run_mla(dims, dims->Nq, q, kv, idx, q_seq, q_len, softmax_scale, out, lse, workspace, L, nullptr,
                   reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_dense_mla_attn(const dsa_dims* dims, const void* q, const void* kv, const int32_t* q_seq,
                                const int32_t* q_len, float softmax_scale, void* out, float* lse, void* workspace,
                                size_t ws_bytes, void* stream) {
    dsa_status_t s = check_dims(dims, false, true);
    if (s != DSA_OK) return s;
    if (dims->kv_dtype == DSA_F32) return DSA_ERR_UNSUPPORTED;
    if (dims->Nq == 0) return DSA_OK;
    if (!q || !kv || !q_seq || !q_len || !out || !std::isfinite(softmax_scale)) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    const Layout L = layout_for(dims, DSA_OP_DENSE_MLA);
    if (workspace == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    const dsa_dims e = dense_dims(dims);
    // no index list: the attention kernel takes entry j of a row as position j, j < q_len[t]
    return run_mla(&e, dims->Nq, q, kv, nullptr, q_seq, q_len, softmax_scale, out, lse, workspace, L, nullptr,
                   reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_sparse_mla_attn_noalloc(const dsa_dims* dims, const void* q, const void* kv, const int32_t* idx,
                                         const int32_t* q_seq, const int32_t* q_len, float softmax_scale, void* out,
                                         float* lse, void* stream) {
    dsa_status_t s = check_dims(dims, false, true);
    if (s != DSA_OK) return s;
    if (dims->kv_dtype == DSA_F32) return DSA_ERR_UNSUPPORTED;
    if (dims->Nq == 0) return DSA_OK;
    if (!q || !kv || !idx || !q_seq || !q_len || !out || !std::isfinite(softmax_scale)) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    const MlaPlan p = plan_mla(dims, dims->Nq);
    // clustered splits merge on chip; only the partials path needs the static scratch
    if (p.splits > 1 && !dsa::mla_cluster_merge(p.splits) && (size_t)p.splits * dims->Nq > dsa::kStaticScratchPartials)
        return DSA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    cudaError_t e = dsa::static_mla_scratch(&scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    dsa::MlaArgs a{};
    a.q = q;
    a.kv = kv;
    a.idx = idx;
    a.q_seq = q_seq;
    a.q_len = q_len;
    a.out = out;
    a.lse = lse;
    a.part_o = reinterpret_cast<float*>(scratch);
    a.part_lse = reinterpret_cast<float*>(static_cast<char*>(scratch) + dsa::kStaticScratchOBytes);
    a.Nq = dims->Nq;
    a.B = dims->B;
    a.T_max = dims->T_max;
    a.k = dims->k;
    a.H = dims->H;
    a.splits = p.splits;
    a.rows_per_split = p.rows_per_split;
    a.kv_fp8 = dims->kv_dtype == DSA_FP8_E4M3 ? 1 : 0;
    a.softmax_scale = softmax_scale;
    a.status = nullptr;  // no caller memory to report device-side errors into
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    e = dsa::launch_sparse_mla_bf16(a, st);
    if (e == cudaSuccess) e = dsa::launch_mla_combine(a, st);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e);
}

}  // extern "C"

namespace {

// The decode step over a contiguous cache (paged == nullptr) or a paged one (k_I, k_scale and
// kv are then the pools and paged holds the block table).
dsa_status_t decode_impl(const dsa_dims* dims, const void* q_I, const float* q_scale, const void* w, const void* k_I,
                         const float* k_scale, const void* q, const void* kv, const dsa_paged_cache* paged,
                         const int32_t* q_seq, const int32_t* q_len, float softmax_scale, void* out, float* lse,
                         float* scores_out, int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream,
                         const dsa_stage_events* events) {
    dsa_status_t s = check_dims(dims, true, true);
    if (s != DSA_OK) return s;
    if (dims->Nq == 0) return DSA_OK;
    const bool fp8 = dims->idx_dtype == DSA_FP8_E4M3;
    if (!q_I || !w || !k_I || !q || !kv || !q_seq || !q_len || !out || (fp8 && (!q_scale || !k_scale)) ||
        !std::isfinite(softmax_scale))
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_I) || !aligned16(k_I) || !aligned16(w) || !aligned16(q) || !aligned16(kv) || !aligned16(out) ||
        (fp8 && (!aligned16(k_scale) || !aligned16(q_scale))) || (scores_out && !aligned16(scores_out)) ||
        (idx_out && !aligned16(idx_out)))
        return DSA_ERR_INVALID_ARG;
    const Layout L = layout_for(dims, DSA_OP_DECODE);
    if (workspace == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    int* status = status_word(workspace);
    float* scores = scores_out ? scores_out : reinterpret_cast<float*>(ws + L.scores);
    int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
    // Short-context dispatch.  Rows with at most k positions select all of them: unless the
    // caller asked for the scores, the indexer skips those rows.  When the whole cache is that
    // short, the attention runs in dense form and the indexer and top-k run only for the
    // outputs the caller asked for (the top-k copies such rows' positions through).
    const bool short_cache = short_cache_decode(dims);
    record_event(events, 0, st);
    if (!short_cache || scores_out) {
        s = run_indexer(dims, dims->Nq, q_I, q_scale, w, k_I, k_scale, q_seq, q_len, scores, status, st, false,
                        scores_out ? 0 : dims->k, paged);
        if (s != DSA_OK) return s;
    }
    record_event(events, 1, st);
    // top-k and attention follow their producer as programmatic dependents: their setup
    // overlaps the previous kernel's tail and they wait on the device for its output
    if (!short_cache || idx_out) {
        s = run_topk(dims, dims->Nq, scores, q_len, idx, status, st, true);
        if (s != DSA_OK) return s;
    }
    record_event(events, 2, st);
    if (short_cache) {
        const dsa_dims e = dense_dims(dims);
        s = run_mla(&e, dims->Nq, q, kv, nullptr, q_seq, q_len, softmax_scale, out, lse, workspace, L, events, st,
                    true, true, paged);
    } else {
        s = run_mla(dims, dims->Nq, q, kv, idx, q_seq, q_len, softmax_scale, out, lse, workspace, L, events, st,
                    true, true, paged);
    }
    if (s != DSA_OK) return s;
    record_event(events, 4, st);
    return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status_t dsa_decode_step(const dsa_dims* dims, const void* q_I, const float* q_scale, const void* w,
                             const void* k_I, const float* k_scale, const void* q, const void* kv,
                             const int32_t* q_seq, const int32_t* q_len, float softmax_scale, void* out, float* lse,
                             float* scores_out, int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream,
                             const dsa_stage_events* events) {
    return decode_impl(dims, q_I, q_scale, w, k_I, k_scale, q, kv, nullptr, q_seq, q_len, softmax_scale, out, lse,
                       scores_out, idx_out, workspace, ws_bytes, stream, events);
}

dsa_status_t dsa_decode_step_paged(const dsa_dims* dims, const void* q_I, const float* q_scale, const void* w,
                                   const dsa_paged_cache* cache, const void* q, const int32_t* q_seq,
                                   const int32_t* q_len, float softmax_scale, void* out, float* lse,
                                   float* scores_out, int32_t* idx_out, void* workspace, size_t ws_bytes,
                                   void* stream, const dsa_stage_events* events) {
    if (dims == nullptr || cache == nullptr || cache->block_table == nullptr || cache->reserved != 0)
        return DSA_ERR_INVALID_ARG;
    if (dims->idx_dtype != DSA_FP8_E4M3 || dims->kv_dtype == DSA_F32) return DSA_ERR_UNSUPPORTED;
    const int bs = cache->block_size;
    if (bs < 64 || (bs & (bs - 1)) != 0 || cache->num_blocks < 1 || cache->max_blocks < 1) return DSA_ERR_INVALID_ARG;
    if ((int64_t)cache->max_blocks * bs != dims->T_max) return DSA_ERR_INVALID_ARG;
    if ((int64_t)cache->num_blocks * bs > (int64_t)INT32_MAX / 2) return DSA_ERR_UNSUPPORTED;
    if (!aligned16(cache->k_scale)) return DSA_ERR_INVALID_ARG;
    return decode_impl(dims, q_I, q_scale, w, cache->k_I, cache->k_scale, q, cache->kv, cache, q_seq, q_len,
                       softmax_scale, out, lse, scores_out, idx_out, workspace, ws_bytes, stream, events);
}

dsa_status_t dsa_prefill(const dsa_dims* dims, const void* q_I, const float* q_scale, const void* w, const void* k_I,
                         const float* k_scale, const void* q, const void* kv, const int32_t* q_seq,
                         const int32_t* q_len, float softmax_scale, void* out, float* lse, int32_t* idx_out,
                         void* workspace, size_t ws_bytes, void* stream) {
    dsa_status_t s = check_dims(dims, true, true, true);
    if (s != DSA_OK) return s;
    if (dims->Nq == 0) return DSA_OK;
    const bool fp8 = dims->idx_dtype == DSA_FP8_E4M3;
    if (!q_I || !w || !k_I || !q || !kv || !q_seq || !q_len || !out || (fp8 && (!q_scale || !k_scale)) ||
        !std::isfinite(softmax_scale))
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_I) || !aligned16(k_I) || !aligned16(w) || !aligned16(q) || !aligned16(kv) || !aligned16(out) ||
        (fp8 && (!aligned16(k_scale) || !aligned16(q_scale))) || (idx_out && !aligned16(idx_out)))
        return DSA_ERR_INVALID_ARG;
    const Layout L = layout_for(dims, DSA_OP_PREFILL);
    if (workspace == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    int* status = status_word(workspace);
    const int chunk = plan_prefill_chunk(dims);
    const size_t qi_row = (size_t)dims->H_I * dims->d_I * (fp8 ? 1 : 4);
    const size_t w_row = (size_t)dims->H_I * (fp8 ? 2 : 4);
    const size_t kv_esz = dims->kv_dtype == DSA_F32 ? 4 : 2;  // q and out are bf16 unless the cache is f32
    const size_t q_row = (size_t)dims->H * dsa::kDK * kv_esz;
    const size_t o_row = (size_t)dims->H * dsa::kDV * kv_esz;
    for (int r0 = 0; r0 < dims->Nq; r0 += chunk) {
        const int nq = dims->Nq - r0 < chunk ? dims->Nq - r0 : chunk;
        float* scores = reinterpret_cast<float*>(ws + L.scores);
        int32_t* idx = idx_out ? idx_out + (size_t)r0 * dims->k : reinterpret_cast<int32_t*>(ws + L.idx);
        const char* qi = static_cast<const char*>(q_I) + r0 * qi_row;
        const float* qs = fp8 ? q_scale + (size_t)r0 * dims->H_I : nullptr;
        const char* wr = static_cast<const char*>(w) + r0 * w_row;
        s = run_indexer(dims, nq, qi, qs, wr, k_I, k_scale, q_seq + r0, q_len + r0, scores, status, st, true,
                        dims->k);
        if (s != DSA_OK) return s;
        // prompt rows at the end of the cache (a causal prompt, or a chunk of one after a cached
        // context: q_len[t] = T_max - Nq + t + 1 at most) hold at most T_max - Nq + r0 + nq
        // positions in rows r0 .. r0 + nq - 1; the top-k's clusters and slices are planned for
        // that (a longer row stays correct, only slower)
        const int64_t before = dims->T_max > dims->Nq ? (int64_t)dims->T_max - dims->Nq : 0;
        s = run_topk(dims, nq, scores, q_len + r0, idx, status, st, true, before + r0 + nq);
        if (s != DSA_OK) return s;
        s = run_mla(dims, nq, static_cast<const char*>(q) + r0 * q_row, kv, idx, q_seq + r0, q_len + r0,
                    softmax_scale, static_cast<char*>(out) + r0 * o_row, lse ? lse + (size_t)r0 * dims->H : nullptr,
                    workspace, L, nullptr, st, true, true);
        if (s != DSA_OK) return s;
    }
    return DSA_OK;
}

dsa_status_t dsa_append_tokens(const dsa_dims* dims, int32_t n, const int32_t* seq, const int32_t* pos,
                               const void* kv_new, const float* k_new, void* kv, void* k_I, float* k_scale,
                               const dsa_paged_cache* paged, void* workspace, size_t ws_bytes, void* stream) {
    dsa_status_t s = check_dims(dims, true, true);
    if (s != DSA_OK) return s;
    if (n < 0 || n > 65535) return n < 0 ? DSA_ERR_INVALID_ARG : DSA_ERR_UNSUPPORTED;
    if (n == 0) return DSA_OK;
    const bool fp8 = dims->idx_dtype == DSA_FP8_E4M3;
    if (dims->kv_dtype == DSA_F32) return DSA_ERR_UNSUPPORTED;
    if (paged != nullptr) {
        if (paged->block_table == nullptr || paged->reserved != 0) return DSA_ERR_INVALID_ARG;
        const int bs = paged->block_size;
        if (bs < 64 || (bs & (bs - 1)) != 0 || paged->num_blocks < 1 ||
            (int64_t)paged->max_blocks * bs != dims->T_max)
            return DSA_ERR_INVALID_ARG;
        kv = const_cast<void*>(paged->kv);
        k_I = const_cast<void*>(paged->k_I);
        k_scale = const_cast<float*>(paged->k_scale);
    }
    if (!seq || !pos || !kv_new || !k_new || !kv || !k_I || (fp8 && !k_scale)) return DSA_ERR_INVALID_ARG;
    if (workspace != nullptr && ws_bytes < kStatusBytes) return DSA_ERR_WORKSPACE;
    dsa::AppendArgs a{};
    a.n = n;
    a.seq = seq;
    a.pos = pos;
    a.kv_new = kv_new;
    a.k_new = k_new;
    a.kv = kv;
    a.k_I = k_I;
    a.k_scale = k_scale;
    a.B = dims->B;
    a.T_max = dims->T_max;
    a.d_I = dims->d_I;
    a.idx_fp8 = fp8 ? 1 : 0;
    a.kv_fp8 = dims->kv_dtype == DSA_FP8_E4M3 ? 1 : 0;
    if (paged != nullptr) {
        a.block_table = paged->block_table;
        a.block_size = paged->block_size;
        a.max_blocks = paged->max_blocks;
        a.num_blocks = paged->num_blocks;
    }
    a.status = workspace ? status_word(workspace) : nullptr;
    const cudaError_t e = dsa::launch_append_tokens(a, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DSA_OK : cuda_fail(e);
}

dsa_status_t dsa_get_device_status(void* workspace, void* stream, int32_t* status) {
    if (workspace == nullptr || status == nullptr) return DSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return cuda_fail(e);
    *status = v;
    return DSA_OK;
}

dsa_status_t dsa_selftest_attention_stall(const dsa_dims* dims, const void* q, const void* kv, const int32_t* idx,
                                          const int32_t* q_seq, const int32_t* q_len, float softmax_scale, void* out,
                                          float* lse, void* workspace, size_t ws_bytes, int32_t timeout_us,
                                          void* stream) {
    dsa_status_t s = check_dims(dims, false, true);
    if (s != DSA_OK) return s;
    if (dims->kv_dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
    if (timeout_us < 1 || timeout_us > 5000000) return DSA_ERR_INVALID_ARG;
    if (dims->Nq == 0) return DSA_OK;
    if (!q || !kv || !idx || !q_seq || !q_len || !out || !std::isfinite(softmax_scale)) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    const Layout L = layout_for(dims, DSA_OP_SPARSE_MLA);
    if (workspace == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    const MlaPlan p = plan_mla(dims, dims->Nq);
    dsa::MlaArgs a{};
    a.q = q;
    a.kv = kv;
    a.idx = idx;
    a.q_seq = q_seq;
    a.q_len = q_len;
    a.out = out;
    a.lse = lse;
    a.part_o = p.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(workspace) + L.part_o) : nullptr;
    a.part_lse = p.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(workspace) + L.part_lse) : nullptr;
    a.Nq = dims->Nq;
    a.B = dims->B;
    a.T_max = dims->T_max;
    a.k = dims->k;
    a.H = dims->H;
    a.splits = p.splits;
    a.rows_per_split = p.rows_per_split;
    a.softmax_scale = softmax_scale;
    a.status = status_word(workspace);
    a.selftest_stall = 1;
    a.wait_budget_ns = (uint64_t)timeout_us * 1000ull;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = dsa::launch_sparse_mla_bf16(a, st);
    if (e == cudaSuccess) e = dsa::launch_mla_combine(a, st);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e);
}

dsa_status_t dsa_selftest_wait_timeout(void* workspace, size_t ws_bytes, int32_t timeout_us, void* stream) {
    if (workspace == nullptr || ws_bytes < kStatusBytes) return DSA_ERR_WORKSPACE;
    if (timeout_us < 1 || timeout_us > 5000000) return DSA_ERR_INVALID_ARG;
    cudaError_t e = dsa::launch_wait_timeout_selftest(status_word(workspace), timeout_us,
                                                      reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DSA_OK : cuda_fail(e);
}

}  // extern "C"
