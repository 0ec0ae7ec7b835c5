/*
 * decode_c_api.c -- the C interface on its own (no Python, no PyTorch).
 *
 * Builds a small synthetic decode batch on the host: 4 sequences of up to
 * 8,192 cached tokens, FP8 indexer keys and queries with fp32 scales, a bf16
 * latent cache.  It copies the batch to the device and runs the decode step
 * twice:
 *   - once through dsa_decode_step (indexer -> top-2048 -> sparse MLA);
 *   - once stage by stage (dsa_indexer_scores, dsa_topk, dsa_sparse_mla_attn).
 * It checks that both select the same positions and give the same attention
 * output within bf16 rounding.  Exit status 0 when they agree.
 *
 * Build (next to the library, which it links):
 *   gcc -O2 -I../../include decode_c_api.c -L.. -ldsa_b200 -L/usr/local/cuda/lib64 -lcudart \
 *       -Wl,-rpath,'$ORIGIN/..' -o decode_c_api
 */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "dsa.h"

#define CHECK_CUDA(x)                                                                   \
    do {                                                                                \
        cudaError_t e_ = (x);                                                           \
        if (e_ != cudaSuccess) {                                                        \
            fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #x, cudaGetErrorString(e_)); \
            exit(2);                                                                    \
        }                                                                               \
    } while (0)
#define CHECK_DSA(x)                                                                    \
    do {                                                                                \
        dsa_status_t s_ = (x);                                                          \
        if (s_ != DSA_OK) {                                                             \
            fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #x, dsa_status_string(s_)); \
            exit(3);                                                                    \
        }                                                                               \
    } while (0)

enum { NSEQ = 4, T_MAX = 8192, H_I = 64, D_I = 64, H = 128, DK = 576, DV = 512, TOPK = 2048 };

/* xorshift32: the example's own seeded generator */
static uint32_t rng_state = 12345u;
static uint32_t rng_next(void) {
    uint32_t x = rng_state;
    x ^= x << 13;
    x ^= x >> 17;
    x ^= x << 5;
    rng_state = x;
    return x;
}
static float rng_uniform(float lo, float hi) { return lo + (hi - lo) * (float)(rng_next() >> 8) * (1.0f / 16777216.0f); }

/* bf16 bits of a finite float, rounded to nearest even */
static uint16_t to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
static float from_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}
/* a random finite e4m3 code: exponent field at most 13 keeps it away from the NaN codes */
static uint8_t random_e4m3(void) {
    const uint32_t r = rng_next();
    const uint8_t mag = (uint8_t)((r >> 8) % 0x70u);
    return (uint8_t)((r & 0x80u) | mag);
}

static void* to_device(const void* host, size_t bytes) {
    void* d = NULL;
    CHECK_CUDA(cudaMalloc(&d, bytes));
    CHECK_CUDA(cudaMemcpy(d, host, bytes, cudaMemcpyHostToDevice));
    return d;
}
static void* device_zeros(size_t bytes) {
    void* d = NULL;
    CHECK_CUDA(cudaMalloc(&d, bytes));
    CHECK_CUDA(cudaMemset(d, 0, bytes));
    return d;
}
static void* workspace_for(const dsa_dims* dims, int op, size_t* bytes) {
    CHECK_DSA(dsa_workspace_size(dims, op, bytes));
    if (*bytes < 256) *bytes = 256;
    void* ws = NULL;
    CHECK_CUDA(cudaMalloc(&ws, *bytes));
    CHECK_DSA(dsa_workspace_init(ws, *bytes, NULL));
    return ws;
}

int main(void) {
    const int32_t lens[NSEQ] = {8192, 5000, 3001, 1000}; /* the last row selects all its positions */
    const int nq = NSEQ;
    dsa_dims dims;
    memset(&dims, 0, sizeof dims);
    dims.B = NSEQ;
    dims.Nq = nq;
    dims.H_I = H_I;
    dims.d_I = D_I;
    dims.H = H;
    dims.k = TOPK;
    dims.T_max = T_MAX;
    dims.idx_dtype = DSA_FP8_E4M3;
    dims.kv_dtype = DSA_BF16;
    dims.ld_scores = T_MAX;

    /* ---- host inputs */
    const size_t n_qI = (size_t)nq * H_I * D_I, n_kI = (size_t)NSEQ * T_MAX * D_I;
    const size_t n_q = (size_t)nq * H * DK, n_kv = (size_t)NSEQ * T_MAX * DK;
    uint8_t* q_I = malloc(n_qI);
    uint8_t* k_I = malloc(n_kI);
    float* q_scale = malloc(sizeof(float) * nq * H_I);
    float* k_scale = malloc(sizeof(float) * NSEQ * T_MAX);
    uint16_t* w = malloc(sizeof(uint16_t) * nq * H_I);
    uint16_t* q = malloc(sizeof(uint16_t) * n_q);
    uint16_t* kv = malloc(sizeof(uint16_t) * n_kv);
    int32_t q_seq[NSEQ], q_len[NSEQ];
    if (!q_I || !k_I || !q_scale || !k_scale || !w || !q || !kv) return 4;
    for (size_t i = 0; i < n_qI; ++i) q_I[i] = random_e4m3();
    for (size_t i = 0; i < n_kI; ++i) k_I[i] = random_e4m3();
    for (int i = 0; i < nq * H_I; ++i) q_scale[i] = rng_uniform(0.005f, 0.02f);
    for (int i = 0; i < NSEQ * T_MAX; ++i) k_scale[i] = rng_uniform(0.005f, 0.02f);
    for (int i = 0; i < nq * H_I; ++i) w[i] = to_bf16(rng_uniform(-0.25f, 0.25f));
    for (size_t i = 0; i < n_q; ++i) q[i] = to_bf16(rng_uniform(-0.25f, 0.25f));
    for (size_t i = 0; i < n_kv; ++i) kv[i] = to_bf16(rng_uniform(-0.25f, 0.25f));
    for (int t = 0; t < nq; ++t) {
        q_seq[t] = t;
        q_len[t] = lens[t];
    }
    const float softmax_scale = 1.0f / sqrtf((float)(128 + 64));

    /* ---- device copies */
    void* d_qI = to_device(q_I, n_qI);
    void* d_kI = to_device(k_I, n_kI);
    float* d_qs = to_device(q_scale, sizeof(float) * nq * H_I);
    float* d_ks = to_device(k_scale, sizeof(float) * NSEQ * T_MAX);
    void* d_w = to_device(w, sizeof(uint16_t) * nq * H_I);
    void* d_q = to_device(q, sizeof(uint16_t) * n_q);
    void* d_kv = to_device(kv, sizeof(uint16_t) * n_kv);
    int32_t* d_seq = to_device(q_seq, sizeof q_seq);
    int32_t* d_len = to_device(q_len, sizeof q_len);
    const size_t out_bytes = sizeof(uint16_t) * nq * H * DV, lse_bytes = sizeof(float) * nq * H;
    const size_t idx_bytes = sizeof(int32_t) * nq * TOPK;
    void* d_out1 = device_zeros(out_bytes);
    float* d_lse1 = device_zeros(lse_bytes);
    int32_t* d_idx1 = device_zeros(idx_bytes);
    void* d_out2 = device_zeros(out_bytes);
    float* d_lse2 = device_zeros(lse_bytes);
    int32_t* d_idx2 = device_zeros(idx_bytes);
    float* d_scores = device_zeros(sizeof(float) * nq * T_MAX);

    /* ---- 1. the whole decode step */
    size_t ws_dec_bytes = 0, ws_idx_bytes = 0, ws_topk_bytes = 0, ws_mla_bytes = 0;
    void* ws_dec = workspace_for(&dims, DSA_OP_DECODE, &ws_dec_bytes);
    CHECK_DSA(dsa_decode_step(&dims, d_qI, d_qs, d_w, d_kI, d_ks, d_q, d_kv, d_seq, d_len, softmax_scale, d_out1,
                              d_lse1, NULL, d_idx1, ws_dec, ws_dec_bytes, NULL, NULL));
    int32_t status = 0;
    CHECK_DSA(dsa_get_device_status(ws_dec, NULL, &status));
    if (status != DSA_OK) {
        fprintf(stderr, "decode step: device status %s\n", dsa_status_string(status));
        return 5;
    }

    /* ---- 2. the same, one stage per call */
    void* ws_idx = workspace_for(&dims, DSA_OP_INDEXER, &ws_idx_bytes);
    void* ws_topk = workspace_for(&dims, DSA_OP_TOPK, &ws_topk_bytes);
    void* ws_mla = workspace_for(&dims, DSA_OP_SPARSE_MLA, &ws_mla_bytes);
    CHECK_DSA(dsa_indexer_scores(&dims, d_qI, d_qs, d_w, d_kI, d_ks, d_seq, d_len, d_scores, ws_idx, ws_idx_bytes,
                                 NULL));
    CHECK_DSA(dsa_topk(&dims, d_scores, d_len, d_idx2, ws_topk, ws_topk_bytes, NULL));
    CHECK_DSA(dsa_sparse_mla_attn(&dims, d_q, d_kv, d_idx2, d_seq, d_len, softmax_scale, d_out2, d_lse2, ws_mla,
                                  ws_mla_bytes, NULL));
    void* wss[3] = {ws_idx, ws_topk, ws_mla};
    for (int i = 0; i < 3; ++i) {
        CHECK_DSA(dsa_get_device_status(wss[i], NULL, &status));
        if (status != DSA_OK) {
            fprintf(stderr, "stage %d: device status %s\n", i, dsa_status_string(status));
            return 5;
        }
    }

    CHECK_CUDA(cudaDeviceSynchronize());

    /* ---- compare */
    int32_t* idx1 = malloc(idx_bytes);
    int32_t* idx2 = malloc(idx_bytes);
    uint16_t* out1 = malloc(out_bytes);
    uint16_t* out2 = malloc(out_bytes);
    float* lse1 = malloc(lse_bytes);
    float* lse2 = malloc(lse_bytes);
    if (!idx1 || !idx2 || !out1 || !out2 || !lse1 || !lse2) return 4;
    CHECK_CUDA(cudaMemcpy(idx1, d_idx1, idx_bytes, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(idx2, d_idx2, idx_bytes, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(out1, d_out1, out_bytes, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(out2, d_out2, out_bytes, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(lse1, d_lse1, lse_bytes, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(lse2, d_lse2, lse_bytes, cudaMemcpyDeviceToHost));

    int bad = 0;
    if (memcmp(idx1, idx2, idx_bytes) != 0) {
        fprintf(stderr, "selected positions differ between the fused step and the staged calls\n");
        bad = 1;
    }
    for (int t = 0; t < nq; ++t) {
        /* ascending positions below q_len, then -1 */
        const int n_sel = lens[t] < TOPK ? lens[t] : TOPK;
        for (int j = 0; j < TOPK; ++j) {
            const int32_t v = idx1[(size_t)t * TOPK + j];
            const int ok = j < n_sel ? (v >= 0 && v < lens[t] && (j == 0 || v > idx1[(size_t)t * TOPK + j - 1]))
                                     : v == -1;
            if (!ok) {
                fprintf(stderr, "row %d entry %d: %d is not a valid selection entry\n", t, j, v);
                bad = 1;
                break;
            }
        }
    }
    double max_err = 0.0, max_lse = 0.0;
    for (size_t i = 0; i < (size_t)nq * H * DV; ++i) {
        const double a = from_bf16(out1[i]), b = from_bf16(out2[i]);
        const double e = fabs(a - b);
        if (e > max_err) max_err = e;
        if (!(e <= 2e-2 + 1e-2 * fabs(b))) bad = 1;
    }
    for (int i = 0; i < nq * H; ++i) {
        const double e = fabs((double)lse1[i] - (double)lse2[i]);
        if (e > max_lse) max_lse = e;
        if (!(e <= 1e-3 * (1.0 + fabs((double)lse2[i])))) bad = 1;
    }
    printf("%s: %s; selections %s, max |out difference| %.3e, max |lse difference| %.3e\n",
           bad ? "FAIL" : "ok", dsa_version(), memcmp(idx1, idx2, idx_bytes) == 0 ? "identical" : "differ", max_err,
           max_lse);
    return bad ? 1 : 0;
}
