/*
 * dsa_oracle.c -- CPU oracle for the DeepSeek Sparse Attention (DSA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * restatement of what the hot path computes, used to check the CUDA library.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no code, header, table or helper with the CUDA path
 * (it includes no header of the library and the library includes none of it).
 *
 * Arithmetic: every sum is a plain sequential loop accumulated in double
 * (fp64); inputs are decoded from their stored bytes here (FP8 e4m3 from the
 * format definition, bf16 by widening the bit pattern).  No blocking, fusion
 * or reordering beyond the definitions below.
 *
 * Sources (page title, section):
 *  - Indexer score: "DeepSeek Sparse Attention Explained" (kgptalkie), section
 *    "How Does the Lightning Indexer Score a Token?": one dot product of the
 *    past token's single shared key with each of H_I small queries, a ReLU on
 *    each, then a sum weighted by per-head weights.  Also "DeepSeek V3.2-Exp
 *    Cuts Long-Context Costs" (kiadev), "How DSA works" (few small heads,
 *    ReLU, FP8), and "DeepSeek Sparse Attention Cuts Long-Context Cost"
 *    (milos-mitrovic), "How Does the Lightning Indexer Pick Which Tokens Matter?".
 *  - Selection: kgptalkie, "How Does the Selector Pick 1,024?": keep the
 *    highest index_topk scores; take min(budget, tokens so far); redo per query.
 *  - Sparse attention: kgptalkie, "What Does the Whole Block Look Like?": the
 *    softmax denominator runs over the selected tokens only; lizeman "DeepSeek
 *    Sparse Attention" section 2 (Stage 2, attention restricted to the
 *    selected positions) and kiadev "Training and implementation details"
 *    (MLA in MQA mode: every query head shares each latent row).
 *  - Mask formulation: kgptalkie, "How Does the Selector Pick 1,024?": top-k,
 *    then a mask that sets every other position to minus infinity.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - FP8 dequantisation: value = e4m3(code) * per-token fp32 scale, applied
 *    before the dot product.
 *  - No internal 1/sqrt(d_I) in the multi-head indexer (a positive constant
 *    folds into w exactly because ReLU(c x) = c ReLU(x) for c > 0).
 *  - Candidates of query row t are positions s < q_len[t].
 *  - Ties in the selection go to the lower position; -0.0 equals +0.0.
 *  - The index list is written in ascending position order, padded with -1.
 *  - Value = the first 512 of the 576 values of the latent row.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_DK 576
#define ORACLE_DV 512

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_FP8 = 2 };

/* OCP FP8 e4m3 ("fn" variant): 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits; exponent field 0 encodes subnormals m/8 * 2^-6; the codes
 * S.1111.111 are NaN; there are no infinities; the largest finite value is
 * 1.75 * 2^8 = 448. */
double dsa_oracle_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32 pattern. */
double dsa_oracle_bf16_decode(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void* base, int64_t i, int dtype) {
    if (dtype == ORACLE_FP8) return dsa_oracle_e4m3_decode(((const uint8_t*)base)[i]);
    if (dtype == ORACLE_BF16) return dsa_oracle_bf16_decode(((const uint16_t*)base)[i]);
    return (double)((const float*)base)[i];
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/*
 * Lightning-indexer scores, literal order.
 *   q[t,j,x] = q_I[t,j,x] * q_scale[t,j]     (FP8 mode; F32 mode: q_I as is)
 *   k[s,x]   = k_I[b,s,x] * k_scale[b,s]     (b = q_seq[t])
 *   I[t,s]   = sum_{j<H_I} w[t,j] * max(sum_{x<d_I} q[t,j,x] k[s,x], 0)
 * for s < q_len[t]; entries s >= q_len[t] are left untouched.
 * idx_dtype: ORACLE_FP8 (q_I/k_I e4m3 bytes, w bf16 bits, scales used) or
 *            ORACLE_F32 (q_I/k_I/w float32, scales ignored).
 * Returns 0, or -1 on an argument error (q_seq/q_len out of range).
 */
int dsa_oracle_indexer(int Nq, int H_I, int d_I, int T_max, int B, int idx_dtype,
                       const void* q_I, const float* q_scale, const void* w,
                       const void* k_I, const float* k_scale,
                       const int32_t* q_seq, const int32_t* q_len,
                       double* scores, int64_t ld, int nthreads) {
    const int wdt = idx_dtype == ORACLE_FP8 ? ORACLE_BF16 : ORACLE_F32;
    if (d_I <= 0 || d_I > 256 || H_I <= 0) return -1;
    for (int t = 0; t < Nq; ++t)
        if (q_seq[t] < 0 || q_seq[t] >= B || q_len[t] < 0 || q_len[t] > T_max || q_len[t] > ld)
            return -1;
    set_threads(nthreads);
    double* q = (double*)malloc(sizeof(double) * (size_t)H_I * d_I);
    double* wt = (double*)malloc(sizeof(double) * (size_t)H_I);
    for (int t = 0; t < Nq; ++t) {
        for (int j = 0; j < H_I; ++j) {
            double qs = idx_dtype == ORACLE_FP8 ? (double)q_scale[(int64_t)t * H_I + j] : 1.0;
            for (int x = 0; x < d_I; ++x)
                q[j * d_I + x] = load_elem(q_I, ((int64_t)t * H_I + j) * d_I + x, idx_dtype) * qs;
            wt[j] = load_elem(w, (int64_t)t * H_I + j, wdt);
        }
        const int b = q_seq[t];
        const int n = q_len[t];
#pragma omp parallel for schedule(static)
        for (int s = 0; s < n; ++s) {
            const int64_t row = (int64_t)b * T_max + s;
            double kk[256];
            double ks = idx_dtype == ORACLE_FP8 ? (double)k_scale[row] : 1.0;
            for (int x = 0; x < d_I; ++x) kk[x] = load_elem(k_I, row * d_I + x, idx_dtype) * ks;
            double I = 0.0;
            for (int j = 0; j < H_I; ++j) {
                double dot = 0.0;
                for (int x = 0; x < d_I; ++x) dot += q[j * d_I + x] * kk[x];
                I += wt[j] * (dot > 0.0 ? dot : 0.0);
            }
            scores[(int64_t)t * ld + s] = I;
        }
    }
    free(q);
    free(wt);
    return 0;
}

typedef struct { double v; int32_t s; } scored_pos;

/* order: larger score first; equal scores -> lower position first */
static int cmp_desc(const void* a, const void* b) {
    const scored_pos* x = (const scored_pos*)a;
    const scored_pos* y = (const scored_pos*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s > y->s) - (x->s < y->s);
}

static int cmp_i32(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/*
 * Per-row causal top-k.  For row t with n = q_len[t] candidates: sort all
 * (score, s) with s < n by score descending, position ascending; keep the
 * first min(k, n); write them in ascending position order; pad with -1.
 * -0.0 compares equal to +0.0 (C comparison already does).  Returns 0, -1 on
 * bad arguments, -2 if a NaN score is met.
 */
int dsa_oracle_topk(int Nq, int64_t ld, const double* scores, const int32_t* q_len, int k,
                    int32_t* idx, int nthreads) {
    if (k <= 0) return -1;
    for (int t = 0; t < Nq; ++t)
        if (q_len[t] < 0 || q_len[t] > ld) return -1;
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
    for (int t = 0; t < Nq; ++t) {
        const int n = q_len[t];
        scored_pos* a = (scored_pos*)malloc(sizeof(scored_pos) * (size_t)(n > 0 ? n : 1));
        for (int s = 0; s < n; ++s) {
            double v = scores[(int64_t)t * ld + s];
            if (v != v) bad = 1;
            a[s].v = v;
            a[s].s = s;
        }
        qsort(a, (size_t)n, sizeof(scored_pos), cmp_desc);
        const int m = n < k ? n : k;
        int32_t* out = idx + (int64_t)t * k;
        for (int i = 0; i < m; ++i) out[i] = a[i].s;
        qsort(out, (size_t)m, sizeof(int32_t), cmp_i32);
        for (int i = m; i < k; ++i) out[i] = -1;
        free(a);
    }
    return bad ? -2 : 0;
}

/* Attention of one (row, head) over an explicit list of positions (two-pass softmax). */
static void attend(const void* q, const void* kv, int kv_dtype, int H, int T_max,
                   int t, int h, int b, const int32_t* pos, int m, double scale,
                   const unsigned char* masked, double* out, double* lse) {
    double* z = (double*)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
    double qv[ORACLE_DK];
    for (int x = 0; x < ORACLE_DK; ++x)
        qv[x] = load_elem(q, ((int64_t)t * H + h) * ORACLE_DK + x, kv_dtype);
    double zmax = -INFINITY;
    int live = 0;
    for (int i = 0; i < m; ++i) {
        if (masked && masked[i]) { z[i] = -INFINITY; continue; }
        const int64_t row = (int64_t)b * T_max + pos[i];
        double dot = 0.0;
        for (int x = 0; x < ORACLE_DK; ++x) dot += qv[x] * load_elem(kv, row * ORACLE_DK + x, kv_dtype);
        z[i] = scale * dot;
        if (z[i] > zmax) zmax = z[i];
        live = 1;
    }
    for (int x = 0; x < ORACLE_DV; ++x) out[x] = 0.0;
    if (!live) {
        *lse = -INFINITY;
        free(z);
        return;
    }
    double l = 0.0;
    for (int i = 0; i < m; ++i) {
        z[i] = (z[i] == -INFINITY) ? 0.0 : exp(z[i] - zmax);
        l += z[i];
    }
    for (int i = 0; i < m; ++i) {
        if (z[i] == 0.0) continue;
        const double p = z[i] / l;
        const int64_t row = (int64_t)b * T_max + pos[i];
        for (int x = 0; x < ORACLE_DV; ++x) out[x] += p * load_elem(kv, row * ORACLE_DK + x, kv_dtype);
    }
    *lse = zmax + log(l);
    free(z);
}

/*
 * Sparse MLA attention in MQA mode over the selected positions.
 * For each row t and head h, over S = {idx[t,i] : idx[t,i] >= 0}:
 *   z_s = scale * sum_{x<576} q[t,h,x] c[s,x];  p_s = exp(z_s - max z) / sum exp(z - max z)
 *   out[t,h,:] = sum_s p_s c[s,0:512];  lse[t,h] = max z + ln sum exp(z - max z)
 * Empty S gives out = 0 and lse = -inf.  kv_dtype: ORACLE_BF16 or ORACLE_F32.
 * Returns 0, -1 on bad arguments, -3 if an index is >= q_len[t] or < -1.
 */
int dsa_oracle_sparse_attn(int Nq, int H, int T_max, int B, int k, int kv_dtype,
                           const void* q, const void* kv, const int32_t* idx,
                           const int32_t* q_seq, const int32_t* q_len, double scale,
                           double* out, double* lse, int nthreads) {
    for (int t = 0; t < Nq; ++t) {
        if (q_seq[t] < 0 || q_seq[t] >= B || q_len[t] < 0 || q_len[t] > T_max) return -1;
        for (int i = 0; i < k; ++i) {
            int32_t s = idx[(int64_t)t * k + i];
            if (s < -1 || s >= q_len[t]) return -3;
        }
    }
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic)
    for (int th = 0; th < Nq * H; ++th) {
        const int t = th / H, h = th % H;
        int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
        int m = 0;
        for (int i = 0; i < k; ++i) {
            int32_t s = idx[(int64_t)t * k + i];
            if (s >= 0) pos[m++] = s;
        }
        attend(q, kv, kv_dtype, H, T_max, t, h, q_seq[t], pos, m, scale, NULL,
               out + (int64_t)th * ORACLE_DV, lse + th);
        free(pos);
    }
    return 0;
}

/* Dense attention over every candidate s < q_len[t] (no selection). */
int dsa_oracle_dense_attn(int Nq, int H, int T_max, int B, int kv_dtype, const void* q,
                          const void* kv, const int32_t* q_seq, const int32_t* q_len,
                          double scale, double* out, double* lse, int nthreads) {
    for (int t = 0; t < Nq; ++t)
        if (q_seq[t] < 0 || q_seq[t] >= B || q_len[t] < 0 || q_len[t] > T_max) return -1;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic)
    for (int th = 0; th < Nq * H; ++th) {
        const int t = th / H, h = th % H;
        const int n = q_len[t];
        int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
        for (int s = 0; s < n; ++s) pos[s] = s;
        attend(q, kv, kv_dtype, H, T_max, t, h, q_seq[t], pos, n, scale, NULL,
               out + (int64_t)th * ORACLE_DV, lse + th);
        free(pos);
    }
    return 0;
}

/* The mask view of selection: dense attention over s < q_len[t] where every
 * position not listed in idx[t] gets logit -inf (weight exactly zero). */
int dsa_oracle_masked_dense_attn(int Nq, int H, int T_max, int B, int k, int kv_dtype,
                                 const void* q, const void* kv, const int32_t* idx,
                                 const int32_t* q_seq, const int32_t* q_len, double scale,
                                 double* out, double* lse, int nthreads) {
    for (int t = 0; t < Nq; ++t)
        if (q_seq[t] < 0 || q_seq[t] >= B || q_len[t] < 0 || q_len[t] > T_max) return -1;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic)
    for (int th = 0; th < Nq * H; ++th) {
        const int t = th / H, h = th % H;
        const int n = q_len[t];
        int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
        unsigned char* masked = (unsigned char*)malloc((size_t)(n > 0 ? n : 1));
        for (int s = 0; s < n; ++s) { pos[s] = s; masked[s] = 1; }
        for (int i = 0; i < k; ++i) {
            int32_t s = idx[(int64_t)t * k + i];
            if (s >= 0 && s < n) masked[s] = 0;
        }
        attend(q, kv, kv_dtype, H, T_max, t, h, q_seq[t], pos, n, scale, masked,
               out + (int64_t)th * ORACLE_DV, lse + th);
        free(pos);
        free(masked);
    }
    return 0;
}

int dsa_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
