// append.cu -- writing a decode step's new tokens into the caches.
//
// What it computes ("DeepSeek Sparse Attention Explained", section "What Does
// the Whole Block Look Like?": on the precise path the token is compressed and
// written to the KV cache; section "What Does the GPU Actually Run?": the
// latent entry is stored in FP8 with one fp32 scale per 128 values and the 64
// rope values in bf16; the indexer's key cache holds FP8 numbers and one scale
// per token): for new token i of sequence seq[i] at position pos[i],
//   * the indexer key k_new[i, 0:d_I] (fp32) becomes e4m3 codes of
//     k_new / s with s = max|k_new| / 448 (1 when all zero), rounded to nearest
//     even and clamped to +-448, and the fp32 scale s;
//   * the latent row kv_new[i, 0:576] (bf16) is copied (bf16 cache) or packed
//     into the 656-byte FP8 entry: four groups of 128 latent values, each
//     quantised like the key with its own scale, then the 64 rope values.
// One CTA of 128 threads per new token; a warp reduces each maximum.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "status.cuh"

namespace dsa {
namespace {

constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// e4m3 code of x / s, rounded to nearest even, clamped to the finite range
__device__ __forceinline__ uint8_t e4m3_of(float x, float s) {
    const float y = fminf(fmaxf(x / s, -kE4m3Max), kE4m3Max);
    return (uint8_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
}

__global__ void __launch_bounds__(128) append_tokens_kernel(const AppendArgs a) {
    const int i = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = a.seq[i], s = a.pos[i];
    if (b < 0 || b >= a.B || s < 0 || s >= a.T_max) {
        if (tid == 0) record_status(a.status, DSA_STATUS_LENGTH);
        return;
    }
    int64_t row = (int64_t)b * a.T_max + s;
    if (a.block_table != nullptr) {
        const int pb = a.block_table[(int64_t)b * a.max_blocks + s / a.block_size];
        if (pb < 0 || pb >= a.num_blocks) {
            if (tid == 0) record_status(a.status, DSA_STATUS_INDEX_OOB);
            return;
        }
        row = (int64_t)pb * a.block_size + s % a.block_size;
    }
    __shared__ float red[4];

    // ---- indexer key: d_I values, one scale
    {
        const float* k = a.k_new + (int64_t)i * a.d_I;
        float m = 0.f;
        for (int x = tid; x < a.d_I; x += 128) m = fmaxf(m, fabsf(k[x]));
        m = warp_max(m);
        if (lane == 0) red[warp] = m;
        __syncthreads();
        const float amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        if (a.idx_fp8) {
            const float sc = amax > 0.f ? amax / kE4m3Max : 1.f;
            uint8_t* dst = reinterpret_cast<uint8_t*>(a.k_I) + row * a.d_I;
            for (int x = tid; x < a.d_I; x += 128) dst[x] = e4m3_of(k[x], sc);
            if (tid == 0) a.k_scale[row] = sc;
        } else {
            float* dst = reinterpret_cast<float*>(a.k_I) + row * a.d_I;
            for (int x = tid; x < a.d_I; x += 128) dst[x] = k[x];
        }
    }

    // ---- latent row
    const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(a.kv_new) + (int64_t)i * kDK;
    if (!a.kv_fp8) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.kv) + row * kDK;
        for (int x = tid; x < kDK; x += 128) dst[x] = v[x];
        return;
    }
    // FP8 entry: warp g quantises latent values [128 g, 128 g + 128) with their own scale
    uint8_t* e = reinterpret_cast<uint8_t*>(a.kv) + row * kFp8EntryBytes;
    float val[4];
    float m = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        val[u] = __bfloat162float(v[128 * warp + 32 * u + lane]);
        m = fmaxf(m, fabsf(val[u]));
    }
    m = warp_max(m);
    const float sc = m > 0.f ? m / kE4m3Max : 1.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) e[128 * warp + 32 * u + lane] = e4m3_of(val[u], sc);
    if (lane == 0) reinterpret_cast<float*>(e + kFp8ScaleOff)[warp] = sc;
    // rope: 64 bf16 values copied as they are
    if (tid < 64) reinterpret_cast<__nv_bfloat16*>(e + kFp8RopeOff)[tid] = v[512 + tid];
}

}  // namespace

cudaError_t launch_append_tokens(const AppendArgs& a, cudaStream_t st) {
    if (a.n == 0) return cudaSuccess;
    append_tokens_kernel<<<a.n, 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
