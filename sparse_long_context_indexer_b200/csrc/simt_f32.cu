// simt_f32.cu -- fp32 CUDA-core kernels for float-typed inputs (small problems:
// the fp32 tiny decode).  Same operations as the tensor-core path:
//   indexer  I[t,s] = sum_j w[t,j] ReLU(q_I[t,j] . k_I[s])
//            ("DeepSeek Sparse Attention Explained", "How Does the Lightning
//            Indexer Score a Token?")
//   attention over the selected rows with the softmax over that set only
//            (same page, "What Does the Whole Block Look Like?"), every head
//            sharing each latent row (MQA mode).
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "status.cuh"

namespace dsa {
namespace {

// One thread per cached token; the query's H_I x d_I block sits in shared memory.
template <int D_I>
__global__ void __launch_bounds__(256) indexer_f32_kernel(const IndexerArgs a) {
    extern __shared__ float qs[];  // [H_I * D_I] then w[H_I]
    float* ws = qs + a.H_I * D_I;
    const int t = blockIdx.y;
    int n = a.q_len[t];
    const int b = a.q_seq[t];
    if (n < 0 || n > a.T_max || (int64_t)n > a.ld || b < 0 || b >= a.B) {
        if (blockIdx.x == 0 && threadIdx.x == 0) record_status(a.status, DSA_STATUS_LENGTH);
        return;
    }
    const float* q = reinterpret_cast<const float*>(a.q_I) + (int64_t)t * a.H_I * D_I;
    for (int i = threadIdx.x; i < a.H_I * D_I; i += blockDim.x) qs[i] = q[i];
    for (int i = threadIdx.x; i < a.H_I; i += blockDim.x) ws[i] = reinterpret_cast<const float*>(a.w)[(int64_t)t * a.H_I + i];
    __syncthreads();
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n) return;
    const float4* kr = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.k_I) + ((int64_t)b * a.T_max + s) * D_I);
    float k[D_I];
#pragma unroll
    for (int x = 0; x < D_I / 4; ++x) {
        const float4 v = __ldg(kr + x);
        k[4 * x] = v.x;
        k[4 * x + 1] = v.y;
        k[4 * x + 2] = v.z;
        k[4 * x + 3] = v.w;
    }
    float acc = 0.f;
    for (int j = 0; j < a.H_I; ++j) {
        const float* qj = qs + j * D_I;
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int x = 0; x < D_I; x += 2) {
            d0 = fmaf(qj[x], k[x], d0);
            d1 = fmaf(qj[x + 1], k[x + 1], d1);
        }
        acc = fmaf(ws[j], fmaxf(d0 + d1, 0.f), acc);
    }
    a.scores[(int64_t)t * a.ld + s] = acc;
}

// One CTA per (head, row): logits of the selected rows, softmax, weighted sum.
__global__ void __launch_bounds__(256) sparse_mla_f32_kernel(const MlaArgs a) {
    extern __shared__ float sm[];
    float* qv = sm;                 // [576]
    float* z = sm + kDK;            // [k]
    int* pos = reinterpret_cast<int*>(z + a.k);  // [k]
    __shared__ float red[32];
    __shared__ float bcast;
    const int h = blockIdx.x, t = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int n_t = a.q_len[t];
    const int b = a.q_seq[t];
    const bool row_ok = n_t >= 0 && n_t <= a.T_max && b >= 0 && b < a.B;
    if (!row_ok) {
        if (h == 0 && tid == 0) record_status(a.status, DSA_STATUS_LENGTH);
        n_t = 0;
    }
    const float* q = reinterpret_cast<const float*>(a.q) + ((int64_t)t * a.H + h) * kDK;
    for (int x = tid; x < kDK; x += blockDim.x) qv[x] = q[x];
    const int32_t* idx = a.idx + (int64_t)t * a.k;
    for (int j = tid; j < a.k; j += blockDim.x) {
        int s = idx[j];
        if (s < -1 || s >= n_t) {
            if (h == 0 && row_ok) record_status(a.status, DSA_STATUS_INDEX_OOB);
            s = -1;
        }
        pos[j] = s;
    }
    __syncthreads();
    const float* kv = reinterpret_cast<const float*>(a.kv) + (int64_t)b * a.T_max * kDK;
    // logits: one warp per selected row, lanes over the 576 values
    for (int j = warp; j < a.k; j += blockDim.x / 32) {
        const int s = pos[j];
        float d = 0.f;
        if (s >= 0) {
            const float* c = kv + (int64_t)s * kDK;
            for (int x = lane; x < kDK; x += 32) d = fmaf(qv[x], c[x], d);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) z[j] = s >= 0 ? d * a.softmax_scale : -CUDART_INF_F;
    }
    __syncthreads();
    float m = -CUDART_INF_F;
    for (int j = tid; j < a.k; j += blockDim.x) m = fmaxf(m, z[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (tid == 0) {
        float mm = -CUDART_INF_F;
        for (int w = 0; w < (int)(blockDim.x / 32); ++w) mm = fmaxf(mm, red[w]);
        bcast = mm;
    }
    __syncthreads();
    m = bcast;
    float l = 0.f;
    for (int j = tid; j < a.k; j += blockDim.x) {
        const float p = (z[j] == -CUDART_INF_F) ? 0.f : expf(z[j] - m);
        z[j] = p;
        l += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    __syncthreads();
    if (lane == 0) red[warp] = l;
    __syncthreads();
    if (tid == 0) {
        float ll = 0.f;
        for (int w = 0; w < (int)(blockDim.x / 32); ++w) ll += red[w];
        bcast = ll;
    }
    __syncthreads();
    l = bcast;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* out = reinterpret_cast<float*>(a.out) + ((int64_t)t * a.H + h) * kDV;
    for (int x = tid; x < kDV; x += blockDim.x) {
        float acc = 0.f;
        for (int j = 0; j < a.k; ++j) {
            const int s = pos[j];
            if (s >= 0 && z[j] != 0.f) acc = fmaf(z[j], kv[(int64_t)s * kDK + x], acc);
        }
        out[x] = acc * inv;
    }
    if (tid == 0 && a.lse) a.lse[(int64_t)t * a.H + h] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
}

}  // namespace

cudaError_t launch_indexer_f32(const IndexerArgs& a, cudaStream_t st) {
    if (a.Nq == 0 || a.T_max == 0) return cudaSuccess;
    const size_t smem = (size_t)(a.H_I * a.d_I + a.H_I) * sizeof(float);
    dim3 grid((a.T_max + 255) / 256, a.Nq);
    if (a.d_I == 64) {
        indexer_f32_kernel<64><<<grid, 256, smem, st>>>(a);
    } else if (a.d_I == 128) {
        indexer_f32_kernel<128><<<grid, 256, smem, st>>>(a);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_sparse_mla_f32(const MlaArgs& a, cudaStream_t st) {
    if (a.Nq == 0) return cudaSuccess;
    const size_t smem = (size_t)kDK * sizeof(float) + (size_t)a.k * (sizeof(float) + sizeof(int));
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.H, a.Nq);
    sparse_mla_f32_kernel<<<grid, 256, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
