// Row-wise kernels of the bidirectional transformer around the Fast-dLLM
// step (LLaDA / Dream family: pre-norm blocks with RMSNorm): RMSNorm of the
// f32 residual stream into the bf16 GEMM input (optionally gathering rows,
// e.g. the current block's rows after a refresh forward), and the token
// embedding gather. Both are HBM-bound copies of one row per CTA.
#include "gemm.h"

namespace fdl {

constexpr int NORM_THREADS = 256;

__global__ void __launch_bounds__(NORM_THREADS)
rmsnorm_kernel(const float* __restrict__ h, const int32_t* __restrict__ row_map,
               const float* __restrict__ weight, float eps, bf16* __restrict__ out, int hidden) {
    pdl_wait();
    pdl_trigger();
    __shared__ float s_red[NORM_THREADS / 32];
    const int i = blockIdx.x;
    const int src = row_map ? row_map[i] : i;
    const float4* x = reinterpret_cast<const float4*>(h + (size_t)src * hidden);
    const int n4 = hidden / 4;
    float ss = 0.f;
    for (int j = threadIdx.x; j < n4; j += NORM_THREADS) {
        const float4 v = x[j];
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = threadIdx.x < NORM_THREADS / 32 ? s_red[threadIdx.x] : 0.f;
        t = warp_sum(t);
        if (threadIdx.x == 0) s_red[0] = t;
    }
    __syncthreads();
    const float inv = rsqrtf(s_red[0] / (float)hidden + eps);
    const float4* w4 = reinterpret_cast<const float4*>(weight);
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(out + (size_t)i * hidden);
    for (int j = threadIdx.x; j < n4; j += NORM_THREADS) {
        const float4 v = x[j], w = w4[j];
        o2[2 * j] = __floats2bfloat162_rn(v.x * inv * w.x, v.y * inv * w.y);
        o2[2 * j + 1] = __floats2bfloat162_rn(v.z * inv * w.z, v.w * inv * w.w);
    }
}

__global__ void __launch_bounds__(NORM_THREADS)
embed_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ row_map,
             const bf16* __restrict__ table, float* __restrict__ h, int hidden) {
    pdl_wait();
    pdl_trigger();
    const int i = blockIdx.x;
    const int id = ids[row_map ? row_map[i] : i];
    const __nv_bfloat162* src = reinterpret_cast<const __nv_bfloat162*>(table + (size_t)id * hidden);
    float2* dst = reinterpret_cast<float2*>(h + (size_t)i * hidden);
    for (int j = threadIdx.x; j < hidden / 2; j += NORM_THREADS) dst[j] = __bfloat1622float2(src[j]);
}

cudaError_t launch_rmsnorm(int rows, int hidden, const float* h, const int32_t* row_map,
                           const float* weight, float eps, bf16* out, cudaStream_t st) {
    return launch_pdl(rmsnorm_kernel, dim3(rows), dim3(NORM_THREADS), 0, st, 0, h, row_map, weight,
                      eps, out, hidden);
}

cudaError_t launch_embed(int rows, int hidden, const int32_t* ids, const int32_t* row_map,
                         const bf16* table, float* h, cudaStream_t st) {
    return launch_pdl(embed_kernel, dim3(rows), dim3(NORM_THREADS), 0, st, 0, ids, row_map, table,
                      h, hidden);
}

}  // namespace fdl
