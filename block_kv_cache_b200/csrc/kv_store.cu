// In-place K/V cache store: the block slot at every DualCache step, or every
// row at a refresh (Fast-dLLM: all K/V are recomputed once a block
// completes; ICLR reviews, review 4 question 2).
//
// Token-major fresh rows [b, n, Hkv, d] are transposed into the head-major
// cache [b, Hkv, L, d]; each head row of d elements is moved as 16-byte
// vectors. Pure copy: HBM-bound at 2 * (read + write) = 4 * b*n*Hkv*d*esize
// bytes per call.
#include "common.cuh"
#include "launch.h"

namespace fdl {

__global__ void kv_store_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                long long total, int n, int Hkv, int chunks, int L, int start) {
    pdl_wait();
    pdl_trigger();
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(idx % chunks);
        long long t = idx / chunks;
        const int h = (int)(t % Hkv);
        t /= Hkv;
        const int i = (int)(t % n);
        const long long bb = t / n;
        const long long src = ((bb * n + i) * Hkv + h) * chunks + c;
        const long long dst = ((bb * Hkv + h) * (long long)L + start + i) * chunks + c;
        k_cache[dst] = k_new[src];
        v_cache[dst] = v_new[src];
    }
}

cudaError_t launch_kv_store(int batch, int n_kv_heads, int head_dim, int seq_len,
                            int elem_bytes, const void* k_new, const void* v_new,
                            int start, int n, void* k_cache, void* v_cache,
                            cudaStream_t st) {
    const int chunks = head_dim * elem_bytes / 16;
    const long long total = (long long)batch * n * n_kv_heads * chunks;
    const int threads = 256;
    long long blocks = (total + threads - 1) / threads;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    return launch_pdl(kv_store_kernel, dim3((int)blocks), dim3(threads), 0, st, 0,
                      (const uint4*)k_new, (const uint4*)v_new, (uint4*)k_cache, (uint4*)v_cache,
                      total, n, n_kv_heads, chunks, seq_len, start);
}

}  // namespace fdl
