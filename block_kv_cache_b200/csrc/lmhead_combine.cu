// Merge of the per-tile (max, sum exp, argmax) partials of the fused LM head:
//   M = max_t m_t,  S = sum_t s_t * exp(m_t - M),  conf = 1 / S,
//   tok = lowest id among the tiles attaining M.
// One warp per row; the partials of a row are strided by M in memory.
#include "lmhead_common.cuh"
#include "launch.h"

namespace fdl {

__global__ void lmhead_combine_kernel(const LMPartial* __restrict__ part, int n_tiles, int M,
                                      float* __restrict__ conf, int32_t* __restrict__ tok) {
    pdl_wait();
    pdl_trigger();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= M) return;
    float mx = -INFINITY;
    int arg = INT_MAX;
    for (int t = lane; t < n_tiles; t += 32) {
        const LMPartial p = part[(size_t)t * M + warp];
        if (p.mx > mx || (p.mx == mx && p.arg < arg)) { mx = p.mx; arg = p.arg; }
    }
    warp_argmax_lowest(mx, arg);
    float se = 0.f;
    for (int t = lane; t < n_tiles; t += 32) {
        const LMPartial p = part[(size_t)t * M + warp];
        if (p.mx != -INFINITY) se += p.se * expf(p.mx - mx);
    }
    se = warp_sum(se);
    if (lane == 0) {
        conf[warp] = 1.0f / se;
        tok[warp] = arg;
    }
}

cudaError_t launch_lmhead_combine(const LMPartial* part, int n_tiles, int M, float* conf,
                                  int32_t* tok, cudaStream_t st) {
    const int threads = 256;
    const int blocks = (M * 32 + threads - 1) / threads;
    return launch_pdl(lmhead_combine_kernel, dim3(blocks), dim3(threads), 0, st, 0, part, n_tiles,
                      M, conf, tok);
}

}  // namespace fdl
