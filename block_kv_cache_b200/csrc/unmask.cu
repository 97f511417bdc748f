// Confidence-aware parallel unmask: threshold select + scatter.
//
// Fast-dLLM (arXiv 2505.22618), abstract and README "Key techniques" 2: at
// each step every masked token whose confidence exceeds the threshold is
// decoded in parallel; the others stay masked for later steps. When no
// candidate exceeds it, the single most confident candidate (lowest position
// on ties) is decoded so that every step makes progress.
//
// One CTA per sequence, one thread per block position. With a compacted batch
// (only the sequences that still have masked positions in the block), CTA i
// reads row i of conf/tok and updates sequence seq_map[i]; with s_map, that
// sequence's block starts at s_map[i] instead of block_start. The work is a few
// compares per position, so the kernel is latency-bound; it reads B floats,
// B ints and B bytes per sequence and writes at most B ints and B bytes.
#include "common.cuh"
#include "launch.h"
#include <climits>

namespace fdl {

__global__ void __launch_bounds__(1024)
threshold_unmask_kernel(const float* __restrict__ conf, const int32_t* __restrict__ tok,
                        int32_t* __restrict__ x, uint8_t* __restrict__ masked,
                        int32_t* __restrict__ remaining, int32_t* __restrict__ n_decoded,
                        int L, int s, int B, float tau, const int32_t* __restrict__ seq_map,
                        const int32_t* __restrict__ s_map, int* err) {
    pdl_wait();
    pdl_trigger();
    __shared__ float s_val[32];
    __shared__ int s_idx[32];
    __shared__ int s_win;
    const int ci = blockIdx.x;                      // row of conf / tok
    const int b = seq_map ? seq_map[ci] : ci;       // sequence updated
    if (s_map) s = s_map[ci];                       // its own block
    const int j = threadIdx.x;
    const int lane = j & 31, warp = j >> 5, nwarps = blockDim.x >> 5;

    bool cand = false;
    float c = 0.f;
    if (j < B) {
        cand = masked[(size_t)b * L + s + j] != 0;
        c = conf[(size_t)ci * B + j];
    }
    const bool above = cand && (c > tau);          // NaN > tau is false
    const int any_above = __syncthreads_or(above);
    const int any_cand = __syncthreads_or(cand);
    bool sel = above;
    if (!any_above && any_cand) {
        // most confident valid candidate, lowest position on ties
        const bool valid = cand && !isnan(c);
        float v = valid ? c : -INFINITY;
        int idx = valid ? j : INT_MAX;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float v2 = __shfl_xor_sync(0xffffffffu, v, o);
            int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
            if (v2 > v || (v2 == v && i2 < idx)) { v = v2; idx = i2; }
        }
        if (lane == 0) { s_val[warp] = v; s_idx[warp] = idx; }
        __syncthreads();
        if (j == 0) {
            float bv = s_val[0];
            int bi = s_idx[0];
            for (int w = 1; w < nwarps; ++w)
                if (s_val[w] > bv || (s_val[w] == bv && s_idx[w] < bi)) { bv = s_val[w]; bi = s_idx[w]; }
            s_win = bi;
            if (bi == INT_MAX) record_error(err, DEV_NO_PROGRESS);
        }
        __syncthreads();
        sel = (j == s_win);
    }
    if (sel) {
        x[(size_t)b * L + s + j] = tok[(size_t)ci * B + j];
        masked[(size_t)b * L + s + j] = 0;
    }
    const int rem = __syncthreads_count(cand && !sel);
    const int nd = __syncthreads_count(sel);
    if (j == 0) {
        remaining[b] = rem;
        if (n_decoded) n_decoded[b] = nd;
    }
}

cudaError_t launch_threshold_unmask(int batch, int seq_len, int block_start,
                                    int block_len, float tau, const float* conf,
                                    const int32_t* tok, int32_t* x, uint8_t* masked,
                                    int32_t* remaining, int32_t* n_decoded,
                                    int* dev_err, cudaStream_t st, const int32_t* seq_map,
                                    const int32_t* s_map) {
    int threads = ((block_len + 31) / 32) * 32;
    return launch_pdl(threshold_unmask_kernel, dim3(batch), dim3(threads), 0, st, 0, conf, tok, x,
                      masked, remaining, n_decoded, seq_len, block_start, block_len, tau,
                      seq_map, s_map, dev_err);
}

}  // namespace fdl
