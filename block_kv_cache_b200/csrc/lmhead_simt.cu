// LM head fused with the vocabulary-wide (max, sum exp, argmax) reduction,
// SIMT FFMA version for f32 inputs (a TF32 tensor-core product would not
// hold the f32 path's tolerances; bf16 inputs go to lmhead_bf16.cu).
//
// Fast-dLLM, confidence-aware parallel decoding (abstract; README "Key
// techniques" 2): each masked row's confidence is the probability of its
// predicted token, exp(max z - logsumexp z), and the token is the argmax.
// The [M, V] logits are reduced where they are produced and never stored.
//
// Pass 1 (this file): CTA tile = 32 rows x 128 vocab entries, K stepped by
// 32 through shared memory, 4x4 outputs per thread. The epilogue adds the
// planted bias, then each warp reduces its 4 rows over the tile's 128
// columns to a partial (max, sum exp(z - max), lowest argmax) per (row, tile).
// Pass 2 (lmhead_combine.cu): per row, merge the partials of all tiles.
#include "common.cuh"
#include "launch.h"
#include "lmhead_common.cuh"

namespace fdl {

constexpr int LS_BM = 32, LS_BN = 128, LS_BK = 32;

template <typename T>
__global__ void __launch_bounds__(256)
lmhead_simt_kernel(const T* __restrict__ h, const T* __restrict__ w,
                   const int32_t* __restrict__ bias_tok, const float* __restrict__ bias_val,
                   LMPartial* __restrict__ part, int M, int D, int V) {
    __shared__ float As[LS_BM][LS_BK];
    __shared__ float Bs[LS_BN][LS_BK + 1];
    const int vt = blockIdx.x, mt = blockIdx.y;
    const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;   // ty = warp: rows 4ty..4ty+3
    const int row0 = mt * LS_BM, col0 = vt * LS_BN;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < D; k0 += LS_BK) {
        __syncthreads();
        for (int e = tid; e < LS_BM * LS_BK; e += 256) {
            const int r = e / LS_BK, kk = e % LS_BK;
            As[r][kk] = (row0 + r < M) ? to_f32(h[(size_t)(row0 + r) * D + k0 + kk]) : 0.f;
        }
        for (int e = tid; e < LS_BN * LS_BK; e += 256) {
            const int c = e / LS_BK, kk = e % LS_BK;
            Bs[c][kk] = (col0 + c < V) ? to_f32(w[(size_t)(col0 + c) * D + k0 + kk]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < LS_BK; ++kk) {
            float a[4], bv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = As[ty * 4 + r][kk];
#pragma unroll
            for (int c = 0; c < 4; ++c) bv[c] = Bs[tx + 32 * c][kk];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], bv[c], acc[r][c]);
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int row = row0 + ty * 4 + r;
        if (row >= M) break;                              // uniform across the warp
        const int bt = bias_tok ? bias_tok[row] : -1;
        const float bv = bias_tok ? bias_val[row] : 0.f;
        float z[4];
        float mx = -INFINITY;
        int arg = INT_MAX;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int col = col0 + tx + 32 * c;
            z[c] = (col < V) ? acc[r][c] + (col == bt ? bv : 0.f) : -INFINITY;
            if (z[c] > mx) { mx = z[c]; arg = col; }       // cols ascending in c
        }
        warp_argmax_lowest(mx, arg);
        float se = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) se += (z[c] == -INFINITY) ? 0.f : expf(z[c] - mx);
        se = warp_sum(se);
        if (tx == 0) part[(size_t)vt * M + row] = LMPartial{mx, se, arg};
    }
}

template <typename T>
static cudaError_t run_lmhead_simt(const LMShape& s, const T* h, const T* w,
                                   const int32_t* bias_tok, const float* bias_val,
                                   float* conf, int32_t* tok, void* ws, cudaStream_t st) {
    const int nvt = (s.vocab + LS_BN - 1) / LS_BN;
    LMPartial* part = (LMPartial*)ws;
    dim3 grid(nvt, (s.rows + LS_BM - 1) / LS_BM);
    lmhead_simt_kernel<T><<<grid, 256, 0, st>>>(h, w, bias_tok, bias_val, part, s.rows, s.hidden,
                                             s.vocab);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_lmhead_combine(part, nvt, s.rows, conf, tok, st);
}

cudaError_t launch_lmhead_f32(const LMShape& s, const float* h, const float* w,
                              const int32_t* bias_tok, const float* bias_val,
                              float* conf, int32_t* tok, void* ws, cudaStream_t st) {
    return run_lmhead_simt<float>(s, h, w, bias_tok, bias_val, conf, tok, ws, st);
}
}  // namespace fdl
