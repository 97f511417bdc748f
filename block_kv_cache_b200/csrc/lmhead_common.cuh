// Partial results of the fused LM-head reduction and their merge.
#pragma once
#include "common.cuh"
#include <climits>

namespace fdl {

// One (row, vocab tile) partial: tile max, sum of exp(z - max) over the tile,
// lowest vocab id attaining the max (INT_MAX if the tile had no valid entry).
struct LMPartial {
    float mx;
    float se;
    int arg;
};

// Warp-wide (max, lowest index attaining it).
__device__ __forceinline__ void warp_argmax_lowest(float& mx, int& arg) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, mx, o);
        const int a2 = __shfl_xor_sync(0xffffffffu, arg, o);
        if (m2 > mx || (m2 == mx && a2 < arg)) { mx = m2; arg = a2; }
    }
}

// part: [n_tiles][M]; writes conf[M], tok[M].
cudaError_t launch_lmhead_combine(const LMPartial* part, int n_tiles, int M, float* conf,
                                  int32_t* tok, cudaStream_t st);

}  // namespace fdl
