// Host-side interface of the fused-epilogue GEMMs (gemm_bf16.cu) and the
// row-wise kernels of the transformer scaffold (norm.cu).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace fdl {

struct GemmShape { int M, N, K; };

struct EpiResid {            // h[M, N] (f32, row stride ldh) += A W^T
    float* h;
    int ldh;
};

struct EpiSwiGLU {           // out[M, N/2] (bf16, row stride ldo)
    bf16* out;
    int ldo;
};

struct EpiQKV {              // N = (n_q_heads + 2 n_kv_heads) * 128
    bf16* q;                 // [M, n_q_heads, 128]
    bf16* k_cache;           // [b, n_kv_heads, seq_len, 128]
    bf16* v_cache;
    const float* bias;       // [N] or null
    const float2* rope;      // [max_pos, 64] (cos, sin)
    int n_q_heads, n_kv_heads, seq_len;
    int rows_per_seq;        // row r belongs to sequence r / rows_per_seq ...
    int pos0;                // ... at position pos0 + r % rows_per_seq
    // Compacted batch: the rows of sequence i write the cache rows of sequence
    // seq_map[i] (null: of sequence i).
    const int32_t* seq_map = nullptr;
    // Sequences at their own positions: sequence i's rows start at position
    // pos0_map[i] (null: at pos0).
    const int32_t* pos0_map = nullptr;
    __device__ __forceinline__ int cache_seq(int i) const {
        return seq_map ? __ldg(seq_map + i) : i;
    }
    __device__ __forceinline__ int pos0_of(int i) const {
        return pos0_map ? __ldg(pos0_map + i) : pos0;
    }
};

cudaError_t launch_gemm_resid(const GemmShape& g, const void* a, const void* w,
                              const EpiResid& p, int sm_count, int* err, cudaStream_t st);
cudaError_t launch_gemm_swiglu(const GemmShape& g, const void* a, const void* w,
                               const EpiSwiGLU& p, int sm_count, int* err, cudaStream_t st);
cudaError_t launch_gemm_qkv(const GemmShape& g, const void* a, const void* w, const EpiQKV& p,
                            int sm_count, int* err, cudaStream_t st);

// Token-few variants (M <= 256, N % 128 == 0): weight rows on the MMA's M side.
bool skinny_ok(const GemmShape& g);
cudaError_t launch_skinny_resid(const GemmShape& g, const void* x, const void* w,
                                const EpiResid& p, int sm_count, int* err, cudaStream_t st);
// acc: f32 scratch of acc_bytes, all zeros; split-K partial sums go there and
// the finishing kernel restores the zeros. Too small or NULL: no K split.
cudaError_t launch_skinny_swiglu(const GemmShape& g, const void* x, const void* w,
                                 const EpiSwiGLU& p, float* acc, size_t acc_bytes, int sm_count,
                                 int* err, cudaStream_t st);
cudaError_t launch_skinny_qkv(const GemmShape& g, const void* x, const void* w, const EpiQKV& p,
                              float* acc, size_t acc_bytes, int sm_count, int* err,
                              cudaStream_t st);

// RMSNorm applied by a fused kernel to its activation rows: x = bf16(h *
// rsqrt(mean(h^2) + eps) * w), x then being the kernel's operand.
struct NormIn {
    const float* h;          // [rows, hidden] f32 residual stream
    const float* w;          // [hidden]
    float eps;
};

// K splits the few-row q/k/v projection uses with an accumulator of acc_bytes
// (1: none), and the projection alone leaving its split-K sums in acc (the
// epilogue is then up to the caller: launch_qkv_attention_bf16).
int skinny_qkv_splits(const GemmShape& g, size_t acc_bytes, int sm_count);
// With norm, the projection's CTAs first write x = RMSNorm(h) (grid barrier
// on the 64-bit counter at bar).
cudaError_t launch_skinny_qkv_sums(const GemmShape& g, const void* x, const void* w, float* acc,
                                   int splits, const NormIn* norm, unsigned* bar, int sm_count,
                                   int* err, cudaStream_t st);

// Feed-forward block for M <= 256 rows: h[M, ld_h] += down(SwiGLU(x W_gu^T)),
// w_gu [2F, K] interleaved (row 2f gate, 2f + 1 up), w_down [ld_h, F], f [M, F]
// bf16 scratch (the down projection's operand). acc/acc_bytes as above; bar:
// four zeroed words for the grid barriers. With norm, x is first written as
// RMSNorm(norm->h) by the gate/up projection's CTAs.
cudaError_t launch_skinny_ffn(const GemmShape& g_gu, const void* x, const void* w_gu,
                              const void* w_down, bf16* f, float* h, int ld_h, float* acc,
                              size_t acc_bytes, unsigned* bar, const NormIn* norm, int sm_count,
                              int* err, cudaStream_t st);

// out[i, :] = bf16(h[src_i, :] / sqrt(mean(h[src_i]^2) + eps) * weight), src_i =
// row_map ? row_map[i] : i.
cudaError_t launch_rmsnorm(int rows, int hidden, const float* h, const int32_t* row_map,
                           const float* weight, float eps, bf16* out, cudaStream_t st);
// h[i, :] = f32(table[ids[j], :]), j = row_map ? row_map[i] : i
cudaError_t launch_embed(int rows, int hidden, const int32_t* ids, const int32_t* row_map,
                         const bf16* table, float* h, cudaStream_t st);

}  // namespace fdl
