// Host-side launchers shared between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gemm.h"

namespace fdl {

struct AttnShape {
    int batch, n_q_heads, n_kv_heads, head_dim, seq_len, block_start, block_len;
    float scale;  // resolved (never 0)
    int bf16;     // 1: bf16 tensors (tcgen05 kernel), 0: f32 (SIMT kernel)
    int q_per_kv = 1;   // query blocks per sequence: batch counts query blocks,
                        // sequence index = batch index / q_per_kv (full attention)
    // Compacted batch (q_per_kv == 1): query block i reads the caches of
    // sequence seq_map[i], and the caches hold kv_batch sequences (null / 0:
    // the identity and batch).
    const int32_t* seq_map = nullptr;
    int kv_batch = 0;
    // Sequences at their own blocks: query block i's block slot starts at
    // blk0_map[i] (null: at block_start for all).
    const int32_t* blk0_map = nullptr;
};

// Query the cluster capacities the attention launches use to size their split
// count (once per process; call outside stream capture).
void attn_tc_warm();

// Scratch for the split-KV partials of either attention kernel.
size_t attn_workspace_bytes(const AttnShape& s, int sm_count);
size_t attn_tc_workspace_bytes(const AttnShape& s, int sm_count);

cudaError_t launch_attention_f32(const AttnShape& s, const float* q, const float* k,
                                 const float* v, float* out, float* lse, void* ws,
                                 int sm_count, cudaStream_t st);
cudaError_t launch_attention_bf16(const AttnShape& s, const void* q, const void* k,
                                  const void* v, void* out, float* lse, void* ws,
                                  int sm_count, int* dev_err, cudaStream_t st);

// Block-slot projection fused with DualCache attention: the split-K sums of
// the q/k/v projection (acc, rows x N f32, zero-kept) are finished (bias,
// RoPE, zeros restored) by the CTAs of the attention kernel: each forms its
// query tile in shared memory (and split 0 writes q) and writes the block-slot
// K/V rows of its own key range, then the attention runs. Only when
// qkv_attention_fusable(s): bf16, head_dim 128, one query block per sequence
// and the whole GQA group of a kv head in one CTA.
bool qkv_attention_fusable(const AttnShape& s, int sm_count);
cudaError_t launch_qkv_attention_bf16(const AttnShape& s, float* acc, const EpiQKV& pq, void* out,
                                      int sm_count, int* err, cudaStream_t st);

// Full bidirectional attention of the last n_q positions of every sequence
// over all seq_len positions (n_q = seq_len: the refresh forward; n_q = L - s:
// a PrefixCache step): q, out [b, n_q, Hq, d] bf16; caches [b, Hkv, L, d].
// With seq_map, sequence i of q/out is sequence seq_map[i] of caches that hold
// kv_batch sequences.
cudaError_t launch_full_attention_bf16(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                       int seq_len, int n_q, float scale, const void* q,
                                       const void* k, const void* v, void* out, int sm_count,
                                       int* dev_err, cudaStream_t st,
                                       const int32_t* seq_map = nullptr, int kv_batch = 0);

cudaError_t launch_kv_store(int batch, int n_kv_heads, int head_dim, int seq_len,
                            int elem_bytes, const void* k_new, const void* v_new,
                            int start, int n, void* k_cache, void* v_cache,
                            cudaStream_t st);

struct LMShape { int rows, hidden, vocab; };
size_t lmhead_workspace_bytes(const LMShape& s);
cudaError_t launch_lmhead_f32(const LMShape& s, const float* h, const float* w,
                              const int32_t* bias_tok, const float* bias_val,
                              float* conf, int32_t* tok, void* ws, cudaStream_t st);
cudaError_t launch_lmhead_bf16(const LMShape& s, const void* h, const void* w,
                               const int32_t* bias_tok, const float* bias_val,
                               float* conf, int32_t* tok, void* ws, int sm_count,
                               int* dev_err, cudaStream_t st);

cudaError_t launch_threshold_unmask(int batch, int seq_len, int block_start,
                                    int block_len, float tau, const float* conf,
                                    const int32_t* tok, int32_t* x, uint8_t* masked,
                                    int32_t* remaining, int32_t* n_decoded,
                                    int* dev_err, cudaStream_t st,
                                    const int32_t* seq_map = nullptr,
                                    const int32_t* s_map = nullptr);

}  // namespace fdl
