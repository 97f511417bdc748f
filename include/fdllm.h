/*
 * fdllm.h - C ABI of the B200 (sm_100a) Fast-dLLM block-decoding step.
 *
 * The library computes one decoding step of a masked diffusion LLM with the
 * two techniques of "Fast-dLLM: Training-free Acceleration of Diffusion LLM
 * by Enabling KV Cache and Parallel Decoding" (arXiv 2505.22618):
 *   (a) DualCache block attention: the current block's queries attend,
 *       without a causal mask, over [cached prefix K/V | fresh block K/V |
 *       cached masked-suffix K/V]; the caches are rewritten when a block
 *       completes;
 *   (b) confidence-aware parallel unmasking: the LM head over the block's
 *       rows is reduced on the fly to (confidence, token) per row, and every
 *       masked position whose confidence exceeds a threshold is decoded.
 *
 * Conventions shared by every entry point
 *  - All pointers named as device buffers are CUDA device pointers on the
 *    context's device, owned by the caller. The library never allocates or
 *    frees them; scratch memory is passed in by the caller (`ws`), sized by
 *    the matching *_workspace_bytes query.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Every compute
 *    call is asynchronous on that stream: it returns after enqueueing. The
 *    exception is fdl_generate, whose decode loop reads a few counters back
 *    after every step and returns when the decode is complete.
 *  - Return value: FDL_OK (0) or a negative fdl_status. Argument errors are
 *    detected on the host before anything is enqueued, so nothing runs on an
 *    error return. fdl_last_error() gives a message for the calling thread's
 *    last failure. No C++ exception crosses this boundary.
 *  - Faults found on the device (a bounded wait that ran out, a confidence
 *    that is NaN for every candidate) never trap: the kernel records a code in
 *    the context's device error word and finishes; fdl_get_device_status()
 *    reports and clears it.
 *  - Layouts are row-major with the last named dimension contiguous.
 *    bf16 is IEEE bfloat16 (as torch.bfloat16); f32 is IEEE single.
 */
#ifndef FDLLM_H
#define FDLLM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FDL_ABI_VERSION 6

#if defined(__GNUC__)
#define FDL_API __attribute__((visibility("default")))
#else
#define FDL_API
#endif

typedef enum {
    FDL_OK = 0,
    FDL_EINVAL = -1,        /* bad argument: null pointer, shape, alignment, value */
    FDL_EUNSUPPORTED = -2,  /* valid but not implemented (e.g. head_dim 96) */
    FDL_ECUDA = -3,         /* a CUDA runtime/driver call failed */
    FDL_ETIMEOUT = -4,      /* device: a bounded wait ran out */
    FDL_EWORKSPACE = -5,    /* ws is NULL or smaller than the query says */
    FDL_EDEVICE = -6        /* device: the step could not make progress (all-NaN confidences) */
} fdl_status;

typedef enum { FDL_F32 = 0, FDL_BF16 = 1 } fdl_dtype;

typedef struct fdl_ctx fdl_ctx;   /* opaque: device id, device error word, launch config */

/* ABI version of the loaded library (FDL_ABI_VERSION it was built with). */
FDL_API int fdl_abi_version(void);

/* Create a context on CUDA device `device`. Allocates, once, here (the only
 * device allocations the library makes): the 4-byte device error word, a 32 MiB
 * zero-filled f32 accumulator used by the few-token projections to add
 * split-K partial sums (every kernel that adds into it leaves it zeroed), and
 * 256 zeroed bytes for the grid-wide barriers of fused kernels. After a call
 * has reported FDL_ETIMEOUT these may be inconsistent: destroy the context.
 * Because of that shared accumulator, the calls made on one context must be
 * ordered on the GPU (one stream, or streams ordered by events); use one
 * context per concurrent stream. Fails with FDL_EUNSUPPORTED unless the device
 * is compute capability 10.0 (B200). *out is set to NULL on failure. */
FDL_API int fdl_create(fdl_ctx** out, int device);

/* Free the context and its device buffers. NULL is accepted. */
FDL_API int fdl_destroy(fdl_ctx* ctx);

/* Message for the calling thread's last non-OK return ("" if none). The
 * pointer stays valid until the thread's next failing call. */
FDL_API const char* fdl_last_error(void);

/* Synchronise `stream`, read the device error word, clear it, and return
 * FDL_OK, FDL_ETIMEOUT or FDL_EDEVICE accordingly. */
FDL_API int fdl_get_device_status(fdl_ctx* ctx, void* stream);

/* Limit, in ns, of the bounded waits with which the kernels launched on this
 * context wait for progress (a TMA load, an MMA, another CTA, another
 * warp's results); 2 s after fdl_create. A wait that runs out makes its CTA
 * give up: it records FDL_ETIMEOUT in the device error word, waits (with the
 * fixed 2 s limit) for the copies and tensor-core operations it has already
 * started, frees its TMEM and returns, leaving the call's outputs undefined;
 * the context must then be destroyed and created again. The library's own
 * failure-detection test shortens the limit to make a wait run out on purpose.
 * Synchronises the device; applies to kernels launched afterwards.
 * ns in [1, 60e9]. Errors: FDL_EINVAL, FDL_ECUDA. */
FDL_API int fdl_set_wait_timeout(fdl_ctx* ctx, uint64_t ns);

/* ------------------------------------------------------------------------
 * (a) DualCache block attention
 * ------------------------------------------------------------------------ */
typedef struct {
    int batch;        /* b  >= 1 sequences (all of length seq_len) */
    int n_q_heads;    /* Hq >= 1 */
    int n_kv_heads;   /* Hkv >= 1, Hq % Hkv == 0; q head h reads kv head h / (Hq/Hkv) */
    int head_dim;     /* d in {64, 128} */
    int seq_len;      /* L = prefix + block + suffix, >= 1 */
    int block_start;  /* s, first position of the current block */
    int block_len;    /* B, 1 <= B <= 128, s + B <= L */
    int dtype;        /* fdl_dtype of q, caches and out; accumulation is f32 */
    float scale;      /* softmax scale; 0 means 1/sqrt(head_dim) */
} fdl_attn_desc;

/* Bytes of scratch fdl_dualcache_attention needs for this shape on ctx's
 * device (split-KV partial results; the split count follows the device's SM
 * count). Returns 0 for an invalid context or descriptor. */
FDL_API size_t fdl_attention_workspace_bytes(const fdl_ctx* ctx, const fdl_attn_desc* desc);

/* DualCache block attention (Fast-dLLM: block-wise approximate KV cache,
 * DualCache variant; aibase news "Innovations" 1, README "Key techniques" 1).
 *
 * For each sequence b, q-head h and block row i:
 *   out[b,i,h,:] = sum_j softmax_j(scale * q[b,i,h,:] . K[b,g,j,:]) V[b,g,j,:]
 * over ALL j in [0, L) (bidirectional: no mask), g = h / (Hq/Hkv). The cache
 * rows [s, s+B) must already hold the block's fresh K/V (fdl_kv_store); the
 * other rows are the cached prefix and masked-suffix K/V.
 *
 *   q       [b, B, Hq, d]   dtype, device, 16-byte aligned
 *   k_cache [b, Hkv, L, d]  dtype, device, 16-byte aligned
 *   v_cache [b, Hkv, L, d]  dtype, device, 16-byte aligned
 *   out     [b, B, Hq, d]   dtype, device (written)
 *   lse     [b, Hq, B] f32, device, optional (NULL = not written):
 *           natural-log softmax denominator, lse = log sum_j exp(scale q.k_j)
 *   ws      device scratch of >= fdl_attention_workspace_bytes(desc) bytes
 * Errors: FDL_EINVAL (shape, null, alignment), FDL_EUNSUPPORTED (head_dim),
 * FDL_EWORKSPACE, FDL_ECUDA. */
FDL_API int fdl_dualcache_attention(fdl_ctx* ctx, const fdl_attn_desc* desc,
                            const void* q, const void* k_cache,
                            const void* v_cache, void* out, float* lse,
                            void* ws, size_t ws_bytes, void* stream);

/* Store fresh K/V rows into the caches in place: the block slot at every
 * step (start = s, n = B) and the whole cache at a refresh after a block
 * completes (start = 0, n = L; ICLR reviews, review 4 question 2: all K/V
 * are recomputed once a block is done).
 *
 *   k_new, v_new [b, n, Hkv, d] dtype, device (token-major, as a projection
 *                writes them), 16-byte aligned
 *   k_cache, v_cache [b, Hkv, L, d] dtype, device; rows [start, start+n)
 *                written, all other rows untouched
 * Uses desc->batch, n_kv_heads, head_dim, seq_len, dtype.
 * Errors: FDL_EINVAL (start < 0, start + n > L, n < 1, null, alignment). */
FDL_API int fdl_kv_store(fdl_ctx* ctx, const fdl_attn_desc* desc, const void* k_new,
                 const void* v_new, int start, int n, void* k_cache,
                 void* v_cache, void* stream);

/* ------------------------------------------------------------------------
 * (b) LM head fused with the vocabulary-wide confidence reduction
 * ------------------------------------------------------------------------ */
typedef struct {
    int rows;     /* M >= 1 hidden rows (the block's masked positions) */
    int hidden;   /* D, multiple of 64 */
    int vocab;    /* V >= 2 */
    int dtype;    /* fdl_dtype of h and w; logits and reductions are f32 */
} fdl_lmhead_desc;

/* Bytes of scratch fdl_lmhead_confidence needs (per-tile partial maxima,
 * sums and arguments). Returns 0 for an invalid context or descriptor. */
FDL_API size_t fdl_lmhead_workspace_bytes(const fdl_ctx* ctx, const fdl_lmhead_desc* desc);

/* Confidence of each row (Fast-dLLM abstract and README "Key techniques" 2:
 * tokens are decoded when their confidence exceeds a threshold; confidence is
 * read as the largest softmax probability of the predicted token).
 *
 *   z[r, v]  = h[r,:] . w[v,:] (+ bias_val[r] if v == bias_tok[r])   (f32)
 *   conf[r]  = exp(max_v z - logsumexp_v z) = 1 / sum_v exp(z[r,v] - max z)
 *   tok[r]   = smallest v with z[r, v] == max z
 * The [M, V] logits are never written to memory.
 *
 *   h        [M, D] dtype, device, 16-byte aligned
 *   w        [V, D] dtype, device, 16-byte aligned (each vocab row contiguous)
 *   bias_tok [M] int32, device, optional (NULL: no bias); entries in [0, V)
 *   bias_val [M] f32, device; required iff bias_tok is given
 *   conf     [M] f32, device (written); tok [M] int32, device (written)
 *   ws       device scratch >= fdl_lmhead_workspace_bytes(desc)
 * Errors: FDL_EINVAL, FDL_EUNSUPPORTED, FDL_EWORKSPACE, FDL_ECUDA. */
FDL_API int fdl_lmhead_confidence(fdl_ctx* ctx, const fdl_lmhead_desc* desc,
                          const void* h, const void* w,
                          const int32_t* bias_tok, const float* bias_val,
                          float* conf, int32_t* tok, void* ws, size_t ws_bytes,
                          void* stream);

/* The same computation as fdl_lmhead_confidence, for callers that cannot
 * provide a workspace: C hosts that own only their inputs and outputs, and
 * engines whose device memory belongs entirely to their own pool, where one
 * more cudaMalloc would fail or would bring the device-wide synchronisation
 * cudaMalloc/cudaFree can cause. (The Fast-dLLM paper has no counterpart to
 * this entry point; it is a deployment convenience of this library.)
 *
 * Its scratch is an 8 MiB array inside the library's device module, so every
 * GPU that loads the library holds those 8 MiB until the process exits; the
 * call itself allocates and frees nothing. Shapes whose scratch would exceed
 * 8 MiB (rows x ceil(vocab / 128) x 12 bytes, e.g. more than 707 rows at a
 * vocabulary of 126464) are rejected with FDL_EINVAL before anything runs.
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture. fdl_create drops the cached address of its device, so after a
 * cudaDeviceReset (which invalidates every context and the address) the
 * first call on a new context looks it up again. All calls share the one array and it keeps the last call's
 * contents; each call writes every entry it later reads. Calls whose
 * executions overlap on the GPU (different streams, or different contexts
 * on one device) race on the array and must be ordered by the caller.
 * Arguments, layouts and other errors as fdl_lmhead_confidence. */
FDL_API int fdl_lmhead_confidence_noalloc(fdl_ctx* ctx, const fdl_lmhead_desc* desc,
                                          const void* h, const void* w,
                                          const int32_t* bias_tok, const float* bias_val,
                                          float* conf, int32_t* tok, void* stream);

/* ------------------------------------------------------------------------
 * (b) threshold select + scatter
 * ------------------------------------------------------------------------ */
typedef struct {
    int batch;        /* b >= 1 */
    int seq_len;      /* L */
    int block_start;  /* s */
    int block_len;    /* B, 1 <= B <= 1024, s + B <= L */
    float tau;        /* threshold, finite */
} fdl_unmask_desc;

/* One confidence-aware parallel unmask step (Fast-dLLM abstract; README "Key
 * techniques" 2; aibase news "Innovations" 2).
 *
 * For each sequence, the candidates are the positions p in [s, s+B) with
 * masked[b,p] != 0. Selected = candidates with conf > tau (strict; NaN never
 * selected). If none is selected but a candidate exists, the single candidate
 * with the largest confidence is selected, the lowest position on ties.
 * For every selected p: x[b,p] = tok[b, p-s], masked[b,p] = 0. Positions
 * outside the block and already-decoded positions are never written.
 *
 *   conf      [b, B] f32, device: slot i describes position s+i (slots of
 *             decoded positions are ignored)
 *   tok       [b, B] int32, device
 *   x         [b, L] int32, device, updated in place
 *   masked    [b, L] uint8, device, updated in place (0 = decoded)
 *   remaining [b] int32, device (written): masked positions left in the block
 *   n_decoded [b] int32, device, optional (NULL = not written)
 * A block whose candidates all have NaN confidence decodes nothing and sets
 * FDL_EDEVICE in the device error word.
 * Errors: FDL_EINVAL (shape, null, non-finite tau), FDL_ECUDA. */
FDL_API int fdl_threshold_unmask(fdl_ctx* ctx, const fdl_unmask_desc* desc,
                         const float* conf, const int32_t* tok, int32_t* x,
                         uint8_t* masked, int32_t* remaining,
                         int32_t* n_decoded, void* stream);

/* ------------------------------------------------------------------------
 * Transformer scaffold of the LLaDA / Dream family (pre-norm, bidirectional):
 * the projections that produce the block's K/V (a cached step) or every
 * position's K/V (a refresh), RMSNorm, SwiGLU FFN, residual stream. All GEMMs
 * are bf16 on tcgen05 with f32 accumulation; the residual stream is f32.
 * ------------------------------------------------------------------------ */

/* Rotary table for rotate-half RoPE: out_host[p][i] = (cos, sin) of
 * p * theta^(-2i/head_dim), p in [0, max_pos), i in [0, head_dim/2), computed
 * in double and rounded to float. out_host holds max_pos*head_dim floats.
 * Host-only; errors: FDL_EINVAL. */
FDL_API int fdl_rope_table(double theta, int max_pos, int head_dim, float* out_host);

/* out[i, :] = bf16( h[src, :] / sqrt(mean(h[src, :]^2) + eps) * weight ),
 * src = row_map ? row_map[i] : i.
 *   h [*, hidden] f32 device; row_map [rows] int32 device or NULL;
 *   weight [hidden] f32 device; out [rows, hidden] bf16 device.
 * hidden % 8 == 0. Errors: FDL_EINVAL, FDL_ECUDA. */
FDL_API int fdl_rmsnorm(fdl_ctx* ctx, int rows, int hidden, const float* h,
                        const int32_t* row_map, const float* weight, float eps, void* out,
                        void* stream);

/* h[i, :] = f32(table[ids[j], :]), j = row_map ? row_map[i] : i (row_map
 * lets a cached step embed the block's tokens straight out of x [b, L]).
 * ids int32, row_map [rows] int32 or NULL, table [V, hidden] bf16,
 * h [rows, hidden] f32 (all device). Errors: FDL_EINVAL, FDL_ECUDA. */
FDL_API int fdl_embed(fdl_ctx* ctx, int rows, int hidden, const int32_t* ids,
                      const int32_t* row_map, const void* table, float* h, void* stream);

typedef struct {
    int rows;          /* M token rows of x */
    int hidden;        /* K, multiple of 64 */
    int n_q_heads;     /* q heads; N = (n_q_heads + 2 n_kv_heads) * head_dim */
    int n_kv_heads;
    int head_dim;      /* 128 */
    int batch;         /* sequences in the caches */
    int seq_len;       /* L, cache rows per (sequence, kv head) */
    int rows_per_seq;  /* row r is sequence r / rows_per_seq ... */
    int pos0;          /* ... at position pos0 + r % rows_per_seq */
    int max_pos;       /* rows of the rope table, > every position used */
} fdl_qkv_desc;

/* Block-slot (or, at a refresh, full) projection with rotary embedding and
 * in-place cache write (Fast-dLLM DualCache: at a cached step only the
 * current block is recomputed; aibase news "Innovations" 1; a refresh
 * recomputes every position, ICLR reviews, review 4 question 2).
 *   [q | k | v] = x w^T (+ bias); q, k rotated (rotate-half RoPE) at their
 *   absolute positions; q -> q_out [rows, n_q_heads, head_dim];
 *   k, v -> k_cache / v_cache [batch, n_kv_heads, seq_len, head_dim] at rows
 *   (sequence, position); other cache rows untouched.
 *   x [rows, hidden] bf16; w [N, hidden] bf16 (q heads, then k, then v);
 *   bias [N] f32 or NULL; rope = fdl_rope_table output on the device.
 * Errors: FDL_EINVAL (shapes, positions beyond seq_len or max_pos,
 * alignment), FDL_EUNSUPPORTED (head_dim != 128), FDL_ECUDA. */
FDL_API int fdl_qkv_rope_store(fdl_ctx* ctx, const fdl_qkv_desc* desc, const void* x,
                               const void* w, const float* bias, const float* rope,
                               void* q_out, void* k_cache, void* v_cache, void* stream);

/* The attention half of a cached DualCache step for the block rows:
 *   x = RMSNorm(h) * norm_w          (when norm_w != NULL; x is then written)
 *   q, k, v = x w^T (+ bias), RoPE, k/v into the cache block slot
 *   out = DualCache attention of the block over the whole cache
 * The result equals fdl_rmsnorm (if norm_w), fdl_qkv_rope_store(desc, ...) and
 * fdl_dualcache_attention with block_start = desc->pos0, block_len =
 * desc->rows_per_seq, scale 1/sqrt(128), no LSE. Requires rows == batch *
 * rows_per_seq (the block rows of every sequence), rows_per_seq <= 128.
 *   h       [rows, hidden] f32 (read; only with norm_w); norm_w [hidden] f32;
 *           eps > 0 the RMSNorm epsilon
 *   x       [rows, hidden] bf16: written when norm_w is given, else the input
 *   out     [batch, rows_per_seq, n_q_heads, 128] bf16 (written)
 *   q_out, k_cache, v_cache, w, bias, rope as for fdl_qkv_rope_store.
 * When the shapes allow (few rows, split-K projection, a whole GQA group of
 * query heads per attention CTA) the RMSNorm runs in the projection's kernel
 * (behind a grid-wide barrier) and the projection's epilogue (bias, RoPE, q
 * and block-slot store) in the attention kernel's CTAs, each forming its own
 * query tile and block-slot rows, instead of in kernels of their own.
 * Errors: as fdl_qkv_rope_store, plus FDL_EINVAL for the row layout or the
 * norm arguments. */
FDL_API int fdl_qkv_attention(fdl_ctx* ctx, const fdl_qkv_desc* desc, const float* h,
                              const float* norm_w, float eps, void* x, const void* w,
                              const float* bias, const float* rope, void* q_out, void* k_cache,
                              void* v_cache, void* out, void* stream);

/* h[rows, out_features] += x w^T  (f32 residual stream; x bf16 [rows, in],
 * w bf16 [out, in]). in % 64 == 0, out % 64 == 0. Errors: FDL_EINVAL, FDL_ECUDA. */
FDL_API int fdl_linear_residual(fdl_ctx* ctx, int rows, int out_features, int in_features,
                                const void* x, const void* w, float* h, void* stream);

/* out[rows, out_features] = silu(x Wg^T) * (x Wu^T), bf16, with the gate and
 * up weights interleaved by rows: w_gu [2*out_features, in], row 2f = gate
 * row f, row 2f+1 = up row f. in % 64 == 0, out_features % 32 == 0.
 * Errors: FDL_EINVAL, FDL_ECUDA. */
FDL_API int fdl_linear_swiglu(fdl_ctx* ctx, int rows, int out_features, int in_features,
                              const void* x, const void* w_gu, void* out, void* stream);

/* Feed-forward half of a layer with its residual (pre-norm SwiGLU MLP):
 *   x  = RMSNorm(h) * norm_w           (when norm_w != NULL; x is then written)
 *   f  = silu(x Wg^T) * (x Wu^T)      bf16 [rows, ffn], written
 *   h += f Wd^T                        f32 [rows, hidden], updated
 * x bf16 [rows, hidden] (the input when norm_w is NULL); norm_w [hidden] f32,
 * eps > 0; w_gu bf16 [2*ffn, hidden] interleaved as for fdl_linear_swiglu;
 * w_down bf16 [hidden, ffn]. hidden % 64 == 0, ffn % 64 == 0. The result
 * equals fdl_rmsnorm (if norm_w), fdl_linear_swiglu and fdl_linear_residual.
 * For the few rows of a cached block step (rows <= 256, hidden and ffn
 * multiples of 128) the RMSNorm runs in the gate/up projection's kernel and
 * the SwiGLU of the split-K gate/up sums in the down projection's kernel,
 * each behind a grid-wide barrier, instead of in kernels of their own.
 * Errors: FDL_EINVAL, FDL_ECUDA. */
FDL_API int fdl_ffn(fdl_ctx* ctx, int rows, int hidden, int ffn, const float* norm_w, float eps,
                    void* x, const void* w_gu, const void* w_down, void* f, float* h,
                    void* stream);

/* Full bidirectional attention of the positions [s, L), s = desc->block_start,
 * over all L positions of the caches: out[b, i, h, :] = sum_j softmax_j(scale *
 * q_i . k_j) v_j over every j in [0, L). s = 0 is the refresh forward after a
 * block completes (ICLR reviews, review 4 question 2: all K/V are recomputed);
 * s = the block start is the attention of a PrefixCache step, where the block
 * and the masked suffix are recomputed over the cached prefix (README usage
 * flag --use_cache without --if_cache_position).
 *   q, out [b, L - s, Hq, d] bf16; caches [b, Hkv, L, d] bf16 (desc->dtype
 *   must be FDL_BF16; block_len is ignored). L - s a positive multiple of 32.
 * Errors: FDL_EINVAL, FDL_EUNSUPPORTED, FDL_ECUDA. */
FDL_API int fdl_full_attention(fdl_ctx* ctx, const fdl_attn_desc* desc, const void* q,
                               const void* k_cache, const void* v_cache, void* out,
                               void* stream);

/* ---- the whole decode: DualCache block decoding with the threshold rule ----
 * Fast-dLLM (README "Key techniques" 1 and 2; aibase news "Innovations" 1
 * and 2): the generated part is split into blocks of `block` positions,
 * decoded left to right. A block starts with a full bidirectional forward
 * over all positions (it rewrites every layer's K/V cache, and its logits
 * serve the block's first step); then cached steps recompute only the
 * block's rows, attending over [prefix | block | suffix] of the cache, until
 * no position of the block is masked. Each step unmasks the masked positions
 * of the block whose confidence exceeds tau, or the single most confident
 * one (lowest position on ties), as fdl_threshold_unmask. The model is a
 * pre-norm bidirectional transformer: x = RMSNorm(h); q/k/v (+ bias), RoPE;
 * attention; h += o W_o^T; x = RMSNorm(h); h += (silu(x W_g^T) * (x W_u^T))
 * W_d^T; final RMSNorm; LM head. */
typedef struct {
    int vocab;        /* V >= 2 */
    int hidden;       /* D, multiple of 128 */
    int n_layers;     /* >= 1 */
    int n_q_heads;    /* Hq, multiple of n_kv_heads */
    int n_kv_heads;   /* Hkv >= 1 */
    int head_dim;     /* 128 */
    int ffn;          /* F, multiple of 64 */
    int mask_id;      /* token id of a masked position, in [0, V) */
    float rope_theta; /* > 0 */
    float rms_eps;    /* > 0 */
} fdl_model_desc;

/* Device pointers of one layer, owned by the caller; every matrix K-major. */
typedef struct {
    const float* attn_norm;  /* f32 [D] */
    const void* w_qkv;       /* bf16 [(Hq + 2 Hkv) * 128, D]: q rows, then k, then v */
    const float* bias;       /* f32 [(Hq + 2 Hkv) * 128] or NULL */
    const void* wo;          /* bf16 [D, Hq * 128] */
    const float* ffn_norm;   /* f32 [D] */
    const void* w_gu;        /* bf16 [2F, D], gate and up rows interleaved (2f, 2f + 1) */
    const void* w_down;      /* bf16 [D, F] */
} fdl_layer_weights;

typedef struct {
    const void* embed;                /* bf16 [V, D] */
    const float* final_norm;          /* f32 [D] */
    const void* lm_head;              /* bf16 [V, D] */
    const fdl_layer_weights* layers;  /* host array of n_layers (copied by create) */
} fdl_model_weights;

typedef struct fdl_model fdl_model;   /* the description and the weight pointers */

/* Record a model: copies the description and the pointers (host memory
 * only; the weights stay the caller's and must outlive the model). Checks
 * shapes, alignment (16 bytes) and non-NULL pointers. *out is NULL on failure.
 * Errors: FDL_EINVAL. */
FDL_API int fdl_model_create(const fdl_model_desc* desc, const fdl_model_weights* weights,
                             fdl_model** out);
FDL_API int fdl_model_destroy(fdl_model* model);

/* Device workspace of fdl_generate for `batch` sequences of length seq_len
 * in blocks of `block` positions: every layer's K/V cache (2 * layers * batch
 * * Hkv * seq_len * 128 bf16), the activations of a full forward and of a
 * block step, the LM-head scratch, the mask state and the rotary table. 0 on
 * bad arguments. */
FDL_API size_t fdl_generate_workspace_bytes(fdl_ctx* ctx, const fdl_model* model, int batch,
                                            int seq_len, int block);

/* Which K/V a decode step after a block's first reuses (Fast-dLLM README,
 * usage flags and the evaluation table's "+cache" columns; aibase news
 * "Innovations" 1). A block's first step is always the full forward that
 * rewrites every layer's cache. */
typedef enum {
    FDL_CACHE_DUAL = 0,    /* DualCache (--use_cache --if_cache_position): only the block's
                              rows are recomputed; prefix and masked suffix come from the cache */
    FDL_CACHE_PREFIX = 1,  /* PrefixCache (--use_cache): the block and the suffix, rows [s, L),
                              are recomputed over the cached prefix */
    FDL_CACHE_NONE = 2     /* no cache: every step is a full forward over all positions */
} fdl_cache_mode;

/* How the sequences of a batch move through their blocks. Every sequence
 * decodes the same tokens in all three; they differ in what a step computes. */
typedef enum {
    FDL_BATCH_LOCKSTEP = 0,   /* every step runs on the whole batch; the batch moves to
                                 the next block (one refresh for all) when every
                                 sequence's block is decoded */
    FDL_BATCH_COMPACT = 1,    /* as lockstep, but a cached step runs only on the sequences
                                 that still have masked positions in the block, compacted
                                 into a smaller batch */
    FDL_BATCH_PER_SEQUENCE = 2 /* every sequence moves to its next block as soon as its own
                                 block is decoded: a step refreshes the sequences that have
                                 just moved on and takes a DualCache step of the others,
                                 each at its own block; steps_out counts these steps */
} fdl_batching;
/* FDL_BATCH_COMPACT and FDL_BATCH_PER_SEQUENCE need FDL_CACHE_DUAL and the host
 * loop (device_loop = 0); otherwise fdl_generate returns FDL_EINVAL. */

typedef struct {
    int cache;                /* fdl_cache_mode */
    /* 0: the host runs the loop, reading the block's masked counts back after
     * every step. 1: the whole decode is one CUDA graph: per block the refresh
     * step, then a conditional WHILE node whose body is one cached step,
     * repeated on the device while a sequence has a masked position left in
     * the block (the condition is set by a small kernel after each step); the
     * host synchronises once per decode. The executable graph is kept in the
     * context and launched again by the next call with the same model,
     * workspace, shapes, tau, cache mode and bias pointers; the first call
     * captures and instantiates it. */
    int device_loop;
    /* Optional planted logit bias per generated position (a synthetic workload
     * device: with random weights no confidence reaches a threshold, and a bias
     * on one token per position makes the parallel rule fire): at the LM head of
     * every step, the logit of token bias_tok[i, p - prompt_len] of position p
     * of sequence i gets + bias_val[i, p - prompt_len]. */
    const int32_t* bias_tok;  /* [batch, gen_len] int32 device, entries in [0, V), or NULL */
    const float* bias_val;    /* [batch, gen_len] f32 device; required iff bias_tok */
    int batching;             /* fdl_batching */
} fdl_generate_opts;

/* Decode gen_len positions after the prompts of `batch` sequences.
 *   prompt  [batch, prompt_len] int32 device (token ids)
 *   out_x   [batch, prompt_len + gen_len] int32 device (written: the prompts,
 *           then the decoded tokens)
 *   block   positions per block, 1..128; prompt_len and gen_len multiples of it,
 *           prompt_len + gen_len a multiple of 32 (FDL_CACHE_PREFIX: prompt_len
 *           and block too, so that every block starts at a multiple of 32)
 *   tau     threshold in [0, 1] (tau = 1 decodes exactly one position per step)
 *   opts    cache mode, loop, optional planted bias, batching; NULL =
 *           FDL_CACHE_DUAL, host loop, no bias, FDL_BATCH_LOCKSTEP
 *   *steps_out (host) the decode steps taken (refresh steps included)
 *   ws      device workspace of fdl_generate_workspace_bytes bytes, 256-byte
 *           aligned
 * With the host loop every step reads `batch` 4-byte counters back to decide
 * between the next cached step and the next block; with opts->device_loop the
 * steps are sequenced on the device. The call returns when the decode is
 * complete (the stream is synchronised). prompt and out_x are only read at
 * the start and written at the end (the decode state lives in ws). The kernels and their
 * order are those of the per-call functions above (fdl_embed, fdl_rmsnorm,
 * fdl_qkv_rope_store, fdl_full_attention, fdl_qkv_attention,
 * fdl_linear_residual, fdl_ffn, fdl_lmhead_confidence, fdl_threshold_unmask).
 * Errors: FDL_EINVAL, FDL_EWORKSPACE, FDL_ECUDA, or those of the calls. */
FDL_API int fdl_generate(fdl_ctx* ctx, const fdl_model* model, const int32_t* prompt, int batch,
                         int prompt_len, int gen_len, int block, float tau,
                         const fdl_generate_opts* opts, int32_t* out_x, int* steps_out, void* ws,
                         size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FDLLM_H */
