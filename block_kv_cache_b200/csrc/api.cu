// C-ABI entry points of the Fast-dLLM step library: argument validation,
// device selection, workspace checks and dispatch to the kernels. See
// include/fdllm.h for the contract of every function.
#include "fdllm.h"
#include "launch.h"
#include "common.cuh"

#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <vector>

// The executable graph of the last device-loop decode of a context, kept for
// the next decode with the same key (fdl_generate with device_loop).
struct GenGraph {
    cudaGraphExec_t exec = nullptr;
    cudaStream_t cap = nullptr, body = nullptr;   // capture streams (non-blocking)
    // key: everything the captured kernels' arguments depend on
    uint64_t model = 0;                           // fdl_model id
    const void* ws = nullptr;
    size_t ws_bytes = 0;
    int b = 0, P = 0, gen = 0, B = 0, mode = 0;
    float tau = 0.f;
    const void* bias_tok = nullptr;
    const void* bias_val = nullptr;
};

struct fdl_ctx {
    int device;
    int sm_count;
    int* d_err;              // device error word (4 bytes), then at +8 the u64 wait limit
    float* d_acc;            // split-K accumulator of the projections, kept all zeros
    size_t acc_bytes;
    unsigned* d_sync;        // grid-barrier words of the fused kernels (zeroed)
    GenGraph* gen;           // cached device-loop decode graph, or NULL
};

// Split-K accumulator of the few-token projections (zeroed at creation; every
// kernel that adds into it leaves it zeroed again): room for 256 rows x 32768.
static const size_t kAccBytes = (size_t)256 * 32768 * 4;
static const size_t kSyncBytes = 256;
// Default limit of the kernels' progress waits (the device-side default too).
static const uint64_t kDefaultWaitNs = 2000000000ull;
static const uint64_t kMaxWaitNs = 60000000000ull;

namespace fdl {
void noalloc_forget(int dev);
}

namespace {

thread_local char g_msg[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char* where) {
    return fail(FDL_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

// Make ctx->device current for the duration of a call; restore afterwards.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int check_attn(const fdl_attn_desc* d) {
    if (!d) return fail(FDL_EINVAL, "attention: desc is NULL");
    if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->seq_len < 1)
        return fail(FDL_EINVAL, "attention: batch, heads and seq_len must be >= 1");
    if (d->n_q_heads % d->n_kv_heads)
        return fail(FDL_EINVAL, "attention: n_q_heads (%d) must be a multiple of n_kv_heads (%d)",
                    d->n_q_heads, d->n_kv_heads);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(FDL_EUNSUPPORTED, "attention: head_dim %d not supported (64 or 128)",
                    d->head_dim);
    if (d->block_len < 1 || d->block_len > 128)
        return fail(FDL_EINVAL, "attention: block_len %d outside [1, 128]", d->block_len);
    if (d->block_start < 0 || d->block_start + d->block_len > d->seq_len)
        return fail(FDL_EINVAL, "attention: block [%d, %d) outside [0, %d)", d->block_start,
                    d->block_start + d->block_len, d->seq_len);
    if (d->dtype != FDL_F32 && d->dtype != FDL_BF16)
        return fail(FDL_EINVAL, "attention: unknown dtype %d", d->dtype);
    if (!(d->scale >= 0.f) || isinf(d->scale))
        return fail(FDL_EINVAL, "attention: scale must be finite and >= 0");
    return FDL_OK;
}

fdl::AttnShape attn_shape(const fdl_attn_desc* d) {
    fdl::AttnShape s{d->batch, d->n_q_heads, d->n_kv_heads, d->head_dim, d->seq_len,
                     d->block_start, d->block_len, d->scale, d->dtype == FDL_BF16 ? 1 : 0};
    if (s.scale == 0.f) s.scale = 1.0f / sqrtf((float)d->head_dim);
    return s;
}

int check_lm(const fdl_lmhead_desc* d) {
    if (!d) return fail(FDL_EINVAL, "lmhead: desc is NULL");
    if (d->rows < 1 || d->vocab < 2 || d->hidden < 64)
        return fail(FDL_EINVAL, "lmhead: need rows >= 1, vocab >= 2, hidden >= 64");
    if (d->hidden % 64)
        return fail(FDL_EUNSUPPORTED, "lmhead: hidden %d must be a multiple of 64", d->hidden);
    if (d->dtype != FDL_F32 && d->dtype != FDL_BF16)
        return fail(FDL_EINVAL, "lmhead: unknown dtype %d", d->dtype);
    return FDL_OK;
}

}  // namespace

void release_gen_graph(fdl_ctx* ctx);

extern "C" {

int fdl_abi_version(void) { return FDL_ABI_VERSION; }

const char* fdl_last_error(void) { return g_msg; }

int fdl_create(fdl_ctx** out, int device) {
    if (!out) return fail(FDL_EINVAL, "fdl_create: out is NULL");
    *out = nullptr;
    int n = 0;
    cudaError_t e = cudaGetDeviceCount(&n);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceCount");
    if (device < 0 || device >= n)
        return fail(FDL_EINVAL, "fdl_create: device %d not in [0, %d)", device, n);
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, device);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major != 10 || prop.minor != 0)
        return fail(FDL_EUNSUPPORTED, "fdl_create: device %d is sm_%d%d; this library is built "
                    "for sm_100a (B200)", device, prop.major, prop.minor);
    DeviceGuard g(device);
    if (!g.ok) return fail(FDL_ECUDA, "fdl_create: cannot select device %d", device);
    fdl_ctx* c = new fdl_ctx;
    c->device = device;
    c->sm_count = prop.multiProcessorCount;
    c->d_err = nullptr;
    c->d_acc = nullptr;
    c->d_sync = nullptr;
    c->gen = nullptr;
    c->acc_bytes = kAccBytes;
    // 16 bytes: the error word, then (8-byte aligned) the limit of the
    // kernels' progress waits in ns
    const uint64_t limit = kDefaultWaitNs;
    e = cudaMalloc(&c->d_err, 16);
    if (e == cudaSuccess) e = cudaMemset(c->d_err, 0, 16);
    if (e == cudaSuccess)
        e = cudaMemcpy(reinterpret_cast<char*>(c->d_err) + 8, &limit, 8, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMalloc(&c->d_acc, kAccBytes);
    if (e == cudaSuccess) e = cudaMemset(c->d_acc, 0, kAccBytes);
    if (e == cudaSuccess) e = cudaMalloc(&c->d_sync, kSyncBytes);
    if (e == cudaSuccess) e = cudaMemset(c->d_sync, 0, kSyncBytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e == cudaSuccess) fdl::attn_tc_warm();   // host-side queries, no launch
    if (e != cudaSuccess) {
        if (c->d_err) cudaFree(c->d_err);
        if (c->d_acc) cudaFree(c->d_acc);
        if (c->d_sync) cudaFree(c->d_sync);
        delete c;
        return cuda_fail(e, "fdl_create: device buffers");
    }
    fdl::noalloc_forget(device);
    *out = c;
    return FDL_OK;
}

int fdl_destroy(fdl_ctx* ctx) {
    if (!ctx) return FDL_OK;
    DeviceGuard g(ctx->device);
    release_gen_graph(ctx);
    if (ctx->d_err) cudaFree(ctx->d_err);
    if (ctx->d_acc) cudaFree(ctx->d_acc);
    if (ctx->d_sync) cudaFree(ctx->d_sync);
    delete ctx;
    return FDL_OK;
}

int fdl_set_wait_timeout(fdl_ctx* ctx, uint64_t ns) {
    if (!ctx) return fail(FDL_EINVAL, "set_wait_timeout: ctx is NULL");
    if (ns < 1 || ns > kMaxWaitNs)
        return fail(FDL_EINVAL, "set_wait_timeout: %llu ns outside [1, %llu]",
                    (unsigned long long)ns, (unsigned long long)kMaxWaitNs);
    DeviceGuard g(ctx->device);
    if (!g.ok) return fail(FDL_ECUDA, "set_wait_timeout: cannot select device");
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(reinterpret_cast<char*>(ctx->d_err) + 8, &ns, 8, cudaMemcpyHostToDevice);
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "set_wait_timeout");
}

int fdl_get_device_status(fdl_ctx* ctx, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "fdl_get_device_status: ctx is NULL");
    DeviceGuard g(ctx->device);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "fdl_get_device_status: sync");
    int code = 0;
    e = cudaMemcpy(&code, ctx->d_err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "fdl_get_device_status: read");
    if (code != 0) {
        e = cudaMemset(ctx->d_err, 0, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "fdl_get_device_status: clear");
    }
    if (code == fdl::DEV_TIMEOUT) return fail(FDL_ETIMEOUT, "device: a bounded wait ran out");
    if (code == fdl::DEV_NO_PROGRESS)
        return fail(FDL_EDEVICE, "device: every candidate of a block had a NaN confidence");
    if (code != 0) return fail(FDL_EDEVICE, "device: error code %d", code);
    return FDL_OK;
}

size_t fdl_attention_workspace_bytes(const fdl_ctx* ctx, const fdl_attn_desc* desc) {
    if (!ctx) { fail(FDL_EINVAL, "attention workspace: ctx is NULL"); return 0; }
    if (check_attn(desc) != FDL_OK) return 0;
    return fdl::attn_workspace_bytes(attn_shape(desc), ctx->sm_count);
}

int fdl_dualcache_attention(fdl_ctx* ctx, const fdl_attn_desc* desc, const void* q,
                            const void* k_cache, const void* v_cache, void* out, float* lse,
                            void* ws, size_t ws_bytes, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "attention: ctx is NULL");
    int rc = check_attn(desc);
    if (rc) return rc;
    if (!q || !k_cache || !v_cache || !out)
        return fail(FDL_EINVAL, "attention: q, k_cache, v_cache and out must be non-NULL");
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (lse && ((uintptr_t)lse & 3u)))
        return fail(FDL_EINVAL, "attention: q/k_cache/v_cache/out must be 16-byte aligned");
    fdl::AttnShape s = attn_shape(desc);
    const size_t need = fdl::attn_workspace_bytes(s, ctx->sm_count);
    if (!ws || ws_bytes < need || !aligned16(ws))
        return fail(FDL_EWORKSPACE, "attention: workspace needs %zu bytes (16-byte aligned), "
                    "got %zu", need, ws ? ws_bytes : (size_t)0);
    DeviceGuard g(ctx->device);
    if (!g.ok) return fail(FDL_ECUDA, "attention: cannot select device");
    cudaError_t e = desc->dtype == FDL_F32
        ? fdl::launch_attention_f32(s, (const float*)q, (const float*)k_cache,
                                    (const float*)v_cache, (float*)out, lse, ws, ctx->sm_count,
                                    (cudaStream_t)stream)
        : fdl::launch_attention_bf16(s, q, k_cache, v_cache, out, lse, ws, ctx->sm_count,
                                     ctx->d_err, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    return FDL_OK;
}

int fdl_kv_store(fdl_ctx* ctx, const fdl_attn_desc* desc, const void* k_new, const void* v_new,
                 int start, int n, void* k_cache, void* v_cache, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "kv_store: ctx is NULL");
    if (!desc) return fail(FDL_EINVAL, "kv_store: desc is NULL");
    if (desc->batch < 1 || desc->n_kv_heads < 1 || desc->seq_len < 1)
        return fail(FDL_EINVAL, "kv_store: batch, n_kv_heads and seq_len must be >= 1");
    if (desc->head_dim != 64 && desc->head_dim != 128)
        return fail(FDL_EUNSUPPORTED, "kv_store: head_dim %d not supported", desc->head_dim);
    if (desc->dtype != FDL_F32 && desc->dtype != FDL_BF16)
        return fail(FDL_EINVAL, "kv_store: unknown dtype %d", desc->dtype);
    if (n < 1 || start < 0 || start + n > desc->seq_len)
        return fail(FDL_EINVAL, "kv_store: rows [%d, %d) outside [0, %d)", start, start + n,
                    desc->seq_len);
    if (!k_new || !v_new || !k_cache || !v_cache)
        return fail(FDL_EINVAL, "kv_store: NULL buffer");
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(FDL_EINVAL, "kv_store: buffers must be 16-byte aligned");
    DeviceGuard g(ctx->device);
    if (!g.ok) return fail(FDL_ECUDA, "kv_store: cannot select device");
    const int eb = desc->dtype == FDL_F32 ? 4 : 2;
    cudaError_t e = fdl::launch_kv_store(desc->batch, desc->n_kv_heads, desc->head_dim,
                                         desc->seq_len, eb, k_new, v_new, start, n, k_cache,
                                         v_cache, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kv_store launch");
    return FDL_OK;
}

size_t fdl_lmhead_workspace_bytes(const fdl_ctx* ctx, const fdl_lmhead_desc* desc) {
    if (!ctx) { fail(FDL_EINVAL, "lmhead workspace: ctx is NULL"); return 0; }
    if (check_lm(desc) != FDL_OK) return 0;
    fdl::LMShape s{desc->rows, desc->hidden, desc->vocab};
    return fdl::lmhead_workspace_bytes(s);
}

int fdl_lmhead_confidence(fdl_ctx* ctx, const fdl_lmhead_desc* desc, const void* h,
                          const void* w, const int32_t* bias_tok, const float* bias_val,
                          float* conf, int32_t* tok, void* ws, size_t ws_bytes, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "lmhead: ctx is NULL");
    int rc = check_lm(desc);
    if (rc) return rc;
    if (!h || !w || !conf || !tok) return fail(FDL_EINVAL, "lmhead: NULL buffer");
    if ((bias_tok == nullptr) != (bias_val == nullptr))
        return fail(FDL_EINVAL, "lmhead: bias_tok and bias_val go together");
    if (!aligned16(h) || !aligned16(w))
        return fail(FDL_EINVAL, "lmhead: h and w must be 16-byte aligned");
    fdl::LMShape s{desc->rows, desc->hidden, desc->vocab};
    const size_t need = fdl::lmhead_workspace_bytes(s);
    if (!ws || ws_bytes < need || !aligned16(ws))
        return fail(FDL_EWORKSPACE, "lmhead: workspace needs %zu bytes (16-byte aligned), got %zu",
                    need, ws ? ws_bytes : (size_t)0);
    DeviceGuard g(ctx->device);
    if (!g.ok) return fail(FDL_ECUDA, "lmhead: cannot select device");
    cudaError_t e = desc->dtype == FDL_F32
        ? fdl::launch_lmhead_f32(s, (const float*)h, (const float*)w, bias_tok, bias_val, conf,
                                 tok, ws, (cudaStream_t)stream)
        : fdl::launch_lmhead_bf16(s, h, w, bias_tok, bias_val, conf, tok, ws, ctx->sm_count,
                                  ctx->d_err, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "lmhead launch");
    return FDL_OK;
}

int fdl_threshold_unmask(fdl_ctx* ctx, const fdl_unmask_desc* desc, const float* conf,
                         const int32_t* tok, int32_t* x, uint8_t* masked, int32_t* remaining,
                         int32_t* n_decoded, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "unmask: ctx is NULL");
    if (!desc) return fail(FDL_EINVAL, "unmask: desc is NULL");
    if (desc->batch < 1 || desc->seq_len < 1)
        return fail(FDL_EINVAL, "unmask: batch and seq_len must be >= 1");
    if (desc->block_len < 1 || desc->block_len > 1024)
        return fail(FDL_EINVAL, "unmask: block_len %d outside [1, 1024]", desc->block_len);
    if (desc->block_start < 0 || desc->block_start + desc->block_len > desc->seq_len)
        return fail(FDL_EINVAL, "unmask: block [%d, %d) outside [0, %d)", desc->block_start,
                    desc->block_start + desc->block_len, desc->seq_len);
    if (!isfinite(desc->tau)) return fail(FDL_EINVAL, "unmask: tau must be finite");
    if (!conf || !tok || !x || !masked || !remaining)
        return fail(FDL_EINVAL, "unmask: NULL buffer");
    DeviceGuard g(ctx->device);
    if (!g.ok) return fail(FDL_ECUDA, "unmask: cannot select device");
    cudaError_t e = fdl::launch_threshold_unmask(desc->batch, desc->seq_len, desc->block_start,
                                                 desc->block_len, desc->tau, conf, tok, x,
                                                 masked, remaining, n_decoded, ctx->d_err,
                                                 (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "unmask launch");
    return FDL_OK;
}

}  // extern "C"

void release_gen_graph(fdl_ctx* ctx) {
    if (!ctx->gen) return;
    if (ctx->gen->exec) cudaGraphExecDestroy(ctx->gen->exec);
    if (ctx->gen->cap) cudaStreamDestroy(ctx->gen->cap);
    if (ctx->gen->body) cudaStreamDestroy(ctx->gen->body);
    delete ctx->gen;
    ctx->gen = nullptr;
}

namespace fdl {
// Device id of a context (for library-internal entry points in other files).
int ctx_device(const fdl_ctx* ctx) { return ctx ? ctx->device : -1; }
}  // namespace fdl

namespace fdl {
// Record `msg` as the calling thread's last error and return `code`.
int report_error(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace fdl

// ----------------------------------------------------------------------------
// transformer scaffold
// ----------------------------------------------------------------------------
#include <cmath>

#include "gemm.h"

extern "C" {

int fdl_rope_table(double theta, int max_pos, int head_dim, float* out_host) {
    if (!out_host || max_pos < 1 || head_dim < 2 || head_dim % 2 || !(theta > 0.0))
        return fail(FDL_EINVAL, "rope_table: need out, max_pos >= 1, even head_dim, theta > 0");
    const int half = head_dim / 2;
    for (int p = 0; p < max_pos; ++p)
        for (int i = 0; i < half; ++i) {
            const double ang = (double)p * std::pow(theta, -2.0 * i / head_dim);
            out_host[((size_t)p * half + i) * 2 + 0] = (float)std::cos(ang);
            out_host[((size_t)p * half + i) * 2 + 1] = (float)std::sin(ang);
        }
    return FDL_OK;
}

int fdl_rmsnorm(fdl_ctx* ctx, int rows, int hidden, const float* h, const int32_t* row_map,
                const float* weight, float eps, void* out, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "rmsnorm: ctx is NULL");
    if (rows < 1 || hidden < 8 || hidden % 8)
        return fail(FDL_EINVAL, "rmsnorm: rows >= 1 and hidden a multiple of 8 required");
    if (!h || !weight || !out || !(eps >= 0.f))
        return fail(FDL_EINVAL, "rmsnorm: NULL buffer or bad eps");
    if (!aligned16(h) || !aligned16(weight) || !aligned16(out))
        return fail(FDL_EINVAL, "rmsnorm: buffers must be 16-byte aligned");
    DeviceGuard g(ctx->device);
    cudaError_t e = fdl::launch_rmsnorm(rows, hidden, h, row_map, weight, eps, (fdl::bf16*)out,
                                        (cudaStream_t)stream);
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "rmsnorm launch");
}

int fdl_embed(fdl_ctx* ctx, int rows, int hidden, const int32_t* ids, const int32_t* row_map,
              const void* table, float* h, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "embed: ctx is NULL");
    if (rows < 1 || hidden < 2 || hidden % 2)
        return fail(FDL_EINVAL, "embed: rows >= 1 and even hidden required");
    if (!ids || !table || !h) return fail(FDL_EINVAL, "embed: NULL buffer");
    DeviceGuard g(ctx->device);
    cudaError_t e = fdl::launch_embed(rows, hidden, ids, row_map, (const fdl::bf16*)table, h,
                                      (cudaStream_t)stream);
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "embed launch");
}

}  // extern "C"

namespace {
int check_qkv(const fdl_ctx* ctx, const fdl_qkv_desc* d, const void* x, const void* w,
              const float* rope, const void* q_out, const void* k_cache, const void* v_cache) {
    if (!ctx) return fail(FDL_EINVAL, "qkv: ctx is NULL");
    if (!d) return fail(FDL_EINVAL, "qkv: desc is NULL");
    if (d->head_dim != 128) return fail(FDL_EUNSUPPORTED, "qkv: head_dim must be 128");
    if (d->rows < 1 || d->hidden < 64 || d->hidden % 64 || d->n_q_heads < 1 ||
        d->n_kv_heads < 1 || d->batch < 1 || d->seq_len < 1 || d->rows_per_seq < 1 ||
        d->pos0 < 0 || d->max_pos < 1)
        return fail(FDL_EINVAL, "qkv: bad shape");
    if ((d->rows + d->rows_per_seq - 1) / d->rows_per_seq > d->batch)
        return fail(FDL_EINVAL, "qkv: rows span more than batch sequences");
    const int last_pos = d->pos0 + (d->rows < d->rows_per_seq ? d->rows : d->rows_per_seq) - 1;
    if (last_pos >= d->seq_len || last_pos >= d->max_pos)
        return fail(FDL_EINVAL, "qkv: position %d beyond seq_len %d or rope rows %d", last_pos,
                    d->seq_len, d->max_pos);
    if (!x || !w || !rope || !q_out || !k_cache || !v_cache)
        return fail(FDL_EINVAL, "qkv: NULL buffer");
    if (!aligned16(x) || !aligned16(w) || !aligned16(q_out) || !aligned16(k_cache) ||
        !aligned16(v_cache) || !aligned16(rope))
        return fail(FDL_EINVAL, "qkv: buffers must be 16-byte aligned");
    return FDL_OK;
}
}  // namespace

int qkv_attention_mapped(fdl_ctx* ctx, const fdl_qkv_desc* d, const float* h,
                         const float* norm_w, float eps, void* x, const void* w,
                         const float* bias, const float* rope, void* q_out, void* k_cache,
                         void* v_cache, void* out, void* stream, const int32_t* seq_map,
                         int kv_batch, const int32_t* pos0_map);
int qkv_rope_store_mapped(fdl_ctx* ctx, const fdl_qkv_desc* d, const void* x, const void* w,
                          const float* bias, const float* rope, void* q_out, void* k_cache,
                          void* v_cache, void* stream, const int32_t* seq_map, int kv_batch);

extern "C" {

int fdl_qkv_rope_store(fdl_ctx* ctx, const fdl_qkv_desc* d, const void* x, const void* w,
                       const float* bias, const float* rope, void* q_out, void* k_cache,
                       void* v_cache, void* stream) {
    return qkv_rope_store_mapped(ctx, d, x, w, bias, rope, q_out, k_cache, v_cache, stream,
                                 nullptr, 0);
}

}  // extern "C"

// fdl_qkv_rope_store with the rows of sequence i going to the caches of
// sequence seq_map[i] of kv_batch (seq_map null: the identity).
int qkv_rope_store_mapped(fdl_ctx* ctx, const fdl_qkv_desc* d, const void* x, const void* w,
                          const float* bias, const float* rope, void* q_out, void* k_cache,
                          void* v_cache, void* stream, const int32_t* seq_map, int kv_batch) {
    const int rc = check_qkv(ctx, d, x, w, rope, q_out, k_cache, v_cache);
    if (rc) return rc;
    if (seq_map && kv_batch < d->batch)
        return fail(FDL_EINVAL, "qkv: the caches hold %d sequences, fewer than the %d of the "
                    "batch", kv_batch, d->batch);
    DeviceGuard g(ctx->device);
    fdl::GemmShape gs{d->rows, (d->n_q_heads + 2 * d->n_kv_heads) * 128, d->hidden};
    fdl::EpiQKV p{(fdl::bf16*)q_out, (fdl::bf16*)k_cache, (fdl::bf16*)v_cache, bias,
                  (const float2*)rope, d->n_q_heads, d->n_kv_heads, d->seq_len,
                  d->rows_per_seq, d->pos0, seq_map};
    cudaError_t e = fdl::skinny_ok(gs)
        ? fdl::launch_skinny_qkv(gs, x, w, p, ctx->d_acc, ctx->acc_bytes, ctx->sm_count,
                                 ctx->d_err, (cudaStream_t)stream)
        : fdl::launch_gemm_qkv(gs, x, w, p, ctx->sm_count, ctx->d_err, (cudaStream_t)stream);
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "qkv launch");
}

extern "C" {

int fdl_qkv_attention(fdl_ctx* ctx, const fdl_qkv_desc* d, const float* h, const float* norm_w,
                      float eps, void* x, const void* w, const float* bias, const float* rope,
                      void* q_out, void* k_cache, void* v_cache, void* out, void* stream) {
    return qkv_attention_mapped(ctx, d, h, norm_w, eps, x, w, bias, rope, q_out, k_cache,
                                v_cache, out, stream, nullptr, 0, nullptr);
}

}  // extern "C"

// fdl_qkv_attention over a compacted batch: the d->batch sequences of the rows
// are sequences seq_map[0 .. d->batch) of caches that hold kv_batch sequences
// (seq_map null: the identity, kv_batch = d->batch); with pos0_map, sequence i's
// block starts at pos0_map[i] instead of d->pos0 (the caller keeps every block
// inside [0, seq_len)).
int qkv_attention_mapped(fdl_ctx* ctx, const fdl_qkv_desc* d, const float* h,
                         const float* norm_w, float eps, void* x, const void* w,
                         const float* bias, const float* rope, void* q_out, void* k_cache,
                         void* v_cache, void* out, void* stream, const int32_t* seq_map,
                         int kv_batch, const int32_t* pos0_map) {
    int rc = check_qkv(ctx, d, x, w, rope, q_out, k_cache, v_cache);
    if (rc) return rc;
    if (norm_w && (!h || !aligned16(h) || !aligned16(norm_w) || !(eps > 0.f)))
        return fail(FDL_EINVAL, "qkv_attention: with norm_w, h must be a 16-byte aligned f32 "
                    "buffer and eps > 0");
    if (d->rows != d->batch * d->rows_per_seq || d->rows_per_seq > 128)
        return fail(FDL_EINVAL, "qkv_attention: rows must be batch * rows_per_seq, "
                    "rows_per_seq <= 128 (one block per sequence)");
    if (d->n_q_heads % d->n_kv_heads)
        return fail(FDL_EINVAL, "qkv_attention: n_q_heads must be a multiple of n_kv_heads");
    if (!out || !aligned16(out)) return fail(FDL_EINVAL, "qkv_attention: out NULL or unaligned");
    DeviceGuard g(ctx->device);
    cudaStream_t st = (cudaStream_t)stream;
    const fdl::GemmShape gs{d->rows, (d->n_q_heads + 2 * d->n_kv_heads) * 128, d->hidden};
    if (seq_map && kv_batch < d->batch)
        return fail(FDL_EINVAL, "qkv_attention: the caches hold %d sequences, fewer than the "
                    "%d of the batch", kv_batch, d->batch);
    const fdl::EpiQKV p{(fdl::bf16*)q_out, (fdl::bf16*)k_cache, (fdl::bf16*)v_cache, bias,
                        (const float2*)rope, d->n_q_heads, d->n_kv_heads, d->seq_len,
                        d->rows_per_seq, d->pos0, seq_map, pos0_map};
    fdl::AttnShape as{d->batch, d->n_q_heads, d->n_kv_heads, 128, d->seq_len, d->pos0,
                      d->rows_per_seq, 1.0f / sqrtf(128.f), 1};
    as.seq_map = seq_map;
    as.kv_batch = seq_map ? kv_batch : 0;
    as.blk0_map = pos0_map;
    const fdl::NormIn ni{h, norm_w, eps};
    cudaError_t e;
    const int splits = fdl::skinny_ok(gs) ? fdl::skinny_qkv_splits(gs, ctx->acc_bytes,
                                                                   ctx->sm_count) : 1;
    if (splits > 1 && fdl::qkv_attention_fusable(as, ctx->sm_count)) {
        e = fdl::launch_skinny_qkv_sums(gs, x, w, ctx->d_acc, splits, norm_w ? &ni : nullptr,
                                        ctx->d_sync + 6, ctx->sm_count, ctx->d_err, st);
        if (e == cudaSuccess)
            e = fdl::launch_qkv_attention_bf16(as, ctx->d_acc, p, out, ctx->sm_count, ctx->d_err,
                                               st);
    } else {
        e = norm_w ? fdl::launch_rmsnorm(d->rows, d->hidden, h, nullptr, norm_w, eps,
                                         (fdl::bf16*)x, st)
                   : cudaSuccess;
        if (e == cudaSuccess)
            e = fdl::skinny_ok(gs)
                ? fdl::launch_skinny_qkv(gs, x, w, p, ctx->d_acc, ctx->acc_bytes, ctx->sm_count,
                                         ctx->d_err, st)
                : fdl::launch_gemm_qkv(gs, x, w, p, ctx->sm_count, ctx->d_err, st);
        if (e == cudaSuccess)
            e = fdl::launch_attention_bf16(as, q_out, k_cache, v_cache, out, nullptr, nullptr,
                                           ctx->sm_count, ctx->d_err, st);
    }
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "qkv_attention launch");
}

extern "C" {

int fdl_linear_residual(fdl_ctx* ctx, int rows, int out_features, int in_features,
                        const void* x, const void* w, float* h, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "linear_residual: ctx is NULL");
    if (rows < 1 || out_features < 64 || out_features % 64 || in_features < 64 ||
        in_features % 64)
        return fail(FDL_EINVAL, "linear_residual: rows >= 1, in and out multiples of 64");
    if (!x || !w || !h) return fail(FDL_EINVAL, "linear_residual: NULL buffer");
    if (!aligned16(x) || !aligned16(w) || !aligned16(h))
        return fail(FDL_EINVAL, "linear_residual: buffers must be 16-byte aligned");
    DeviceGuard g(ctx->device);
    fdl::GemmShape gs{rows, out_features, in_features};
    const fdl::EpiResid ep{h, out_features};
    cudaError_t e = fdl::skinny_ok(gs)
        ? fdl::launch_skinny_resid(gs, x, w, ep, ctx->sm_count, ctx->d_err,
                                   (cudaStream_t)stream)
        : fdl::launch_gemm_resid(gs, x, w, ep, ctx->sm_count, ctx->d_err, (cudaStream_t)stream);
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "linear_residual launch");
}

int fdl_linear_swiglu(fdl_ctx* ctx, int rows, int out_features, int in_features, const void* x,
                      const void* w_gu, void* out, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "linear_swiglu: ctx is NULL");
    if (rows < 1 || out_features < 32 || out_features % 32 || in_features < 64 ||
        in_features % 64)
        return fail(FDL_EINVAL, "linear_swiglu: rows >= 1, out % 32 == 0, in % 64 == 0");
    if (!x || !w_gu || !out) return fail(FDL_EINVAL, "linear_swiglu: NULL buffer");
    if (!aligned16(x) || !aligned16(w_gu) || !aligned16(out))
        return fail(FDL_EINVAL, "linear_swiglu: buffers must be 16-byte aligned");
    DeviceGuard g(ctx->device);
    fdl::GemmShape gs{rows, 2 * out_features, in_features};
    const fdl::EpiSwiGLU ep{(fdl::bf16*)out, out_features};
    cudaError_t e = fdl::skinny_ok(gs)
        ? fdl::launch_skinny_swiglu(gs, x, w_gu, ep, ctx->d_acc, ctx->acc_bytes, ctx->sm_count,
                                    ctx->d_err, (cudaStream_t)stream)
        : fdl::launch_gemm_swiglu(gs, x, w_gu, ep, ctx->sm_count, ctx->d_err,
                                  (cudaStream_t)stream);
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "linear_swiglu launch");
}

int fdl_ffn(fdl_ctx* ctx, int rows, int hidden, int ffn, const float* norm_w, float eps, void* x,
            const void* w_gu, const void* w_down, void* f, float* h, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "ffn: ctx is NULL");
    if (rows < 1 || hidden < 64 || hidden % 64 || ffn < 64 || ffn % 64)
        return fail(FDL_EINVAL, "ffn: rows >= 1, hidden % 64 == 0, ffn % 64 == 0");
    if (!x || !w_gu || !w_down || !f || !h) return fail(FDL_EINVAL, "ffn: NULL buffer");
    if (!aligned16(x) || !aligned16(w_gu) || !aligned16(w_down) || !aligned16(f) ||
        !aligned16(h) || (norm_w && !aligned16(norm_w)))
        return fail(FDL_EINVAL, "ffn: buffers must be 16-byte aligned");
    if (norm_w && !(eps > 0.f)) return fail(FDL_EINVAL, "ffn: eps must be > 0");
    DeviceGuard g(ctx->device);
    cudaStream_t st = (cudaStream_t)stream;
    const fdl::GemmShape gu{rows, 2 * ffn, hidden}, dn{rows, hidden, ffn};
    const fdl::NormIn ni{h, norm_w, eps};
    cudaError_t e;
    if (fdl::skinny_ok(gu) && fdl::skinny_ok(dn)) {
        e = fdl::launch_skinny_ffn(gu, x, w_gu, w_down, (fdl::bf16*)f, h, hidden, ctx->d_acc,
                                   ctx->acc_bytes, ctx->d_sync, norm_w ? &ni : nullptr,
                                   ctx->sm_count, ctx->d_err, st);
    } else {
        e = norm_w ? fdl::launch_rmsnorm(rows, hidden, h, nullptr, norm_w, eps, (fdl::bf16*)x, st)
                   : cudaSuccess;
        if (e != cudaSuccess) return cuda_fail(e, "ffn launch");
        const fdl::EpiSwiGLU es{(fdl::bf16*)f, ffn};
        e = fdl::skinny_ok(gu)
            ? fdl::launch_skinny_swiglu(gu, x, w_gu, es, ctx->d_acc, ctx->acc_bytes,
                                        ctx->sm_count, ctx->d_err, st)
            : fdl::launch_gemm_swiglu(gu, x, w_gu, es, ctx->sm_count, ctx->d_err, st);
        if (e == cudaSuccess) {
            const fdl::EpiResid er{h, hidden};
            e = fdl::skinny_ok(dn)
                ? fdl::launch_skinny_resid(dn, f, w_down, er, ctx->sm_count, ctx->d_err, st)
                : fdl::launch_gemm_resid(dn, f, w_down, er, ctx->sm_count, ctx->d_err, st);
        }
    }
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "ffn launch");
}

int fdl_full_attention(fdl_ctx* ctx, const fdl_attn_desc* desc, const void* q,
                       const void* k_cache, const void* v_cache, void* out, void* stream) {
    if (!ctx) return fail(FDL_EINVAL, "full_attention: ctx is NULL");
    if (!desc) return fail(FDL_EINVAL, "full_attention: desc is NULL");
    if (desc->dtype != FDL_BF16) return fail(FDL_EUNSUPPORTED, "full_attention: bf16 only");
    if (desc->head_dim != 64 && desc->head_dim != 128)
        return fail(FDL_EUNSUPPORTED, "full_attention: head_dim %d", desc->head_dim);
    if (desc->batch < 1 || desc->n_q_heads < 1 || desc->n_kv_heads < 1 ||
        desc->n_q_heads % desc->n_kv_heads || desc->block_start < 0 ||
        desc->seq_len - desc->block_start < 32 || (desc->seq_len - desc->block_start) % 32)
        return fail(FDL_EINVAL, "full_attention: bad shape (batch, heads; seq_len - block_start "
                    "a positive multiple of 32)");
    if (!q || !k_cache || !v_cache || !out) return fail(FDL_EINVAL, "full_attention: NULL");
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return fail(FDL_EINVAL, "full_attention: buffers must be 16-byte aligned");
    DeviceGuard g(ctx->device);
    const float scale = desc->scale == 0.f ? 1.0f / sqrtf((float)desc->head_dim) : desc->scale;
    cudaError_t e = fdl::launch_full_attention_bf16(desc->batch, desc->n_q_heads,
                                                    desc->n_kv_heads, desc->head_dim,
                                                    desc->seq_len, desc->seq_len -
                                                    desc->block_start, scale, q, k_cache,
                                                    v_cache, out, ctx->sm_count, ctx->d_err,
                                                    (cudaStream_t)stream);
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "full_attention launch");
}

}  // extern "C"

// ---- the whole decode ------------------------------------------------------------
struct fdl_model {
    uint64_t id;              // unique per fdl_model_create (keys the cached decode graph)
    fdl_model_desc d;
    const void* embed;
    const float* final_norm;
    const void* lm_head;
    std::vector<fdl_layer_weights> layers;
};

namespace {

__global__ void fill_i32_kernel(int32_t* __restrict__ p, size_t n, int32_t v) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        p[i] = v;
}

// rows of block k of every sequence in the flattened [b * L] token rows:
// maps[k][i * B + j] = i * L + k * B + j (clamped to the last row)
__global__ void block_rows_kernel(int32_t* __restrict__ maps, int b, int L, int B, int nblk) {
    const size_t n = (size_t)nblk * b * B;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
         e += (size_t)gridDim.x * blockDim.x) {
        const int k = (int)(e / ((size_t)b * B)), r = (int)(e % ((size_t)b * B));
        const int i = r / B, j = r % B;
        const long v = (long)i * L + (long)k * B + j;
        maps[e] = (int32_t)(v < (long)b * L ? v : (long)b * L - 1);
    }
}

// PrefixCache row maps of the block at s: tail[i * n + j] = i * L + s + j for
// j < n = L - s (rows [s, L) of sequence i in the [b * L] token rows) and
// blk[i * B + j] = i * n + j (the block's rows among those b * n rows).
__global__ void tail_rows_kernel(int32_t* __restrict__ tail, int32_t* __restrict__ blk, int b,
                                 int L, int s, int B) {
    const int n = L - s;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < b * n; e += gridDim.x * blockDim.x) {
        const int i = e / n, j = e % n;
        tail[e] = i * L + s + j;
        if (j < B) blk[i * B + j] = i * n + j;
    }
}

// A compacted DualCache step of the block at s: the sequences with masked
// positions left in the block (remaining > 0), in order, become the batch;
// seq_map[i] is the sequence of batch entry i, rows[i * B + j] the token row
// of its block position j, and the block's planted bias rows are gathered to
// match. One CTA; returns nothing (the host derives the same count from the
// same counts).
__global__ void compact_batch_kernel(const int32_t* __restrict__ remaining, int b, int L, int s,
                                     int B, int32_t* __restrict__ seq_map,
                                     int32_t* __restrict__ rows, const int32_t* __restrict__ btok,
                                     const float* __restrict__ bval, int32_t* __restrict__ btok_c,
                                     float* __restrict__ bval_c) {
    __shared__ int n_act;
    if (threadIdx.x == 0) {
        int n = 0;
        for (int i = 0; i < b; ++i)
            if (remaining[i] > 0) seq_map[n++] = i;
        n_act = n;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n_act * B; e += blockDim.x) {
        const int i = e / B, j = e % B, sq = seq_map[i];
        rows[e] = sq * L + s + j;
        if (btok) {
            btok_c[e] = btok[sq * B + j];
            bval_c[e] = bval[sq * B + j];
        }
    }
}

// The planted-bias rows of n sequences at their own blocks: row i * B + j is
// position s_of[i] + j of sequence seq[i] (bias arrays [b, gen] from prompt_len
// P on).
__global__ void gather_bias_kernel(const int32_t* __restrict__ btok,
                                   const float* __restrict__ bval, int gen, int P, int B,
                                   const int32_t* __restrict__ seq,
                                   const int32_t* __restrict__ s_of, int n,
                                   int32_t* __restrict__ btok_c, float* __restrict__ bval_c) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n * B; e += gridDim.x * blockDim.x) {
        const int i = e / B, j = e % B;
        const size_t src = (size_t)seq[i] * gen + (s_of[i] - P) + j;
        btok_c[e] = btok[src];
        bval_c[e] = bval[src];
    }
}

// Byte offsets of the generate workspace (256-byte aligned pieces).
struct GenLayout {
    size_t kc, vc, h_full, x_full, q_full, o_full, f_full, h_blk, x_blk, q_blk, o_blk, f_blk,
        xn, conf, tok, masked, counts, maps, tail_map, tail_blk, bias_tok, bias_val, rope, lm_ws,
        x, steps, seq_map, row_map_c, bias_tok_c, bias_val_c, ps_maps, total;
    size_t kv_layer;    // bytes of one layer's K (or V) cache
    size_t lm_bytes;
};

GenLayout gen_layout(const fdl_model_desc& d, int b, int L, int B, size_t lm_bytes) {
    GenLayout g{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    const size_t D = d.hidden, F = d.ffn, hd = 128, Hq = d.n_q_heads, Hkv = d.n_kv_heads;
    const size_t rf = (size_t)b * L, rb = (size_t)b * B;
    const int nblk = (L + B - 1) / B;
    g.kv_layer = (size_t)b * Hkv * L * hd * 2;
    g.kc = take(g.kv_layer * d.n_layers);
    g.vc = take(g.kv_layer * d.n_layers);
    g.h_full = take(rf * D * 4);
    g.x_full = take(rf * D * 2);
    g.q_full = take(rf * Hq * hd * 2);
    g.o_full = take(rf * Hq * hd * 2);
    g.f_full = take(rf * F * 2);
    g.h_blk = take(rb * D * 4);
    g.x_blk = take(rb * D * 2);
    g.q_blk = take(rb * Hq * hd * 2);
    g.o_blk = take(rb * Hq * hd * 2);
    g.f_blk = take(rb * F * 2);
    g.xn = take(rb * D * 2);
    g.conf = take(rb * 4);
    g.tok = take(rb * 4);
    g.masked = take(rf);
    g.counts = take((size_t)2 * b * 4);
    g.maps = take((size_t)nblk * rb * 4);
    g.tail_map = take(rf * 4);       // PrefixCache: rows [s, L) of every sequence
    g.tail_blk = take(rb * 4);       // ... and the block's rows among them
    g.bias_tok = take(rb * 4);       // the planted bias of the current block's rows
    g.bias_val = take(rb * 4);
    g.rope = take((size_t)L * hd * 4);
    g.lm_bytes = lm_bytes;
    g.lm_ws = take(lm_bytes);
    g.x = take(rf * 4);              // the decode's token ids (copied out at the end)
    g.steps = take(16);              // decode steps taken (device loop)
    g.seq_map = take((size_t)b * 4); // compacted steps: the sequences still decoding,
    g.row_map_c = take(rb * 4);      // ... their block rows among the token rows,
    g.bias_tok_c = take(rb * 4);     // ... and their rows of the planted bias
    g.bias_val_c = take(rb * 4);
    // sequences at their own blocks: the maps of one step, written by the host
    // (sequence ids, block starts, token rows of up to b whole sequences, and
    // the block rows among them)
    g.ps_maps = take(((size_t)2 * b + rf + rb) * 4);
    g.total = off;
    return g;
}

// One decode of fdl_generate: its shapes, the workspace pieces, and the
// issuing of a block's set-up and of one decode step on a given stream (used by
// the host loop and, captured, by the device loop).
struct GenRun {
    fdl_ctx* ctx;
    const fdl_model* m;
    int b, P, gen, B, L, mode;
    float tau;
    const int32_t* bias_tok;
    const float* bias_val;
    GenLayout g;
    char* base;

    void* at(size_t off) const { return static_cast<void*>(base + off); }
    int32_t* x() const { return (int32_t*)at(g.x); }
    uint8_t* masked() const { return (uint8_t*)at(g.masked); }
    int32_t* remaining() const { return (int32_t*)at(g.counts); }
    int32_t* maps() const { return (int32_t*)at(g.maps); }

    // per block, before its first step: the planted bias of its rows and, for
    // the PrefixCache, its row maps
    int block_prep(int blk, cudaStream_t st) const {
        const int s = P + blk * B;
        cudaError_t e = cudaSuccess;
        if (bias_tok) {
            // this block's planted bias, [b, gen] -> [b, B] contiguous
            e = cudaMemcpy2DAsync(at(g.bias_tok), (size_t)B * 4, bias_tok + (s - P),
                                  (size_t)gen * 4, (size_t)B * 4, b, cudaMemcpyDeviceToDevice, st);
            if (e == cudaSuccess)
                e = cudaMemcpy2DAsync(at(g.bias_val), (size_t)B * 4, bias_val + (s - P),
                                      (size_t)gen * 4, (size_t)B * 4, b,
                                      cudaMemcpyDeviceToDevice, st);
        }
        if (e == cudaSuccess && mode == FDL_CACHE_PREFIX) {
            tail_rows_kernel<<<64, 256, 0, st>>>((int32_t*)at(g.tail_map),
                                                 (int32_t*)at(g.tail_blk), b, L, s, B);
            e = cudaGetLastError();
        }
        return e == cudaSuccess ? FDL_OK : cuda_fail(e, "generate: block set-up");
    }

    // The layers over rows = b * n token rows at positions [pos0, pos0 + n) of
    // every sequence. full: their K/V go into the caches and they attend over
    // the whole cache (refresh: pos0 = 0, n = L; PrefixCache step: pos0 = s,
    // n = L - s); otherwise the fused DualCache step of the block rows.
    // With seq_map, the rows are those of nb sequences, batch entry i being
    // sequence seq_map[i] of the caches; with pos0_map (a DualCache step of
    // sequences at their own blocks), entry i's block starts at pos0_map[i].
    int layers(float* h, void* xb, void* q, void* o, void* f, int rows, bool full, int pos0,
               int n, cudaStream_t st, int nb = -1, const int32_t* seq_map = nullptr,
               const int32_t* pos0_map = nullptr) const {
        const fdl_model_desc& d = m->d;
        const int D = d.hidden, F = d.ffn, Hq = d.n_q_heads, Hkv = d.n_kv_heads, hd = 128;
        void* stream = (void*)st;
        const float* rope = (const float*)at(g.rope);
        int rc = FDL_OK;
        for (int li = 0; li < d.n_layers && rc == FDL_OK; ++li) {
            const fdl_layer_weights& W = m->layers[li];
            void* kl = base + g.kc + g.kv_layer * li;
            void* vl = base + g.vc + g.kv_layer * li;
            const fdl_qkv_desc qd{rows, D, Hq, Hkv, hd, nb > 0 ? nb : b, L, n, pos0, L};
            if (full) {
                rc = fdl_rmsnorm(ctx, rows, D, h, nullptr, W.attn_norm, d.rms_eps, xb, stream);
                if (!rc) rc = qkv_rope_store_mapped(ctx, &qd, xb, W.w_qkv, W.bias, rope, q, kl,
                                                    vl, stream, seq_map, b);
                if (!rc && !seq_map) {
                    const fdl_attn_desc ad{b, Hq, Hkv, hd, L, pos0, n, FDL_BF16, 0.f};
                    rc = fdl_full_attention(ctx, &ad, q, kl, vl, o, stream);
                } else if (!rc) {
                    // the whole-sequence forward of the nb sequences of seq_map
                    const cudaError_t e = fdl::launch_full_attention_bf16(
                        nb, Hq, Hkv, hd, L, n, 1.0f / sqrtf((float)hd), q, kl, vl, o,
                        ctx->sm_count, ctx->d_err, st, seq_map, b);
                    if (e != cudaSuccess) rc = cuda_fail(e, "generate: full attention");
                }
            } else {
                rc = qkv_attention_mapped(ctx, &qd, h, W.attn_norm, d.rms_eps, xb, W.w_qkv,
                                          W.bias, rope, q, kl, vl, o, stream, seq_map, b,
                                          pos0_map);
            }
            if (!rc) rc = fdl_linear_residual(ctx, rows, D, Hq * hd, o, W.wo, h, stream);
            if (!rc) rc = fdl_ffn(ctx, rows, D, F, W.ffn_norm, d.rms_eps, xb, W.w_gu, W.w_down, f,
                                  h, stream);
        }
        return rc;
    }

    // A cached DualCache step over only the n_act < b sequences that still
    // have masked positions in the block (the others' rows would decode
    // nothing): the same step on a compacted batch, whose rows read and write
    // the caches, tokens and counts of the sequences they stand for.
    int compact_step(int blk, int n_act, cudaStream_t st) const {
        const fdl_model_desc& d = m->d;
        const int D = d.hidden, rc_rows = n_act * B, s = P + blk * B;
        void* stream = (void*)st;
        int32_t* smap = (int32_t*)at(g.seq_map);
        int32_t* rows = (int32_t*)at(g.row_map_c);
        compact_batch_kernel<<<1, 256, 0, st>>>(
            remaining(), b, L, s, B, smap, rows, bias_tok ? (const int32_t*)at(g.bias_tok) : nullptr,
            (const float*)at(g.bias_val), (int32_t*)at(g.bias_tok_c), (float*)at(g.bias_val_c));
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "generate: compaction");
        float* h_blk = (float*)at(g.h_blk);
        int rc = fdl_embed(ctx, rc_rows, D, x(), rows, m->embed, h_blk, stream);
        if (!rc) rc = layers(h_blk, at(g.x_blk), at(g.q_blk), at(g.o_blk), at(g.f_blk), rc_rows,
                             false, s, B, st, n_act, smap);
        if (!rc) rc = fdl_rmsnorm(ctx, rc_rows, D, h_blk, nullptr, m->final_norm, d.rms_eps,
                                  at(g.xn), stream);
        const fdl_lmhead_desc lmd{rc_rows, D, d.vocab, FDL_BF16};
        if (!rc) rc = fdl_lmhead_confidence(ctx, &lmd, at(g.xn), m->lm_head,
                                            bias_tok ? (const int32_t*)at(g.bias_tok_c) : nullptr,
                                            bias_tok ? (const float*)at(g.bias_val_c) : nullptr,
                                            (float*)at(g.conf), (int32_t*)at(g.tok), at(g.lm_ws),
                                            g.lm_bytes, stream);
        if (rc) return rc;
        e = fdl::launch_threshold_unmask(n_act, L, s, B, tau, (const float*)at(g.conf),
                                         (const int32_t*)at(g.tok), x(), masked(), remaining(),
                                         remaining() + b, ctx->d_err, st, smap);
        return e == cudaSuccess ? FDL_OK : cuda_fail(e, "generate: unmask");
    }

    // Sequences at their own blocks. The host writes the step's maps into
    // ps_maps: n sequence ids, their n block starts, then the token rows the
    // step embeds, then (a refresh) the block rows among the forward's rows.
    int32_t* ps_seq() const { return (int32_t*)at(g.ps_maps); }
    int32_t* ps_start() const { return ps_seq() + b; }
    int32_t* ps_rows() const { return ps_seq() + 2 * b; }
    int32_t* ps_blk_rows() const { return ps_rows() + (size_t)b * L; }

    // The step's maps to the device (stream-ordered; `host` may be reused once
    // this returns) and the gather of the planted bias of the n sequences'
    // blocks.
    int ps_upload(const std::vector<int32_t>& host, int n, cudaStream_t st) const {
        cudaError_t e = cudaMemcpyAsync(ps_seq(), host.data(), host.size() * 4,
                                        cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess && bias_tok) {
            gather_bias_kernel<<<32, 256, 0, st>>>(bias_tok, bias_val, gen, P, B, ps_seq(),
                                                   ps_start(), n, (int32_t*)at(g.bias_tok_c),
                                                   (float*)at(g.bias_val_c));
            e = cudaGetLastError();
        }
        return e == cudaSuccess ? FDL_OK : cuda_fail(e, "generate: step maps");
    }

    // LM head over the n sequences' block rows in xn, then the unmask of each
    // at its own block.
    int ps_decide(int n, cudaStream_t st) const {
        const fdl_model_desc& d = m->d;
        const fdl_lmhead_desc lmd{n * B, d.hidden, d.vocab, FDL_BF16};
        int rc = fdl_lmhead_confidence(ctx, &lmd, at(g.xn), m->lm_head,
                                       bias_tok ? (const int32_t*)at(g.bias_tok_c) : nullptr,
                                       bias_tok ? (const float*)at(g.bias_val_c) : nullptr,
                                       (float*)at(g.conf), (int32_t*)at(g.tok), at(g.lm_ws),
                                       g.lm_bytes, (void*)st);
        if (rc) return rc;
        const cudaError_t e = fdl::launch_threshold_unmask(
            n, L, P, B, tau, (const float*)at(g.conf), (const int32_t*)at(g.tok), x(), masked(),
            remaining(), remaining() + b, ctx->d_err, st, ps_seq(), ps_start());
        return e == cudaSuccess ? FDL_OK : cuda_fail(e, "generate: unmask");
    }

    // The refresh of n sequences that have just moved to a new block: the full
    // forward over all their positions (their caches rewritten), then the
    // first step of their new blocks.
    int ps_refresh(int n, cudaStream_t st) const {
        const fdl_model_desc& d = m->d;
        float* h_full = (float*)at(g.h_full);
        int rc = fdl_embed(ctx, n * L, d.hidden, x(), ps_rows(), m->embed, h_full, (void*)st);
        if (!rc) rc = layers(h_full, at(g.x_full), at(g.q_full), at(g.o_full), at(g.f_full),
                             n * L, true, 0, L, st, n, ps_seq());
        if (!rc) rc = fdl_rmsnorm(ctx, n * B, d.hidden, h_full, ps_blk_rows(), m->final_norm,
                                  d.rms_eps, at(g.xn), (void*)st);
        return rc ? rc : ps_decide(n, st);
    }

    // A DualCache step of n sequences, each at its own block.
    int ps_cached(int n, cudaStream_t st) const {
        const fdl_model_desc& d = m->d;
        float* h_blk = (float*)at(g.h_blk);
        int rc = fdl_embed(ctx, n * B, d.hidden, x(), ps_rows(), m->embed, h_blk, (void*)st);
        if (!rc) rc = layers(h_blk, at(g.x_blk), at(g.q_blk), at(g.o_blk), at(g.f_blk), n * B,
                             false, P, B, st, n, ps_seq(), ps_start());
        if (!rc) rc = fdl_rmsnorm(ctx, n * B, d.hidden, h_blk, nullptr, m->final_norm,
                                  d.rms_eps, at(g.xn), (void*)st);
        return rc ? rc : ps_decide(n, st);
    }

    // One decode step of block blk: the forward (the refresh when `first` or
    // without a cache, else the cache mode's step), the LM head with the
    // confidence reduction, and the threshold unmask (remaining[] written).
    int step(int blk, bool first, cudaStream_t st) const {
        const fdl_model_desc& d = m->d;
        const int D = d.hidden, rf = b * L, rb = b * B, s = P + blk * B;
        void* stream = (void*)st;
        const int32_t* row_map = maps() + (size_t)(s / B) * rb;
        float* h_full = (float*)at(g.h_full);
        float* h_blk = (float*)at(g.h_blk);
        int rc;
        if (first || mode == FDL_CACHE_NONE) {
            // full forward over every position: all K/V caches rewritten
            rc = fdl_embed(ctx, rf, D, x(), nullptr, m->embed, h_full, stream);
            if (!rc) rc = layers(h_full, at(g.x_full), at(g.q_full), at(g.o_full), at(g.f_full),
                                 rf, true, 0, L, st);
            if (!rc) rc = fdl_rmsnorm(ctx, rb, D, h_full, row_map, m->final_norm, d.rms_eps,
                                      at(g.xn), stream);
        } else if (mode == FDL_CACHE_PREFIX) {
            // PrefixCache step: the block and the suffix over the cached prefix
            const int n = L - s;
            rc = fdl_embed(ctx, b * n, D, x(), (const int32_t*)at(g.tail_map), m->embed, h_full,
                           stream);
            if (!rc) rc = layers(h_full, at(g.x_full), at(g.q_full), at(g.o_full), at(g.f_full),
                                 b * n, true, s, n, st);
            if (!rc) rc = fdl_rmsnorm(ctx, rb, D, h_full, (const int32_t*)at(g.tail_blk),
                                      m->final_norm, d.rms_eps, at(g.xn), stream);
        } else {
            // DualCache step: only the block's rows
            rc = fdl_embed(ctx, rb, D, x(), row_map, m->embed, h_blk, stream);
            if (!rc) rc = layers(h_blk, at(g.x_blk), at(g.q_blk), at(g.o_blk), at(g.f_blk), rb,
                                 false, s, B, st);
            if (!rc) rc = fdl_rmsnorm(ctx, rb, D, h_blk, nullptr, m->final_norm, d.rms_eps,
                                      at(g.xn), stream);
        }
        const fdl_lmhead_desc lmd{rb, D, d.vocab, FDL_BF16};
        if (!rc) rc = fdl_lmhead_confidence(ctx, &lmd, at(g.xn), m->lm_head,
                                            bias_tok ? (const int32_t*)at(g.bias_tok) : nullptr,
                                            bias_tok ? (const float*)at(g.bias_val) : nullptr,
                                            (float*)at(g.conf), (int32_t*)at(g.tok), at(g.lm_ws),
                                            g.lm_bytes, stream);
        const fdl_unmask_desc ud{b, L, s, B, tau};
        if (!rc) rc = fdl_threshold_unmask(ctx, &ud, (const float*)at(g.conf),
                                           (const int32_t*)at(g.tok), x(), masked(), remaining(),
                                           remaining() + b, stream);
        return rc;
    }
};

// After a step of the device loop: count it, and set the block's loop
// condition to "a sequence still has a masked position in the block".
__global__ void loop_cond_kernel(cudaGraphConditionalHandle h, const int32_t* __restrict__ rem,
                                 int b, int32_t* __restrict__ steps) {
    if (threadIdx.x != 0) return;
    int any = 0;
    for (int i = 0; i < b; ++i) any |= rem[i] > 0;
    cudaGraphSetConditional(h, any ? 1u : 0u);
    *steps += 1;
}

bool same_key(const GenGraph* c, const GenRun& r, size_t ws_bytes) {
    return c && c->exec && c->model == r.m->id && c->ws == r.base && c->ws_bytes == ws_bytes &&
           c->b == r.b && c->P == r.P && c->gen == r.gen && c->B == r.B && c->mode == r.mode &&
           c->tau == r.tau && c->bias_tok == r.bias_tok && c->bias_val == r.bias_val;
}

// Capture the whole decode as one CUDA graph: per block its set-up and first
// step (the refresh), then a conditional WHILE node whose body is one cached
// step; a small kernel after every step sets the condition from the counts of
// masked positions left, so the block's steps repeat on the device with no
// host round trip. Captured on the context's own non-blocking streams.
int build_gen_graph(const GenRun& r, GenGraph* c, cudaGraphExec_t* out) {
    *out = nullptr;
    cudaError_t e = cudaSuccess;
    if (!c->cap) e = cudaStreamCreateWithFlags(&c->cap, cudaStreamNonBlocking);
    if (e == cudaSuccess && !c->body) e = cudaStreamCreateWithFlags(&c->body, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "generate: capture streams");
    cudaStream_t cs = c->cap;
    e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return cuda_fail(e, "generate: begin capture");
    int32_t* steps = (int32_t*)r.at(r.g.steps);
    int rc = FDL_OK;
    cudaGraph_t graph = nullptr;
    for (int blk = 0; rc == FDL_OK && blk < r.gen / r.B; ++blk) {
        cudaStreamCaptureStatus status;
        const cudaGraphNode_t* deps = nullptr;
        size_t ndeps = 0;
        e = cudaStreamGetCaptureInfo(cs, &status, nullptr, &graph, &deps, &ndeps);
        cudaGraphConditionalHandle h = 0;
        if (e == cudaSuccess) e = cudaGraphConditionalHandleCreate(&h, graph, 0, 0);
        if (e != cudaSuccess) { rc = cuda_fail(e, "generate: condition"); break; }
        rc = r.block_prep(blk, cs);
        if (!rc) rc = r.step(blk, true, cs);
        if (rc) break;
        loop_cond_kernel<<<1, 32, 0, cs>>>(h, r.remaining(), r.b, steps);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaStreamGetCaptureInfo(cs, &status, nullptr, &graph, &deps, &ndeps);
        cudaGraphNodeParams cp = {};
        cp.type = cudaGraphNodeTypeConditional;
        cp.conditional.handle = h;
        cp.conditional.type = cudaGraphCondTypeWhile;
        cp.conditional.size = 1;
        cudaGraphNode_t node = nullptr;
        if (e == cudaSuccess) e = cudaGraphAddNode(&node, graph, deps, ndeps, &cp);
        if (e == cudaSuccess)
            e = cudaStreamUpdateCaptureDependencies(cs, &node, 1, cudaStreamSetCaptureDependencies);
        if (e != cudaSuccess) { rc = cuda_fail(e, "generate: loop node"); break; }
        // the body: one cached step, then the condition again
        cudaGraph_t body = cp.conditional.phGraph_out[0];
        e = cudaStreamBeginCaptureToGraph(c->body, body, nullptr, nullptr, 0,
                                          cudaStreamCaptureModeThreadLocal);
        if (e != cudaSuccess) { rc = cuda_fail(e, "generate: body capture"); break; }
        rc = r.step(blk, false, c->body);
        if (!rc) {
            loop_cond_kernel<<<1, 32, 0, c->body>>>(h, r.remaining(), r.b, steps);
            e = cudaGetLastError();
        }
        cudaGraph_t body_out = nullptr;
        const cudaError_t e2 = cudaStreamEndCapture(c->body, &body_out);
        if (!rc && e == cudaSuccess) e = e2;
        if (!rc && e != cudaSuccess) rc = cuda_fail(e, "generate: body");
    }
    cudaGraph_t whole = nullptr;
    const cudaError_t e3 = cudaStreamEndCapture(cs, &whole);
    if (!rc && e3 != cudaSuccess) rc = cuda_fail(e3, "generate: end capture");
    if (!rc) {
        e = cudaGraphInstantiate(out, whole, 0);
        if (e != cudaSuccess) rc = cuda_fail(e, "generate: instantiate");
    }
    if (whole) cudaGraphDestroy(whole);
    return rc;
}

int run_device_loop(const GenRun& r, cudaStream_t st) {
    fdl_ctx* ctx = r.ctx;
    const size_t ws_bytes = r.g.total;
    if (!same_key(ctx->gen, r, ws_bytes)) {
        if (!ctx->gen) ctx->gen = new GenGraph;
        GenGraph* c = ctx->gen;
        if (c->exec) {
            cudaGraphExecDestroy(c->exec);
            c->exec = nullptr;
        }
        cudaGraphExec_t exec = nullptr;
        const int rc = build_gen_graph(r, c, &exec);
        if (rc) return rc;
        c->exec = exec;
        c->model = r.m->id;
        c->ws = r.base;
        c->ws_bytes = ws_bytes;
        c->b = r.b;
        c->P = r.P;
        c->gen = r.gen;
        c->B = r.B;
        c->mode = r.mode;
        c->tau = r.tau;
        c->bias_tok = r.bias_tok;
        c->bias_val = r.bias_val;
    }
    const cudaError_t e = cudaGraphLaunch(ctx->gen->exec, st);
    return e == cudaSuccess ? FDL_OK : cuda_fail(e, "generate: graph launch");
}

bool model_desc_ok(const fdl_model_desc* d) {
    return d && d->vocab >= 2 && d->hidden >= 128 && d->hidden % 128 == 0 && d->n_layers >= 1 &&
           d->n_kv_heads >= 1 && d->n_q_heads >= d->n_kv_heads &&
           d->n_q_heads % d->n_kv_heads == 0 && d->head_dim == 128 && d->ffn >= 64 &&
           d->ffn % 64 == 0 && d->mask_id >= 0 && d->mask_id < d->vocab && d->rope_theta > 0.f &&
           d->rms_eps > 0.f;
}

size_t lm_ws_bytes(fdl_ctx* ctx, const fdl_model_desc& d, int rows) {
    const fdl_lmhead_desc ld{rows, d.hidden, d.vocab, FDL_BF16};
    const size_t n = fdl_lmhead_workspace_bytes(ctx, &ld);
    return n > 16 ? n : 16;
}

}  // namespace

extern "C" {

int fdl_model_create(const fdl_model_desc* desc, const fdl_model_weights* w, fdl_model** out) {
    if (!out) return fail(FDL_EINVAL, "model_create: out is NULL");
    *out = nullptr;
    if (!model_desc_ok(desc))
        return fail(FDL_EINVAL, "model_create: bad description (hidden a multiple of 128, "
                    "head_dim 128, Hq a multiple of Hkv, ffn a multiple of 64, 0 <= mask_id < "
                    "vocab, rope_theta and rms_eps > 0)");
    if (!w || !w->embed || !w->final_norm || !w->lm_head || !w->layers)
        return fail(FDL_EINVAL, "model_create: NULL weight pointer");
    if (!aligned16(w->embed) || !aligned16(w->final_norm) || !aligned16(w->lm_head))
        return fail(FDL_EINVAL, "model_create: weights must be 16-byte aligned");
    static std::atomic<uint64_t> next_id{1};
    fdl_model* m = new fdl_model;
    m->id = next_id++;
    m->d = *desc;
    m->embed = w->embed;
    m->final_norm = w->final_norm;
    m->lm_head = w->lm_head;
    m->layers.assign(w->layers, w->layers + desc->n_layers);
    for (int l = 0; l < desc->n_layers; ++l) {
        const fdl_layer_weights& L = m->layers[l];
        if (!L.attn_norm || !L.w_qkv || !L.wo || !L.ffn_norm || !L.w_gu || !L.w_down ||
            !aligned16(L.attn_norm) || !aligned16(L.w_qkv) || !aligned16(L.wo) ||
            !aligned16(L.ffn_norm) || !aligned16(L.w_gu) || !aligned16(L.w_down) ||
            (L.bias && !aligned16(L.bias))) {
            delete m;
            return fail(FDL_EINVAL, "model_create: layer %d: NULL or unaligned weight", l);
        }
    }
    *out = m;
    return FDL_OK;
}

int fdl_model_destroy(fdl_model* model) {
    delete model;
    return FDL_OK;
}

size_t fdl_generate_workspace_bytes(fdl_ctx* ctx, const fdl_model* m, int batch, int seq_len,
                                    int block) {
    if (!ctx || !m || batch < 1 || seq_len < 1 || block < 1 || block > 128) return 0;
    return gen_layout(m->d, batch, seq_len, block, lm_ws_bytes(ctx, m->d, batch * block)).total;
}

int fdl_generate(fdl_ctx* ctx, const fdl_model* m, const int32_t* prompt, int b, int P, int gen,
                 int B, float tau, const fdl_generate_opts* opts, int32_t* out_x, int* steps_out,
                 void* ws, size_t ws_bytes, void* stream) {
    if (!ctx || !m) return fail(FDL_EINVAL, "generate: ctx or model is NULL");
    if (!prompt || !out_x || !steps_out) return fail(FDL_EINVAL, "generate: NULL buffer");
    if (b < 1 || B < 1 || B > 128 || P < 0 || gen < B || P % B || gen % B)
        return fail(FDL_EINVAL, "generate: need batch >= 1, 1 <= block <= 128, prompt_len and "
                    "gen_len (>= block) multiples of block");
    if (!(tau >= 0.f && tau <= 1.f)) return fail(FDL_EINVAL, "generate: tau must be in [0, 1]");
    GenRun r;
    r.ctx = ctx;
    r.m = m;
    r.b = b;
    r.P = P;
    r.gen = gen;
    r.B = B;
    r.tau = tau;
    r.mode = opts ? opts->cache : FDL_CACHE_DUAL;
    const bool device_loop = opts && opts->device_loop;
    const int batching = opts ? opts->batching : FDL_BATCH_LOCKSTEP;
    const bool compact = batching == FDL_BATCH_COMPACT;
    const bool per_seq = batching == FDL_BATCH_PER_SEQUENCE;
    if (batching != FDL_BATCH_LOCKSTEP && !compact && !per_seq)
        return fail(FDL_EINVAL, "generate: unknown batching %d", batching);
    if (r.mode != FDL_CACHE_DUAL && r.mode != FDL_CACHE_PREFIX && r.mode != FDL_CACHE_NONE)
        return fail(FDL_EINVAL, "generate: unknown cache mode %d", r.mode);
    r.bias_tok = opts ? opts->bias_tok : nullptr;
    r.bias_val = opts ? opts->bias_val : nullptr;
    if ((r.bias_tok == nullptr) != (r.bias_val == nullptr))
        return fail(FDL_EINVAL, "generate: bias_tok and bias_val go together");
    if ((compact || per_seq) && (device_loop || r.mode != FDL_CACHE_DUAL))
        return fail(FDL_EINVAL, "generate: compacted or per-sequence batching needs the "
                    "DualCache mode and the host loop");
    const fdl_model_desc& d = m->d;
    r.L = P + gen;
    if (r.L % 32)   // the refresh's full attention takes query blocks of 32 rows
        return fail(FDL_EINVAL, "generate: prompt_len + gen_len must be a multiple of 32");
    if (r.mode == FDL_CACHE_PREFIX && (P % 32 || B % 32))
        return fail(FDL_EINVAL, "generate: the PrefixCache mode needs the block starts at "
                    "multiples of 32 (prompt_len and block)");
    const int rf = b * r.L, rb = b * B;
    r.g = gen_layout(d, b, r.L, B, lm_ws_bytes(ctx, d, rb));
    if (!ws || ws_bytes < r.g.total)
        return fail(FDL_EWORKSPACE, "generate: workspace of %zu bytes needed", r.g.total);
    if (((uintptr_t)ws & 255u) != 0) return fail(FDL_EINVAL, "generate: ws must be 256-byte aligned");
    r.base = static_cast<char*>(ws);
    DeviceGuard guard(ctx->device);
    if (!guard.ok) return fail(FDL_ECUDA, "generate: cannot select device");
    cudaStream_t st = (cudaStream_t)stream;
    int32_t* x = r.x();
    const int nblk = (r.L + B - 1) / B;

    // state: x = prompts then mask ids, masked = the generated positions
    cudaError_t e = cudaSuccess;
    fill_i32_kernel<<<148, 256, 0, st>>>(x, (size_t)rf, d.mask_id);
    if (e == cudaSuccess && P > 0)
        e = cudaMemcpy2DAsync(x, (size_t)r.L * 4, prompt, (size_t)P * 4, (size_t)P * 4, b,
                              cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(r.masked(), 0, (size_t)rf, st);
    if (e == cudaSuccess)
        e = cudaMemset2DAsync(r.masked() + P, (size_t)r.L, 1, (size_t)gen, b, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(r.at(r.g.steps), 0, 16, st);
    block_rows_kernel<<<64, 256, 0, st>>>(r.maps(), b, r.L, B, nblk);
    if (e == cudaSuccess) e = cudaGetLastError();
    {
        std::vector<float> host_rope((size_t)r.L * 128);
        int rc = fdl_rope_table((double)d.rope_theta, r.L, 128, host_rope.data());
        if (rc) return rc;
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(r.at(r.g.rope), host_rope.data(), host_rope.size() * 4,
                                cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);   // host_rope goes out of scope
    }
    if (e != cudaSuccess) return cuda_fail(e, "generate: set-up");

    int steps = 0;
    if (device_loop) {
        int rc = run_device_loop(r, st);
        if (rc) return rc;
        int32_t dev_steps = 0;
        e = cudaMemcpyAsync(&dev_steps, r.at(r.g.steps), 4, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "generate: step count");
        steps = dev_steps;
    } else if (per_seq) {
        // Every sequence moves to its next block as soon as its own block is
        // decoded: a step refreshes the sequences that have just moved on
        // (their forward also decodes the first step of the new block) and
        // takes one DualCache step of the others, each at its own block.
        const int nblk_gen = gen / B;
        std::vector<int32_t> host_rem(b), blk(b, 0), state(b, 0);   // 0 refresh, 1 cached, 2 done
        std::vector<int32_t> up;
        for (;;) {
            int stepped = 0;
            for (int kind = 0; kind < 2; ++kind) {
                up.assign((size_t)2 * b, 0);
                int n = 0;
                for (int i = 0; i < b; ++i)
                    if (state[i] == kind) {
                        up[n] = i;
                        up[b + n] = P + blk[i] * B;
                        ++n;
                    }
                if (n == 0) continue;
                // token rows embedded: every position (refresh) or the block's
                for (int k = 0; k < n; ++k) {
                    const int i = up[k], s = up[b + k];
                    if (kind == 0)
                        for (int j = 0; j < r.L; ++j) up.push_back(i * r.L + j);
                    else
                        for (int j = 0; j < B; ++j) up.push_back(i * r.L + s + j);
                }
                if (kind == 0) {   // the new blocks' rows among the forward's rows
                    up.resize((size_t)2 * b + (size_t)b * r.L, 0);
                    for (int k = 0; k < n; ++k)
                        for (int j = 0; j < B; ++j) up.push_back(k * r.L + up[b + k] + j);
                }
                int rc = r.ps_upload(up, n, st);
                if (!rc) rc = kind == 0 ? r.ps_refresh(n, st) : r.ps_cached(n, st);
                if (rc) return rc;
                stepped += n;
            }
            if (stepped == 0) break;
            ++steps;
            e = cudaMemcpyAsync(host_rem.data(), r.remaining(), (size_t)b * 4,
                                cudaMemcpyDeviceToHost, st);
            if (e == cudaSuccess) e = cudaStreamSynchronize(st);
            if (e != cudaSuccess) return cuda_fail(e, "generate: counters");
            for (int i = 0; i < b; ++i) {
                if (state[i] == 2 || host_rem[i] > 0) {
                    if (state[i] == 0) state[i] = 1;
                    continue;
                }
                state[i] = ++blk[i] < nblk_gen ? 0 : 2;
            }
        }
    } else {
        std::vector<int32_t> host_rem(b);
        for (int blk = 0; blk < gen / B; ++blk) {
            int rc = r.block_prep(blk, st);
            if (rc) return rc;
            int n_act = b;              // sequences with masked positions left in the block
            for (bool first = true;; first = false) {
                rc = !first && compact && n_act < b ? r.compact_step(blk, n_act, st)
                                                    : r.step(blk, first, st);
                if (rc) return rc;
                ++steps;
                e = cudaMemcpyAsync(host_rem.data(), r.remaining(), (size_t)b * 4,
                                    cudaMemcpyDeviceToHost, st);
                if (e == cudaSuccess) e = cudaStreamSynchronize(st);
                if (e != cudaSuccess) return cuda_fail(e, "generate: counters");
                n_act = 0;
                for (int i = 0; i < b; ++i) n_act += host_rem[i] > 0;
                if (n_act == 0) break;
            }
        }
    }
    e = cudaMemcpyAsync(out_x, x, (size_t)rf * 4, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "generate: output");
    *steps_out = steps;
    return FDL_OK;
}

}  // extern "C"
