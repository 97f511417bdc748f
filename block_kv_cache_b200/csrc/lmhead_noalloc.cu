// fdl_lmhead_confidence_noalloc: the LM-head confidence call without a
// caller-provided workspace.
//
// Some callers cannot hand this library a scratch buffer: plain C hosts that
// only own the input and output tensors, and engines whose device memory is
// entirely held by their own pool, where an extra cudaMalloc would fail or
// would force the device-wide synchronisation that cudaMalloc and cudaFree
// can cause. For them this entry point keeps its scratch (the per-tile
// partial maxima, sums and arguments of the vocabulary reduction) in a
// fixed-size array in the library's own device memory. The array is part of
// the loaded module, so every GPU that loads the library holds its 8 MiB
// until the process exits; the entry point itself allocates nothing.
#include <stdio.h>

#include <mutex>

#include "fdllm.h"
#include "launch.h"
#include "lmhead_common.cuh"

namespace fdl {
int ctx_device(const fdl_ctx* ctx);
int report_error(int code, const char* msg);
}

namespace {

constexpr size_t kScratchBytes = 8u << 20;     // 8 MiB
constexpr int kMaxDevices = 64;

// Shared by every call on a device: each call overwrites the part it uses.
static __device__ __align__(256) unsigned char g_lmhead_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_lmhead_scratch on `dev`, looked up once per device with
// that device current (in host code the symbol names a host-side stand-in, not
// device memory, so it must never be passed to a kernel directly).
cudaError_t scratch_address(int dev, void** out) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_addr[dev]) {
        *out = g_scratch_addr[dev];
        return cudaSuccess;
    }
    int prev = -1;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess) return e;
    if (prev != dev && (e = cudaSetDevice(dev)) != cudaSuccess) return e;
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lmhead_scratch);
    if (prev != dev) cudaSetDevice(prev);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
    *out = p;
    return cudaSuccess;
}

}  // namespace

namespace fdl {
// Drop the cached address of `dev` (called by fdl_create): after a device
// reset the module is loaded again and the array may sit elsewhere, and any
// context used after a reset is a new one.
void noalloc_forget(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return;
    std::lock_guard<std::mutex> lk(g_mu);
    g_scratch_addr[dev] = nullptr;
}
}  // namespace fdl

extern "C" FDL_API int fdl_lmhead_confidence_noalloc(fdl_ctx* ctx, const fdl_lmhead_desc* desc,
                                                     const void* h, const void* w,
                                                     const int32_t* bias_tok,
                                                     const float* bias_val, float* conf,
                                                     int32_t* tok, void* stream) {
    if (!ctx) return fdl_lmhead_confidence(ctx, desc, h, w, bias_tok, bias_val, conf, tok,
                                           nullptr, 0, stream);
    const size_t need = fdl_lmhead_workspace_bytes(ctx, desc);
    if (need == 0)   // invalid descriptor: let the regular entry point report it
        return fdl_lmhead_confidence(ctx, desc, h, w, bias_tok, bias_val, conf, tok, nullptr, 0,
                                     stream);
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "lmhead_noalloc: this shape needs %zu bytes of scratch, more than the built-in "
                 "%zu; call fdl_lmhead_confidence with a workspace instead", need, kScratchBytes);
        return fdl::report_error(FDL_EINVAL, msg);
    }
    const int dev = fdl::ctx_device(ctx);
    if (dev < 0 || dev >= kMaxDevices)
        return fdl::report_error(FDL_EUNSUPPORTED, "lmhead_noalloc: device id above 63");
    void* ws = nullptr;
    const cudaError_t e = scratch_address(dev, &ws);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "lmhead_noalloc: cudaGetSymbolAddress: %s",
                 cudaGetErrorString(e));
        return fdl::report_error(FDL_ECUDA, msg);
    }
    return fdl_lmhead_confidence(ctx, desc, h, w, bias_tok, bias_val, conf, tok, ws,
                                 kScratchBytes, stream);
}
