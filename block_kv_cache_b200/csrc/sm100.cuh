// sm_100a building blocks written as inline PTX: mbarriers with bounded
// waits, TMA tile loads, TMEM allocation, tcgen05 MMA (bf16 -> f32) and
// TMEM loads. Host side: tensor-map encoding through the driver entry point.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace fdl {
namespace sm100 {

// A wait that has not completed after this long gives up and records
// DEV_TIMEOUT; a correct launch of any kernel here finishes in milliseconds.
// This is the default of the per-context limit of the progress waits (below)
// and the fixed limit of the drain waits that follow a give-up.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

// The limit of the progress waits of a context: the 64-bit word 8 bytes after
// the context's 4-byte device error word (set by fdl_create to kWaitTimeoutNs
// and changed by fdl_set_wait_timeout). Read when a wait starts its clock.
__device__ __forceinline__ uint64_t wait_limit_ns(const int* err) {
    if (!err) return kWaitTimeoutNs;
    // constant while a kernel runs (set with the device idle): read through the
    // non-coherent cache, a hit in L1 after the first read on an SM
    return __ldg(reinterpret_cast<const unsigned long long*>(
        reinterpret_cast<const char*>(err) + 8));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Orders this thread's generic-proxy global accesses with later async-proxy
// (TMA) accesses to global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Non-blocking: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Poll budget of a producer loop that waits on several barriers at once:
// returns false (after raising *abort and recording DEV_TIMEOUT) once it has
// found nothing to do for longer than the timeout, or when another thread has
// given up. Call reset() whenever the loop made progress.
struct PollBudget {
    uint32_t n = 0;
    uint64_t t0 = 0;
    uint64_t limit = 0;
    __device__ __forceinline__ void reset() { n = 0; t0 = 0; }
    __device__ __forceinline__ bool idle(volatile int* abort, int* err) {
        if ((++n & 63u) != 0) return true;
        if (*abort) return false;
        const uint64_t now = globaltimer();
        if (t0 == 0) {
            t0 = now;
            limit = wait_limit_ns(err);
        } else if (now - t0 > limit) {
            *abort = 1;
            record_error(err, DEV_TIMEOUT);
            return false;
        }
        return true;
    }
};

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete. Returns false
// (after raising *abort and recording DEV_TIMEOUT) if it does not complete in
// time, or at once if another thread of the CTA has already given up.
// The clock and the abort flag are consulted only every 64 polls, so a wait
// that completes soon costs no more than the try_wait itself.
// The clock starts at the first unsuccessful poll; with the default limit it
// is read every 64 polls, with a limit under 1 ms (a shortened limit, set to
// make waits run out) at every poll, so that a short wait can run out too.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    const uint64_t limit = wait_limit_ns(err);
    const uint32_t every = limit < 1000000ull ? 0u : 63u;
    uint32_t n = 0;
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((++n & every) == 0) {
            if (*abort) return false;
            if (globaltimer() - t0 > limit) {
                *abort = 1;
                record_error(err, DEV_TIMEOUT);
                return false;
            }
        }
    }
}

// Wait of the give-up path: for an asynchronous operation this thread (or a
// copy it requested) has already started and that completes by itself (a TMA
// load landing, a tcgen05 commit arriving), so that nothing is still on its
// way into the CTA's shared memory or TMEM when the CTA leaves. Ignores the
// abort flag and has the fixed limit kWaitTimeoutNs (records DEV_TIMEOUT and
// returns false if even that runs out).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, int* err) {
    uint32_t n = 0;
    uint64_t t0 = 0;
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((++n & 63u) == 0) {
            const uint64_t now = globaltimer();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kWaitTimeoutNs) {
                record_error(err, DEV_TIMEOUT);
                return false;
            }
        }
    }
}

// Whole-warp wait: every lane polls the barrier, then the warp agrees on the
// outcome (all lanes leave together, also on the give-up path).
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile int* abort, int* err) {
    const bool ok = mbar_wait(bar, parity, abort, err);
    return __all_sync(0xffffffffu, ok);
}

// Barrier over every CTA of the grid. Only for grids whose CTAs are all
// resident at once (persistent grids of at most one CTA per SM, launched when
// nothing else can hold an SM indefinitely). The two words at bar hold one
// 64-bit arrival counter (8-byte aligned, zero at first use) that only grows:
// one barrier adds exactly kBarrierQuantum to it whatever the grid size (CTA 0
// adds the quantum less the other CTAs' ones), so a CTA that arrives at count
// c leaves once the count reaches the next multiple of the quantum above c.
// One release add and acquire polls: no reset, no second word, no full
// fences. Bounded: a CTA that waits longer than the timeout raises *abort,
// records DEV_TIMEOUT and returns false; afterwards the counter is no longer
// at a multiple of the quantum, so the caller's context has to be recreated.
constexpr unsigned long long kBarrierQuantum = 1ull << 20;   // > any grid size

__device__ __forceinline__ unsigned long long atom_add_release_gpu(unsigned long long* p,
                                                                   unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.release.gpu.global.add.u64 %0, [%1], %2;"
                 : "=l"(old)
                 : "l"(p), "l"(v)
                 : "memory");
    return old;
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ bool grid_barrier(unsigned* bar, volatile int* abort, int* err) {
    __syncthreads();                                 // the CTA's writes precede the release
    if (threadIdx.x == 0) {
        unsigned long long* cnt = reinterpret_cast<unsigned long long*>(bar);
        const unsigned long long nb = (unsigned long long)gridDim.x * gridDim.y * gridDim.z;
        const bool first = (blockIdx.x | blockIdx.y | blockIdx.z) == 0;
        const unsigned long long old =
            atom_add_release_gpu(cnt, first ? kBarrierQuantum - (nb - 1) : 1ull);
        const unsigned long long target = (old / kBarrierQuantum + 1) * kBarrierQuantum;
        uint32_t n = 0;
        uint64_t t0 = 0, limit = 0;
        while (ld_acquire_gpu(cnt) < target) {
            if ((++n & 63u) == 0) {
                const uint64_t now = globaltimer();
                if (t0 == 0) {
                    t0 = now;
                    limit = wait_limit_ns(err);
                } else if (now - t0 > limit) {
                    *abort = 1;
                    record_error(err, DEV_TIMEOUT);
                    break;
                }
            }
        }
    }
    __syncthreads();
    return *abort == 0;
}

// 2-D TMA tile load global -> shared, completion counted on `bar` in bytes.
// c0 is the innermost (contiguous) coordinate in elements; c0 * elem_size must
// be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// 3-D TMA tile load (c0 innermost).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// L2 policy for data read once per pass (weights, K/V caches streamed past a
// handful of rows): such lines are the first to be evicted, so a stream far
// larger than L2 does not push out the small tensors that the next kernels
// read back (split-K sums, the residual stream, activations).
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// tma_load_2d with an L2 cache policy (l2_evict_first()).
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int c0, int c1, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

// tma_load_3d with an L2 cache policy (l2_evict_first()).
__device__ __forceinline__ void tma_load_3d_hint(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int c0, int c1, int c2,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- TMEM ------------------------------------------------------------------
// Executed by one full warp. Writes the allocated base address to *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     slot_smem),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- UMMA descriptors --------------------------------------------------------
// Shared-memory matrix descriptor for a K-major tile written by TMA with
// 128-byte swizzle: rows of 64 bf16 (128 B), 8-row groups 1024 B apart.
// Fields: start address >> 4 (bits 0-13), leading byte offset >> 4 (16-29,
// unused for swizzled K-major, 1), stride byte offset >> 4 (32-45) = 1024 B,
// version 1 (46-47), base offset 0 (49-51), layout SWIZZLE_128B = 2 (61-63).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Shared-memory descriptor for an MN-major operand tile written by TMA with
// 128-byte swizzle: each K index is a 128-byte row of 64 consecutive MN
// elements, 8 K-rows form a 1024-byte atom (stride byte offset), and the next
// 64 MN elements start `mn_chunk_bytes` further on (leading byte offset).
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t smem_addr,
                                                       uint32_t mn_chunk_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((mn_chunk_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor, kind::f16: f32 accumulator, bf16 A and B, shape
// M x N; A K-major; B K-major unless b_mn_major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N, bool b_mn_major = false) {
    return (1u << 4)                       // D format f32
           | (1u << 7)                     // A format bf16
           | (1u << 10)                    // B format bf16
           | ((b_mn_major ? 1u : 0u) << 16)  // B major-ness
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by a single thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05.mma of this thread
// have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// lane (base lane + t), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- thread-block clusters --------------------------------------------------------
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// Address in the shared::cluster window of `smem_addr` of CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// Split cluster barrier: every thread of every CTA of the cluster arrives
// once and later waits once (not necessarily warp-converged).
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

// Store to (possibly another CTA's) shared memory at a shared::cluster address,
// counted in bytes on the mbarrier at `bar` (a shared::cluster address in the
// same CTA as `addr`), which completes its phase once the expected bytes have
// all landed.
__device__ __forceinline__ void st_async_f4(uint32_t addr, float4 v, uint32_t bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, "
        "[%5];" ::"r"(addr),
        "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void st_async_f2(uint32_t addr, float2 v, uint32_t bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
            addr),
        "f"(v.x), "f"(v.y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ float2 ld_cluster_f2(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
    return v;
}

}  // namespace sm100

// ---- host: tensor maps ---------------------------------------------------------
// 2-D bf16 tensor map over a row-major [rows, cols] matrix (cols contiguous),
// box = box_rows x box_cols with 128-byte swizzle (box_cols * 2 must be 128).
// Returns cudaSuccess or the error of the driver call.
cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t box_rows, uint32_t box_cols);

// Tensor map over a row-major [rows, cols] bf16 matrix (cols % 64 == 0) whose
// box is box_rows rows x (n_chunks * 64) columns, delivered as n_chunks
// consecutive [box_rows][64] sub-tiles of 128-byte rows (128-byte swizzle):
// the K-major operand layout of the MMAs, fetched with one copy instead of
// one per 64 columns. Copy coordinates: (0, row, first chunk).
cudaError_t make_tmap_bf16_rows(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                uint32_t box_rows, uint32_t n_chunks);

// General rank-2..5 bf16 tensor map, 128-byte swizzle: dims[0] is the
// contiguous dimension (box[0] must be 64 elements = 128 bytes);
// strides_bytes[i] is the byte stride of dimension i+1 (multiple of 16).
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box);

}  // namespace fdl
