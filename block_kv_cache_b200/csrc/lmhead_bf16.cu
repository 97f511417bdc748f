// LM head fused with the vocabulary-wide confidence reduction, bf16 on the
// 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Fast-dLLM, confidence-aware parallel decoding (abstract; README "Key
// techniques" 2): a masked row's confidence is the probability of its
// predicted token, exp(max z - logsumexp z); the token is the argmax. The
// [M, V] logits are reduced in the epilogue and never reach memory.
//
// Persistent, warp-specialised kernel. A work item is one (row tile of 128,
// vocab tile of 256) pair; items are ordered vocab-tile-major so the row
// tiles that share a weight tile run at about the same time and the weight
// tile is read from HBM once and from L2 afterwards.
//   warp 0      TMA producer: h tile [128 x 64] and W tile [256 x 64] per
//               K-step into a 4-stage shared-memory ring (128-byte swizzle)
//   warp 1      TMEM owner and MMA issuer (one thread): 4 x tcgen05.mma
//               (M=128, N=256, K=16) per K-step into one of two 256-column
//               f32 accumulators, so the epilogue of item i overlaps the
//               mainloop of item i+1
//   warps 2..5  epilogue: thread = tile row; tcgen05.ld 32 columns at a time,
//               planted bias, running (max, sum exp, lowest argmax), one
//               12-byte partial per (row, vocab tile)
// A second tiny kernel merges the partials of each row (lmhead_combine.cu).
//
// Roofline: weight bytes V*D*2 are read once (1.036 GB at 126464 x 4096);
// 2*M*D*V flops. At M <= ~256 rows the kernel is bound by HBM, above by the
// tensor pipe. Row tiles are padded to 128 by TMA zero fill (no memory read).
#include "lmhead_common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace fdl {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
constexpr float LOG2E = 1.4426950408889634f;

__global__ void __launch_bounds__(THREADS, 1)
lmhead_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const int32_t* __restrict__ bias_tok, const float* __restrict__ bias_val,
                 LMPartial* __restrict__ part, int M, int D, int V, int num_m, int num_items,
                 int* err) {
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto full_bar = [&](int s) { return smem_u32(bars + s); };
    auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
    auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * STAGES + 2 + a); };
    auto sA = [&](int s) { return sbase + s * STAGE_BYTES; };
    auto sB = [&](int s) { return sbase + s * STAGE_BYTES + A_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 128);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_wait();
    pdl_trigger();
    const uint32_t tmem_base = *tmem_slot;
    const int k_iters = D / BK;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int issued = 0;                              // loads requested (load u: stage u % STAGES)
            const uint64_t w_policy = l2_evict_first();
            for (int item = blockIdx.x; ok && item < num_items; item += gridDim.x) {
                const int m_tile = item % num_m, n_tile = item / num_m;
                for (int k = 0; k < k_iters; ++k) {
                    if (!(ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, err))) break;
                    mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
                    tma_load_2d(sA(stage), &tmA, full_bar(stage), k * BK, m_tile * BM);
                    if (num_m == 1)                      // the vocabulary matrix is read once
                        tma_load_2d_hint(sB(stage), &tmB, full_bar(stage), k * BK, n_tile * BN,
                                         w_policy);
                    else
                        tma_load_2d(sB(stage), &tmB, full_bar(stage), k * BK, n_tile * BN);
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            // tail: every stage handed to the MMA has been released again, so
            // no tcgen05.commit arrival is still on its way to this CTA's smem
            for (int s = 0; ok && s < STAGES; ++s) {
                ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, err);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) {
                // gave up: the loads still in flight (at most one per stage, the
                // last STAGES requested) land before the CTA may leave
                for (int u = issued > STAGES ? issued - STAGES : 0; u < issued; ++u)
                    mbar_wait_drain(full_bar(u % STAGES), (uint32_t)((u / STAGES) & 1), err);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
            int consumed = 0;                            // stages committed back (u: stage u % STAGES)
            int tcommits = 0;                            // accumulators committed (i: acc i & 1)
            for (int item = blockIdx.x; ok && item < num_items; item += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t aphase = (it >> 1) & 1;
                if (!(ok = mbar_wait(tempty_bar(acc), aphase ^ 1, abort_flag, err))) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int k = 0; k < k_iters; ++k) {
                    if (!(ok = mbar_wait(full_bar(stage), phase, abort_flag, err))) break;
                    tc_fence_after();
                    const uint64_t a0 = umma_desc_sw128(sA(stage));
                    const uint64_t b0 = umma_desc_sw128(sB(stage));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // +32 bytes per K=16 step inside the 128-byte swizzle atom
                        umma_bf16(d_tmem, a0 + (uint64_t)(kk * 2), b0 + (uint64_t)(kk * 2), idesc,
                                  (k | kk) != 0);
                    }
                    umma_commit(empty_bar(stage));
                    ++consumed;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (ok) {
                    umma_commit(tfull_bar(acc));
                    ++tcommits;
                }
            }
            if (!ok) {
                // gave up: every MMA issued is followed by a commit on its stage's
                // empty barrier (at most one outstanding per stage, the last
                // STAGES) and each finished item by one on its accumulator's full
                // barrier (at most the last two): once those arrivals have
                // landed, no MMA writes TMEM and no arrival is on its way here
                for (int u = consumed > STAGES ? consumed - STAGES : 0; u < consumed; ++u)
                    mbar_wait_drain(empty_bar(u % STAGES), (uint32_t)((u / STAGES) & 1), err);
                for (int i = tcommits > 2 ? tcommits - 2 : 0; i < tcommits; ++i)
                    mbar_wait_drain(tfull_bar(i & 1), (uint32_t)((i >> 1) & 1), err);
            }
        }
    } else {
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int r_in = q * 32 + lane;
        int it = 0;
        for (int item = blockIdx.x; item < num_items; item += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t aphase = (it >> 1) & 1;
            const int m_tile = item % num_m, n_tile = item / num_m;
            const int row = m_tile * BM + r_in;
            const int n0 = n_tile * BN;
            if (!mbar_wait_warp(tfull_bar(acc), aphase, abort_flag, err)) break;
            tc_fence_after();
            int bt = -1;
            float bv = 0.f;
            if (bias_tok != nullptr && row < M) {
                bt = bias_tok[row];
                bv = bias_val[row];
            }
            float mx = -INFINITY, se = 0.f;
            int arg = INT_MAX;
            const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(t0 + c * 32, r);
                tmem_wait_ld();
                const int cbase = n0 + c * 32;
                float z[32];
                float cm = -INFINITY;
                int ca = INT_MAX;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float v = __uint_as_float(r[j]);
                    if (cbase + j == bt) v += bv;
                    if (cbase + j >= V) v = -INFINITY;
                    z[j] = v;
                    if (v > cm) { cm = v; ca = cbase + j; }
                }
                if (cm > mx) {
                    se *= exp2f((mx - cm) * LOG2E);
                    mx = cm;
                    arg = ca;
                }
                const float mxl = mx * LOG2E;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    se += (z[j] == -INFINITY) ? 0.f : exp2f(fmaf(z[j], LOG2E, -mxl));
            }
            tc_fence_before();
            mbar_arrive(tempty_bar(acc));
            if (row < M) part[(size_t)n_tile * M + row] = LMPartial{mx, se, arg};
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace

size_t lmhead_workspace_bytes(const LMShape& s) {
    // per-128-column partials of the f32 path bound the 256-column ones here
    const size_t tiles = (s.vocab + 127) / 128;
    return tiles * (size_t)s.rows * sizeof(LMPartial);
}

cudaError_t launch_lmhead_bf16(const LMShape& s, const void* h, const void* w,
                               const int32_t* bias_tok, const float* bias_val, float* conf,
                               int32_t* tok, void* ws, int sm_count, int* dev_err,
                               cudaStream_t st) {
    CUtensorMap ta, tb;
    cudaError_t e = make_tmap_bf16_2d(&ta, h, s.rows, s.hidden, BM, BK);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_2d(&tb, w, s.vocab, s.hidden, BN, BK);
    if (e != cudaSuccess) return e;
    const int num_m = (s.rows + BM - 1) / BM;
    const int num_n = (s.vocab + BN - 1) / BN;
    const int items = num_m * num_n;
    const int grid = items < sm_count ? items : sm_count;
    e = cudaFuncSetAttribute(lmhead_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    LMPartial* part = (LMPartial*)ws;
    e = launch_pdl(lmhead_tc_kernel, dim3(grid), dim3(THREADS), SMEM_BYTES, st, 0, ta, tb,
                   bias_tok, bias_val, part, s.rows, s.hidden, s.vocab, num_m, items, dev_err);
    if (e != cudaSuccess) return e;
    return launch_lmhead_combine(part, num_n, s.rows, conf, tok, st);
}

}  // namespace fdl
