// Transformer GEMMs of the block step and of the refresh forward, bf16 on
// tcgen05 with fused epilogues:  C[M, N] = A[M, K] . W[N, K]^T  (both K-major)
//
//   EpiQKV    the block's (or, at a refresh, every position's) q/k/v
//             projection (Fast-dLLM DualCache: only the current block is
//             recomputed at a cached step; aibase news "Innovations" 1):
//             optional bias, rotary embedding of q and k at each row's
//             absolute position, q to [rows, Hq, d], k and v written in place
//             into the head-major caches [b, Hkv, L, d]
//   EpiResid  h[M, N] += C (f32 residual stream): attention output and FFN
//             down projections
//   EpiSwiGLU out[M, N/2] = silu(C[:, 2f]) * C[:, 2f+1] (bf16), with the gate
//             and up weight rows stored interleaved (row 2f = gate f, 2f+1 =
//             up f), so a tile holds both halves of its features
//
// Same persistent, warp-specialised structure as the LM-head kernel: warp 0
// TMA producer (4-stage ring, 128-byte swizzle), warp 1 TMEM owner and
// single-thread tcgen05.mma issuer (M=128, N=256, K=16) into two 256-column
// accumulators, warps 2-5 the epilogue (thread = tile row). Work items are
// ordered vocab/N-tile-major so row tiles sharing a weight tile run together
// and the weight is read from HBM once. Rows past M are TMA zero-fill.
//
// Roofline: at the block step (M = 32 rows per sequence) the weight stream
// bounds it (N*K*2 bytes per call, HBM); at a refresh (M = b*L) the tensor
// pipe does (2*M*N*K flops).
#include "common.cuh"
#include "gemm.h"
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

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void tmem_ld32_f(uint32_t taddr, float* v) {
    sm100::tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(v));
}

// ---- epilogues: each processes one accumulator tile row [n0, n0 + BN) ---------
struct EpiResidOp {
    EpiResid p;
    __device__ void operator()(uint32_t tacc, int row, int M, int n0, int N) const {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            float v[32];
            tmem_ld32_f(tacc + c, v);
            sm100::tmem_wait_ld();
            if (row < M && n0 + c < N) {
                float* dst = p.h + (size_t)row * p.ldh + n0 + c;
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 o = *reinterpret_cast<float4*>(dst + j);
                    o.x += v[j]; o.y += v[j + 1]; o.z += v[j + 2]; o.w += v[j + 3];
                    *reinterpret_cast<float4*>(dst + j) = o;
                }
            }
        }
    }
};

struct EpiSwiGLUOp {
    EpiSwiGLU p;
    __device__ void operator()(uint32_t tacc, int row, int M, int n0, int N) const {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            float v[32];
            tmem_ld32_f(tacc + c, v);
            sm100::tmem_wait_ld();
            if (row < M && n0 + c < N) {
                uint32_t pk[8];
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const float g0 = v[2 * j], u0 = v[2 * j + 1];
                    const float g1 = v[2 * j + 2], u1 = v[2 * j + 3];
                    const float a0 = g0 / (1.f + __expf(-g0)) * u0;
                    const float a1 = g1 / (1.f + __expf(-g1)) * u1;
                    pk[j >> 1] = pack_bf16x2(a0, a1);
                }
                bf16* dst = p.out + (size_t)row * p.ldo + (n0 + c) / 2;
                *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4*>(dst + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }
};

struct EpiQKVOp {
    EpiQKV p;
    // one head (128 columns) at a time: q heads, then k heads, then v heads
    __device__ void operator()(uint32_t tacc, int row, int M, int n0, int N) const {
        constexpr int D = 128;
        const int nq = p.n_q_heads * D, nk = p.n_kv_heads * D;
        const int seq = row < M ? p.cache_seq(row / p.rows_per_seq) : 0;
        const int pos = (row < M ? p.pos0_of(row / p.rows_per_seq) : p.pos0) + row % p.rows_per_seq;
#pragma unroll 1
        for (int hc = 0; hc < BN; hc += D) {
            const int col = n0 + hc;
            float v[D];
#pragma unroll
            for (int c = 0; c < D; c += 32) tmem_ld32_f(tacc + hc + c, v + c);
            sm100::tmem_wait_ld();
            if (row >= M || col >= N) continue;
            if (p.bias) {
#pragma unroll
                for (int j = 0; j < D; ++j) v[j] += p.bias[col + j];
            }
            bf16* dst;
            if (col < nq + nk) {
                // rotate-half RoPE: (x_i, x_{i+64}) rotated by pos * theta^(-2i/128)
                const float2* cs = p.rope + (size_t)pos * (D / 2);
#pragma unroll
                for (int j = 0; j < D / 2; ++j) {
                    const float2 t = cs[j];             // (cos, sin)
                    const float a = v[j], b = v[j + D / 2];
                    v[j] = a * t.x - b * t.y;
                    v[j + D / 2] = a * t.y + b * t.x;
                }
                if (col < nq) {
                    dst = p.q + ((size_t)row * p.n_q_heads + col / D) * D;
                } else {
                    const int h = (col - nq) / D;
                    dst = p.k_cache + (((size_t)seq * p.n_kv_heads + h) * p.seq_len + pos) * D;
                }
            } else {
                const int h = (col - nq - nk) / D;
                dst = p.v_cache + (((size_t)seq * p.n_kv_heads + h) * p.seq_len + pos) * D;
            }
#pragma unroll
            for (int j = 0; j < D; j += 8)
                *reinterpret_cast<uint4*>(dst + j) =
                    make_uint4(pack_bf16x2(v[j], v[j + 1]), pack_bf16x2(v[j + 2], v[j + 3]),
                               pack_bf16x2(v[j + 4], v[j + 5]), pack_bf16x2(v[j + 6], v[j + 7]));
        }
    }
};

template <class Epi>
__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               int M, int N, int K, int num_m, int num_items, int* err, const Epi epi) {
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
    const int k_iters = K / BK;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < num_items; item += gridDim.x) {
                const int m_tile = item % num_m, n_tile = item / num_m;
                for (int k = 0; k < k_iters; ++k) {
                    if (!(ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, err))) break;
                    mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
                    tma_load_2d(sA(stage), &tmA, full_bar(stage), k * BK, m_tile * BM);
                    tma_load_2d(sB(stage), &tmB, full_bar(stage), k * BK, n_tile * BN);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            for (int s = 0; ok && s < STAGES; ++s) {
                ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, err);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
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
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_bf16(d_tmem, a0 + (uint64_t)(kk * 2), b0 + (uint64_t)(kk * 2), idesc,
                                  (k | kk) != 0);
                    umma_commit(empty_bar(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (ok) umma_commit(tfull_bar(acc));
            }
        }
    } else {
        const int q = warp & 3;
        const int r_in = q * 32 + lane;
        int it = 0;
        for (int item = blockIdx.x; item < num_items; item += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t aphase = (it >> 1) & 1;
            const int m_tile = item % num_m, n_tile = item / num_m;
            if (!mbar_wait_warp(tfull_bar(acc), aphase, abort_flag, err)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            epi(tacc, m_tile * BM + r_in, M, n_tile * BN, N);
            tc_fence_before();
            mbar_arrive(tempty_bar(acc));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <class Epi>
cudaError_t run_gemm(const GemmShape& g, const void* a, const void* w, const Epi& epi,
                     int sm_count, int* err, cudaStream_t st) {
    CUtensorMap ta, tb;
    cudaError_t e = make_tmap_bf16_2d(&ta, a, g.M, g.K, BM, BK);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_2d(&tb, w, g.N, g.K, BN, BK);
    if (e != cudaSuccess) return e;
    const int num_m = (g.M + BM - 1) / BM;
    const int num_n = (g.N + BN - 1) / BN;
    const int items = num_m * num_n;
    const int grid = items < sm_count ? items : sm_count;
    e = cudaFuncSetAttribute(gemm_tc_kernel<Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(gemm_tc_kernel<Epi>, dim3(grid), dim3(THREADS), SMEM_BYTES, st, 0, ta, tb,
                      g.M, g.N, g.K, num_m, items, err, epi);
}

}  // namespace

cudaError_t launch_gemm_resid(const GemmShape& g, const void* a, const void* w,
                              const EpiResid& p, int sm_count, int* err, cudaStream_t st) {
    return run_gemm(g, a, w, EpiResidOp{p}, sm_count, err, st);
}

cudaError_t launch_gemm_swiglu(const GemmShape& g, const void* a, const void* w,
                               const EpiSwiGLU& p, int sm_count, int* err, cudaStream_t st) {
    return run_gemm(g, a, w, EpiSwiGLUOp{p}, sm_count, err, st);
}

cudaError_t launch_gemm_qkv(const GemmShape& g, const void* a, const void* w, const EpiQKV& p,
                            int sm_count, int* err, cudaStream_t st) {
    return run_gemm(g, a, w, EpiQKVOp{p}, sm_count, err, st);
}

}  // namespace fdl
