// DualCache block attention, bf16, on the 5th-generation tensor cores.
//
// Fast-dLLM, DualCache (aibase news "Innovations" 1; README "Key techniques"
// 1): the block's queries attend, without a mask, over the whole cache
// [prefix | block slot | masked suffix]; the block slot holds fresh K/V.
//
// One CTA = one key tile of KT keys of one (sequence, kv head, head chunk).
// All query heads that share the kv head (GQA group, or a chunk of it) are
// packed into the MMA's M dimension, so each K/V tile is read from HBM once
// per group: rows r = i * hc + j hold query i of head (chunk*hc + j).
//   warp 4 (one thread): TMA loads of Q (3-D box: d x heads x queries), K and
//          V tiles (128-byte swizzle); tcgen05.mma S = Q K^T into TMEM
//          (M=128 per row tile, N=KT, K=d); after the softmax, O = P V with V
//          as an MN-major operand (N=d, K=KT)
//   warps 0-3: thread = query row: read S from TMEM, softmax in the log2
//          domain (scale * log2 e folded in), P as bf16 into shared memory in
//          the swizzled K-major layout the MMA reads, then O from TMEM to
//          the split-KV workspace with the row's (max, sum)
// A second kernel merges the splits (attention.cu, attn_combine_kernel).
//
// Roofline: HBM. Algorithmic bytes per call = K and V once (2*b*Hkv*L*d*2)
// + q and out (2*b*B*Hq*d*2); the MMAs run at ~30 flop per byte.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace fdl {

struct AttnPlan {
    int kt;        // keys per CTA
    int mt;        // 128-row tiles of packed queries (1 or 2)
    int hc;        // query heads packed per CTA
    int n_chunks;  // head chunks per kv head
    int n_splits;  // key tiles per (sequence, kv head)
};

AttnPlan attn_tc_plan(const AttnShape& s, int sm_count) {
    AttnPlan p;
    const int grp = s.n_q_heads / s.n_kv_heads;
    p.hc = 256 / s.block_len;
    if (p.hc > grp) p.hc = grp;
    if (p.hc < 1) p.hc = 1;
    p.n_chunks = (grp + p.hc - 1) / p.hc;
    p.mt = p.hc * s.block_len > 128 ? 2 : 1;
    const int units = s.batch * s.n_kv_heads * p.n_chunks;
    static const int kts1[] = {192, 128, 64}, kts2[] = {128, 64};
    const int* kts = p.mt == 1 ? kts1 : kts2;
    const int nk = p.mt == 1 ? 3 : 2;
    long best_waves = -1;
    p.kt = kts[0];
    for (int i = 0; i < nk; ++i) {
        const long ctas = (long)units * ((s.seq_len + kts[i] - 1) / kts[i]);
        const long waves = (ctas + sm_count - 1) / sm_count;
        if (best_waves < 0 || waves <= best_waves) {   // ties: the smaller tile, more CTAs
            best_waves = waves;
            p.kt = kts[i];
        }
    }
    p.n_splits = (s.seq_len + p.kt - 1) / p.kt;
    return p;
}

namespace {

constexpr int TC_THREADS = 160;

template <int D, int KT, int MT>
struct AttnSmem {
    static constexpr int DC = D / 64;                       // 64-wide d chunks
    static constexpr int Q_CHUNK = MT * 128 * 128;          // bytes per d chunk of Q
    static constexpr int Q_BYTES = DC * Q_CHUNK;
    static constexpr int KV_CHUNK = KT * 128;               // bytes per d chunk of K or V
    static constexpr int KV_BYTES = DC * KV_CHUNK;
    static constexpr int P_CHUNK = 128 * 128;               // 64 keys x 128 rows
    static constexpr int P_TILE = (KT / 64) * P_CHUNK;      // one 128-row tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + KV_BYTES;
    static constexpr int OFF_P = OFF_V + KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + MT * P_TILE;
    static constexpr size_t TOTAL = 1024 + OFF_BAR + 128;
    static constexpr uint32_t TMEM_S = 0;                    // S[mt] at mt*KT
    static constexpr uint32_t TMEM_O = MT * KT;              // O[mt] at MT*KT + mt*D
    static constexpr uint32_t TMEM_USED = MT * (KT + D);
    static constexpr uint32_t TMEM_ALLOC = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64
                                         : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert(TOTAL <= 227 * 1024, "shared memory budget");
};

template <int D, int KT, int MT>
__global__ void __launch_bounds__(TC_THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, float* __restrict__ ws_o,
               float* __restrict__ ws_ml, int B, int Hq, int Hkv, int L, int hc, int n_chunks,
               int n_splits, float scale_log2, int* err) {
    using namespace sm100;
    using S = AttnSmem<D, KT, MT>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sb = raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t bar_qk = smem_u32(bars + 0), bar_v = smem_u32(bars + 1);
    const uint32_t bar_s = smem_u32(bars + 2), bar_p = smem_u32(bars + 3);
    const uint32_t bar_o = smem_u32(bars + 4);

    const int split = blockIdx.x;
    const int g = blockIdx.y / n_chunks, chunk = blockIdx.y % n_chunks;
    const int bb = blockIdx.z;
    const int grp = Hq / Hkv;
    const int k0 = split * KT;
    const int nk = min(KT, L - k0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(bar_qk, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_p, 128);
        mbar_init(bar_o, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4) tmem_alloc(smem_u32(tmem_slot), S::TMEM_ALLOC);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            const int krow = (bb * Hkv + g) * L + k0;
            const int head0 = g * grp + chunk * hc;
            mbar_arrive_expect_tx(bar_qk, (uint32_t)(S::DC * hc * B * 128 + S::KV_BYTES));
            for (int c = 0; c < S::DC; ++c) {
                tma_load_3d(sb + S::OFF_Q + c * S::Q_CHUNK, &tmQ, bar_qk, c * 64, head0, bb * B);
                tma_load_2d(sb + S::OFF_K + c * S::KV_CHUNK, &tmK, bar_qk, c * 64, krow);
            }
            mbar_arrive_expect_tx(bar_v, (uint32_t)S::KV_BYTES);
            for (int c = 0; c < S::DC; ++c)
                tma_load_2d(sb + S::OFF_V + c * S::KV_CHUNK, &tmV, bar_v, c * 64, krow);

            bool ok = mbar_wait(bar_qk, 0, abort_flag, err);
            if (ok) {
                tc_fence_after();
                constexpr uint32_t idesc_s = umma_idesc_bf16_f32(128, KT);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t qa = sb + S::OFF_Q + (kk >> 2) * S::Q_CHUNK + m * 16384 +
                                            (kk & 3) * 32;
                        const uint32_t ka = sb + S::OFF_K + (kk >> 2) * S::KV_CHUNK + (kk & 3) * 32;
                        umma_bf16(tmem + S::TMEM_S + m * KT, umma_desc_sw128(qa),
                                  umma_desc_sw128(ka), idesc_s, kk > 0);
                    }
                }
                umma_commit(bar_s);
                ok = mbar_wait(bar_v, 0, abort_flag, err) && mbar_wait(bar_p, 0, abort_flag, err);
            }
            if (ok) {
                tc_fence_after();
                constexpr uint32_t idesc_o = umma_idesc_bf16_f32(128, D, true);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
#pragma unroll
                    for (int ks = 0; ks < KT / 16; ++ks) {
                        const uint32_t pa = sb + S::OFF_P + m * S::P_TILE + (ks >> 2) * S::P_CHUNK +
                                            (ks & 3) * 32;
                        const uint32_t va = sb + S::OFF_V + ks * 2048;
                        umma_bf16(tmem + S::TMEM_O + m * D, umma_desc_sw128(pa),
                                  umma_desc_sw128_mn(va, S::KV_CHUNK), idesc_o, ks > 0);
                    }
                }
                umma_commit(bar_o);
            }
        }
    } else {
        // softmax / epilogue warps: warp w reads TMEM lanes [32w, 32w+32)
        int ok = 1;
        if (lane == 0) ok = mbar_wait(bar_s, 0, abort_flag, err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        float mrow[MT], lrow[MT];
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint32_t tS = tmem + ((uint32_t)(warp * 32) << 16) + S::TMEM_S + m * KT;
                float mx = -INFINITY;
#pragma unroll 1
                for (int c = 0; c < KT / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tS + c * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c * 32 + j < nk) mx = fmaxf(mx, __uint_as_float(r[j]) * scale_log2);
                }
                float l = 0.f;
                const int row = warp * 32 + lane;                    // row within the tile
                uint8_t* prow = smem + S::OFF_P + m * S::P_TILE + row * 128;
#pragma unroll 1
                for (int c = 0; c < KT / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tS + c * 32, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const int key = c * 32 + j;
                        const float p0 = key < nk ? exp2f(fmaf(__uint_as_float(r[j]), scale_log2, -mx)) : 0.f;
                        const float p1 = key + 1 < nk ? exp2f(fmaf(__uint_as_float(r[j + 1]), scale_log2, -mx)) : 0.f;
                        l += p0 + p1;
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                        pk[j >> 1] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    // 32 keys = 4 pieces of 16 B in chunk (c/2), pieces 4*(c&1)..+3
                    uint8_t* pc = prow + (c >> 1) * S::P_CHUNK;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int piece = (c & 1) * 4 + q4;
                        const int phys = piece ^ (row & 7);
                        *reinterpret_cast<uint4*>(pc + phys * 16) =
                            make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                    }
                }
                mrow[m] = mx;
                lrow[m] = l;
            }
            fence_proxy_async();          // P (generic-proxy stores) -> MMA (async proxy)
            tc_fence_before();
            mbar_arrive(bar_p);
            if (lane == 0) ok = mbar_wait(bar_o, 0, abort_flag, err);
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int r = m * 128 + warp * 32 + lane;            // packed row
                const int i = r / hc, j = r % hc;
                const int head_in_grp = chunk * hc + j;
                const bool valid = i < B && head_in_grp < grp;
                const int head = g * grp + head_in_grp;
                const uint32_t tO = tmem + ((uint32_t)(warp * 32) << 16) + S::TMEM_O + m * D;
                const size_t prow = valid ? (((size_t)bb * Hq + head) * n_splits + split) * B + i : 0;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(tO + c * 32, rr);
                    tmem_wait_ld();
                    if (valid) {
                        float4* dst = reinterpret_cast<float4*>(ws_o + prow * D + c * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            dst[q4] = make_float4(__uint_as_float(rr[4 * q4]),
                                                  __uint_as_float(rr[4 * q4 + 1]),
                                                  __uint_as_float(rr[4 * q4 + 2]),
                                                  __uint_as_float(rr[4 * q4 + 3]));
                    }
                }
                if (valid) {
                    ws_ml[prow * 2 + 0] = mrow[m];
                    ws_ml[prow * 2 + 1] = lrow[m];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_ALLOC);
    }
}

template <int D, int KT, int MT>
cudaError_t run_tc(const AttnShape& s, const AttnPlan& p, const CUtensorMap& tq,
                   const CUtensorMap& tk, const CUtensorMap& tv, float* ws_o, float* ws_ml,
                   int* err, cudaStream_t st) {
    using S = AttnSmem<D, KT, MT>;
    auto kfn = attn_tc_kernel<D, KT, MT>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)S::TOTAL);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_splits, s.n_kv_heads * p.n_chunks, s.batch);
    kfn<<<grid, TC_THREADS, S::TOTAL, st>>>(tq, tk, tv, ws_o, ws_ml, s.block_len, s.n_q_heads,
                                            s.n_kv_heads, s.seq_len, p.hc, p.n_chunks,
                                            p.n_splits, s.scale * 1.4426950408889634f, err);
    return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_tc(const AttnShape& s, const AttnPlan& p, const CUtensorMap& tq,
                        const CUtensorMap& tk, const CUtensorMap& tv, float* ws_o, float* ws_ml,
                        int* err, cudaStream_t st) {
    if (p.mt == 1) {
        if (p.kt == 192) return run_tc<D, 192, 1>(s, p, tq, tk, tv, ws_o, ws_ml, err, st);
        if (p.kt == 128) return run_tc<D, 128, 1>(s, p, tq, tk, tv, ws_o, ws_ml, err, st);
        return run_tc<D, 64, 1>(s, p, tq, tk, tv, ws_o, ws_ml, err, st);
    }
    if (p.kt == 128) return run_tc<D, 128, 2>(s, p, tq, tk, tv, ws_o, ws_ml, err, st);
    return run_tc<D, 64, 2>(s, p, tq, tk, tv, ws_o, ws_ml, err, st);
}

}  // namespace

size_t attn_tc_workspace_bytes(const AttnShape& s, int sm_count) {
    const AttnPlan p = attn_tc_plan(s, sm_count);
    const size_t rows = (size_t)s.batch * s.n_q_heads * p.n_splits * s.block_len;
    return rows * (s.head_dim + 2) * sizeof(float);
}

cudaError_t launch_attn_combine_bf16(const float* ws_o, const float* ws_ml, void* out, float* lse,
                                     int batch, int B, int Hq, int D, int n_splits,
                                     cudaStream_t st);

cudaError_t launch_attention_bf16(const AttnShape& s, const void* q, const void* k,
                                  const void* v, void* out, float* lse, void* ws, int sm_count,
                                  int* err, cudaStream_t st) {
    const AttnPlan p = attn_tc_plan(s, sm_count);
    const int D = s.head_dim;
    CUtensorMap tq, tk, tv;
    const uint64_t qdims[3] = {(uint64_t)D, (uint64_t)s.n_q_heads,
                               (uint64_t)s.batch * s.block_len};
    const uint64_t qstr[2] = {(uint64_t)D * 2, (uint64_t)s.n_q_heads * D * 2};
    const uint32_t qbox[3] = {64, (uint32_t)p.hc, (uint32_t)s.block_len};
    cudaError_t e = make_tmap_bf16(&tq, q, 3, qdims, qstr, qbox);
    if (e != cudaSuccess) return e;
    const uint64_t kv_rows = (uint64_t)s.batch * s.n_kv_heads * s.seq_len;
    e = make_tmap_bf16_2d(&tk, k, kv_rows, D, p.kt, 64);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_2d(&tv, v, kv_rows, D, p.kt, 64);
    if (e != cudaSuccess) return e;
    float* ws_o = (float*)ws;
    const size_t rows = (size_t)s.batch * s.n_q_heads * p.n_splits * s.block_len;
    float* ws_ml = ws_o + rows * D;
    e = D == 128 ? dispatch_tc<128>(s, p, tq, tk, tv, ws_o, ws_ml, err, st)
                 : dispatch_tc<64>(s, p, tq, tk, tv, ws_o, ws_ml, err, st);
    if (e != cudaSuccess) return e;
    return launch_attn_combine_bf16(ws_o, ws_ml, out, lse, s.batch, s.block_len, s.n_q_heads, D,
                                    p.n_splits, st);
}

}  // namespace fdl
