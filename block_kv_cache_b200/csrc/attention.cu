// DualCache block attention, split-KV (flash-decoding style).
//
// Fast-dLLM, DualCache (aibase news "Innovations" 1; README "Key techniques"
// 1): the B queries of the current block attend, with no mask, over the
// whole cache [prefix | block slot | masked suffix]. The block slot already
// holds the block's fresh K/V.
//
// Pass 1: CTA (split, q-head, sequence) streams a contiguous range of keys of
// its kv head, keeps an online softmax per query row (running max m, sum l,
// unnormalised o) and writes (m, l, o) to the workspace. Scores are kept in
// the log2 domain (scale * log2(e) folded in) so exp2f serves the softmax.
// Pass 2: per (query row, head, sequence) the partials are merged.
//
// This SIMT version serves f32 tensors: it computes in f32 FFMA, because the
// f32 path must stay within 1e-4 relative error, out of reach of TF32 tensor
// cores. bf16 tensors go to the tcgen05 kernel (attention_tc.cu), which
// writes the same partials and is merged by the same combine kernel.
#include "common.cuh"
#include "launch.h"

namespace fdl {

constexpr int ATT_THREADS = 256;          // 8 warps
constexpr int ATT_KT = 32;                // keys per smem tile (one per lane)

static int attn_num_splits(const AttnShape& s, int sm_count) {
    const int heads = s.batch * s.n_q_heads;
    const int max_splits = (s.seq_len + ATT_KT - 1) / ATT_KT;
    int want = (2 * sm_count + heads - 1) / heads;
    if (want < 1) want = 1;
    if (want > max_splits) want = max_splits;
    return want;
}

size_t attn_workspace_bytes(const AttnShape& s, int sm_count) {
    if (s.bf16) return attn_tc_workspace_bytes(s, sm_count);
    const size_t ns = attn_num_splits(s, sm_count);
    const size_t rows = (size_t)s.batch * s.n_q_heads * ns * s.block_len;
    return rows * (s.head_dim + 2) * sizeof(float);
}

// QPW: query rows per warp (ceil(B / 8)); D: head dim.
template <typename T, int D, int QPW>
__global__ void __launch_bounds__(ATT_THREADS)
attn_split_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                  float* __restrict__ ws_o, float* __restrict__ ws_ml, int B, int Hq, int Hkv,
                  int L, int n_splits, int keys_per_split, float scale_log2) {
    extern __shared__ float smem[];
    float* Qs = smem;                                 // [B][D]
    float* Ks = Qs + B * D;                           // [KT][D+1]
    float* Vs = Ks + ATT_KT * (D + 1);                // [KT][D]
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (Hq / Hkv);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int DL = D / 32;                        // dims per lane

    for (int e = tid; e < B * D; e += ATT_THREADS) {
        const int i = e / D, dd = e % D;
        Qs[e] = to_f32(q[(((size_t)b * B + i) * Hq + h) * D + dd]);
    }
    float m[QPW], l[QPW], o[QPW][DL];
#pragma unroll
    for (int r = 0; r < QPW; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int t = 0; t < DL; ++t) o[r][t] = 0.f;
    }
    const int k0 = split * keys_per_split;
    const int k1 = min(L, k0 + keys_per_split);
    const T* kh = kc + ((size_t)b * Hkv + g) * (size_t)L * D;
    const T* vh = vc + ((size_t)b * Hkv + g) * (size_t)L * D;

    for (int t0 = k0; t0 < k1; t0 += ATT_KT) {
        const int nk = min(ATT_KT, k1 - t0);
        __syncthreads();
        for (int e = tid; e < ATT_KT * D; e += ATT_THREADS) {
            const int j = e / D, dd = e % D;
            float kv = 0.f, vv = 0.f;
            if (j < nk) {
                kv = to_f32(kh[(size_t)(t0 + j) * D + dd]);
                vv = to_f32(vh[(size_t)(t0 + j) * D + dd]);
            }
            Ks[j * (D + 1) + dd] = kv;
            Vs[j * D + dd] = vv;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < QPW; ++r) {
            const int i = warp + 8 * r;
            if (i >= B) break;
            // lane j scores key t0 + j
            float sc = 0.f;
            const float* qi = Qs + i * D;
            const float* kj = Ks + lane * (D + 1);
#pragma unroll 8
            for (int dd = 0; dd < D; ++dd) sc = fmaf(qi[dd], kj[dd], sc);
            sc = (lane < nk) ? sc * scale_log2 : -INFINITY;
            const float mt = warp_max(sc);
            const float mn = fmaxf(m[r], mt);
            const float alpha = exp2f(m[r] - mn);     // m = -inf first: exp2(-inf) = 0
            const float p = (lane < nk) ? exp2f(sc - mn) : 0.f;
            l[r] = l[r] * alpha + warp_sum(p);
            m[r] = mn;
#pragma unroll
            for (int t = 0; t < DL; ++t) o[r][t] *= alpha;
            for (int j = 0; j < nk; ++j) {
                const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
                for (int t = 0; t < DL; ++t) o[r][t] = fmaf(pj, Vs[j * D + lane + 32 * t], o[r][t]);
            }
        }
    }
    // partials: row index ((b*Hq + h)*n_splits + split)*B + i
#pragma unroll
    for (int r = 0; r < QPW; ++r) {
        const int i = warp + 8 * r;
        if (i >= B) break;
        const size_t row = (((size_t)b * Hq + h) * n_splits + split) * B + i;
#pragma unroll
        for (int t = 0; t < DL; ++t) ws_o[row * D + lane + 32 * t] = o[r][t];
        if (lane == 0) {
            ws_ml[row * 2 + 0] = m[r];
            ws_ml[row * 2 + 1] = l[r];
        }
    }
}

// One CTA of D threads per (query row, head, sequence).
template <typename T, int D>
__global__ void attn_combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_ml,
                                    T* __restrict__ out, float* __restrict__ lse, int B, int Hq,
                                    int n_splits) {
    const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z, dd = threadIdx.x;
    const size_t base = ((size_t)b * Hq + h) * n_splits;
    float M = -INFINITY;
    for (int sp = 0; sp < n_splits; ++sp) M = fmaxf(M, ws_ml[((base + sp) * B + i) * 2]);
    float Lsum = 0.f, acc = 0.f;
    for (int sp = 0; sp < n_splits; ++sp) {
        const size_t row = (base + sp) * B + i;
        const float ms = ws_ml[row * 2];
        if (ms == -INFINITY) continue;                // split with no keys
        const float w = exp2f(ms - M);
        Lsum = fmaf(ws_ml[row * 2 + 1], w, Lsum);
        acc = fmaf(ws_o[row * D + dd], w, acc);
    }
    out[(((size_t)b * B + i) * Hq + h) * D + dd] = from_f32<T>(acc / Lsum);
    if (lse && dd == 0)
        lse[((size_t)b * Hq + h) * B + i] = (M + log2f(Lsum)) * 0.69314718055994530942f;
}

template <typename T, int D, int QPW>
static cudaError_t run_attn(const AttnShape& s, const T* q, const T* k, const T* v, T* out,
                            float* lse, void* ws, int sm_count, cudaStream_t st) {
    const int ns = attn_num_splits(s, sm_count);
    int kps = (s.seq_len + ns - 1) / ns;
    kps = ((kps + ATT_KT - 1) / ATT_KT) * ATT_KT;
    const int ns_eff = (s.seq_len + kps - 1) / kps;
    float* ws_o = (float*)ws;
    const size_t rows = (size_t)s.batch * s.n_q_heads * ns_eff * s.block_len;
    float* ws_ml = ws_o + rows * D;
    const size_t smem = ((size_t)s.block_len * D + ATT_KT * (D + 1) + ATT_KT * D) * sizeof(float);
    auto kfn = attn_split_kernel<T, D, QPW>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const float scale_log2 = s.scale * 1.4426950408889634f;
    dim3 grid(ns_eff, s.n_q_heads, s.batch);
    kfn<<<grid, ATT_THREADS, smem, st>>>(q, k, v, ws_o, ws_ml, s.block_len, s.n_q_heads,
                                         s.n_kv_heads, s.seq_len, ns_eff, kps, scale_log2);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2(s.block_len, s.n_q_heads, s.batch);
    attn_combine_kernel<T, D><<<g2, D, 0, st>>>(ws_o, ws_ml, out, lse, s.block_len, s.n_q_heads,
                                                ns_eff);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t dispatch_attn(const AttnShape& s, const T* q, const T* k, const T* v, T* out,
                                 float* lse, void* ws, int sm_count, cudaStream_t st) {
    const int qpw = (s.block_len + 7) / 8;
#define FDL_ATT_CASE(DD, QQ)                                                              \
    if (s.head_dim == DD && qpw <= QQ)                                                    \
        return run_attn<T, DD, QQ>(s, q, k, v, out, lse, ws, sm_count, st);
    FDL_ATT_CASE(64, 1) FDL_ATT_CASE(64, 2) FDL_ATT_CASE(64, 4) FDL_ATT_CASE(64, 8)
    FDL_ATT_CASE(64, 16) FDL_ATT_CASE(128, 1) FDL_ATT_CASE(128, 2) FDL_ATT_CASE(128, 4)
    FDL_ATT_CASE(128, 8) FDL_ATT_CASE(128, 16)
#undef FDL_ATT_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_attention_f32(const AttnShape& s, const float* q, const float* k,
                                 const float* v, float* out, float* lse, void* ws,
                                 int sm_count, cudaStream_t st) {
    return dispatch_attn<float>(s, q, k, v, out, lse, ws, sm_count, st);
}


}  // namespace fdl
