// Weight-streaming GEMMs of the cached block step (few token rows, M <= 256):
//   C^T[N, M] = W[N, K] . X[M, K]^T      ("swap AB": the weight is the MMA's
// A operand, 128 weight rows per tile; the tokens are its N dimension).
//
// At a cached DualCache step only the block's rows (32 per sequence) pass
// through the layers (Fast-dLLM; aibase news "Innovations" 1), so every
// projection is a stream of the weight matrix past a handful of activation
// rows: HBM-bound, N*K*2 bytes per call. Putting the weight rows on the MMA's
// M side keeps the tensor-core work per weight byte at the token count
// instead of padding the tokens to 128 rows, and gives twice as many tiles as
// 256-wide token-major tiles; the residual projections also split K so that
// every SM streams (partial sums added atomically into the f32 residual).
//
// Persistent, warp-specialised: warp 0 TMA (ring of 128-wide K steps, each one
// copy of the 128-row weight tile and one of the NT activation rows, landing
// as two 64-column 128-byte-swizzled sub-tiles), warp 1 TMEM owner + single-thread tcgen05.mma (M=128,
// N=NT, K=16) into two NT-column accumulators, warps 2-5 epilogue with
// thread = weight row (output feature), columns = tokens.
//
// The weights never depend on the kernel before this one, so under
// programmatic dependent launch the TMA warp requests the first ring of weight
// tiles before it waits for that kernel; only the activation boxes wait.
#include "common.cuh"
#include "gemm.h"
#include "sm100.cuh"
#include "timeline.cuh"

#include <type_traits>

namespace fdl {
namespace {

constexpr int SK_BM = 128, SK_BK = 128, SK_THREADS = 192;

template <int NT>
struct Sk {
    static constexpr int A_BYTES = SK_BM * SK_BK * 2;        // weight tile (2 chunks of 64)
    static constexpr int B_BYTES = NT * SK_BK * 2;           // activation tile (2 chunks)
    static constexpr int A_CHUNK = SK_BM * 128, B_CHUNK = NT * 128;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = (176 * 1024) / STAGE > 8 ? 8 : (176 * 1024) / STAGE;
    static constexpr int OFF_X = STAGES * STAGE;             // epilogue exchange (QKV)
    // exchange buffer: RoPE partners (128 rows x 33) or the split-K transpose (32 x 132)
    static constexpr int X_BYTES = SK_BM * 33 * 4;
    static constexpr int OFF_BAR = OFF_X + X_BYTES;
    static constexpr size_t TOTAL = 1024 + OFF_BAR + 256;
    static constexpr uint32_t TMEM_COLS = 2 * NT < 32 ? 32 : 2 * NT;
    static_assert(STAGE % 1024 == 0, "stage alignment");
    static_assert(TOTAL <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Each epilogue gets (feature index within [0, N), token count M, first token
// of the 32-token chunk, the 32 accumulator values of the chunk, the shared
// exchange buffer, first feature of the tile).

// dst[t * ld + n0 + c] += C[c][t] for the tile's 128 features c and the chunk's
// tokens t < M, with 16-byte vector atomics: the chunk is transposed through
// shared memory (token-major, rows of 132 floats) so that a thread adds 4
// consecutive features of one token and a warp instruction covers 128
// consecutive features (512 bytes): a quarter of the atomic operations of one
// per element, which the L2 has to absorb when several splits add into a tile.
__device__ __forceinline__ void add_tile_v4(float* dst, int ld, int n0, int M, int j0, int r,
                                            const float* v, uint8_t* xbuf) {
    float* xs = reinterpret_cast<float*>(xbuf);
#pragma unroll
    for (int j = 0; j < 32; ++j) xs[j * 132 + r] = v[j];
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int et = threadIdx.x - 64;                 // epilogue thread 0..127
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int i = et + 128 * k, g4 = i & 31, tl = i >> 5;
        if (j0 + tl < M)
            atomicAdd(reinterpret_cast<float4*>(dst + (size_t)(j0 + tl) * ld + n0 + 4 * g4),
                      *reinterpret_cast<const float4*>(xs + tl * 132 + 4 * g4));
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");   // exchange buffer free again
}

struct SkResid {
    EpiResid p;
    int split;          // > 1: partial sums are added atomically
    __device__ void chunk(int f, int M, int j0, const float* v, uint8_t* xbuf, int n0) const {
        if (split > 1) {
            add_tile_v4(p.h, p.ldh, n0, M, j0, f - n0, v, xbuf);
            return;
        }
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
            const int t = j0 + j;
            if (t < M) p.h[(size_t)t * p.ldh + f] += v[j];
        }
    }
};

struct SkSwiGLU {
    EpiSwiGLU p;
    // rows 2g and 2g+1 of the tile are gate and up of feature g: adjacent lanes
    __device__ void chunk(int f, int M, int j0, const float* v, uint8_t*, int) const {
        const int lane = threadIdx.x & 31;
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
            const float up = __shfl_down_sync(0xffffffffu, v[j], 1);
            const int t = j0 + j;
            if (!(lane & 1) && t < M) {
                const float g = v[j];
                p.out[(size_t)t * p.ldo + (f >> 1)] =
                    __float2bfloat16_rn(g / (1.f + __expf(-g)) * up);
            }
        }
    }
};

struct SkQKV {
    EpiQKV p;
    // one tile = one head (128 dims); RoPE partners are 64 rows apart, so the
    // chunk is exchanged through shared memory (row = dim, 32 tokens, +1 pad)
    __device__ void chunk(int f, int M, int j0, const float* v, uint8_t* xbuf, int n0) const {
        constexpr int D = 128;
        const int r = f - n0;                      // dim within the head
        float* xs = reinterpret_cast<float*>(xbuf);
        const int nq = p.n_q_heads * D, nk = p.n_kv_heads * D;
        const bool rot = n0 < nq + nk;
        if (rot) {
#pragma unroll
            for (int j = 0; j < 32; ++j) xs[r * 33 + j] = v[j];
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const float bias = p.bias ? p.bias[f] : 0.f;
        const float pb = (rot && p.bias) ? p.bias[n0 + (r ^ 64)] : 0.f;
        float2 cs[32];                             // all table loads in flight at once
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int t = j0 + j;
            cs[j] = rot && t < M
                        ? __ldg(p.rope + (size_t)(p.pos0_of(t / p.rows_per_seq) + t % p.rows_per_seq) *
                                             (D / 2) + (r & 63))
                        : make_float2(1.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int t = j0 + j;
            if (t >= M) break;
            const int seq = p.cache_seq(t / p.rows_per_seq);
            const int pos = p.pos0_of(t / p.rows_per_seq) + t % p.rows_per_seq;
            float y = v[j] + bias;
            if (rot) {
                const float other = xs[(r ^ 64) * 33 + j] + pb;
                y = r < 64 ? y * cs[j].x - other * cs[j].y : other * cs[j].y + y * cs[j].x;
            }
            bf16* dst;
            if (n0 < nq)
                dst = p.q + ((size_t)t * p.n_q_heads + n0 / D) * D + r;
            else if (n0 < nq + nk)
                dst = p.k_cache + (((size_t)seq * p.n_kv_heads + (n0 - nq) / D) * p.seq_len + pos) *
                                      D + r;
            else
                dst = p.v_cache +
                      (((size_t)seq * p.n_kv_heads + (n0 - nq - nk) / D) * p.seq_len + pos) * D + r;
            *dst = __float2bfloat16_rn(y);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");   // exchange buffer free again
    }
};

// Split-K partial sums of a non-linear projection: acc[t][f] += C (f32,
// token-major); the epilogue proper runs in a finish_* kernel that also
// restores the zeros.
struct SkAccum {
    float* acc;
    int ldn;
    __device__ void chunk(int f, int M, int j0, const float* v, uint8_t* xbuf, int n0) const {
        add_tile_v4(acc, ldn, n0, M, j0, f - n0, v, xbuf);
    }
};

// ---- prologues: work every CTA does after the preceding kernel, before the GEMM --
struct NoPro {
    static constexpr bool kActive = false;
};

// The SwiGLU of a split-K gate/up projection, done by the CTAs of the GEMM that
// consumes it (the down projection) instead of a kernel of its own: the CTAs
// share out[t, f] = bf16(silu(g) * u) over the f32 sums acc[t, 2f + {0, 1}]
// (restoring the zeros), then meet at a grid barrier before the TMA reads
// `out` as the activation operand. Thread item = 4 consecutive features of
// one token (two float4 of interleaved sums in, 8 bytes out).
struct ProSwiGLU {
    static constexpr bool kActive = true;
    unsigned* bar;           // grid barrier words
    float* acc;
    int M, F;                // tokens, features
    bf16* out;               // [M, F] row stride F: the GEMM's X
    __device__ void work(int part, int nparts) const {
        constexpr int U = 4;                         // items in flight per thread
        const int fq = F / 4, n = M * fq, stride = nparts * blockDim.x;
        for (int e0 = part * blockDim.x + threadIdx.x; e0 < n; e0 += U * stride) {
            float4 a[U], b[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {           // every load first, then the math
                const int e = e0 + u * stride;
                if (e < n) {
                    const int t = e / fq, f = (e - t * fq) * 4;
                    const float4* pg = reinterpret_cast<const float4*>(acc + (size_t)t * 2 * F + 2 * f);
                    a[u] = __ldcg(pg);
                    b[u] = __ldcg(pg + 1);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int e = e0 + u * stride;
                if (e < n) {
                    const int t = e / fq, f = (e - t * fq) * 4;
                    float4* pg = reinterpret_cast<float4*>(acc + (size_t)t * 2 * F + 2 * f);
                    __stcg(pg, make_float4(0.f, 0.f, 0.f, 0.f));
                    __stcg(pg + 1, make_float4(0.f, 0.f, 0.f, 0.f));
                    uint2 o;
                    o.x = pack2(a[u].x / (1.f + __expf(-a[u].x)) * a[u].y,
                                a[u].z / (1.f + __expf(-a[u].z)) * a[u].w);
                    o.y = pack2(b[u].x / (1.f + __expf(-b[u].x)) * b[u].y,
                                b[u].z / (1.f + __expf(-b[u].z)) * b[u].w);
                    *reinterpret_cast<uint2*>(out + (size_t)t * F + f) = o;
                }
            }
        }
    }
};

// RMSNorm of the rows of the f32 residual stream that the GEMM consumes,
// done by its own CTAs instead of a kernel of its own: CTA c normalises rows
// c, c + grid, ... (a block reduction of the sum of squares, then
// out = bf16(h * rsqrt(mean(h^2) + eps) * w)), then all CTAs meet at a grid
// barrier before the TMA reads `out` as the activation operand.
struct ProRMSNorm {
    static constexpr bool kActive = true;
    unsigned* bar;           // grid barrier words
    const float* h;          // [M, D] f32
    const float* w;          // [D]
    float eps;
    int M, D;
    bf16* out;               // [M, D]: the GEMM's X
    __device__ void work(int part, int nparts) const {
        constexpr int RV = 8;                        // float4 of a row held per thread
        __shared__ float red[SK_THREADS / 32];
        const int n4 = D / 4;
        const bool in_regs = n4 <= RV * (int)blockDim.x;
        for (int r = part; r < M; r += nparts) {
            const float4* x = reinterpret_cast<const float4*>(h + (size_t)r * D);
            const float4* w4 = reinterpret_cast<const float4*>(w);
            float4 v[RV], gw[RV];
            float ss = 0.f;
            if (in_regs) {                           // one pass: the row stays in registers
                // the row and the norm weights in one round of loads
#pragma unroll
                for (int k = 0; k < RV; ++k) {
                    const int j = threadIdx.x + k * blockDim.x;
                    v[k] = j < n4 ? __ldcg(x + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                    gw[k] = j < n4 ? __ldg(w4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int k = 0; k < RV; ++k)
                    ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
            } else {
                for (int j = threadIdx.x; j < n4; j += blockDim.x) {
                    const float4 u = __ldcg(x + j);
                    ss += u.x * u.x + u.y * u.y + u.z * u.z + u.w * u.w;
                }
            }
            ss = warp_sum(ss);
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
            __syncthreads();
            float tot = 0.f;
#pragma unroll
            for (int k = 0; k < SK_THREADS / 32; ++k) tot += red[k];
            const float inv = rsqrtf(tot / (float)D + eps);
            __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(out + (size_t)r * D);
            if (in_regs) {
#pragma unroll
                for (int k = 0; k < RV; ++k) {
                    const int j = threadIdx.x + k * blockDim.x;
                    if (j < n4) {
                        const float4 g = gw[k];
                        o2[2 * j] = __floats2bfloat162_rn(v[k].x * inv * g.x, v[k].y * inv * g.y);
                        o2[2 * j + 1] =
                            __floats2bfloat162_rn(v[k].z * inv * g.z, v[k].w * inv * g.w);
                    }
                }
            } else {
                for (int j = threadIdx.x; j < n4; j += blockDim.x) {
                    const float4 u = __ldcg(x + j), g = __ldg(w4 + j);
                    o2[2 * j] = __floats2bfloat162_rn(u.x * inv * g.x, u.y * inv * g.y);
                    o2[2 * j + 1] = __floats2bfloat162_rn(u.z * inv * g.z, u.w * inv * g.w);
                }
            }
            __syncthreads();                        // red[] is reused by the next row
        }
    }
};

// Kind of an instrumented launch (timeline builds): which call it serves.
template <class Epi, class Pro>
__device__ __forceinline__ constexpr int sk_tl_kind() {
    if constexpr (std::is_same<Epi, SkAccum>::value && std::is_same<Pro, ProRMSNorm>::value)
        return 0;                                    // q/k/v or gate/up sums with the RMSNorm
    else if constexpr (std::is_same<Epi, SkResid>::value && std::is_same<Pro, ProSwiGLU>::value)
        return 1;                                    // down projection with the SwiGLU
    else if constexpr (std::is_same<Epi, SkResid>::value)
        return 2;                                    // O projection
    else if constexpr (std::is_same<Epi, SkAccum>::value)
        return 3;
    else if constexpr (std::is_same<Epi, SkSwiGLU>::value)
        return 4;
    else
        return 5;
}

// Timeline events of the skinny GEMM (timeline builds): 0 entry, 1 after the
// dependency wait, 2 after the prologue's grid barrier, 3 first MMA issued,
// 4 last MMA issued, 5 last epilogue chunk done, 7 exit.
template <int NT, class Epi, class Pro>
__global__ void __launch_bounds__(SK_THREADS, 1)
gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   int M, int N, int K, int splits, int num_items, int* err, const Epi epi,
                   const Pro pro) {
    using namespace sm100;
    using S = Sk<NT>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S::STAGES + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto full_bar = [&](int s) { return smem_u32(bars + s); };
    auto empty_bar = [&](int s) { return smem_u32(bars + S::STAGES + s); };
    auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * S::STAGES + a); };
    auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * S::STAGES + 2 + a); };
    auto sA = [&](int s) { return sbase + s * S::STAGE; };
    auto sB = [&](int s) { return sbase + s * S::STAGE + S::A_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k_iters = K / SK_BK;
    const int kps = (k_iters + splits - 1) / splits;        // k iterations per split
    constexpr int tlk = sk_tl_kind<Epi, Pro>();
    if (threadIdx.x == 0) FDL_TL(tlk, 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
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
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), S::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // (item, k) steps of this CTA in order; the first npre of them get their
    // weight boxes before the dependency wait (the weights never depend on the
    // preceding kernel)
    int npre = 0;
    int pre_k[S::STAGES];                            // K step of each of them
    const uint64_t w_policy = l2_evict_first();      // weights: read once per call
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmW);
        prefetch_tmap(&tmX);
        for (int item = blockIdx.x; npre < S::STAGES && item < num_items; item += gridDim.x) {
            const int n_tile = item / splits, ks = item % splits;
            const int k0 = ks * kps, k1 = min(k_iters, k0 + kps);
            for (int k = k0; npre < S::STAGES && k < k1; ++k, ++npre) {
                pre_k[npre] = k;
                mbar_arrive_expect_tx(full_bar(npre), S::STAGE);
                tma_load_3d_hint(sA(npre), &tmW, full_bar(npre), 0, n_tile * SK_BM, k * 2,
                                 w_policy);
            }
        }
    }
    pdl_wait();
    if (threadIdx.x == 0) FDL_TL(tlk, 1);
    if constexpr (Pro::kActive) {
        pro.work(blockIdx.x, gridDim.x);
        fence_proxy_async_global();                 // the TMA below reads what was written
        grid_barrier(pro.bar, abort_flag, err);
    }
    if (threadIdx.x == 0) FDL_TL(tlk, 2);
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            if constexpr (Pro::kActive) fence_proxy_async_global();
            int stage = 0, n = 0;
            uint32_t phase = 0;
            bool ok = *abort_flag == 0;
            for (int item = blockIdx.x; ok && item < num_items; item += gridDim.x) {
                const int n_tile = item / splits, ks = item % splits;
                const int k0 = ks * kps, k1 = min(k_iters, k0 + kps);
                for (int k = k0; k < k1; ++k, ++n) {
                    if (n >= npre) {
                        if (!(ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, err))) break;
                        mbar_arrive_expect_tx(full_bar(stage), S::STAGE);
                        tma_load_3d_hint(sA(stage), &tmW, full_bar(stage), 0, n_tile * SK_BM,
                                         k * 2, w_policy);
                    }
                    tma_load_3d(sB(stage), &tmX, full_bar(stage), 0, 0, k * 2);
                    if (++stage == S::STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            for (int s = 0; ok && s < S::STAGES; ++s) {
                ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, err);
                if (++stage == S::STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) {
                // gave up: wait (bounded) until every copy issued into this
                // CTA's shared memory has landed before the CTA may exit; a
                // step whose weights went out early gets its activation box
                // now, so that its barrier phase completes
                for (int j = n; j < npre; ++j)
                    tma_load_3d(sB(j), &tmX, full_bar(j), 0, 0, pre_k[j] * 2);
                const int issued = n > npre ? n : npre;
                for (int s = 0; s < S::STAGES && s < issued; ++s) {
                    const int j = s + ((issued - 1 - s) / S::STAGES) * S::STAGES;
                    mbar_wait_drain(full_bar(s), (uint32_t)((j / S::STAGES) & 1), err);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(SK_BM, NT);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
            for (int item = blockIdx.x; ok && item < num_items; item += gridDim.x, ++it) {
                const int ks = item % splits;
                const int k0 = ks * kps, k1 = min(k_iters, k0 + kps);
                const int acc = it & 1;
                const uint32_t aphase = (it >> 1) & 1;
                if (!(ok = mbar_wait(tempty_bar(acc), aphase ^ 1, abort_flag, err))) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * NT;
                for (int k = k0; k < k1; ++k) {
                    if (!(ok = mbar_wait(full_bar(stage), phase, abort_flag, err))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < SK_BK / 16; ++kk) {
                        const uint64_t a0 = umma_desc_sw128(sA(stage) + (kk >> 2) * S::A_CHUNK);
                        const uint64_t b0 = umma_desc_sw128(sB(stage) + (kk >> 2) * S::B_CHUNK);
                        umma_bf16(d_tmem, a0 + (uint64_t)((kk & 3) * 2), b0 + (uint64_t)((kk & 3) * 2),
                                  idesc, (k > k0 || kk > 0) ? 1u : 0u);
                    }
                    if (it == 0 && k == k0) FDL_TL(tlk, 3);
                    umma_commit(empty_bar(stage));
                    if (++stage == S::STAGES) { stage = 0; phase ^= 1; }
                }
                if (ok) umma_commit(tfull_bar(acc));
            }
            FDL_TL(tlk, 4);
        }
    } else {
        const int q = warp & 3;                     // TMEM lane quarter = 32 weight rows
        const int r = q * 32 + lane;
        int it = 0;
        for (int item = blockIdx.x; item < num_items; item += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t aphase = (it >> 1) & 1;
            const int n0 = (item / splits) * SK_BM;
            if (!mbar_wait_warp(tfull_bar(acc), aphase, abort_flag, err)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * NT;
#pragma unroll 1
            for (int j0 = 0; j0 < NT; j0 += 32) {
                float v[32];
                tmem_ld32(tacc + j0, *reinterpret_cast<uint32_t(*)[32]>(v));
                tmem_wait_ld();
                if (j0 >= M) break;                           // no token left (uniform)
                epi.chunk(n0 + r, M, j0, v, smem + S::OFF_X, n0);
            }
            tc_fence_before();
            mbar_arrive(tempty_bar(acc));
        }
        if (threadIdx.x == 64) FDL_TL(tlk, 5);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
    if (threadIdx.x == 0) FDL_TL(tlk, 7);
}

template <int NT, class Epi, class Pro = NoPro>
cudaError_t run_skinny(const GemmShape& g, const void* x, const void* w, const Epi& epi,
                       int splits, int sm_count, int* err, cudaStream_t st, const Pro& pro = Pro{}) {
    using S = Sk<NT>;
    CUtensorMap tw, tx;
    // one copy per K step and operand: 128 columns as two 64-column sub-tiles
    cudaError_t e = make_tmap_bf16_rows(&tw, w, g.N, g.K, SK_BM, 2);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_rows(&tx, x, g.M, g.K, NT, 2);
    if (e != cudaSuccess) return e;
    const int items = (g.N / SK_BM) * splits;
    const int grid = items < sm_count ? items : sm_count;
    e = cudaFuncSetAttribute(gemm_skinny_kernel<NT, Epi, Pro>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::TOTAL);
    if (e != cudaSuccess) return e;
    return launch_pdl(gemm_skinny_kernel<NT, Epi, Pro>, dim3(grid), dim3(SK_THREADS), S::TOTAL, st,
                      0, tw, tx, g.M, g.N, g.K, splits, items, err, epi, pro);
}

template <class Epi, class Pro = NoPro>
cudaError_t dispatch_skinny(const GemmShape& g, const void* x, const void* w, const Epi& epi,
                            int splits, int sm_count, int* err, cudaStream_t st,
                            const Pro& pro = Pro{}) {
    if (g.M <= 32) return run_skinny<32>(g, x, w, epi, splits, sm_count, err, st, pro);
    if (g.M <= 64) return run_skinny<64>(g, x, w, epi, splits, sm_count, err, st, pro);
    if (g.M <= 128) return run_skinny<128>(g, x, w, epi, splits, sm_count, err, st, pro);
    return run_skinny<256>(g, x, w, epi, splits, sm_count, err, st, pro);
}

// K splits: the (tiles x splits) work items should fill whole waves of the
// persistent grid (a partly filled last wave leaves SMs idle while the others
// stream), with at least 4 K steps per split. Among splits with the best wave
// efficiency the smallest wins (fewer partial-sum additions).
int choose_splits(const GemmShape& g, int sm_count, int max_splits) {
    const int tiles = g.N / SK_BM, k_iters = g.K / SK_BK;
    int best = 1;
    double best_eff = 0.0;
    for (int s = 1; s <= max_splits && s <= k_iters / 4; ++s) {
        const int items = tiles * s;
        const int waves = (items + sm_count - 1) / sm_count;
        const double eff = (double)items / ((double)waves * sm_count);
        if (eff > best_eff + 0.02) {
            best_eff = eff;
            best = s;
        }
    }
    const int kps = (k_iters + best - 1) / best;
    return (k_iters + kps - 1) / kps;            // every split gets at least one K step
}

// ---- epilogues of split-K projections: consume the f32 sums, leave zeros ----------
// SwiGLU: thread = 4 consecutive features of one token (two float4 of
// interleaved gate/up sums in, 8 bytes of bf16 out).
__global__ void finish_swiglu_kernel(float* __restrict__ acc, int M, int F, bf16* __restrict__ out,
                                     int ldo) {
    pdl_wait();
    pdl_trigger();
    const int fq = F / 4;
    const int n = M * fq;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
        const int t = e / fq, f = (e - t * fq) * 4;
        float4* pg = reinterpret_cast<float4*>(acc + (size_t)t * 2 * F + 2 * f);
        const float4 a = __ldcs(pg), b = __ldcs(pg + 1);
        __stcs(pg, make_float4(0.f, 0.f, 0.f, 0.f));
        __stcs(pg + 1, make_float4(0.f, 0.f, 0.f, 0.f));
        uint2 o;
        o.x = pack2(a.x / (1.f + __expf(-a.x)) * a.y, a.z / (1.f + __expf(-a.z)) * a.w);
        o.y = pack2(b.x / (1.f + __expf(-b.x)) * b.y, b.z / (1.f + __expf(-b.z)) * b.w);
        *reinterpret_cast<uint2*>(out + (size_t)t * ldo + f) = o;
    }
}

// one CTA of 128 threads per (token, head of q, k or v); thread = dim
__global__ void finish_qkv_kernel(float* __restrict__ acc, int M, EpiQKV p) {
    pdl_wait();
    pdl_trigger();
    constexpr int D = 128;
    const int heads = p.n_q_heads + 2 * p.n_kv_heads;
    const int t = blockIdx.x / heads, h = blockIdx.x % heads, r = threadIdx.x;
    const int N = heads * D;
    float* row = acc + (size_t)t * N + h * D;
    float y = row[r] + (p.bias ? p.bias[h * D + r] : 0.f);
    const int seq = p.cache_seq(t / p.rows_per_seq);
            const int pos = p.pos0_of(t / p.rows_per_seq) + t % p.rows_per_seq;
    if (h < p.n_q_heads + p.n_kv_heads) {
        const float other = row[r ^ 64] + (p.bias ? p.bias[h * D + (r ^ 64)] : 0.f);
        const float2 cs = p.rope[(size_t)pos * (D / 2) + (r & 63)];
        y = r < 64 ? y * cs.x - other * cs.y : other * cs.y + y * cs.x;
    }
    __syncthreads();                               // both halves read before zeroing
    row[r] = 0.f;
    bf16* dst;
    if (h < p.n_q_heads)
        dst = p.q + ((size_t)t * p.n_q_heads + h) * D + r;
    else if (h < p.n_q_heads + p.n_kv_heads)
        dst = p.k_cache + (((size_t)seq * p.n_kv_heads + h - p.n_q_heads) * p.seq_len + pos) * D + r;
    else
        dst = p.v_cache +
              (((size_t)seq * p.n_kv_heads + h - p.n_q_heads - p.n_kv_heads) * p.seq_len + pos) * D + r;
    *dst = __float2bfloat16_rn(y);
}

}  // namespace

bool skinny_ok(const GemmShape& g) { return g.M <= 256 && g.N % SK_BM == 0 && g.K % SK_BK == 0; }

cudaError_t launch_skinny_resid(const GemmShape& g, const void* x, const void* w,
                                const EpiResid& p, int sm_count, int* err, cudaStream_t st) {
    // partial sums go straight into the f32 residual stream (coalesced atomics)
    const int splits = choose_splits(g, sm_count, 16);
    return dispatch_skinny(g, x, w, SkResid{p, splits}, splits, sm_count, err, st);
}

cudaError_t launch_skinny_swiglu(const GemmShape& g, const void* x, const void* w,
                                 const EpiSwiGLU& p, float* acc, size_t acc_bytes, int sm_count,
                                 int* err, cudaStream_t st) {
    const int splits = acc && (size_t)g.M * g.N * 4 <= acc_bytes
                           ? choose_splits(g, sm_count, 8) : 1;
    if (splits == 1) return dispatch_skinny(g, x, w, SkSwiGLU{p}, 1, sm_count, err, st);
    cudaError_t e = dispatch_skinny(g, x, w, SkAccum{acc, g.N}, splits, sm_count, err, st);
    if (e != cudaSuccess) return e;
    const int n = g.M * (g.N / 8);                 // 4 output features per thread
    const int blocks = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
    return launch_pdl(finish_swiglu_kernel, dim3(blocks), dim3(256), 0, st, 0, acc, g.M, g.N / 2,
                      p.out, p.ldo);
}

cudaError_t launch_skinny_qkv(const GemmShape& g, const void* x, const void* w, const EpiQKV& p,
                              float* acc, size_t acc_bytes, int sm_count, int* err,
                              cudaStream_t st) {
    const int splits = acc && (size_t)g.M * g.N * 4 <= acc_bytes
                           ? choose_splits(g, sm_count, 8) : 1;
    if (splits == 1) return dispatch_skinny(g, x, w, SkQKV{p}, 1, sm_count, err, st);
    cudaError_t e = dispatch_skinny(g, x, w, SkAccum{acc, g.N}, splits, sm_count, err, st);
    if (e != cudaSuccess) return e;
    return launch_pdl(finish_qkv_kernel, dim3(g.M * (g.N / 128)), dim3(128), 0, st, 0, acc, g.M,
                      p);
}

int skinny_qkv_splits(const GemmShape& g, size_t acc_bytes, int sm_count) {
    return (size_t)g.M * g.N * 4 <= acc_bytes ? choose_splits(g, sm_count, 8) : 1;
}

cudaError_t launch_skinny_qkv_sums(const GemmShape& g, const void* x, const void* w, float* acc,
                                   int splits, const NormIn* norm, unsigned* bar, int sm_count,
                                   int* err, cudaStream_t st) {
    if (norm)
        return dispatch_skinny(g, x, w, SkAccum{acc, g.N}, splits, sm_count, err, st,
                               ProRMSNorm{bar, norm->h, norm->w, norm->eps, g.M, g.K, (bf16*)x});
    return dispatch_skinny(g, x, w, SkAccum{acc, g.N}, splits, sm_count, err, st);
}

// h += down(SwiGLU(x W_gu^T)) for few rows: the gate/up projection with split-K
// partial sums in acc, then the down projection whose CTAs first turn the
// sums into f = bf16(silu(g) * u) (grid barrier, no kernel in between).
cudaError_t launch_skinny_ffn(const GemmShape& g_gu, const void* x, const void* w_gu,
                              const void* w_down, bf16* f, float* h, int ld_h, float* acc,
                              size_t acc_bytes, unsigned* bar, const NormIn* norm, int sm_count,
                              int* err, cudaStream_t st) {
    const int F = g_gu.N / 2;
    const GemmShape g_dn{g_gu.M, ld_h, F};
    const int splits = acc && (size_t)g_gu.M * g_gu.N * 4 <= acc_bytes
                           ? choose_splits(g_gu, sm_count, 8) : 1;
    const EpiResid pr{h, ld_h};
    const int dn_splits = choose_splits(g_dn, sm_count, 16);
    cudaError_t e;
    if (splits == 1) {
        if (norm) {
            e = launch_rmsnorm(g_gu.M, g_gu.K, norm->h, nullptr, norm->w, norm->eps, (bf16*)x, st);
            if (e != cudaSuccess) return e;
        }
        e = dispatch_skinny(g_gu, x, w_gu, SkSwiGLU{EpiSwiGLU{f, F}}, 1, sm_count, err, st);
        if (e != cudaSuccess) return e;
        return dispatch_skinny(g_dn, f, w_down, SkResid{pr, dn_splits}, dn_splits, sm_count, err,
                               st);
    }
    if (norm)
        e = dispatch_skinny(g_gu, x, w_gu, SkAccum{acc, g_gu.N}, splits, sm_count, err, st,
                            ProRMSNorm{bar + 2, norm->h, norm->w, norm->eps, g_gu.M, g_gu.K,
                                       (bf16*)x});
    else
        e = dispatch_skinny(g_gu, x, w_gu, SkAccum{acc, g_gu.N}, splits, sm_count, err, st);
    if (e != cudaSuccess) return e;
    return dispatch_skinny(g_dn, f, w_down, SkResid{pr, dn_splits}, dn_splits, sm_count, err, st,
                           ProSwiGLU{bar, acc, g_gu.M, F, f});
}

}  // namespace fdl

FDL_TL_READER(fdl_timeline_skinny)
