// DualCache block attention, bf16, on the 5th-generation tensor cores.
//
// Fast-dLLM, DualCache (aibase news "Innovations" 1; README "Key techniques"
// 1): the block's queries attend, without a mask, over the whole cache
// [prefix | block slot | masked suffix]; the block slot holds fresh K/V.
//
// Work decomposition. The query heads that share a kv head (the GQA group,
// or a chunk of it) are packed as R = hc * B query rows, row r = i*hc + j
// holding query i of head j of the chunk. A CTA owns one (sequence, kv head,
// head chunk) and a contiguous range ("split") of 64-key tiles streamed
// through a TMA ring, so every K/V byte is read from HBM once. The splits of
// one (sequence, kv head, chunk) form a thread-block cluster and merge their
// partial softmaxes on chip: with one 128-row tile each split pushes its
// partial rows into the receive buffer of the CTA that owns them (st.async,
// counted in bytes on the owner's mbarrier); otherwise the owners pull them
// through distributed shared memory between two cluster barriers. The owners
// write the final bf16 output and LSE, with no second pass over memory.
//
// The 128 TMEM lanes are the MMA's M dimension: R <= 128 packed rows use one
// 128-row tile, R in (128, 256] two, each with its own softmax warpgroup. A
// softmax warp reads only its own 32-lane quarter of TMEM; warps whose rows
// are all padding sit out. (With one block of 32 queries per head, one warp
// per tile does the softmax: 64 exponentials and bf16 packs per thread, about
// 1240 of the ~1550 cycles a 64-key tile takes on this B200 at L = 2048;
// replicating the query rows into all four lane quarters, each warp taking a
// quarter of the keys, measured slower.)
//
//   softmax warps (4 per 128-row tile): thread = TMEM lane; online softmax in
//       the log2 domain (scale*log2 e folded into one FFMA); P(t) as bf16 into
//       one of two shared-memory buffers; O rescaled in TMEM only when the
//       running max grows by more than 8 (a factor 2^8)
//   TMA warp (1 thread): Q once, then K and V tiles; a K stage is released
//       as soon as S(t) is done, a V stage once PV(t) is, so the next K tile
//       does not wait for the softmax
//   MMA warp (1 thread): TMEM owner; tcgen05.mma S(t) = Q K(t)^T into one of
//       two S buffers and O += P(u) V(u) with V as an MN-major operand, each
//       issued as soon as its operands are there (non-blocking barrier polls),
//       so a PV never queues behind the wait for the next K tile
//
// Roofline: HBM. Algorithmic bytes per call = K and V once (2*b*Hkv*L*d*2)
// + q and out (2*b*B*Hq*d*2).
#include <atomic>

#include "common.cuh"
#include "gemm.h"
#include "launch.h"
#include "sm100.cuh"
#include "timeline.cuh"

namespace fdl {

constexpr int ATT_KT = 64;          // keys per tile
constexpr int ATT_MAX_SPLITS = 8;   // portable cluster size

struct AttnPlan {
    int hc;        // query heads packed per CTA
    int n_chunks;  // head chunks per kv head
    int rows;      // packed rows R = hc * B
    int mt;        // 128-row MMA tiles (1 or 2)
    int tiles;     // 64-key tiles per (sequence, kv head)
    int tps;       // tiles per split
    int n_splits;  // cluster size
    int units;     // (query block, kv head, chunk) units the split count is planned for
};

// At most `splits` splits of the key tiles (at least one tile each).
void attn_set_splits(AttnPlan& p, int splits) {
    if (splits > ATT_MAX_SPLITS) splits = ATT_MAX_SPLITS;
    if (splits > p.tiles) splits = p.tiles;
    if (splits < 1) splits = 1;
    p.tps = (p.tiles + splits - 1) / splits;
    p.n_splits = (p.tiles + p.tps - 1) / p.tps;
}

AttnPlan attn_tc_plan(const AttnShape& s, int sm_count) {
    AttnPlan p;
    const int grp = s.n_q_heads / s.n_kv_heads;
    p.hc = 256 / s.block_len;
    if (p.hc > grp) p.hc = grp;
    if (p.hc < 1) p.hc = 1;
    p.n_chunks = (grp + p.hc - 1) / p.hc;
    p.rows = p.hc * s.block_len;
    p.mt = p.rows > 128 ? 2 : 1;
    p.tiles = (s.seq_len + ATT_KT - 1) / ATT_KT;
    // A compacted batch (seq_map) is planned as the whole batch of kv_batch
    // sequences, so that a sequence's splits, and with them the order of its
    // sums, do not depend on which other sequences are in the launch.
    const int blocks = s.kv_batch > 0 ? s.kv_batch * s.q_per_kv : s.batch;
    const int units = blocks * s.n_kv_heads * p.n_chunks;
    p.units = units;
    attn_set_splits(p, sm_count / units);
    return p;
}

namespace {

template <int D, int MT>
struct Att4 {
    static constexpr int STAGES = MT == 1 ? 3 : 2;
    static constexpr int THREADS = 32 * (4 * MT + 2);
    static constexpr int TMA_WARP = 4 * MT, MMA_WARP = 4 * MT + 1;
    static constexpr int DC = D / 64;
    static constexpr int Q_CHUNK = MT * 128 * 128;
    static constexpr int KV_CHUNK = ATT_KT * 128;
    static constexpr int KV_TILE = DC * KV_CHUNK;
    static constexpr int P_TILE = 128 * 128;                // 128 rows x 64 keys
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + DC * Q_CHUNK;
    static constexpr int OFF_V = OFF_K + STAGES * KV_TILE;
    static constexpr int OFF_P = OFF_V + STAGES * KV_TILE;   // P[buffer][m]
    static constexpr int OFF_RED = OFF_P + 2 * MT * P_TILE;  // 128 MT x (max, sum) floats
    static constexpr int OFF_BAR = OFF_RED + 128 * MT * 2 * 4;
    // Receive buffer of the pushed split merge (single-tile shapes): partial
    // rows of every split for the rows this CTA owns, (D + 4) floats each.
    static constexpr int OFF_RCV = OFF_BAR + 256;
    static constexpr int RCV_BYTES = MT == 1 ? 65536 : 0;
    static constexpr int RCV_ROW = (D + 4) * 4;
    static constexpr size_t TOTAL = 1024 + OFF_RCV + RCV_BYTES;
    // After the last MMA, [OFF_K, OFF_RED) holds this CTA's partial output
    // (R rows x D floats, float4 slots XOR-swizzled by row) for the cluster.
    static_assert(128 * MT * D * 4 <= OFF_RED - OFF_K, "partial buffer");
    static constexpr uint32_t TMEM_S = 0;                    // S[b2][m] at (b2*MT + m)*64
    static constexpr uint32_t TMEM_O = 2 * MT * ATT_KT;      // O[m] at TMEM_O + m*D
    static constexpr uint32_t TMEM_USED = 2 * MT * ATT_KT + MT * D;
    static constexpr uint32_t TMEM_ALLOC = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert(TOTAL <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// 2^x on the special-function unit (PTX ex2.approx, flush-to-zero); -inf -> 0.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct AttnArgs {
    bf16* out;
    float* lse;         // optional
    int B, Hq, Hkv, L, hc, n_chunks, rows, tiles, tps, n_splits, q_per_kv;
    int blk0, blk1;     // block slot [blk0, blk1) of every sequence
    int push;           // splits push their partial rows to the owner's buffer
    float scale_log2;
    int* err;
    const int32_t* seq_map;   // compacted batch: caches of sequence seq_map[bb / q_per_kv]
    const int32_t* blk0_map;  // sequences at their own blocks: slot of bb at blk0_map[bb]
};

// ---- prologues: work every CTA does after the preceding kernel -----------------
struct AttNoPro {
    static constexpr bool kActive = false;
};

// The epilogue of a split-K block-slot projection (bias, RoPE, q and the K/V
// block slot), done by the attention CTAs that consume it, with no kernel of
// its own and no wait on another CTA. Each CTA forms its own query tile in
// shared memory straight from the f32 sums, then its first MMA can go; the
// block-slot K/V rows that fall in its own key range (only it reads them) are
// written by its idle softmax warps while the others run, and the tiles that
// hold them come last in its tile order. The sums read are zeroed again (the
// q sums, which every split of a head reads, by split 0 once the cluster has
// merged). One query chunk per kv head (hc == grp), one query block per
// sequence.
struct ProQKV {
    static constexpr bool kActive = true;
    float* acc;              // [M, N] sums, N = (Hq + 2 Hkv) * 128
    EpiQKV p;
};

// Item = 8 consecutive dimensions d of one row and their rotation partners
// d + 64 (RoPE over 128-dimensional heads). Loads of a batch first, then math.
// Items [0, nq) are the query tile's, the rest block-slot K/V rows from kv0 on;
// thread tid of nthreads takes every nthreads-th item.
template <int QCHUNK>
__device__ __forceinline__ void qkv_items(const ProQKV& pro, const AttnArgs& a, uint8_t* sq,
                                          int g, int bb, int kv0, int nq, int n, int tid,
                                          int nthreads, bool write_q) {
    constexpr int U = 2;
    const EpiQKV& p = pro.p;
    const int N = (p.n_q_heads + 2 * p.n_kv_heads) * 128;
    const int kv_seq = p.cache_seq(bb);         // whose cache rows the block slot is
    const int blk0 = p.pos0_of(bb);             // where its block slot starts
    for (int e0 = tid; e0 < n; e0 += U * nthreads) {
        float4 v[U][4], bs[U][4], cs[U][4];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * nthreads;
            if (e >= n) continue;
            int i, col, pc;
            bool rot = true;
            if (e < nq) {                        // q: packed row r = i * hc + j
                const int r = e >> 3;
                pc = e & 7;
                i = r / a.hc;
                col = (g * a.hc + r % a.hc) * 128;
            } else {                             // k or v of a block-slot row
                const int f = e - nq, kind = (f >> 3) & 1;
                pc = f & 7;
                i = kv0 + (f >> 4) - blk0;
                col = (p.n_q_heads + kind * p.n_kv_heads + g) * 128;
                rot = kind == 0;
            }
            const float* src = pro.acc + (size_t)(bb * a.B + i) * N + col + pc * 8;
            v[u][0] = __ldcg(reinterpret_cast<const float4*>(src));
            v[u][1] = __ldcg(reinterpret_cast<const float4*>(src + 4));
            v[u][2] = __ldcg(reinterpret_cast<const float4*>(src + 64));
            v[u][3] = __ldcg(reinterpret_cast<const float4*>(src + 68));
            if (p.bias) {
                const float4* b4 = reinterpret_cast<const float4*>(p.bias + col + pc * 8);
                bs[u][0] = __ldg(b4);
                bs[u][1] = __ldg(b4 + 1);
                bs[u][2] = __ldg(b4 + 16);
                bs[u][3] = __ldg(b4 + 17);
            } else {
#pragma unroll
                for (int x = 0; x < 4; ++x) bs[u][x] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (rot) {
                const float4* c4 = reinterpret_cast<const float4*>(
                    p.rope + (size_t)(blk0 + i) * 64 + pc * 8);
#pragma unroll
                for (int x = 0; x < 4; ++x) cs[u][x] = __ldg(c4 + x);
            } else {
#pragma unroll
                for (int x = 0; x < 4; ++x) cs[u][x] = make_float4(1.f, 0.f, 1.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * nthreads;
            if (e >= n) continue;
            const float* lo = reinterpret_cast<const float*>(&v[u][0]);
            const float* hi = reinterpret_cast<const float*>(&v[u][2]);
            const float* blo = reinterpret_cast<const float*>(&bs[u][0]);
            const float* bhi = reinterpret_cast<const float*>(&bs[u][2]);
            const float* c = reinterpret_cast<const float*>(&cs[u][0]);
            uint32_t o0[4], o1[4];
#pragma unroll
            for (int x = 0; x < 8; x += 2) {
                float r0[2], r1[2];
#pragma unroll
                for (int y = 0; y < 2; ++y) {
                    const float y0 = lo[x + y] + blo[x + y], y1 = hi[x + y] + bhi[x + y];
                    const float co = c[2 * (x + y)], si = c[2 * (x + y) + 1];
                    r0[y] = y0 * co - y1 * si;
                    r1[y] = y1 * co + y0 * si;
                }
                o0[x >> 1] = pack_bf16(r0[0], r0[1]);
                o1[x >> 1] = pack_bf16(r1[0], r1[1]);
            }
            const uint4 w0 = make_uint4(o0[0], o0[1], o0[2], o0[3]);
            const uint4 w1 = make_uint4(o1[0], o1[1], o1[2], o1[3]);
            if (e < nq) {
                const int r = e >> 3, pc = e & 7;
                uint8_t* dst = sq + r * 128 + ((pc ^ (r & 7)) << 4);
                *reinterpret_cast<uint4*>(dst) = w0;
                *reinterpret_cast<uint4*>(dst + QCHUNK) = w1;
                if (write_q) {
                    const int i = r / a.hc;
                    bf16* q = p.q + ((size_t)(bb * a.B + i) * p.n_q_heads + g * a.hc + r % a.hc) *
                                        128 + pc * 8;
                    *reinterpret_cast<uint4*>(q) = w0;
                    *reinterpret_cast<uint4*>(q + 64) = w1;
                }
            } else {
                const int f = e - nq, kind = (f >> 3) & 1, pc = f & 7, row = kv0 + (f >> 4);
                bf16* dst = (kind ? p.v_cache : p.k_cache) +
                            (((size_t)kv_seq * p.n_kv_heads + g) * p.seq_len + row) * 128 + pc * 8;
                *reinterpret_cast<uint4*>(dst) = w0;
                *reinterpret_cast<uint4*>(dst + 64) = w1;
                // only this thread reads these sums: zero them for the next call
                float* src = pro.acc + (size_t)(bb * a.B + row - blk0) * N +
                             (p.n_q_heads + kind * p.n_kv_heads + g) * 128 + pc * 8;
                const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
                __stcg(reinterpret_cast<float4*>(src), z);
                __stcg(reinterpret_cast<float4*>(src + 4), z);
                __stcg(reinterpret_cast<float4*>(src + 64), z);
                __stcg(reinterpret_cast<float4*>(src + 68), z);
            }
        }
    }
}

// Zero the q sums of this CTA's query rows (after every split has read them).
__device__ __forceinline__ void qkv_zero_q(const ProQKV& pro, const AttnArgs& a, int g, int bb) {
    const int N = (pro.p.n_q_heads + 2 * pro.p.n_kv_heads) * 128;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = threadIdx.x; e < a.rows * 8; e += blockDim.x) {
        const int r = e >> 3, pc = e & 7;
        float* src = pro.acc + (size_t)(bb * a.B + r / a.hc) * N + (g * a.hc + r % a.hc) * 128 +
                     pc * 8;
        __stcg(reinterpret_cast<float4*>(src), z);
        __stcg(reinterpret_cast<float4*>(src + 4), z);
        __stcg(reinterpret_cast<float4*>(src + 64), z);
        __stcg(reinterpret_cast<float4*>(src + 68), z);
    }
}

// Timeline events (timeline builds): 0 entry, 1 after the dependency wait and
// the prologue, 2 first S MMA issued, 3 last PV committed, 4 first P tile
// written, 5 epilogue start, 6 split merge done, 7 exit.
template <int D, int MT, class Pro>
__global__ void __launch_bounds__(Att4<D, MT>::THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const AttnArgs a, const Pro pro) {
    using namespace sm100;
    using S = Att4<D, MT>;
    constexpr int KT = ATT_KT, STAGES = S::STAGES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sb = raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    const uint32_t bar_q = smem_u32(bars + 0);
    auto k_full = [&](int s) { return smem_u32(bars + 1 + s); };
    auto v_full = [&](int s) { return smem_u32(bars + 1 + STAGES + s); };
    // K and V stages are released separately: K once S(t) is done, V once PV(t) is
    auto k_empty = [&](int s) { return smem_u32(bars + 1 + 2 * STAGES + s); };
    auto v_empty = [&](int s) { return smem_u32(bars + 1 + 3 * STAGES + s); };
    auto s_full = [&](int b) { return smem_u32(bars + 1 + 4 * STAGES + b); };
    auto s_free = [&](int b) { return smem_u32(bars + 3 + 4 * STAGES + b); };
    auto p_full = [&](int b) { return smem_u32(bars + 5 + 4 * STAGES + b); };
    auto o_done = [&](int b) { return smem_u32(bars + 7 + 4 * STAGES + b); };
    const uint32_t bar_kv = smem_u32(bars + 9 + 4 * STAGES);   // block-slot rows written
    const uint32_t bar_rcv = smem_u32(bars + 10 + 4 * STAGES);  // pushed partials landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11 + 4 * STAGES);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    constexpr int tlk = Pro::kActive ? 1 : (MT == 2 ? 2 : 0);
    if (threadIdx.x == 0) FDL_TL(tlk, 0);
    const int split = blockIdx.x;                    // == rank in the cluster
    const int g = blockIdx.y / a.n_chunks, chunk = blockIdx.y % a.n_chunks;
    const int bb = blockIdx.z;
    const int grp = a.Hq / a.Hkv;
    const int t_begin = split * a.tps;
    const int nt = min(a.tps, a.tiles - t_begin);
    const int k_begin = t_begin * KT;
    const int k_end = min(a.L, k_begin + nt * KT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // softmax warps with at least one real row (a warp covers 32 packed rows)
    const int live_warps = (a.rows + 31) / 32;
    const int live_threads = live_warps * 32;
    // warps that write the block-slot K/V rows: the idle softmax warps, else all
    const int kv_w0 = live_warps < 4 * MT ? live_warps : 0;
    // Tile order: with the fused prologue the tiles holding block-slot rows of
    // this split come last (a rotation; the online softmax is order-free).
    // this sequence's block slot [blk0, blk1)
    const int blk0 = a.blk0_map ? __ldg(a.blk0_map + bb) : a.blk0, blk1 = blk0 + (a.blk1 - a.blk0);
    int rot = 0;
    if constexpr (Pro::kActive) {
        if (blk0 < k_end && blk1 > k_begin)
            rot = ((min(blk1, k_end) - 1 - k_begin) / KT + 1) % nt;
    }
    auto tile_of = [&](int t) { const int u = t + rot; return u >= nt ? u - nt : u; };
    auto in_block = [&](int tile) {
        const int k0 = k_begin + tile * KT;
        return k0 < blk1 && k0 + KT > blk0;
    };
    // split merge: split c owns packed rows [c * rpc, c * rpc + own)
    const int rpc = (a.rows + a.n_splits - 1) / a.n_splits;
    const int own = max(0, min(rpc, a.rows - split * rpc));
    const bool push = a.push != 0 && a.n_splits > 1 &&
                      a.n_splits * rpc * S::RCV_ROW <= S::RCV_BYTES;

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_rcv, 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(v_full(s), 1);
            mbar_init(k_empty(s), 1);
            mbar_init(v_empty(s), 1);
        }
        mbar_init(bar_kv, (4 * MT - kv_w0) * 32);
        for (int b2 = 0; b2 < 2; ++b2) {
            mbar_init(s_full(b2), 1);
            mbar_init(s_free(b2), live_threads);
            mbar_init(p_full(b2), live_threads);
            mbar_init(o_done(b2), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
        // every split pushes D + 2 floats for each row this CTA owns
        if (push) mbar_arrive_expect_tx(bar_rcv, (uint32_t)(a.n_splits * own * (D * 4 + 8)));
    }
    if (warp == S::MMA_WARP) tmem_alloc(smem_u32(tmem_slot), S::TMEM_ALLOC);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the receive barriers of the cluster are initialised once every thread
    // has arrived here; the matching wait comes just before the first push
    if (push) cluster_arrive();
    bool rcv_ready = !push;
    const uint32_t tmem = *tmem_slot;
    const int kv_seq = a.seq_map ? __ldg(a.seq_map + bb / a.q_per_kv) : bb / a.q_per_kv;
    const int krow0 = (kv_seq * a.Hkv + g) * a.L + k_begin;
    const uint64_t kv_policy = l2_evict_first();
    // one copy per tile and operand: all D columns as DC sub-tiles
    auto load_k = [&](int t, int st) {
        mbar_arrive_expect_tx(k_full(st), S::KV_TILE);
        if (a.q_per_kv == 1)   // one query block: every K/V byte is read once
            tma_load_3d_hint(sb + S::OFF_K + st * S::KV_TILE, &tmK, k_full(st), 0,
                             krow0 + t * KT, 0, kv_policy);
        else
            tma_load_3d(sb + S::OFF_K + st * S::KV_TILE, &tmK, k_full(st), 0, krow0 + t * KT, 0);
    };
    auto load_v = [&](int t, int st) {
        mbar_arrive_expect_tx(v_full(st), S::KV_TILE);
        if (a.q_per_kv == 1)
            tma_load_3d_hint(sb + S::OFF_V + st * S::KV_TILE, &tmV, v_full(st), 0,
                             krow0 + t * KT, 0, kv_policy);
        else
            tma_load_3d(sb + S::OFF_V + st * S::KV_TILE, &tmV, v_full(st), 0, krow0 + t * KT, 0);
    };
    // With a prologue, the preceding kernel is this call's own projection,
    // which writes no cache row: the first tile, when it lies outside the block
    // slot, can be requested before that kernel ends (its ring stage is fresh,
    // so no empty wait). One tile only: a larger burst delays the loads of the
    // prologue that follows (measured).
    uint32_t early = 0;
    if constexpr (!Pro::kActive) {
        // the tensor maps are kernel parameters: fetch them while the
        // preceding kernel finishes, so the first copies do not wait for them
        if (warp == S::TMA_WARP && lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
        }
    }
    if constexpr (Pro::kActive) {
        if (warp == S::TMA_WARP && lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            for (int t = 0; t < nt && t < 1; ++t) {
                const int tile = tile_of(t);
                if (k_begin + (tile + 1) * KT <= a.L && !in_block(tile)) {
                    load_k(tile, t);
                    load_v(tile, t);
                    early |= 1u << t;
                }
            }
        }
    }
    pdl_wait();
    if constexpr (Pro::kActive) {
        static_assert(D == 128, "the q/k/v prologue rotates 128-dim heads");
        qkv_items<S::Q_CHUNK>(pro, a, smem + S::OFF_Q, g, bb, 0, a.rows * 8, a.rows * 8,
                              threadIdx.x, blockDim.x, split == 0);
        fence_proxy_async();                        // the MMA reads the Q tile written here
        __syncthreads();
    }
    pdl_trigger();
    if (threadIdx.x == 0) FDL_TL(tlk, 1);
    bool ok = *abort_flag == 0;

    if (warp == S::TMA_WARP) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0) {
            bool q_issued = false;
            if constexpr (Pro::kActive) {
                mbar_arrive(bar_q);                 // the Q tile is already in place
            } else if (ok) {
                q_issued = true;
                const int head0 = g * grp + chunk * a.hc;
                mbar_arrive_expect_tx(bar_q, (uint32_t)(S::DC * a.rows * 128));
                for (int dc = 0; dc < S::DC; ++dc)
                    tma_load_3d(sb + S::OFF_Q + dc * S::Q_CHUNK, &tmQ, bar_q, dc * 64, head0,
                                bb * a.B);
            }
            // K and V tiles are requested as their stages come free, in tile
            // order each; whichever can go first does (non-blocking polls)
            int nk = 0, nv = 0;
            bool kv_rows = !Pro::kActive;           // block-slot rows in place
            PollBudget pb;
            while (ok && (nk < nt || nv < nt)) {
                bool moved = false;
                if (nk < nt) {
                    const int st = nk % STAGES, tile = tile_of(nk);
                    if (nk < STAGES && ((early >> nk) & 1u)) {
                        ++nk;
                        moved = true;
                    } else {
                        if (!kv_rows && in_block(tile) && mbar_test(bar_kv, 0)) {
                            fence_proxy_async_global();
                            kv_rows = true;
                        }
                        if ((kv_rows || !in_block(tile)) &&
                            mbar_test(k_empty(st), ((nk / STAGES) & 1) ^ 1)) {
                            load_k(tile, st);
                            ++nk;
                            moved = true;
                        }
                    }
                }
                if (nv < nk) {
                    const int st = nv % STAGES, tile = tile_of(nv);
                    if (nv < STAGES && ((early >> nv) & 1u)) {
                        ++nv;
                        moved = true;
                    } else if (mbar_test(v_empty(st), ((nv / STAGES) & 1) ^ 1)) {
                        load_v(tile, st);
                        ++nv;
                        moved = true;
                    }
                }
                if (moved) {
                    pb.reset();
                } else {
                    __nanosleep(32);                // leave issue slots to the softmax warps
                    ok = pb.idle(abort_flag, a.err);
                }
            }
            // tail: every stage handed out has been released again
            for (int u = nt; ok && u < nt + STAGES; ++u) {
                ok = mbar_wait(k_empty(u % STAGES), ((u / STAGES) & 1) ^ 1, abort_flag, a.err);
                if (ok)
                    ok = mbar_wait(v_empty(u % STAGES), ((u / STAGES) & 1) ^ 1, abort_flag,
                                   a.err);
            }
            if (!ok) {
                // gave up: every copy requested into this CTA's shared memory must
                // land before the CTA exits (the last STAGES of each operand)
                for (int u = (nk > STAGES ? nk - STAGES : 0); u < nk; ++u)
                    mbar_wait_drain(k_full(u % STAGES), (u / STAGES) & 1, a.err);
                for (int u = (nv > STAGES ? nv - STAGES : 0); u < nv; ++u)
                    mbar_wait_drain(v_full(u % STAGES), (u / STAGES) & 1, a.err);
                for (int u = nv; u < STAGES && u < nt; ++u)   // early V not yet counted
                    if ((early >> u) & 1u)
                        mbar_wait_drain(v_full(u), 0, a.err);
                for (int u = nk; u < STAGES && u < nt; ++u)
                    if ((early >> u) & 1u)
                        mbar_wait_drain(k_full(u), 0, a.err);
                if (q_issued) mbar_wait_drain(bar_q, 0, a.err);
            }
        }
    } else if (warp == S::MMA_WARP) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16_f32(128, KT);
            constexpr uint32_t idesc_o = umma_idesc_bf16_f32(128, D, true);
            ok = mbar_wait(bar_q, 0, abort_flag, a.err);
            // S(t) = Q K(t)^T and O += P(u) V(u), each issued as soon as its
            // operands are there: a PV never queues behind the next tile's K
            int ns = 0, npv = 0;
            PollBudget pb;
            while (ok && npv < nt) {
                bool moved = false;
                if (npv < ns) {
                    const int u = npv, su = u % STAGES, pbuf = u & 1;
                    if (mbar_test(p_full(pbuf), (u >> 1) & 1) &&
                        mbar_test(v_full(su), (u / STAGES) & 1)) {
                        tc_fence_after();
#pragma unroll
                        for (int m = 0; m < MT; ++m)
#pragma unroll
                            for (int ks = 0; ks < KT / 16; ++ks) {
                                const uint32_t pa = sb + S::OFF_P + (pbuf * MT + m) * S::P_TILE +
                                                    (ks & 3) * 32;
                                const uint32_t va = sb + S::OFF_V + su * S::KV_TILE + ks * 2048;
                                umma_bf16(tmem + S::TMEM_O + m * D, umma_desc_sw128(pa),
                                          umma_desc_sw128_mn(va, S::KV_CHUNK), idesc_o,
                                          (u > 0 || ks > 0) ? 1u : 0u);
                            }
                        umma_commit(o_done(pbuf));
                        umma_commit(v_empty(su));
                        if (npv + 1 == nt) FDL_TL(tlk, 3);
                        ++npv;
                        moved = true;
                    }
                }
                if (ns < nt) {
                    const int t = ns, st = t % STAGES, b2 = t & 1;
                    if (mbar_test(k_full(st), (t / STAGES) & 1) &&
                        mbar_test(s_free(b2), ((t >> 1) & 1) ^ 1)) {
                        tc_fence_after();
#pragma unroll
                        for (int m = 0; m < MT; ++m)
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t qa = sb + S::OFF_Q + (kk >> 2) * S::Q_CHUNK +
                                                    m * 16384 + (kk & 3) * 32;
                                const uint32_t ka = sb + S::OFF_K + st * S::KV_TILE +
                                                    (kk >> 2) * S::KV_CHUNK + (kk & 3) * 32;
                                umma_bf16(tmem + S::TMEM_S + (b2 * MT + m) * KT,
                                          umma_desc_sw128(qa), umma_desc_sw128(ka), idesc_s,
                                          kk > 0);
                            }
                        umma_commit(s_full(b2));
                        umma_commit(k_empty(st));
                        if (ns == 0) FDL_TL(tlk, 2);
                        ++ns;
                        moved = true;
                    }
                }
                if (moved) {
                    pb.reset();
                } else {
                    __nanosleep(32);                // leave issue slots to the softmax warps
                    ok = pb.idle(abort_flag, a.err);
                }
            }
        }
    } else {
        if constexpr (Pro::kActive) {
            if (warp >= kv_w0) {
                // the block-slot K/V rows of this split's key range
                const int kv0 = max(blk0, k_begin), kv1 = min(blk1, k_end);
                qkv_items<S::Q_CHUNK>(pro, a, smem + S::OFF_Q, g, bb, kv0, 0,
                                      kv1 > kv0 ? (kv1 - kv0) * 16 : 0,
                                      threadIdx.x - kv_w0 * 32, (4 * MT - kv_w0) * 32, false);
                fence_proxy_async_global();         // the TMA reads these rows
                mbar_arrive(bar_kv);
            }
        }
        if (warp < live_warps) {
            // ------------------------------------------------------------ softmax
            const int q = warp & 3;                          // TMEM lane quarter
            const int m = warp >> 2;                         // 128-row tile
            const int r = q * 32 + lane;                     // row within the tile
            const uint32_t lane_base = (uint32_t)(q * 32) << 16;
            float m_run = -INFINITY, l_run = 0.f;            // running max (log2 units), sum
            for (int t = 0; t < nt; ++t) {
                const int b2 = t & 1;
                if (!(ok = mbar_wait_warp(s_full(b2), (t >> 1) & 1, abort_flag, a.err))) break;
                tc_fence_after();
                float sr[KT];
#pragma unroll
                for (int j = 0; j < KT; j += 16)
                    tmem_ld16(tmem + lane_base + S::TMEM_S + (b2 * MT + m) * KT + j,
                              reinterpret_cast<uint32_t*>(sr) + j);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(s_free(b2));

                const int kbase = k_begin + tile_of(t) * KT; // global key of sr[0]
                if (kbase + KT > k_end) {                    // ragged last tile
#pragma unroll
                    for (int j = 0; j < KT; ++j)
                        if (kbase + j >= k_end) sr[j] = -INFINITY;
                }
                float m8[8];                                 // 8 independent max chains
#pragma unroll
                for (int j = 0; j < 8; ++j) m8[j] = sr[j];
#pragma unroll
                for (int j = 8; j < KT; ++j) m8[j & 7] = fmaxf(m8[j & 7], sr[j]);
                float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                 fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                mx *= a.scale_log2;                          // scale > 0 commutes with max
                float alpha = 1.f;
                bool rescale = false;
                if (mx > m_run + 8.f || m_run == -INFINITY) {
                    const float mn = fmaxf(m_run, mx);
                    if (mn != -INFINITY) {
                        alpha = ex2(m_run - mn);             // 0 on the first update
                        rescale = m_run != -INFINITY;
                        m_run = mn;
                    }
                }
                const float nmr = m_run == -INFINITY ? 0.f : -m_run;
                float l = 0.f;
                uint32_t pk[KT / 2];
#pragma unroll
                for (int j = 0; j < KT; j += 2) {
                    const float p0 = ex2(fmaf(sr[j], a.scale_log2, nmr));
                    const float p1 = ex2(fmaf(sr[j + 1], a.scale_log2, nmr));
                    l += p0 + p1;
                    pk[j >> 1] = pack_bf16(p0, p1);
                }
                l_run = l_run * alpha + l;
                if (__any_sync(0xffffffffu, rescale)) {
                    // O holds P V up to tile t-1: wait for PV(t-1), then scale it
                    if (t > 0) {
                        if (!(ok = mbar_wait_warp(o_done((t - 1) & 1), ((t - 1) >> 1) & 1, abort_flag,
                                                  a.err)))
                            break;
                        tc_fence_after();
#pragma unroll
                        for (int d0 = 0; d0 < D; d0 += 16) {
                            uint32_t o[16];
                            const uint32_t ta = tmem + lane_base + S::TMEM_O + m * D + d0;
                            tmem_ld16(ta, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int x = 0; x < 16; ++x)
                                o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
                            tmem_st16(ta, o);
                        }
                        tmem_wait_st();
                    }
                }
                // P buffer b2 is free once PV(t-2) is done
                if (!(ok = mbar_wait_warp(o_done(b2), ((t >> 1) & 1) ^ 1, abort_flag, a.err))) break;
                uint8_t* prow = smem + S::OFF_P + (b2 * MT + m) * S::P_TILE + r * 128;
#pragma unroll
                for (int piece = 0; piece < 8; ++piece)      // 8 keys per 16-byte piece
                    *reinterpret_cast<uint4*>(prow + ((piece ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * piece], pk[4 * piece + 1], pk[4 * piece + 2],
                                   pk[4 * piece + 3]);
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(p_full(b2));
                if (t == 0 && threadIdx.x == 0) FDL_TL(tlk, 4);
            }
            // ----------------------------------------------------------- epilogue
            if (ok)
                ok = mbar_wait_warp(o_done((nt - 1) & 1), ((nt - 1) >> 1) & 1, abort_flag, a.err);
            if (threadIdx.x == 0) FDL_TL(tlk, 5);
            // the live softmax warps agree on running the epilogue; every wait
            // above is bounded, so all of them get here
            named_sync(1, live_threads);
            ok = __all_sync(0xffffffffu, ok && *abort_flag == 0);
            if (push) {                     // the owners' receive barriers exist
                cluster_wait();
                rcv_ready = true;
            }
            if (ok) {
                tc_fence_after();
                float o[D];
#pragma unroll
                for (int d0 = 0; d0 < D; d0 += 16)
                    tmem_ld16(tmem + lane_base + S::TMEM_O + m * D + d0,
                              reinterpret_cast<uint32_t*>(o) + d0);
                tmem_wait_ld();
                const int pr = m * 128 + r;                  // packed row
                const int i = pr / a.hc, hig = chunk * a.hc + pr % a.hc;
                const bool row_ok = pr < a.rows;
                const bool valid = row_ok && i < a.B && hig < grp;
                if (a.n_splits == 1) {
                    if (valid) {
                        const int head = g * grp + hig;
                        const float inv = 1.f / l_run;
                        bf16* dst = a.out + (((size_t)bb * a.B + i) * a.Hq + head) * D;
#pragma unroll
                        for (int d = 0; d < D; d += 8)
                            *reinterpret_cast<uint4*>(dst + d) = make_uint4(
                                pack_bf16(o[d] * inv, o[d + 1] * inv),
                                pack_bf16(o[d + 2] * inv, o[d + 3] * inv),
                                pack_bf16(o[d + 4] * inv, o[d + 5] * inv),
                                pack_bf16(o[d + 6] * inv, o[d + 7] * inv));
                        if (a.lse)
                            a.lse[((size_t)bb * a.Hq + head) * a.B + i] =
                                (m_run + log2f(l_run)) * 0.69314718055994530942f;
                    }
                } else if (row_ok && push) {
                    // push this row's partial into the owner's receive buffer
                    const int oc = pr / rpc, j = pr - oc * rpc;
                    const uint32_t dst = cluster_map(
                        sb + S::OFF_RCV + (uint32_t)((split * rpc + j) * S::RCV_ROW), oc);
                    const uint32_t rbar = cluster_map(bar_rcv, oc);
#pragma unroll
                    for (int d4 = 0; d4 < D / 4; ++d4)
                        st_async_f4(dst + d4 * 16,
                                    make_float4(o[4 * d4], o[4 * d4 + 1], o[4 * d4 + 2],
                                                o[4 * d4 + 3]),
                                    rbar);
                    st_async_f2(dst + D * 4, make_float2(m_run, l_run), rbar);
                } else if (row_ok) {
                    // publish this CTA's partial for the cluster merge
                    float* part = reinterpret_cast<float*>(smem + S::OFF_K) + (size_t)pr * D;
#pragma unroll
                    for (int d4 = 0; d4 < D / 4; ++d4)
                        *reinterpret_cast<float4*>(part + ((d4 ^ (pr & 7)) << 2)) =
                            make_float4(o[4 * d4], o[4 * d4 + 1], o[4 * d4 + 2], o[4 * d4 + 3]);
                    float* red = reinterpret_cast<float*>(smem + S::OFF_RED);
                    red[2 * pr] = m_run;
                    red[2 * pr + 1] = l_run;
                }
            }
        }
    }

    if (push) {
        // -------------------------------------- merge of the pushed split partials
        if (!rcv_ready) cluster_wait();
        // every split's rows have landed (bounded; on the give-up path still wait
        // for what is in flight, so that no push lands after this CTA has left)
        const bool got = own == 0 || mbar_wait_drain(bar_rcv, 0, a.err);
        const int items = got && *abort_flag == 0 ? own * (D / 8) : 0;
        for (int it = threadIdx.x; it < items; it += S::THREADS) {
            const int j = it / (D / 8), d8 = it % (D / 8);
            const int pr = split * rpc + j;
            const int i = pr / a.hc, hig = chunk * a.hc + pr % a.hc;
            if (i >= a.B || hig >= grp) continue;
            float2 ml[ATT_MAX_SPLITS];
            float4 v0[ATT_MAX_SPLITS], v1[ATT_MAX_SPLITS];
#pragma unroll
            for (int cc = 0; cc < ATT_MAX_SPLITS; ++cc) {
                if (cc < a.n_splits) {
                    const uint8_t* row = smem + S::OFF_RCV + (cc * rpc + j) * S::RCV_ROW;
                    ml[cc] = *reinterpret_cast<const float2*>(row + D * 4);
                    v0[cc] = *reinterpret_cast<const float4*>(row + d8 * 32);
                    v1[cc] = *reinterpret_cast<const float4*>(row + d8 * 32 + 16);
                }
            }
            float M = -INFINITY;
#pragma unroll
            for (int cc = 0; cc < ATT_MAX_SPLITS; ++cc)
                if (cc < a.n_splits) M = fmaxf(M, ml[cc].x);
            float Lsum = 0.f;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int cc = 0; cc < ATT_MAX_SPLITS; ++cc) {
                if (cc < a.n_splits && ml[cc].x != -INFINITY) {
                    const float w = ex2(ml[cc].x - M);
                    Lsum += ml[cc].y * w;
                    acc[0] += v0[cc].x * w; acc[1] += v0[cc].y * w;
                    acc[2] += v0[cc].z * w; acc[3] += v0[cc].w * w;
                    acc[4] += v1[cc].x * w; acc[5] += v1[cc].y * w;
                    acc[6] += v1[cc].z * w; acc[7] += v1[cc].w * w;
                }
            }
            const float inv = 1.f / Lsum;
            const int head = g * grp + hig;
            bf16* dst = a.out + (((size_t)bb * a.B + i) * a.Hq + head) * D + d8 * 8;
            *reinterpret_cast<uint4*>(dst) =
                make_uint4(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv),
                           pack_bf16(acc[4] * inv, acc[5] * inv), pack_bf16(acc[6] * inv, acc[7] * inv));
            if (a.lse && d8 == 0)
                a.lse[((size_t)bb * a.Hq + head) * a.B + i] =
                    (M + log2f(Lsum)) * 0.69314718055994530942f;
        }
    } else if (a.n_splits > 1) {
        // ------------------------------------------------ cluster merge of splits
        // every thread of every CTA of the cluster takes part in both barriers
        cluster_sync();
        const int r0 = split * rpc, r1 = min(a.rows, r0 + rpc);
        // item = 8 output columns of one row: two float4 slots per split
        const int items = (r1 > r0 ? r1 - r0 : 0) * (D / 8);
        const uint32_t part_base = sb + S::OFF_K, red_base = sb + S::OFF_RED;
        for (int it = threadIdx.x; it < items; it += S::THREADS) {
            const int pr = r0 + it / (D / 8), d8 = it % (D / 8);
            const int i = pr / a.hc, hig = chunk * a.hc + pr % a.hc;
            if (i >= a.B || hig >= grp) continue;
            float2 ml[ATT_MAX_SPLITS];
            float4 v0[ATT_MAX_SPLITS], v1[ATT_MAX_SPLITS];
            const uint32_t off_ml = red_base + pr * 8;
            const uint32_t off_0 =
                part_base + (uint32_t)(pr * D + (((2 * d8) ^ (pr & 7)) << 2)) * 4;
            const uint32_t off_1 =
                part_base + (uint32_t)(pr * D + (((2 * d8 + 1) ^ (pr & 7)) << 2)) * 4;
#pragma unroll
            for (int cc = 0; cc < ATT_MAX_SPLITS; ++cc) {    // issue every remote load first
                if (cc < a.n_splits) {
                    ml[cc] = ld_cluster_f2(cluster_map(off_ml, cc));
                    v0[cc] = ld_cluster_f4(cluster_map(off_0, cc));
                    v1[cc] = ld_cluster_f4(cluster_map(off_1, cc));
                }
            }
            float M = -INFINITY;
#pragma unroll
            for (int cc = 0; cc < ATT_MAX_SPLITS; ++cc)
                if (cc < a.n_splits) M = fmaxf(M, ml[cc].x);
            float Lsum = 0.f;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int cc = 0; cc < ATT_MAX_SPLITS; ++cc) {
                if (cc < a.n_splits && ml[cc].x != -INFINITY) {
                    const float w = ex2(ml[cc].x - M);
                    Lsum += ml[cc].y * w;
                    acc[0] += v0[cc].x * w; acc[1] += v0[cc].y * w;
                    acc[2] += v0[cc].z * w; acc[3] += v0[cc].w * w;
                    acc[4] += v1[cc].x * w; acc[5] += v1[cc].y * w;
                    acc[6] += v1[cc].z * w; acc[7] += v1[cc].w * w;
                }
            }
            const float inv = 1.f / Lsum;
            const int head = g * grp + hig;
            bf16* dst = a.out + (((size_t)bb * a.B + i) * a.Hq + head) * D + d8 * 8;
            *reinterpret_cast<uint4*>(dst) =
                make_uint4(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv),
                           pack_bf16(acc[4] * inv, acc[5] * inv), pack_bf16(acc[6] * inv, acc[7] * inv));
            if (a.lse && d8 == 0)
                a.lse[((size_t)bb * a.Hq + head) * a.B + i] =
                    (M + log2f(Lsum)) * 0.69314718055994530942f;
        }
        cluster_sync();                    // no CTA leaves while others read its smem
    }
    if (threadIdx.x == 0) FDL_TL(tlk, 6);
    // every split of this head has read the q sums (split 0 has received every
    // split's partial, or passed the cluster barrier above, or, with one split,
    // the barrier after the prologue)
    if constexpr (Pro::kActive)
        if (split == 0) qkv_zero_q(pro, a, g, bb);
    tc_fence_before();
    __syncthreads();
    if (warp == S::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_ALLOC);
    }
    if (threadIdx.x == 0) FDL_TL(tlk, 7);
}

// Clusters of s CTAs of this kernel that the GPU holds at once. A cluster
// must fit in one GPC, so with one CTA per SM fewer clusters of 8 are resident
// than 148 / 8 (measured: 16 clusters of 8 ran in two waves). Queried once per
// cluster size, never while the stream is being captured (fdl_create warms the
// values up); 0 while unknown.
template <int D, int MT, class Pro>
int cluster_capacity(int s, cudaStream_t st) {
    using S = Att4<D, MT>;
    static std::atomic<int> cap[ATT_MAX_SPLITS + 1];
    if (s < 2 || s > ATT_MAX_SPLITS) return 0;
    const int known = cap[s].load(std::memory_order_relaxed);
    if (known > 0) return known;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
        (void)cudaGetLastError();
        return 0;
    }
    auto kfn = attn_tc_kernel<D, MT, Pro>;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::TOTAL) !=
        cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(s, 1, 1);
    cfg.blockDim = dim3(S::THREADS, 1, 1);
    cfg.dynamicSmemBytes = S::TOTAL;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = s;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kfn, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    cap[s].store(n, std::memory_order_relaxed);
    return n;
}

template <int D, int MT, class Pro>
void warm_clusters() {
    for (int s = 2; s <= ATT_MAX_SPLITS; ++s) (void)cluster_capacity<D, MT, Pro>(s, nullptr);
}

template <int D, int MT, class Pro>
cudaError_t run_tc(AttnPlan p, const CUtensorMap& tq, const CUtensorMap& tk,
                   const CUtensorMap& tv, AttnArgs a, int batch, int hkv,
                   cudaStream_t st, const Pro& pro) {
    using S = Att4<D, MT>;
    auto kfn = attn_tc_kernel<D, MT, Pro>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)S::TOTAL);
    if (e != cudaSuccess) return e;
    // fewer splits while the grid's clusters would not all be resident at once
    while (p.n_splits > 1) {
        const int cap = cluster_capacity<D, MT, Pro>(p.n_splits, st);
        if (cap <= 0 || p.units <= cap) break;
        attn_set_splits(p, p.n_splits - 1);
    }
    a.tps = p.tps;
    a.n_splits = p.n_splits;
    // pushed merge when every split's rows for one owner fit its buffer
    const int rpc = (p.rows + p.n_splits - 1) / p.n_splits;
    a.push = MT == 1 && p.n_splits > 1 && p.n_splits * rpc * S::RCV_ROW <= S::RCV_BYTES ? 1 : 0;
    return launch_pdl(kfn, dim3(p.n_splits, hkv * p.n_chunks, batch), dim3(S::THREADS), S::TOTAL,
                      st, p.n_splits, tq, tk, tv, a, pro);
}

}  // namespace

// The cluster capacities of every attention kernel, queried once per process
// outside any stream capture (GPUs of one kind in a process).
void attn_tc_warm() {
    warm_clusters<128, 1, AttNoPro>();
    warm_clusters<128, 2, AttNoPro>();
    warm_clusters<64, 1, AttNoPro>();
    warm_clusters<64, 2, AttNoPro>();
    warm_clusters<128, 1, ProQKV>();
    warm_clusters<128, 2, ProQKV>();
}

size_t attn_tc_workspace_bytes(const AttnShape&, int) {
    return 16;   // the splits merge on chip; no scratch is needed
}

namespace {

template <class Pro>
cudaError_t launch_attn(const AttnShape& s, const void* q, const void* k, const void* v,
                        void* out, float* lse, int sm_count, int* err, cudaStream_t st,
                        const Pro& pro) {
    const AttnPlan p = attn_tc_plan(s, sm_count);
    const int D = s.head_dim;
    CUtensorMap tq, tk, tv;
    const uint64_t qdims[3] = {(uint64_t)D, (uint64_t)s.n_q_heads,
                               (uint64_t)s.batch * s.block_len};
    const uint64_t qstr[2] = {(uint64_t)D * 2, (uint64_t)s.n_q_heads * D * 2};
    const uint32_t qbox[3] = {64, (uint32_t)p.hc, (uint32_t)s.block_len};
    cudaError_t e = make_tmap_bf16(&tq, q, 3, qdims, qstr, qbox);
    if (e != cudaSuccess) return e;
    const uint64_t kv_rows =
        (uint64_t)(s.kv_batch > 0 ? s.kv_batch : s.batch / s.q_per_kv) * s.n_kv_heads * s.seq_len;
    e = make_tmap_bf16_rows(&tk, k, kv_rows, D, ATT_KT, D / 64);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_rows(&tv, v, kv_rows, D, ATT_KT, D / 64);
    if (e != cudaSuccess) return e;
    AttnArgs a;
    a.out = (bf16*)out;
    a.lse = lse;
    a.B = s.block_len;
    a.Hq = s.n_q_heads;
    a.Hkv = s.n_kv_heads;
    a.L = s.seq_len;
    a.hc = p.hc;
    a.n_chunks = p.n_chunks;
    a.rows = p.rows;
    a.tiles = p.tiles;
    a.tps = p.tps;
    a.n_splits = p.n_splits;
    a.q_per_kv = s.q_per_kv;
    a.blk0 = s.block_start;
    a.blk1 = s.block_start + s.block_len;
    a.push = 0;   // set by run_tc with the split count it launches
    a.scale_log2 = s.scale * 1.4426950408889634f;
    a.err = err;
    a.seq_map = s.seq_map;
    a.blk0_map = s.blk0_map;
    const int hb = s.batch, hk = s.n_kv_heads;
    if (D == 128)
        return p.mt == 2 ? run_tc<128, 2>(p, tq, tk, tv, a, hb, hk, st, pro)
                         : run_tc<128, 1>(p, tq, tk, tv, a, hb, hk, st, pro);
    if constexpr (Pro::kActive) return cudaErrorInvalidValue;   // 128-dim heads only
    else
        return p.mt == 2 ? run_tc<64, 2>(p, tq, tk, tv, a, hb, hk, st, pro)
                         : run_tc<64, 1>(p, tq, tk, tv, a, hb, hk, st, pro);
}

}  // namespace

cudaError_t launch_attention_bf16(const AttnShape& s, const void* q, const void* k,
                                  const void* v, void* out, float* lse, void* ws, int sm_count,
                                  int* err, cudaStream_t st) {
    (void)ws;
    return launch_attn(s, q, k, v, out, lse, sm_count, err, st, AttNoPro{});
}

bool qkv_attention_fusable(const AttnShape& s, int sm_count) {
    if (s.head_dim != 128 || !s.bf16 || s.q_per_kv != 1) return false;
    // each CTA forms the query tile of one whole GQA group
    return attn_tc_plan(s, sm_count).n_chunks == 1;
}

cudaError_t launch_qkv_attention_bf16(const AttnShape& s, float* acc, const EpiQKV& pq, void* out,
                                      int sm_count, int* err, cudaStream_t st) {
    return launch_attn(s, pq.q, pq.k_cache, pq.v_cache, out, nullptr, sm_count, err, st,
                       ProQKV{acc, pq});
}

cudaError_t launch_full_attention_bf16(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                       int seq_len, int n_q, float scale, const void* q,
                                       const void* k, const void* v, void* out, int sm_count,
                                       int* dev_err, cudaStream_t st, const int32_t* seq_map,
                                       int kv_batch) {
    // The n_q query rows of a sequence (the last n_q positions; all of them at
    // a refresh) in query blocks of Bq rows: as many whole heads of a GQA group
    // per 256 rows. Each query block is one "sequence" of the attention kernel
    // whose K/V are its sequence's (q_per_kv blocks per sequence).
    const int grp = n_q_heads / n_kv_heads;
    int bq = grp == 1 ? 256 : grp == 2 ? 128 : grp <= 4 ? 64 : 32;
    while (bq > 32 && n_q % bq) bq /= 2;
    if (n_q < 1 || n_q > seq_len || n_q % bq) return cudaErrorInvalidValue;
    AttnShape s{batch * (n_q / bq), n_q_heads, n_kv_heads, head_dim, seq_len, 0, bq, scale,
                1, n_q / bq};
    s.seq_map = seq_map;
    s.kv_batch = seq_map ? kv_batch : 0;
    return launch_attention_bf16(s, q, k, v, out, nullptr, nullptr, sm_count, dev_err, st);
}

}  // namespace fdl

FDL_TL_READER(fdl_timeline_attention)
