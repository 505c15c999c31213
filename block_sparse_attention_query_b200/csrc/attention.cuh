// Block-sparse attention on tcgen05 tensor cores (PARK: Accurate Block Retrieval for Sparse
// Attention in Video Diffusion Transformers, Abstract: attention computed only within the
// retrieved blocks; cost motive "quadratic complexity of full attention", HASTE abstract).
//
// Persistent kernel: one CTA per SM walks work items round-robin. A work item is (head h,
// query block i, range [e0, e0+n) of its kept list): video query rows are one item each;
// the dense text query rows are split into chunks whose partial results (normalised O and
// log2-sum-exp) go to the workspace and are merged by merge_text_kernel. Text items come
// first in the item order, so the long ones start early.
//
// Warp roles (512 threads):
//   warps 0-7  softmax, two groups of four warps. Group G takes the blocks g of the stream
//              with g%2 == G, so the two groups work on consecutive blocks at the same time
//              (one in its exponentials while the other reads and reduces its scores);
//              warp w owns query rows 32*(w%4) .. +31 (its TMEM lane quarter), whole rows.
//              The reference max of a row is chained from block to block through shared
//              memory (a light dependency on the other group's first pass only).
//   warps 8-11 epilogue: once the MMA has committed an item's last PV, read O[item&1] out of
//              TMEM, divide by the row sum and store the rows (bf16 O, or the text rows'
//              float32 partials); also writes the rows of items with nothing kept.
//   warp 12    TMEM allocation; one elected thread issues every tcgen05.mma.
//   warps 13-15 loaders: gather Q / K / V rows of a block (raster rows from the block-slot
//              table) with 16-byte cp.async into 128B-swizzled K-major tiles; completion
//              arrives on the tile's mbarrier asynchronously.
// The kept blocks of all items of a CTA form one stream g = 0, 1, 2, ...:
//   S[g&1] = Q K_g^T (TMEM fp32) -> softmax: row max of the block (pass 1), P = 2^(s-m) as
//   bf16 pairs written back over S in TMEM (pass 2) -> O[item&1] += P V_g with P read from
//   TMEM (V is an MN-major smem operand). The reference max m only moves when a row max
//   grows by more than 2^8, so O (in TMEM) is rarely rescaled; P <= 2^8 fits bf16 and the
//   final division by the row sum is exact either way.
// S/P is double-buffered (buffer g&1 belongs to softmax group g&1); Q, O, K and V are
// double-buffered. Each group keeps its row sum relative to its own latest reference max; the
// epilogue combines the two. Every wait is bounded: one that runs out raises
// BSA_ERR_TIMEOUT and all roles wind down. tcgen05.ld/st are warp-collective, so every
// condition around them is warp-uniform.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace attn {

constexpr int BQ = 128;                 // query rows per tile (MMA M)
constexpr int kSoftmaxThreads = 256;    // 8 warps: 2 groups of 4 (one per TMEM lane quarter)
constexpr int kGroupThreads = 128;
constexpr int kEpiWarp0 = 8;
constexpr int kEpiThreads = 128;
constexpr int kMmaWarp = 12;
constexpr int kLoadWarp0 = 13;
constexpr int kLoadThreads = 96;        // a warp of 16-byte gathers moves ~12 B per cycle
constexpr int kThreads = kSoftmaxThreads + kEpiThreads + 32 + kLoadThreads;   // 512
constexpr int NK = 2;                   // K pipeline stages
constexpr int NV = 2;                   // V pipeline stages
constexpr int kTextChunk = 64;          // kept blocks per work item of a text query row
constexpr float kRescaleLog2 = 8.0f;    // O is rescaled only when a row max grows by > 2^8

template <int D, int BK>
struct Cfg {
    static constexpr int Q_BYTES = BQ * D * 2;
    static constexpr int KV_BYTES = BK * D * 2;
    static constexpr int OFF_Q = 0;                          // 2 buffers
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;        // NK stages
    static constexpr int OFF_V = OFF_K + NK * KV_BYTES;      // NV stages
    static constexpr int OFF_ML = OFF_V + NV * KV_BYTES;     // [2 O buffers][m0, l0, m1, l1][BQ]
    static constexpr int OFF_MCH = OFF_ML + 2 * 4 * BQ * 4;  // [2 S buffers][BQ] chained maxima
    static constexpr int OFF_STG = OFF_MCH + 2 * BQ * 4;     // [4 epilogue warps][32 rows][128 B]
    static constexpr int OFF_BAR = OFF_STG + 4 * 32 * 128;
    // q_full[2] q_empty[2] k_full[NK] k_empty[NK] v_full[NV] v_empty[NV] s_full[2] s_free[2]
    // p_full[2] pv_done o_full[2] ml_ready[2] o_free[2] fin m_ready[2]
    // (s_free[b]: the PV that read P out of S buffer b is done; o_full[b]: the item's last
    // PV into O buffer b is done; ml_ready[b]: both groups' row max and sum are in shared
    // memory; o_free[b]: the epilogue has read O buffer b and its row maxima and sums;
    // m_ready[b]: the reference max of the latest block of S buffer b is published)
    static constexpr int NBAR = 4 + 2 * NK + 2 * NV + 4 + 2 + 1 + 6 + 1 + 2;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 8;         // +8: TMEM address slot
    static constexpr int TMEM_S = 0;            // S buffers: [0, 2*BK); P (bf16 pairs, key k at
                                                // column k/2) overwrites the first BK/2 columns
    static constexpr int TMEM_O = 2 * BK;       // O buffers: [2*BK, 2*BK + 2*D)
    static constexpr int TMEM_COLS = (2 * BK + 2 * D) <= 256 ? 256 : 512;
    static constexpr int Q_PANEL = BQ * 128;    // bytes per 64-column swizzle panel
    static constexpr int KV_PANEL = BK * 128;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BQ, BK, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, 0, 1);
    static_assert(2 * BK + 2 * D <= 512, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
    Geom g;
    const bsa_bf16* Q;
    const bsa_bf16* K;
    const bsa_bf16* V;
    const int* idx;     // kept lists; idx == cnt == nullptr: every block, in index order
    const int* cnt;
    const int* head_mask;   // nullable: heads with head_mask[h] == 0 are skipped, nothing written
    const int* perm;    // [nb*B] raster token of every block slot, -1 = padding
    const int* kperm;   // nullable, [heads][nb*B]: key-side slot table (query-aware key blocks);
                        // NULL: keys and values use perm like the queries
    bsa_bf16* O;
    float* lse;         // nullable, [heads][N]: log2 of the row's softmax denominator in log2
                        // units of the scaled logits (-inf when nothing is kept)
    float* part_o;      // [n_text_items][BQ][D] normalised partial outputs
    float* part_lse;    // [n_text_items][BQ] log2-sum-exp of each partial row
    int n_text_items;   // heads * nbt * nsplit
    int nsplit;         // chunks per text query row
    int n_items;        // n_text_items + heads * nbv
    float scale_log2;   // log2(e) / sqrt(d)
};

// One work item, decoded identically by every role.
struct Item {
    int h, i, e0, n;
    bool split;
    bool skip;          // head masked out: no work, no output
};

__device__ inline Item decode_item(const Params& P, int item) {
    const Geom& g = P.g;
    Item it;
    if (item < P.n_text_items) {
        it.split = true;
        const int per_head = g.nbt * P.nsplit;
        it.h = item / per_head;
        const int rem = item - it.h * per_head;
        it.i = g.nbv + rem / P.nsplit;
        it.e0 = (rem % P.nsplit) * kTextChunk;
    } else {
        it.split = false;
        const int v = item - P.n_text_items;
        it.h = v / g.nbv;
        it.i = v - it.h * g.nbv;
        it.e0 = 0;
    }
    it.skip = P.head_mask != nullptr && P.head_mask[it.h] == 0;
    if (it.skip) {
        it.n = 0;
        return it;
    }
    const int c = P.cnt != nullptr ? P.cnt[(size_t)it.h * g.nb + it.i] : g.nb;
    if (c < 1 || c > g.nb) it.n = -1;   // invalid count: flagged by the epilogue
    else it.n = it.split ? max(0, min(c, it.e0 + kTextChunk) - it.e0) : c;
    return it;
}

__device__ inline float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Packed float32 pairs (fma.rn.f32x2 / add.rn.f32x2 run both lanes in one instruction).
__device__ inline unsigned long long pack2(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ inline float2 unpack2(unsigned long long r) {
    float2 v;
    asm("mov.b64 {%0,%1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
__device__ inline unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ inline unsigned long long add2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x on the FMA pipe, for x <= 8 (larger x is never passed here). Range reduction x = n + f
// with n = round(x) by the 1.5*2^23 magic-constant add, f in [-0.5, 0.5]; 2^f from a degree-3
// polynomial fitted by relative-error-weighted least squares (Lawson iterations) at Chebyshev
// nodes of [-0.5, 0.5]; then n is added to the exponent field. Max relative error 7.5e-5 for
// x >= -125 (well under the 2^-9 of the bf16 that P is rounded to); x below -125 is clamped
// there (2^-125 ~ 2.4e-38 stands in for 0, and keeps the exponent field normal).
constexpr float kExp2Clamp = -125.0f;
constexpr float kExp2Magic = 12582912.0f;     // 1.5 * 2^23: low mantissa bits hold round(x)
constexpr float kExp2C3 = 0.0551716648042202f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C0 = 0.9999280571937561f;

__device__ inline float exp2_fma(float x) {
    x = fmaxf(x, kExp2Clamp);
    const float t = x + kExp2Magic;
    const float f = x - (t - kExp2Magic);
    float p = fmaf(kExp2C3, f, kExp2C2);
    p = fmaf(p, f, kExp2C1);
    p = fmaf(p, f, kExp2C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// The same function on a pair, in packed float32x2 arithmetic (bit-identical results).
__device__ inline float2 exp2_fma_pair(float2 x) {
    const unsigned long long xx = pack2(fmaxf(x.x, kExp2Clamp), fmaxf(x.y, kExp2Clamp));
    const unsigned long long t = add2(xx, pack2(kExp2Magic, kExp2Magic));
    const unsigned long long n = add2(t, pack2(-kExp2Magic, -kExp2Magic));   // round(x), exact
    const unsigned long long f = fma2(n, pack2(-1.0f, -1.0f), xx);           // x - round(x), exact
    unsigned long long p = fma2(pack2(kExp2C3, kExp2C3), f, pack2(kExp2C2, kExp2C2));
    p = fma2(p, f, pack2(kExp2C1, kExp2C1));
    p = fma2(p, f, pack2(kExp2C0, kExp2C0));
    const float2 pv = unpack2(p), tv = unpack2(t);
    return make_float2(__int_as_float(__float_as_int(pv.x) + (__float_as_int(tv.x) << 23)),
                       __int_as_float(__float_as_int(pv.y) + (__float_as_int(tv.y) << 23)));
}

// Pairs e (of 16 per 32 keys) whose exponentials run on the FMA pipe instead of the MUFU:
// bit (e % 8) of this mask.
#ifndef BSA_SOFT_EXP_MASK
#define BSA_SOFT_EXP_MASK 0x00
#endif

__device__ inline float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Loader thread lt owns 16-byte chunk (lt % CH) of up to TPT consecutive rows of a tile: rows
// (lt / CH) * TPT + k below ROWS (G = kLoadThreads / CH row groups; the last one may be
// shorter). Its tokens come from the block-slot table in independent loads issued together, so
// one tile's tokens are a single round trip; K and V of a block share them.
template <int D, int ROWS>
struct RowToks {
    static constexpr int CH = D / 8;                      // 16-byte chunks per row
    static constexpr int G = kLoadThreads / CH;           // row groups
    static constexpr int TPT = (ROWS + G - 1) / G;        // rows per loader thread (at most)
    static_assert(kLoadThreads % CH == 0, "whole rows per loader pass");
    int t[TPT];
};

// Tokens of rows [block*B + (lt/CH)*TPT, +TPT); rows beyond the block, and padding slots,
// read token row 0 of the head: finite values that the softmax masks (keys) or the epilogue
// never stores (queries).
// Entries outside [0, N) (padding, or a bad caller-supplied key table) read a row in range.
template <int D, int ROWS>
__device__ inline RowToks<D, ROWS> load_tokens(const int* table, int B, int N, int block, int lt) {
    using RT = RowToks<D, ROWS>;
    RT rt;
    const int r0 = (lt / RT::CH) * RT::TPT;
#pragma unroll
    for (int k = 0; k < RT::TPT; ++k) {
        const int r = r0 + k;
        const int q = (r < ROWS && r < B) ? __ldg(table + block * B + r) : 0;
        rt.t[k] = min(max(q, 0), N - 1);
    }
    return rt;
}

template <int D, int ROWS>
__device__ inline void gather_tile(const RowToks<D, ROWS>& rt, const bsa_bf16* head_base,
                                   uint32_t tile_smem, int lt) {
    using RT = RowToks<D, ROWS>;
    const int c = lt % RT::CH;
    const int r0 = (lt / RT::CH) * RT::TPT;
#pragma unroll
    for (int k = 0; k < RT::TPT; ++k)
        if (r0 + k < ROWS)
            cp_async_16(tile_smem + sw128_offset(ROWS, r0 + k, c), head_base + (size_t)rt.t[k] * D + c * 8);
}

#ifdef BSA_TEST_HOOKS
// Test builds only (never in the product library): while set, CTA 0 withholds the arrival of
// its first query tile, so the MMA warp's bounded wait on it runs out and the launch takes
// the timeout path (BSA_ERR_TIMEOUT, every role winds down, TMEM is freed).
__device__ int g_test_withhold_q;
#endif

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1) sparse_attention_kernel(Params P) {
    using C = Cfg<D, BK>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    // the swizzled tiles need 1024-byte alignment: refuse to run (flagged, no access) without it
    if ((smem_u32(sm) & 1023u) != 0) {
        if (threadIdx.x == 0) raise_error(BSA_ERR_DEVICE_ARG);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 2;
    uint64_t* k_full = bars + 4;
    uint64_t* k_empty = k_full + NK;
    uint64_t* v_full = k_empty + NK;
    uint64_t* v_empty = v_full + NV;
    uint64_t* s_full = v_empty + NV;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* pv_done = p_full + 2;
    uint64_t* o_full = pv_done + 1;
    uint64_t* ml_ready = o_full + 2;
    uint64_t* o_free = ml_ready + 2;
    uint64_t* fin_bar = o_free + 2;
    uint64_t* m_ready = fin_bar + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_BAR + C::NBAR * 8);
    float* ml = reinterpret_cast<float*>(sm + C::OFF_ML);     // [ob][m0, l0, m1, l1][row]
    float* mch = reinterpret_cast<float*>(sm + C::OFF_MCH);   // [S buffer][row]

    const Geom& g = P.g;
    const int warp = threadIdx.x >> 5;
    const unsigned epoch = timeout_epoch();   // waits give up early only on a newer timeout
    const int nb = g.nb;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], kLoadThreads);
            mbar_init(&q_empty[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 1);
            mbar_init(&o_full[b], 1);
            mbar_init(&ml_ready[b], kSoftmaxThreads);
            mbar_init(&o_free[b], kEpiThreads);
        }
        for (int s = 0; s < NK; ++s) {
            mbar_init(&k_full[s], kLoadThreads);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(&v_full[s], kLoadThreads);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&p_full[b], kGroupThreads);
            mbar_init(&m_ready[b], kGroupThreads);
        }
        mbar_init(pv_done, 1);
        mbar_init(fin_bar, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const uint32_t sQ = smem_u32(sm + C::OFF_Q);
    const uint32_t sK = smem_u32(sm + C::OFF_K);
    const uint32_t sV = smem_u32(sm + C::OFF_V);
    const int first_item = blockIdx.x, stride = gridDim.x;

    auto kept_block = [&](const Item& it, int j) -> int {
        if (P.idx == nullptr) return it.e0 + j;
        int kb = P.idx[((size_t)it.h * nb + it.i) * nb + it.e0 + j];
        if (kb < 0 || kb >= nb) { raise_error(BSA_ERR_DEVICE_ARG); kb = 0; }
        return kb;
    };

    if (warp >= kLoadWarp0) {
        // ================================================================ loaders
        // Each loader thread gathers its share of a tile, then has the hardware arrive on the
        // tile's full barrier once its copies land (cp.async.mbarrier.arrive.noinc), so the
        // loaders run ahead as far as free stages allow.
        const int lt = threadIdx.x - kLoadWarp0 * 32;
        bool ok = true;
        int gblk = 0, k = 0;
        for (int item = first_item; item < P.n_items && ok; item += stride) {
            const Item it = decode_item(P, item);
            if (it.n <= 0) continue;
            const size_t head_off = (size_t)it.h * g.N * D;
            const int qb = k & 1;
            // tokens of the query block and of the first kept block, and the index of the
            // second kept block, are all in flight before the first wait
            // key and value rows come from the key-side table of this head
            const int* ktab = P.kperm != nullptr ? P.kperm + (size_t)it.h * nb * g.B : P.perm;
            const RowToks<D, BQ> tq = load_tokens<D, BQ>(P.perm, g.B, g.N, it.i, lt);
            RowToks<D, BK> tk = load_tokens<D, BK>(ktab, g.B, g.N, kept_block(it, 0), lt);
            int kb_ahead = it.n > 1 ? kept_block(it, 1) : 0;
            if (k >= 2) ok = mbar_wait(&q_empty[qb], ((k >> 1) - 1) & 1, epoch);
            if (!ok) break;
            gather_tile<D, BQ>(tq, P.Q + head_off, sQ + qb * C::Q_BYTES, lt);
#ifdef BSA_TEST_HOOKS
            if (!(k == 0 && blockIdx.x == 0 && *(volatile int*)&g_test_withhold_q != 0))
#endif
            cp_async_arrive_noinc(&q_full[qb]);
            for (int j = 0; j < it.n && ok; ++j, ++gblk) {
                const int ks = gblk % NK, vs = gblk % NV;
                const RowToks<D, BK> cur = tk;
                if (j + 1 < it.n) {          // prefetch: next block's tokens, index two ahead
                    tk = load_tokens<D, BK>(ktab, g.B, g.N, kb_ahead, lt);
                    if (j + 2 < it.n) kb_ahead = kept_block(it, j + 2);
                }
                if (gblk >= NK) ok = mbar_wait(&k_empty[ks], ((gblk / NK) - 1) & 1, epoch);
                if (!ok) break;
                gather_tile<D, BK>(cur, P.K + head_off, sK + ks * C::KV_BYTES, lt);
                cp_async_arrive_noinc(&k_full[ks]);
                if (gblk >= NV) ok = mbar_wait(&v_empty[vs], ((gblk / NV) - 1) & 1, epoch);
                if (!ok) break;
                gather_tile<D, BK>(cur, P.V + head_off, sV + vs * C::KV_BYTES, lt);
                cp_async_arrive_noinc(&v_full[vs]);
            }
            ++k;
        }
        cp_async_wait_all();   // no copy may still target shared memory at teardown
    } else if (warp == kMmaWarp) {
        // ================================================================ MMA issuer
        if (elect_one()) {
            bool ok = true;
            // PV for stream block gb, the j-th block of the item with local index kitem. P is
            // read from S buffer gb&1 (key k at column k/2: 8 columns per 16 keys).
            auto issue_pv = [&](int gb, int j, int kitem, bool last) -> bool {
                const int ob = kitem & 1;
                if (j == 0 && kitem >= 2 && !mbar_wait(&o_free[ob], ((kitem >> 1) - 1) & 1, epoch)) return false;
                if (!mbar_wait(&p_full[gb & 1], (gb >> 1) & 1, epoch)) return false;
                if (!mbar_wait(&v_full[gb % NV], (gb / NV) & 1, epoch)) return false;
                tc_fence_after();
                const uint32_t vbase = sV + (gb % NV) * C::KV_BYTES;
                const uint32_t pcol = tmem + C::TMEM_S + (gb & 1) * BK;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint64_t b = smem_desc_sw128(vbase + kk * 2048, C::KV_PANEL, 1024);
                    mma_bf16_ts(tmem + C::TMEM_O + ob * D, pcol + kk * 8, b, C::IDESC_PV,
                                (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(pv_done);
                tc_commit(&s_free[gb & 1]);
                tc_commit(&v_empty[gb % NV]);
                if (last) tc_commit(&o_full[ob]);
                return true;
            };
            int gblk = 0, k = 0;
            int prev_g = -1, prev_j = 0, prev_k = 0;
            bool prev_last = false;
            for (int item = first_item; item < P.n_items && ok; item += stride) {
                const Item it = decode_item(P, item);
                if (it.n <= 0) continue;
                const int qb = k & 1;
                ok = mbar_wait(&q_full[qb], (k >> 1) & 1, epoch);
                for (int j = 0; j < it.n && ok; ++j, ++gblk) {
                    const int ks = gblk % NK, sb = gblk & 1;
                    ok = mbar_wait(&k_full[ks], (gblk / NK) & 1, epoch);
                    if (ok && gblk >= 2) ok = mbar_wait(&s_free[sb], ((gblk >> 1) - 1) & 1, epoch);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t qbase = sQ + qb * C::Q_BYTES;
                    const uint32_t kbase = sK + ks * C::KV_BYTES;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = smem_desc_sw128(qbase + (kk >> 2) * C::Q_PANEL + (kk & 3) * 32, 16, 1024);
                        const uint64_t b = smem_desc_sw128(kbase + (kk >> 2) * C::KV_PANEL + (kk & 3) * 32, 16, 1024);
                        mma_bf16_ss(tmem + C::TMEM_S + sb * BK, a, b, C::IDESC_QK, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&s_full[sb]);
                    tc_commit(&k_empty[ks]);
                    if (j == it.n - 1) tc_commit(&q_empty[qb]);
                    if (prev_g >= 0) ok = issue_pv(prev_g, prev_j, prev_k, prev_last);
                    prev_g = gblk;
                    prev_j = j;
                    prev_k = k;
                    prev_last = (j == it.n - 1);
                }
                ++k;
            }
            if (ok && prev_g >= 0) ok = issue_pv(prev_g, prev_j, prev_k, prev_last);
            // every MMA issued by this thread has completed once fin_bar flips
            tc_commit(fin_bar);
            mbar_drain(fin_bar, 0);
        }
        __syncwarp();
    } else if (warp < kEpiWarp0) {
        // ================================================================ softmax
        const int lane = threadIdx.x & 31;
        const int quarter = warp & 3;                    // TMEM lane quarter
        const int grp = warp >> 2;                       // owns the blocks g with g%2 == grp
        const int r = quarter * 32 + lane;               // query row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t s_col = lane_base + C::TMEM_S + grp * BK;
        const unsigned long long scale2 = pack2(P.scale_log2, P.scale_log2);
        bool ok = true;
        int gblk = 0, k = 0;
        for (int item = first_item; item < P.n_items && ok; item += stride) {
            const Item it = decode_item(P, item);
            if (it.n <= 0) continue;                     // the epilogue warps write zeros
            const int ob = k & 1;
            const uint32_t o_col = lane_base + C::TMEM_O + ob * D;
            // this group's reference max (log2 units) and row sum relative to it
            float mref = -INFINITY, l = 0.f;
            const int j0 = (gblk & 1) == grp ? 0 : 1;    // this group's first block of the item
            int kb = j0 < it.n ? kept_block(it, j0) : 0;
            for (int j = j0; j < it.n && ok; j += 2) {
                const int g_cur = gblk + j;              // stream index of this block
                const int kcount = block_count(g, kb);
                if (j + 2 < it.n) kb = kept_block(it, j + 2);   // prefetch for the next block
                ok = __all_sync(0xffffffffu, mbar_wait(&s_full[grp], (g_cur >> 1) & 1, epoch));
                if (!ok) break;
                tc_fence_after();
                // pass 1: max of the row's raw scores (padding keys excluded)
                float mx = -INFINITY;
#pragma unroll 1
                for (int c = 0; c < BK / 32; ++c) {
                    uint32_t t[32];
                    tmem_ld32(s_col + c * 32, t);
                    tmem_wait_ld();
                    if (kcount >= BK) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) mx = max3(mx, __uint_as_float(t[e]), __uint_as_float(t[e + 1]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (c * 32 + e < kcount) mx = fmaxf(mx, __uint_as_float(t[e]));
                    }
                }
                const float m_blk = mx * P.scale_log2;
                // reference max chain: block g takes the previous block's reference (published
                // by the other group) and moves it only when its own max exceeds it by more
                // than 2^8; the first block of an item starts afresh. Every block waits for
                // its predecessor's entry, which keeps the two groups' entries in step.
                float mprev = -INFINITY;
                if (g_cur >= 1) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&m_ready[grp ^ 1], ((g_cur - 1) >> 1) & 1, epoch));
                    if (!ok) break;
                    mprev = mch[(grp ^ 1) * BQ + r];
                }
                const float m = (j == 0 || m_blk > mprev + kRescaleLog2) ? m_blk : mprev;
                mch[grp * BQ + r] = m;
                mbar_arrive(&m_ready[grp]);
                // this group's sum follows its own reference
                if (mref != -INFINITY && m != mref) l *= ex2(mref - m);
                mref = m;
                // pass 2: P = 2^(s*scale - m) as bf16 pairs, key k at column k/2 of the buffer
                const unsigned long long negm2 = pack2(-m, -m);
                unsigned long long sum2 = pack2(0.f, 0.f);
#pragma unroll 1
                for (int c = 0; c < BK / 32; ++c) {
                    uint32_t t[32];
                    tmem_ld32(s_col + c * 32, t);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 x = unpack2(fma2(pack2(__uint_as_float(t[2 * e]), __uint_as_float(t[2 * e + 1])),
                                                      scale2, negm2));
                        float p0, p1;
                        if ((BSA_SOFT_EXP_MASK >> (e % 8)) & 1) {
                            const float2 q = exp2_fma_pair(x);
                            p0 = q.x;
                            p1 = q.y;
                        } else {
                            p0 = ex2(x.x);
                            p1 = ex2(x.y);
                        }
                        if (kcount < BK) {
                            if (c * 32 + 2 * e >= kcount) p0 = 0.f;
                            if (c * 32 + 2 * e + 1 >= kcount) p1 = 0.f;
                        }
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                        pk[e] = *reinterpret_cast<uint32_t*>(&b2);
                        sum2 = add2(sum2, pack2(p0, p1));
                    }
                    // keys [32c, 32c+32) -> P columns [16c, 16c+16): S columns already read
                    tmem_st16(s_col + c * 16, pk);
                }
                const float2 sum = unpack2(sum2);
                l += sum.x + sum.y;
                // O holds the PVs of the blocks before this one at reference mprev: rescale it
                // (whole warp, when any of its rows moved) once the previous PV is done.
                // pv_done is at most one phase ahead of block g-1 here (S of this block was
                // issued after the PV two blocks back completed, and PV of this block waits
                // for p_full), so a parity wait is exact even though most blocks skip it.
                if (j >= 1 && __any_sync(0xffffffffu, m != mprev)) {
                    ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (g_cur - 1) & 1, epoch));
                    if (!ok) break;
                    tc_fence_after();
                    const float alpha = ex2(mprev - m);   // 1 for rows that kept their max
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(o_col + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(o_col + c * 32, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[grp]);
            }
            if (!ok) break;
            gblk += it.n;
            // hand this group's reference max and row sum to the epilogue; O buffer ob (and
            // its slots) must have been released by the epilogue of the item two back
            if (k >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&o_free[ob], ((k >> 1) - 1) & 1, epoch));
            if (!ok) break;
            ml[(ob * 4 + 2 * grp) * BQ + r] = mref;
            ml[(ob * 4 + 2 * grp + 1) * BQ + r] = l;
            mbar_arrive(&ml_ready[ob]);
            ++k;
        }
    } else if (warp < kMmaWarp) {
        // ================================================================ epilogue
        const int quarter = warp - kEpiWarp0;
        const int r = quarter * 32 + (threadIdx.x & 31);  // query row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        bool ok = true;
        int k = 0;
        int item = first_item;
        Item it;
        if (item < P.n_items) it = decode_item(P, item);
        while (item < P.n_items && ok) {
            const int next_item = item + stride;
            Item nxt;
            if (next_item < P.n_items) nxt = decode_item(P, next_item);   // prefetched
            const size_t head_off = (size_t)it.h * g.N * D;
            const int q_token = (r < g.B) ? __ldg(P.perm + it.i * g.B + r) : -1;
            if (it.skip) {
                // head masked out: nothing to write
            } else if (it.n <= 0) {
                // nothing kept (an empty text chunk, or an invalid count): zero output
                if (it.n < 0 && r == 0) raise_error(BSA_ERR_DEVICE_ARG);
                if (it.split) {
                    float* po = P.part_o + ((size_t)item * BQ + r) * D;
                    for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(po + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                    P.part_lse[(size_t)item * BQ + r] = -INFINITY;
                } else if (q_token >= 0) {
                    bsa_bf16* orow = P.O + head_off + (size_t)q_token * D;
                    for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
                    if (P.lse != nullptr) P.lse[(size_t)it.h * g.N + q_token] = -INFINITY;
                }
            } else {
                const int ob = k & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&o_full[ob], (k >> 1) & 1, epoch));
                if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&ml_ready[ob], (k >> 1) & 1, epoch));
                if (!ok) break;
                tc_fence_after();
                // O is relative to the reference of the item's last block, the larger of the two
                // groups' final references; each group's sum is relative to its own
                const float m0 = ml[(ob * 4 + 0) * BQ + r], l0 = ml[(ob * 4 + 1) * BQ + r];
                const float m1 = ml[(ob * 4 + 2) * BQ + r], l1 = ml[(ob * 4 + 3) * BQ + r];
                const float m = fmaxf(m0, m1);
                const float l = (l0 > 0.f ? l0 * ex2(m0 - m) : 0.f) + (l1 > 0.f ? l1 * ex2(m1 - m) : 0.f);
                const float inv = 1.0f / l;
                const uint32_t o_col = lane_base + C::TMEM_O + ob * D;
                if (it.split) {
                    float* po = P.part_o + ((size_t)item * BQ + r) * D;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t t[32];
                        tmem_ld32(o_col + c * 32, t);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(po + c * 32 + e) =
                                make_float4(__uint_as_float(t[e]) * inv, __uint_as_float(t[e + 1]) * inv,
                                            __uint_as_float(t[e + 2]) * inv, __uint_as_float(t[e + 3]) * inv);
                    }
                    P.part_lse[(size_t)item * BQ + r] = m + __log2f(l);
                } else {
                    if (P.lse != nullptr && q_token >= 0) P.lse[(size_t)it.h * g.N + q_token] = m + __log2f(l);
                    // 64 columns at a time: the warp's 32 rows go through a 128B-swizzled staging
                    // tile in shared memory so that each global store instruction writes four
                    // whole 128-byte row segments
                    const uint32_t stg = smem_u32(sm + C::OFF_STG) + (warp - kEpiWarp0) * 32 * 128;
                    const int lane = threadIdx.x & 31;
#pragma unroll 1
                    for (int hc = 0; hc < D / 64; ++hc) {
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            uint32_t t[32];
                            tmem_ld32(o_col + hc * 64 + c * 32, t);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; e += 8) {
                                uint32_t pk[4];
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(t[e + 2 * u]) * inv,
                                                                              __uint_as_float(t[e + 2 * u + 1]) * inv);
                                    pk[u] = *reinterpret_cast<uint32_t*>(&b2);
                                }
                                const int chunk = c * 4 + e / 8;
                                st_shared_v4(stg + lane * 128 + ((chunk ^ (lane & 7)) << 4), pk);
                            }
                        }
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int row = i * 4 + (lane >> 3), chunk = lane & 7;
                            const int tok = __shfl_sync(0xffffffffu, q_token, row);
                            const uint4 v = ld_shared_v4(stg + row * 128 + ((chunk ^ (row & 7)) << 4));
                            if (tok >= 0)
                                *reinterpret_cast<uint4*>(P.O + head_off + (size_t)tok * D + hc * 64 + chunk * 8) = v;
                        }
                        __syncwarp();
                    }
                }
                tc_fence_before();
                mbar_arrive(&o_free[ob]);            // O buffer and its m, l are free again
                ++k;
            }
            item = next_item;
            it = nxt;
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// grid (heads * nbt, BQ), D threads: merges the partial rows of one text query row.
template <int D>
__global__ void merge_text_kernel(Params P) {
    const Geom& g = P.g;
    const int hr = blockIdx.x, r = blockIdx.y;
    const int h = hr / g.nbt, ti = hr - h * g.nbt;
    const int i = g.nbv + ti;
    if (r >= g.B) return;
    if (P.head_mask != nullptr && P.head_mask[h] == 0) return;
    const int tok = P.perm[i * g.B + r];
    if (tok < 0) return;
    const int first = (h * g.nbt + ti) * P.nsplit;
    float mx = -INFINITY;
    for (int c = 0; c < P.nsplit; ++c) mx = fmaxf(mx, P.part_lse[(size_t)(first + c) * BQ + r]);
    float wsum = 0.f, acc = 0.f;
    for (int c = 0; c < P.nsplit; ++c) {
        const float lse = P.part_lse[(size_t)(first + c) * BQ + r];
        if (lse == -INFINITY) continue;
        const float w = exp2f(lse - mx);
        wsum += w;
        acc += w * P.part_o[((size_t)(first + c) * BQ + r) * D + threadIdx.x];
    }
    const float o = wsum > 0.f ? acc / wsum : 0.f;
    P.O[(size_t)h * g.N * D + (size_t)tok * D + threadIdx.x] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    if (P.lse != nullptr && threadIdx.x == 0)
        P.lse[(size_t)h * g.N + tok] = wsum > 0.f ? mx + log2f(wsum) : -INFINITY;
}

}  // namespace attn
}  // namespace bsa
