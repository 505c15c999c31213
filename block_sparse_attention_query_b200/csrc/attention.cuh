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
// Warp roles (352 threads):
//   warps 0-7  softmax + epilogue. Warp w owns query rows 32*(w%4) .. +31 (its TMEM lane
//              quarter) and column half w/4 of S, P and O. The two warps of a row group
//              exchange their half-row maxima once per block (bounded mbarrier), then each
//              writes P only over its own S columns.
//   warp 8     TMEM allocation; one elected thread issues every tcgen05.mma.
//   warps 9-10 loaders: gather Q / K / V rows of a block (raster rows from the block-slot
//              table) with 16-byte cp.async into 128B-swizzled K-major tiles; completion
//              arrives on the tile's mbarrier asynchronously.
// The kept blocks of all items of a CTA form one stream g = 0, 1, 2, ...:
//   S[g&1] = Q K_g^T (TMEM fp32) -> softmax: row max of the block (pass 1), P = 2^(s-m) as
//   bf16 pairs written back over S in TMEM (pass 2) -> O[item&1] += P V_g with P read from
//   TMEM (V is an MN-major smem operand). The reference max m only moves when a row max
//   grows by more than 2^8, so O (in TMEM) is rarely rescaled; P <= 2^8 fits bf16 and the
//   final division by the row sum is exact either way.
// S/P is double-buffered (QK^T of block g+1 overlaps the softmax of block g, and the
// softmax of block g+1 overlaps PV of block g); Q and O are double-buffered across items
// (the next item's loads and QK^T overlap this item's epilogue). Every wait is bounded: one that runs out raises BSA_ERR_TIMEOUT and all roles
// wind down. tcgen05.ld/st are warp-collective, so every condition around them is
// warp-uniform.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace attn {

constexpr int BQ = 128;                 // query rows per tile (MMA M)
constexpr int kSoftmaxThreads = 256;    // 8 warps: 2 per row group, each half the columns
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp0 = 9;
constexpr int kLoadThreads = 64;        // 11 warps in all: at most 3 per SM sub-partition
constexpr int kThreads = kSoftmaxThreads + 32 + kLoadThreads;   // 352
constexpr int NS = 2;                   // K and V pipeline stages
constexpr int kTextChunk = 64;          // kept blocks per work item of a text query row
constexpr float kRescaleLog2 = 8.0f;    // O is rescaled only when a row max grows by > 2^8

template <int D, int BK>
struct Cfg {
    static constexpr int Q_BYTES = BQ * D * 2;
    static constexpr int KV_BYTES = BK * D * 2;
    static constexpr int OFF_Q = 0;                          // 2 buffers
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;        // NS stages
    static constexpr int OFF_V = OFF_K + NS * KV_BYTES;      // NS stages
    static constexpr int OFF_STAGE = OFF_V + NS * KV_BYTES;  // bf16 O rows of one item
    static constexpr int OFF_STAGE_TOK = OFF_STAGE + BQ * D * 2;
    // [2 slots][2 halves][BQ]: half-row maxima of a block (slot = block parity); during an
    // epilogue the slot of the next block holds the two halves' row sums instead
    static constexpr int OFF_PMAX = OFF_STAGE_TOK + BQ * 4;
    static constexpr int OFF_BAR = OFF_PMAX + 4 * BQ * 4;
    // q_full[2] q_empty[2] k_full[NS] v_full[NS] k_empty[NS] v_empty[NS] s_full[2] s_free[2]
    // p_full pv_done o_free[2] fin stage  (s_free[b]: the PV that read P out of S buffer b is
    // done; stage: the 128 softmax threads meet around the epilogue's staging tile)
    static constexpr int NBAR = 4 + 4 * NS + 4 + 2 + 2 + 1 + 1 + 4;   // + pair[4]
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 8;         // +8: TMEM address slot
    static constexpr int TMEM_S = 0;            // S buffers: [0, 2*BK); P (bf16 pairs) overwrites
                                                // the first BK/2 columns of its S buffer
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
    const int* idx;
    const int* cnt;
    const int* perm;    // [nb*B] raster token of every block slot, -1 = padding
    bsa_bf16* O;
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
    const int c = P.cnt[(size_t)it.h * g.nb + it.i];
    if (c < 1 || c > g.nb) it.n = -1;   // invalid count: flagged by the softmax role
    else it.n = it.split ? max(0, min(c, it.e0 + kTextChunk) - it.e0) : c;
    return it;
}

__device__ inline float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x on the FMA pipe, for x <= 8 (larger x is never passed here). Range reduction x = n + f
// with n = round(x) by the 1.5*2^23 magic-constant add, f in [-0.5, 0.5]; 2^f from a degree-3
// polynomial fitted by relative-error-weighted least squares (Lawson iterations) at Chebyshev
// nodes of [-0.5, 0.5]; then n is added to the exponent field. Max relative error 7.5e-5 for
// x >= -125 (well under the 2^-9 of the bf16 that P is rounded to); x below -125 is clamped
// there (2^-125 ~ 2.4e-38 stands in for 0, and keeps the exponent field normal).
__device__ inline float exp2_fma(float x) {
    x = fmaxf(x, -125.0f);
    const float t = x + 12582912.0f;            // 1.5 * 2^23: low mantissa bits hold round(x)
    const float f = x - (t - 12582912.0f);
    float p = fmaf(0.0551716648042202f, f, 0.2426111251115799f);
    p = fmaf(p, f, 0.6932609677314758f);
    p = fmaf(p, f, 0.9999280571937561f);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
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

// Loader thread lt owns 16-byte chunk (lt % CH) of TPT consecutive rows of a tile: rows
// (lt / CH) * TPT + k. Its tokens come from the block-slot table in TPT/4 int4 loads, so
// one tile's tokens are a single round trip; K and V of a block share them.
template <int D, int ROWS>
struct RowToks {
    static constexpr int CH = D / 8;                      // 16-byte chunks per row
    static constexpr int TPT = ROWS * CH / kLoadThreads;  // rows per loader thread
    static_assert(TPT % 4 == 0, "whole int4 loads");
    int t[TPT];
};

// Tokens of rows [block*B + (lt/CH)*TPT, +TPT); rows beyond the block, and padding slots,
// read token row 0 of the head: finite values that the softmax masks (keys) or the epilogue
// never stores (queries).
template <int D, int ROWS>
__device__ inline RowToks<D, ROWS> load_tokens(const Params& P, int block, int lt) {
    using RT = RowToks<D, ROWS>;
    RT rt;
    const int r0 = (lt / RT::CH) * RT::TPT;
    const int B = P.g.B;
#pragma unroll
    for (int v = 0; v < RT::TPT / 4; ++v) {
        int4 q = make_int4(0, 0, 0, 0);
        if (r0 + 4 * v < B) q = __ldg(reinterpret_cast<const int4*>(P.perm + block * B + r0 + 4 * v));
        rt.t[4 * v + 0] = max(q.x, 0);
        rt.t[4 * v + 1] = max(q.y, 0);
        rt.t[4 * v + 2] = max(q.z, 0);
        rt.t[4 * v + 3] = max(q.w, 0);
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
        cp_async_16(tile_smem + sw128_offset(ROWS, r0 + k, c), head_base + (size_t)rt.t[k] * D + c * 8);
}

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
    uint64_t* v_full = k_full + NS;
    uint64_t* k_empty = v_full + NS;
    uint64_t* v_empty = k_empty + NS;
    uint64_t* s_full = v_empty + NS;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* pv_done = p_full + 1;
    uint64_t* o_free = pv_done + 1;
    uint64_t* fin_bar = o_free + 2;
    uint64_t* stage_bar = fin_bar + 1;
    uint64_t* pair_bar = stage_bar + 1;   // [4]: the two warps of a TMEM lane quarter
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_BAR + C::NBAR * 8);

    const Geom& g = P.g;
    const int warp = threadIdx.x >> 5;
    const int nb = g.nb;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], kLoadThreads);
            mbar_init(&q_empty[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 1);
            mbar_init(&o_free[b], kSoftmaxThreads);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], kLoadThreads);
            mbar_init(&v_full[s], kLoadThreads);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(p_full, kSoftmaxThreads);
        mbar_init(pv_done, 1);
        mbar_init(fin_bar, 1);
        mbar_init(stage_bar, kSoftmaxThreads);
        for (int q = 0; q < 4; ++q) mbar_init(&pair_bar[q], 64);
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
            const RowToks<D, BQ> tq = load_tokens<D, BQ>(P, it.i, lt);
            RowToks<D, BK> tk = load_tokens<D, BK>(P, kept_block(it, 0), lt);
            int kb_ahead = it.n > 1 ? kept_block(it, 1) : 0;
            if (k >= 2) ok = mbar_wait(&q_empty[qb], ((k >> 1) - 1) & 1);
            if (!ok) break;
            gather_tile<D, BQ>(tq, P.Q + head_off, sQ + qb * C::Q_BYTES, lt);
            cp_async_arrive_noinc(&q_full[qb]);
            for (int j = 0; j < it.n && ok; ++j, ++gblk) {
                const int s = gblk % NS;
                const RowToks<D, BK> cur = tk;
                if (j + 1 < it.n) {          // prefetch: next block's tokens, index two ahead
                    tk = load_tokens<D, BK>(P, kb_ahead, lt);
                    if (j + 2 < it.n) kb_ahead = kept_block(it, j + 2);
                }
                if (gblk >= NS) ok = mbar_wait(&k_empty[s], ((gblk / NS) - 1) & 1);
                if (!ok) break;
                gather_tile<D, BK>(cur, P.K + head_off, sK + s * C::KV_BYTES, lt);
                cp_async_arrive_noinc(&k_full[s]);
                if (gblk >= NS) ok = mbar_wait(&v_empty[s], ((gblk / NS) - 1) & 1);
                if (!ok) break;
                gather_tile<D, BK>(cur, P.V + head_off, sV + s * C::KV_BYTES, lt);
                cp_async_arrive_noinc(&v_full[s]);
            }
            ++k;
        }
        cp_async_wait<0>();   // no copy may still target shared memory at teardown
    } else if (warp == kMmaWarp) {
        // ================================================================ MMA issuer
        if (elect_one()) {
            bool ok = true;
            // PV for stream block gb, the j-th block of the item with local index kitem. P is
            // read from the first BK/4 columns of each column half of S buffer gb&1: key k of
            // half h sits at column h*BK/2 + (k - h*BK/2)/2.
            auto issue_pv = [&](int gb, int j, int kitem) -> bool {
                const int ob = kitem & 1;
                if (j == 0 && kitem >= 2 && !mbar_wait(&o_free[ob], ((kitem >> 1) - 1) & 1)) return false;
                if (!mbar_wait(p_full, gb & 1)) return false;
                if (!mbar_wait(&v_full[gb % NS], (gb / NS) & 1)) return false;
                tc_fence_after();
                const uint32_t vbase = sV + (gb % NS) * C::KV_BYTES;
                const uint32_t pcol = tmem + C::TMEM_S + (gb & 1) * BK;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const int hk = kk / (BK / 32);
                    const uint32_t acol = kk * 8 + hk * (BK / 4);
                    const uint64_t b = smem_desc_sw128(vbase + kk * 2048, C::KV_PANEL, 1024);
                    mma_bf16_ts(tmem + C::TMEM_O + ob * D, pcol + acol, b, C::IDESC_PV,
                                (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(pv_done);
                tc_commit(&s_free[gb & 1]);
                tc_commit(&v_empty[gb % NS]);
                return true;
            };
            int gblk = 0, k = 0;
            int prev_g = -1, prev_j = 0, prev_k = 0;
            for (int item = first_item; item < P.n_items && ok; item += stride) {
                const Item it = decode_item(P, item);
                if (it.n <= 0) continue;
                const int qb = k & 1;
                ok = mbar_wait(&q_full[qb], (k >> 1) & 1);
                for (int j = 0; j < it.n && ok; ++j, ++gblk) {
                    const int s = gblk % NS, sb = gblk & 1;
                    ok = mbar_wait(&k_full[s], (gblk / NS) & 1);
                    if (ok && gblk >= 2) ok = mbar_wait(&s_free[sb], ((gblk >> 1) - 1) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t qbase = sQ + qb * C::Q_BYTES;
                    const uint32_t kbase = sK + s * C::KV_BYTES;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = smem_desc_sw128(qbase + (kk >> 2) * C::Q_PANEL + (kk & 3) * 32, 16, 1024);
                        const uint64_t b = smem_desc_sw128(kbase + (kk >> 2) * C::KV_PANEL + (kk & 3) * 32, 16, 1024);
                        mma_bf16_ss(tmem + C::TMEM_S + sb * BK, a, b, C::IDESC_QK, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&s_full[sb]);
                    tc_commit(&k_empty[s]);
                    if (j == it.n - 1) tc_commit(&q_empty[qb]);
                    if (prev_g >= 0) ok = issue_pv(prev_g, prev_j, prev_k);
                    prev_g = gblk;
                    prev_j = j;
                    prev_k = k;
                }
                ++k;
            }
            if (ok && prev_g >= 0) ok = issue_pv(prev_g, prev_j, prev_k);
            // every MMA issued by this thread has completed once fin_bar flips
            tc_commit(fin_bar);
            mbar_wait(fin_bar, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ softmax
        const int lane = threadIdx.x & 31;
        const int quarter = warp & 3;                    // TMEM lane quarter
        const int half = warp >> 2;                      // column half of S / P / O
        const int r = quarter * 32 + lane;               // query row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        constexpr int HB = BK / 2;                       // S / P columns of a half (keys)
        constexpr int HD = D / 2;                        // O columns of a half
        constexpr int CH = D / 8;                        // 16-byte chunks per O row
        const uint32_t s_stage = smem_u32(sm + C::OFF_STAGE);
        int* stage_tok = reinterpret_cast<int*>(sm + C::OFF_STAGE_TOK);
        float* pmax = reinterpret_cast<float*>(sm + C::OFF_PMAX);
        bool ok = true;
        uint32_t pair_phase = 0;
        int gblk = 0, k = 0;

        // The epilogue of a finished item is deferred until the next item's first block has
        // been handed to the MMA, so the item's last PV runs while that block is processed.
        struct Pending {
            bool active, split;
            int item, h, q_token, ob;
            float m, l;                                  // l: this half's partial row sum
        };
        Pending pend;
        pend.active = false;

        // all softmax threads meet here (bounded: a wait that runs out returns false)
        uint32_t stage_phase = 0;
        auto stage_sync = [&]() -> bool {
            mbar_arrive(stage_bar);
            const bool done = mbar_wait(stage_bar, stage_phase & 1);
            ++stage_phase;
            return __all_sync(0xffffffffu, done);
        };

        // gnext: index of the next block in the stream; its max-exchange slot is idle now
        auto epilogue = [&](const Pending& pe, int gnext) -> bool {
            const uint32_t o_col = lane_base + C::TMEM_O + pe.ob * D + half * HD;
            float* lsum = pmax + (gnext & 1) * 2 * BQ;
            // row sum: the two halves' partial sums meet in shared memory
            if (!stage_sync()) return false;         // previous epilogue done with the tile
            lsum[half * BQ + r] = pe.l;
            if (half == 0) stage_tok[r] = pe.split ? -1 : pe.q_token;
            uint32_t t0[32], t1[32];
            tmem_ld32(o_col, t0);
            if (HD > 32) tmem_ld32(o_col + 32, t1);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&o_free[pe.ob]);             // O has been read out of TMEM
            if (!stage_sync()) return false;         // both halves of lsum are written
            const float l = lsum[r] + lsum[BQ + r];
            const float inv = 1.0f / l;
            if (pe.split) {
                float* po = P.part_o + ((size_t)pe.item * BQ + r) * D + half * HD;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4*>(po + e) =
                        make_float4(__uint_as_float(t0[e]) * inv, __uint_as_float(t0[e + 1]) * inv,
                                    __uint_as_float(t0[e + 2]) * inv, __uint_as_float(t0[e + 3]) * inv);
                if (HD > 32) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(po + 32 + e) =
                            make_float4(__uint_as_float(t1[e]) * inv, __uint_as_float(t1[e + 1]) * inv,
                                        __uint_as_float(t1[e + 2]) * inv, __uint_as_float(t1[e + 3]) * inv);
                }
                if (half == 0) P.part_lse[(size_t)pe.item * BQ + r] = pe.m + __log2f(l);
                return stage_sync();                 // lsum slot read by every thread
            }
            // bf16 rows into the staging tile: 16-byte chunk c of row r at slot c ^ (r % CH)
#pragma unroll
            for (int u = 0; u < HD / 8; ++u) {
                const uint32_t* t = u < 4 ? t0 : t1;
                const int e0 = (u & 3) * 8;
                uint32_t pk[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(t[e0 + 2 * v]) * inv,
                                                              __uint_as_float(t[e0 + 2 * v + 1]) * inv);
                    pk[v] = *reinterpret_cast<uint32_t*>(&b2);
                }
                const int chunk = half * (HD / 8) + u;
                const uint32_t dst = s_stage + r * (D * 2) + ((chunk ^ (r & (CH - 1))) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(pk[0]), "r"(pk[1]),
                             "r"(pk[2]), "r"(pk[3]) : "memory");
            }
            if (!stage_sync()) return false;         // the tile is complete
            // coalesced write-out: warp w writes rows 16w .. 16w+15, CH lanes per row
            bsa_bf16* Oh = P.O + (size_t)pe.h * g.N * D;
            constexpr int RPI = 32 / CH;             // rows per instruction
            constexpr int NIT = 16 / RPI;
            const int cc = lane % CH;
            uint4 v[NIT];
            int tok[NIT];
#pragma unroll
            for (int q = 0; q < NIT; ++q) {
                const int R = warp * 16 + q * RPI + lane / CH;
                tok[q] = stage_tok[R];
                const uint32_t src = s_stage + R * (D * 2) + ((cc ^ (R & (CH - 1))) << 4);
                asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                             : "=r"(v[q].x), "=r"(v[q].y), "=r"(v[q].z), "=r"(v[q].w) : "r"(src));
            }
#pragma unroll
            for (int q = 0; q < NIT; ++q)
                if (tok[q] >= 0) *reinterpret_cast<uint4*>(Oh + (size_t)tok[q] * D + cc * 8) = v[q];
            return true;
        };

        int item = first_item;
        Item it;
        if (item < P.n_items) it = decode_item(P, item);
        while (item < P.n_items && ok) {
            const int next_item = item + stride;
            Item nxt;
            if (next_item < P.n_items) nxt = decode_item(P, next_item);   // prefetched
            const size_t head_off = (size_t)it.h * g.N * D;
            const int q_token = (r < g.B) ? __ldg(P.perm + it.i * g.B + r) : -1;
            if (it.n <= 0) {
                // nothing kept (an empty text chunk, or an invalid count): zero output
                if (it.n < 0 && threadIdx.x == 0) raise_error(BSA_ERR_DEVICE_ARG);
                if (it.split) {
                    float* po = P.part_o + ((size_t)item * BQ + r) * D + half * HD;
                    for (int c = 0; c < HD; c += 4) *reinterpret_cast<float4*>(po + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (half == 0) P.part_lse[(size_t)item * BQ + r] = -INFINITY;
                } else if (q_token >= 0) {
                    bsa_bf16* orow = P.O + head_off + (size_t)q_token * D + half * HD;
                    for (int c = 0; c < HD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
                }
                item = next_item;
                it = nxt;
                continue;
            }
            const int ob = k & 1;
            const uint32_t o_col = lane_base + C::TMEM_O + ob * D + half * HD;
            float m = -INFINITY, l = 0.f;   // reference max (log2 units), this half's row sum
            int kb_next = kept_block(it, 0);
            for (int j = 0; j < it.n && ok; ++j, ++gblk) {
                const int sb = gblk & 1;
                const uint32_t s_col = lane_base + C::TMEM_S + sb * BK;
                const int kcount = block_count(g, kb_next);
                if (j + 1 < it.n) kb_next = kept_block(it, j + 1);   // prefetch for the next block
                ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (gblk >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
                // pass 1: max of this half's raw scores (padding keys excluded), then the two
                // halves of the row swap maxima so both use the same reference max
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < HB / 32; ++c) {
                    const int key0 = half * HB + c * 32;
                    uint32_t t[32];
                    tmem_ld32(s_col + key0, t);
                    tmem_wait_ld();
                    if (kcount >= BK) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) mx = max3(mx, __uint_as_float(t[e]), __uint_as_float(t[e + 1]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (key0 + e < kcount) mx = fmaxf(mx, __uint_as_float(t[e]));
                    }
                }
                {
                    float* slot = pmax + (gblk & 1) * 2 * BQ;
                    slot[half * BQ + r] = mx;
                    mbar_arrive(&pair_bar[quarter]);
                    ok = __all_sync(0xffffffffu, mbar_wait(&pair_bar[quarter], pair_phase & 1));
                    ++pair_phase;
                    if (!ok) break;
                    mx = fmaxf(mx, slot[(half ^ 1) * BQ + r]);
                }
                const float m_blk = mx * P.scale_log2;
                float alpha = 1.0f;
                if (j == 0) {
                    m = m_blk;
                } else if (m_blk > m + kRescaleLog2) {
                    alpha = ex2(m - m_blk);
                    m = m_blk;
                }
                // pass 2 on this half: P = 2^(s*scale - m) as bf16 pairs over the S columns
                const unsigned long long scale2 = pack2(P.scale_log2, P.scale_log2);
                const unsigned long long negm2 = pack2(-m, -m);
                unsigned long long sum2 = pack2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < HB / 32; ++c) {
                    const int key0 = half * HB + c * 32;         // first key of this chunk
                    uint32_t t[32];
                    tmem_ld32(s_col + key0, t);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 x = unpack2(fma2(pack2(__uint_as_float(t[2 * e]), __uint_as_float(t[2 * e + 1])),
                                                      scale2, negm2));
                        const bool soft = (BSA_SOFT_EXP_MASK >> (e % 8)) & 1;
                        float p0 = soft ? exp2_fma(x.x) : ex2(x.x);
                        float p1 = soft ? exp2_fma(x.y) : ex2(x.y);
                        if (kcount < BK) {
                            if (key0 + 2 * e >= kcount) p0 = 0.f;
                            if (key0 + 2 * e + 1 >= kcount) p1 = 0.f;
                        }
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                        pk[e] = *reinterpret_cast<uint32_t*>(&b2);
                        sum2 = add2(sum2, pack2(p0, p1));
                    }
                    // keys [key0, key0+32) -> P columns half*HB + (key0 - half*HB)/2 + [0,16),
                    // inside this half's S region and already read
                    tmem_st16(s_col + half * HB + (key0 - half * HB) / 2, pk);
                }
                const float2 sum = unpack2(sum2);
                const float rs = sum.x + sum.y;
                l = l * alpha + rs;
                if (j >= 1 || pend.active) {
                    // the previous PV (this item's, or the pending item's last) must be done
                    // before O may be rescaled or PV of this block is issued; every PV is
                    // waited for here, in order
                    ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (gblk - 1) & 1));
                    if (!ok) break;
                    tc_fence_after();
                    // the whole warp takes part when any of its rows moved its reference max
                    if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
                        for (int c = 0; c < HD / 32; ++c) {
                            uint32_t t[32];
                            tmem_ld32(o_col + c * 32, t);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
                            tmem_st32(o_col + c * 32, t);
                        }
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(p_full);
                if (j == 0 && pend.active) {
                    ok = epilogue(pend, gblk + 1);
                    pend.active = false;
                }
            }
            if (!ok) break;
            pend.active = true;
            pend.split = it.split;
            pend.item = item;
            pend.h = it.h;
            pend.q_token = q_token;
            pend.ob = ob;
            pend.m = m;
            pend.l = l;
            ++k;
            item = next_item;
            it = nxt;
        }
        if (ok && pend.active) {
            ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (gblk - 1) & 1));
            if (ok) {
                tc_fence_after();
                ok = epilogue(pend, gblk);
            }
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
}

}  // namespace attn
}  // namespace bsa
