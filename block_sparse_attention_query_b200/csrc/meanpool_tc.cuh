// Mean-pooled block scorer on tcgen05 tensor cores (PARK: Accurate Block Retrieval for Sparse
// Attention in Video Diffusion Transformers, Abstract: block retrieval from the averaged
// representations of query and key blocks).
//
//   S[h][i][j] = softmax_j(qbar_i . kbar_j / sqrt(d))
//
// Float32-grade logits from bf16 tensor cores: both pooled operands (float32) are split into
// three bf16 parts x = hi + mid + lo (hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid);
// 24 significant bits), and the six part products down to relative order 2^-16
//   mid.mid + lo.hi + hi.lo + mid.hi + hi.mid + hi.hi     (issued in this order)
// accumulate in fp32 TMEM; the dropped terms are of order 2^-24 of the logit, the size of a
// float32 rounding.
//
// Persistent kernel, one CTA per SM, work item = (head, tile of 128 pooled query rows, share of
// the key tiles: all of them, or one of two halves when there are too few items to fill the
// SMs twice). Key blocks come in tiles of 64 (one MMA N), one pass: per tile, each query row's
// scaled logits (log2 units) go to the output row through a padded staging tile (each store
// instruction writes 32 consecutive entries of one row) while the row keeps an online max m and
// sum l of 2^logit; after the item's last tile the row's log-sum-exp m + log2 l over its share
// goes to rowoff, and normalize_rows_kernel combines the shares and rewrites every row as
// 2^(logit - lse).
// Roles (224 threads): warps 0-3 softmax (thread r = pooled query row r = TMEM lane r), warp 4
// MMA issuer + TMEM allocation, warps 5-6 loaders (contiguous split rows, 16-byte cp.async).
// Every wait is bounded.
#pragma once

#include "bsa_common.cuh"
#include "park_tc.cuh"

namespace bsa {
namespace mp {

constexpr int BQ = 128;                 // pooled query rows per item (MMA M)
constexpr int NT = 64;                  // key blocks per tile (MMA N)
constexpr int kSoftmaxThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp0 = 5;
constexpr int kLoadThreads = 64;
constexpr int kThreads = kSoftmaxThreads + 32 + kLoadThreads;   // 224
constexpr int NS = 2;                   // key-split tile stages

template <int D>
struct Cfg {
    static constexpr int QS_BYTES = BQ * D * 2;              // one split of the query tile
    static constexpr int KT_BYTES = NT * D * 2;              // one split of one key tile
    static constexpr int STAGE_BYTES = 3 * KT_BYTES;
    static constexpr int OFF_Q = 0;                          // 3 splits, single buffer
    static constexpr int OFF_K = OFF_Q + 3 * QS_BYTES;       // NS stages of 3 splits
    static constexpr int OFF_STG = OFF_K + NS * STAGE_BYTES; // [4 warps][32 rows][33] fp32 staging
    static constexpr int OFF_BAR = OFF_STG + 4 * 32 * 33 * 4;
    // q_full q_empty k_full[NS] k_empty[NS] l_full[2] l_free[2] fin
    static constexpr int NBAR = 2 + 2 * NS + 4 + 1;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 8;
    static constexpr int TMEM_COLS = 128;                    // 2 logit buffers of NT columns
    static constexpr int Q_PANEL = BQ * 128;
    static constexpr int KT_PANEL = NT * 128;
    static constexpr uint32_t IDESC = idesc_bf16_f32(BQ, NT, 0, 0);
    static_assert(SMEM <= 232448, "shared memory budget");
};

// The six (query part, key part) products, SMALLEST first: the tensor cores round the fp32
// accumulator at every K step, so each step costs up to an ulp of the accumulator's current
// size. Accumulating the correction products while the sum is still small, and the large
// hi.hi product last, leaves only hi.hi's own K steps at full size.
__device__ constexpr int kProdA[6] = {1, 2, 0, 1, 0, 0};
__device__ constexpr int kProdB[6] = {1, 0, 2, 0, 1, 0};

struct Params {
    Geom g;
    const bsa_bf16* qsplit;   // [heads][3][nbq][D] bf16: hi, mid, lo of the pooled queries
    const bsa_bf16* ksplit;   // [heads][3][nbp][D] bf16: hi, mid, lo of the pooled keys
    const int* head_mask;
    float* scores;
    float* rowoff;            // [heads][nb][nsplit] log-sum-exp (log2 units) of each row's share
    int nsplit;               // shares of the key tiles per (head, query tile): 1 or 2
    int tps;                  // key tiles per share
    int nbq;                  // nb rounded up to a multiple of BQ
    int nbp;                  // nb rounded up to a multiple of NT
    int n_items;              // heads * nbq / BQ * nsplit
    float scale_log2;         // log2(e) / sqrt(d)
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) meanpool_tc_kernel(Params P) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    if ((smem_u32(sm) & 1023u) != 0) {
        if (threadIdx.x == 0) raise_error(BSA_ERR_DEVICE_ARG);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 1;
    uint64_t* k_full = bars + 2;
    uint64_t* k_empty = k_full + NS;
    uint64_t* l_full = k_empty + NS;
    uint64_t* l_free = l_full + 2;
    uint64_t* fin_bar = l_free + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_BAR + C::NBAR * 8);

    const Geom& g = P.g;
    const int warp = threadIdx.x >> 5;
    const unsigned epoch = timeout_epoch();   // waits give up early only on a newer timeout
    const int nb = g.nb;
    const int ntiles = P.nbp / NT;
    const int qtiles = P.nbq / BQ;

    if (threadIdx.x == 0) {
        mbar_init(q_full, kLoadThreads);
        mbar_init(q_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&l_full[b], 1);
            mbar_init(&l_free[b], kSoftmaxThreads);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], kLoadThreads);
            mbar_init(&k_empty[s], 1);
        }
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

    auto skip_item = [&](int item) -> bool {
        const int h = item / (qtiles * P.nsplit);
        return P.head_mask != nullptr && P.head_mask[h] == 0;
    };
    // item -> head, query tile, key tiles [t0, t1)
    auto decode = [&](int item, int& h, int& qt, int& t0, int& t1) {
        const int sp = item % P.nsplit, hq = item / P.nsplit;
        h = hq / qtiles;
        qt = hq - h * qtiles;
        t0 = sp * P.tps;
        t1 = min(ntiles, t0 + P.tps);
    };

    if (warp >= kLoadWarp0) {
        // ================================================================ loaders
        constexpr int CH = D / 8;                           // 16-byte chunks per row
        const int lt = threadIdx.x - kLoadWarp0 * 32;
        const int c = lt % CH;
        bool ok = true;
        int gt = 0, k = 0;
        for (int item = blockIdx.x; item < P.n_items && ok; item += gridDim.x) {
            if (skip_item(item)) continue;
            int h, qt, t0, t1;
            decode(item, h, qt, t0, t1);
            if (k >= 1) ok = mbar_wait(q_empty, (k - 1) & 1, epoch);
            if (!ok) break;
            const bsa_bf16* qh = P.qsplit + (size_t)h * 3 * P.nbq * D;
#pragma unroll
            for (int sp = 0; sp < 3; ++sp) {
                const bsa_bf16* src = qh + ((size_t)sp * P.nbq + (size_t)qt * BQ) * D;
                for (int r = lt / CH; r < BQ; r += kLoadThreads / CH)
                    cp_async_16(sQ + sp * C::QS_BYTES + sw128_offset(BQ, r, c), src + (size_t)r * D + c * 8);
            }
            cp_async_arrive_noinc(q_full);
            const bsa_bf16* kh = P.ksplit + (size_t)h * 3 * P.nbp * D;
            for (int t = t0; t < t1 && ok; ++t, ++gt) {
                const int s = gt % NS;
                if (gt >= NS) ok = mbar_wait(&k_empty[s], ((gt / NS) - 1) & 1, epoch);
                if (!ok) break;
#pragma unroll
                for (int sp = 0; sp < 3; ++sp) {
                    const bsa_bf16* src = kh + ((size_t)sp * P.nbp + (size_t)t * NT) * D;
                    for (int r = lt / CH; r < NT; r += kLoadThreads / CH)
                        cp_async_16(sK + s * C::STAGE_BYTES + sp * C::KT_BYTES + sw128_offset(NT, r, c),
                                    src + (size_t)r * D + c * 8);
                }
                cp_async_arrive_noinc(&k_full[s]);
            }
            ++k;
        }
        cp_async_wait_all();   // no copy may still target shared memory at teardown
    } else if (warp == kMmaWarp) {
        // ================================================================ MMA issuer
        if (elect_one()) {
            bool ok = true;
            int gt = 0, k = 0;
            for (int item = blockIdx.x; item < P.n_items && ok; item += gridDim.x) {
                if (skip_item(item)) continue;
                int h, qt, t0, t1;
                decode(item, h, qt, t0, t1);
                ok = mbar_wait(q_full, k & 1, epoch);
                for (int t = t0; t < t1 && ok; ++t, ++gt) {
                    const int s = gt % NS, lb = gt & 1;
                    ok = mbar_wait(&k_full[s], (gt / NS) & 1, epoch);
                    if (ok && gt >= 2) ok = mbar_wait(&l_free[lb], ((gt >> 1) - 1) & 1, epoch);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int pr = 0; pr < 6; ++pr) {
                        const uint32_t qbase = sQ + kProdA[pr] * C::QS_BYTES;
                        const uint32_t kbase = sK + s * C::STAGE_BYTES + kProdB[pr] * C::KT_BYTES;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t a = smem_desc_sw128(qbase + (kk >> 2) * C::Q_PANEL + (kk & 3) * 32, 16, 1024);
                            const uint64_t b = smem_desc_sw128(kbase + (kk >> 2) * C::KT_PANEL + (kk & 3) * 32, 16, 1024);
                            mma_bf16_ss(tmem + lb * NT, a, b, C::IDESC, (pr > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(&l_full[lb]);
                    tc_commit(&k_empty[s]);
                    if (t == t1 - 1) tc_commit(q_empty);
                }
                ++k;
            }
            tc_commit(fin_bar);
            mbar_drain(fin_bar, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ softmax
        const int r = threadIdx.x;                       // pooled query row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        bool ok = true;
        int gt = 0;
        for (int item = blockIdx.x; item < P.n_items && ok; item += gridDim.x) {
            if (skip_item(item)) continue;
            int h, qt, t0, t1;
            decode(item, h, qt, t0, t1);
            const int sp = item % P.nsplit;
            float m = -INFINITY, l = 0.f;
            const int lane = r & 31;
            float* stg = reinterpret_cast<float*>(sm + C::OFF_STG) + warp * 32 * 33;
            const int row0 = qt * BQ + warp * 32;           // the warp's first query block
            for (int t = t0; t < t1 && ok; ++t, ++gt) {
                const int lb = gt & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&l_full[lb], (gt >> 1) & 1, epoch));
                if (!ok) break;
                tc_fence_after();
                uint32_t v0[32], v1[32];
                tmem_ld32(lane_base + lb * NT, v0);
                tmem_ld32(lane_base + lb * NT + 32, v1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&l_free[lb]);                // logits are in registers
                const int jbase = t * NT;
                float mx = -INFINITY;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    if (jbase + e < nb) mx = fmaxf(mx, __uint_as_float(v0[e]));
                    if (jbase + 32 + e < nb) mx = fmaxf(mx, __uint_as_float(v1[e]));
                }
                const float m_new = fmaxf(m, mx * P.scale_log2);
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    if (jbase + e < nb) s += park::ex2(fmaf(__uint_as_float(v0[e]), P.scale_log2, -m_new));
                    if (jbase + 32 + e < nb) s += park::ex2(fmaf(__uint_as_float(v1[e]), P.scale_log2, -m_new));
                }
                l = l * park::ex2(m - m_new) + s;
                m = m_new;
                // scaled logits to the rows, 32 columns at a time through the staging tile
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    const uint32_t* v = hc == 0 ? v0 : v1;
#pragma unroll
                    for (int e = 0; e < 32; ++e) stg[lane * 33 + e] = __uint_as_float(v[e]) * P.scale_log2;
                    __syncwarp();
                    const int j = jbase + hc * 32 + lane;
#pragma unroll 4
                    for (int rr = 0; rr < 32; ++rr) {
                        if (row0 + rr < nb && j < nb) P.scores[((size_t)h * nb + row0 + rr) * nb + j] = stg[rr * 33 + lane];
                    }
                    __syncwarp();
                }
            }
            if (!ok) break;
            if (row0 + lane < nb) P.rowoff[((size_t)h * nb + row0 + lane) * P.nsplit + sp] = m + __log2f(l);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// grid (heads * nb), 128 threads: row (h, i) of the scores, logits (log2 units) ->
// probabilities 2^(logit - lse), lse combining the row's nsplit shares (each share holds at
// least one real key block). Skips heads that were not scored.
__global__ void __launch_bounds__(128) normalize_rows_kernel(Geom g, const int* __restrict__ head_mask,
                                                             const float* __restrict__ rowoff, int nsplit,
                                                             float* __restrict__ scores) {
    const int row = blockIdx.x;
    const int h = row / g.nb;
    if (head_mask != nullptr && head_mask[h] == 0) return;
    float lse = rowoff[(size_t)row * nsplit];
    if (nsplit == 2) {
        const float b = rowoff[(size_t)row * nsplit + 1];
        const float mx = fmaxf(lse, b);
        lse = mx + __log2f(park::ex2(lse - mx) + park::ex2(b - mx));
    }
    const float off = -lse;
    float* p = scores + (size_t)row * g.nb;
    for (int j = threadIdx.x; j < g.nb; j += 128) p[j] = park::ex2(p[j] + off);
}

}  // namespace mp
}  // namespace bsa
