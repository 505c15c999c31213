// PARK per-query-normalised block scorer on tcgen05 tensor cores (PARK: Accurate Block
// Retrieval for Sparse Attention in Video Diffusion Transformers, Abstract: every original
// query is kept, its attention over key blocks is normalised on its own, and the
// distributions are averaged within the query block).
//
//   P[h][i][j] = (1/n_i) * sum over real queries q of block i of softmax_j(q . kbar_j / sqrt(d))
//
// Float32-grade logits from bf16 tensor cores: Q is exact in bf16, and each pooled key
// kbar (float32) is split into three bf16 parts hi + mid + lo (hi = bf16(kbar), mid =
// bf16(kbar - hi), lo = bf16(kbar - hi - mid); 24 significant bits), so
// q . kbar = q . lo + q . mid + q . hi accumulates in fp32 TMEM from three MMAs, smallest
// first (the tensor cores round the accumulator at every K step, at its current size).
//
// Persistent kernel, one CTA per SM, work item = (head, query block). Key blocks come in
// tiles of 64 (one MMA N). Two passes over the tiles of an item:
//   pass A: per query row, online max and sum of 2^(logit*scale) over all key blocks;
//   pass B: the tiles again, p = 2^(logit*scale - m - log2 l) for real rows, summed over
//           the 128 rows (warp transpose-reduce, then the four warps) and written once.
// Roles (224 threads): warps 0-3 softmax (thread r = query row r = TMEM lane r), warp 4 MMA
// issuer + TMEM allocation, warps 5-6 loaders (Q rows by the block-slot table, key-split
// rows contiguous). Every wait is bounded.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace park {

constexpr int BQ = 128;
constexpr int NT = 64;                  // key blocks per tile (MMA N)
constexpr int kSoftmaxThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp0 = 5;
constexpr int kLoadThreads = 64;
constexpr int kThreads = kSoftmaxThreads + 32 + kLoadThreads;   // 224
constexpr int NS = 2;                   // key-split tile stages

template <int D>
struct Cfg {
    static constexpr int Q_BYTES = BQ * D * 2;
    static constexpr int KT_BYTES = NT * D * 2;              // one split of one tile
    static constexpr int STAGE_BYTES = 3 * KT_BYTES;
    static constexpr int OFF_Q = 0;                          // 2 buffers
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;        // NS stages of 3 splits
    static constexpr int OFF_COL = OFF_K + NS * STAGE_BYTES; // [2][4 warps][NT] column sums
    static constexpr int OFF_TOK = OFF_COL + 2 * 4 * NT * 4;  // [2 loader warps][BQ] int: query-tile tokens
    static constexpr int OFF_BAR = OFF_TOK + 2 * BQ * 4;
    // q_full[2] q_empty[2] k_full[NS] k_empty[NS] l_full[2] l_free[2] col[1] fin
    static constexpr int NBAR = 4 + 2 * NS + 4 + 1 + 1;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 8;
    static constexpr int TMEM_COLS = 128;                    // 2 logit buffers of NT columns
    static constexpr int Q_PANEL = BQ * 128;
    static constexpr int KT_PANEL = NT * 128;
    static constexpr uint32_t IDESC = idesc_bf16_f32(BQ, NT, 0, 0);
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
    Geom g;
    const bsa_bf16* Q;
    const bsa_bf16* ksplit;   // [heads][3][nbp][D] bf16: hi, mid, lo of the pooled keys
    const int* perm;
    const int* head_mask;
    float* scores;
    int nbp;                  // nb rounded up to a multiple of NT
    int n_items;              // heads * nb
    float scale_log2;         // log2(e) / sqrt(d)
};

__device__ inline float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// kbar (float32) -> three bf16 parts; padding rows j >= nb are zero.
template <int D>
__global__ void split_kbar_kernel(Geom g, const float* __restrict__ kbar, int nbp, bsa_bf16* __restrict__ ks) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long per_head = (long long)nbp * D;
    if (e >= (long long)g.heads * per_head) return;
    const int h = (int)(e / per_head);
    const long long r = e - (long long)h * per_head;
    const int j = (int)(r / D), c = (int)(r % D);
    float x = j < g.nb ? kbar[((size_t)h * g.nb + j) * D + c] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    x -= __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(x);
    x -= __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x);
    bsa_bf16* base = ks + (size_t)h * 3 * per_head + r;
    base[0] = __bfloat16_as_ushort(hi);
    base[per_head] = __bfloat16_as_ushort(mid);
    base[2 * per_head] = __bfloat16_as_ushort(lo);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) park_tc_kernel(Params P) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    if ((smem_u32(sm) & 1023u) != 0) {
        if (threadIdx.x == 0) raise_error(BSA_ERR_DEVICE_ARG);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 2;
    uint64_t* k_full = bars + 4;
    uint64_t* k_empty = k_full + NS;
    uint64_t* l_full = k_empty + NS;
    uint64_t* l_free = l_full + 2;
    uint64_t* col_bar = l_free + 2;
    uint64_t* fin_bar = col_bar + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_BAR + C::NBAR * 8);
    float* colpart = reinterpret_cast<float*>(sm + C::OFF_COL);
    int* qtok = reinterpret_cast<int*>(sm + C::OFF_TOK);

    const Geom& g = P.g;
    const int warp = threadIdx.x >> 5;
    const unsigned epoch = timeout_epoch();   // waits give up early only on a newer timeout
    const int nb = g.nb;
    const int ntiles = P.nbp / NT;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], kLoadThreads);
            mbar_init(&q_empty[b], 1);
            mbar_init(&l_full[b], 1);
            mbar_init(&l_free[b], kSoftmaxThreads);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], kLoadThreads);
            mbar_init(&k_empty[s], 1);
        }
        mbar_init(col_bar, kSoftmaxThreads);
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
        const int h = item / nb;
        return P.head_mask != nullptr && P.head_mask[h] == 0;
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
            const int h = item / nb, i = item - h * nb;
            const int qb = k & 1;
            // loader waits are warp-uniform (__all_sync): the warp syncs below need every lane
            if (k >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&q_empty[qb], ((k >> 1) - 1) & 1, epoch));
            if (!ok) break;
            const bsa_bf16* Qh = P.Q + (size_t)h * g.N * D;
            // the tile's tokens: one coalesced load per loader warp into its own copy in shared
            // memory, then the row gathers (no gather waits on a load of its own token)
            {
                int* wtok = qtok + (lt >> 5) * BQ;
                const int ln = lt & 31;
                int4 t4 = make_int4(-1, -1, -1, -1);
                if (4 * ln < g.B) t4 = __ldg(reinterpret_cast<const int4*>(P.perm + (size_t)i * g.B) + ln);
                reinterpret_cast<int4*>(wtok)[ln] = t4;
                __syncwarp();
                for (int r = lt / CH; r < BQ; r += kLoadThreads / CH) {
                    const int tok = max(wtok[r], 0);
                    cp_async_16(sQ + qb * C::Q_BYTES + sw128_offset(BQ, r, c), Qh + (size_t)tok * D + c * 8);
                }
                __syncwarp();                            // the copy is rewritten for the next item
            }
            cp_async_arrive_noinc(&q_full[qb]);
            const bsa_bf16* kh = P.ksplit + (size_t)h * 3 * P.nbp * D;
            for (int t2 = 0; t2 < 2 * ntiles && ok; ++t2, ++gt) {
                const int t = t2 % ntiles;                   // pass A tiles, then pass B tiles
                const int s = gt % NS;
                if (gt >= NS) ok = __all_sync(0xffffffffu, mbar_wait(&k_empty[s], ((gt / NS) - 1) & 1, epoch));
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
                const int qb = k & 1;
                ok = mbar_wait(&q_full[qb], (k >> 1) & 1, epoch);
                for (int t2 = 0; t2 < 2 * ntiles && ok; ++t2, ++gt) {
                    const int s = gt % NS, lb = gt & 1;
                    ok = mbar_wait(&k_full[s], (gt / NS) & 1, epoch);
                    if (ok && gt >= 2) ok = mbar_wait(&l_free[lb], ((gt >> 1) - 1) & 1, epoch);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t qbase = sQ + qb * C::Q_BYTES;
                    // lo, then mid, then hi: the small products accumulate while the sum is
                    // small (each K step rounds the fp32 accumulator at its current size)
#pragma unroll
                    for (int sp = 2; sp >= 0; --sp) {
                        const uint32_t kbase = sK + s * C::STAGE_BYTES + sp * C::KT_BYTES;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t a = smem_desc_sw128(qbase + (kk >> 2) * C::Q_PANEL + (kk & 3) * 32, 16, 1024);
                            const uint64_t b = smem_desc_sw128(kbase + (kk >> 2) * C::KT_PANEL + (kk & 3) * 32, 16, 1024);
                            mma_bf16_ss(tmem + lb * NT, a, b, C::IDESC, (sp < 2 || kk > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(&l_full[lb]);
                    tc_commit(&k_empty[s]);
                    if (t2 == 2 * ntiles - 1) tc_commit(&q_empty[qb]);
                }
                ++k;
            }
            tc_commit(fin_bar);
            mbar_drain(fin_bar, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ softmax
        const int r = threadIdx.x;                       // query row == TMEM lane
        const int lane = r & 31;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        bool ok = true;
        int gt = 0;
        uint32_t col_phase = 0;
        for (int item = blockIdx.x; item < P.n_items && ok; item += gridDim.x) {
            if (skip_item(item)) continue;
            const int h = item / nb, i = item - h * nb;
            const bool row_real = r < g.B && __ldg(P.perm + i * g.B + r) >= 0;
            const float inv_n = 1.0f / (float)block_count(g, i);
            float m = -INFINITY, l = 0.f;
            float* out = P.scores + ((size_t)h * nb + i) * nb;
            for (int t2 = 0; t2 < 2 * ntiles && ok; ++t2, ++gt) {
                const int t = t2 % ntiles, lb = gt & 1;
                const bool pass_b = t2 >= ntiles;
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
                if (!pass_b) {
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
                        if (jbase + e < nb) s += ex2(fmaf(__uint_as_float(v0[e]), P.scale_log2, -m_new));
                        if (jbase + 32 + e < nb) s += ex2(fmaf(__uint_as_float(v1[e]), P.scale_log2, -m_new));
                    }
                    l = l * ex2(m - m_new) + s;
                    m = m_new;
                    continue;
                }
                // pass B: normalised probabilities of this row (0 for padding rows)
                const float off = -(m + __log2f(l));
                float p[64];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    p[e] = (row_real && jbase + e < nb) ? ex2(fmaf(__uint_as_float(v0[e]), P.scale_log2, off)) : 0.f;
                    p[32 + e] = (row_real && jbase + 32 + e < nb) ? ex2(fmaf(__uint_as_float(v1[e]), P.scale_log2, off)) : 0.f;
                }
                // warp transpose-reduce: after five halvings lane l holds the column sums of
                // columns 2*l and 2*l+1 over the warp's 32 rows
#pragma unroll
                for (int o = 16, n = 64; o > 0; o >>= 1, n >>= 1) {
                    const bool upper = (lane & o) != 0;
#pragma unroll
                    for (int e = 0; e < n / 2; ++e) {
                        const float send = upper ? p[e] : p[e + n / 2];
                        const float keep = upper ? p[e + n / 2] : p[e];
                        p[e] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                    }
                }
                // the halving with offset 2^b moved columns by 2^(b+1) for lanes with bit b
                // set, so lane l now holds columns 2l and 2l+1
                const int colbase = 2 * lane;
                float* cp = colpart + (gt & 1) * 4 * NT + warp * NT;
                cp[colbase] = p[0];
                cp[colbase + 1] = p[1];
                // the four warps meet; threads 0..NT-1 finish their column
                mbar_arrive(col_bar);
                ok = __all_sync(0xffffffffu, mbar_wait(col_bar, col_phase & 1, epoch));
                ++col_phase;
                if (!ok) break;
                if (r < NT && jbase + r < nb) {
                    const float* cq = colpart + (gt & 1) * 4 * NT;
                    out[jbase + r] = (cq[r] + cq[NT + r] + cq[2 * NT + r] + cq[3 * NT + r]) * inv_n;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace park
}  // namespace bsa
