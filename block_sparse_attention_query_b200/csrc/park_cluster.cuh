// PARK per-query-normalised block scorer in one pass: the logits of an item stay in tensor
// memory (PARK: Accurate Block Retrieval for Sparse Attention in Video Diffusion Transformers,
// Abstract: each query's attention over key blocks is normalised on its own, then these
// distributions are averaged within the query block).
//
//   P[h][i][j] = (1/n_i) * sum over real queries q of block i of softmax_j(q . kbar_j / sqrt(d))
//
// Logits are float32-grade as in park_tc.cuh: Q is exact in bf16, each pooled key is split
// into three bf16 parts, and the products are issued smallest part first. Instead of two
// passes over the key tiles, the key blocks of a head are split over a cluster of C CTAs. CTA c
// keeps the three parts of its W pooled keys (key blocks [cW, cW + W)) resident in shared
// memory while the cluster works on that head, and per item (head, query block) issues one
// M = 128, N = W product per part and K step. The 128 x W logits stay in TMEM, in one of three
// buffers used in turn; two softmax teams take the items alternately, so one team's
// exponentials, the other's column sums and the next items' products overlap:
//   pass A   per row, in one thread (two 32-column chunks loaded at a time): the running max
//            m_t and sum l_t of 2^(x - m_t); the exponentials, relative to the running max of
//            their pair, are written back over the logits;
//   exchange each CTA stores its rows' (m, l) into every CTA of the cluster with st.async,
//            which counts the bytes on the receiver's mbarrier (armed one item ahead with the
//            bytes it expects); every CTA combines the C pairs in rank order, so all of them
//            hold the same row normaliser;
//   pass B   p = e * 2^(m_pair - m) / l for real rows, summed over the 128 rows (warp
//            transpose-reduce, then the four lane quarters in a fixed order), written once.
// Roles (384 threads): warps 0-3 and 4-7 the two softmax teams (warp w: TMEM lane quarter
// w & 3), warp 8 MMA issuer and TMEM allocation, warps 9-11 loaders. Every wait is bounded. The
// CTAs of a cluster meet at a cluster barrier before the first remote store and again before
// exit; a team whose exchange was cut short first waits until the bytes of its armed phases
// have landed, so no CTA's shared memory goes away while a peer's store to it may be in flight.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace parkc {

constexpr int BQ = 128;
constexpr int kTeamThreads = 128;        // one softmax thread per query row
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp0 = 9;
constexpr int kLoadWarps = 3;            // a cp.async gather warp moves ~5 B per cycle
constexpr int kLoadThreads = 32 * kLoadWarps;
constexpr int kThreads = 2 * kTeamThreads + 32 + kLoadThreads;   // 384
constexpr int kMaxCluster = 8;
constexpr int kBufs = 3;          // TMEM logit buffers, used in turn by consecutive items
constexpr int kTmemCols = 512;
constexpr int kNumBars = 19;

// Most key blocks one CTA holds (five chunks of 32 per row; for d = 128 the three parts of 160
// pooled keys take 120 KB of shared memory).
constexpr int kMaxCols = 160;     // also the TMEM buffer stride: 3 x 160 columns of the 512
constexpr int kChunks = kMaxCols / 32;
constexpr int kGroup = 2;                                   // chunks loaded together
constexpr int kGroups = (kChunks + kGroup - 1) / kGroup;

struct Layout {
    int part_bytes;   // one bf16 part of the W resident pooled keys, W * D * 2
    int off_q;        // two query tiles, 128 x D bf16 each
    int off_col;      // [2 teams][4][kMaxCols] float: column sums of each TMEM lane quarter
    int off_stats;    // [2 teams][2][C][BQ] float2: (m, l) of each row from every CTA of the cluster
    int off_tok;      // [kLoadWarps][BQ] int: each loader warp's copy of the query tile's tokens
    int off_bar;
    int total;
};

template <int D>
__host__ __device__ inline Layout layout(int W, int C) {
    Layout L;
    L.part_bytes = W * D * 2;                   // a multiple of 4096 for W a multiple of 16
    L.off_q = 3 * L.part_bytes;
    L.off_col = L.off_q + 2 * BQ * D * 2;
    L.off_stats = L.off_col + 2 * 4 * kMaxCols * 4;
    L.off_tok = L.off_stats + 4 * C * BQ * 8;
    L.off_bar = L.off_tok + kLoadWarps * BQ * 4;
    L.total = L.off_bar + kNumBars * 8 + 8;
    return L;
}

struct Params {
    Geom g;
    const bsa_bf16* Q;
    const bsa_bf16* ksplit;   // [heads][3][nbp][D] bf16: hi, mid, lo of the pooled keys (rows >= nb zero)
    const int* perm;
    const int* head_mask;
    float* scores;
    int nbp;                  // rows of each part per head, >= C * W
    int W;                    // key blocks per CTA: a multiple of 16, <= kMaxCols
    int C;                    // CTAs per cluster, (C - 1) * W < nb <= C * W
    int n_items;              // heads * nb
    int n_clusters;
    float scale_log2;         // log2(e) / sqrt(d)
};

__device__ inline float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed float32 pairs: one fma.rn.f32x2 / add.rn.f32x2 does both lanes (each lane rounds as
// the scalar instruction would).
__device__ inline unsigned long long pk2(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ inline float2 up2(unsigned long long r) {
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
__device__ inline float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Pass A over NC consecutive 32-column chunks of a row (tcgen05 loads in flight together); the
// last chunk holds `nv_last` real columns (the rest is masked to -inf). Updates the running max
// mt (scaled logits) and the sum lt of 2^(x - mt); writes 2^(x - mn) back (mn = the new
// running max, returned as the chunks' reference).
template <int NC>
__device__ inline float pass_a_chunks(uint32_t taddr, int nv_last, float sc, float& mt, float& lt) {
    uint32_t v[NC][32];
#pragma unroll
    for (int u = 0; u < NC; ++u) tmem_ld32(taddr + u * 32, v[u]);
    tmem_wait_ld();
    if (nv_last < 32) {                                  // warp-uniform: only a row's last chunk
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (e >= nv_last) v[NC - 1][e] = __float_as_uint(-INFINITY);
    }
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int u = 0; u < NC; ++u)
#pragma unroll
        for (int e = 0; e < 32; e += 2)
            mx[(e >> 1) & 3] = max3(mx[(e >> 1) & 3], __uint_as_float(v[u][e]), __uint_as_float(v[u][e + 1]));
    const float mn = fmaxf(mt, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sc);
    const unsigned long long sc2 = pk2(sc, sc), neg2 = pk2(-mn, -mn);
    unsigned long long ls[2] = {pk2(0.f, 0.f), pk2(0.f, 0.f)};
#pragma unroll
    for (int u = 0; u < NC; ++u) {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const float2 x = up2(fma2(pk2(__uint_as_float(v[u][e]), __uint_as_float(v[u][e + 1])), sc2, neg2));
            const float p0 = ex2(x.x), p1 = ex2(x.y);                   // -inf -> 0
            ls[(e >> 1) & 1] = add2(ls[(e >> 1) & 1], pk2(p0, p1));
            v[u][e] = __float_as_uint(p0);
            v[u][e + 1] = __float_as_uint(p1);
        }
        tmem_st32(taddr + u * 32, v[u]);
    }
    const float2 l2 = up2(add2(ls[0], ls[1]));
    lt = lt * ex2(mt - mn) + (l2.x + l2.y);              // the first chunks: 0 * 0
    mt = mn;
    return mn;
}

// Pass B over NC consecutive chunks: p = e * f summed over the warp's 32 rows (transpose-reduce:
// after five halvings lane l holds column l's sum), written to col[u * 32 + lane].
template <int NC>
__device__ inline void pass_b_chunks(uint32_t taddr, float f, int lane, float* col) {
    uint32_t v[NC][32];
#pragma unroll
    for (int u = 0; u < NC; ++u) tmem_ld32(taddr + u * 32, v[u]);
    tmem_wait_ld();
    const unsigned long long f2 = pk2(f, f), zero2 = pk2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < NC; ++u) {
        float p[32];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const float2 y = up2(fma2(pk2(__uint_as_float(v[u][e]), __uint_as_float(v[u][e + 1])), f2, zero2));
            p[e] = y.x;
            p[e + 1] = y.y;
        }
#pragma unroll
        for (int o = 16, m = 32; o > 1; o >>= 1, m >>= 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int e = 0; e < m / 2; e += 2) {
                const float s0 = upper ? p[e] : p[e + m / 2], s1 = upper ? p[e + 1] : p[e + 1 + m / 2];
                const float k0 = upper ? p[e + m / 2] : p[e], k1 = upper ? p[e + 1 + m / 2] : p[e + 1];
                const float r0 = __shfl_xor_sync(0xffffffffu, s0, o), r1 = __shfl_xor_sync(0xffffffffu, s1, o);
                const float2 y = up2(add2(pk2(k0, k1), pk2(r0, r1)));
                p[e] = y.x;
                p[e + 1] = y.y;
            }
        }
        {   // the last halving (offset 1): one column left per lane
            const bool upper = (lane & 1) != 0;
            const float sd = upper ? p[0] : p[1], kp = upper ? p[1] : p[0];
            p[0] = kp + __shfl_xor_sync(0xffffffffu, sd, 1);
        }
        col[u * 32 + lane] = p[0];
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) park_cluster_kernel(Params P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    const Layout L = layout<D>(P.W, P.C);
    // the same in every CTA, so a whole cluster returns here before any cluster barrier
    if ((smem_u32(sm) & 1023u) != 0) {
        if (threadIdx.x == 0) raise_error(BSA_ERR_DEVICE_ARG);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.off_bar);
    uint64_t* q_full = bars;          // [2] query tile landed (loaders)
    uint64_t* q_empty = bars + 2;     // [2] query tile read by the products (commit)
    uint64_t* kb_full = bars + 4;     // resident pooled keys landed (loaders)
    uint64_t* kb_free = bars + 5;     // last product of a head done (commit)
    uint64_t* s_full = bars + 6;      // [3] logits in TMEM buffer (commit)
    uint64_t* s_free = bars + 9;      // [3] TMEM buffer read for the last time (softmax team)
    uint64_t* st_full = bars + 12;    // [2 teams][2] the cluster's (m, l) pairs landed (st.async bytes)
    uint64_t* col_bar = bars + 16;    // [2 teams] the four lane quarters' column sums written
    uint64_t* fin_bar = bars + 18;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
    float* colsum = reinterpret_cast<float*>(sm + L.off_col);
    float2* stats = reinterpret_cast<float2*>(sm + L.off_stats);
    int* qtok = reinterpret_cast<int*>(sm + L.off_tok);

    const Geom& g = P.g;
    const int warp = threadIdx.x >> 5;
    const unsigned epoch = timeout_epoch();   // waits give up early only on a newer timeout
    const int nb = g.nb, W = P.W, C = P.C;
    const int rank = (int)cluster_rank();
    const int col0 = rank * W;                          // first key block of this CTA
    const int Wc = max(0, min(W, nb - col0));           // its real key blocks
    const int nch = (Wc + 31) / 32;                     // 32-column chunks holding them
    const int cid = blockIdx.x / C;
    const long long it_begin = (long long)cid * P.n_items / P.n_clusters;
    const long long it_end = (long long)(cid + 1) * P.n_items / P.n_clusters;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], kLoadThreads);
            mbar_init(&q_empty[b], 1);
            mbar_init(&col_bar[b], kTeamThreads);
        }
        for (int b = 0; b < kBufs; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], kTeamThreads);
        }
        for (int b = 0; b < 4; ++b) mbar_init(&st_full[b], 1);   // the local expect_tx arrival; bytes from the peers
        mbar_init(kb_full, kLoadThreads);
        mbar_init(kb_free, 1);
        mbar_init(fin_bar, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // every CTA's barriers are initialised before the first remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sK = smem_u32(sm);
    const uint32_t sQ = smem_u32(sm + L.off_q);
    constexpr uint32_t Q_BYTES = BQ * D * 2;

    // masked heads are skipped; the mask of the last head looked at is kept (items come in
    // head order, so the mask is read about once per head and thread)
    int mask_h = -1;
    bool mask_skip = false;
    auto skip_item = [&](long long item) -> bool {
        if (P.head_mask == nullptr) return false;
        const int h = (int)(item / nb);
        if (h != mask_h) {
            mask_h = h;
            mask_skip = P.head_mask[h] == 0;
        }
        return mask_skip;
    };

    if (warp >= kLoadWarp0) {
        // ================================================================ loaders
        constexpr int CH = D / 8;                           // 16-byte chunks per row
        const int lt = threadIdx.x - kLoadWarp0 * 32;
        const int c = lt % CH;
        bool ok = true;
        int k = 0, kload = 0, prev_h = -1;
        for (long long item = it_begin; item < it_end && ok; ++item) {
            if (skip_item(item)) continue;
            const int h = (int)(item / nb), i = (int)(item - (long long)h * nb);
            if (h != prev_h) {
                // this CTA's pooled keys of head h, once the last product of the previous head is done
                // loader waits are warp-uniform (__all_sync): the warp syncs below need every lane
                if (kload >= 1) ok = __all_sync(0xffffffffu, mbar_wait(kb_free, (kload - 1) & 1, epoch));
                if (!ok) break;
                const bsa_bf16* kh = P.ksplit + (size_t)h * 3 * P.nbp * D;
                for (int sp = 0; sp < 3; ++sp) {
                    const bsa_bf16* src = kh + ((size_t)sp * P.nbp + col0) * D;
                    for (int r = lt / CH; r < W; r += kLoadThreads / CH)
                        cp_async_16(sK + sp * L.part_bytes + sw128_offset(W, r, c), src + (size_t)r * D + c * 8);
                }
                cp_async_arrive_noinc(kb_full);
                ++kload;
                prev_h = h;
            }
            const int qb = k & 1;
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
                constexpr int RPP = kLoadThreads / CH;          // rows per pass
                constexpr int NP = (BQ + RPP - 1) / RPP;
                int tok[NP];
#pragma unroll
                for (int pi = 0; pi < NP; ++pi) {
                    const int r = lt / CH + pi * RPP;
                    tok[pi] = r < BQ ? max(wtok[r], 0) : 0;
                }
#pragma unroll
                for (int pi = 0; pi < NP; ++pi) {              // all gathers issued back to back
                    const int r = lt / CH + pi * RPP;
                    if (r < BQ)
                        cp_async_16(sQ + qb * Q_BYTES + sw128_offset(BQ, r, c), Qh + (size_t)tok[pi] * D + c * 8);
                }
                __syncwarp();                            // the copy is rewritten for the next item
            }
            cp_async_arrive_noinc(&q_full[qb]);
            ++k;
        }
        cp_async_wait_all();   // no copy may still target shared memory at teardown
    } else if (warp == kMmaWarp) {
        // ================================================================ MMA issuer
        if (elect_one()) {
            const uint32_t idesc = idesc_bf16_f32(BQ, W, 0, 0);
            bool ok = true;
            int k = 0, kload = 0, prev_h = -1;
            for (long long item = it_begin; item < it_end && ok; ++item) {
                if (skip_item(item)) continue;
                const int h = (int)(item / nb);
                if (h != prev_h) {
                    ok = mbar_wait(kb_full, kload & 1, epoch);
                    ++kload;
                    prev_h = h;
                    if (!ok) break;
                }
                const int qb = k & 1, sb = k % kBufs, su = k / kBufs;   // buffer sb, its use su
                ok = mbar_wait(&q_full[qb], (k >> 1) & 1, epoch);
                if (ok && su >= 1) ok = mbar_wait(&s_free[sb], (su - 1) & 1, epoch);
                if (!ok) break;
                tc_fence_after();
                const uint32_t qbase = sQ + qb * Q_BYTES;
                // lo, then mid, then hi: the small products accumulate while the sum is small
#pragma unroll
                for (int sp = 2; sp >= 0; --sp) {
                    const uint32_t kbase = sK + sp * L.part_bytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = smem_desc_sw128(qbase + (kk >> 2) * (BQ * 128) + (kk & 3) * 32, 16, 1024);
                        const uint64_t b = smem_desc_sw128(kbase + (kk >> 2) * (W * 128) + (kk & 3) * 32, 16, 1024);
                        mma_bf16_ss(tmem + sb * kMaxCols, a, b, idesc, (sp < 2 || kk > 0) ? 1u : 0u);
                    }
                }
                tc_commit(&s_full[sb]);
                tc_commit(&q_empty[qb]);
                if (item + 1 >= it_end || (int)((item + 1) / nb) != h) tc_commit(kb_free);
                ++k;
            }
            // every MMA issued by this thread has completed once fin_bar flips
            tc_commit(fin_bar);
            mbar_drain(fin_bar, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ softmax teams
        const int team = warp >> 2, q4 = warp & 3;
        const int lane = threadIdx.x & 31;
        const int r = q4 * 32 + lane;                    // query row == TMEM lane
        const int tt = threadIdx.x & (kTeamThreads - 1);
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);   // this warp's lane quarter
        const float sc = P.scale_log2;
        const uint32_t xbytes = (uint32_t)(C * BQ * 8);  // (m, l) pairs one CTA receives per item
        float* csum = colsum + team * 4 * kMaxCols;
        // the CTA's items in order, masked heads left out; this team takes every other one
        auto next_item = [&](long long item) -> long long {
            for (++item; item < it_end; ++item)
                if (!skip_item(item)) return item;
            return -1;
        };
        auto team_next = [&](long long item) -> long long {
            item = next_item(item);
            return item >= 0 ? next_item(item) : -1;
        };
        long long item = it_begin < it_end ? (skip_item(it_begin) ? next_item(it_begin) : it_begin) : -1;
        if (team == 1 && item >= 0) item = next_item(item);
        // team thread 0 arms each item's exchange barrier (expected bytes) one item ahead, so no
        // peer stores into a phase that is not armed; it drains armed phases before exit
        int armed = -1, waited = -1;
        if (tt == 0 && item >= 0) {
            mbar_arrive_expect_tx(&st_full[team * 2], xbytes);
            armed = 0;
        }
        bool ok = true;
        int n = 0;                                       // this team's item count
        for (long long nx; item >= 0 && ok; item = nx, ++n) {
            nx = team_next(item);                        // this team's next item, -1 at the end
            const int h = (int)(item / nb), i = (int)(item - (long long)h * nb);
            const bool row_real = r < g.B && __ldg(P.perm + (size_t)i * g.B + r) >= 0;
            const int k = 2 * n + team, sb = k % kBufs;  // the CTA's item index, its TMEM buffer
            const uint32_t tb = tl + sb * kMaxCols;
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (k / kBufs) & 1, epoch));
            if (!ok) break;
            tc_fence_after();
            // pass A: the row's logits, two chunks of 32 at a time (both loads in flight): the
            // running max m_t and sum l_t of 2^(x - m_t); the exponentials, relative to the
            // running max of their pair (ref), are written back over the logits
            float mt = -INFINITY, lt = 0.f;
            float ref[kGroups];
#pragma unroll 1
            for (int gi = 0; gi * kGroup < nch; ++gi) {
                const int ch = gi * kGroup;
                const uint32_t ta = tb + ch * 32;
                float rf;
                if (ch + 1 < nch) rf = pass_a_chunks<2>(ta, min(32, Wc - (ch + 1) * 32), sc, mt, lt);
                else rf = pass_a_chunks<1>(ta, min(32, Wc - ch * 32), sc, mt, lt);
#pragma unroll
                for (int q = 0; q < kGroups; ++q)
                    if (q == gi) ref[q] = rf;                // registers, not local memory
            }
            tmem_wait_st();
            // exchange: this row's (m, l) over the CTA's key blocks, into every CTA of the cluster
            const int xb = team * 2 + (n & 1);
            {
                const uint32_t slot = smem_u32(&stats[(xb * C + rank) * BQ + r]);
                const uint32_t bar = smem_u32(&st_full[xb]);
                for (int c2 = 0; c2 < C; ++c2)
                    st_async_f32x2(cluster_map(slot, (uint32_t)c2), mt, lt, cluster_map(bar, (uint32_t)c2));
            }
            if (tt == 0 && nx >= 0) {
                // the team's next item uses the other barrier, whose previous phase (the team's
                // item n - 1) was waited on during that item
                mbar_arrive_expect_tx(&st_full[team * 2 + ((n + 1) & 1)], xbytes);
                armed = n + 1;
            }
            ok = __all_sync(0xffffffffu, mbar_wait_cluster(&st_full[xb], (n >> 1) & 1, epoch));
            if (!ok) break;
            waited = n;
            // the row normaliser over all key blocks, combined in rank order (the same in every CTA)
            float mg = -INFINITY;
            for (int c2 = 0; c2 < C; ++c2) mg = fmaxf(mg, stats[(xb * C + c2) * BQ + r].x);
            float lg = 0.f;
            for (int c2 = 0; c2 < C; ++c2) {
                const float2 s2 = stats[(xb * C + c2) * BQ + r];
                if (s2.y > 0.f) lg += s2.y * ex2(s2.x - mg);
            }
            // pass B: probabilities, summed over the warp's 32 rows per column
#pragma unroll 1
            for (int gi = 0; gi * kGroup < nch; ++gi) {
                const int ch = gi * kGroup;
                float rf = ref[0];
#pragma unroll
                for (int q = 1; q < kGroups; ++q)
                    if (q == gi) rf = ref[q];
                const float f = (row_real && lg > 0.f) ? ex2(rf - mg) / lg : 0.f;
                if (ch + 1 < nch) pass_b_chunks<2>(tb + ch * 32, f, lane, csum + q4 * kMaxCols + ch * 32);
                else pass_b_chunks<1>(tb + ch * 32, f, lane, csum + q4 * kMaxCols + ch * 32);
            }
            tc_fence_before();
            mbar_arrive(&s_free[sb]);                    // TMEM buffer read for this item
            mbar_arrive(&col_bar[team]);
            ok = __all_sync(0xffffffffu, mbar_wait(&col_bar[team], n & 1, epoch));
            if (!ok) break;
            const float inv_n = 1.0f / (float)block_count(g, i);
            float* out = P.scores + ((size_t)h * nb + i) * nb + col0;
            for (int t = tt; t < Wc; t += kTeamThreads)
                out[t] = (csum[t] + csum[kMaxCols + t] + csum[2 * kMaxCols + t] + csum[3 * kMaxCols + t]) * inv_n;
            // the next item's pass B writes csum only after the exchange, which every thread of
            // the team reaches after these reads
        }
        // an item whose exchange was cut short: wait (to the cycle limit at most) until whatever
        // the peers stored for the armed phases has landed, before this CTA may exit
        if (tt == 0)
            for (int j = waited + 1; j <= armed; ++j) mbar_drain(&st_full[team * 2 + (j & 1)], (j >> 1) & 1);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    cluster_sync_all();   // no CTA leaves while a peer may still write to its shared memory
}

}  // namespace parkc
}  // namespace bsa
