// Block-sparse attention on tcgen05 tensor cores (PARK: Accurate Block Retrieval for Sparse
// Attention in Video Diffusion Transformers, Abstract: attention computed only within the
// retrieved blocks; cost motive "quadratic complexity of full attention", HASTE abstract).
//
// One CTA per work item = (head h, query block i, range [e0, e1) of its kept list). Video
// query rows are one item each; the dense text query rows are split into chunks whose
// partial results (normalised O and log2-sum-exp) go to the workspace and are merged by
// merge_text_kernel.
//
// Warp roles (288 threads):
//   warps 0-3  softmax + epilogue. Thread r owns query row r = TMEM lane r.
//   warp 4     TMEM allocation; one elected thread issues every tcgen05.mma.
//   warps 5-8  loaders: gather Q / K / V rows of a block (raster rows found on the fly)
//              with 16-byte cp.async into 128B-swizzled K-major tiles.
// Per kept block j:  S[j&1] = Q K_j^T (TMEM, fp32)  ->  softmax threads: scale, mask padding
// keys, online max / sum, rescale O in TMEM when the max grows, P = exp2(.) as bf16 into a
// swizzled smem tile  ->  O += P V_j (TMEM, fp32; V used as an MN-major operand).
// S is double-buffered so QK^T of block j+1 overlaps the softmax of block j. Every wait is
// bounded: a wait that runs out raises BSA_ERR_TIMEOUT and every role winds down.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace attn {

constexpr int BQ = 128;                 // query rows per tile (MMA M)
constexpr int kThreads = 288;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp0 = 5;
constexpr int kLoadThreads = 128;
constexpr int NS = 2;                   // K and V pipeline stages
constexpr int kTextChunk = 64;          // kept blocks per work item of a text query row

template <int D, int BK>
struct Cfg {
    static constexpr int Q_BYTES = BQ * D * 2;
    static constexpr int KV_BYTES = BK * D * 2;
    static constexpr int P_BYTES = BQ * BK * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
    static constexpr int OFF_P = OFF_V + NS * KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;
    static constexpr int NBAR = 1 + 4 * NS + 2 + 2 + 2 + 1;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 8 + 1024;  // +8: TMEM address slot, +1024: alignment slack
    static constexpr int TMEM_S0 = 0;
    static constexpr int TMEM_O = 2 * BK;
    static constexpr int TMEM_COLS = (2 * BK + D) <= 256 ? 256 : 512;
    static constexpr int Q_PANEL = BQ * 128;   // bytes per 64-column swizzle panel
    static constexpr int KV_PANEL = BK * 128;
    static constexpr int P_PANEL = BQ * 128;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BQ, BK, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, 0, 1);
};

struct Params {
    Geom g;
    const bsa_bf16* Q;
    const bsa_bf16* K;
    const bsa_bf16* V;
    const int* idx;
    const int* cnt;
    bsa_bf16* O;
    float* part_o;      // [n_text_items][BQ][D] normalised partial outputs
    float* part_lse;    // [n_text_items][BQ] log2-sum-exp of each partial row
    int n_text_items;   // heads * nbt * nsplit
    int nsplit;         // chunks per text query row
    float scale_log2;   // log2(e) / sqrt(d)
};

// Gather rows [block*B, block*B + rows) of one head into a swizzled tile. Rows that are
// padding (or beyond the block) read token row 0 of the head: finite values that the
// softmax masks (keys) or the epilogue never stores (queries).
template <int D>
__device__ inline void gather_tile(const Geom& g, const bsa_bf16* head_base, int block, int rows,
                                   uint32_t tile_smem, int lt) {
    constexpr int CH = D / 8;                 // 16-byte chunks per row
    constexpr int RPR = kLoadThreads / CH;    // rows per round
    const int c = lt % CH;
    for (int r = lt / CH; r < rows; r += RPR) {
        int tok = (r < g.B) ? slot_to_token(g, block * g.B + r) : -1;
        if (tok < 0) tok = 0;
        cp_async_16(tile_smem + sw128_offset(rows, r, c), head_base + (size_t)tok * D + c * 8);
    }
}

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1) sparse_attention_kernel(Params P) {
    using C = Cfg<D, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;
    uint64_t* v_full = bars + 1 + NS;
    uint64_t* k_empty = bars + 1 + 2 * NS;
    uint64_t* v_empty = bars + 1 + 3 * NS;
    uint64_t* s_full = bars + 1 + 4 * NS;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* pv_done = p_full + 1;
    uint64_t* fin_bar = pv_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_BAR + C::NBAR * 8);

    const Geom& g = P.g;
    const int warp = threadIdx.x >> 5;
    const int nb = g.nb;

    // ---- work item
    int h, i, e0, n;
    bool split = false;
    int item = blockIdx.x;
    if (item < P.n_text_items) {
        split = true;
        const int per_head = g.nbt * P.nsplit;
        h = item / per_head;
        const int rem = item - h * per_head;
        i = g.nbv + rem / P.nsplit;
        e0 = (rem % P.nsplit) * kTextChunk;
    } else {
        item -= P.n_text_items;
        h = item / g.nbv;
        i = item - h * g.nbv;
        e0 = 0;
    }
    const int row_cnt = P.cnt[(size_t)h * nb + i];
    if (row_cnt < 1 || row_cnt > nb) {
        if (threadIdx.x == 0) raise_error(BSA_ERR_DEVICE_ARG);
        n = 0;
    } else {
        n = split ? max(0, min(row_cnt, e0 + kTextChunk) - e0) : row_cnt;
    }
    const int* kept = P.idx + ((size_t)h * nb + i) * nb + e0;
    const size_t head_off = (size_t)h * g.N * D;

    // ---- setup
    if (threadIdx.x == 0) {
        mbar_init(q_full, kLoadThreads);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], kLoadThreads);
            mbar_init(&v_full[s], kLoadThreads);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], 128);
        }
        mbar_init(p_full, 128);
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
    const uint32_t sP = smem_u32(sm + C::OFF_P);

    auto block_of = [&](int j) -> int {
        int kb = kept[j];
        if (kb < 0 || kb >= nb) { raise_error(BSA_ERR_DEVICE_ARG); kb = 0; }
        return kb;
    };

    if (warp >= kLoadWarp0) {
        // ================================================================ loaders
        const int lt = threadIdx.x - kLoadWarp0 * 32;
        const bsa_bf16* Qh = P.Q + head_off;
        const bsa_bf16* Kh = P.K + head_off;
        const bsa_bf16* Vh = P.V + head_off;
        bool ok = true;
        gather_tile<D>(g, Qh, i, BQ, sQ, lt);
        cp_async_commit();
        uint64_t* pending = q_full;     // barrier of the last committed group
        for (int j = 0; j < n && ok; ++j) {
            const int s = j % NS;
            const int kb = block_of(j);
            if (j >= NS) ok = mbar_wait(&k_empty[s], ((j / NS) - 1) & 1);
            if (!ok) break;
            gather_tile<D>(g, Kh, kb, BK, sK + s * C::KV_BYTES, lt);
            cp_async_commit();
            cp_async_wait<1>();
            fence_proxy_async_smem();
            mbar_arrive(pending);
            pending = &k_full[s];
            if (j >= NS) ok = mbar_wait(&v_empty[s], ((j / NS) - 1) & 1);
            if (!ok) break;
            gather_tile<D>(g, Vh, kb, BK, sV + s * C::KV_BYTES, lt);
            cp_async_commit();
            cp_async_wait<1>();
            fence_proxy_async_smem();
            mbar_arrive(pending);
            pending = &v_full[s];
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        if (ok) mbar_arrive(pending);
    } else if (warp == kMmaWarp) {
        // ================================================================ MMA issuer
        if (elect_one()) {
            bool ok = mbar_wait(q_full, 0);
            auto issue_pv = [&](int jj) -> bool {
                if (!mbar_wait(p_full, jj & 1)) return false;
                if (!mbar_wait(&v_full[jj % NS], (jj / NS) & 1)) return false;
                tc_fence_after();
                const uint32_t vbase = sV + (jj % NS) * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint64_t a = smem_desc_sw128(sP + (kk >> 2) * C::P_PANEL + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = smem_desc_sw128(vbase + kk * 2048, C::KV_PANEL, 1024);
                    mma_bf16_ss(tmem + C::TMEM_O, a, b, C::IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(pv_done);
                tc_commit(&v_empty[jj % NS]);
                return true;
            };
            for (int j = 0; j < n && ok; ++j) {
                const int s = j % NS, sb = j & 1;
                ok = mbar_wait(&k_full[s], (j / NS) & 1);
                if (ok && j >= 2) ok = mbar_wait(&s_free[sb], ((j >> 1) - 1) & 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kbase = sK + s * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = smem_desc_sw128(sQ + (kk >> 2) * C::Q_PANEL + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = smem_desc_sw128(kbase + (kk >> 2) * C::KV_PANEL + (kk & 3) * 32, 16, 1024);
                    mma_bf16_ss(tmem + C::TMEM_S0 + sb * BK, a, b, C::IDESC_QK, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[sb]);
                tc_commit(&k_empty[s]);
                if (j >= 1) ok = issue_pv(j - 1);
            }
            if (ok && n > 0) ok = issue_pv(n - 1);
            // all MMAs issued by this thread have completed once fin_bar flips
            tc_commit(fin_bar);
            mbar_wait(fin_bar, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ softmax
        const int r = threadIdx.x;                       // query row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n && ok; ++j) {
            const int sb = j & 1;
            const int kb = block_of(j);
            const int kcount = block_count(g, kb);
            // keep `ok` warp-uniform: the tcgen05.ld/st below are .sync.aligned
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j >> 1) & 1));
            if (!ok) break;
            tc_fence_after();
            float sv[BK];
#pragma unroll
            for (int c = 0; c < BK / 32; ++c) {
                uint32_t t[32];
                tmem_ld32(lane_base + C::TMEM_S0 + sb * BK + c * 32, t);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(t[e]);
            }
            tc_fence_before();
            mbar_arrive(&s_free[sb]);
            float mx = -INFINITY;
#pragma unroll
            for (int k = 0; k < BK; ++k) {
                sv[k] = (k < kcount) ? sv[k] * P.scale_log2 : -INFINITY;
                mx = fmaxf(mx, sv[k]);
            }
            const float m_new = fmaxf(m, mx);
            if (j >= 1) {
                ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1));
                if (!ok) break;
                tc_fence_after();
                // tcgen05.ld/st are warp-collective (.sync.aligned): the rescale runs for the
                // whole warp when any of its rows saw a larger max (alpha = 1 elsewhere)
                const bool grow = m_new > m;
                if (__any_sync(0xffffffffu, grow)) {
                    const float alpha = grow ? exp2f(m - m_new) : 1.0f;
                    l *= alpha;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t t[32];
                        tmem_ld32(lane_base + C::TMEM_O + c * 32, t);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
                        tmem_st32(lane_base + C::TMEM_O + c * 32, t);
                    }
                    tmem_wait_st();
                }
            }
            m = m_new;
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < BK / 8; ++c) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float p0 = exp2f(sv[c * 8 + 2 * e] - m);
                    const float p1 = exp2f(sv[c * 8 + 2 * e + 1] - m);
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                    // the row sum uses the rounded weights the MMA sees, so they sum to 1
                    const float2 pr = __bfloat1622float2(b2);
                    rs += pr.x + pr.y;
                    pk[e] = *reinterpret_cast<uint32_t*>(&b2);
                }
                const uint32_t dst = sP + sw128_offset(BQ, r, c);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(pk[0]), "r"(pk[1]),
                             "r"(pk[2]), "r"(pk[3]) : "memory");
            }
            l += rs;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        // ---- epilogue
        if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (n - 1) & 1));
        tc_fence_after();
        // recomputed here rather than read from the loaders' table: no barrier orders
        // the loaders' shared-memory writes before this point for these threads
        const int q_token = (r < g.B) ? slot_to_token(g, i * g.B + r) : -1;
        const bool row_real = q_token >= 0;
        if (split) {
            const int t_item = blockIdx.x;
            float* po = P.part_o + ((size_t)t_item * BQ + r) * D;
            const float inv = (ok && n > 0) ? 1.0f / l : 0.f;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t t[32];
                if (ok && n > 0) {
                    tmem_ld32(lane_base + C::TMEM_O + c * 32, t);
                    tmem_wait_ld();
                }
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    float4 v;
                    v.x = (ok && n > 0) ? __uint_as_float(t[e]) * inv : 0.f;
                    v.y = (ok && n > 0) ? __uint_as_float(t[e + 1]) * inv : 0.f;
                    v.z = (ok && n > 0) ? __uint_as_float(t[e + 2]) * inv : 0.f;
                    v.w = (ok && n > 0) ? __uint_as_float(t[e + 3]) * inv : 0.f;
                    *reinterpret_cast<float4*>(po + c * 32 + e) = v;
                }
            }
            P.part_lse[(size_t)t_item * BQ + r] = (ok && n > 0) ? m + log2f(l) : -INFINITY;
        } else {
            // every lane takes part in the warp-collective TMEM loads; only real rows store
            bsa_bf16* orow = P.O + head_off + (size_t)(row_real ? q_token : 0) * D;
            const float inv = (ok && n > 0) ? 1.0f / l : 0.f;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t t[32];
                if (ok && n > 0) {
                    tmem_ld32(lane_base + C::TMEM_O + c * 32, t);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) t[e] = 0u;
                }
                if (!row_real) continue;
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint32_t pk[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(t[e + 2 * u]) * inv,
                                                                  __uint_as_float(t[e + 2 * u + 1]) * inv);
                        pk[u] = *reinterpret_cast<uint32_t*>(&b2);
                    }
                    *reinterpret_cast<uint4*>(orow + c * 32 + e) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
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
    const int tok = slot_to_token(g, i * g.B + r);
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
