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
// Warp roles (288 threads):
//   warps 0-3  softmax + epilogue. Thread r owns query row r = TMEM lane r.
//   warp 4     TMEM allocation; one elected thread issues every tcgen05.mma.
//   warps 5-8  loaders: gather Q / K / V rows of a block (raster rows from the block-slot
//              table) with 16-byte cp.async into 128B-swizzled K-major tiles.
// The kept blocks of all items of a CTA form one stream g = 0, 1, 2, ...:
//   S[g&1] = Q K_g^T (TMEM fp32) -> softmax: scale, mask padding keys, online max/sum,
//   rescale O in TMEM when a row max grows, P = 2^(s-m) as bf16 into swizzled smem ->
//   O[item&1] += P V_g (TMEM fp32; V is an MN-major operand).
// S is double-buffered (QK^T of block g+1 overlaps the softmax of block g); Q and O are
// double-buffered across items (the next item's loads and QK^T overlap this item's
// epilogue). Every wait is bounded: one that runs out raises BSA_ERR_TIMEOUT and all roles
// wind down. tcgen05.ld/st are warp-collective, so every condition around them is
// warp-uniform.
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
    static constexpr int OFF_Q = 0;                          // 2 buffers
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;        // NS stages
    static constexpr int OFF_V = OFF_K + NS * KV_BYTES;      // NS stages
    static constexpr int OFF_P = OFF_V + NS * KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;
    // q_full[2] q_empty[2] k_full[NS] v_full[NS] k_empty[NS] v_empty[NS] s_full[2] s_free[2]
    // p_full pv_done o_free[2] fin
    static constexpr int NBAR = 4 + 4 * NS + 4 + 2 + 2 + 1;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 8 + 1024;  // +8 TMEM slot, +1024 alignment
    static constexpr int TMEM_S = 0;            // S buffers: [0, 2*BK)
    static constexpr int TMEM_O = 2 * BK;       // O buffers: [2*BK, 2*BK + 2*D)
    static constexpr int TMEM_COLS = (2 * BK + 2 * D) <= 256 ? 256 : 512;
    static constexpr int Q_PANEL = BQ * 128;    // bytes per 64-column swizzle panel
    static constexpr int KV_PANEL = BK * 128;
    static constexpr int P_PANEL = BQ * 128;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BQ, BK, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, 0, 1);
    static_assert(2 * BK + 2 * D <= 512, "TMEM budget");
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

__device__ inline float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Gather rows [block*B, block*B + rows) of one head into a swizzled tile. Rows that are
// padding (or beyond the block) read token row 0 of the head: finite values that the
// softmax masks (keys) or the epilogue never stores (queries).
template <int D>
__device__ inline void gather_tile(const Params& P, const bsa_bf16* head_base, int block, int rows,
                                   uint32_t tile_smem, int lt) {
    constexpr int CH = D / 8;                 // 16-byte chunks per row
    constexpr int RPR = kLoadThreads / CH;    // rows per round
    const int B = P.g.B;
    const int c = lt % CH;
    const int* slot = P.perm + block * B;
#pragma unroll 4
    for (int r = lt / CH; r < rows; r += RPR) {
        int tok = (r < B) ? __ldg(slot + r) : -1;
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
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_BAR + C::NBAR * 8);

    const Geom& g = P.g;
    const int warp = threadIdx.x >> 5;
    const int nb = g.nb;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], kLoadThreads);
            mbar_init(&q_empty[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 128);
            mbar_init(&o_free[b], 128);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], kLoadThreads);
            mbar_init(&v_full[s], kLoadThreads);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_empty[s], 1);
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
    const int first_item = blockIdx.x, stride = gridDim.x;

    auto kept_block = [&](const Item& it, int j) -> int {
        int kb = P.idx[((size_t)it.h * nb + it.i) * nb + it.e0 + j];
        if (kb < 0 || kb >= nb) { raise_error(BSA_ERR_DEVICE_ARG); kb = 0; }
        return kb;
    };

    if (warp >= kLoadWarp0) {
        // ================================================================ loaders
        const int lt = threadIdx.x - kLoadWarp0 * 32;
        bool ok = true;
        uint64_t* pending = nullptr;     // full barrier of the last committed cp.async group
        auto complete_previous = [&]() {
            cp_async_wait<1>();
            fence_proxy_async_smem();
            if (pending != nullptr) mbar_arrive(pending);
        };
        int gblk = 0, k = 0;
        for (int item = first_item; item < P.n_items && ok; item += stride) {
            const Item it = decode_item(P, item);
            if (it.n <= 0) continue;
            const size_t head_off = (size_t)it.h * g.N * D;
            const int qb = k & 1;
            if (k >= 2) ok = mbar_wait(&q_empty[qb], ((k >> 1) - 1) & 1);
            if (!ok) break;
            gather_tile<D>(P, P.Q + head_off, it.i, BQ, sQ + qb * C::Q_BYTES, lt);
            cp_async_commit();
            complete_previous();
            pending = &q_full[qb];
            for (int j = 0; j < it.n && ok; ++j, ++gblk) {
                const int s = gblk % NS;
                const int kb = kept_block(it, j);
                if (gblk >= NS) ok = mbar_wait(&k_empty[s], ((gblk / NS) - 1) & 1);
                if (!ok) break;
                gather_tile<D>(P, P.K + head_off, kb, BK, sK + s * C::KV_BYTES, lt);
                cp_async_commit();
                complete_previous();
                pending = &k_full[s];
                if (gblk >= NS) ok = mbar_wait(&v_empty[s], ((gblk / NS) - 1) & 1);
                if (!ok) break;
                gather_tile<D>(P, P.V + head_off, kb, BK, sV + s * C::KV_BYTES, lt);
                cp_async_commit();
                complete_previous();
                pending = &v_full[s];
            }
            ++k;
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        if (ok && pending != nullptr) mbar_arrive(pending);
    } else if (warp == kMmaWarp) {
        // ================================================================ MMA issuer
        if (elect_one()) {
            bool ok = true;
            // PV for stream block gb, the j-th block of the item with local index kitem
            auto issue_pv = [&](int gb, int j, int kitem) -> bool {
                const int ob = kitem & 1;
                if (j == 0 && kitem >= 2 && !mbar_wait(&o_free[ob], ((kitem >> 1) - 1) & 1)) return false;
                if (!mbar_wait(p_full, gb & 1)) return false;
                if (!mbar_wait(&v_full[gb % NS], (gb / NS) & 1)) return false;
                tc_fence_after();
                const uint32_t vbase = sV + (gb % NS) * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint64_t a = smem_desc_sw128(sP + (kk >> 2) * C::P_PANEL + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = smem_desc_sw128(vbase + kk * 2048, C::KV_PANEL, 1024);
                    mma_bf16_ss(tmem + C::TMEM_O + ob * D, a, b, C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(pv_done);
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
        const int r = threadIdx.x;                       // query row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        bool ok = true;
        int gblk = 0, k = 0;
        for (int item = first_item; item < P.n_items && ok; item += stride) {
            const Item it = decode_item(P, item);
            const size_t head_off = (size_t)it.h * g.N * D;
            const int q_token = (r < g.B) ? __ldg(P.perm + it.i * g.B + r) : -1;
            const bool row_real = q_token >= 0;
            if (it.n <= 0) {
                // nothing kept (an empty text chunk, or an invalid count): zero output
                if (it.n < 0 && r == 0) raise_error(BSA_ERR_DEVICE_ARG);
                if (it.split) {
                    float* po = P.part_o + ((size_t)item * BQ + r) * D;
                    for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(po + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                    P.part_lse[(size_t)item * BQ + r] = -INFINITY;
                } else if (row_real) {
                    bsa_bf16* orow = P.O + head_off + (size_t)q_token * D;
                    for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
                }
                continue;
            }
            const int ob = k & 1;
            const uint32_t o_col = C::TMEM_O + ob * D;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < it.n && ok; ++j, ++gblk) {
                const int sb = gblk & 1;
                const int kcount = block_count(g, kept_block(it, j));
                ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (gblk >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
                float sv[BK];
#pragma unroll
                for (int c = 0; c < BK / 32; ++c) {
                    uint32_t t[32];
                    tmem_ld32(lane_base + C::TMEM_S + sb * BK + c * 32, t);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(t[e]);
                }
                tc_fence_before();
                mbar_arrive(&s_free[sb]);
                float mx = -INFINITY;
#pragma unroll
                for (int e = 0; e < BK; ++e) {
                    sv[e] = (e < kcount) ? sv[e] * P.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, sv[e]);
                }
                const float m_new = fmaxf(m, mx);
                if (j >= 1) {
                    // PV of the previous block is done: P is free and O is stable
                    ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (gblk - 1) & 1));
                    if (!ok) break;
                    tc_fence_after();
                    // the whole warp rescales when any of its rows saw a larger max
                    const bool grow = m_new > m;
                    if (__any_sync(0xffffffffu, grow)) {
                        const float alpha = grow ? ex2(m - m_new) : 1.0f;
                        l *= alpha;
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t t[32];
                            tmem_ld32(lane_base + o_col + c * 32, t);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
                            tmem_st32(lane_base + o_col + c * 32, t);
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
                        const float p0 = ex2(sv[c * 8 + 2 * e] - m);
                        const float p1 = ex2(sv[c * 8 + 2 * e + 1] - m);
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
            // ---- epilogue of this item: wait for its last PV, read O, release the buffer
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (gblk - 1) & 1));
            if (!ok) break;
            tc_fence_after();
            const float inv = 1.0f / l;
            if (it.split) {
                float* po = P.part_o + ((size_t)item * BQ + r) * D;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t t[32];
                    tmem_ld32(lane_base + o_col + c * 32, t);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(po + c * 32 + e) =
                            make_float4(__uint_as_float(t[e]) * inv, __uint_as_float(t[e + 1]) * inv,
                                        __uint_as_float(t[e + 2]) * inv, __uint_as_float(t[e + 3]) * inv);
                }
                P.part_lse[(size_t)item * BQ + r] = m + __log2f(l);
            } else {
                bsa_bf16* orow = P.O + head_off + (size_t)(row_real ? q_token : 0) * D;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t t[32];
                    tmem_ld32(lane_base + o_col + c * 32, t);
                    tmem_wait_ld();
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
            tc_fence_before();
            mbar_arrive(&o_free[ob]);
            ++k;
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

// perm[s] = raster token of block slot s (-1 = padding), for s in [0, nb*B).
__global__ void perm_kernel(Geom g, int* perm) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s < g.nb * g.B) perm[s] = slot_to_token(g, s);
}

}  // namespace attn
}  // namespace bsa
