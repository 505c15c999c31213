// Per-head top-p block selection (HASTE: Training-Free Video Diffusion Acceleration via
// Head-Wise Adaptive Sparse Attention, abstract: online top-p sparse attention with
// per-head thresholds).
//
// CTAs walk (head, query block) rows. A row's scores become 64-bit keys
// (~float_bits << 32 | j) so that one ascending bitonic sort in shared memory orders them
// by score descending, then index ascending. A block-wide float32 inclusive scan of the
// sorted scores finds the first position whose cumulative mass reaches p; the kept set is
// that prefix plus the forced text key blocks (all blocks for text query rows), compacted in
// sorted order.
#pragma once

#include "bsa_common.cuh"

namespace bsa {

constexpr int kSelectThreads = 256;
constexpr int kWarpSelectCap = 64;      // extractions before a row falls back to the full sort

// Rows the per-warp kernel below does not finish: text query rows and heads with p >= 1
// (every block kept), rows it marked with cnt = -1 (more than kWarpSelectCap blocks to
// extract), and every row when sort_all is set (more than 1024 blocks per row).
template <int N2>
__global__ void __launch_bounds__(kSelectThreads) select_topp_kernel(
    Geom g, const float* __restrict__ scores, const float* __restrict__ p,
    const int* __restrict__ head_mask, int* __restrict__ idx, int* __restrict__ cnt, int sort_all) {
    constexpr int NT = kSelectThreads;
    constexpr int E = (N2 + NT - 1) / NT;   // sorted elements owned per thread in the scan
    __shared__ unsigned long long key[N2];
    __shared__ float warp_tot[NT / 32];
    __shared__ int warp_cnt[NT / 32];
    __shared__ int cut_pos;

    const int nb = g.nb;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int rowi = blockIdx.x; rowi < g.heads * nb; rowi += gridDim.x) {
    const int h = rowi / nb, i = rowi - h * nb;
    if (head_mask != nullptr && head_mask[h] == 0) continue;
    if (!sort_all && i < g.nbv && p[h] < 1.0f && cnt[(size_t)h * nb + i] != -1) continue;
    __syncthreads();                       // the previous row is finished with shared memory
    const float* row = scores + ((size_t)h * nb + i) * nb;

    for (int e = tid; e < N2; e += NT) {
        unsigned long long k = ~0ull;
        if (e < nb) {
            const float s = row[e];
            // scores are probabilities; anything not > 0 (0, -0, NaN, negative) orders as 0
            const uint32_t bits = (s > 0.f) ? __float_as_uint(s) : 0u;
            k = ((unsigned long long)(~bits) << 32) | (uint32_t)e;
        }
        key[e] = k;
    }
    if (tid == 0) cut_pos = nb;   // "none reached": keep all
    __syncthreads();

    // bitonic sort, ascending
    for (int k = 2; k <= N2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int t = tid; t < N2 / 2; t += NT) {
                const int a = ((t & ~(j - 1)) << 1) | (t & (j - 1));
                const int b = a + j;
                const unsigned long long x = key[a], y = key[b];
                const bool up = (a & k) == 0;
                if ((x > y) == up) { key[a] = y; key[b] = x; }
            }
            __syncthreads();
        }
    }

    const bool text_row = i >= g.nbv;
    const float pth = p[h];
    const bool keep_all = text_row || !(pth < 1.0f);

    // inclusive scan of sorted scores: thread t owns positions [t*E, t*E+E)
    float v[E];
    float run = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int pos = tid * E + e;
        float s = 0.f;
        if (pos < nb) s = __uint_as_float(~(uint32_t)(key[pos] >> 32));
        run += s;
        v[e] = run;
    }
    float incl = run;   // warp-level inclusive scan of thread totals
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    float off = incl - run;
    for (int w = 0; w < warp; ++w) off += warp_tot[w];
    if (!keep_all) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int pos = tid * E + e;
            if (pos < nb && off + v[e] >= pth) { atomicMin(&cut_pos, pos); break; }
        }
    }
    __syncthreads();
    const int last = keep_all ? nb - 1 : min(cut_pos, nb - 1);

    // compaction in sorted order: kept = position <= last, or a text key block
    int flags[E];
    int mine = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int pos = tid * E + e;
        int f = 0;
        if (pos < nb) {
            const int j = (int)(uint32_t)key[pos];
            f = (pos <= last) || (j >= g.nbv);
        }
        flags[e] = f;
        mine += f;
    }
    int ic = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ic, o);
        if (lane >= o) ic += y;
    }
    if (lane == 31) warp_cnt[warp] = ic;
    __syncthreads();
    int base = ic - mine;
    int total = 0;
    for (int w = 0; w < NT / 32; ++w) {
        if (w < warp) base += warp_cnt[w];
        total += warp_cnt[w];
    }
    int* out = idx + ((size_t)h * nb + i) * nb;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if (flags[e]) out[base++] = (int)(uint32_t)key[tid * E + e];
    }
    if (tid == 0) cnt[(size_t)h * nb + i] = total;
    }
}


// One warp per video query row with p < 1 (rows up to 1024 blocks). Block j's key is
// ~float_bits(score), so an ascending key order is score descending, and among equal keys the
// lower block index wins; the row's keys sit in shared memory (lane l owns blocks l, l+32, ...),
// which keeps registers, and so the number of resident warps, low. The warp extracts the best
// remaining block, adds its score to a float32 running sum (sequentially, in sorted order) and
// stops once the sum reaches p -- usually after a handful of blocks. The kept list is then
// merged with the forced text key blocks in the same order. A row that needs more than
// kWarpSelectCap extractions is marked cnt = -1 for the sorting kernel.
constexpr int kWarpSelectMaxBlocks = 1024;

template <int E>
__global__ void __launch_bounds__(256) select_topp_warp_kernel(
    Geom g, const float* __restrict__ scores, const float* __restrict__ p,
    const int* __restrict__ head_mask, int* __restrict__ idx, int* __restrict__ cnt) {
    static_assert(E * 32 <= kWarpSelectMaxBlocks, "row fits the key buffer");
    __shared__ uint32_t key_s[8][E * 32];
    __shared__ int kept_s[8][kWarpSelectCap];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = g.nb;
    const long long row = (long long)blockIdx.x * 8 + warp;
    if (row >= (long long)g.heads * nb) return;
    const int h = (int)(row / nb), i = (int)(row - (long long)h * nb);
    if (i >= g.nbv) return;                                   // text rows: sorting kernel
    if (head_mask != nullptr && head_mask[h] == 0) return;
    const float pth = p[h];
    if (!(pth < 1.0f)) return;                                // keep-all rows: sorting kernel
    const float* srow = scores + (size_t)row * nb;
    uint32_t* keys = key_s[warp];
    float sc[E];
#pragma unroll
    for (int m = 0; m < E; ++m) {
        const int j = lane + 32 * m;
        sc[m] = j < nb ? srow[j] : 0.f;                       // all loads in flight together
    }
    // lane-local best untaken block as (key << 32 | index); all ones when none is left (no
    // real block has that value: indices stay below 2^31)
    uint32_t taken = 0;                                     // bit m: block lane + 32m retired
    unsigned long long mine = ~0ull;
#pragma unroll
    for (int m = 0; m < E; ++m) {
        const int j = lane + 32 * m;
        if (j < nb) {
            const uint32_t k = ~((sc[m] > 0.f) ? __float_as_uint(sc[m]) : 0u);   // not > 0 orders as 0
            keys[j] = k;
            const unsigned long long c = ((unsigned long long)k << 32) | (uint32_t)j;
            if (c < mine) mine = c;
        } else {
            taken |= 1u << m;
        }
    }
    __syncwarp();
    auto local_best = [&]() -> unsigned long long {
        unsigned long long b = ~0ull;
        for (int m = 0; m < E; ++m) {
            if ((taken >> m) & 1u) continue;
            const int j = lane + 32 * m;
            const unsigned long long c = ((unsigned long long)keys[j] << 32) | (uint32_t)j;
            if (c < b) b = c;
        }
        return b;
    };
    float cum = 0.f;
    int n = 0;
    bool done = false;
    while (!done && n < kWarpSelectCap) {
        unsigned long long best = mine;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other < best ? other : best;
        }
        if (best == ~0ull) { done = true; break; }            // every block kept: sum stayed < p
        const uint32_t bkey = (uint32_t)(best >> 32);
        const int bj = (int)(uint32_t)best;
        if (lane == 0) kept_s[warp][n] = bj;
        ++n;
        cum += __uint_as_float(~bkey);                       // sequential float32 sum
        if (cum >= pth) done = true;
        if ((bj & 31) == lane) {                             // owner retires the block
            taken |= 1u << (bj >> 5);
            mine = local_best();
        }
    }
    if (!done) {                                            // too many blocks: full sort
        if (lane == 0) cnt[row] = -1;
        return;
    }
    __syncwarp();
    if (lane == 0) {
        // merge the kept prefix (already in key order) with the forced text blocks, taken
        // in key order too (at most 64 text blocks reach this kernel); keys from shared memory
        auto key_of = [&](int j) -> unsigned long long {
            return ((unsigned long long)keys[j] << 32) | (uint32_t)j;
        };
        int* out = idx + (size_t)row * nb;
        unsigned long long used = 0;                     // bit t - nbv: text block placed
        for (int q = 0; q < n; ++q)
            if (kept_s[warp][q] >= g.nbv) used |= 1ull << (kept_s[warp][q] - g.nbv);
        int a = 0, o = 0;
        while (true) {
            int bt = -1;
            unsigned long long bk = ~0ull;
            for (int t = g.nbv; t < nb; ++t) {
                if ((used >> (t - g.nbv)) & 1ull) continue;
                const unsigned long long k = key_of(t);
                if (k < bk) { bk = k; bt = t; }
            }
            if (bt < 0) break;
            used |= 1ull << (bt - g.nbv);
            while (a < n && key_of(kept_s[warp][a]) < bk) out[o++] = kept_s[warp][a++];
            out[o++] = bt;
        }
        while (a < n) out[o++] = kept_s[warp][a++];
        cnt[row] = o;
    }
}

}  // namespace bsa
