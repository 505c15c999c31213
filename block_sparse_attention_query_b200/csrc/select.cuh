// Per-head top-p block selection (HASTE: Training-Free Video Diffusion Acceleration via
// Head-Wise Adaptive Sparse Attention, abstract: online top-p sparse attention with
// per-head thresholds).
//
// One CTA per (query block i, head h). The row's scores become 64-bit keys
// (~float_bits << 32 | j) so that one ascending bitonic sort in shared memory orders them
// by score descending, then index ascending. A block-wide float32 inclusive scan of the
// sorted scores finds the first position whose cumulative mass reaches p; the kept set is
// that prefix plus the forced text key blocks (all blocks for text query rows), compacted in
// sorted order.
#pragma once

#include "bsa_common.cuh"

namespace bsa {

constexpr int kSelectThreads = 256;

template <int N2>
__global__ void __launch_bounds__(kSelectThreads) select_topp_kernel(
    Geom g, const float* __restrict__ scores, const float* __restrict__ p,
    const int* __restrict__ head_mask, int* __restrict__ idx, int* __restrict__ cnt) {
    constexpr int NT = kSelectThreads;
    constexpr int E = (N2 + NT - 1) / NT;   // sorted elements owned per thread in the scan
    __shared__ unsigned long long key[N2];
    __shared__ float warp_tot[NT / 32];
    __shared__ int warp_cnt[NT / 32];
    __shared__ int cut_pos;

    const int i = blockIdx.x, h = blockIdx.y;
    if (head_mask != nullptr && head_mask[h] == 0) return;
    const int nb = g.nb;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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

}  // namespace bsa
