// Block pooling and the CUDA-core mean-pooled block scorer.
//
// pool_kernel:  qbar[h][i] = mean of Q over the real tokens of block i (same for K).
//   HBM-bound: every real row of Q and K is read exactly once, 16-byte loads, CD/8 lanes
//   per 2*d-byte row, float32 accumulation, shared-memory tree reduction.
// meanpool_score_kernel: S[h][i][j] = softmax_j(qbar_i . kbar_j / sqrt(d)) for 8, 16 or 32
//   query rows per CTA against every key block; register-blocked float32 dot products, row
//   softmax in shared memory. Used when the problem is too small to fill the SMs with the
//   tensor-core scorer's 128-row items (meanpool_tc.cuh); same logits to float32 rounding.
// (PARK: Accurate Block Retrieval for Sparse Attention in Video Diffusion Transformers,
// Abstract: block retrieval from the averaged representations of query and key blocks.)
#pragma once

#include "bsa_common.cuh"

namespace bsa {

template <int D>
__device__ inline void accum_bf16x8(float (&acc)[8], const uint4& v) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float2 f = __bfloat1622float2(p[k]);
        acc[2 * k] += f.x;
        acc[2 * k + 1] += f.y;
    }
}

// grid (nb, heads), 256 threads. Pools Q and K of block i, head h into qbar/kbar [heads][nb][D].
// kperm (nullable): per-head key-side block-slot table [heads][nb*B] (query-aware key
// blocks); NULL: keys use the tile layout like the queries.
template <int D, int B>
__global__ void __launch_bounds__(256) pool_kernel(Geom g, const bsa_bf16* __restrict__ Q,
                                                   const bsa_bf16* __restrict__ K,
                                                   const int* __restrict__ perm,
                                                   const int* __restrict__ kperm,
                                                   const int* __restrict__ head_mask,
                                                   float* __restrict__ qbar, float* __restrict__ kbar) {
    constexpr int CH = D / 8;               // 16-byte chunks per row
    constexpr int RPP = 256 / CH;           // rows per pass
    constexpr int NIT = B / RPP;            // passes
    const int i = blockIdx.x, h = blockIdx.y;
    if (head_mask != nullptr && head_mask[h] == 0) return;
    const int c = threadIdx.x % CH, rs = threadIdx.x / CH;
    const size_t head_off = (size_t)h * g.N * D;

    int tok[NIT], tokk[NIT];
    const int* kp = kperm != nullptr ? kperm + (size_t)h * g.nb * B : perm;
#pragma unroll
    for (int k = 0; k < NIT; ++k) {
        tok[k] = __ldg(perm + i * B + rs + k * RPP);
        tokk[k] = min(__ldg(kp + i * B + rs + k * RPP), g.N - 1);   // a bad caller table stays in range
    }
    uint4 vq[NIT], vk[NIT];
#pragma unroll
    for (int k = 0; k < NIT; ++k) {
        vq[k] = tok[k] >= 0 ? __ldg(reinterpret_cast<const uint4*>(Q + head_off + (size_t)tok[k] * D + c * 8))
                            : make_uint4(0, 0, 0, 0);
        vk[k] = tokk[k] >= 0 ? __ldg(reinterpret_cast<const uint4*>(K + head_off + (size_t)tokk[k] * D + c * 8))
                             : make_uint4(0, 0, 0, 0);
    }
    float aq[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ak[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int k = 0; k < NIT; ++k) {
        accum_bf16x8<D>(aq, vq[k]);
        accum_bf16x8<D>(ak, vk[k]);
    }
    __shared__ float red[2][RPP][D + 4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        red[0][rs][c * 8 + e] = aq[e];
        red[1][rs][c * 8 + e] = ak[e];
    }
    __syncthreads();
    if (threadIdx.x < 2 * D) {
        const int which = threadIdx.x / D, col = threadIdx.x % D;
        float s = 0.f;
#pragma unroll 8
        for (int r = 0; r < RPP; ++r) s += red[which][r][col];
        const float n = (float)block_count(g, i);
        float* out = which == 0 ? qbar : kbar;
        out[((size_t)h * g.nb + i) * D + col] = s / n;
    }
}

// grid (ceil(nb/R), heads), 256 threads; dynamic smem = (R*D + KC*(D+4) + R*nbp) floats.
// Rows i0..i0+R-1 of head h: logits against every key block (pooled keys staged through
// shared memory KC at a time), then row softmax.
constexpr int kScoreKeyChunk = 64;

template <int D, int R>
__global__ void __launch_bounds__(256) meanpool_score_kernel(Geom g, const float* __restrict__ qbar,
                                                             const float* __restrict__ kbar,
                                                             const int* __restrict__ head_mask,
                                                             float* __restrict__ scores, float scale) {
    constexpr int KC = kScoreKeyChunk;
    constexpr int KS = D + 4;              // padded row stride of the staged keys
    constexpr int RPT = R / 4;             // rows per thread (4 row groups x 64 keys)
    extern __shared__ float4 smem_f4[];
    const int h = blockIdx.y, i0 = blockIdx.x * R;
    if (head_mask != nullptr && head_mask[h] == 0) return;
    const int nb = g.nb;
    const int nbp = (nb + 3) & ~3;
    float* sq = reinterpret_cast<float*>(smem_f4);      // [R][D]
    float* sk = sq + R * D;                              // [KC][KS]
    float* slog = sk + KC * KS;                          // [R][nbp]
    const float* qh = qbar + (size_t)h * nb * D;
    const float* kh = kbar + (size_t)h * nb * D;
    for (int e = threadIdx.x; e < R * D; e += 256) {
        const int r = e / D;
        sq[e] = (i0 + r < nb) ? qh[(size_t)(i0 + r) * D + (e % D)] : 0.f;
    }
    const int kk = threadIdx.x % KC, rg = threadIdx.x / KC;   // key in chunk, row group
    const float4* sq4 = reinterpret_cast<const float4*>(sq);
    for (int j0 = 0; j0 < nb; j0 += KC) {
        __syncthreads();                                 // previous chunk consumed
        for (int e = threadIdx.x; e < KC * (D / 4); e += 256) {
            const int j = e / (D / 4), c4 = e % (D / 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j0 + j < nb) v = __ldg(reinterpret_cast<const float4*>(kh + (size_t)(j0 + j) * D) + c4);
            *reinterpret_cast<float4*>(sk + j * KS + c4 * 4) = v;
        }
        __syncthreads();
        float acc[RPT];
#pragma unroll
        for (int q = 0; q < RPT; ++q) acc[q] = 0.f;
        const float4* krow = reinterpret_cast<const float4*>(sk + kk * KS);
#pragma unroll 4
        for (int c4 = 0; c4 < D / 4; ++c4) {
            const float4 kv = krow[c4];
#pragma unroll
            for (int q = 0; q < RPT; ++q) {
                const float4 qv = sq4[(rg * RPT + q) * (D / 4) + c4];
                acc[q] = fmaf(qv.x, kv.x, acc[q]);
                acc[q] = fmaf(qv.y, kv.y, acc[q]);
                acc[q] = fmaf(qv.z, kv.z, acc[q]);
                acc[q] = fmaf(qv.w, kv.w, acc[q]);
            }
        }
        if (j0 + kk < nb) {
#pragma unroll
            for (int q = 0; q < RPT; ++q) slog[(rg * RPT + q) * nbp + j0 + kk] = acc[q] * scale;
        }
    }
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int r = warp; r < R; r += 8) {
        if (i0 + r >= nb) break;
        float* row = slog + r * nbp;
        float mx = -INFINITY;
        for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, row[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        for (int j = lane; j < nb; j += 32) {
            const float e = expf(row[j] - mx);
            row[j] = e;
            sum += e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = 1.0f / sum;
        float* out = scores + ((size_t)h * nb + i0 + r) * nb;
        for (int j = lane; j < nb; j += 32) out[j] = row[j] * inv;
    }
}

}  // namespace bsa
