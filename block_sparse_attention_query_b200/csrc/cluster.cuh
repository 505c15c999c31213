// Query-aware key blocks (PARK: Accurate Block Retrieval for Sparse Attention in Video Diffusion
// Transformers, Abstract: keys are transformed with information from the current queries before
// clustering, so that keys receiving similar QK scores are grouped together).
//
// Per head: M = Q^T Q / N over the real queries; (k1 - k2)^T M (k1 - k2) is the mean-square
// difference of the scores the queries give two keys. Lloyd's k-means with that metric over
// the video keys, one cluster per video block, started from the tile-block means: each round
// assigns every key to argmin_j (c_j^T M c_j - 2 k . M c_j) (the squared metric distance minus
// the key's own term; ties to the lowest j), then moves each non-empty cluster's centroid to
// the mean of its keys. The key table lists the video keys in (cluster, raster index) order;
// it is cut into blocks of B keys like the query side, so block sizes do not change.
//
// Kernels (all deterministic: fixed summation orders, no float atomics):
//   qtq_partial_kernel / qtq_reduce_kernel   M (float32 partials of 4096 rows, float64 sum)
//   centroid_init_kernel                     the tile-block means of the keys
//   centroid_prep_kernel                     w_j = M c_j, b_j = c_j . w_j
//   assign_kernel                            argmin over all centroids, 4 keys x 8 centroids
//                                            per thread, centroid chunks staged in smem
//   cluster_sort_kernel                      one warp per head: counting sort of the keys by
//                                            cluster, stable in the raster index
//   centroid_update_kernel                   per cluster: mean of its keys in sorted order
//   key_table_kernel                         sorted video keys, then the tile layout's slots
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace clu {

constexpr int kQtqRows = 4096;          // query rows per partial of M
constexpr int kQtqThreads = 256;
constexpr int kAssignKeys = 128;        // keys per CTA of the assignment
constexpr int kAssignChunk = 64;        // centroids staged per step
constexpr int kAssignThreads = 256;     // 32 key groups of 4 x 8 centroid groups of 8

// grid (chunks, heads), 256 threads: part[h][c] = sum over rows [c*4096, +4096) of q q^T.
// Thread (ti, tj), 16 x 16, owns the 8 x 8 tile rows 8ti.., columns 8tj.. of the D x D sum
// (D = 128; for D = 64 the threads with ti or tj >= 8 idle in the accumulation).
template <int D>
__global__ void __launch_bounds__(kQtqThreads) qtq_partial_kernel(const bsa_bf16* __restrict__ Q, int N,
                                                                 float* __restrict__ part) {
    constexpr int RS = 64;                          // rows staged at a time
    __shared__ float sq[RS][D + 4];
    const int c = blockIdx.x, h = blockIdx.y, nchunks = gridDim.x;
    const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
    const bool active = ti * 8 < D && tj * 8 < D;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
    const bsa_bf16* Qh = Q + (size_t)h * N * D;
    const int r0 = c * kQtqRows, r1 = min(N, r0 + kQtqRows);
    for (int rs = r0; rs < r1; rs += RS) {
        __syncthreads();
        for (int e = threadIdx.x; e < RS * (D / 8); e += kQtqThreads) {
            const int r = e / (D / 8), c8 = e % (D / 8);
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (rs + r < r1) {
                const uint4 u = *reinterpret_cast<const uint4*>(Qh + (size_t)(rs + r) * D + c8 * 8);
                const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 f = __bfloat1622float2(p2[k]);
                    v[2 * k] = f.x;
                    v[2 * k + 1] = f.y;
                }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) sq[r][c8 * 8 + k] = v[k];
        }
        __syncthreads();
        if (active) {
            const int nr = min(RS, r1 - rs);
            for (int r = 0; r < nr; ++r) {
                float x[8], y[8];
#pragma unroll
                for (int a = 0; a < 8; ++a) x[a] = sq[r][ti * 8 + a];
#pragma unroll
                for (int b = 0; b < 8; ++b) y[b] = sq[r][tj * 8 + b];
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(x[a], y[b], acc[a][b]);
            }
        }
    }
    if (active) {
        float* out = part + ((size_t)h * nchunks + c) * D * D;
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b) out[(ti * 8 + a) * D + tj * 8 + b] = acc[a][b];
    }
}

// grid (heads), D*D/... threads loop: M[h] = (sum of the partials, float64, in chunk order) / N.
template <int D>
__global__ void qtq_reduce_kernel(const float* __restrict__ part, int nchunks, int N, float* __restrict__ M) {
    const int h = blockIdx.x;
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
        double s = 0.0;
        for (int c = 0; c < nchunks; ++c) s += (double)part[((size_t)h * nchunks + c) * D * D + e];
        M[(size_t)h * D * D + e] = (float)(s / N);
    }
}

// grid (C, heads), D threads: w_j = M c_j and b_j = c_j . w_j (float32; M is symmetric).
template <int D>
__global__ void centroid_prep_kernel(const float* __restrict__ M, const float* __restrict__ cent, int C,
                                     float* __restrict__ W, float* __restrict__ bvec) {
    const int j = blockIdx.x, h = blockIdx.y, r = threadIdx.x;
    __shared__ float sc[D];
    __shared__ float red[D];
    const float* cj = cent + ((size_t)h * C + j) * D;
    sc[r] = cj[r];
    __syncthreads();
    const float* Mr = M + (size_t)h * D * D + (size_t)r * D;
    float w = 0.f;
    for (int k = 0; k < D; ++k) w = fmaf(Mr[k], sc[k], w);
    W[((size_t)h * C + j) * D + r] = w;
    red[r] = w * sc[r];
    __syncthreads();
    if (r == 0) {
        float b = 0.f;
        for (int k = 0; k < D; ++k) b += red[k];
        bvec[(size_t)h * C + j] = b;
    }
}

// grid (ceil(Nv/128), heads), 256 threads: a[h][u] = argmin_j (b_j - 2 K_u . w_j), ties to
// the lowest j. Thread t: keys (t%32) + 32q, q < 4, of the CTA's 128 (consecutive lanes read
// consecutive padded rows: no bank conflicts), centroids 8*(t/32) .. +7 of each staged chunk of
// 64 (one warp reads the same centroid row: broadcast); a final pass over shared memory picks
// each key's best of the 8 groups.
template <int D>
__global__ void __launch_bounds__(kAssignThreads) assign_kernel(const bsa_bf16* __restrict__ K, int N, int Nv,
                                                                const float* __restrict__ W,
                                                                const float* __restrict__ bvec, int C,
                                                                int* __restrict__ assign) {
    constexpr int KS = D + 4;                      // padded row stride (floats)
    extern __shared__ float4 smem_f4[];
    float* sk = reinterpret_cast<float*>(smem_f4);             // [128][KS]
    float* sw = sk + kAssignKeys * KS;                          // [64][KS]
    float* sb = sw + kAssignChunk * KS;                         // [64]
    float* bestv = sb + kAssignChunk;                           // [8][128]
    int* besti = reinterpret_cast<int*>(bestv + 8 * kAssignKeys);   // [8][128]
    const int h = blockIdx.y, u0 = blockIdx.x * kAssignKeys;
    const int kg = threadIdx.x % 32, cg = threadIdx.x / 32;
    const bsa_bf16* Kh = K + (size_t)h * N * D;
    for (int e = threadIdx.x; e < kAssignKeys * (D / 8); e += kAssignThreads) {
        const int r = e / (D / 8), c8 = e % (D / 8);
        float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (u0 + r < Nv) {
            const uint4 q = *reinterpret_cast<const uint4*>(Kh + (size_t)(u0 + r) * D + c8 * 8);
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = __bfloat1622float2(p2[k]);
                v[2 * k] = f.x;
                v[2 * k + 1] = f.y;
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) sk[r * KS + c8 * 8 + k] = v[k];
    }
    float bv[4];
    int bi[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        bv[q] = INFINITY;
        bi[q] = 0x7fffffff;
    }
    const float* Wh = W + (size_t)h * C * D;
    for (int j0 = 0; j0 < C; j0 += kAssignChunk) {
        __syncthreads();
        for (int e = threadIdx.x; e < kAssignChunk * (D / 4); e += kAssignThreads) {
            const int j = e / (D / 4), c4 = e % (D / 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j0 + j < C) v = *reinterpret_cast<const float4*>(Wh + (size_t)(j0 + j) * D + c4 * 4);
            *reinterpret_cast<float4*>(sw + j * KS + c4 * 4) = v;
        }
        if (threadIdx.x < kAssignChunk)
            sb[threadIdx.x] = j0 + threadIdx.x < C ? bvec[(size_t)h * C + j0 + threadIdx.x] : INFINITY;
        __syncthreads();
        float acc[4][8];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[q][c] = 0.f;
#pragma unroll 2
        for (int k4 = 0; k4 < D / 4; ++k4) {
            float4 kv[4], wv[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) kv[q] = *reinterpret_cast<const float4*>(sk + (kg + 32 * q) * KS + k4 * 4);
#pragma unroll
            for (int c = 0; c < 8; ++c) wv[c] = *reinterpret_cast<const float4*>(sw + (cg * 8 + c) * KS + k4 * 4);
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    acc[q][c] = fmaf(kv[q].x, wv[c].x, acc[q][c]);
                    acc[q][c] = fmaf(kv[q].y, wv[c].y, acc[q][c]);
                    acc[q][c] = fmaf(kv[q].z, wv[c].z, acc[q][c]);
                    acc[q][c] = fmaf(kv[q].w, wv[c].w, acc[q][c]);
                }
        }
        // centroids in increasing index order: strict < keeps the lowest index on ties
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int j = j0 + cg * 8 + c;
            if (j >= C) continue;
            const float bj = sb[cg * 8 + c];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float obj = fmaf(-2.f, acc[q][c], bj);
                if (obj < bv[q]) {
                    bv[q] = obj;
                    bi[q] = j;
                }
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        bestv[cg * kAssignKeys + kg + 32 * q] = bv[q];
        besti[cg * kAssignKeys + kg + 32 * q] = bi[q];
    }
    __syncthreads();
    if (threadIdx.x < kAssignKeys && u0 + threadIdx.x < Nv) {
        float v = INFINITY;
        int i = 0x7fffffff;
        for (int c = 0; c < 8; ++c) {          // lexicographic (value, index): lowest index on ties
            const float cv = bestv[c * kAssignKeys + threadIdx.x];
            const int ci = besti[c * kAssignKeys + threadIdx.x];
            if (cv < v || (cv == v && ci < i)) {
                v = cv;
                i = ci;
            }
        }
        assign[(size_t)h * Nv + u0 + threadIdx.x] = i < C ? i : 0;   // no finite objective (NaN input): 0
    }
}

// grid (heads), 32 threads (one warp), dynamic smem 2*(C+1) ints: order[h] = the video keys sorted
// by (cluster, raster index); start[h][j] = first position of cluster j, start[h][C] = Nv.
__global__ void cluster_sort_kernel(const int* __restrict__ assign, int Nv, int C, int* __restrict__ order,
                                    int* __restrict__ start) {
    extern __shared__ int sh[];
    int* cnt = sh;             // [C + 1]
    int* cur = sh + C + 1;     // [C + 1]
    const int h = blockIdx.x, lane = threadIdx.x;
    const int* a = assign + (size_t)h * Nv;
    for (int j = lane; j <= C; j += 32) cnt[j] = 0;
    __syncwarp();
    for (int u0 = 0; u0 < Nv; u0 += 32) {
        const int u = u0 + lane;
        const int j = u < Nv ? min(max(a[u], 0), C - 1) : C;   // lanes past the end count into bin C
        const unsigned peers = __match_any_sync(0xffffffffu, j);
        if ((peers & ((1u << lane) - 1u)) == 0) cnt[j] += __popc(peers);   // one lane per bin
        __syncwarp();
    }
    if (lane == 0) {                                 // exclusive scan of the C bins
        int s = 0;
        for (int j = 0; j < C; ++j) {
            const int c = cnt[j];
            cur[j] = s;
            start[(size_t)h * (C + 1) + j] = s;
            s += c;
        }
        start[(size_t)h * (C + 1) + C] = s;
    }
    __syncwarp();
    for (int u0 = 0; u0 < Nv; u0 += 32) {
        const int u = u0 + lane;
        const int j = u < Nv ? min(max(a[u], 0), C - 1) : C;
        const unsigned peers = __match_any_sync(0xffffffffu, j);
        const unsigned below = peers & ((1u << lane) - 1u);
        if (j < C) order[(size_t)h * Nv + cur[j] + __popc(below)] = u;
        __syncwarp();
        if (j < C && below == 0) cur[j] += __popc(peers);
        __syncwarp();
    }
}

// grid (C, heads), D threads: initial centroids = the first C rows (video blocks) of the pooled
// key means [heads][nb][D].
template <int D>
__global__ void centroid_init_kernel(const float* __restrict__ kbar, int nb, int C, float* __restrict__ cent) {
    const int j = blockIdx.x, h = blockIdx.y;
    cent[((size_t)h * C + j) * D + threadIdx.x] = kbar[((size_t)h * nb + j) * D + threadIdx.x];
}

// grid (C, heads), D threads: centroid j = mean of K over its keys (in sorted order); an empty
// cluster keeps its centroid.
template <int D>
__global__ void centroid_update_kernel(const bsa_bf16* __restrict__ K, int N, int Nv, int C,
                                       const int* __restrict__ order, const int* __restrict__ start,
                                       float* __restrict__ cent) {
    const int j = blockIdx.x, h = blockIdx.y, r = threadIdx.x;
    const int s0 = start[(size_t)h * (C + 1) + j], s1 = start[(size_t)h * (C + 1) + j + 1];
    if (s1 <= s0) return;
    const bsa_bf16* Kh = K + (size_t)h * N * D;
    float s = 0.f;
    for (int p = s0; p < s1; ++p) {
        const int u = order[(size_t)h * Nv + p];
        s += __bfloat162float(__ushort_as_bfloat16(Kh[(size_t)u * D + r]));
    }
    cent[((size_t)h * C + j) * D + r] = s / (float)(s1 - s0);
}

// grid (ceil(nb*B/256), heads): table[h][s] = order[h][s] for the video keys (s < Nv), else the
// tile layout's slot (padding, text).
__global__ void key_table_kernel(Geom g, const int* __restrict__ order, int* __restrict__ table) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x, h = blockIdx.y;
    if (s >= g.nb * g.B) return;
    table[(size_t)h * g.nb * g.B + s] = s < g.Nv ? order[(size_t)h * g.Nv + s] : slot_to_token(g, s);
}

}  // namespace clu
}  // namespace bsa
