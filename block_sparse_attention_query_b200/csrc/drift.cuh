// Temporal Mask Reuse gate (HEART: Exploiting Head Heterogeneity in Sparse Attention for
// Video Diffusion, abstract: a per-head query-key drift signal decides whether the cached
// mask is refreshed; HASTE abstract: mask prediction skipped on small drift).
//
// drift_partial_kernel  grid (chunks, heads): streams Q, K, Q_ref, K_ref once with 16-byte
//   loads and writes four float64 partial sums per chunk (|Q-Qref|^2, |Qref|^2, |K-Kref|^2,
//   |Kref|^2). With force_all it also writes the new reference in the same pass.
// drift_pool_kernel     grid (nb, heads), the same sums taken block by block (rows through the
//   block-slot tables), also writing the block means of Q and K: the pooling that the scores
//   need, from the same pass over Q and K (bsa_problem.block_means).
// drift_finalize_kernel grid (chunks, heads): every CTA reduces its head's partials in a
//   fixed order (deterministic), so all of them agree on the decision; CTA 0 publishes
//   drift/refresh and, for a refreshed head, each CTA copies its chunk of Q, K to the
//   reference.
#pragma once

#include "bsa_common.cuh"

namespace bsa {

constexpr int kDriftThreads = 256;
constexpr int kDriftVecPerThread = 8;                                   // 16-byte vectors
constexpr int kDriftChunkElems = kDriftThreads * kDriftVecPerThread * 8; // 16384 bf16

__device__ inline void drift_accum(const uint4& a, const uint4& r, float& diff2, float& ref2) {
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 x = __bfloat1622float2(pa[k]);
        const float2 y = __bfloat1622float2(pr[k]);
        const float dx = x.x - y.x, dy = x.y - y.y;
        diff2 = fmaf(dx, dx, diff2);
        diff2 = fmaf(dy, dy, diff2);
        ref2 = fmaf(y.x, y.x, ref2);
        ref2 = fmaf(y.y, y.y, ref2);
    }
}

__device__ inline double block_sum_double(double v, double* scratch) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0) {
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += scratch[w];
    }
    return s;   // valid in thread 0
}

// elems = tokens * d per head (a multiple of 8).
__global__ void __launch_bounds__(kDriftThreads) drift_partial_kernel(
    const bsa_bf16* __restrict__ Q, const bsa_bf16* __restrict__ K, bsa_bf16* Qref,
    bsa_bf16* Kref, long long elems, int force_all, double* __restrict__ part) {
    const int c = blockIdx.x, h = blockIdx.y, nchunks = gridDim.x;
    const long long base = (long long)h * elems;
    const long long v0 = (long long)c * (kDriftChunkElems / 8);
    const long long nvec = elems / 8;
    const uint4* q4 = reinterpret_cast<const uint4*>(Q + base);
    const uint4* k4 = reinterpret_cast<const uint4*>(K + base);
    uint4* qr4 = reinterpret_cast<uint4*>(Qref + base);
    uint4* kr4 = reinterpret_cast<uint4*>(Kref + base);
    float dq = 0.f, rq = 0.f, dk = 0.f, rk = 0.f;
    uint4 a[kDriftVecPerThread], b[kDriftVecPerThread], ar[kDriftVecPerThread], br[kDriftVecPerThread];
#pragma unroll
    for (int k = 0; k < kDriftVecPerThread; ++k) {
        const long long v = v0 + threadIdx.x + (long long)k * kDriftThreads;
        if (v < nvec) {
            a[k] = __ldg(q4 + v);
            b[k] = __ldg(k4 + v);
            ar[k] = qr4[v];
            br[k] = kr4[v];
        } else {
            a[k] = b[k] = ar[k] = br[k] = make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int k = 0; k < kDriftVecPerThread; ++k) {
        drift_accum(a[k], ar[k], dq, rq);
        drift_accum(b[k], br[k], dk, rk);
    }
    if (force_all) {
#pragma unroll
        for (int k = 0; k < kDriftVecPerThread; ++k) {
            const long long v = v0 + threadIdx.x + (long long)k * kDriftThreads;
            if (v < nvec) { qr4[v] = a[k]; kr4[v] = b[k]; }
        }
    }
    __shared__ double scratch[kDriftThreads / 32];
    const double s0 = block_sum_double((double)dq, scratch);
    const double s1 = block_sum_double((double)rq, scratch);
    const double s2 = block_sum_double((double)dk, scratch);
    const double s3 = block_sum_double((double)rk, scratch);
    if (threadIdx.x == 0) {
        double* o = part + ((size_t)h * nchunks + c) * 4;
        o[0] = s0; o[1] = s1; o[2] = s2; o[3] = s3;
    }
}

// grid (nb, heads), kDriftPoolThreads threads: block i of head h. Query rows come from perm,
// key rows from kperm (per head, nullable: perm). Each thread owns 16-byte chunk c of NIT rows,
// taken two rows at a time (eight 16-byte loads of the four tensors in flight per thread, few
// registers, three CTAs per SM so that one CTA's loads overlap another's stores). Writes the
// four drift sums of the block (float64, fixed order) to part[h][i] and the means of Q and K
// over the block's real tokens to qbar/kbar [heads][nb][D]; with force_all also the snapshot
// (Q -> Qref, K -> Kref).
constexpr int kDriftPoolThreads = 256;

template <int D, int B>
__global__ void __launch_bounds__(kDriftPoolThreads, 3) drift_pool_kernel(
    Geom g, const bsa_bf16* __restrict__ Q, const bsa_bf16* __restrict__ K, bsa_bf16* Qref, bsa_bf16* Kref,
    const int* __restrict__ perm, const int* __restrict__ kperm, int force_all, double* __restrict__ part,
    float* __restrict__ qbar, float* __restrict__ kbar) {
    constexpr int CH = D / 8;                       // 16-byte chunks per row
    constexpr int RPP = kDriftPoolThreads / CH;     // rows per pass
    constexpr int NIT = B / RPP;                    // passes
    constexpr int PH = NIT >= 2 ? 2 : 1;            // rows loaded together
    static_assert(NIT >= 1 && RPP * NIT == B && NIT % PH == 0, "block rows per thread");
    const int i = blockIdx.x, h = blockIdx.y;
    const int c = threadIdx.x % CH, rs = threadIdx.x / CH;
    const size_t head_off = (size_t)h * g.N * D;
    const int* kp = kperm != nullptr ? kperm + (size_t)h * g.nb * B : perm;
    float dq = 0.f, sq = 0.f, dk = 0.f, sk = 0.f;
    float aq[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ak[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int k0 = 0; k0 < NIT; k0 += PH) {
        uint4 vq[PH], vk[PH], rq[PH], rk[PH];
        int tq[PH], tk[PH];
#pragma unroll
        for (int u = 0; u < PH; ++u) {
            const int slot = i * B + rs + (k0 + u) * RPP;
            tq[u] = __ldg(perm + slot);
            tk[u] = min(__ldg(kp + slot), g.N - 1);
            const size_t oq = head_off + (size_t)max(tq[u], 0) * D + c * 8;
            const size_t ok = head_off + (size_t)max(tk[u], 0) * D + c * 8;
            vq[u] = tq[u] >= 0 ? __ldg(reinterpret_cast<const uint4*>(Q + oq)) : z;
            vk[u] = tk[u] >= 0 ? __ldg(reinterpret_cast<const uint4*>(K + ok)) : z;
            rq[u] = tq[u] >= 0 ? *reinterpret_cast<const uint4*>(Qref + oq) : z;
            rk[u] = tk[u] >= 0 ? *reinterpret_cast<const uint4*>(Kref + ok) : z;
        }
#pragma unroll
        for (int u = 0; u < PH; ++u) {
            drift_accum(vq[u], rq[u], dq, sq);
            drift_accum(vk[u], rk[u], dk, sk);
            const __nv_bfloat162* pq = reinterpret_cast<const __nv_bfloat162*>(&vq[u]);
            const __nv_bfloat162* pk = reinterpret_cast<const __nv_bfloat162*>(&vk[u]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 a = __bfloat1622float2(pq[e]), b = __bfloat1622float2(pk[e]);
                aq[2 * e] += a.x;
                aq[2 * e + 1] += a.y;
                ak[2 * e] += b.x;
                ak[2 * e + 1] += b.y;
            }
            if (force_all) {
                if (tq[u] >= 0) *reinterpret_cast<uint4*>(Qref + head_off + (size_t)tq[u] * D + c * 8) = vq[u];
                if (tk[u] >= 0) *reinterpret_cast<uint4*>(Kref + head_off + (size_t)tk[u] * D + c * 8) = vk[u];
            }
        }
    }
    // block means: the RPP row groups' sums through shared memory, in a fixed order
    __shared__ float red[2][RPP][D + 4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        red[0][rs][c * 8 + e] = aq[e];
        red[1][rs][c * 8 + e] = ak[e];
    }
    __shared__ double scratch[kDriftPoolThreads / 32];
    const double s0 = block_sum_double((double)dq, scratch);   // (its first __syncthreads also
    const double s1 = block_sum_double((double)sq, scratch);   //  orders the stores to red)
    const double s2 = block_sum_double((double)dk, scratch);
    const double s3 = block_sum_double((double)sk, scratch);
    if (threadIdx.x == 0) {
        double* o = part + ((size_t)h * g.nb + i) * 4;
        o[0] = s0; o[1] = s1; o[2] = s2; o[3] = s3;
    }
    for (int t = threadIdx.x; t < 2 * D; t += kDriftPoolThreads) {
        const int which = t / D, col = t % D;
        float s = 0.f;
#pragma unroll 8
        for (int r = 0; r < RPP; ++r) s += red[which][r][col];
        const float n = (float)block_count(g, i);
        float* out = which == 0 ? qbar : kbar;
        out[((size_t)h * g.nb + i) * D + col] = s / n;
    }
}

__device__ inline double rel_change(double diff2, double ref2) {
    if (ref2 == 0.0) return diff2 == 0.0 ? 0.0 : (double)INFINITY;
    return sqrt(diff2 / ref2);
}

// grid (copy chunks of kDriftChunkElems, or 1 with force_all, heads); nparts partials per head.
__global__ void __launch_bounds__(kDriftThreads) drift_finalize_kernel(
    const bsa_bf16* __restrict__ Q, const bsa_bf16* __restrict__ K, bsa_bf16* Qref,
    bsa_bf16* Kref, long long elems, int force_all, float tau,
    const double* __restrict__ part, float* __restrict__ drift, int* __restrict__ refresh, int nparts) {
    const int c = blockIdx.x, h = blockIdx.y;
    __shared__ double scratch[kDriftThreads / 32];
    __shared__ int s_refresh;
    double acc[4] = {0, 0, 0, 0};
    const double* ph = part + (size_t)h * nparts * 4;
    for (int k = threadIdx.x; k < nparts; k += kDriftThreads) {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] += ph[(size_t)k * 4 + e];
    }
    double tot[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) tot[e] = block_sum_double(acc[e], scratch);
    if (threadIdx.x == 0) {
        const double dlt = fmax(rel_change(tot[0], tot[1]), rel_change(tot[2], tot[3]));
        const int fresh = force_all || dlt > (double)tau;
        s_refresh = fresh;
        if (c == 0) {
            drift[h] = (float)dlt;
            refresh[h] = fresh;
        }
    }
    __syncthreads();
    if (!s_refresh || force_all) return;   // with force_all the copy already happened
    const long long base = (long long)h * elems;
    const long long v0 = (long long)c * (kDriftChunkElems / 8);
    const long long nvec = elems / 8;
    const uint4* q4 = reinterpret_cast<const uint4*>(Q + base);
    const uint4* k4 = reinterpret_cast<const uint4*>(K + base);
    uint4* qr4 = reinterpret_cast<uint4*>(Qref + base);
    uint4* kr4 = reinterpret_cast<uint4*>(Kref + base);
#pragma unroll
    for (int k = 0; k < kDriftVecPerThread; ++k) {
        const long long v = v0 + threadIdx.x + (long long)k * kDriftThreads;
        if (v < nvec) { qr4[v] = __ldg(q4 + v); kr4[v] = __ldg(k4 + v); }
    }
}

}  // namespace bsa
