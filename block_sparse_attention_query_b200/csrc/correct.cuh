// Cached dense correction of sparse attention (RECAP: Reciprocal Sparse Attention and
// Hierarchical Caching for Efficient Video Diffusion, Abstract: a cached dense refinement
// corrects the interactions the current sparse estimate omits; fresh statistics of the
// inputs regulate the aging correction).
//
// correct_kernel, grid (chunks, heads), after the dense attention of the refreshed heads was
// written into R: for a refreshed head, R = D - O (the new correction, D the dense output
// held in R) and O = D; for every other head, O = O + R (the sparse output plus the cached
// correction). bf16 in and out, float32 arithmetic, 16-byte loads: HBM-bound.
#pragma once

#include "bsa_common.cuh"

namespace bsa {

constexpr int kCorrThreads = 256;
constexpr int kCorrVecPerThread = 4;                                          // 16-byte vectors
constexpr int kCorrChunkElems = kCorrThreads * kCorrVecPerThread * 8;        // 8192 bf16

__device__ inline uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// elems = tokens * d per head (a multiple of 8).
__global__ void __launch_bounds__(kCorrThreads) correct_kernel(const int* __restrict__ refresh, long long elems,
                                                              bsa_bf16* __restrict__ O, bsa_bf16* __restrict__ R) {
    const int c = blockIdx.x, h = blockIdx.y;
    const bool fresh = refresh[h] != 0;
    const long long nvec = elems / 8;
    uint4* o4 = reinterpret_cast<uint4*>(O + (long long)h * elems);
    uint4* r4 = reinterpret_cast<uint4*>(R + (long long)h * elems);
    const long long v0 = (long long)c * (kCorrChunkElems / 8) + threadIdx.x;
    uint4 ov[kCorrVecPerThread], rv[kCorrVecPerThread];
#pragma unroll
    for (int k = 0; k < kCorrVecPerThread; ++k) {
        const long long v = v0 + (long long)k * kCorrThreads;
        if (v < nvec) {
            ov[k] = o4[v];
            rv[k] = r4[v];
        }
    }
#pragma unroll
    for (int k = 0; k < kCorrVecPerThread; ++k) {
        const long long v = v0 + (long long)k * kCorrThreads;
        if (v >= nvec) continue;
        const __nv_bfloat162* op = reinterpret_cast<const __nv_bfloat162*>(&ov[k]);
        const __nv_bfloat162* rp = reinterpret_cast<const __nv_bfloat162*>(&rv[k]);
        uint4 a;
        uint32_t* ap = reinterpret_cast<uint32_t*>(&a);
        if (fresh) {
            // R holds the dense output D: the new correction is D - O, the output D
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 o = __bfloat1622float2(op[e]);
                const float2 d = __bfloat1622float2(rp[e]);
                ap[e] = pack_bf16x2(d.x - o.x, d.y - o.y);
            }
            o4[v] = rv[k];
            r4[v] = a;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 o = __bfloat1622float2(op[e]);
                const float2 r = __bfloat1622float2(rp[e]);
                ap[e] = pack_bf16x2(o.x + r.x, o.y + r.y);
            }
            o4[v] = a;
        }
    }
}

}  // namespace bsa
