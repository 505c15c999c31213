// Retrieval accuracy: the share of each query's exact attention mass that its kept key blocks
// hold (PARK: Accurate Block Retrieval for Sparse Attention in Video Diffusion Transformers,
// Abstract: inaccurate retrieval degrades quality or wastes computation; methods are judged by
// block retrieval accuracy).
//
// For a real query t, with lse_kept(t) and lse_all(t) the log2-sum-exp of its scaled logits
// over the kept keys and over all keys (both from the attention kernel), the captured mass is
// 2^(lse_kept - lse_all). mass_kernel averages it over the real queries of each query block.
#pragma once

#include "bsa_common.cuh"

namespace bsa {

constexpr int kMassThreads = 128;   // one thread per block slot (B <= 128)

// grid (nb, heads): mass[h][i] = mean over the real queries t of block i of
// 2^(lse_kept[h][t] - lse_all[h][t]). Fixed reduction order (deterministic).
__global__ void __launch_bounds__(kMassThreads) mass_kernel(Geom g, const int* __restrict__ perm,
                                                           const float* __restrict__ lse_kept,
                                                           const float* __restrict__ lse_all,
                                                           float* __restrict__ mass) {
    const int i = blockIdx.x, h = blockIdx.y, r = threadIdx.x;
    float v = 0.f;
    if (r < g.B) {
        const int tok = perm[i * g.B + r];
        if (tok >= 0) {
            const size_t o = (size_t)h * g.N + tok;
            v = exp2f(lse_kept[o] - lse_all[o]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    __shared__ float part[kMassThreads / 32];
    if ((r & 31) == 0) part[r >> 5] = v;
    __syncthreads();
    if (r == 0) {
        float s = 0.f;
        for (int w = 0; w < kMassThreads / 32; ++w) s += part[w];
        mass[(size_t)h * g.nb + i] = s / (float)block_count(g, i);
    }
}

}  // namespace bsa
