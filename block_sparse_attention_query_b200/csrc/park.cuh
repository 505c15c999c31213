// PARK per-query-normalised block scorer (PARK: Accurate Block Retrieval for Sparse
// Attention in Video Diffusion Transformers, Abstract: every original query is kept, its
// attention over key blocks is normalised on its own, and the distributions are averaged
// within the query block).
//
//   P[h][i][j] = (1/n_i) * sum over real queries q of block i of softmax_j(q . kbar_j / sqrt(d))
//
// CUDA-core version: one CTA per (query block, head); queries in groups of R; float32 logits
// against every pooled key (kbar from the pooling pass, L2-resident), row softmax in shared
// memory, then a fixed-order column sum over the group's real queries.
#pragma once

#include "bsa_common.cuh"

namespace bsa {

template <int D, int R>
__global__ void __launch_bounds__(256) park_score_kernel(Geom g, const bsa_bf16* __restrict__ Q,
                                                         const float* __restrict__ kbar,
                                                         const int* __restrict__ head_mask,
                                                         float* __restrict__ scores, float scale) {
    extern __shared__ float4 smem_f4[];
    const int i = blockIdx.x, h = blockIdx.y;
    if (head_mask != nullptr && head_mask[h] == 0) return;
    const int nb = g.nb;
    const int nbp = (nb + 3) & ~3;
    float* sq = reinterpret_cast<float*>(smem_f4);   // [R][D]
    float* slog = sq + R * D;                         // [R][nbp]
    float* colsum = slog + R * nbp;                   // [nbp]
    __shared__ int s_tok[R];
    const float* kh = kbar + (size_t)h * nb * D;
    const bsa_bf16* Qh = Q + (size_t)h * g.N * D;
    const int n_real = block_count(g, i);
    for (int j = threadIdx.x; j < nbp; j += 256) colsum[j] = 0.f;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    for (int r0 = 0; r0 < g.B; r0 += R) {
        __syncthreads();
        if (threadIdx.x < R) s_tok[threadIdx.x] = slot_to_token(g, i * g.B + r0 + threadIdx.x);
        __syncthreads();
        for (int e = threadIdx.x; e < R * D; e += 256) {
            const int r = e / D, c = e % D;
            const int tok = s_tok[r];
            sq[e] = tok >= 0 ? __bfloat162float(__ushort_as_bfloat16(Qh[(size_t)tok * D + c])) : 0.f;
        }
        __syncthreads();
        const float4* sq4 = reinterpret_cast<const float4*>(sq);
        for (int jb = 0; jb < nb; jb += 512) {
            const int ja = jb + threadIdx.x, jbb = ja + 256;
            const float4* ka = reinterpret_cast<const float4*>(kh + (size_t)min(ja, nb - 1) * D);
            const float4* kb = reinterpret_cast<const float4*>(kh + (size_t)min(jbb, nb - 1) * D);
            float acc0[R], acc1[R];
#pragma unroll
            for (int r = 0; r < R; ++r) { acc0[r] = 0.f; acc1[r] = 0.f; }
#pragma unroll 2
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 a = __ldg(ka + c4), b = __ldg(kb + c4);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float4 q = sq4[r * (D / 4) + c4];
                    acc0[r] = fmaf(q.x, a.x, acc0[r]);
                    acc0[r] = fmaf(q.y, a.y, acc0[r]);
                    acc0[r] = fmaf(q.z, a.z, acc0[r]);
                    acc0[r] = fmaf(q.w, a.w, acc0[r]);
                    acc1[r] = fmaf(q.x, b.x, acc1[r]);
                    acc1[r] = fmaf(q.y, b.y, acc1[r]);
                    acc1[r] = fmaf(q.z, b.z, acc1[r]);
                    acc1[r] = fmaf(q.w, b.w, acc1[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if (ja < nb) slog[r * nbp + ja] = acc0[r] * scale;
                if (jbb < nb) slog[r * nbp + jbb] = acc1[r] * scale;
            }
        }
        __syncthreads();
        for (int r = warp; r < R; r += 8) {
            float* row = slog + r * nbp;
            if (s_tok[r] < 0) {
                for (int j = lane; j < nb; j += 32) row[j] = 0.f;
                continue;
            }
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
            for (int j = lane; j < nb; j += 32) row[j] *= inv;
        }
        __syncthreads();
        for (int j = threadIdx.x; j < nb; j += 256) {
            float s = colsum[j];
#pragma unroll
            for (int r = 0; r < R; ++r) s += slog[r * nbp + j];
            colsum[j] = s;
        }
    }
    __syncthreads();
    const float inv_n = 1.0f / (float)n_real;
    float* out = scores + ((size_t)h * nb + i) * nb;
    for (int j = threadIdx.x; j < nb; j += 256) out[j] = colsum[j] * inv_n;
}

inline int launch_park(const Geom& g, const bsa_bf16* Q, const float* kbar, const int* head_mask,
                       float* scores, cudaStream_t st) {
    const bool wide = g.nb > 1024;
    const int R = wide ? 16 : 32;
    const int nbp = (g.nb + 3) & ~3;
    const size_t smem = (size_t)(R * g.d + R * nbp + nbp) * sizeof(float);
    const dim3 grid(g.nb, g.heads);
    const float scale = 1.0f / std::sqrt((float)g.d);
    if (smem > 227 * 1024) return BSA_ERR_UNSUPPORTED;
#define BSA_PARK(DD, RR)                                                                           \
    do {                                                                                           \
        if (cudaFuncSetAttribute(park_score_kernel<DD, RR>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                 (int)smem) != cudaSuccess)                                        \
            return BSA_ERR_CUDA;                                                                   \
        park_score_kernel<DD, RR><<<grid, 256, smem, st>>>(g, Q, kbar, head_mask, scores, scale);  \
    } while (0)
    if (g.d == 128) { if (wide) BSA_PARK(128, 16); else BSA_PARK(128, 32); }
    else { if (wide) BSA_PARK(64, 16); else BSA_PARK(64, 32); }
#undef BSA_PARK
    return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

}  // namespace bsa
