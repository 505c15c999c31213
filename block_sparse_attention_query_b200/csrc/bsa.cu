// libbsa host side: argument validation, planning and kernel launches behind the C ABI of
// include/bsa.h. Single translation unit so that the device error word is shared by every
// kernel of the library.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "bsa_common.cuh"
#include "score.cuh"
#include "park_tc.cuh"
#include "park_cluster.cuh"
#include "meanpool_tc.cuh"
#include "select.cuh"
#include "drift.cuh"
#include "attention.cuh"
#include "mass.cuh"
#include "correct.cuh"
#include "cluster.cuh"

using namespace bsa;

namespace {

constexpr int kMaxBlocks = 2048;   // top-p sorts at most 2048 keys per row in shared memory

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int resolve_tile(const bsa_problem& pr, int* tt, int* th, int* tw) {
    if (pr.tile_t == 0 && pr.tile_h == 0 && pr.tile_w == 0) {
        *tt = pr.block == 64 ? 1 : 2;
        *th = 8;
        *tw = 8;
        return BSA_OK;
    }
    if (pr.tile_t < 1 || pr.tile_h < 1 || pr.tile_w < 1) return BSA_ERR_ARG;
    if ((long long)pr.tile_t * pr.tile_h * pr.tile_w != pr.block) return BSA_ERR_ARG;
    *tt = pr.tile_t;
    *th = pr.tile_h;
    *tw = pr.tile_w;
    return BSA_OK;
}

// Validates the problem and fills the device geometry.
int make_geom(const bsa_problem* prob, Geom* g) {
    if (prob == nullptr) return BSA_ERR_ARG;
    const bsa_problem& pr = *prob;
    if (pr.d != 64 && pr.d != 128) return BSA_ERR_UNSUPPORTED;
    if (pr.block != 64 && pr.block != 128) return BSA_ERR_UNSUPPORTED;
    if (pr.score_mode != BSA_SCORE_MEANPOOL && pr.score_mode != BSA_SCORE_PARK) return BSA_ERR_ARG;
    if (pr.heads < 1 || pr.T < 1 || pr.H < 1 || pr.W < 1 || pr.text_tokens < 0) return BSA_ERR_ARG;
    const long long nv = (long long)pr.T * pr.H * pr.W;
    if (nv + pr.text_tokens != (long long)pr.tokens) return BSA_ERR_ARG;
    if ((long long)pr.heads * pr.tokens * pr.d >= (1LL << 40)) return BSA_ERR_UNSUPPORTED;
    if (pr.tokens >= (1 << 30)) return BSA_ERR_UNSUPPORTED;
    int tt, th, tw;
    const int rc = resolve_tile(pr, &tt, &th, &tw);
    if (rc != BSA_OK) return rc;
    Geom x;
    x.heads = pr.heads;
    x.N = pr.tokens;
    x.d = pr.d;
    x.B = pr.block;
    x.T = pr.T;
    x.H = pr.H;
    x.W = pr.W;
    x.text = pr.text_tokens;
    x.tt = tt;
    x.th = th;
    x.tw = tw;
    x.Nv = (int)nv;
    x.nbv = (int)((nv + pr.block - 1) / pr.block);
    x.nbt = (pr.text_tokens + pr.block - 1) / pr.block;
    x.nb = x.nbv + x.nbt;
    if ((long long)tt * pr.H * pr.W >= (1LL << 30)) return BSA_ERR_UNSUPPORTED;
    x.slab = tt * pr.H * pr.W;
    if (x.nb > kMaxBlocks) return BSA_ERR_UNSUPPORTED;
    *g = x;
    return BSA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Kernels this library has launched in this process (every launch is followed by exactly one
// launch_status() call, which counts it).
std::atomic<unsigned long long> g_launch_count{0};

int launch_status() {
    g_launch_count.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

size_t perm_bytes(const Geom& g) { return align256((size_t)g.nb * g.B * sizeof(int)); }

// Score workspace: [pooled Q means | pooled K means: heads*nb*d fp32 each][block-slot table]
size_t pooled_bytes(const Geom& g) { return align256((size_t)2 * g.heads * g.nb * g.d * sizeof(float)); }
// bsa_set_park_kernel: BSA_PARK_TWO_PASS forces the two-pass PARK kernel.
std::atomic<int> g_park_two_pass{0};

int tile_nbp(const Geom& g) { return (g.nb + park::NT - 1) / park::NT * park::NT; }
// PARK in one pass: key blocks split over a cluster of C CTAs, W per CTA (a multiple of 16);
// false when nb needs more than the largest portable cluster.
bool park_cluster_shape(const Geom& g, int* C, int* W) {
    const int wmax = parkc::kMaxCols;
    const int c = (g.nb + wmax - 1) / wmax;
    if (c < 1 || c > parkc::kMaxCluster) return false;
    const int w = ((g.nb + c - 1) / c + 15) / 16 * 16;
    if ((c - 1) * w >= g.nb) return false;   // every CTA holds at least one real key block
    *C = c;
    *W = w;
    return true;
}
// Rows of each bf16 part of the pooled keys per head: the tile count of the two-pass kernels,
// or the cluster's C * W, whichever is larger.
int park_nbp(const Geom& g) {
    int C = 0, W = 0, n = tile_nbp(g);
    if (park_cluster_shape(g, &C, &W) && C * W > n) n = (C * W + park::NT - 1) / park::NT * park::NT;
    return n;
}
// Both scorers keep the three bf16 parts of the pooled keys, [heads][3][nbp][d]; the
// mean-pooled one also those of the pooled queries, [heads][3][nbq][d] (nbq: nb rounded up to
// a multiple of 128), then one float per score row (its softmax offset).
size_t ksplit_bytes(const Geom& g) { return align256((size_t)g.heads * 3 * park_nbp(g) * g.d * 2); }
int mp_nbq(const Geom& g) { return (g.nb + mp::BQ - 1) / mp::BQ * mp::BQ; }
size_t qsplit_bytes(const Geom& g) { return align256((size_t)g.heads * 3 * mp_nbq(g) * g.d * 2); }
size_t rowoff_bytes(const Geom& g) { return align256((size_t)g.heads * g.nb * 2 * sizeof(float)); }
size_t score_ws_bytes(const Geom& g, int mode) {
    return pooled_bytes(g) + perm_bytes(g) + ksplit_bytes(g) +
           (mode == BSA_SCORE_MEANPOOL ? qsplit_bytes(g) + rowoff_bytes(g) : 0);
}

int sm_count();

// One-pass PARK on clusters; BSA_ERR_UNSUPPORTED when the shape or the device leaves it out
// (the caller then runs the two-pass kernel).
template <int D>
int launch_park_cluster(const Geom& g, const bsa_bf16* Q, const int* perm, const int* head_mask, float* scores,
                        const bsa_bf16* ksplit, int nbp, cudaStream_t st) {
    int C = 0, W = 0;
    if (!park_cluster_shape(g, &C, &W) || C * W > nbp) return BSA_ERR_UNSUPPORTED;
    const parkc::Layout L = parkc::layout<D>(W, C);
    if (L.total > 232448) return BSA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(parkc::park_cluster_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total) !=
        cudaSuccess)
        return BSA_ERR_CUDA;
    const int sms = sm_count();
    if (sms <= 0) return BSA_ERR_CUDA;
    parkc::Params P;
    P.g = g;
    P.Q = Q;
    P.ksplit = ksplit;
    P.perm = perm;
    P.head_mask = head_mask;
    P.scores = scores;
    P.nbp = nbp;
    P.W = W;
    P.C = C;
    P.n_items = g.heads * g.nb;
    P.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sms / C * C));
    cfg.blockDim = dim3(parkc::kThreads);
    cfg.dynamicSmemBytes = (size_t)L.total;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, parkc::park_cluster_kernel<D>, &cfg) != cudaSuccess || ncl <= 0) {
        (void)cudaGetLastError();
        return BSA_ERR_UNSUPPORTED;
    }
    if (ncl > P.n_items) ncl = P.n_items;
    P.n_clusters = ncl;
    cfg.gridDim = dim3((unsigned)(ncl * C));
    if (cudaLaunchKernelEx(&cfg, parkc::park_cluster_kernel<D>, P) != cudaSuccess) {
        launch_status();
        return BSA_ERR_CUDA;
    }
    return launch_status();
}

template <int D>
int launch_park(const Geom& g, const bsa_bf16* Q, const float* kbar, const int* perm, const int* head_mask,
                float* scores, bsa_bf16* ksplit, cudaStream_t st) {
    using C = park::Cfg<D>;
    const int nbp = park_nbp(g);
    const long long n = (long long)g.heads * nbp * D;
    park::split_kbar_kernel<D><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(g, kbar, nbp, ksplit);
    if (launch_status() != BSA_OK) return BSA_ERR_CUDA;
    if (!g_park_two_pass) {
        const int rc = launch_park_cluster<D>(g, Q, perm, head_mask, scores, ksplit, nbp, st);
        if (rc != BSA_ERR_UNSUPPORTED) return rc;
    }
    if (cudaFuncSetAttribute(park::park_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
        return BSA_ERR_CUDA;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return BSA_ERR_CUDA;
    park::Params P;
    P.g = g;
    P.Q = Q;
    P.ksplit = ksplit;
    P.perm = perm;
    P.head_mask = head_mask;
    P.scores = scores;
    P.nbp = nbp;
    P.n_items = g.heads * g.nb;
    P.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    const int grid = P.n_items < sms ? P.n_items : sms;
    park::park_tc_kernel<D><<<grid, park::kThreads, C::SMEM, st>>>(P);
    return launch_status();
}

template <int D>
int launch_meanpool(const Geom& g, const float* qbar, const float* kbar, const int* head_mask, float* scores,
                    bsa_bf16* qsplit, bsa_bf16* ksplit, float* rowoff, cudaStream_t st) {
    using C = mp::Cfg<D>;
    const int nbq = mp_nbq(g), nbp = tile_nbp(g);
    const long long nq = (long long)g.heads * nbq * D, nk = (long long)g.heads * nbp * D;
    park::split_kbar_kernel<D><<<(unsigned)((nq + 255) / 256), 256, 0, st>>>(g, qbar, nbq, qsplit);
    if (launch_status() != BSA_OK) return BSA_ERR_CUDA;
    park::split_kbar_kernel<D><<<(unsigned)((nk + 255) / 256), 256, 0, st>>>(g, kbar, nbp, ksplit);
    if (launch_status() != BSA_OK) return BSA_ERR_CUDA;
    if (cudaFuncSetAttribute(mp::meanpool_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
        return BSA_ERR_CUDA;
    const int sms = sm_count();
    if (sms <= 0) return BSA_ERR_CUDA;
    mp::Params P;
    P.g = g;
    P.qsplit = qsplit;
    P.ksplit = ksplit;
    P.head_mask = head_mask;
    P.scores = scores;
    P.rowoff = rowoff;
    P.nbq = nbq;
    P.nbp = nbp;
    // too few (head, query tile) items to fill the SMs twice: each item's key tiles in two
    // halves, the halves' log-sum-exps combined by the normalisation pass
    const int base_items = g.heads * (nbq / mp::BQ), ntiles = nbp / mp::NT;
    P.nsplit = (base_items < 2 * sms && ntiles >= 2) ? 2 : 1;
    P.tps = (ntiles + P.nsplit - 1) / P.nsplit;
    P.n_items = base_items * P.nsplit;
    P.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    const int grid = P.n_items < sms ? P.n_items : sms;
    mp::meanpool_tc_kernel<D><<<grid, mp::kThreads, C::SMEM, st>>>(P);
    if (launch_status() != BSA_OK) return BSA_ERR_CUDA;
    mp::normalize_rows_kernel<<<g.heads * g.nb, 128, 0, st>>>(g, head_mask, rowoff, P.nsplit, scores);
    return launch_status();
}

int drift_chunks(const Geom& g) {
    const long long elems = (long long)g.N * g.d;
    return (int)((elems + kDriftChunkElems - 1) / kDriftChunkElems);
}

// Drift workspace: [float64 partial sums: heads * max(chunks, nb) * 4][block-slot table (fused
// path with bsa_problem.block_means)]
size_t drift_part_bytes(const Geom& g) {
    const int parts = drift_chunks(g) > g.nb ? drift_chunks(g) : g.nb;
    return align256((size_t)g.heads * parts * 4 * sizeof(double));
}
size_t drift_ws_bytes(const Geom& g) { return drift_part_bytes(g) + perm_bytes(g); }

int text_splits(const Geom& g) { return (g.nb + attn::kTextChunk - 1) / attn::kTextChunk; }

// Attention workspace: [perm: nb*B int32][text partial O: items*BQ*d fp32][text lse: items*BQ fp32]

size_t attention_ws_bytes(const Geom& g) {
    size_t bytes = perm_bytes(g);
    if (g.nbt > 0) {
        const size_t items = (size_t)g.heads * g.nbt * text_splits(g);
        bytes += align256(items * attn::BQ * (size_t)g.d * sizeof(float));
        bytes += align256(items * attn::BQ * sizeof(float));
    }
    return bytes;
}

// Captured-mass workspace: [attention workspace][O scratch: heads*N*d bf16]
// [kept-set lse: heads*N fp32][all-blocks lse: heads*N fp32]
size_t mass_ws_bytes(const Geom& g) {
    const size_t rows = (size_t)g.heads * g.N;
    return attention_ws_bytes(g) + align256(rows * g.d * 2) + 2 * align256(rows * sizeof(float));
}

// Clustering workspace: [M partials: heads*chunks*d*d f32][M: heads*d*d f32][pooled means:
// 2*heads*nb*d f32][block-slot table][centroids, M c: 2*heads*C*d f32][c.Mc: heads*C f32]
// [assignment, order: 2*heads*Nv i32][cluster starts: heads*(C+1) i32]
int qtq_chunks(const Geom& g) { return (g.N + clu::kQtqRows - 1) / clu::kQtqRows; }
size_t cluster_ws_bytes(const Geom& g) {
    const size_t h = g.heads, d = g.d, C = g.nbv, Nv = g.Nv;
    return align256(h * qtq_chunks(g) * d * d * 4) + align256(h * d * d * 4) + pooled_bytes(g) + perm_bytes(g) +
           2 * align256(h * C * d * 4) + align256(h * C * 4) + 2 * align256(h * Nv * 4) + align256(h * (C + 1) * 4);
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
}


template <int D, int BK>
int launch_attention(const attn::Params& P, cudaStream_t st) {
    using C = attn::Cfg<D, BK>;
    // set on every call: the attribute is per device and the call is cheap
    if (cudaFuncSetAttribute(attn::sparse_attention_kernel<D, BK>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return BSA_ERR_CUDA;
    const int sms = sm_count();
    if (sms <= 0) return BSA_ERR_CUDA;
    const int grid = P.n_items < sms ? P.n_items : sms;   // persistent: one CTA per SM
    const int total = P.g.nb * P.g.B;
    perm_kernel<<<(total + 255) / 256, 256, 0, st>>>(P.g, const_cast<int*>(P.perm));
    int rc = launch_status();
    if (rc != BSA_OK) return rc;
    attn::sparse_attention_kernel<D, BK><<<grid, attn::kThreads, C::SMEM, st>>>(P);
    rc = launch_status();
    if (rc != BSA_OK) return rc;
    if (P.n_text_items > 0) {
        dim3 grid(P.g.heads * P.g.nbt, attn::BQ);
        attn::merge_text_kernel<D><<<grid, D, 0, st>>>(P);
        rc = launch_status();
    }
    return rc;
}

attn::Params attention_params(const Geom& g, const bsa_bf16* Q, const bsa_bf16* K, const bsa_bf16* V,
                              const int* idx, const int* cnt, bsa_bf16* O, float* lse, void* ws,
                              const int* key_table) {
    attn::Params P;
    P.g = g;
    P.kperm = key_table;
    P.Q = Q;
    P.K = K;
    P.V = V;
    P.idx = idx;
    P.cnt = cnt;
    P.O = O;
    P.lse = lse;
    P.head_mask = nullptr;
    P.nsplit = g.nbt > 0 ? text_splits(g) : 1;
    P.n_text_items = g.heads * g.nbt * (g.nbt > 0 ? P.nsplit : 0);
    uint8_t* w = static_cast<uint8_t*>(ws);
    P.perm = reinterpret_cast<int*>(w);
    P.part_o = g.nbt > 0 ? reinterpret_cast<float*>(w + perm_bytes(g)) : nullptr;
    P.part_lse = g.nbt > 0 ? reinterpret_cast<float*>(w + perm_bytes(g) +
                                                      align256((size_t)P.n_text_items * attn::BQ * g.d * sizeof(float)))
                           : nullptr;
    P.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.d));
    P.n_items = P.n_text_items + g.heads * g.nbv;
    return P;
}

template <int D>
int run_cluster(const Geom& g, const bsa_bf16* Q, const bsa_bf16* K, int iters, int nchunks, float* part,
                float* M, const float* kbar, float* cent, float* Wc, float* bvec, int* assign, int* order,
                int* start, int* key_table, cudaStream_t st) {
    int rc;
    const int C = g.nbv, Nv = g.Nv;
    clu::qtq_partial_kernel<D><<<dim3(nchunks, g.heads), clu::kQtqThreads, 0, st>>>(Q, g.N, part);
    if ((rc = launch_status()) != BSA_OK) return rc;
    clu::qtq_reduce_kernel<D><<<g.heads, 256, 0, st>>>(part, nchunks, g.N, M);
    if ((rc = launch_status()) != BSA_OK) return rc;
    clu::centroid_init_kernel<D><<<dim3(C, g.heads), D, 0, st>>>(kbar, g.nb, C, cent);
    if ((rc = launch_status()) != BSA_OK) return rc;
    constexpr int KS = D + 4;
    const int asmem = (clu::kAssignKeys * KS + clu::kAssignChunk * KS + clu::kAssignChunk +
                       2 * 8 * clu::kAssignKeys) * 4;
    if (cudaFuncSetAttribute(clu::assign_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, asmem) != cudaSuccess)
        return BSA_ERR_CUDA;
    const dim3 agrid((Nv + clu::kAssignKeys - 1) / clu::kAssignKeys, g.heads);
    for (int t = 0; t < iters; ++t) {
        clu::centroid_prep_kernel<D><<<dim3(C, g.heads), D, 0, st>>>(M, cent, C, Wc, bvec);
        if ((rc = launch_status()) != BSA_OK) return rc;
        clu::assign_kernel<D><<<agrid, clu::kAssignThreads, asmem, st>>>(K, g.N, Nv, Wc, bvec, C, assign);
        if ((rc = launch_status()) != BSA_OK) return rc;
        clu::cluster_sort_kernel<<<g.heads, 32, 2 * (C + 1) * sizeof(int), st>>>(assign, Nv, C, order, start);
        if ((rc = launch_status()) != BSA_OK) return rc;
        if (t + 1 < iters) {
            clu::centroid_update_kernel<D><<<dim3(C, g.heads), D, 0, st>>>(K, g.N, Nv, C, order, start, cent);
            if ((rc = launch_status()) != BSA_OK) return rc;
        }
    }
    clu::key_table_kernel<<<dim3((g.nb * g.B + 255) / 256, g.heads), 256, 0, st>>>(g, order, key_table);
    return launch_status();
}

int run_attention(const attn::Params& P, cudaStream_t st) {
    const Geom& g = P.g;
    if (g.d == 128 && g.B == 128) return launch_attention<128, 128>(P, st);
    if (g.d == 128) return launch_attention<128, 64>(P, st);
    if (g.B == 128) return launch_attention<64, 128>(P, st);
    return launch_attention<64, 64>(P, st);
}

}  // namespace

extern "C" {

int bsa_plan(const bsa_problem* prob, bsa_plan_info* out) {
    if (out == nullptr) return BSA_ERR_ARG;
    Geom g;
    const int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    bsa_plan_info info;
    std::memset(&info, 0, sizeof(info));
    info.nb = g.nb;
    info.nb_video = g.nbv;
    info.nb_text = g.nbt;
    info.npad = g.nb * g.B;
    info.tile_t = g.tt;
    info.tile_h = g.th;
    info.tile_w = g.tw;
    info.score_workspace_bytes = score_ws_bytes(g, prob->score_mode);
    info.drift_workspace_bytes = drift_ws_bytes(g);
    info.attention_workspace_bytes = attention_ws_bytes(g);
    info.mass_workspace_bytes = mass_ws_bytes(g);
    info.cluster_workspace_bytes = cluster_ws_bytes(g);
    int pc = 0, pw = 0;
    if (park_cluster_shape(g, &pc, &pw)) {
        info.park_cluster = pc;
        info.park_cols = pw;
    }
    *out = info;
    return BSA_OK;
}

int bsa_block_layout(const bsa_problem* prob, int* perm_host) {
    if (perm_host == nullptr) return BSA_ERR_ARG;
    Geom g;
    const int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    for (int s = 0; s < g.nb * g.B; ++s) perm_host[s] = slot_to_token(g, s);
    return BSA_OK;
}

int bsa_score_blocks(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                     const int* head_mask, float* scores, void* ws, size_t ws_bytes,
                     bsa_stream_t stream) {
    Geom g;
    int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    if (Q == nullptr || K == nullptr || scores == nullptr) return BSA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(scores) || !aligned16(head_mask) ||
        !aligned16(prob->key_table))
        return BSA_ERR_ALIGN;
    if (ws == nullptr || ws_bytes < score_ws_bytes(g, prob->score_mode)) return BSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return BSA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (!aligned16(prob->block_means)) return BSA_ERR_ALIGN;
    // block means: from the drift pass of this step (bsa_problem.block_means), else pooled here
    float* qbar = prob->block_means != nullptr ? prob->block_means : static_cast<float*>(ws);
    float* kbar = qbar + (size_t)g.heads * g.nb * g.d;
    int* perm = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + pooled_bytes(g));
    const int total = g.nb * g.B;
    perm_kernel<<<(total + 255) / 256, 256, 0, st>>>(g, perm);
    if ((rc = launch_status()) != BSA_OK) return rc;
    const dim3 pgrid(g.nb, g.heads);
    if (prob->block_means == nullptr) {
    const int* kperm = prob->key_table;
    if (g.d == 128 && g.B == 128) pool_kernel<128, 128><<<pgrid, 256, 0, st>>>(g, Q, K, perm, kperm, head_mask, qbar, kbar);
    else if (g.d == 128) pool_kernel<128, 64><<<pgrid, 256, 0, st>>>(g, Q, K, perm, kperm, head_mask, qbar, kbar);
    else if (g.B == 128) pool_kernel<64, 128><<<pgrid, 256, 0, st>>>(g, Q, K, perm, kperm, head_mask, qbar, kbar);
    else pool_kernel<64, 64><<<pgrid, 256, 0, st>>>(g, Q, K, perm, kperm, head_mask, qbar, kbar);
    if ((rc = launch_status()) != BSA_OK) return rc;
    }
    bsa_bf16* ksplit = reinterpret_cast<bsa_bf16*>(static_cast<uint8_t*>(ws) + pooled_bytes(g) + perm_bytes(g));
    if (prob->score_mode == BSA_SCORE_MEANPOOL && (long long)g.heads * mp_nbq(g) / mp::BQ < sm_count()) {
        // fewer 128-row items than SMs: the CUDA-core scorer with 8-32 rows per CTA
        const float scale = 1.0f / std::sqrt((float)g.d);
        const int nbp = (g.nb + 3) & ~3;
        int R = 32;
        if (g.nb > 1024) R = 16;
        while (R > 8 && (long long)((g.nb + R - 1) / R) * g.heads < 296) R >>= 1;
        const size_t smem = (size_t)(R * g.d + kScoreKeyChunk * (g.d + 4) + R * nbp) * sizeof(float);
        const dim3 grid((g.nb + R - 1) / R, g.heads);
#define BSA_MP(DD, RR)                                                                             \
    do {                                                                                           \
        if (cudaFuncSetAttribute(meanpool_score_kernel<DD, RR>,                                    \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
            return BSA_ERR_CUDA;                                                                   \
        meanpool_score_kernel<DD, RR><<<grid, 256, smem, st>>>(g, qbar, kbar, head_mask, scores, scale); \
    } while (0)
        if (g.d == 128) { if (R == 32) BSA_MP(128, 32); else if (R == 16) BSA_MP(128, 16); else BSA_MP(128, 8); }
        else { if (R == 32) BSA_MP(64, 32); else if (R == 16) BSA_MP(64, 16); else BSA_MP(64, 8); }
#undef BSA_MP
        return launch_status();
    }
    if (prob->score_mode == BSA_SCORE_MEANPOOL) {
        bsa_bf16* qsplit = reinterpret_cast<bsa_bf16*>(reinterpret_cast<uint8_t*>(ksplit) + ksplit_bytes(g));
        float* rowoff = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(qsplit) + qsplit_bytes(g));
        if (g.d == 128) return launch_meanpool<128>(g, qbar, kbar, head_mask, scores, qsplit, ksplit, rowoff, st);
        return launch_meanpool<64>(g, qbar, kbar, head_mask, scores, qsplit, ksplit, rowoff, st);
    }
    if (g.d == 128) return launch_park<128>(g, Q, kbar, perm, head_mask, scores, ksplit, st);
    return launch_park<64>(g, Q, kbar, perm, head_mask, scores, ksplit, st);
}

int bsa_select_topp(const bsa_problem* prob, const float* scores, const float* p,
                    const int* head_mask, int* idx, int* cnt, bsa_stream_t stream) {
    Geom g;
    const int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    if (scores == nullptr || p == nullptr || idx == nullptr || cnt == nullptr) return BSA_ERR_ARG;
    if (!aligned16(scores) || !aligned16(idx) || !aligned16(cnt) || !aligned16(head_mask)) return BSA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // pass 1: one warp per video row extracts the top-p prefix (rows of up to 1024 blocks)
    const int sort_all = (g.nb > 1024 || g.nbt > 64) ? 1 : 0;
    if (!sort_all) {
        const long long rows = (long long)g.heads * g.nb;
        const int wgrid = (int)((rows + 7) / 8);
#define BSA_WSEL(EE) select_topp_warp_kernel<EE><<<wgrid, 256, 0, st>>>(g, scores, p, head_mask, idx, cnt)
        if (g.nb <= 64) BSA_WSEL(2);
        else if (g.nb <= 128) BSA_WSEL(4);
        else if (g.nb <= 256) BSA_WSEL(8);
        else if (g.nb <= 512) BSA_WSEL(16);
        else BSA_WSEL(32);
#undef BSA_WSEL
        const int rc = launch_status();
        if (rc != BSA_OK) return rc;
    }
    // pass 2: CTAs walk the rows (grid-stride) and fully sort the remaining ones (text rows,
    // p >= 1, overflow, or all of them)
    const int rows_all = g.heads * g.nb;
    const int grid = sort_all ? rows_all : (rows_all < 1184 ? rows_all : 1184);
    if (g.nb <= 64) select_topp_kernel<64><<<grid, kSelectThreads, 0, st>>>(g, scores, p, head_mask, idx, cnt, sort_all);
    else if (g.nb <= 128) select_topp_kernel<128><<<grid, kSelectThreads, 0, st>>>(g, scores, p, head_mask, idx, cnt, sort_all);
    else if (g.nb <= 256) select_topp_kernel<256><<<grid, kSelectThreads, 0, st>>>(g, scores, p, head_mask, idx, cnt, sort_all);
    else if (g.nb <= 512) select_topp_kernel<512><<<grid, kSelectThreads, 0, st>>>(g, scores, p, head_mask, idx, cnt, sort_all);
    else if (g.nb <= 1024) select_topp_kernel<1024><<<grid, kSelectThreads, 0, st>>>(g, scores, p, head_mask, idx, cnt, sort_all);
    else select_topp_kernel<2048><<<grid, kSelectThreads, 0, st>>>(g, scores, p, head_mask, idx, cnt, sort_all);
    return launch_status();
}

int bsa_drift_check(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                    bsa_bf16* Q_ref, bsa_bf16* K_ref, float tau, int force_all, float* drift,
                    int* refresh, void* ws, size_t ws_bytes, bsa_stream_t stream) {
    Geom g;
    const int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    if (Q == nullptr || K == nullptr || Q_ref == nullptr || K_ref == nullptr || drift == nullptr ||
        refresh == nullptr)
        return BSA_ERR_ARG;
    if (!(tau >= 0.0f) || std::isinf(tau)) return BSA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(Q_ref) || !aligned16(K_ref) || !aligned16(drift) ||
        !aligned16(refresh))
        return BSA_ERR_ALIGN;
    if (!aligned16(prob->block_means) || !aligned16(prob->key_table)) return BSA_ERR_ALIGN;
    const int chunks = drift_chunks(g);
    const bool fused = prob->block_means != nullptr;
    const size_t need = fused ? drift_ws_bytes(g) : (size_t)g.heads * chunks * 4 * sizeof(double);
    if (ws == nullptr || ws_bytes < need) return BSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return BSA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const long long elems = (long long)g.N * g.d;
    double* part = static_cast<double*>(ws);
    int nparts = chunks;
    int r2;
    if (fused) {
        // one pass over Q, K, Q_ref, K_ref block by block: the drift sums and the block means
        int* perm = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + drift_part_bytes(g));
        perm_kernel<<<(g.nb * g.B + 255) / 256, 256, 0, st>>>(g, perm);
        if ((r2 = launch_status()) != BSA_OK) return r2;
        float* qbar = prob->block_means;
        float* kbar = qbar + (size_t)g.heads * g.nb * g.d;
        const dim3 pgrid(g.nb, g.heads);
        const int f = force_all ? 1 : 0;
        const int* kp = prob->key_table;
#define BSA_DP(DD, BB) drift_pool_kernel<DD, BB><<<pgrid, kDriftPoolThreads, 0, st>>>(g, Q, K, Q_ref, K_ref, perm, kp, f, part, qbar, kbar)
        if (g.d == 128 && g.B == 128) BSA_DP(128, 128);
        else if (g.d == 128) BSA_DP(128, 64);
        else if (g.B == 128) BSA_DP(64, 128);
        else BSA_DP(64, 64);
#undef BSA_DP
        nparts = g.nb;
    } else {
        drift_partial_kernel<<<dim3(chunks, g.heads), kDriftThreads, 0, st>>>(Q, K, Q_ref, K_ref, elems,
                                                                             force_all ? 1 : 0, part);
    }
    if ((r2 = launch_status()) != BSA_OK) return r2;
    // with force_all the snapshot was taken in the first pass: one CTA per head publishes
    const dim3 fgrid(force_all ? 1 : chunks, g.heads);
    drift_finalize_kernel<<<fgrid, kDriftThreads, 0, st>>>(Q, K, Q_ref, K_ref, elems, force_all ? 1 : 0, tau,
                                                          part, drift, refresh, nparts);
    return launch_status();
}

int bsa_sparse_attention(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                         const bsa_bf16* V, const int* idx, const int* cnt, bsa_bf16* O, void* ws,
                         size_t ws_bytes, bsa_stream_t stream) {
    Geom g;
    const int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr) return BSA_ERR_ARG;
    if ((idx == nullptr) != (cnt == nullptr)) return BSA_ERR_ARG;   // both NULL: dense
    if (!aligned16(prob->key_table)) return BSA_ERR_ALIGN;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(cnt) || !aligned16(O))
        return BSA_ERR_ALIGN;
    const size_t need = attention_ws_bytes(g);
    if (ws == nullptr || ws_bytes < need) return BSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return BSA_ERR_ALIGN;
    const attn::Params P = attention_params(g, Q, K, V, idx, cnt, O, nullptr, ws, prob->key_table);
    return run_attention(P, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_cluster_keys(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K, int iters,
                     int* key_table, int* assignment, void* ws, size_t ws_bytes, bsa_stream_t stream) {
    Geom g;
    int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    if (Q == nullptr || K == nullptr || key_table == nullptr) return BSA_ERR_ARG;
    if (iters < 1 || iters > 64 || g.nbv < 1) return BSA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(key_table) || !aligned16(assignment)) return BSA_ERR_ALIGN;
    if (ws == nullptr || ws_bytes < cluster_ws_bytes(g)) return BSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return BSA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t h = g.heads, d = g.d, C = g.nbv, Nv = g.Nv;
    const int nchunks = qtq_chunks(g);
    uint8_t* w = static_cast<uint8_t*>(ws);
    float* part = reinterpret_cast<float*>(w);                        w += align256(h * nchunks * d * d * 4);
    float* M = reinterpret_cast<float*>(w);                           w += align256(h * d * d * 4);
    float* qbar = reinterpret_cast<float*>(w);
    float* kbar = qbar + h * g.nb * d;                                w += pooled_bytes(g);
    int* perm = reinterpret_cast<int*>(w);                            w += perm_bytes(g);
    float* cent = reinterpret_cast<float*>(w);                        w += align256(h * C * d * 4);
    float* Wc = reinterpret_cast<float*>(w);                          w += align256(h * C * d * 4);
    float* bvec = reinterpret_cast<float*>(w);                        w += align256(h * C * 4);
    int* assign = assignment != nullptr ? assignment : reinterpret_cast<int*>(w);
    w += align256(h * Nv * 4);
    int* order = reinterpret_cast<int*>(w);                           w += align256(h * Nv * 4);
    int* start = reinterpret_cast<int*>(w);
    perm_kernel<<<(g.nb * g.B + 255) / 256, 256, 0, st>>>(g, perm);
    if ((rc = launch_status()) != BSA_OK) return rc;
    const dim3 pgrid(g.nb, g.heads);
    if (g.d == 128 && g.B == 128) pool_kernel<128, 128><<<pgrid, 256, 0, st>>>(g, Q, K, perm, nullptr, nullptr, qbar, kbar);
    else if (g.d == 128) pool_kernel<128, 64><<<pgrid, 256, 0, st>>>(g, Q, K, perm, nullptr, nullptr, qbar, kbar);
    else if (g.B == 128) pool_kernel<64, 128><<<pgrid, 256, 0, st>>>(g, Q, K, perm, nullptr, nullptr, qbar, kbar);
    else pool_kernel<64, 64><<<pgrid, 256, 0, st>>>(g, Q, K, perm, nullptr, nullptr, qbar, kbar);
    if ((rc = launch_status()) != BSA_OK) return rc;
    return g.d == 128 ? run_cluster<128>(g, Q, K, iters, nchunks, part, M, kbar, cent, Wc, bvec, assign, order,
                                         start, key_table, st)
                      : run_cluster<64>(g, Q, K, iters, nchunks, part, M, kbar, cent, Wc, bvec, assign, order,
                                        start, key_table, st);
}

int bsa_dense_correction(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                         const bsa_bf16* V, const int* refresh, bsa_bf16* O, bsa_bf16* R,
                         void* ws, size_t ws_bytes, bsa_stream_t stream) {
    Geom g;
    int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    if (Q == nullptr || K == nullptr || V == nullptr || refresh == nullptr || O == nullptr || R == nullptr)
        return BSA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(refresh) || !aligned16(O) || !aligned16(R) ||
        !aligned16(prob->key_table))
        return BSA_ERR_ALIGN;
    if (ws == nullptr || ws_bytes < attention_ws_bytes(g)) return BSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return BSA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // dense attention of the refreshed heads, written into their rows of R
    attn::Params P = attention_params(g, Q, K, V, nullptr, nullptr, R, nullptr, ws, prob->key_table);
    P.head_mask = refresh;
    if ((rc = run_attention(P, st)) != BSA_OK) return rc;
    const long long elems = (long long)g.N * g.d;
    const dim3 grid((unsigned)((elems + kCorrChunkElems - 1) / kCorrChunkElems), g.heads);
    correct_kernel<<<grid, kCorrThreads, 0, st>>>(refresh, elems, O, R);
    return launch_status();
}

int bsa_captured_mass(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K, const int* idx,
                      const int* cnt, float* mass, void* ws, size_t ws_bytes, bsa_stream_t stream) {
    Geom g;
    int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    if (Q == nullptr || K == nullptr || idx == nullptr || cnt == nullptr || mass == nullptr) return BSA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(idx) || !aligned16(cnt) || !aligned16(mass) ||
        !aligned16(prob->key_table))
        return BSA_ERR_ALIGN;
    if (ws == nullptr || ws_bytes < mass_ws_bytes(g)) return BSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return BSA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t rows = (size_t)g.heads * g.N;
    uint8_t* w = static_cast<uint8_t*>(ws);
    bsa_bf16* o_scratch = reinterpret_cast<bsa_bf16*>(w + attention_ws_bytes(g));
    float* lse_kept = reinterpret_cast<float*>(w + attention_ws_bytes(g) + align256(rows * g.d * 2));
    float* lse_all = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(lse_kept) + align256(rows * sizeof(float)));
    // the log-sum-exp over the kept keys, then over every key; the outputs themselves are not
    // needed, so K stands in for V
    attn::Params P = attention_params(g, Q, K, K, idx, cnt, o_scratch, lse_kept, ws, prob->key_table);
    if ((rc = run_attention(P, st)) != BSA_OK) return rc;
    P = attention_params(g, Q, K, K, nullptr, nullptr, o_scratch, lse_all, ws, prob->key_table);
    if ((rc = run_attention(P, st)) != BSA_OK) return rc;
    mass_kernel<<<dim3(g.nb, g.heads), kMassThreads, 0, st>>>(g, P.perm, lse_kept, lse_all, mass);
    return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Drift check without a caller workspace.
//
// Some callers cannot allocate device memory when they call in: inference servers and
// real-time pipelines that reserve all device memory at start-up and forbid allocation
// afterwards, and plugin interfaces that hand a kernel only its input and output buffers
// with no way to ask for scratch space. bsa_drift_check_noalloc serves them: its float64
// partial sums live in the library's own static device array below instead of a caller
// workspace. That array exists once per device that loads the library and stays until the
// process exits; every call on a device shares it.
namespace {

constexpr size_t kNoallocDriftDoubles = 262144;   // 2 MiB: heads * chunks * 4 doubles
static __device__ __align__(256) double g_noalloc_drift_scratch[kNoallocDriftDoubles];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
double* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the static scratch on the current device, looked up once per device.
// The name g_noalloc_drift_scratch is only a host-side stand-in; kernels must get this
// address instead.
int noalloc_scratch(double** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_drift_scratch) != cudaSuccess) return BSA_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<double*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return BSA_OK;
}

}  // namespace

extern "C" {

int bsa_drift_check_noalloc(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                            bsa_bf16* Q_ref, bsa_bf16* K_ref, float tau, int force_all, float* drift,
                            int* refresh, bsa_stream_t stream) {
    Geom g;
    const int rc = make_geom(prob, &g);
    if (rc != BSA_OK) return rc;
    const size_t need = (size_t)g.heads * drift_chunks(g) * 4;
    if (need > kNoallocDriftDoubles) return BSA_ERR_SCRATCH_LIMIT;
    double* scratch = nullptr;
    const int sc = noalloc_scratch(&scratch);
    if (sc != BSA_OK) return sc;
    // every partial that the finalize pass reads is written first by the partial pass of
    // the same call, so the shared array needs no clearing between calls; the block means of a
    // fused pass are not written by this entry point (its scratch holds only the partials)
    bsa_problem p = *prob;
    p.block_means = nullptr;
    return bsa_drift_check(&p, Q, K, Q_ref, K_ref, tau, force_all, drift, refresh, scratch,
                           kNoallocDriftDoubles * sizeof(double), stream);
}

int bsa_device_status(bsa_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return BSA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
    }
    return word;
}

const char* bsa_error_string(int status) {
    switch (status) {
        case BSA_OK: return "ok";
        case BSA_ERR_ARG: return "invalid argument";
        case BSA_ERR_UNSUPPORTED: return "unsupported size (d and block must be 64 or 128; at most 2048 blocks)";
        case BSA_ERR_ALIGN: return "pointer not 16-byte aligned";
        case BSA_ERR_WORKSPACE: return "workspace missing or too small";
        case BSA_ERR_CUDA: return "CUDA launch or runtime error";
        case BSA_ERR_TIMEOUT: return "device: a bounded wait in a kernel ran out";
        case BSA_ERR_DEVICE_ARG: return "device: kept-block index or count out of range";
        case BSA_ERR_SCRATCH_LIMIT:
            return "problem too large for the static scratch of bsa_drift_check_noalloc "
                   "(needs heads * ceil(tokens * d / 16384) <= 65536)";
        default: return "unknown status";
    }
}

const char* bsa_version(void) { return "bsa 0.3.0 sm_100a"; }

int bsa_set_park_kernel(int which) {
    if (which != BSA_PARK_AUTO && which != BSA_PARK_TWO_PASS) return BSA_ERR_ARG;
    g_park_two_pass.store(which == BSA_PARK_TWO_PASS ? 1 : 0);
    return BSA_OK;
}

unsigned long long bsa_launch_count(void) { return g_launch_count.load(std::memory_order_relaxed); }

#ifdef BSA_TEST_HOOKS
// Test builds only: makes the next attention launches take their timeout path (see
// attn::g_test_withhold_q). Not declared in bsa.h and not in the product library.
int bsa_test_withhold_q_arrival(int on) {
    return cudaMemcpyToSymbol(attn::g_test_withhold_q, &on, sizeof(int)) == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}
#endif

}  // extern "C"
