/*
 * bsa.h — C ABI of libbsa: training-free block-sparse 3D attention for video diffusion
 * transformers on NVIDIA B200 (sm_100a).
 *
 * One attention layer's hot path, per denoising step:
 *   bsa_drift_check      per-head query/key drift against the cached reference; decides
 *                        which heads refresh their mask (HEART: Exploiting Head
 *                        Heterogeneity in Sparse Attention for Video Diffusion, abstract,
 *                        "Temporal Mask Reuse"; HASTE, abstract)
 *   bsa_score_blocks     query-block x key-block importance, mean-pooled or per-query
 *                        normalised (PARK: Accurate Block Retrieval for Sparse Attention in
 *                        Video Diffusion Transformers, Abstract)
 *   bsa_select_topp      per-head top-p kept-block lists (HASTE: Training-Free Video
 *                        Diffusion Acceleration via Head-Wise Adaptive Sparse Attention,
 *                        abstract)
 *   bsa_sparse_attention softmax attention over the kept key blocks only (PARK, Abstract:
 *                        attention computed only within the retrieved blocks)
 *
 * Conventions shared by every call
 *   - Tensors Q, K, V, O are bfloat16 (raw 16-bit patterns, bsa_bf16), row-major
 *     [heads, tokens, d] in RASTER order of the 3D grid (t slowest, x fastest), video tokens
 *     first, then `text_tokens` text tokens. The library never permutes them in memory: the
 *     kernels gather rows in block order on the fly.
 *   - Block order: the video grid is cut into tiles (tile_t x tile_h x tile_w) visited in
 *     raster order of tile coordinates; tokens inside a tile are in raster order and edge
 *     tiles are truncated. That concatenated order is cut into blocks of `block` tokens; only
 *     the last video block can be partial (its missing slots are padding, masked as keys and
 *     never written as queries). Text tokens follow as their own blocks (nb_text of them).
 *     nb = nb_video + nb_text blocks per head.
 *   - All pointers are DEVICE pointers to caller-owned memory, 16-byte aligned, unless a
 *     parameter says "host". The library allocates and frees nothing; scratch comes from the
 *     caller's workspace, sized by bsa_plan.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and returns a status code. Argument errors are detected on the host before anything is
 *     launched; nothing is written then. Device-side problems (a bounded wait that ran out, an
 *     out-of-range kept-block index) set a device error word read by bsa_device_status.
 *     The word is sticky: it keeps the FIRST problem's code until bsa_device_status reads and
 *     clears it, so read it after any sequence of calls whose results matter. No kernel reads
 *     the word: later calls run normally whether or not it is set. A bad kept-block index
 *     or count only spoils its own query block's output; a wait that ran out (about 2 s; a
 *     hang) ends that launch early, and every output of that call is then unspecified.
 *   - Thread safety: calls only read their arguments; concurrent calls on different streams
 *     are safe as long as their output buffers and workspaces do not overlap.
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t bsa_bf16;                 /* bfloat16 bit pattern */
typedef struct CUstream_st* bsa_stream_t;  /* identical to cudaStream_t */

/* status codes */
#define BSA_OK               0
#define BSA_ERR_ARG         -1   /* null pointer, bad size, inconsistent problem */
#define BSA_ERR_UNSUPPORTED -2   /* d or block outside the supported set */
#define BSA_ERR_ALIGN       -3   /* a pointer is not 16-byte aligned */
#define BSA_ERR_WORKSPACE   -4   /* workspace missing or smaller than bsa_plan asks */
#define BSA_ERR_CUDA        -5   /* a CUDA launch or runtime call failed */
#define BSA_ERR_TIMEOUT     -6   /* device: a bounded wait inside a kernel ran out */
#define BSA_ERR_DEVICE_ARG  -7   /* device: a kept-block index or count was out of range */
#define BSA_ERR_SCRATCH_LIMIT -8 /* problem exceeds the static scratch of bsa_drift_check_noalloc */

/* scorers (PARK, Abstract) */
#define BSA_SCORE_MEANPOOL   0   /* softmax_j( mean(Q in block i) . mean(K in block j) / sqrt(d) ) */
#define BSA_SCORE_PARK       1   /* mean over real q in block i of softmax_j( q . mean(K in block j) / sqrt(d) ) */

/* One attention layer. Plain struct, passed by pointer, read only. */
typedef struct bsa_problem {
    int heads;          /* >= 1 */
    int tokens;         /* must equal T*H*W + text_tokens */
    int d;              /* head dimension: 64 or 128 */
    int T, H, W;        /* 3D video grid, each >= 1 */
    int text_tokens;    /* >= 0, appended after the video tokens */
    int block;          /* tokens per block: 64 or 128 */
    int tile_t, tile_h, tile_w;  /* tile shape; all 0 = default (1x8x8 for 64, 2x8x8 for 128);
                                    otherwise tile_t*tile_h*tile_w must equal block */
    int score_mode;     /* BSA_SCORE_MEANPOOL or BSA_SCORE_PARK */
    const int* key_table;   /* DEVICE pointer, nullable: per-head key-side block-slot table
                               [heads][nb*block] written by bsa_cluster_keys (query-aware key
                               blocks). When set, bsa_score_blocks pools keys and
                               bsa_sparse_attention / bsa_captured_mass gather keys and values
                               through it; queries always use the tile layout. NULL: keys use
                               the tile layout too. Entries outside [-1, tokens) are clamped
                               into range (a wrong table gives wrong results, never a fault). */
    float* block_means;     /* DEVICE pointer, nullable: caller-owned [2][heads][nb][d] float32.
                               When set, bsa_drift_check reads Q, K, Q_ref, K_ref block by block
                               and also writes the block means of Q (first half) and K (second
                               half; through key_table when set) over each block's real tokens,
                               and bsa_score_blocks takes its means from there instead of reading
                               Q and K again: call them in that order on the same Q, K. NULL: each
                               call reads what it needs. */
} bsa_problem;

/* Derived sizes, filled by bsa_plan (host only, no CUDA call). */
typedef struct bsa_plan_info {
    int nb;             /* blocks per head = nb_video + nb_text */
    int nb_video;       /* ceil(T*H*W / block) */
    int nb_text;        /* ceil(text_tokens / block) */
    int npad;           /* nb * block */
    int tile_t, tile_h, tile_w;  /* tile actually used */
    size_t score_workspace_bytes;      /* bsa_score_blocks */
    size_t drift_workspace_bytes;      /* bsa_drift_check */
    size_t attention_workspace_bytes;  /* bsa_sparse_attention */
    size_t mass_workspace_bytes;       /* bsa_captured_mass */
    size_t cluster_workspace_bytes;    /* bsa_cluster_keys */
    int park_cluster;   /* PARK scorer under BSA_PARK_AUTO: CTAs per thread-block cluster of the
                           one-pass kernel (1..8), or 0 when nb needs the two-pass kernel */
    int park_cols;      /* key blocks each CTA of that cluster holds (0 with park_cluster 0) */
} bsa_plan_info;

/* Validate `prob` and fill `out`. Host only; launches nothing.
 * Returns BSA_OK, BSA_ERR_ARG or BSA_ERR_UNSUPPORTED. */
int bsa_plan(const bsa_problem* prob, bsa_plan_info* out);

/* Block layout on the host: perm_host[s] = raster token index held by block slot s, or -1
 * for a padding slot, for s in [0, plan.npad). Host memory, caller-owned, plan.npad ints.
 * Host only (the kernels compute the same map on the fly). Returns BSA_OK or BSA_ERR_ARG. */
int bsa_block_layout(const bsa_problem* prob, int* perm_host);

/* Block importance scores (PARK, Abstract: retrieval from averaged query/key block
 * representations, and PARK's per-query normalisation averaged within the query block).
 *   Q, K       [heads, tokens, d] bf16, raster order.
 *   head_mask  [heads] int, device, nullable. Heads with head_mask[h] == 0 are skipped and
 *              their rows of `scores` are left untouched (the cached-mask case).
 *   scores     [heads, nb, nb] float32 out. Row (h, i) is a probability distribution over
 *              key blocks j (including text blocks); logits are scaled by 1/sqrt(d).
 *   ws         workspace of at least plan.score_workspace_bytes: pooled block means, the
 *              block-slot table, the bf16 three-way splits of the pooled keys (and, for the
 *              mean-pooled mode, of the pooled queries and two log-sum-exps per score row). Its
 *              size depends on the mode, so plan with the mode that will run.
 * Mode is prob->score_mode. Mean-pooled scores are float32-grade: float32 dot products on
 * CUDA cores for problems too small to fill the GPU, otherwise tensor-core products of the
 * bf16 splits; both agree with exact arithmetic to float32 rounding. PARK scores are
 * float32-grade too, from one of two tensor-core kernels (bsa_set_park_kernel). */
int bsa_score_blocks(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                     const int* head_mask, float* scores,
                     void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Per-head top-p kept-block lists (HASTE, abstract: online top-p with per-head thresholds).
 * For each row (h, i): key blocks ordered by score descending, then index ascending; the
 * shortest prefix whose float32 cumulative score reaches p[h] (>=) is kept (at least one
 * block; p[h] >= 1 keeps all). Video query rows additionally keep every text key block; text
 * query rows keep every block. The kept list is written in that same order.
 *   scores     [heads, nb, nb] float32 (from bsa_score_blocks).
 *   p          [heads] float32, device.
 *   head_mask  [heads] int, device, nullable: heads with 0 are skipped (idx/cnt untouched).
 *   idx        [heads, nb, nb] int32 out: idx[h][i][0..cnt-1] are kept block indices;
 *              entries at and after cnt are not written.
 *   cnt        [heads, nb] int32 out, 1 <= cnt <= nb. */
int bsa_select_topp(const bsa_problem* prob, const float* scores, const float* p,
                    const int* head_mask, int* idx, int* cnt, bsa_stream_t stream);

/* Temporal mask reuse gate (HEART, abstract: refresh a head's cached mask only when its
 * query-key drift exceeds a prescribed threshold).
 *   drift[h]   = max(||Q_h - Qref_h||_F / ||Qref_h||_F, ||K_h - Kref_h||_F / ||Kref_h||_F)
 *                over all tokens of head h (0 when both norms are 0; +inf when only the
 *                reference norm is 0).
 *   refresh[h] = force_all || drift[h] > tau.
 * For every refreshed head the call then copies Q_h -> Q_ref_h and K_h -> K_ref_h (the new
 * reference), after the decision is made. Pass force_all = 1 on the first step, when there is
 * no reference yet (Q_ref/K_ref may then hold anything finite or not).
 *   Q, K           [heads, tokens, d] bf16, current step.
 *   Q_ref, K_ref   [heads, tokens, d] bf16, in/out reference snapshots.
 *   drift          [heads] float32 out;  refresh [heads] int32 out (0/1; usable as head_mask).
 *   ws             at least plan.drift_workspace_bytes. The reduction order is fixed, so the
 *                  result is deterministic. With prob->block_means set, the same pass also
 *                  writes the block means (see bsa_problem). */
int bsa_drift_check(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                    bsa_bf16* Q_ref, bsa_bf16* K_ref, float tau, int force_all,
                    float* drift, int* refresh,
                    void* ws, size_t ws_bytes, bsa_stream_t stream);

/* bsa_drift_check for callers that cannot allocate device memory. The paper has no
 * counterpart; this is a deployment convenience. Some callers cannot call cudaMalloc when
 * they call in: servers and real-time pipelines that reserve all device memory at start-up
 * and forbid allocation afterwards, and plugin interfaces that pass a kernel only its inputs
 * and outputs. This entry point takes no workspace and allocates nothing: its scratch is a
 * 2 MiB static device array inside the library (held on every device that loads the library
 * until the process exits).
 *   Arguments, results and determinism are those of bsa_drift_check; prob->block_means is
 *   ignored (the means are not written).
 *   Limit: heads * ceil(tokens * d / 16384) <= 65536; larger problems return
 *          BSA_ERR_SCRATCH_LIMIT and launch nothing.
 *   The first call on a device looks up the scratch address on that device (make that first
 *   call before any stream capture). All calls on a device share the one array: calls that
 *   may overlap on the GPU (different streams without ordering) race and must not be made. */
int bsa_drift_check_noalloc(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                            bsa_bf16* Q_ref, bsa_bf16* K_ref, float tau, int force_all,
                            float* drift, int* refresh, bsa_stream_t stream);

/* Block-sparse attention (PARK, Abstract: attention computed only within the retrieved
 * blocks). For every real query t of query block i of head h:
 *   O_t = sum over the real keys u of blocks idx[h][i][0..cnt[h][i]-1] of
 *         softmax_u(Q_t . K_u / sqrt(d)) V_u
 * bf16 inputs, float32 accumulation and softmax, bf16 output.
 *   Q, K, V    [heads, tokens, d] bf16, raster order.
 *   idx, cnt   as written by bsa_select_topp (any lists with 1 <= cnt <= nb and distinct
 *              indices in [0, nb) are accepted; a bad entry sets BSA_ERR_DEVICE_ARG in the
 *              device error word and the row's output is unspecified). Both NULL: every
 *              block is kept (dense attention, e.g. the steps before a one-shot estimate, or a
 *              dense refresh); only one NULL is BSA_ERR_ARG.
 *   O          [heads, tokens, d] bf16 out, raster order. Every real token is written.
 *   ws         at least plan.attention_workspace_bytes, always required: the block-slot ->
 *              token table, and the partial results of the dense text rows, which are split
 *              across CTAs and merged. */
int bsa_sparse_attention(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                         const bsa_bf16* V, const int* idx, const int* cnt, bsa_bf16* O,
                         void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Query-aware key blocks (PARK, Abstract: keys are transformed with information from the
 * current queries before clustering, so that keys receiving similar QK scores are grouped
 * together). Per head: M = Q^T Q / tokens over the real queries, so (k1-k2)^T M (k1-k2) is the
 * mean-square difference of the scores the queries give two keys; Lloyd's k-means with that
 * metric over the video keys, one cluster per video block, started from the tile-block means;
 * each of `iters` rounds assigns every key to argmin_j (k-c_j)^T M (k-c_j) (ties to the lowest
 * j) and, except in the last round, moves each non-empty cluster's centroid to the mean of
 * its keys. The table lists the video keys in (cluster, raster index) order followed by the
 * tile layout's padding and text slots: cut every `block` keys it gives key blocks of the same
 * sizes as the tile layout. Pass it as prob->key_table to the scoring and attention calls.
 *   Q, K        [heads, tokens, d] bf16, raster order.
 *   iters       1..64 rounds.
 *   key_table   [heads, nb*block] int32 out (raster token per slot, -1 = padding).
 *   assignment  [heads, T*H*W] int32 out, nullable: cluster of every video key (raster order)
 *               in the last round.
 *   ws          at least plan.cluster_workspace_bytes (M and its partial sums, centroids, the
 *               assignment and the sorted order). prob->key_table is ignored here.
 * Deterministic (fixed summation orders). Not a per-step call: it costs a pass over Q (M) and
 * heads x video keys x clusters x d multiply-adds per round. */
int bsa_cluster_keys(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K, int iters,
                     int* key_table, int* assignment, void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Cached dense correction of this step's sparse output (RECAP: Reciprocal Sparse Attention
 * and Hierarchical Caching for Efficient Video Diffusion, Abstract: a cached dense refinement
 * corrects the interactions the current sparse estimate omits, and fresh statistics of the
 * inputs regulate the aging correction). Call after bsa_sparse_attention of the same step,
 * with the refresh flags of bsa_drift_check (the fresh statistics):
 *   refresh[h] != 0: D = dense attention of head h (every key block); R_h = D - O_h (the new
 *                    correction); O_h = D.
 *   refresh[h] == 0: O_h = O_h + R_h (the sparse output plus the head's cached correction).
 * bf16 in and out, float32 arithmetic.
 *   Q, K, V    [heads, tokens, d] bf16, raster order (this step's).
 *   refresh    [heads] int, device (from bsa_drift_check; all 1 on the first step).
 *   O          [heads, tokens, d] bf16 in/out: this step's sparse output in, corrected out.
 *   R          [heads, tokens, d] bf16 in/out: the cached corrections, caller-owned across
 *              steps; its contents only matter for heads that are not refreshed.
 *   ws         at least plan.attention_workspace_bytes. */
int bsa_dense_correction(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                         const bsa_bf16* V, const int* refresh, bsa_bf16* O, bsa_bf16* R,
                         void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Retrieval accuracy of a set of kept-block lists (PARK, Abstract: inaccurate block
 * retrieval either degrades quality or wastes computation; retrieval is judged by its
 * accuracy). For every real query t of query block i of head h, the captured mass is the
 * share of t's exact attention softmax over ALL real keys that falls on the real keys of the
 * kept blocks idx[h][i][0..cnt[h][i]-1]; mass[h][i] is its mean over the block's real
 * queries (1 when every block is kept). A measurement, not a step of the hot path: it runs
 * the attention kernel twice (kept blocks, then every block) for the two log-sum-exps of
 * each query and takes 2^(difference), so it costs one dense attention pass.
 *   Q, K       [heads, tokens, d] bf16, raster order.
 *   idx, cnt   kept lists as bsa_select_topp writes them (same checks as bsa_sparse_attention).
 *   mass       [heads, nb] float32 out.
 *   ws         at least plan.mass_workspace_bytes: the attention workspace, an output scratch
 *              [heads, tokens, d] bf16 and two [heads, tokens] float32 log-sum-exps. */
int bsa_captured_mass(const bsa_problem* prob, const bsa_bf16* Q, const bsa_bf16* K,
                      const int* idx, const int* cnt, float* mass,
                      void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word of the current device.
 * Returns BSA_OK, BSA_ERR_TIMEOUT, BSA_ERR_DEVICE_ARG or BSA_ERR_CUDA. */
int bsa_device_status(bsa_stream_t stream);

/* Static description of a status code (never NULL). */
const char* bsa_error_string(int status);

/* Which kernel bsa_score_blocks runs in PARK mode (process-wide host setting, no CUDA call;
 * takes effect at the next call):
 *   BSA_PARK_AUTO      one pass, each item's logits held in tensor memory, the key blocks of
 *                      a head split over a thread-block cluster of up to 8 CTAs (nb up to
 *                      1280); larger nb, or a device that cannot place the cluster, falls
 *                      back to the two-pass kernel. The default.
 *   BSA_PARK_TWO_PASS  always the two-pass kernel (64-block tiles, logits computed twice).
 * Both give the same scores to float32 rounding. Returns BSA_OK or BSA_ERR_ARG. */
#define BSA_PARK_AUTO     0
#define BSA_PARK_TWO_PASS 1
int bsa_set_park_kernel(int which);

/* Library version, e.g. "bsa 0.3.0 sm_100a". */
const char* bsa_version(void);

/* Number of kernels this library has launched in this process so far (all devices, all
 * streams; host counter, no CUDA call). A caller that wants the launches of a stretch of
 * calls takes the difference of two readings. */
unsigned long long bsa_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H */
