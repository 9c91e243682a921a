/*
 * sbsa.h -- block-sparse attention prefill on NVIDIA B200 (sm_100a).
 *
 * A C ABI over four device stages: pool key/query blocks, select a block
 * list per query block, attend over the listed blocks, and the whole
 * prefill.  All tensor arguments are DEVICE pointers owned by the caller;
 * the library never allocates, frees or retains memory between calls.
 * Every call is asynchronous on the caller's stream (a cudaStream_t passed
 * as `void*`; NULL means the legacy default stream) and returns a status
 * code.  Argument errors are detected on the host before any launch; in
 * that case nothing is enqueued.  Errors detected by a kernel (a bounded
 * wait that expired, an index out of range) are recorded in a per-device
 * status word read by sbsa_get_status().
 *
 * Sources of the operations (web pages, by title and section):
 *   [RBS]  "RBS-Attention: un metodo de prefill disperso para modelos de
 *          lenguaje con contexto largo" (iaonda.com), method paragraph: key
 *          blocks summarised by a centroid and a dynamic radius; a base
 *          branch (centroid relevance) and a rescue branch (blocks at risk
 *          of being underestimated) each with an independent threshold;
 *          masks united; sparse-FlashAttention-compatible prefill.
 *   [UGS]  "Uncertainty-gated selection for block-sparse attention"
 *          (gist.science, paper 2607.07724), technical summary,
 *          Metodologia steps 1-5: mean-pooled block scores, per-query-tile
 *          top-k lists kv_idx, expansion to 2k where the top-k cut is
 *          ambiguous, sentinel padding for uniform dispatch shapes.
 *   [MSA]  "MiniMax presenta MSA ..." (iaonda.com), "Que es MSA y como
 *          funciona?": one top-k selection per GQA group from a light index
 *          branch; full attention over the preselected blocks only.
 *
 * Layout (all tensors contiguous, batch 1, one layer):
 *   Q  [Hq,  N, d]      K, V [Hkv, N, d]      O [Hq, N, d]
 *   Q_idx [Hq, N, d_idx], K_idx [Hkv, N, d_idx]   (optional index tensors)
 * Element type of Q/K/V/O and of the index tensors: p->dtype.
 * Query head h reads kv head h / (Hq/Hkv).  Token t belongs to block t / B;
 * NB = ceil(N / B) and the last block may be partial.
 */
#ifndef SBSA_H_
#define SBSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define SBSA_OK 0
#define SBSA_ERR_INVALID_ARG 1 /* null pointer, inconsistent shape or option  */
#define SBSA_ERR_UNSUPPORTED 2 /* valid but not built: d, B, d_idx, dtype, or
                                  NB beyond what one CTA's shared memory holds:
                                  the selection keeps two score rows (NB <= 23424
                                  at d_s = 128, <= 15616 with the rescue branch), the row-max
                                  scores a tile's running maxima (NB <= 16897 at
                                  d_s = 128), the percentile gate NB doubles   */
#define SBSA_ERR_WORKSPACE 3   /* workspace too small or misaligned           */
#define SBSA_ERR_CUDA 4        /* a CUDA runtime/driver call failed           */
#define SBSA_ERR_TIMEOUT 5     /* a kernel's bounded wait expired             */
#define SBSA_ERR_DEVICE 6      /* a kernel met an out-of-range list entry     */

/* ---- element types ---- */
#define SBSA_BF16 0 /* bfloat16 storage, bf16 tensor-core products, fp32 accumulate */
#define SBSA_FP32 1 /* fp32 storage, tf32 tensor-core products, fp32 accumulate     */

/* ---- base-branch selection rules ---- */
#define SBSA_TOPK 0    /* [UGS] step 2: the top_k best-scoring past blocks           */
#define SBSA_CUMMASS 1 /* [RBS] base branch: shortest score-ranked prefix whose
                          softmax mass over the candidates reaches mass_threshold */

/* ---- block-scoring backbones ([UGS] Metodologia step 1, Componibilidad) ---- */
#define SBSA_BACKBONE_MEAN 0   /* centroid: s_j = q . c_j (SSA-style K-mean)          */
#define SBSA_BACKBONE_MINMAX 1 /* per-coordinate upper bound from the block's K-min /
                                  K-max: s_j = sum_d max(q_d min_jd, q_d max_jd),
                                  the largest q.k over the block's coordinate box
                                  (Quest-style K-max)                               */

typedef struct sbsa_params {
  int n_q_heads;        /* Hq >= 1                                             */
  int n_kv_heads;       /* Hkv >= 1, divides Hq (GQA group G = Hq/Hkv)         */
  int seq_len;          /* N >= 1                                              */
  int head_dim;         /* d in {64, 128}                                      */
  int block_size;       /* B in {64, 128}; query tile = key block = B tokens   */
  int dtype;            /* SBSA_BF16 | SBSA_FP32 (fp32 attention: d = 64 only) */
  int select_mode;      /* SBSA_TOPK | SBSA_CUMMASS                            */
  int group_shared;     /* 0: one list per query head; 1: one per GQA group    */
  int index_dim;        /* 0: score on Q/K; else d_idx in {64,128} of Q_idx/K_idx */
  int top_k;            /* TOPK budget k >= 1                                  */
  float mass_threshold; /* CUMMASS threshold in (0, 1]                         */
  int rescue;           /* 1: unite with the rescue branch (needs radii)       */
  float rescue_tau;     /* rescue keeps j when (q.c_j + |q| r_j)*score_scale > tau */
  int gate;             /* TOPK only. 0: none; SBSA_GATE_GAP: a row takes 2k when
                           s_(k) - s_(k+1) < gate_margin * std(s);
                           SBSA_GATE_PERCENTILE: the page's gate, see below    */
  float gate_margin;    /* SBSA_GATE_GAP margin                                */
  int max_blocks;       /* list width Kmax; must hold the widest possible list:
                           TOPK min(k,NB-1)+1, gated min(2k,NB-1)+1,
                           CUMMASS or rescue NB                                */
  float sm_scale;       /* attention logit scale; 0 => 1/sqrt(head_dim)       */
  float score_scale;    /* block-score scale;     0 => 1/sqrt(score dim)      */
  int backbone;         /* SBSA_BACKBONE_MEAN | SBSA_BACKBONE_MINMAX; MINMAX
                           excludes the rescue branch (which needs radii)    */
  float gate_quantile;  /* SBSA_GATE_PERCENTILE: q in [0, 1]                  */
  int gate_rho;         /* SBSA_GATE_PERCENTILE: fired tiles take rho*k, rho >= 1 */
  int tile_score;       /* SBSA_TILE_MEAN | SBSA_TILE_ROWMAX; ROWMAX needs the
                           mean backbone, bf16 inputs and no rescue branch   */
} sbsa_params;

/* ---- query side of a tile score ([UGS] Metodologia step 2) ---- */
#define SBSA_TILE_MEAN 0   /* the pooled (mean) query of the tile: one dot per block     */
#define SBSA_TILE_ROWMAX 1 /* the page's tile score: the largest q_t . c_j over the
                              tile's query rows (and, per GQA group, the group's heads),
                              a tensor-core contraction with exact products (each fp32
                              centroid split exactly into three bf16 parts) */

/* ---- gates ([UGS] Metodologia steps 3-5) ---- */
#define SBSA_GATE_GAP 1        /* per row: gap at the cut below margin * std -> 2k   */
#define SBSA_GATE_PERCENTILE 2 /* the page's gate: per row with more than k
     candidates, sigma = (s_(k-1) - s_(k)) / (s_(0) - s_(k)) on the descending
     0-based order (0 when s_(0) = s_(k)); per query tile, the mean of sigma over
     the selection heads; the floor(q T) of the T eligible tiles with the
     smallest mean (lower tile first on equal means) fire and take the top
     rho*k in every head; max_blocks must hold min(rho*k, NB-1)+1.  Needs a
     workspace (sbsa_select_ws or sbsa_prefill). */

/*
 * sbsa_pool_blocks -- [RBS] centroid and radius of each block; [UGS] step 1
 * mean pooling; [MSA] group-level pooled queries.
 *   x         device [n_heads, N, dim], element type p->dtype.
 *   group     consecutive heads averaged into one output head (1 = none);
 *             must divide n_heads.
 *   centroids device fp32 [n_heads/group, NB, dim]:
 *             mean over the group's heads of each head's mean over the rows
 *             of block j (rows t with t/B == j, t < N).
 *   radii     device fp32 [n_heads, NB] or NULL: max_t |x_t - c_j|_2 over the
 *             block's rows (group must be 1 when radii is given).
 * Uses N and B from p; dim in {64, 128}.  Reads x once.
 */
int sbsa_pool_blocks(const sbsa_params* p, const void* x, int n_heads, int dim, int group,
                     float* centroids, float* radii, void* stream);

/*
 * sbsa_pool_minmax -- [UGS] step 1 with the K-min / K-max backbone.
 *   x       device [n_heads, N, dim], element type p->dtype.
 *   minmax  device fp32 [n_heads, NB, 2, dim]: for block j, the coordinate-wise
 *           minimum over the block's rows (t/B == j, t < N), then the maximum.
 * Uses N and B from p; dim in {64, 128}.  Reads x once; exact (no rounding).
 * Errors: SBSA_ERR_INVALID_ARG for null or misaligned pointers or n_heads < 1,
 * SBSA_ERR_UNSUPPORTED for other dim or B; SBSA_ERR_CUDA on a launch failure.
 * The pages have the backbone only by name; the table layout is this library's.
 */
int sbsa_pool_minmax(const sbsa_params* p, const void* x, int n_heads, int dim, float* minmax,
                     void* stream);

/*
 * sbsa_select -- [UGS] steps 1-5 on pooled tables; [RBS] base and rescue
 * branches with their union; [MSA] group-shared lists.
 *   q_cent   device fp32 [Hs, NB, ds]  pooled queries, Hs = group_shared ? Hkv : Hq
 *   k_cent   device fp32 [Hkv, NB, ds] key centroids
 *   k_radius device fp32 [Hkv, NB] (required when p->rescue, else ignored)
 *   idx      device int32 [Hs, NB, max_blocks] out: ascending block ids, then -1
 *   cnt      device int32 [Hs, NB] out: number of valid ids per row
 *   flags    device uint8 [Hs, NB] out or NULL: bit0 gate fired, bit1 rescue
 *            added a block the base branch missed
 * ds = index_dim if set, else head_dim.  Selection head hs scores against kv
 * head (group_shared ? hs : hs / G).  Candidates of query block i are the
 * blocks j < i with score s_j = (q_cent[hs,i] . k_cent[g,j]) * score_scale,
 * ranked by score descending, lower id first on equal scores.  The diagonal
 * block i is always appended.
 */
int sbsa_select(const sbsa_params* p, const float* q_cent, const float* k_cent,
                const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags, void* stream);
/* With p->backbone == SBSA_BACKBONE_MINMAX, k_cent is the [Hkv, NB, 2, ds]
 * table of sbsa_pool_minmax and s_j = sum_d max(q_d min_jd, q_d max_jd) *
 * score_scale; everything else is unchanged.  With p->gate ==
 * SBSA_GATE_PERCENTILE sbsa_select returns SBSA_ERR_WORKSPACE: use
 * sbsa_select_ws. */

/*
 * sbsa_score_centroids -- [UGS] step 1 / [RBS] base branch scores as one
 * dense product on the tensor cores (mean backbone, mean tile scores).
 *   q_cent   device fp32 [Hs, NB, ds] pooled queries (sbsa_pool_blocks).
 *   k_cent   device fp32 [Hkv, NB, ds] key centroids.
 *   scores   device fp32 [Hs, NB, NB] out: scores[hs, i, j] for j < i is
 *            (q_cent[hs,i] . k_cent[g,j]) * score_scale, g as in sbsa_select;
 *            entries j >= i are not written.
 *   workspace device, 256-byte aligned, >= sbsa_score_centroids_workspace_bytes(p)
 *            (tf32 hi / lo parts of both tables).
 * Each product is taken as three tf32 products of the split operands
 * (x = hi + lo), within a few fp32 roundings of the exact dot product; the
 * summation order is the tensor core's.
 * Errors as sbsa_select, plus SBSA_ERR_UNSUPPORTED unless p->backbone is
 * SBSA_BACKBONE_MEAN and p->tile_score is SBSA_TILE_MEAN, and
 * SBSA_ERR_WORKSPACE for a missing, misaligned or short workspace.
 */
size_t sbsa_score_centroids_workspace_bytes(const sbsa_params* p);
int sbsa_score_centroids(const sbsa_params* p, const float* q_cent, const float* k_cent,
                         float* scores, void* workspace, size_t ws_bytes, void* stream);

/*
 * sbsa_score_rowmax -- the page's tile scores (SBSA_TILE_ROWMAX).
 *   q_src    device [Hq, N, ds] bf16: Q, or Q_idx when p->index_dim is set.
 *   k_cent   device fp32 [Hkv, NB, ds] key centroids (sbsa_pool_blocks).
 *   scores   device fp32 [Hs, NB, NB] out: scores[hs, i, j] for j < i is
 *            max_t (q_t . c_j) * score_scale over the query rows t of
 *            block i (rows t < N) of head hs, or of every head of group hs
 *            when p->group_shared; entries j >= i are not written.
 *   workspace device, 256-byte aligned, >= sbsa_score_rowmax_workspace_bytes(p)
 *            (the centroids split exactly into three bf16 parts).
 * The products are exact (bf16 rows times the exact bf16 parts of each fp32
 * centroid); the only rounding is the tensor core's fp32 accumulation.
 * Errors as sbsa_select, plus SBSA_ERR_UNSUPPORTED when p->tile_score is not
 * SBSA_TILE_ROWMAX.
 */
size_t sbsa_score_rowmax_workspace_bytes(const sbsa_params* p);
int sbsa_score_rowmax(const sbsa_params* p, const void* q_src, const float* k_cent,
                      float* scores, void* workspace, size_t ws_bytes, void* stream);

/*
 * sbsa_select_scores -- the selection on a precomputed score table
 * [Hs, NB, NB] (sbsa_score_rowmax or sbsa_score_centroids; row i holds the
 * scores of candidates j < i, the rest is not read) instead of pooled
 * tables; every rule (top-k, the gates, cumulative mass, the diagonal)
 * applies unchanged.  Outputs as sbsa_select.
 *   workspace  used only by the percentile gate (its per-row margins and
 *              per-tile decisions); a workspace of sbsa_select_workspace_bytes(p)
 *              bytes, 256-byte aligned, always suffices.
 * Errors as sbsa_select; SBSA_ERR_INVALID_ARG with p->rescue (the rescue bound
 * needs the pooled tables); SBSA_ERR_WORKSPACE for a missing or short
 * workspace under the percentile gate.
 */
int sbsa_select_scores(const sbsa_params* p, const float* scores, int32_t* idx, int32_t* cnt,
                       uint8_t* flags, void* workspace, size_t ws_bytes, void* stream);

/* Device workspace sbsa_select_ws needs: the percentile gate's scratch,
 * and with the mean backbone and mean tile scores the score table and the
 * scratch of sbsa_score_centroids.  0 when neither applies or p is invalid. */
size_t sbsa_select_workspace_bytes(const sbsa_params* p);

/*
 * sbsa_select_ws -- sbsa_select with a caller workspace (256-byte aligned,
 * ws_bytes >= sbsa_select_workspace_bytes(p)) for the percentile gate's
 * per-row margins and per-tile decisions: three launches (top-k lists and
 * margins; the tile decisions; top-rho*k lists of the fired tiles).  The
 * pages have no entry point; the gate is theirs.  With the mean backbone and
 * mean tile scores the scores come from sbsa_score_centroids into the
 * workspace (tensor cores) instead of fp32 FMA inside the selection kernel,
 * as they do in sbsa_prefill; sbsa_select keeps the FMA form.
 */
int sbsa_select_ws(const sbsa_params* p, const float* q_cent, const float* k_cent,
                   const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags,
                   void* workspace, size_t ws_bytes, void* stream);

/*
 * sbsa_select_gate_partial / sbsa_select_gate_finish -- sbsa_select_ws under
 * the percentile gate ([UGS] Metodologia steps 3-5), split in two so that the
 * selection heads may be spread over several processes (one sequence sharded
 * by kv head).  The gate is the only rule that couples heads: a tile's
 * decision uses the mean of its cut margins over ALL selection heads.  The
 * pages have no entry point for this; the split is this library's.
 *   partial: centroid scores (tensor cores) into the workspace, top-k lists and
 *            per-row margins of this call's heads, then
 *            tile_sums[i] = sum over this call's heads (head order, double) of
 *            the margin of tile i (NaN for tiles with at most k candidates).
 *   The caller sums tile_sums over the processes (an all-reduce), then
 *   finish:  mean margin = tile_sums / total_heads, the floor(q T) smallest of
 *            the T tiles with more than k candidates fire, and the rows of the
 *            fired tiles are redone with top rho*k.
 *   Both calls take the same arguments as sbsa_select_ws and the SAME
 *   workspace (finish reads the scores and margins partial left in it).
 *   tile_sums    device double [NB], 8-byte aligned.
 *   total_heads  selection heads over all processes (>= this call's Hs).
 * With total_heads = Hs and tile_sums untouched between the calls the result
 * is that of sbsa_select_ws.  Errors as sbsa_select_ws; SBSA_ERR_INVALID_ARG
 * unless p->gate is SBSA_GATE_PERCENTILE with mean tile scores, for a missing
 * or misaligned tile_sums, or total_heads < Hs.
 */
int sbsa_select_gate_partial(const sbsa_params* p, const float* q_cent, const float* k_cent,
                             const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags,
                             void* workspace, size_t ws_bytes, double* tile_sums, void* stream);
int sbsa_select_gate_finish(const sbsa_params* p, const float* q_cent, const float* k_cent,
                            const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags,
                            void* workspace, size_t ws_bytes, const double* tile_sums,
                            int total_heads, void* stream);

/*
 * sbsa_attend -- [RBS] sparse prefill attention; [MSA] main branch.
 *   q [Hq,N,d], k/v [Hkv,N,d], o [Hq,N,d]: device, element type p->dtype.
 *   idx/cnt: lists as produced by sbsa_select (Hs rows per p->group_shared).
 * O[h,t] = sum over u in the listed blocks of (h, t/B) with u <= t of
 * softmax_u(Q[h,t].K[g,u] * sm_scale) V[g,u]; rows that see no key are 0.
 * List entries outside [0, i] are skipped and reported as SBSA_ERR_DEVICE
 * through sbsa_get_status; a repeated entry is attended twice.
 */
int sbsa_attend(const sbsa_params* p, const void* q, const void* k, const void* v,
                const int32_t* idx, const int32_t* cnt, void* o, void* stream);

/* Bytes of device workspace sbsa_prefill needs for these parameters
 * (pooled tables; the score table with its scratch for the mean backbone
 * and for row-max tile scores; the percentile gate's scratch; plus lists when
 * the caller does not provide them).  Returns 0 when p is invalid. */
size_t sbsa_prefill_workspace_bytes(const sbsa_params* p);

/*
 * sbsa_prefill -- pool (keys and queries), select, attend, on one stream.
 *   q_idx/k_idx: index tensors when p->index_dim != 0 (else NULL).
 *   workspace:   device, 256-byte aligned, ws_bytes >= sbsa_prefill_workspace_bytes(p).
 *   idx_out/cnt_out/flags_out: optional device outputs (layout of sbsa_select);
 *   when NULL the lists live in the workspace.
 */
int sbsa_prefill(const sbsa_params* p, const void* q, const void* k, const void* v,
                 const void* q_idx, const void* k_idx, void* o, void* workspace,
                 size_t ws_bytes, int32_t* idx_out, int32_t* cnt_out, uint8_t* flags_out,
                 void* stream);

/*
 * sbsa_prefill_host -- sbsa_prefill from and to HOST memory.  The pages have
 * no such call; it is the end-to-end form of the prefill for a caller whose
 * tensors live on the host.
 *   q, k, v, q_idx, k_idx: host, layouts as in sbsa_prefill (page-locked
 *                memory lets the copies overlap the computation; pageable
 *                memory is correct but the copies then wait for the host).
 *   o:           host [Hq, N, d] out, written when the call's work on
 *                `stream` completes.
 *   workspace:   device, 256-byte aligned, ws_bytes >=
 *                sbsa_prefill_host_workspace_bytes(p): two staging sets of one
 *                chunk's inputs and output, and the chunk prefill's workspace.
 * The request is cut into chunks of kv heads (each kv head with the query
 * heads that read it; one chunk under the percentile gate, which averages
 * over every head): chunk c + 1 is copied in while chunk c is prefilled on
 * `stream` and chunk c - 1 is copied out.  The copies run on two streams of
 * the library's own per device, created on the first call (make that call
 * before any stream capture), ordered after the work already on `stream`;
 * everything the call enqueues is complete once `stream` reaches its end.
 * Calls that overlap on one device share those copy streams and run in turn.
 * Lists are not returned (they stay in the workspace).  Errors as
 * sbsa_prefill.
 */
size_t sbsa_prefill_host_workspace_bytes(const sbsa_params* p);
int sbsa_prefill_host(const sbsa_params* p, const void* q, const void* k, const void* v,
                      const void* q_idx, const void* k_idx, void* o, void* workspace,
                      size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the current device's status
 * word into *device_status (SBSA_OK when no kernel reported an error).
 * Returns SBSA_ERR_CUDA when the synchronisation itself failed. */
int sbsa_get_status(void* stream, int* device_status);

/* Static description of a status code. */
const char* sbsa_status_string(int code);

/* Library ABI version (major * 100 + minor). */
int sbsa_version(void);

/*
 * sbsa_debug_wait_timeout -- test hook for the failure path of the bounded
 * device waits used by the kernels (no counterpart on the pages).  Launches
 * one CTA that waits on an mbarrier nothing ever arrives on, using the same
 * bounded-wait primitive as the attention pipeline with a limit of
 * `timeout_ns` nanoseconds (clamped to [1 us, 10 s]); when the limit expires
 * the kernel records SBSA_ERR_TIMEOUT in the device status word and returns.
 * No copy or MMA is in flight, so the context stays usable.  Read the result
 * with sbsa_get_status().
 */
int sbsa_debug_wait_timeout(uint64_t timeout_ns, void* stream);

/*
 * sbsa_exp2_fma_eval -- test hook for the exponential that the persistent
 * 128-token attention kernel can take on the FMA pipe for one score in four
 * (the option SBSA_ATTEND_EXP2=fma in the environment; the default keeps
 * every exponential on the MUFU).  [RBS] method paragraph: the prefill's
 * softmax.  Writes y[e] = exp2_fma(x[e]) for e < n: Cody-Waite reduction
 * x = n + f, f in [-1/2, 1/2], and a degree-3 minimax polynomial for 2^f,
 * relative error below 7.5e-5 for x in [-125, 8], exactly 0 below -125.
 *   x, y  device fp32 [n]; may not overlap unless equal.
 *   n     elements; 0 enqueues nothing.
 * Returns SBSA_ERR_INVALID_ARG for n < 0 or a NULL pointer with n > 0.
 */
int sbsa_exp2_fma_eval(const float* x, float* y, int64_t n, void* stream);

/*
 * sbsa_prefill_noalloc -- sbsa_prefill for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is a deployment
 * convenience of this library.
 *
 * Some callers have no way to supply a workspace: a plugin inside a host
 * framework that owns all device memory and gives its operators no
 * allocator, a latency-critical path where cudaMalloc's implicit device
 * synchronisation is not acceptable, or a process whose device memory
 * budget is fixed at start-up.  This entry point takes the same inputs and
 * outputs as sbsa_prefill minus the workspace; its temporaries (those of
 * sbsa_prefill_workspace_bytes: pooled tables, score table and scratch and,
 * when idx_out/cnt_out are NULL, the block lists) live in one
 * fixed array of SBSA_NOALLOC_SCRATCH_BYTES compiled into the library.  It
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *
 *  - Limit: problems whose temporaries exceed SBSA_NOALLOC_SCRATCH_BYTES are
 *    rejected with SBSA_ERR_WORKSPACE before anything is launched (pass
 *    idx_out/cnt_out to keep the lists out of the scratch).
 *  - Memory: every GPU that loads the library holds the array (32 MiB) until
 *    the process exits.
 *  - Set-up: the first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Sharing: all calls on a device use the same array and it keeps the last
 *    call's contents.  Nothing in it needs to start at zero (every byte a
 *    call reads is written earlier by the same call), but calls whose kernels
 *    overlap on the GPU (different streams without ordering) race on it:
 *    serialise them.
 * Arguments, layouts and errors otherwise as sbsa_prefill.
 */
#define SBSA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int sbsa_prefill_noalloc(const sbsa_params* p, const void* q, const void* k, const void* v,
                         const void* q_idx, const void* k_idx, void* o, int32_t* idx_out,
                         int32_t* cnt_out, uint8_t* flags_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SBSA_H_ */
