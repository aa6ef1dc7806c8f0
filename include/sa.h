/*
 * sa.h - dynamic tile-sparse global attention for feed-forward 3-D
 * reconstruction transformers, on B200 (sm_100a).
 *
 * The operation.  In VGGT-style backbones a "global" attention layer lets
 * every query token of each of S frames attend to all S*N tokens, which costs
 * O((S*N)^2) ("AVGGT: Rethinking Global Attention for Accelerating VGGT",
 * technical summary, section 1; "(Full) Attention is More Than You Need",
 * full vs sparse global attention).  The sparse layer keeps only the most
 * promising interactions, chosen per input and per head ("SAF3R: Dynamic
 * Sparse Attention for Feed-Forward 3D Reconstruction Transformers",
 * abstract), at tile granularity with landmark summaries of the rest
 * ("Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D
 * Reconstruction", abstract).  The path is four calls:
 *
 *   sa_tile_pool        tile means of Q and K (and V for landmarks)
 *   sa_tile_scores      per-head tile-score matrix  s = mean(Q) . mean(K)^T
 *   sa_select_topk      per query tile: own-frame tiles + top-k other tiles
 *   sa_sparse_attn_fwd  block-sparse softmax attention over the kept tiles,
 *                       every frame's special tokens, and (optionally) one
 *                       landmark token per unselected tile
 *
 * plus sa_dense_attn_fwd, the dense (sparsity 0) control at the same shape.
 *
 * Conventions shared by every call
 * --------------------------------
 * Tokens.  t = s*N + n for frame s < S and token n < N.  Tokens n < n_sink
 *   of every frame are the camera/register ("sink") tokens.
 * Layout.  Q, K, V, O are contiguous [bh][S*N][head_dim] arrays of the
 *   shape's dtype (bf16 or f32); bh folds batch and heads, which are
 *   independent problems.
 * Tiles.  Tiles are frame aligned: frame s has tpf = ceil(N/tile) tiles, the
 *   last one partial; tile j covers frame j / tpf, tokens
 *   [(j%tpf)*tile, min(N, (j%tpf+1)*tile)).  nt = S*tpf (sa_num_tiles).
 *   A tile's KEY rows are its tokens with n >= n_sink; sink keys are never
 *   part of a tile and are attended once by every query instead.
 * Pointers.  Every array argument is a DEVICE pointer on the current device,
 *   16-byte aligned and contiguous; the caller allocates and owns all of
 *   them (the library keeps only a device error word and per-device launch
 *   attributes).  Optional arguments are marked _or_null.
 * Streams.  Every compute call is asynchronous on `stream` (NULL = legacy
 *   default stream) and never synchronises, except sa_check_device_error.
 * Errors.  Arguments are validated on the host before any launch: an invalid
 *   shape, a NULL required pointer or a misaligned pointer returns
 *   SA_ERR_INVALID_ARG (or SA_ERR_UNSUPPORTED for a shape outside the built
 *   kernels) and touches no output.  A failed launch returns SA_ERR_CUDA.
 *   Errors found on the device (a bounded wait that ran out, a kept list
 *   with an out-of-range entry) are recorded in a device error word that
 *   sa_check_device_error reads and clears.
 * Threads.  Calls on different streams with disjoint outputs may run
 *   concurrently from several host threads.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* sa_stream_t;

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,   /* bad shape, NULL or misaligned pointer, bad size */
    SA_ERR_UNSUPPORTED = 2,   /* valid, but outside what the built kernels handle */
    SA_ERR_CUDA = 3,          /* a CUDA runtime/driver call or a launch failed */
    SA_ERR_TIMEOUT = 4,       /* a device-side wait ran out of its time limit */
    SA_ERR_BAD_LIST = 5,      /* a kept list held an index outside [0, nt) */
    SA_ERR_WORKSPACE = 6      /* workspace NULL or smaller than the _workspace_size query */
} sa_status;

typedef enum { SA_F32 = 0, SA_BF16 = 1 } sa_dtype;

typedef struct {
    int32_t bh;            /* batch * heads: independent problems (>= 1) */
    int32_t frames;        /* S (>= 1) */
    int32_t tokens;        /* N tokens per frame (>= 1) */
    int32_t head_dim;      /* d; 64 is built (else SA_ERR_UNSUPPORTED) */
    int32_t tile;          /* T in {64, 128} */
    int32_t n_sink;        /* special tokens per frame, 0 <= n_sink < tokens */
    sa_dtype dtype;        /* element type of Q, K, V, O, sink_k, sink_v */
    float softmax_scale;   /* logit scale; 0 selects 1/sqrt(head_dim) */
} sa_shape;

/* Number of tiles nt = frames * ceil(tokens / tile); -1 for an invalid shape. */
int32_t sa_num_tiles(const sa_shape* shape);

/* Length of every kept list for budget k: tpf + min(k, C), C the number of tiles
 * outside one frame that have at least one key row.  -1 for an invalid shape or k < 0. */
int32_t sa_max_kept(const sa_shape* shape, int32_t k);

/*
 * Step 1 - tile pooling (Zebra3D abstract: tiles and their landmark summaries;
 * AVGGT technical summary 2.B.2: a mean key/value pair stands for discarded columns).
 *
 *   q_pool[h][j][:] = mean of q over every row of tile j                 (f32 [bh][nt][d])
 *   k_pool[h][j][:] = mean of k over the key rows of tile j (0 if none)  (f32 [bh][nt][d])
 *   v_pool[h][j][:] = mean of v over the key rows (only if v and v_pool are both non-NULL)
 *   k_cnt[j]        = number of key rows of tile j                       (int32 [nt])
 *   sink_k[h][s*n_sink + n][:] = k[h][s*N + n][:]  for n < n_sink  ([bh][S*n_sink][d], dtype)
 *   sink_v likewise from v.
 * Means accumulate in f32.  sink_k/sink_v may be NULL only when n_sink == 0; sink_v is
 * required whenever n_sink > 0 and v is non-NULL.
 */
sa_status sa_tile_pool(const sa_shape* shape, const void* q, const void* k, const void* v_or_null,
                       float* q_pool, float* k_pool, float* v_pool_or_null, int32_t* k_cnt,
                       void* sink_k_or_null, void* sink_v_or_null, sa_stream_t stream);

/*
 * Step 2 - tile scores (SAF3R abstract: rank the candidate interactions per head).
 *
 *   scores[h][i][j] = sum_e q_pool[h][i][e] * k_pool[h][j][e]     (f32 [bh][nt][nt])
 *
 * f32-accurate dot products on the tensor cores: each f32 operand is split into two tf32 parts
 * (hi = x rounded to tf32, lo = x - hi rounded to tf32) and hi.hi + hi.lo + lo.hi is accumulated
 * in f32; the error stays below about 2^-21 * sum_e |q_e k_e|.  No 1/sqrt(d): it does not change
 * a ranking.  q_pool, k_pool and scores 16-byte aligned; rows of nt scores (a row length that is a
 * multiple of 4 gets 16-byte stores).
 */
sa_status sa_tile_scores(const sa_shape* shape, const float* q_pool, const float* k_pool,
                         float* scores, sa_stream_t stream);

/* Bytes of workspace sa_select_topk needs: 0 when scores are given (streamed == 0); with
 * streamed != 0 the size of one L2-resident block of score rows (a few tens of MB at most). */
size_t sa_select_workspace_size(const sa_shape* shape, int32_t streamed);

/*
 * Step 3 - top-k tile selection (SAF3R abstract: dynamic, input-dependent selection; AVGGT
 * technical summary 2.B.1/2.B.2: the own frame and the diagonal are always kept).
 *
 * For query tile i of head h in frame f: the kept list is every tile of frame f plus the k
 * highest-scoring candidate tiles (tiles of other frames with at least one key row), ranked
 * by score descending and, among equal scores, by lower tile index; all candidates when k
 * is at least their number.  Output:
 *   kept_idx[h][i][0..kept_cnt) ascending tile indices, the rest of the row set to -1
 *                               (int32 [bh][nt][max_kept], max_kept = sa_max_kept(shape,k))
 *   kept_cnt[h][i]              list length                  (int32 [bh][nt])
 * scores_or_null != NULL: read the materialised matrix of sa_tile_scores.
 * scores_or_null == NULL: "streamed" mode - the scores are recomputed from q_pool/k_pool one
 *   block of rows at a time into `workspace` (>= sa_select_workspace_size(shape, 1) bytes),
 *   so the [bh][nt][nt] matrix is never materialised.  q_pool/k_pool are ignored otherwise.
 * Scores that are NaN give unspecified (but in-range) lists.  nt <= 32768 is built.
 */
sa_status sa_select_topk(const sa_shape* shape, const float* scores_or_null,
                         const float* q_pool, const float* k_pool, int32_t k,
                         int32_t* kept_idx, int32_t* kept_cnt, int32_t max_kept,
                         void* workspace_or_null, size_t workspace_bytes, sa_stream_t stream);

/*
 * sa_select_topk with a budget per head (SAF3R abstract: attention sparsity differs across
 * heads, and the budgets come from offline head profiling and online adaptation; neither the
 * profile nor the adaptation rule is part of this library - the caller supplies the budgets).
 *   k_per_head  int32 [bh], DEVICE memory, 4-byte aligned: head h keeps the k_per_head[h]
 *               best candidate tiles (all of them when the budget reaches their number, i.e.
 *               a dense head; 0 keeps the own frame only).  Read on the device when the
 *               kernels run, so the budgets may be computed on the GPU in the same stream.
 *   k_max       an upper bound on every entry, >= 0; max_kept >= sa_max_kept(shape, k_max).
 *               An entry below 0 or above k_max is clamped into [0, k_max] and reported as
 *               SA_ERR_INVALID_ARG by sa_check_device_error.
 * Everything else, outputs included, is as for sa_select_topk; kept_cnt varies by head and
 * sa_sparse_attn_fwd consumes the lists unchanged.  Returns SA_ERR_INVALID_ARG for a NULL or
 * misaligned k_per_head or k_max < 0, before any launch.
 */
sa_status sa_select_topk_per_head(const sa_shape* shape, const float* scores_or_null,
                                  const float* q_pool, const float* k_pool,
                                  const int32_t* k_per_head, int32_t k_max,
                                  int32_t* kept_idx, int32_t* kept_cnt, int32_t max_kept,
                                  void* workspace_or_null, size_t workspace_bytes, sa_stream_t stream);

/* Bytes of workspace sa_head_budgets needs: one f32 per (head, query tile). */
size_t sa_head_budget_workspace_size(const sa_shape* shape);

/*
 * Per-head budgets from an online statistic of each head's own pooled scores (SAF3R
 * abstract: sparsity differs across heads and each head's budget is adapted online).  The
 * pages give no formula; this call computes, for every head h,
 *   H_i  = entropy (natural log) of softmax_j(temperature * s_ij) over the candidate tiles j
 *          of query tile i (the tiles sa_select_topk may choose), 0 without candidates
 *   P_h  = (1/nt) sum_i exp(H_i)   (mean perplexity: how many candidates a tile spreads over;
 *          a tile without candidates adds 0)
 *   k_h  = min(k_hi, max(k_lo, floor(beta * P_h + 1/2)))
 * with s_ij = q_pool[h][i] . k_pool[h][j] (the f32 FMA chain of sa_tile_scores, recomputed:
 * no score matrix is read or written).  Outputs, DEVICE memory:
 *   k_per_head          int32 [bh], 4-byte aligned - ready for sa_select_topk_per_head with
 *                       k_max = k_hi in the same stream
 *   perplexity_or_null  f32 [bh] P_h (may be NULL)
 * temperature > 0 and beta >= 0 finite, 0 <= k_lo <= k_hi, else SA_ERR_INVALID_ARG;
 * workspace >= sa_head_budget_workspace_size(shape) bytes, 16-byte aligned, else
 * SA_ERR_WORKSPACE.  Deterministic (fixed summation orders).  Uniform scores give P_h = the
 * candidate count, so beta = 1 with k_hi at or above it makes that head dense.
 */
sa_status sa_head_budgets(const sa_shape* shape, const float* q_pool, const float* k_pool, float temperature,
                          float beta, int32_t k_lo, int32_t k_hi, int32_t* k_per_head,
                          float* perplexity_or_null, void* workspace, size_t workspace_bytes,
                          sa_stream_t stream);

/*
 * sa_select_topk in streamed mode without any caller-provided memory.  No passage of the
 * pages corresponds to this call; it exists for callers that cannot allocate device memory
 * where this step runs - for instance plugin code inside a host framework that owns the
 * device memory pool and hands out no allocator, or a latency-bound loop that forbids
 * allocation after start-up.  Instead of a workspace it uses a fixed 8 MiB scratch array that
 * is part of the library image: every GPU that loads the library holds it until the process
 * exits.  The result is the same as sa_select_topk(shape, NULL, q_pool, k_pool, k, ...).
 *   Limit: nt <= 32768 (the scratch holds at least 64 whole score rows); larger shapes
 *          return SA_ERR_UNSUPPORTED.
 *   Set-up: the first call on a device looks up the scratch array's device address (a host-
 *          side runtime query); make that first call before any stream capture begins.  The
 *          address is kept for the life of the process: after cudaDeviceReset the module may
 *          load at another address, so this call is not valid across a device reset (nor is
 *          any other entry point, whose one-time kernel attributes a reset also clears).
 *   Sharing: all calls on a device use the same array and it keeps the last call's contents
 *          (every score row is written before it is read, so nothing needs clearing).  Calls
 *          whose kernels overlap on the GPU (e.g. on different streams) race on it.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine is called.
 */
sa_status sa_select_topk_noalloc(const sa_shape* shape, const float* q_pool, const float* k_pool, int32_t k,
                                 int32_t* kept_idx, int32_t* kept_cnt, int32_t max_kept, sa_stream_t stream);

/* Bytes of workspace sa_sparse_attn_fwd needs: a transposed copy of every V tile it may gather
 * (the size of V plus the sink segment) and, in landmark mode, the landmark tables, in the
 * input type; for f32 inputs also Q, K and the sink keys rounded to tf32. */
size_t sa_sparse_attn_workspace_size(const sa_shape* shape, int32_t landmark);

/*
 * Step 4 - block-sparse attention forward (Zebra3D abstract: tile-sparse attention with
 * landmark summaries of the unselected context; AVGGT 2.B.2: all queries and special tokens
 * kept, discarded columns approximated by mean key/value pairs).
 *
 * For every query row r of query tile i (head h) the attended keys are
 *   (i)   the key rows of every tile listed in kept_idx[h][i][0..kept_cnt[h][i]),
 *   (ii)  every frame's sink token, once each (sink_k/sink_v from sa_tile_pool),
 *   (iii) if landmark != 0: one token (k_pool[h][j], v_pool[h][j]) with logit bias ln(k_cnt[j])
 *         for every tile j that is not listed and has k_cnt[j] > 0,
 * and   O[h][r] = sum_t softmax_t(scale * q_r . k_t + b_t) v_t,
 *       lse[h][r] = ln sum_t exp(scale * q_r . k_t + b_t)       (natural log; optional).
 * O has the shape's dtype, [bh][S*N][d]; lse is f32 [bh][S*N].  Products run on the tensor
 * cores with f32 accumulation and an f32 softmax: bf16 operands for bf16 inputs (landmark means
 * enter rounded to bf16), tf32 operands (each f32 rounded to the nearest tf32) for f32 inputs.
 * With bf16 tile-128 inputs the masks of partial tiles and listed landmark tiles (-2^100) and
 * the landmark terms b_t (divided by scale, as three bf16 parts: about f32 accuracy) are added
 * to the scores by one more tensor-core product.
 * Lists must be ascending with entries in [0, nt) and no repeats; a list from sa_select_topk
 * always is.  Entries beyond kept_cnt are ignored.  An out-of-range entry is skipped and
 * reported as SA_ERR_BAD_LIST by sa_check_device_error.
 * workspace: >= sa_sparse_attn_workspace_size(shape, landmark) bytes (NULL when that is 0).
 */
sa_status sa_sparse_attn_fwd(const sa_shape* shape, const void* q, const void* k, const void* v,
                             const int32_t* kept_idx, const int32_t* kept_cnt, int32_t max_kept,
                             const void* sink_k_or_null, const void* sink_v_or_null,
                             int32_t landmark, const float* k_pool_or_null,
                             const float* v_pool_or_null, const int32_t* k_cnt_or_null,
                             void* workspace_or_null, size_t workspace_bytes,
                             void* o, float* lse_or_null, sa_stream_t stream);

/* Bytes of workspace sa_sparse_attn_bwd needs for these lists and mode (bf16, tile 128 only;
 * 0 otherwise): transposed tiles of Q, dO and K, fp32 accumulators of dK and dV, the reverse
 * lists and, in landmark mode, the landmark tables - roughly 8x the size of Q. */
size_t sa_sparse_attn_bwd_workspace_size(const sa_shape* shape, int32_t max_kept, int32_t landmark);

/*
 * Backward of step 4, for training a backbone whose global layers are made sparse after
 * conversion (Zebra3D abstract: tile-sparse attention with landmark summaries).
 *
 * Gradients of sum(d_o * O) for O = sa_sparse_attn_fwd(q, k, v, lists, ...), the lists held
 * fixed (selection is piecewise constant in its inputs, so no gradient flows into it).  With
 * P the forward's probabilities over each row's attended set and D_r = sum_e d_o[r][e] o[r][e]:
 *   dS = P * (d_o V^T - D),  dq = scale dS K,  dk = scale dS^T Q,  dv = P^T d_o,
 * summed over every query row that attends a key; a sink row receives its sink-segment terms;
 * in landmark mode the landmark of tile j (the mean of its k_cnt[j] non-sink rows) passes its
 * gradient to each of those rows divided by k_cnt[j].
 *   q, k, v, o    the forward's inputs and output, [bh][S*N][64] bf16
 *   lse           the forward's lse (natural log), f32 [bh][S*N]; required
 *   d_o           upstream gradient, [bh][S*N][64] bf16
 *   lists, sinks, landmark, pools: exactly as passed to sa_sparse_attn_fwd
 *   dq, dk, dv    outputs, [bh][S*N][64] bf16, written in full (caller-owned, 16-byte aligned)
 * Products run on the tensor cores (bf16 operands, f32 accumulation; P and dS enter rounded to
 * bf16).  dk and dv are accumulated with f32 atomics, so the last bits of their values may
 * vary between calls.  bf16, d = 64, tile = 128 only (else SA_ERR_UNSUPPORTED).  Bad list
 * entries are skipped and reported as SA_ERR_BAD_LIST by sa_check_device_error.
 * workspace: >= sa_sparse_attn_bwd_workspace_size(shape, max_kept, landmark) bytes.
 */
sa_status sa_sparse_attn_bwd(const sa_shape* shape, const void* q, const void* k, const void* v,
                             const void* o, const float* lse, const void* d_o,
                             const int32_t* kept_idx, const int32_t* kept_cnt, int32_t max_kept,
                             const void* sink_k_or_null, const void* sink_v_or_null,
                             int32_t landmark, const float* k_pool_or_null,
                             const float* v_pool_or_null, const int32_t* k_cnt_or_null,
                             void* workspace, size_t workspace_bytes,
                             void* dq, void* dk, void* dv, sa_stream_t stream);

/* Bytes of workspace sa_dense_attn_fwd needs (a transposed copy of V; for f32 inputs also Q
 * and K rounded to tf32). */
size_t sa_dense_attn_workspace_size(const sa_shape* shape);

/*
 * The dense control: softmax(scale * Q K^T) V over all S*N keys of each head, no tiles,
 * sinks or landmarks ("AVGGT" section 1: global attention; "(Full) Attention is More Than
 * You Need": full attention).  Same layouts and precision as sa_sparse_attn_fwd; n_sink is
 * ignored.  workspace: >= sa_dense_attn_workspace_size(shape) bytes (NULL when that is 0).
 */
sa_status sa_dense_attn_fwd(const sa_shape* shape, const void* q, const void* k, const void* v,
                            void* workspace_or_null, size_t workspace_bytes,
                            void* o, float* lse_or_null, sa_stream_t stream);

/* Static description of a status code (never NULL). */
const char* sa_status_string(sa_status status);

/* Synchronises `stream`, then returns and clears the first device-detected error on the
 * current device (SA_OK if none).  Returns SA_ERR_CUDA if the synchronisation itself fails. */
sa_status sa_check_device_error(sa_stream_t stream);

/* Upper bound in nanoseconds on every device-side wait of later launches on the current
 * device (default 2e9, i.e. 2 s; must be > 0).  A wait that runs out ends its kernel early
 * with SA_ERR_TIMEOUT recorded; outputs of that launch are then undefined. */
sa_status sa_set_wait_limit_ns(int64_t limit_ns);

/*
 * Subsampled global attention ("AVGGT: Rethinking Global Attention for Accelerating VGGT",
 * technical summary 2.B.2, SGA), an alternative to steps 1-4 for the later global layers.
 * Every frame is shape->n_sink special tokens followed by a grid_h x grid_w patch grid in
 * row-major order (shape->tokens == n_sink + grid_h * grid_w).  Keys and values are kept for
 * the special tokens of every frame and for the patches at (r, c) with r a multiple of s_h
 * and c a multiple of s_w (one per s_h x s_w window); every query is kept.  Query t attends to
 *   - every kept key of every frame,
 *   - its own key (the diagonal), when its token is not among the kept ones,
 *   - one mean key/value pair standing for the other discarded tokens of all frames
 *     (mean K, mean V over them; logit scale * q.k_mean + ln(their count)),
 * with softmax_scale as for sa_sparse_attn_fwd.  Output O [bh][S*N][64] and, when lse_or_null
 * is given, the natural-log LSE [bh][S*N] of that softmax.
 * Built for bf16, head_dim 64 and tile 128 (the tensor-core path; SA_ERR_UNSUPPORTED else).
 * workspace: >= sa_sga_workspace_size(...) bytes, 16-byte aligned (the compacted K/V
 * sequence, fp32 sums of the discarded rows, an LSE scratch and the attention's V^T tiles).
 * SA_ERR_INVALID_ARG for a grid that does not match shape->tokens, strides < 1, NULL or
 * misaligned pointers; all checked on the host before any launch.
 */
size_t sa_sga_workspace_size(const sa_shape* shape, int32_t grid_h, int32_t grid_w, int32_t s_h, int32_t s_w);
sa_status sa_sga_fwd(const sa_shape* shape, int32_t grid_h, int32_t grid_w, int32_t s_h, int32_t s_w,
                     const void* q, const void* k, const void* v, void* workspace, size_t workspace_bytes,
                     void* o, float* lse_or_null, sa_stream_t stream);

/* Test facility for the failure path (not for production use): while enable != 0, later
 * launches of the tensor-core attention kernels (bf16, tile 128: the forward and the dQ kernel
 * of sa_sparse_attn_bwd) on the current device never issue the first query-tile load of their
 * first CTA, so that CTA's MMA warp waits for data that cannot arrive.  The wait runs out after the wait limit, the CTA drains what it has in
 * flight and exits, and sa_check_device_error reports SA_ERR_TIMEOUT; the outputs of such a
 * launch are undefined and the device stays usable.  Returns SA_ERR_CUDA if the setting
 * cannot be written. */
sa_status sa_test_withhold_query_load(int32_t enable);

#ifdef __cplusplus
}
#endif

#endif /* SA_H_ */
