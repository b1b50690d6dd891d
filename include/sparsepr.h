/*
 * sparsepr.h -- C ABI of the SparsePR attention operator for NVIDIA B200 (sm_100a).
 *
 * SparsePR (arXiv 2608.18484) replaces one dense softmax-attention call by
 *   (a) Response-Coupled Partitioning: keys, with their paired values, are grouped by
 *       their responses to a sample of queries; queries are then grouped by their
 *       responses to the key-group centroids, in one asymmetric pass;
 *   (b) shared block routing: each query block evaluates the key groups with the
 *       largest centroid score, up to an executed-pair density budget that counts the
 *       probe rows;
 *   (c) block-sparse softmax attention over the routed (query block, key group) pairs;
 *   (d) Probe-Fitted Residual Reconstruction: exact attention on a few probe rows per
 *       head calibrates a weighted-ridge affine map from sparse output to residual,
 *       restricted to the top-r subspace of the probe residuals; the predicted residual
 *       is added to every unprobed row.
 * Sources: the paper's abstract (English text on the arxivdaily.com page for
 * 2608.18484; also reprinted on the peercurrent.com digest) and the skillfed.io article
 * "Partition the Support, Reconstruct the Residual", paragraph on the two components.
 * The pages give the method in prose only; the readings this library takes where they
 * are silent are stated at each call below.
 *
 * Conventions (all calls):
 *  - Tensor arguments are DEVICE pointers owned by the caller; the library never
 *    allocates, frees or synchronises on them.  Scratch space is the caller's
 *    workspace `ws` of sparsepr_workspace_size() bytes (256-byte aligned), which
 *    must not be shared by calls that may overlap on the GPU.  Its first 256 bytes
 *    are a status header that must be zero before the first call on a new workspace
 *    (sparsepr_partition zeroes it again at the start of every call sequence).
 *  - Every call is asynchronous on `stream` (0 = legacy default stream).
 *  - Q, K and V start on 16-byte boundaries (else SPARSEPR_ERR_INVALID_ARG).
 *  - Layouts are contiguous row-major: Q, K, V, O are [Bt, H, N, d]; per-head index
 *    arrays are [Bt, H, ...] as stated.  dtype is SPARSEPR_BF16 or SPARSEPR_F32;
 *    d is 64 or 128; block B is 64 or 128; indices are int32, pair counts int64.
 *  - Return value: SPARSEPR_OK or an error code; on error nothing was launched and
 *    sparsepr_last_error() returns a message (thread-local).  Errors found on the
 *    device (a NaN reaching a decision, a bounded wait that ran out) are recorded in a
 *    status word inside `ws`; sparsepr_check() reads it.
 *  - Partition state never persists between calls: each call's map is call-specific.
 *  - Key-group copy (bf16, d = 128, B = 128): sparsepr_probe_dense, sparsepr_sparse_attn
 *    and sparsepr_sparse_attn_apply gather K and V into key-group order inside `ws`.
 *    The header records the K, V, key_perm and key_gsize pointers and the shape the
 *    copy was made from, and a later call with the same ones reuses it instead of
 *    copying again (the probe-first pipeline copies once).  sparsepr_partition clears
 *    the record.  A caller that rewrites K, V, key_perm or key_gsize in place between
 *    such calls, with no partition call in between, calls sparsepr_reset_workspace.
 */
#ifndef SPARSEPR_H
#define SPARSEPR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SPARSEPR_API __attribute__((visibility("default")))
#else
#define SPARSEPR_API
#endif

typedef struct CUstream_st* sparsepr_stream_t; /* same type as cudaStream_t */

enum {
  SPARSEPR_OK = 0,
  SPARSEPR_ERR_INVALID_ARG = 1,
  SPARSEPR_ERR_UNSUPPORTED = 2,
  SPARSEPR_ERR_CUDA = 3,
  SPARSEPR_ERR_TIMEOUT = 4,   /* a bounded device-side wait gave up */
  SPARSEPR_ERR_NONFINITE = 5  /* a NaN reached a clustering or routing decision */
};

enum { SPARSEPR_BF16 = 0, SPARSEPR_F32 = 1 };

enum { SPARSEPR_WEIGHT_INV_NORM = 0, SPARSEPR_WEIGHT_UNIFORM = 1 };

/* Option bit of weight_mode (the fit's parameters): the ridge lambda is taken relative to
 * the scale of the probe outputs, lambda_eff = lambda * tr(X_c^T W X_c) / d, instead of
 * as an absolute number.  The abstract says "weighted ridge regression" without the scale
 * of lambda; absolute lambda (the default) is the plain reading, the relative one makes
 * the fit invariant to the scale of the outputs and is what the probe-budget study
 * compares it with. */
enum { SPARSEPR_RIDGE_RELATIVE = 0x100 };

/* Partition rule.  RESPONSE: Response-Coupled Partitioning (the method).  SEMANTIC: the
 * semantic block-sparse baseline the pages compare against, read as balanced k-means on
 * the raw keys and on the raw queries (same start, fill, iterations and routing); the
 * pages do not state that rule. */
enum { SPARSEPR_PARTITION_RESPONSE = 0, SPARSEPR_PARTITION_SEMANTIC = 1 };

/* Block-routing score (one uniform k either way, so the executed-pair count is the
 * same).  CENTROID: tau qbar_b . mu_g (the method's reading).  SIZE_CORRECTED:
 * tau qbar_b . mu_g + log n_g (first-order log attention mass of the block's mean query
 * on group g).  LSE: log sum_{j in g} exp(tau qbar_b . k_j) (that mass itself).  The
 * pages say "up to a target density" without the score; these are the readings the
 * comparison covers. */
enum { SPARSEPR_ROUTE_CENTROID = 0, SPARSEPR_ROUTE_SIZE_CORRECTED = 1, SPARSEPR_ROUTE_LSE = 2 };

/* How the executed-pair budget floor(rho*N*N - P*N) is spent (SparsePR abstract: routing
 * "up to a target density" names the budget, not its split).  UNIFORM: every query block
 * takes the same number k of key groups (the plain reading).  GLOBAL: the head's budget
 * is shared by its blocks: every block keeps its best group, then the remaining
 * (block, group) pairs are taken in descending score order (ties to the lower block,
 * then the lower group) while the cumulative n_b * n_g stays within the budget. */
enum { SPARSEPR_BUDGET_UNIFORM = 0, SPARSEPR_BUDGET_GLOBAL = 1 };

typedef struct sparsepr_params {
  int32_t block;        /* B: query-block and key-group capacity (64 or 128)            */
  int32_t n_sampled;    /* S: sampled queries that define key response profiles        */
  int32_t n_probe;      /* P: exact probe rows per head                                 */
  int32_t kmeans_iters; /* T: balanced k-means iterations on each side (>= 0)           */
  int32_t rank;         /* r: residual subspace rank (clamped to d)                    */
  int32_t weight_mode;  /* SPARSEPR_WEIGHT_* (probe weights when none are supplied),
                           optionally | SPARSEPR_RIDGE_RELATIVE                           */
  double density;       /* rho: executed-pair budget / N^2, probe rows counted          */
  double ridge_lambda;  /* lambda: ridge on the centred weighted Gram (sum w = P)       */
  float scale;          /* softmax scale tau; <= 0 selects 1/sqrt(d)                    */
  int32_t partition_mode; /* SPARSEPR_PARTITION_*                                        */
  int32_t route_scores;   /* SPARSEPR_ROUTE_*: what block_scores hold                    */
  int32_t route_budget;   /* SPARSEPR_BUDGET_*: uniform k per block or one budget per head */
} sparsepr_params;

/* Number of groups G = Gq = ceil(N / B): capacity-B groups that cover all N tokens. */
SPARSEPR_API int32_t sparsepr_num_groups(int32_t N, int32_t block);

/* Routed key groups per query block (host arithmetic, no device work):
 * k = clamp(floor((rho*N*N - P*N) / (N*B)), 1, G), evaluated in IEEE double in this
 * order.  Reading: one uniform k for every block, so that k*N*B + P*N <= rho*N^2
 * (the budget counts probes, as the abstract's density figure does). */
SPARSEPR_API int32_t sparsepr_route_k(int32_t N, int32_t block, double density, int32_t n_probe);

/* Probe rows of every (batch, head): the midpoint stride floor((2p+1)N/(2P)), p < P,
 * in raster token order (reading: the pages do not say how probe rows are chosen; a
 * stride spreads them over all frames).  probe_idx [Bt,H,P] int32, device. */
SPARSEPR_API int sparsepr_probe_rows(int32_t N, int32_t P, int32_t Bt, int32_t H, int32_t* probe_idx,
                        sparsepr_stream_t stream);

/* Bytes of workspace one call sequence needs for these sizes (0 on invalid sizes). */
SPARSEPR_API size_t sparsepr_workspace_size(int32_t Bt, int32_t H, int32_t N, int32_t d,
                               const sparsepr_params* params);

/* (a) Response-Coupled Partitioning.
 *   Q, K        [Bt,H,N,d] dtype.  V is not read: values follow their keys.
 *   sample_idx  [S] int32 token indices of the sampled queries, or NULL for the
 *               midpoint stride floor((2m+1)N/(2S)) (reading: the pages do not say
 *               how queries are sampled).
 *   Outputs:
 *   key_perm    [Bt,H,G*B]  member tokens of key group g at [g*B, g*B+size), in
 *               ascending token order, -1 in the padding slots.
 *   key_gsize   [Bt,H,G]    members per key group (1..B).
 *   query_perm  [Bt,H,Gq*B], qblock_size [Bt,H,Gq]: the same for query blocks.
 *   block_scores[Bt,H,Gq,G] fp32 routing score of (query block b, key group g): the
 *               mean over b's members of tau * q_i . mu_g, mu_g = mean key of g.
 * Method: keys are clustered on profiles r_j[m] = tau q_{s_m} . k_j by T iterations of
 * balanced k-means (start: contiguous chunks of B tokens; assignment: capacity-B
 * proposal rounds, ties to lower group, then lower token); queries are clustered the
 * same way on coordinates u_i[g] = tau q_i . mu_g.  Both clusterings run in the
 * exactly equivalent head-dim form |x - c|_Gamma^2 with Gamma = Q_S^T Q_S (keys) or
 * mu^T mu (queries), on tensor cores.  Resets the status word in ws. */
SPARSEPR_API int sparsepr_partition(const void* Q, const void* K, int dtype, int32_t Bt, int32_t H,
                       int32_t N, int32_t d, const sparsepr_params* params,
                       const int32_t* sample_idx, int32_t* key_perm, int32_t* key_gsize,
                       int32_t* query_perm, int32_t* qblock_size, float* block_scores,
                       void* ws, sparsepr_stream_t stream);

/* (b) Centroid routing.  UNIFORM budget: for every query block, the k key groups with
 * the largest block score (ties to the lower group index), written in ascending group
 * order, with k = sparsepr_route_k(N, B, density, P).  GLOBAL budget: the groups that
 * the head-wide allocation (SPARSEPR_BUDGET_GLOBAL) gives each block, in ascending
 * order, then -1 up to k = G (at most 8192 groups per head, else UNSUPPORTED; density
 * must be finite, else INVALID_ARG).  The row capacity k is returned in *k_out (host
 * memory); the attention and probe calls take it and stop at the first -1.
 *   route          [Bt,H,Gq,k] int32
 *   executed_pairs [Bt,H] int64 = sum_b qblock_size[b] * sum_{g in route(b)} key_gsize[g]
 *                  + P*N: every evaluated (query, key) pair, probe rows counted.
 * A NaN score sets SPARSEPR_ERR_NONFINITE in the status word (NaN ranks lowest). */
SPARSEPR_API int sparsepr_route(const float* block_scores, const int32_t* key_gsize,
                   const int32_t* qblock_size, int32_t Bt, int32_t H, int32_t N,
                   const sparsepr_params* params, int32_t* route, int32_t* k_out,
                   int64_t* executed_pairs, void* ws, sparsepr_stream_t stream);

/* (c) Block-sparse softmax attention.  Row i of query block b attends to the union of
 * the members of the routed key groups of b, softmax renormalised over that support:
 *   S_out[i] = sum_j softmax_j(tau q_i . k_j) v_j,  written fp32 in token order
 *   [Bt,H,N,d].  bf16 inputs run on tensor cores with fp32 accumulation.  route is
 *   [Bt,H,Gq,k] as written by sparsepr_route (k its *k_out): every row's groups in
 *   ascending order, each row ending at k entries or at its first -1 (global budget).
 *   The same holds for the route argument of the calls below. */
SPARSEPR_API int sparsepr_sparse_attn(const void* Q, const void* K, const void* V, int dtype,
                         int32_t Bt, int32_t H, int32_t N, int32_t d, int32_t block,
                         const int32_t* key_perm, const int32_t* key_gsize,
                         const int32_t* query_perm, const int32_t* qblock_size,
                         const int32_t* route, int32_t k, float scale, float* S_out,
                         void* ws, sparsepr_stream_t stream);

/* (c + e, fused) Block-sparse attention with the residual correction applied in the
 * attention kernel's epilogue (probe-first order: sparsepr_probe_dense and
 * sparsepr_fit_residual run before it):
 *   O[i] = s_i + M s_i + beta for every row, then the probe rows set to probe_out;
 * s_i as in sparsepr_sparse_attn, never written to memory.  M s_i is formed on the
 * tensor cores from bf16 hi + lo parts of s_i and M (three products, ~16-bit operands).
 * O [Bt,H,N,d] bf16.  Built for dtype BF16, d = 128, block = 128 (other shapes:
 * SPARSEPR_ERR_UNSUPPORTED; use sparsepr_sparse_attn + sparsepr_apply_residual).  The
 * workspace is required.  Source: the abstract (the fitted map predicts each unprobed
 * query's residual, added to its sparse output); the order of the steps is free. */
SPARSEPR_API int sparsepr_sparse_attn_apply(const void* Q, const void* K, const void* V, int dtype,
                         int32_t Bt, int32_t H, int32_t N, int32_t d, int32_t block,
                         const int32_t* key_perm, const int32_t* key_gsize,
                         const int32_t* query_perm, const int32_t* qblock_size,
                         const int32_t* route, int32_t k, float scale, const float* M,
                         const float* beta, const int32_t* probe_idx, int32_t P,
                         const float* probe_out, void* O, void* ws, sparsepr_stream_t stream);

/* One whole SparsePR call on device tensors (S1-S10 in one entry point): partition,
 * route, probe rows (midpoint stride), then -- for bf16, d = 128, B = 128 -- probe rows,
 * fit and the sparse attention with the correction in its epilogue; for other shapes the
 * sparse attention, probe rows, fit and apply.  Every intermediate lives in `ws`, of
 * sparsepr_call_workspace_size() bytes (256-byte aligned, first 256 bytes zero before the
 * first call); O [Bt,H,N,d] in dtype.  params->n_probe must be >= 1.  Errors as for the
 * stage calls; sparsepr_check(ws) reads the device status. */
SPARSEPR_API size_t sparsepr_call_workspace_size(int dtype, int32_t Bt, int32_t H, int32_t N, int32_t d,
                                                 const sparsepr_params* params);
SPARSEPR_API int sparsepr_attention(const void* Q, const void* K, const void* V, int dtype, int32_t Bt,
                                    int32_t H, int32_t N, int32_t d, const sparsepr_params* params, void* O,
                                    void* ws, sparsepr_stream_t stream);

/* The same call with Q, K, V and O in HOST memory (page-locked, or the copies do not
 * overlap).  The Bt*H heads are processed in `groups` consecutive groups, the first about
 * half the size of the others so that only a short copy precedes the first compute (every
 * head is an independent problem, so the result is the same for any grouping): while the group
 * g runs on `stream`, `copy_stream` carries group g + 1 to the device and group g - 1
 * back.  ws: sparsepr_host_workspace_size() bytes (first 256 bytes zero before the first
 * call; sparsepr_check(ws) then reports a device error of any group).  Returns after
 * enqueueing; the host O is complete once `stream` is.  Host calls on one device must not
 * overlap in time (they share the device's copy events). */
SPARSEPR_API size_t sparsepr_host_workspace_size(int dtype, int32_t Bt, int32_t H, int32_t N, int32_t d,
                                                 const sparsepr_params* params, int32_t groups);
SPARSEPR_API int sparsepr_attention_host(const void* Q, const void* K, const void* V, int dtype, int32_t Bt,
                                         int32_t H, int32_t N, int32_t d, const sparsepr_params* params,
                                         void* O, int32_t groups, void* ws, sparsepr_stream_t stream,
                                         sparsepr_stream_t copy_stream);

/* Dense softmax attention of every row against all N keys with the same kernel
 * family (the comparator the density budget is measured against):
 *   O_out [Bt,H,N,d] fp32. */
SPARSEPR_API int sparsepr_dense_attn(const void* Q, const void* K, const void* V, int dtype,
                        int32_t Bt, int32_t H, int32_t N, int32_t d, int32_t block,
                        float scale, float* O_out, void* ws, sparsepr_stream_t stream);

/* (d1) Probe rows.  For each probe token p (probe_idx [Bt,H,P], distinct, in [0,N)):
 *   probe_out    [Bt,H,P,d] fp32: exact attention of p against all N keys;
 *   probe_sparse [Bt,H,P,d] fp32: p's block-sparse output over its block's route.
 * Both are computed with the softmax weights carried at ~16-bit precision (split
 * bf16 hi+lo products), because they are the only inputs of the residual fit. */
SPARSEPR_API int sparsepr_probe_dense(const void* Q, const void* K, const void* V, int dtype,
                         int32_t Bt, int32_t H, int32_t N, int32_t d, int32_t block,
                         const int32_t* probe_idx, int32_t P, const int32_t* key_perm,
                         const int32_t* key_gsize, const int32_t* query_perm,
                         const int32_t* route, int32_t k, float scale, float* probe_out,
                         float* probe_sparse, void* ws, sparsepr_stream_t stream);

/* (d2) Residual fit, per (batch, head), in fp64:
 *   y_p = probe_out_p - probe_sparse_p;  w_p from `weights` [Bt,H,P] if not NULL,
 *   else weight_mode (inverse squared norm of probe_out_p, or uniform), then scaled
 *   so sum_p w_p = P;  U_r = top-r eigenvectors of sum_p w_p y_p y_p^T;
 *   z_p = U_r^T y_p;  A = (Z_c^T W X_c)(X_c^T W X_c + lambda I)^-1 with X = probe_sparse
 *   centred at its weighted mean (lambda times tr(X_c^T W X_c) / d when weight_mode has
 *   SPARSEPR_RIDGE_RELATIVE);  b = zbar - A xbar.
 *   Outputs M = U_r A [Bt,H,d,d] and beta = U_r b [Bt,H,d], fp32. */
SPARSEPR_API int sparsepr_fit_residual(const float* probe_sparse, const float* probe_out,
                          const float* weights, int32_t Bt, int32_t H, int32_t d,
                          int32_t P, double ridge_lambda, int32_t rank,
                          int32_t weight_mode, float* M, float* beta, void* ws,
                          sparsepr_stream_t stream);

/* Allocation-free variant of sparsepr_fit_residual (no counterpart in the paper: it is
 * an interface for callers that cannot allocate device memory, such as an inference-
 * engine plugin bound to a memory plan fixed before execution, or a latency-critical
 * loop that cannot take cudaMalloc's implicit synchronisation).  Same arguments, layout
 * and result as sparsepr_fit_residual, but no workspace: the scratch is a 32 MiB static
 * device array inside the library, held by every GPU that loads it until the process
 * exits.  Limit: 256 + 8 * Bt*H * (2 d^2 + P d + 4 d) bytes <= 32 MiB (d = 128, P = 256:
 * 63 heads); larger calls return SPARSEPR_ERR_UNSUPPORTED without launching.  The call
 * allocates nothing (no cudaMalloc/cudaFree).  The first call on each device (and the
 * first after the device's context changed, e.g. after cudaDeviceReset) looks up the
 * array's device address; make that first call before any stream capture.  Every call
 * shares the one array (it keeps the last call's contents; the kernel rewrites all of it
 * before reading it), so calls that overlap on the GPU race: serialise them, e.g. on one
 * stream.
 *   status  optional DEVICE int32 (NULL: not reported): receives this call's device
 *           status on `stream` after the fit, SPARSEPR_OK or the first error code.  As in
 *           sparsepr_fit_residual, a weight sum that is not positive records
 *           SPARSEPR_ERR_INVALID_ARG and the head is fitted with uniform weights; a ridge
 *           system whose Cholesky fails (lambda = 0 on a singular Gram) records
 *           SPARSEPR_ERR_INVALID_ARG and writes M = 0, beta = 0 for the head. */
SPARSEPR_API int sparsepr_fit_residual_noalloc(const float* probe_sparse, const float* probe_out,
                                               const float* weights, int32_t Bt, int32_t H,
                                               int32_t d, int32_t P, double ridge_lambda,
                                               int32_t rank, int32_t weight_mode, float* M,
                                               float* beta, int32_t* status,
                                               sparsepr_stream_t stream);

/* (d3) Apply: O_i = S_i + M S_i + beta for unprobed rows, O_p = probe_out_p for probe
 * rows.  O [Bt,H,N,d] in out_dtype.  O may alias S_out when out_dtype is F32. */
SPARSEPR_API int sparsepr_apply_residual(const float* S_out, const float* M, const float* beta,
                            const int32_t* probe_idx, const float* probe_out,
                            int32_t Bt, int32_t H, int32_t N, int32_t d, int32_t P,
                            void* O, int out_dtype, sparsepr_stream_t stream);

/* Measurement: per-row relative L2 error against a reference output (the metric the
 * abstract reports, averaged there over unprobed queries):
 *   err[b,h,i] = |O_i - O_ref_i|_2 / |O_ref_i|_2, and NaN for the P probe rows listed in
 *   probe_idx [Bt,H,P] (NULL or P = 0: no row is marked).
 *   O [Bt,H,N,d] in o_dtype; O_ref [Bt,H,N,d] fp32; err [Bt,H,N] fp32. */
SPARSEPR_API int sparsepr_row_errors(const void* O, int o_dtype, const float* O_ref,
                                     const int32_t* probe_idx, int32_t Bt, int32_t H,
                                     int32_t N, int32_t d, int32_t P, float* err,
                                     sparsepr_stream_t stream);

/* Number of kernels this library has enqueued since it was loaded (host counter). */
SPARSEPR_API uint64_t sparsepr_launch_count(void);

/* Measurement hook for the tensor-core attention kernels.  sparsepr_kernel_timing(1)
 * makes every later sparse or dense attention call record a CUDA event pair on its
 * stream immediately around the attention kernel itself (the sparse path's copy of K
 * and V into group order is outside the pair); sparsepr_kernel_timing(0) stops it.
 * sparsepr_kernel_timing_read waits for the recorded pairs, returns their summed device
 * time in milliseconds and their number, and forgets them.  Process-wide state meant
 * for timing runs (not for concurrent callers); errors: SPARSEPR_ERR_CUDA. */
SPARSEPR_API int sparsepr_kernel_timing(int enable);
SPARSEPR_API int sparsepr_kernel_timing_read(double* ms_total, int64_t* launches);

/* Wait for `stream` and return the device status word in `ws` (SPARSEPR_OK, or the
 * first device-side error since the last sparsepr_partition).  Apart from the timing
 * hook's read, this is the only call that synchronises. */
SPARSEPR_API int sparsepr_check(const void* ws, sparsepr_stream_t stream);

/* Zero the workspace's 256-byte header on `stream`: clears the status word and the
 * record of the key-group copy (so the next call copies K and V again). */
SPARSEPR_API int sparsepr_reset_workspace(void* ws, sparsepr_stream_t stream);

/* Message of the last host-side error on this thread ("" if none). */
SPARSEPR_API const char* sparsepr_last_error(void);

/* ---- decision kernels on injected scores (used by the parity tests) ---------------
 * sparsepr_test_fill: the capacity-B assignment of a k-means iteration (the fill kernel
 *   of the fp32 and d = 64 partitions; the bf16, d = 128 partition runs the same decision
 *   rule inside its tensor-core assignment kernel, whose decisions the partition trace
 *   exposes), run on caller-supplied fp32 distances D [H, n, G] (device); labels [H, n]
 *   int32; workspace of sparsepr_test_fill_workspace_size bytes.
 * sparsepr_test_topk: the routing selection on caller-supplied scores Sc [H, Gq, G];
 *   route [H, Gq, k] int32.  Both use the same kernels as the operator. */
SPARSEPR_API size_t sparsepr_test_fill_workspace_size(int32_t H, int32_t n, int32_t G);
SPARSEPR_API int sparsepr_test_fill(const float* D, int32_t H, int32_t n, int32_t G, int32_t cap,
                       int32_t* labels, void* ws, sparsepr_stream_t stream);
SPARSEPR_API int sparsepr_test_topk(const float* Sc, int32_t H, int32_t Gq, int32_t G, int32_t k,
                       int32_t* route, void* ws, sparsepr_stream_t stream);

/* sparsepr_test_partition_trace: sparsepr_partition (same arguments, same kernels, same
 * outputs) that also copies its internal state into the caller's DEVICE buffers, so the
 * parity tests can compare every continuous quantity of Response-Coupled Partitioning
 * with the oracle (SparsePR abstract: keys grouped by their responses to sampled
 * queries, queries by their responses to the key-group centroids).  Any member may be
 * NULL (not captured).  T = params->kmeans_iters, HH = Bt*H, G = ceil(N/B):
 *   sample_idx   [S]           sampled query tokens used (midpoint stride or the given ones)
 *   key_gamma    [HH,d,d]      head-dim metric of the key side, Q_S^T Q_S (identity: semantic)
 *   key_dist     [T,HH,N,G]    fp32 distances handed to each key-side capacity fill, in
 *                              response-space units tau^2 |x - c|_Gamma^2 (semantic:
 *                              the raw squared distances |x - c|^2)
 *   key_labels   [T,HH,N]      key-group labels after each fill
 *   mu           [HH,G,d]      key-group mean keys after the last key iteration
 *   query_gamma  [HH,d,d]      metric of the query side, mu^T mu (identity: semantic)
 *   query_dist   [T,HH,N,G], query_labels [T,HH,N]: the same for the query side
 *   qbar         [HH,G,d]      query-block mean queries after the last query iteration
 * The copies are asynchronous on `stream` and do not change what the call computes. */
typedef struct sparsepr_partition_trace {
  int32_t* sample_idx;
  float* key_gamma;
  float* key_dist;
  int32_t* key_labels;
  float* mu;
  float* query_gamma;
  float* query_dist;
  int32_t* query_labels;
  float* qbar;
} sparsepr_partition_trace;
SPARSEPR_API int sparsepr_test_partition_trace(const void* Q, const void* K, int dtype, int32_t Bt, int32_t H,
                       int32_t N, int32_t d, const sparsepr_params* params,
                       const int32_t* sample_idx, int32_t* key_perm, int32_t* key_gsize,
                       int32_t* query_perm, int32_t* qblock_size, float* block_scores,
                       const sparsepr_partition_trace* trace, void* ws, sparsepr_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SPARSEPR_H */
