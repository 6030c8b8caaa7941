/*
 * sparsepr.h -- C ABI of the SparsePR per-call sparse attention path on one
 * NVIDIA B200 (sm_100a).
 *
 * Method sources (web pages, cited by title and section):
 *   [SPR]  "Partition the Support, Reconstruct the Residual: Training-Free
 *          Sparse Attention for Video Generation and World Models" --
 *          section 2 "Methodology": A. response-coupled partitioning,
 *          B. probe-fitted residual reconstruction, C. sparse execution.
 *   [SVOO] "Attention Sparsity is Input-Stable: Training-Free Sparse
 *          Attention for Video Generation via Offline Sparsity Profiling and
 *          Online QK Co-Clustering" -- method details, block selection and
 *          sparse attention assembly.
 *
 * One attention call on H independent heads runs the five calls below in
 * order on one CUDA stream:
 *   sparsepr_partition -> sparsepr_permute -> sparsepr_route
 *   -> sparsepr_block_sparse_attn -> sparsepr_probe_correct
 *
 * Conventions shared by every call
 *   - Tensors are row-major [H, N, d] with d contiguous (Q, K, V and the
 *     outputs) or [H, n] (integer arrays). All tensor pointers are DEVICE
 *     pointers owned by the caller; the library never allocates, frees or
 *     synchronises on them. Q/K/V-shaped tensors (inputs, permuted copies,
 *     outputs) must be 16-byte aligned; a misaligned pointer is rejected
 *     with SPARSEPR_ERR_INVALID_ARG.
 *   - `ws` is a caller-owned device workspace of at least
 *     sparsepr_workspace_bytes(p) bytes, 256-byte aligned. The same `ws` is
 *     passed to every call of one attention call; its first bytes hold the
 *     device status word and per-call statistics (see sparsepr_read_stats).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call only enqueues work on it and returns.
 *   - Argument errors are found on the host before anything is enqueued and
 *     are returned as SPARSEPR_ERR_INVALID_ARG / _UNSUPPORTED / _WORKSPACE.
 *     A failed launch returns SPARSEPR_ERR_CUDA. Errors that only the device
 *     can see (an empty kept key set, a non-finite value, a wait that ran
 *     out) are OR-ed into the status word in `ws`; read it after the stream
 *     has been synchronised.
 *   - Supported: d in {64, 128}; dtype bf16 or fp32 (the attention MMAs run
 *     in bf16 with fp32 accumulation for both); 1 <= H <= SPARSEPR_MAX_HEADS.
 *   - Text tokens (n_text > 0, the trailing tokens of every head; the
 *     HunyuanVideo-shaped joint attention): they take part in neither
 *     k-means nor the sampled queries; they form one extra key group (index
 *     Ck) that every query group keeps outside its budget, and one extra
 *     query group (index Cq) that keeps every key; text rows are never probes
 *     and are not corrected. With text tokens the group counts below are
 *     Ckt = Ck + 1 and Cqt = Cq + 1, otherwise Ckt = Ck and Cqt = Cq.
 */
#ifndef SPARSEPR_H_
#define SPARSEPR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPARSEPR_MAX_HEADS 256

typedef enum {
  SPARSEPR_OK = 0,
  SPARSEPR_ERR_INVALID_ARG = 1, /* null pointer, inconsistent sizes, bad parameter */
  SPARSEPR_ERR_UNSUPPORTED = 2, /* valid but not built: head dim, dtype, text tokens */
  SPARSEPR_ERR_WORKSPACE = 3,   /* ws smaller than sparsepr_workspace_bytes() or misaligned */
  SPARSEPR_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  SPARSEPR_ERR_TIMEOUT = 5,     /* device status: a bounded wait ran out */
  SPARSEPR_ERR_NUMERIC = 6      /* device status: empty kept set or non-finite value */
} sparsepr_status;

typedef enum { SPARSEPR_BF16 = 0, SPARSEPR_F32 = 1 } sparsepr_dtype;

/* Partition computed by sparsepr_partition (sparsepr_params.partition).
 *   RESPONSE  [SPR 2.A]: keys by k-means on their response coordinates in
 *             the eigenbasis of M_K, then queries by k-means on their logit
 *             profiles against the K/V group means (the method).
 *   SEMANTIC  [SPR 4, ablations: the comparison partition]: keys and queries
 *             each by plain Euclidean k-means on their own rows, no coupling.
 *   COCLUSTER ["Attention Sparsity is Input-Stable", online bidirectional
 *             QK co-clustering]: rounds that assign each key to the key block
 *             whose mean affinity vector (scale * k . query centres) is
 *             nearest, update the key centres, then do the same for the
 *             queries against the new key centres.
 * All three use the same initial rows (partial Fisher-Yates draws), pass cap
 * (kmeans_iters), lowest-index ties and empty-group rule (the group keeps its
 * centre). */
typedef enum {
  SPARSEPR_PARTITION_RESPONSE = 0,
  SPARSEPR_PARTITION_SEMANTIC = 1,
  SPARSEPR_PARTITION_COCLUSTER = 2
} sparsepr_partition_mode;

/* Method parameters, passed by const pointer; the callee copies what it
 * needs before returning. */
typedef struct {
  int32_t H;            /* heads, 1..SPARSEPR_MAX_HEADS */
  int32_t N;            /* tokens per head (video tokens + n_text) */
  int32_t d;            /* head dim: 64 or 128 */
  int32_t n_text;       /* trailing text tokens (0 <= n_text < N) */
  int32_t Ck;           /* key (K/V) groups, 1..min(Nv, 4096) */
  int32_t Cq;           /* query groups, 1..min(Nv, 4096) */
  int32_t Ms;           /* sampled queries for M_K, 1..Nv */
  int32_t n_eig;        /* eigenvectors e of M_K used as key coordinates, 1..min(d,32) */
  int32_t kmeans_iters; /* cap on k-means assignment passes (stops early when labels repeat) */
  int32_t M;            /* probe rows per head, 0..Nv */
  int32_t r;            /* rank of the residual subspace, 1..d */
  int32_t partition;    /* SPARSEPR_PARTITION_*: 0 (the default) is the method's
                           response-coupled partition */
  double lambda;        /* ridge penalty, >= 0 */
  double scale;         /* softmax scale; 0 selects 1/sqrt(d) */
  uint64_t seed;        /* k-means initialisation seed */
  const double* keep;   /* HOST array [H]: kept fraction of key groups per head, (0, 1] */
} sparsepr_params;

/* Device statistics of the last attention call, copied out by
 * sparsepr_read_stats. */
typedef struct {
  uint32_t status;       /* OR of (1 << sparsepr_status) device-detected errors; 0 = fine */
  int32_t H;
  int32_t key_passes[SPARSEPR_MAX_HEADS];   /* k-means assignment passes run per head */
  int32_t query_passes[SPARSEPR_MAX_HEADS];
  int64_t pairs_sparse[SPARSEPR_MAX_HEADS]; /* routed (row, key) pairs per head */
  int64_t pairs_exec[SPARSEPR_MAX_HEADS];   /* pairs_sparse + M*N (probe rows) */
  int64_t recheck_rows[2]; /* k-means rows decided again in fp64 (keys, queries), all passes */
  int32_t eig_sweeps[2];   /* Jacobi sweeps, max over heads: [1] = probe residual Gram when r > 64 (the tridiagonal solver serves r <= 64 and M_K, and leaves 0) */
  int64_t near_ties[2];    /* k-means rows (keys, queries), summed over heads and passes, whose
                              two smallest fp64 squared distances d1 <= d2 satisfy
                              d2 - d1 <= 1e-12 d2: their label is decided by the lowest-index
                              rule or by rounding, not by the data (expected 0 on generic data;
                              exact ties such as two identical centroids count) */
} sparsepr_stats;

/* Bytes of device workspace the five calls need for these parameters
 * (0 if the parameters are invalid). */
size_t sparsepr_workspace_bytes(const sparsepr_params* p);

/* Human-readable name of a status code (static string). */
const char* sparsepr_status_string(sparsepr_status s);

/* Stage 1 [SPR 2.A, response-coupled partitioning].
 * Keys: M_K = Q_s^T Q_s / Ms from Ms strided sampled queries; top-n_eig
 * eigenpairs (U, L) of M_K; key coordinates z = L^{1/2} U^T k; Lloyd k-means
 * into Ck groups (lowest index on ties, empty groups keep their centroid,
 * at most kmeans_iters passes, stop when labels repeat).
 * Queries: logit profiles p = scale * C_K q against the K/V group centroids
 * C_K (original-space means); Lloyd k-means into Cq groups, evaluated in the
 * exact d-space form (q - qbar)^T G (q - qbar), G = scale^2 C_K^T C_K.
 * Initial centroids: rows chosen by a partial Fisher-Yates shuffle driven by
 * SplitMix64 seeded with seed ^ (2*head + {0 keys, 1 queries}).
 *   q, k      [H, N, d] input dtype (device, read only)
 *   label_q   [H, N] int32 out: query group of each token, 0..Cqt-1
 *   label_k   [H, N] int32 out: key group of each token, 0..Ckt-1
 *             (text tokens: Cq and Ck) */
sparsepr_status sparsepr_partition(const void* q, const void* k, sparsepr_dtype dt,
                                   const sparsepr_params* p, int32_t* label_q,
                                   int32_t* label_k, void* ws, size_t ws_bytes,
                                   void* stream);

/* Stage 2 [SPR 2.C, contiguous group-major layout].
 * Stable counting sort of the tokens by group: perm[h, i] is the token at
 * group-major row i (ascending token order inside a group); off[h, c] is
 * the first row of group c (off[h, C] = N). qp = q[perm_q], kp = k[perm_k],
 * vp = v[perm_k] (K and V share the key partition).
 *   label_q, label_k   [H, N] int32 in (values must lie in 0..Cqt-1 / 0..Ckt-1)
 *   perm_q, perm_k     [H, N] int32 out
 *   off_q [H, Cqt+1], off_k [H, Ckt+1] int32 out
 *   qp, kp, vp         [H, N, d] input dtype out (must not alias q, k, v) */
sparsepr_status sparsepr_permute(const void* q, const void* k, const void* v,
                                 sparsepr_dtype dt, const sparsepr_params* p,
                                 const int32_t* label_q, const int32_t* label_k,
                                 int32_t* perm_q, int32_t* perm_k, int32_t* off_q,
                                 int32_t* off_k, void* qp, void* kp, void* vp,
                                 void* ws, size_t ws_bytes, void* stream);

/* Stage 3a [SVOO block selection].
 * Block scores A[g, c] = scale * C_Q[g] . C_K[c] in fp64 from the group mean
 * rows of qp / kp (zero vector for an empty group); each query group keeps
 * its top-k_h key groups, ties to the lowest index, listed ascending. Only
 * the Cq x Ck video groups are routed (off_q, off_k as from sparsepr_permute,
 * Cqt + 1 / Ckt + 1 entries per head).
 * k_h = max(1, min(Ck, ceil(keep[h] * Ck - 1e-9))).
 *   csr         [H, Cq, kmax] int32 out, kmax = max_h k_h; entries past
 *               k_h are -1
 *   k_per_head  [H] int32 out */
sparsepr_status sparsepr_route(const void* qp, const void* kp, sparsepr_dtype dt,
                               const sparsepr_params* p, const int32_t* off_q,
                               const int32_t* off_k, int32_t* csr,
                               int32_t* k_per_head, void* ws, size_t ws_bytes,
                               void* stream);

/* Largest k_h of sparsepr_route for these parameters (the csr row width),
 * or -1 if the parameters are invalid. */
int32_t sparsepr_route_width(const sparsepr_params* p);

/* sparsepr_route without a workspace, for callers that cannot allocate
 * device memory or pass a workspace (code that must not trigger the implicit
 * device synchronisation of cudaMalloc, or that works inside a memory pool
 * reserved up front). No counterpart in the paper: it is a memory-management
 * variant of the routing call above, with the same arguments (minus ws), the
 * same kernels and therefore the same routes, bit for bit.
 * Its scratch is one fixed 8 MiB device array per GPU, held until the
 * process exits. Under CUDA's default lazy module loading the array is
 * committed by the first call on each device (that call may allocate and
 * synchronise); with eager loading (CUDA_MODULE_LOADING=EAGER) it is
 * committed when the library is loaded. Heads are processed in chunks that
 * fit: a single head needs ((Cq + Ck) * d + Cq * Ck) * 8 bytes, and larger
 * parameters are rejected with SPARSEPR_ERR_WORKSPACE before anything is
 * enqueued. It calls no allocating routine.
 * The first call on each device looks up the array's device address with
 * that device current; make that first call before any stream capture.
 * All calls share the array and the last call's contents stay in it (every
 * call overwrites what it reads, nothing needs clearing). Calls that overlap
 * on the GPU race on the array: issue them in order on one stream.
 * qp and kp must be 16-byte aligned (SPARSEPR_ERR_INVALID_ARG otherwise). */
sparsepr_status sparsepr_route_noalloc(const void* qp, const void* kp, sparsepr_dtype dt,
                                       const sparsepr_params* p, const int32_t* off_q,
                                       const int32_t* off_k, int32_t* csr,
                                       int32_t* k_per_head, void* stream);

/* Stage 3b [SPR 2.C variable-block sparse attention; SVOO: the softmax is
 * normalised over the kept logits only].
 * For group-major query row i of group g:
 *   o_sparse[i] = sum_{j in S(g)} softmax_{S(g)}(scale * qp_i . kp_j) vp_j,
 * S(g) = union of the key ranges off_k[c]..off_k[c+1] of the kept groups c
 * in csr[g] (plus the text key group when n_text > 0; the text query group
 * keeps every key). Skipped key groups are never multiplied. bf16
 * tensor-core MMAs (tcgen05, fp32 accumulation in tensor memory).
 *   o_sparse      [H, N, d] fp32 out, group-major row order
 *   pairs_sparse  [H] int64 out: sum_g n_g * |S(g)| (exact pair count)
 * A query group whose kept set is empty raises SPARSEPR_ERR_NUMERIC in the
 * status word and its rows are written as 0. */
sparsepr_status sparsepr_block_sparse_attn(const void* qp, const void* kp, const void* vp,
                                           sparsepr_dtype dt, const sparsepr_params* p,
                                           const int32_t* off_q, const int32_t* off_k,
                                           const int32_t* csr, const int32_t* k_per_head,
                                           float* o_sparse, int64_t* pairs_sparse,
                                           void* ws, size_t ws_bytes, void* stream);

/* Stage 4 [SPR 2.B, probe-fitted residual reconstruction].
 * Probes: m_g rows of query group g, m_g proportional to the group size by
 * largest remainder (ties to the lower group, sum M), at group-major offsets
 * floor((t + 1/2) n_g / m_g). O_dense of the probe rows is exact softmax
 * attention over all N keys; R = O_dense - O_sparse on the probes.
 * Ridge fit (fp64, intercept unpenalised): B = (Xc^T Xc + lambda I)^{-1}
 * Xc^T Rc, b = rbar - xbar B with X = O_sparse[probes]. Subspace: V_r = top-r
 * right singular vectors of R; B' = B V_r V_r^T, b' = b V_r V_r^T.
 * Output: out[perm_q[i]] = O_dense(i) for probe rows, o_sparse[i] for text
 * rows, else o_sparse[i] + b' + o_sparse[i] B', rounded to the input dtype
 * (RNE). Probes are drawn from the Cq video query groups only.
 *   perm_q         [H, N] int32 in (from sparsepr_permute)
 *   o_sparse       [H, N, d] fp32 in (from sparsepr_block_sparse_attn)
 *   pairs_sparse   [H] int64 in
 *   out            [H, N, d] input dtype out, ORIGINAL token order
 *   probes         [H, M] int32 out: group-major probe rows, ascending
 *   pairs_exec     [H] int64 out: pairs_sparse + M * N
 *   fit            [H, d*d + d] fp64 out, optional (NULL = skip): B' row-major
 *                  then b' */
sparsepr_status sparsepr_probe_correct(const void* qp, const void* kp, const void* vp,
                                       sparsepr_dtype dt, const sparsepr_params* p,
                                       const int32_t* off_q, const int32_t* perm_q,
                                       const float* o_sparse, const int64_t* pairs_sparse,
                                       void* out, int32_t* probes, int64_t* pairs_exec,
                                       double* fit, void* ws, size_t ws_bytes,
                                       void* stream);

/* Buffers of sparsepr_attention: every output of the five calls, with the
 * shapes and types given there (caller-owned device memory). fit may be
 * NULL; probes may be NULL when M = 0. */
typedef struct {
  int32_t* label_q;       /* [H, N] */
  int32_t* label_k;       /* [H, N] */
  int32_t* perm_q;        /* [H, N] */
  int32_t* perm_k;        /* [H, N] */
  int32_t* off_q;         /* [H, Cq + 1 (+1 with text)] */
  int32_t* off_k;         /* [H, Ck + 1 (+1 with text)] */
  void* qp;               /* [H, N, d] input dtype: permuted Q, K, V */
  void* kp;
  void* vp;
  int32_t* csr;           /* [H, Cq, sparsepr_route_width(p)] */
  int32_t* k_per_head;    /* [H] */
  float* o_sparse;        /* [H, N, d] fp32 */
  int64_t* pairs_sparse;  /* [H] */
  int32_t* probes;        /* [H, M] */
  int64_t* pairs_exec;    /* [H] */
  double* fit;            /* [H, d*d + d] or NULL */
} sparsepr_call_buffers;

/* The whole call [SPR 2.A-2.C] in one entry point: sparsepr_partition,
 * sparsepr_permute and sparsepr_route as above, then the attention of all
 * rows while the probe fit of stage 4 runs beside it on a second stream. The
 * probe rows' dense outputs and their sparse outputs X come from one pass
 * over all keys (for X each probe row's keys are limited to its query
 * group's kept runs, with the same masking and fp32 arithmetic as
 * sparsepr_block_sparse_attn, taken over the key tiles in another order);
 * then come the ridge fit and the residual subspace, and only the correction
 * waits for both. The overlap is taken while that extra pass is cheaper than
 * the fit latency it hides (4 d H M N < 4e11 flop); wider calls run the
 * probe rows after the attention of all rows, as the five calls do (X =
 * o_sparse at the probe rows). Outputs are those of the five calls; integer
 * outputs (labels, permutations, offsets, routes, pair counts, probes) are
 * identical to theirs, and X, hence fit and out, may differ from theirs in
 * the rounding of fp32 sums. q, k, v [H, N, d] in the dtype dt; out
 * [H, N, d] dt, original token order. Errors: those of the five calls (no
 * work is enqueued after a host-side error). */
sparsepr_status sparsepr_attention(const void* q, const void* k, const void* v, sparsepr_dtype dt,
                                   const sparsepr_params* p, const sparsepr_call_buffers* b,
                                   void* out, void* ws, size_t ws_bytes, void* stream);

/* Where a stage's intermediate results sit inside `ws`, for stage-level
 * tests and debugging (the workspace layout depends only on the
 * parameters): the byte offset and size of the named region. Contents
 * (row-major) after the call that writes them, until a later call reuses the
 * region:
 *   written by sparsepr_partition [SPR 2.A]:
 *     "init_k" [H, Ck] int32, "init_q" [H, Cq] int32: initial centroid rows
 *             (partial Fisher-Yates draws, token indices of the video tokens)
 *     "mk"     [H, d, d] fp64: M_K = Q_s^T Q_s / M_s
 *     "eval"   [H, n_eig] fp64: the leading eigenvalues of M_K, descending
 *     "evec"   [H, d, n_eig] fp64: their unit eigenvectors as columns (the
 *             sign of each column is arbitrary)
 *     "wk"     [H, d, n_eig] fp64: key projector U_e Lambda_e^{1/2}
 *     "z"      [H, Nv, n_eig] fp64: key response coordinates z_j = W_K^T k_j
 *     "ck"     [H, Ck, d] fp64: K group means in the original space over the
 *             final key labels (the zero vector for an empty group)
 *     "g"      [H, d, d] fp64: query metric G = scale^2 C_K^T C_K
 *     "zplanes" [3, H, Nv, Dp] bf16 (Dp = 16 for n_eig <= 16, else 64): z
 *             split into three bf16 planes (each the rounding of what the
 *             planes before it leave of z; zero padded to Dp columns), the
 *             operands of the tensor-core key assignment
 *     "xnk"    [H, Nv] fp32: |z_j| rounded up, for the assignment's bound
 *   written by sparsepr_probe_correct [SPR 2.B] (M > 0; it also reuses
 *   "mk", "eval" and "evec" for R^T R and its eigenpairs):
 *     "bmat"   [H, d, d] fp64, "bvec" [H, d] fp64: the ridge solution B, b
 *             before the subspace projection
 *     "xr"     [H, 2, M, d] fp64: X = O_sparse of the probe rows, then
 *             R = O_dense - X
 *     "vr"     [H, d, r] fp64: the leading r right singular vectors of R (columns)
 * Errors: INVALID_ARG for invalid parameters, a NULL pointer or an unknown
 * name; UNSUPPORTED as sparsepr_workspace_bytes. Host only, enqueues nothing. */
sparsepr_status sparsepr_workspace_region(const sparsepr_params* p, const char* name,
                                          size_t* offset, size_t* bytes);

/* Structural diagnostics of the probe rows [SPR 3, structural analysis:
 * retained attention mass does not bound the post-softmax error, and the
 * partition's geometry decides how much of the residual is affine-
 * explainable; SPR 4, ablations: orthogonal residual energy]. Call after
 * sparsepr_probe_correct with the same parameters and `ws` (M > 0), before
 * the workspace is reused; `probes` as written by that call.
 *   mass    [H, M] fp64 out: dense softmax mass of probe row t on the keys its
 *           query group keeps, sum over kept keys of softmax(scale q.k) over
 *           all N keys (from the log-sum-exps of the sparse and dense passes)
 *   error   [H, M] fp64 out: ||O_dense - O_sparse||_2 of probe row t
 *   energy  [H, 4] fp64 out, over the probe rows with R = O_dense - O_sparse,
 *           X = O_sparse, the fitted map F = b + X B and P_r = V_r V_r^T:
 *           { ||R||_F^2, ||R P_r||^2 / ||R||^2 (explainable share),
 *             ||R - F||^2 / ||R||^2, ||R - F P_r||^2 / ||R||^2 } (a zero R gives
 *           {0, 1, 0, 0})
 * Errors: INVALID_ARG for M = 0 or a NULL pointer; UNSUPPORTED for r > 64. */
sparsepr_status sparsepr_probe_diagnostics(const sparsepr_params* p, const int32_t* probes,
                                           double* mass, double* error, double* energy,
                                           void* ws, size_t ws_bytes, void* stream);

/* Support expansion of a shared route [SPR 3, structural analysis: the
 * support that the rows of a query group need together is several times the
 * support each needs alone]. For every group_stride-th video query group g
 * of a permuted call (qp, kp, off_q, off_k as from sparsepr_permute): a row's
 * individual support at mass tau is the smallest set of key groups (the text
 * key group, when present, counts as one) whose dense softmax mass reaches
 * tau (within 1e-15), taken by decreasing mass with ties to the lower index,
 * from the row's scaled logits over all N keys in fp64; the group's
 * aggregate support is the union of its rows' supports.
 *   individual [H, Cq] fp64 out: mean individual support size of the group's
 *              rows (0 for an empty group; NaN for a group not sampled)
 *   aggregate  [H, Cq] fp64 out: size of the union (NaN when not sampled)
 * Cost: 2 N d fp64 FMA per sampled row. Uses the diagnostics scratch of `ws`;
 * call it after the attention call. Errors: INVALID_ARG for tau outside
 * (0, 1], group_stride < 1, NULL or misaligned pointers; UNSUPPORTED when
 * the key-group count does not fit one CTA's shared memory. */
sparsepr_status sparsepr_support_expansion(const void* qp, const void* kp, sparsepr_dtype dt,
                                           const sparsepr_params* p, const int32_t* off_q,
                                           const int32_t* off_k, double tau, int32_t group_stride,
                                           double* individual, double* aggregate, void* ws,
                                           size_t ws_bytes, void* stream);

/* Per-head attention density ["Attention Sparsity is Input-Stable", offline
 * layer-wise sparsity profiling: the share of attention weights a head needs
 * for a mass tau]. For every row_stride-th video row i of q (original token
 * order): n_i = the smallest number of row i's N softmax weights over k,
 * largest first, whose sum reaches tau (within 1e-15), from fp64 logits;
 *   density [H] fp64 out: mean over the sampled rows of n_i / N
 * (1 - density is the head's sparsity at tau; fitting it over calibration
 * inputs is the caller's). Cost: N d fp64 FMA per sampled row. Uses the
 * diagnostics scratch of `ws`. Errors as sparsepr_support_expansion. */
sparsepr_status sparsepr_density_profile(const void* q, const void* k, sparsepr_dtype dt,
                                         const sparsepr_params* p, double tau, int32_t row_stride,
                                         double* density, void* ws, size_t ws_bytes,
                                         void* stream);

/* Copy the device statistics of the last call out of `ws` (a blocking
 * device-to-host copy; call after the stream has been synchronised). */
sparsepr_status sparsepr_read_stats(const void* ws, sparsepr_stats* out);

/* Zero the status word and statistics in `ws` (enqueued on `stream`).
 * sparsepr_partition does this itself at the start of every call. */
sparsepr_status sparsepr_reset_stats(void* ws, void* stream);

/* Check of the device-side failure path, for tests and health checks: one
 * kernel whose thread waits, through the same bounded mbarrier wait as every
 * kernel of the library, on a barrier that nothing completes. After the wait
 * limit (2 s) the wait gives up, SPARSEPR_ERR_TIMEOUT is OR-ed into the status
 * word of `ws` and the kernel returns; the device and the CUDA context stay
 * usable. Enqueued on `stream`; read the result with sparsepr_read_stats after
 * synchronising. Errors: INVALID_ARG for a NULL or not 256-byte-aligned `ws`,
 * CUDA for a failed launch. */
sparsepr_status sparsepr_check_wait_limit(void* ws, void* stream);

/* Check of the reciprocal the eigenvalue multisection uses in its Sturm
 * counts (Golub & Van Loan, Matrix Computations, sec. 8.4.1): the PTX
 * approximate reciprocal refined by two Newton-Raphson steps, which is not
 * correctly rounded. For n device doubles x (finite, nonzero, of normal
 * magnitude) it writes to the device array err[n] the distance of that
 * reciprocal from the correctly rounded 1/x, in units of the last place of
 * the latter. Enqueued on `stream`. Errors: INVALID_ARG for n < 0 or a NULL
 * array with n > 0, CUDA for a failed launch. */
sparsepr_status sparsepr_check_reciprocal(const double* x, int64_t n, double* err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEPR_H_ */
