// Host-side launchers of the SparsePR kernels (one translation unit per
// stage); called by the C-ABI layer in api.cu. Every launcher enqueues on
// `st` and returns cudaGetLastError().
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.h"

namespace spr {

// cuTensorMapEncodeTiled, fetched once through the runtime's driver entry point
// (null if the driver does not provide it).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// ---- sort.cu: stable counting sort of per-head labels ----------------------
// labels [H, n] in 0..C-1 -> perm [H, n] (group-major order, ascending token
// index inside a group) and off [H, C+1]. Heads with skip[h] != 0 are left
// untouched (skip may be null).
cudaError_t launch_counting_sort(const int32_t* labels, int H, int n, int C, int nchunk,
                                 int32_t* hist, int32_t* perm, int32_t* off,
                                 const int32_t* skip, int skip_stride, DeviceStats* stats,
                                 cudaStream_t st);

// ---- partition.cu ----------------------------------------------------------
cudaError_t launch_fy_init(int H, int Nv, int Ck, int Cq, uint64_t seed, int32_t* init_k,
                           int32_t* init_q, cudaStream_t st);
// Gram matrices in fp64. A Gram over S rows is split into up to kGramSplits
// ranges of rows (CTAs of their own); their partial sums go to `part`
// ([kGramJobs, H, kGramSplits, d, d] fp64 scratch) and a second kernel adds
// them in range order, so results do not depend on scheduling.
// out[h] = (1 / Ms) * sum_s x_s x_s^T over the Ms strided sampled query rows.
cudaError_t launch_metric_mk(const void* q, bool bf16, int H, int N, int Nv, int d, int Ms,
                             double* out, double* part, cudaStream_t st);
// out[h] = factor * sum_s (x_s - xm)(y_s - ym)^T + diag * I over S fp64 rows;
// xm / ym (may be null) advance by mean_stride per head.
struct GramJob {
  const double *X, *Y, *xm, *ym;
  long long hsx, hsy, ms;  // per-head strides of X, Y and the means
  double* out;
  long long os;            // per-head stride of out
  double factor, diag;
};
// Up to kGramJobs Grams over the same S rows (row stride ld) in one launch.
struct GramJobs {
  GramJob job[kGramJobs];
  int njobs, ld, S, d, H;
  double* part;  // partial sums (set by the caller)
  int splits;    // set by the launcher
};
cudaError_t launch_gram_f64(GramJobs g, cudaStream_t st);
cudaError_t launch_gram_f64(const double* X, const double* Y, const double* xm,
                            const double* ym, long long head_stride_x, long long head_stride_y,
                            int ld, int S, int H, int d, double factor, double diag,
                            double* out, long long out_stride, long long mean_stride,
                            double* part, cudaStream_t st);
// z = k W_K; with zp given (e = 16, d a multiple of 8, k 16-byte aligned)
// also z's three bf16 planes (plane stride zps elements) and its row norms
// rounded up, as launch_split_rows forms them
cudaError_t launch_zproj(const void* k, bool bf16, int H, int N, int Nv, int d, int e,
                         const double* wk, double* z, __nv_bfloat16* zp, long long zps,
                         float* xnorm, cudaStream_t st);
// dst[h, c, :] = src[h, idx[h, c], :] (as fp64) and norms[h, c] = |dst|^2 (norms may be null)
cudaError_t launch_gather_init(const void* src, int src_kind, long long head_stride, int ld,
                               int D, const int32_t* idx, int C, int H, double* dst,
                               double* norms, cudaStream_t st);
// labels[h, i] = argmin_j (c[h, j] - 2 x_i . y[h, j]) (lowest j on ties);
// changes[h] += number of labels that differ from the previous value.
cudaError_t launch_argmin(const void* X, int x_kind, long long head_stride_x, int ldx, int n,
                          int D, const double* Y, const double* c, int m, int H,
                          int32_t* labels, int32_t* flags, int flag_base, const double* G,
                          DeviceStats* stats, cudaStream_t st);
cudaError_t launch_finalize_pass(int H, int pass, int32_t* flags, int flag_base,
                                 int32_t* passes_out, cudaStream_t st);
// out[h, c, :] = mean of the rows perm[off[c]..off[c+1]) of X (fp64 sums in
// ascending position order); empty group: keep (keep_prev) or zero.
// norms[h, c] = |out[h, c]|^2 if norms is non-null.
cudaError_t launch_group_mean(const void* X, int x_kind, long long head_stride_x, int ldx, int D,
                              const int32_t* perm, int perm_stride, const int32_t* off,
                              int off_stride, int C, int H, bool keep_prev, double* out,
                              double* norms, const int32_t* skip, int skip_stride,
                              cudaStream_t st);
cudaError_t launch_query_metric_apply(const double* G, const double* qbar, int Cq, int H, int d,
                                      double* wg, double* cg, const int32_t* skip,
                                      int skip_stride, cudaStream_t st);
cudaError_t launch_identity(double* G, int H, int d, cudaStream_t st);
cudaError_t launch_group_counts(const int32_t* off, int off_stride, int C, int H, int32_t* cnt,
                                cudaStream_t st);
cudaError_t launch_affinity_centres(const double* xbar, const double* C, int m1, int m2, int d,
                                    int H, double scale, const int32_t* cnt, bool first,
                                    double* pbar, cudaStream_t st);
cudaError_t launch_dspace_centres(const double* pbar, const double* C, int m1, int m2, int d,
                                  int H, double scale, double* y, double* c, cudaStream_t st);
cudaError_t launch_finalize_round(int H, int round, int32_t* flags, int32_t* passes_k,
                                  int32_t* passes_q, cudaStream_t st);
cudaError_t launch_write_labels(const int32_t* lab, int H, int N, int Nv, int C_text,
                                int32_t* out, cudaStream_t st);

// x_kind values
constexpr int kXf64 = 0;
constexpr int kXbf16 = 1;
constexpr int kXf32 = 2;

// ---- assign.cu: certified tensor-core nearest-centroid assignment ----------
struct AssignTC {
  const __nv_bfloat16* a_planes;  // [nA][a_rows_total][Dp]
  long long a_plane_stride;       // elements between planes
  size_t a_rows_total;
  int a_head;                     // rows between heads in the A planes
  int nA;
  const __nv_bfloat16* b_planes;  // [nB][H * Cpad][Dp]
  long long b_plane_stride;
  int nB;
  int Dp;                         // 16 (32-byte rows) or a multiple of 64
  int Cpad;                       // centroids per head padded to a multiple of 16
  int H, n;                       // heads, rows per head
  int npairs;
  int pairs[6];
  const float* cvals;             // [H, Cpad]
  const float* xnorm;             // [H, n]
  const float* hmax;              // [H, 2]
  int32_t* labels;                // [H, n]
  int32_t* flags;
  int flag_base;
  int32_t* recheck;               // [H, n]
  int32_t* nrecheck;              // [H]
  DeviceStats* stats;
  int sm_count;
  // exact operands for the fp64 decision of flagged rows
  const void* x_exact;
  int x_kind;
  long long x_hs;
  int x_ld;
  int D;
  const double* y_tr;             // [H, D, m] centroid side transposed (prep_centroids)
  const double* c_exact;          // [H, m] (unused when direct)
  int m;
  int direct;                     // 1: d = |x - y|^2, 0: d = c - 2 x.y
  const double* metric;           // [H, D, D] G of d = c - 2 x.y + x^T G x (near-tie count; direct: unused)
};
size_t assign_tc_smem_bytes(int nA, int nB, int Dp, int Cpad);
cudaError_t launch_split_rows(const void* X, int kind, long long hsx, int ldx, int n, int D,
                              int Dp, int P, int H, __nv_bfloat16* planes, long long plane_stride,
                              float* norms, cudaStream_t st);
cudaError_t launch_prep_centroids(const double* Y, const double* c, int m, int D, int Dp,
                                  int Cpad, int P, int H, __nv_bfloat16* planes,
                                  long long plane_stride, float* cf, float* hmax, double* ytr,
                                  const int32_t* flags, int flag_base, cudaStream_t st);
cudaError_t launch_argmin_tc(const AssignTC& a, cudaStream_t st);

// ---- linalg.cu -------------------------------------------------------------
// Cyclic-parallel Jacobi eigensolver, one CTA per head: A [H, d, d] fp64
// symmetric -> eval [H, d], evec [H, d, d] (eigenvectors in columns).
cudaError_t launch_jacobi(const double* A, int H, int d, double* eval, double* evec,
                          DeviceStats* stats, int which, cudaStream_t st);
// wk[h, a, t] = evec[h, a, j_t] (* sqrt(max(eval_j_t, 0)) if sqrt_scale) for
// the e largest eigenvalues (t = rank, ties to the lower index).
cudaError_t launch_top_eig_projector(const double* eval, const double* evec, int H, int d, int e,
                                     double* wk, bool sqrt_scale, cudaStream_t st);
// wk[h, a, t] = vecs[h, a, t] * sqrt(max(vals[h, t], 0)), t < e.
cudaError_t launch_scale_columns(const double* vals, const double* vecs, int H, int d, int e,
                                 double* wk, cudaStream_t st);

// ---- eigen.cu: top-ne eigenpairs (ne <= 64) by tridiagonal reduction,
// bisection and inverse iteration ---------------------------------------------
size_t sym_eigs_scratch_doubles(int H, int d);
// evals [H, ne] descending, evecs [H, d, ne].
// err[i]: distance in ulp of rcp_newton(x[i]) from the correctly rounded 1/x[i]
cudaError_t launch_check_reciprocal(const double* x, long long n, double* err, cudaStream_t st);
cudaError_t launch_sym_eigs(const double* A, int H, int d, int ne, double* evals, double* evecs,
                            double* scratch, cudaStream_t st);

// ---- permute.cu ------------------------------------------------------------
// dst = src gathered by `perm` (and dst2 = src2, the same rows, when src2 is
// given; both null otherwise)
cudaError_t launch_gather_rows(const void* src, void* dst, const void* src2, void* dst2,
                               const int32_t* perm, int H, int N, int d, int elem_bytes,
                               cudaStream_t st);
// Score GEMM + warp top-k, heads in groups whose scores fit in `scores`
// (route_scores_bytes(H, Cq, Ck) bytes in the workspace).
size_t route_scores_bytes(int H, int Cq, int Ck);
cudaError_t launch_route_gemm(const double* cq, const double* ckr, int H, int Cq, int Ck, int d,
                              double scale, const int32_t* kh, int kmax, double* scores,
                              size_t scores_bytes, int32_t* csr, cudaStream_t st);
// out[h, c] = mean of rows off[h, c]..off[h, c+1] (c < C; off rows of off_stride entries)
cudaError_t launch_range_mean(const void* X, int x_kind, int H, int N, int d, const int32_t* off,
                              int C, int off_stride, double* out, cudaStream_t st);
cudaError_t launch_write_k(const int32_t* kh_host_vals, int H, int32_t* k_per_head,
                           cudaStream_t st);

// ---- attn.cu ---------------------------------------------------------------
struct AttnArgs {
  const void* qp;   // bf16 [H*Nq_total rows, d] (row = h * q_rows + i)
  const void* kp;   // bf16 [H*N, d]
  const void* vp;   // bf16 [H*N, d]
  int H, N, d;
  int q_rows;       // rows per head of the query tensor
  int Cq, Ck;       // query groups per head (work list), key groups (with the text group)
  int text = 0;     // 1: the last query group (Cq - 1) is the text group and keeps every
                    // key; every other group also keeps the last key group (Ck - 1)
  const int32_t* off_q;  // [H, Cq+1]
  const int32_t* off_k;  // [H, Ck+1]
  const int32_t* csr;    // [H, Cq - text, kmax] routes of the (video) query groups
  const int32_t* kh;     // [H]
  int kmax;
  float scale;
  float* out;            // [H, q_rows, d] fp32
  int32_t* work;         // [H, tiles_per_head]
  int32_t* nwork;        // [H]
  int tiles_per_head;
  int32_t* nslots;       // [H, Cq]
  int2* runs;            // [H, Cq, kmax + 1] merged key runs (start, length)
  int32_t* nruns;        // [H, Cq]
  int64_t* pairs;        // [H] (may be null)
  DeviceStats* stats;
  // split of every unit's key tiles into `splits` contiguous ranges run by
  // separate CTAs (1: off). With splits > 1 each CTA writes its normalised
  // partial output and log2-sum-exp to opart [H, units, splits, 256, d] /
  // lpart [H, units, splits, 256] (units = partial-buffer units per head),
  // and a combine kernel writes `out`.
  int splits = 1;
  int units = 0;
  float* opart = nullptr;
  float* lpart = nullptr;
  // log2-sum-exp of every row's scaled logits over its kept keys (log2
  // units: m + log2 l), [H, q_rows]; may be null
  float* lse = nullptr;
  // dual probe pass (dense routes, units of 128 rows): every row is computed
  // twice over all keys, once densely (out, lse, opart, lpart) and once with
  // its keys limited to the kept runs of its query group pgrp[h, row] in the
  // routed pass's run lists gruns [H, gCq, gkmax + 1] / gnruns [H, gCq]
  // (out2, lse2, opart2, lpart2; partial buffers with 128-row units)
  int dual = 0;
  float* out2 = nullptr;
  float* lse2 = nullptr;
  float* opart2 = nullptr;
  float* lpart2 = nullptr;
  const int32_t* pgrp = nullptr;
  const int2* gruns = nullptr;
  const int32_t* gnruns = nullptr;
  int gCq = 0, gkmax = 0;
};
// the work list and the slot / run / pair metadata of a pass
cudaError_t launch_attn_meta(const AttnArgs& a, cudaStream_t st);
// the attention kernel (and split-KV combine) over metadata already formed
cudaError_t launch_attn_kernel(const AttnArgs& a, cudaStream_t st);
// both, in order
cudaError_t launch_block_sparse_attn(const AttnArgs& a, cudaStream_t st);
cudaError_t launch_cast_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t st);

// ---- diag.cu ---------------------------------------------------------------
cudaError_t launch_probe_diagnostics(const int32_t* probes, const float* lse_s, const float* lse_d,
                                     const double* xr, const double* bmat, const double* bvec,
                                     const double* vr, int H, int N, int M, int d, int r,
                                     double* mass, double* err, double* energy_rows,
                                     double* energy, cudaStream_t st);

cudaError_t launch_support_expansion(const void* qp, const void* kp, bool bf16,
                                     const int32_t* off_q, int oq_stride, const int32_t* off_k,
                                     int Ckt, int H, int N, int d, int Cqv, int stride,
                                     double scale, double tau, uint32_t* union_bits,
                                     unsigned long long* size_sum, double* indiv,
                                     double* aggregate, cudaStream_t st);
size_t support_smem_bytes(int Ckt, int d, int* R, int* P);
cudaError_t launch_density(const void* q, const void* k, bool bf16, int H, int N, int Nv, int d,
                           int row_stride, double scale, double tau, double* scratch,
                           unsigned long long* count_sum, double* density, cudaStream_t st);

// ---- fit.cu ----------------------------------------------------------------
// probes [H, M]; pgrp [H, M] (may be null): the query group of each probe
cudaError_t launch_probe_select(const int32_t* off_q, int off_stride, int H, int Cq, int M,
                                int32_t* probes, int32_t* pgrp, cudaStream_t st);
cudaError_t launch_gather_probe_rows(const void* qp, bool bf16, const int32_t* probes, int H,
                                     int N, int M, int d, __nv_bfloat16* dst, cudaStream_t st);
// X from o_sparse at the probe rows, or from x_rows [H, M, d] when not null;
// part: scratch of part_doubles fp64 for per-block column sums.
cudaError_t launch_probe_residuals(const float* o_sparse, const float* x_rows, const float* od,
                                   const int32_t* probes, int H, int N, int M, int d, double* xr,
                                   double* means, double* part, size_t part_doubles,
                                   cudaStream_t st);
cudaError_t launch_ridge_solve(double* gram, int H, int d, double* bmat, double* bvec,
                               const double* means, DeviceStats* stats, cudaStream_t st);
// B' = (B V_r) V_r^T, b' = (b V_r) V_r^T with vr [H, d, r]; bp32 holds B'^T
// ([H, column, row]), fit_out (optional) B' row-major and b' in fp64.
cudaError_t launch_project_map(const double* bmat, const double* bvec, const double* vr, int H,
                               int d, int r, float* bp32, float* bv32, double* fit_out,
                               cudaStream_t st);
// ---- correct.cu: tensor-core residual correction ---------------------------
bool correct_tc_supported(int H, int N, int d);
// out[perm_q[i]] = od[probe] for probe rows, else x + x B' + b' (bpT = B'^T).
// Rows >= n_corr (text tokens) are copied uncorrected.
cudaError_t launch_correct_tc(const float* o_sparse, const float* od, const int32_t* probes,
                              const int32_t* perm_q, const float* bpT, const float* bv32, int H,
                              int N, int n_corr, int M, int d, void* out, bool out_bf16,
                              int sm_count, DeviceStats* stats, cudaStream_t st);
cudaError_t launch_correct(const float* o_sparse, const float* od, const int32_t* probes,
                           const int32_t* perm_q, const float* bp32, const float* bv32, int H,
                           int N, int n_corr, int M, int d, void* out, bool out_bf16,
                           cudaStream_t st);
cudaError_t launch_pairs_exec(const int64_t* pairs_sparse, int H, int64_t add, int64_t* pairs_exec,
                              DeviceStats* stats, cudaStream_t st);

}  // namespace spr
