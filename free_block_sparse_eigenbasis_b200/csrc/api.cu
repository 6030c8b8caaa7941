// C ABI of the SparsePR library: argument checks, workspace carving and the
// per-stage launch sequences. Declarations and the contract of every entry
// point are in include/sparsepr.h.
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

using namespace spr;

namespace {

struct Ctx {
  sparsepr_params p;
  Layout L;
  cudaStream_t st;
  DeviceStats* stats;
  double scale;
  bool bf16;
  int kind;
};

bool finite_nonneg(double x) { return isfinite(x) && x >= 0.0; }

// Tensor rows are read with 16-byte vector loads and TMA: every tensor
// pointer must be 16-byte aligned.
inline bool al16(const void* a) { return (reinterpret_cast<uintptr_t>(a) & 15) == 0; }
template <typename... Ts>
inline bool al16(const void* a, Ts... rest) { return al16(a) && al16(rest...); }

sparsepr_status check_params(const sparsepr_params* p) {
  if (!p || !p->keep) return SPARSEPR_ERR_INVALID_ARG;
  if (p->H < 1 || p->H > SPARSEPR_MAX_HEADS) return SPARSEPR_ERR_INVALID_ARG;
  if (p->n_text < 0 || p->N < 16) return SPARSEPR_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return SPARSEPR_ERR_UNSUPPORTED;
  const long long Nv = static_cast<long long>(p->N) - p->n_text;
  if (Nv < 1) return SPARSEPR_ERR_INVALID_ARG;
  if (static_cast<long long>(p->H) * p->N >= (1LL << 31)) return SPARSEPR_ERR_UNSUPPORTED;
  if (p->Ck < 1 || p->Ck > Nv || p->Ck > kMaxGroups) return SPARSEPR_ERR_INVALID_ARG;
  if (p->Cq < 1 || p->Cq > Nv || p->Cq > kMaxGroups) return SPARSEPR_ERR_INVALID_ARG;
  if (p->Ms < 1 || p->Ms > Nv) return SPARSEPR_ERR_INVALID_ARG;
  if (p->n_eig < 1 || p->n_eig > p->d || p->n_eig > 32) return SPARSEPR_ERR_INVALID_ARG;
  if (p->kmeans_iters < 1 || p->kmeans_iters > 1000) return SPARSEPR_ERR_INVALID_ARG;
  if (p->M < 0 || p->M > Nv) return SPARSEPR_ERR_INVALID_ARG;
  if (p->r < 1 || p->r > p->d) return SPARSEPR_ERR_INVALID_ARG;
  if (p->partition < SPARSEPR_PARTITION_RESPONSE || p->partition > SPARSEPR_PARTITION_COCLUSTER)
    return SPARSEPR_ERR_INVALID_ARG;
  if (!finite_nonneg(p->lambda) || !finite_nonneg(p->scale)) return SPARSEPR_ERR_INVALID_ARG;
  for (int h = 0; h < p->H; ++h)
    if (!(p->keep[h] > 0.0 && p->keep[h] <= 1.0)) return SPARSEPR_ERR_INVALID_ARG;
  return SPARSEPR_OK;
}

sparsepr_status setup(Ctx* c, const sparsepr_params* p, sparsepr_dtype dt, void* ws,
                      size_t ws_bytes, void* stream) {
  sparsepr_status s = check_params(p);
  if (s != SPARSEPR_OK) return s;
  if (dt != SPARSEPR_BF16 && dt != SPARSEPR_F32) return SPARSEPR_ERR_UNSUPPORTED;
  c->p = *p;
  compute_layout(c->p, &c->L);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) != 0 || ws_bytes < c->L.total)
    return SPARSEPR_ERR_WORKSPACE;
  c->st = static_cast<cudaStream_t>(stream);
  c->stats = at<DeviceStats>(ws, c->L.stats);
  c->scale = p->scale > 0.0 ? p->scale : 1.0 / sqrt(static_cast<double>(p->d));
  c->bf16 = (dt == SPARSEPR_BF16);
  c->kind = c->bf16 ? kXbf16 : kXf32;
  return SPARSEPR_OK;
}

sparsepr_status cuda_status(cudaError_t e) {
  return e == cudaSuccess ? SPARSEPR_OK : SPARSEPR_ERR_CUDA;
}

#define SPR_TRY(expr)                                \
  do {                                               \
    cudaError_t _e = (expr);                         \
    if (_e != cudaSuccess) return SPARSEPR_ERR_CUDA; \
  } while (0)

__global__ void set_i32_kernel(int32_t* p, int v) { *p = v; }


// Side streams per device for independent work beside the caller's stream:
// stream 0 for small kernels that occupy few SMs (the Fisher-Yates init
// beside the M_K eigen solve, the ridge solve beside the residual eigen
// solve) and, in sparsepr_attention, for the probe rows and the fit beside
// the attention of all rows; stream 1 for the ridge solve inside that probe
// branch. They are created with the highest priority, so that their
// latency-bound kernels take SMs as soon as blocks of the caller's kernels
// retire. Each forks from and joins its parent stream through events, so a
// stream capture of the caller's stream follows it. The streams and events
// are created by the first call on a device (make that call before
// capturing); `g_side_mu` is held from fork to join so that concurrent
// callers do not interleave the event records.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
SideStream g_side[64][2];

SideStream* side_stream(int which = 0) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream& ss = g_side[dev][which];
  if (!ss.s) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) greatest = 0;
    if (cudaStreamCreateWithPriority(&ss.s, cudaStreamNonBlocking, greatest) != cudaSuccess) {
      ss.s = nullptr;
      return nullptr;
    }
    if (cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
  }
  return &ss;
}

// fork: work enqueued on the returned stream runs beside `st` (st itself if
// no side stream could be made); join: `st` waits for it.
cudaStream_t fork_side(SideStream* ss, cudaStream_t st) {
  if (!ss) return st;
  if (cudaEventRecord(ss->fork, st) != cudaSuccess || cudaStreamWaitEvent(ss->s, ss->fork, 0) != cudaSuccess)
    return st;
  return ss->s;
}
cudaError_t join_side(SideStream* ss, cudaStream_t side, cudaStream_t st) {
  if (!ss || side == st) return cudaSuccess;
  cudaError_t e = cudaEventRecord(ss->join, side);
  if (e != cudaSuccess) return e;
  return cudaStreamWaitEvent(st, ss->join, 0);
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

AssignTC assign_common(const Ctx& c, void* ws, int32_t* labels, int32_t* flags, int flag_base,
                       int sms) {
  AssignTC a = {};
  a.H = c.p.H;
  a.n = c.L.Nv;
  a.labels = labels;
  a.flags = flags;
  a.flag_base = flag_base;
  a.recheck = at<int32_t>(ws, c.L.recheck);
  a.nrecheck = at<int32_t>(ws, c.L.nrecheck);
  a.stats = c.stats;
  a.sm_count = sms;
  return a;
}

// Nearest-centroid pass in the d-space form argmin_j (cy_j - 2 x . y_j) of
// the video rows x of X [H, N, d] (bf16 or fp32, exact) against the centroid
// side y [H, m, d], cy [H, m] (fp64): on the tensor cores (one exact bf16
// plane of x, two or three planes of y, certified, fp64 recheck) when the
// centroid planes fit in shared memory, else in fp64 on the CUDA cores.
// G: the metric of the true distance x^T G x + cy_j - 2 x . y_j, used only to
// count near ties; the alternative partitions pass null and count none.
struct DPass {
  int nb = 0;  // centroid planes on the tensor cores; 0: fp64 path
  AssignTC a = {};
  const void* X = nullptr;
  int m = 0, Cpad = 0, flag_base = 0;
  int32_t* labels = nullptr;
  const double* G = nullptr;
};

cudaError_t dpass_setup(const Ctx& c, void* ws, const void* X, int m, int Cpad, int32_t* labels,
                        int flag_base, float* xnorm, const double* cy, const double* G, int sms,
                        DPass* P, cudaStream_t st) {
  const int H = c.p.H, N = c.p.N, d = c.p.d, Nv = c.L.Nv;
  const long long hs_in = static_cast<long long>(N) * d;
  P->X = X;
  P->m = m;
  P->Cpad = Cpad;
  P->flag_base = flag_base;
  P->labels = labels;
  P->G = G;
  P->nb = 0;
  // (a 128-row TMA box needs at least 128 rows in the tensor)
  if (c.bf16 && static_cast<size_t>(H) * N >= static_cast<size_t>(kTileM)) {
    if (assign_tc_smem_bytes(1, 3, d, Cpad) <= kMaxDynSmem)
      P->nb = 3;
    else if (assign_tc_smem_bytes(1, 2, d, Cpad) <= kMaxDynSmem)
      P->nb = 2;
  }
  if (!P->nb) return cudaSuccess;
  const cudaError_t e = launch_split_rows(X, c.kind, hs_in, d, Nv, d, d, 0, H, nullptr, 0, xnorm,
                                          st);
  if (e != cudaSuccess) return e;
  AssignTC& a = P->a;
  a = assign_common(c, ws, labels, at<int32_t>(ws, c.L.flags), flag_base, sms);
  a.a_planes = static_cast<const __nv_bfloat16*>(X);
  a.a_plane_stride = 0;
  a.a_rows_total = static_cast<size_t>(H) * N;
  a.a_head = N;
  a.nA = 1;
  a.b_planes = at<__nv_bfloat16>(ws, c.L.wplanes);
  a.b_plane_stride = static_cast<long long>(H) * Cpad * d;
  a.nB = P->nb;
  a.Dp = d;
  a.Cpad = Cpad;
  a.npairs = P->nb;
  for (int i = 0; i < 6; ++i) a.pairs[i] = (i < P->nb) ? i : 0;
  a.cvals = at<float>(ws, c.L.cfq);
  a.xnorm = xnorm;
  a.hmax = at<float>(ws, c.L.hmq);
  a.x_exact = X;
  a.x_kind = c.kind;
  a.x_hs = hs_in;
  a.x_ld = d;
  a.D = d;
  a.y_tr = at<double>(ws, c.L.ytr);
  a.c_exact = cy;
  a.m = m;
  a.direct = 0;
  a.metric = G;
  return cudaSuccess;
}

cudaError_t dpass_run(const Ctx& c, void* ws, const DPass& P, const double* y, const double* cy) {
  const int H = c.p.H, N = c.p.N, d = c.p.d, Nv = c.L.Nv;
  int32_t* flags = at<int32_t>(ws, c.L.flags);
  if (P.nb) {
    const cudaError_t e = launch_prep_centroids(
        y, cy, P.m, d, d, P.Cpad, P.nb, H, at<__nv_bfloat16>(ws, c.L.wplanes),
        static_cast<long long>(H) * P.Cpad * d, at<float>(ws, c.L.cfq), at<float>(ws, c.L.hmq),
        at<double>(ws, c.L.ytr), flags, P.flag_base, c.st);
    if (e != cudaSuccess) return e;
    return launch_argmin_tc(P.a, c.st);
  }
  return launch_argmin(P.X, c.kind, static_cast<long long>(N) * d, d, Nv, d, y, cy, P.m, H,
                       P.labels, flags, P.flag_base, P.G, P.G ? c.stats : nullptr, c.st);
}

// The alternative partitions ([SPR 4] ablations' semantic k-means; the
// co-clustering page's bidirectional rounds), both on the d-space pass.
// Initial rows, pass cap, ties and empty groups as in the method's partition.
sparsepr_status partition_alternative(const Ctx& c, const void* q, const void* k,
                                      int32_t* label_q, int32_t* label_k, void* ws) {
  const Layout& L = c.L;
  const int H = c.p.H, N = c.p.N, d = c.p.d, Nv = L.Nv, Ck = c.p.Ck, Cq = c.p.Cq;
  const int iters = c.p.kmeans_iters;
  const long long hs_in = static_cast<long long>(N) * d;
  cudaStream_t st = c.st;
  int32_t* flags = at<int32_t>(ws, L.flags);
  int32_t* init_k = at<int32_t>(ws, L.init_k);
  int32_t* init_q = at<int32_t>(ws, L.init_q);
  int32_t* lab_k = at<int32_t>(ws, L.lab_k);
  int32_t* lab_q = at<int32_t>(ws, L.lab_q);
  int32_t* hist = at<int32_t>(ws, L.hist);
  int32_t* sperm = at<int32_t>(ws, L.sortperm);
  int32_t* soff = at<int32_t>(ws, L.sortoff);
  int32_t* cnt_k = at<int32_t>(ws, L.cnt);
  int32_t* cnt_q = cnt_k + static_cast<size_t>(H) * Ck;
  double* ck = at<double>(ws, L.ck);    // key centres [H, Ck, d]
  double* qbar = at<double>(ws, L.qbar);  // query centres [H, Cq, d]
  double* G = at<double>(ws, L.g);
  double* wg = at<double>(ws, L.wg);    // centroid side y [H, max(Ck, Cq), d]
  double* cg = at<double>(ws, L.cg);    // offsets cy [H, max(Ck, Cq)]
  const int sms = sm_count();
  SPR_TRY(launch_fy_init(H, Nv, Ck, Cq, c.p.seed, init_k, init_q, st));
  SPR_TRY(launch_gather_init(k, c.kind, hs_in, d, d, init_k, Ck, H, ck, nullptr, st));
  SPR_TRY(launch_gather_init(q, c.kind, hs_in, d, d, init_q, Cq, H, qbar, nullptr, st));
  DPass pk, pq;
  SPR_TRY(dpass_setup(c, ws, k, Ck, L.CpadK, lab_k, 0, at<float>(ws, L.xnk), cg, nullptr, sms, &pk,
                      c.st));
  SPR_TRY(dpass_setup(c, ws, q, Cq, L.CpadQ, lab_q, 2, at<float>(ws, L.xnq), cg, nullptr, sms, &pq,
                      c.st));
  if (c.p.partition == SPARSEPR_PARTITION_SEMANTIC) {
    // plain Euclidean Lloyd on each side: the d-space form with G = I
    // (y = centre, cy = |centre|^2)
    SPR_TRY(launch_identity(G, H, d, st));
    for (int side = 0; side < 2; ++side) {
      const void* X = side ? q : k;
      double* cen = side ? qbar : ck;
      const int m = side ? Cq : Ck;
      const int fb = side ? 2 : 0;
      int32_t* lab = side ? lab_q : lab_k;
      const DPass& P = side ? pq : pk;
      for (int t = 0; t < iters; ++t) {
        SPR_TRY(launch_query_metric_apply(G, cen, m, H, d, wg, cg, flags + fb + 1, 4, st));
        SPR_TRY(dpass_run(c, ws, P, wg, cg));
        SPR_TRY(launch_finalize_pass(H, t, flags, fb,
                                     side ? c.stats->query_passes : c.stats->key_passes, st));
        if (t + 1 < iters) {
          SPR_TRY(launch_counting_sort(lab, H, Nv, m, L.nchunk, hist, sperm, soff, flags + fb + 1,
                                       4, nullptr, st));
          SPR_TRY(launch_group_mean(X, c.kind, hs_in, d, d, sperm, Nv, soff, m + 1, m, H, true,
                                    cen, nullptr, flags + fb + 1, 4, st));
        }
      }
    }
  } else {
    // co-clustering rounds: keys against the query centres' affinity space,
    // then queries against the new key centres'
    if (static_cast<size_t>(8) * (Ck > Cq ? Ck : Cq) * 8 > kMaxDynSmem) return SPARSEPR_ERR_UNSUPPORTED;
    double* pkbar = at<double>(ws, L.pkbar);
    double* pqbar = at<double>(ws, L.pqbar);
    for (int t = 0; t < iters; ++t) {
      // key blocks: mean affinity vectors (from the seed keys in the first
      // round, then from the blocks' mean keys; an empty block keeps its
      // vector), their d-space form, the assignment
      SPR_TRY(launch_affinity_centres(ck, qbar, Ck, Cq, d, H, c.scale, cnt_k, t == 0, pkbar, st));
      SPR_TRY(launch_dspace_centres(pkbar, qbar, Ck, Cq, d, H, c.scale, wg, cg, st));
      SPR_TRY(dpass_run(c, ws, pk, wg, cg));
      // key centres: the blocks' mean keys (zero for an empty block)
      SPR_TRY(launch_counting_sort(lab_k, H, Nv, Ck, L.nchunk, hist, sperm, soff, flags + 1, 4,
                                   nullptr, st));
      SPR_TRY(launch_group_mean(k, c.kind, hs_in, d, d, sperm, Nv, soff, Ck + 1, Ck, H, false, ck,
                                nullptr, flags + 1, 4, st));
      SPR_TRY(launch_group_counts(soff, Ck + 1, Ck, H, cnt_k, st));
      // query blocks against the new key centres
      SPR_TRY(launch_affinity_centres(qbar, ck, Cq, Ck, d, H, c.scale, cnt_q, t == 0, pqbar, st));
      SPR_TRY(launch_dspace_centres(pqbar, ck, Cq, Ck, d, H, c.scale, wg, cg, st));
      SPR_TRY(dpass_run(c, ws, pq, wg, cg));
      // query centres: the blocks' mean queries (an empty block keeps its centre)
      SPR_TRY(launch_counting_sort(lab_q, H, Nv, Cq, L.nchunk, hist, sperm, soff, flags + 3, 4,
                                   nullptr, st));
      SPR_TRY(launch_group_mean(q, c.kind, hs_in, d, d, sperm, Nv, soff, Cq + 1, Cq, H, true, qbar,
                                nullptr, flags + 3, 4, st));
      SPR_TRY(launch_group_counts(soff, Cq + 1, Cq, H, cnt_q, st));
      SPR_TRY(launch_finalize_round(H, t, flags, c.stats->key_passes, c.stats->query_passes, st));
    }
  }
  SPR_TRY(launch_write_labels(lab_q, H, N, Nv, Cq, label_q, st));
  SPR_TRY(launch_write_labels(lab_k, H, N, Nv, Ck, label_k, st));
  return SPARSEPR_OK;
}

// Dense-mode routing metadata per head: one query group [0, M), one key
// group [0, N) kept by it.
__global__ void dense_meta_kernel(int32_t* meta, int H, int M, int N) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  int32_t* offq = meta;
  int32_t* offk = meta + 2 * H;
  int32_t* csr = meta + 4 * H;
  int32_t* kh = meta + 5 * H;
  offq[2 * h] = 0;
  offq[2 * h + 1] = M;
  offk[2 * h] = 0;
  offk[2 * h + 1] = N;
  csr[h] = 0;
  kh[h] = 1;
}

// sparsepr_attention overlaps the probe fit with the attention of all rows
// while the dual pass's extra work stays below this many flop.
constexpr double kDualFlopMax = 4e11;

// bf16 copies of the permuted Q, K, V for the attention kernels (fp32 inputs
// are rounded into the workspace; bf16 inputs are used in place).
struct Bf16Qkv {
  const void *q = nullptr, *k = nullptr, *v = nullptr;
};

cudaError_t bf16_inputs(const Ctx& c, void* ws, const void* qp, const void* kp, const void* vp,
                        bool cast_q, Bf16Qkv* t) {
  t->q = qp;
  t->k = kp;
  t->v = vp;
  if (c.bf16) return cudaSuccess;
  const size_t n = static_cast<size_t>(c.p.H) * c.p.N * c.p.d;
  __nv_bfloat16* b = at<__nv_bfloat16>(ws, c.L.bf16_qkv);
  cudaError_t e = cudaSuccess;
  if (cast_q) {
    e = launch_cast_bf16(static_cast<const float*>(qp), b, n, c.st);
    t->q = b;
  }
  if (e == cudaSuccess) e = launch_cast_bf16(static_cast<const float*>(kp), b + n, n, c.st);
  if (e == cudaSuccess) e = launch_cast_bf16(static_cast<const float*>(vp), b + 2 * n, n, c.st);
  t->k = b + n;
  t->v = b + 2 * n;
  return e;
}

// The routed attention of every row ([SPR 2.C]).
AttnArgs main_attn_args(const Ctx& c, void* ws, const Bf16Qkv& t, const int32_t* off_q,
                        const int32_t* off_k, const int32_t* csr, const int32_t* k_per_head,
                        float* o_sparse, int64_t* pairs_sparse) {
  AttnArgs a;
  a.qp = t.q;
  a.kp = t.k;
  a.vp = t.v;
  a.H = c.p.H;
  a.N = c.p.N;
  a.d = c.p.d;
  a.q_rows = c.p.N;
  a.Cq = c.L.Cqt;
  a.Ck = c.L.Ckt;
  a.text = c.p.n_text > 0 ? 1 : 0;
  a.off_q = off_q;
  a.off_k = off_k;
  a.csr = csr;
  a.kh = k_per_head;
  a.kmax = c.L.kmax;
  a.scale = static_cast<float>(c.scale);
  a.out = o_sparse;
  a.work = at<int32_t>(ws, c.L.work);
  a.nwork = at<int32_t>(ws, c.L.nwork);
  a.tiles_per_head = c.L.tiles_per_head;
  a.nslots = at<int32_t>(ws, c.L.nslots);
  a.runs = at<int2>(ws, c.L.runs);
  a.nruns = at<int32_t>(ws, c.L.nruns);
  a.pairs = pairs_sparse;
  a.stats = c.stats;
  a.lse = at<float>(ws, c.L.lse_s);
  return a;
}

cudaError_t zero_fit(const Ctx& c, void* ws, double* fit, cudaStream_t st) {
  const size_t H = c.p.H, d = c.p.d;
  cudaError_t e = cudaMemsetAsync(at<float>(ws, c.L.bp32), 0, H * d * d * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(at<float>(ws, c.L.bv32), 0, H * d * 4, st);
  if (e == cudaSuccess && fit) e = cudaMemsetAsync(fit, 0, H * (d * d + d) * 8, st);
  return e;
}

// The probe rows of [SPR 2.B] (M > 0) on stream st: stratified probe rows and
// their exact dense outputs over all keys.
//   o_sparse given: the dense pass covers the probe rows alone (X is read
//     later from o_sparse at the probe rows);
//   o_sparse null (dual): one pass also forms X = their sparse outputs (each
//     row's keys limited to its query group's kept runs, from the routed
//     pass's metadata), so the fit does not wait for the attention of all rows.
// qsrc: the permuted queries the probe rows are gathered from (bf16 or, with
// fp32 inputs, fp32).
sparsepr_status probe_pass(const Ctx& c, void* ws, const Bf16Qkv& t, const void* qsrc,
                           const int32_t* off_q, int32_t* probes, bool dual, cudaStream_t st) {
  const Layout& L = c.L;
  const int H = c.p.H, N = c.p.N, d = c.p.d, M = c.p.M, Cq = c.p.Cq;
  float* od = at<float>(ws, L.od);
  int32_t* pgrp = dual ? at<int32_t>(ws, L.pgrp) : nullptr;
  SPR_TRY(launch_probe_select(off_q, L.Cqt + 1, H, Cq, M, probes, pgrp, st));  // video groups only
  __nv_bfloat16* pq = at<__nv_bfloat16>(ws, L.probe_q);
  SPR_TRY(launch_gather_probe_rows(qsrc, c.bf16, probes, H, N, M, d, pq, st));
  int32_t* meta = at<int32_t>(ws, L.pmeta);
  dense_meta_kernel<<<(H + 127) / 128, 128, 0, st>>>(meta, H, M, N);
  SPR_TRY(cudaGetLastError());
  {
    AttnArgs a;
    a.qp = pq;
    a.kp = t.k;
    a.vp = t.v;
    a.H = H;
    a.N = N;
    a.d = d;
    a.q_rows = M;
    a.Cq = 1;
    a.Ck = 1;
    a.off_q = meta;
    a.off_k = meta + 2 * H;
    a.csr = meta + 4 * H;
    a.kh = meta + 5 * H;
    a.kmax = 1;
    a.scale = static_cast<float>(c.scale);
    a.out = od;
    a.work = at<int32_t>(ws, L.pwork);
    a.nwork = at<int32_t>(ws, L.pnwork);
    a.tiles_per_head = M / kTileM + 2;
    a.nslots = meta + 6 * H;
    a.nruns = meta + 7 * H;
    a.runs = reinterpret_cast<int2*>(meta + 8 * H);
    a.pairs = nullptr;
    a.stats = c.stats;
    a.lse = at<float>(ws, L.lse_d);
    // few units over all N keys: split the key tiles so that about one CTA
    // per SM runs
    const int urows = dual ? kTileM : 256;
    const int units = (M + urows - 1) / urows;
    const int ktiles = (N + kTileN - 1) / kTileN;
    int sp = sm_count() / (H * units > 0 ? H * units : 1);
    if (sp > kMaxSplits) sp = kMaxSplits;
    if (sp > ktiles) sp = ktiles;
    if (sp < 1) sp = 1;
    a.splits = sp;
    a.units = dual ? M / kTileM + 1 : L.punits;
    a.opart = at<float>(ws, L.opart);
    a.lpart = at<float>(ws, L.lpart);
    if (dual) {
      a.dual = 1;
      a.out2 = at<float>(ws, L.xp);
      a.opart2 = at<float>(ws, L.opart2);
      a.lpart2 = at<float>(ws, L.lpart2);
      a.pgrp = pgrp;
      a.gruns = at<int2>(ws, L.runs);
      a.gnruns = at<int32_t>(ws, L.nruns);
      a.gCq = L.Cqt;
      a.gkmax = L.kmax;
    }
    SPR_TRY(launch_block_sparse_attn(a, st));
  }
  return SPARSEPR_OK;
}

// The fit of [SPR 2.B] on stream st after probe_pass: R = O_dense - X (X from
// o_sparse at the probe rows, or from the dual pass when o_sparse is null),
// the ridge solution (B, b) and the leading-r subspace of R; writes the
// projected map (bp32, bv32; `fit` when not null). ridge_ss: the side stream
// the ridge solve runs on beside the subspace solve (null: in order on st);
// the caller holds g_side_mu. The side stream is joined on every path.
sparsepr_status probe_solve(const Ctx& c, void* ws, const int32_t* probes, const float* o_sparse,
                            double* fit, cudaStream_t st, SideStream* ridge_ss) {
  const Layout& L = c.L;
  const int H = c.p.H, N = c.p.N, d = c.p.d, M = c.p.M;
  const bool dual = (o_sparse == nullptr);
  const float* od = at<float>(ws, L.od);
  double* xr = at<double>(ws, L.xr);
  double* means = at<double>(ws, L.means);
  double* gram = at<double>(ws, L.gram);
  const long long hs = 2LL * M * d;
  // the block sums of the residual pass live in the Gram region until the
  // Grams are formed
  SPR_TRY(launch_probe_residuals(o_sparse, dual ? at<float>(ws, L.xp) : nullptr, od, probes, H, N,
                                 M, d, xr, means, gram, static_cast<size_t>(H) * 2 * d * d, st));
  double* bmat = at<double>(ws, L.bmat);
  double* bvec = at<double>(ws, L.bvec);
  double* rtr = at<double>(ws, L.mk);
  {
    // one launch for the three Grams over the probe rows: the centred
    // X^T X + lambda I and X^T R of the ridge system, and the uncentred R^T R
    const double* R = xr + static_cast<size_t>(M) * d;
    GramJobs g = {};
    g.part = at<double>(ws, L.gpart);
    g.job[0] = GramJob{xr, xr, means, means, hs, hs, 2LL * d, gram, 2LL * d * d, 1.0, c.p.lambda};
    g.job[1] = GramJob{xr, R, means, means + d, hs, hs, 2LL * d, gram + static_cast<size_t>(d) * d,
                       2LL * d * d, 1.0, 0.0};
    g.job[2] = GramJob{R, R, nullptr, nullptr, hs, hs, 0, rtr, static_cast<long long>(d) * d, 1.0,
                       0.0};
    g.njobs = 3;
    g.ld = d;
    g.S = M;
    g.d = d;
    g.H = H;
    SPR_TRY(launch_gram_f64(g, st));
  }
  // the ridge solve (reads the Grams) runs beside the eigen solve of R^T R
  // (they touch other regions); with r > kTriEigMax the Gram region is
  // reused below, so the two stay in order
  SideStream* ss = (c.p.r <= kTriEigMax) ? ridge_ss : nullptr;
  const cudaStream_t side = fork_side(ss, st);
  cudaError_t err = launch_ridge_solve(gram, H, d, bmat, bvec, means, c.stats, side);
  double* evl = at<double>(ws, L.eval);
  double* evc = at<double>(ws, L.evec);
  // leading-r right singular vectors of R = top-r eigenvectors of R^T R
  const double* vr = evc;
  if (c.p.r <= kTriEigMax) {
    if (err == cudaSuccess)
      err = launch_sym_eigs(rtr, H, d, c.p.r, evl, evc, at<double>(ws, L.eigscr), st);
  } else {
    double* sel = gram;  // free after the ridge solve: [H, d, r] selected vectors
    if (err == cudaSuccess) err = launch_jacobi(rtr, H, d, evl, evc, c.stats, 1, st);
    if (err == cudaSuccess)
      err = launch_top_eig_projector(evl, evc, H, d, c.p.r, sel, false, st);
    vr = sel;
  }
  const cudaError_t ej = join_side(ss, side, st);
  SPR_TRY(err);
  SPR_TRY(ej);
  SPR_TRY(launch_project_map(bmat, bvec, vr, H, d, c.p.r, at<float>(ws, L.bp32),
                             at<float>(ws, L.bv32), fit, st));
  return SPARSEPR_OK;
}

// The correction of the unprobed rows and the unpermute [SPR 2.B]; the
// executed-pair counts.
cudaError_t probe_apply(const Ctx& c, void* ws, const float* o_sparse, const int32_t* probes,
                        const int32_t* perm_q, const int64_t* pairs_sparse, void* out,
                        int64_t* pairs_exec, cudaStream_t st) {
  const Layout& L = c.L;
  const int H = c.p.H, N = c.p.N, d = c.p.d, M = c.p.M;
  const float* bp32 = at<float>(ws, L.bp32);
  const float* bv32 = at<float>(ws, L.bv32);
  const float* od = at<float>(ws, L.od);
  cudaError_t e;
  if (correct_tc_supported(H, N, d))
    e = launch_correct_tc(o_sparse, od, probes, perm_q, bp32, bv32, H, N, L.Nv, M, d, out,
                          c.bf16, sm_count(), c.stats, st);
  else
    e = launch_correct(o_sparse, od, probes, perm_q, bp32, bv32, H, N, L.Nv, M, d, out, c.bf16,
                       st);
  if (e != cudaSuccess) return e;
  return launch_pairs_exec(pairs_sparse, H, static_cast<int64_t>(M) * N, pairs_exec, c.stats, st);
}

// One thread waits, through the same bounded mbarrier wait as every kernel
// of the library, on a barrier that nothing completes; when the limit runs
// out the wait gives up and the status word gets SPARSEPR_ERR_TIMEOUT.
__global__ void wait_limit_kernel(DeviceStats* stats) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort)) raise_status(stats, SPARSEPR_ERR_TIMEOUT);
}

// The sorts and the gathers of q and k (and of v when `with_v`; K and V
// share their permutation and move in one launch).
sparsepr_status permute_rows(const Ctx& c, const void* q, const void* k, const void* v,
                             const int32_t* label_q, const int32_t* label_k, int32_t* perm_q,
                             int32_t* perm_k, int32_t* off_q, int32_t* off_k, void* qp, void* kp,
                             void* vp, bool with_v, void* ws) {
  const int H = c.p.H, N = c.p.N, d = c.p.d;
  const int nchunk = c.L.nchunk;  // chunks of all N tokens
  int32_t* hist = at<int32_t>(ws, c.L.hist);
  // with text tokens the last group of each side is the text group
  SPR_TRY(launch_counting_sort(label_q, H, N, c.L.Cqt, nchunk, hist, perm_q, off_q, nullptr, 0,
                               c.stats, c.st));
  SPR_TRY(launch_counting_sort(label_k, H, N, c.L.Ckt, nchunk, hist, perm_k, off_k, nullptr, 0,
                               c.stats, c.st));
  const int eb = c.bf16 ? 2 : 4;
  SPR_TRY(launch_gather_rows(q, qp, nullptr, nullptr, perm_q, H, N, d, eb, c.st));
  SPR_TRY(launch_gather_rows(k, kp, with_v ? v : nullptr, with_v ? vp : nullptr, perm_k, H, N, d,
                             eb, c.st));
  return SPARSEPR_OK;
}

sparsepr_status check_permute_args(const void* q, const void* k, const void* v,
                                   const int32_t* label_q, const int32_t* label_k,
                                   const int32_t* perm_q, const int32_t* perm_k,
                                   const int32_t* off_q, const int32_t* off_k, const void* qp,
                                   const void* kp, const void* vp) {
  if (!q || !k || !v || !label_q || !label_k || !perm_q || !perm_k || !off_q || !off_k || !qp ||
      !kp || !vp)
    return SPARSEPR_ERR_INVALID_ARG;
  if (qp == q || kp == k || vp == v) return SPARSEPR_ERR_INVALID_ARG;
  if (!al16(q, k, v, qp, kp, vp)) return SPARSEPR_ERR_INVALID_ARG;
  return SPARSEPR_OK;
}

}  // namespace

extern "C" {

size_t sparsepr_workspace_bytes(const sparsepr_params* p) {
  if (check_params(p) != SPARSEPR_OK) return 0;
  Layout L;
  compute_layout(*p, &L);
  return L.total;
}

const char* sparsepr_status_string(sparsepr_status s) {
  switch (s) {
    case SPARSEPR_OK: return "ok";
    case SPARSEPR_ERR_INVALID_ARG: return "invalid argument";
    case SPARSEPR_ERR_UNSUPPORTED: return "unsupported configuration";
    case SPARSEPR_ERR_WORKSPACE: return "workspace too small or misaligned";
    case SPARSEPR_ERR_CUDA: return "CUDA error";
    case SPARSEPR_ERR_TIMEOUT: return "device wait limit reached";
    case SPARSEPR_ERR_NUMERIC: return "numerical error (empty kept set or non-finite value)";
  }
  return "unknown status";
}

int32_t sparsepr_route_width(const sparsepr_params* p) {
  if (check_params(p) != SPARSEPR_OK) return -1;
  Layout L;
  compute_layout(*p, &L);
  return L.kmax;
}

sparsepr_status sparsepr_workspace_region(const sparsepr_params* p, const char* name,
                                          size_t* offset, size_t* bytes) {
  if (!name || !offset || !bytes) return SPARSEPR_ERR_INVALID_ARG;
  const sparsepr_status s = check_params(p);
  if (s != SPARSEPR_OK) return s;
  Layout L;
  compute_layout(*p, &L);
  return named_region(*p, L, name, offset, bytes) ? SPARSEPR_OK : SPARSEPR_ERR_INVALID_ARG;
}

sparsepr_status sparsepr_check_wait_limit(void* ws, void* stream) {
  if (!ws) return SPARSEPR_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return SPARSEPR_ERR_INVALID_ARG;
  wait_limit_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<DeviceStats*>(ws));
  return cuda_status(cudaGetLastError());
}

sparsepr_status sparsepr_check_reciprocal(const double* x, int64_t n, double* err, void* stream) {
  if (n < 0 || (n > 0 && (!x || !err))) return SPARSEPR_ERR_INVALID_ARG;
  return cuda_status(launch_check_reciprocal(x, n, err, static_cast<cudaStream_t>(stream)));
}

sparsepr_status sparsepr_reset_stats(void* ws, void* stream) {
  if (!ws) return SPARSEPR_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(DeviceStats), static_cast<cudaStream_t>(stream)));
}

sparsepr_status sparsepr_read_stats(const void* ws, sparsepr_stats* out) {
  if (!ws || !out) return SPARSEPR_ERR_INVALID_ARG;
  return cuda_status(cudaMemcpy(out, ws, sizeof(DeviceStats), cudaMemcpyDeviceToHost));
}

sparsepr_status sparsepr_partition(const void* q, const void* k, sparsepr_dtype dt,
                                   const sparsepr_params* p, int32_t* label_q, int32_t* label_k,
                                   void* ws, size_t ws_bytes, void* stream) {
  Ctx c;
  sparsepr_status s = setup(&c, p, dt, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  if (!q || !k || !label_q || !label_k) return SPARSEPR_ERR_INVALID_ARG;
  if (!al16(q, k)) return SPARSEPR_ERR_INVALID_ARG;
  const Layout& L = c.L;
  const int H = c.p.H, N = c.p.N, d = c.p.d, Nv = L.Nv, e = c.p.n_eig, Ck = c.p.Ck, Cq = c.p.Cq;
  const int iters = c.p.kmeans_iters;
  cudaStream_t st = c.st;
  int32_t* flags = at<int32_t>(ws, L.flags);
  SPR_TRY(cudaMemsetAsync(ws, 0, sizeof(DeviceStats), st));
  SPR_TRY(cudaMemsetAsync(flags, 0, static_cast<size_t>(H) * 16, st));
  set_i32_kernel<<<1, 1, 0, st>>>(&c.stats->H, H);
  int32_t* init_k = at<int32_t>(ws, L.init_k);
  int32_t* init_q = at<int32_t>(ws, L.init_q);
  double* mk = at<double>(ws, L.mk);
  double* evl = at<double>(ws, L.eval);
  double* evc = at<double>(ws, L.evec);
  double* wk = at<double>(ws, L.wk);
  double* z = at<double>(ws, L.z);
  double* mu = at<double>(ws, L.mu);
  double* mun = at<double>(ws, L.munorm);
  int32_t* lab_k = at<int32_t>(ws, L.lab_k);
  int32_t* lab_q = at<int32_t>(ws, L.lab_q);
  int32_t* hist = at<int32_t>(ws, L.hist);
  int32_t* sperm = at<int32_t>(ws, L.sortperm);
  int32_t* soff = at<int32_t>(ws, L.sortoff);
  double* ck = at<double>(ws, L.ck);
  double* G = at<double>(ws, L.g);
  double* qbar = at<double>(ws, L.qbar);
  double* wg = at<double>(ws, L.wg);
  double* cg = at<double>(ws, L.cg);
  const long long hs_in = static_cast<long long>(N) * d;
  if (c.p.partition != SPARSEPR_PARTITION_RESPONSE)
    return partition_alternative(c, q, k, label_q, label_k, ws);

  // keys: metric, eigenbasis, response coordinates, Lloyd passes
  DPass pq;  // the query passes (set up beside the key eigen solve)
  // tensor-core assignment when the centroid planes fit in shared memory
  // (a 128-row TMA box needs at least 128 rows in the tensor)
  const bool tc_keys = assign_tc_smem_bytes(3, 3, L.Dpk, L.CpadK) <= kMaxDynSmem &&
                       static_cast<size_t>(H) * Nv >= static_cast<size_t>(kTileM);
  __nv_bfloat16* zp = at<__nv_bfloat16>(ws, L.zplanes);
  const long long zps = static_cast<long long>(H) * Nv * L.Dpk;
  // the projection writes z's planes and row norms itself when its two-row
  // form runs
  const bool zproj_planes = tc_keys && e == 16 && L.Dpk == 16 && d % 8 == 0;
  {
    // the side stream is joined on every path, also after a failed launch,
    // so that a stream capture in progress stays valid
    std::lock_guard<std::mutex> lk(g_side_mu);
    SideStream* ss = side_stream();
    const cudaStream_t side = fork_side(ss, st);
    cudaError_t err = launch_fy_init(H, Nv, Ck, Cq, c.p.seed, init_k, init_q, side);
    // the query side's first centroids and row norms need only q: beside the
    // key metric and its eigen solve (few SMs)
    if (err == cudaSuccess)
      err = launch_gather_init(q, c.kind, hs_in, d, d, init_q, Cq, H, qbar, nullptr, side);
    if (err == cudaSuccess)
      err = dpass_setup(c, ws, q, Cq, L.CpadQ, lab_q, 2, at<float>(ws, L.xnq), cg, G, sm_count(),
                        &pq, side);
    if (err == cudaSuccess)
      err = launch_metric_mk(q, c.bf16, H, N, Nv, d, c.p.Ms, mk, at<double>(ws, L.gpart), st);
    if (err == cudaSuccess)
      err = launch_sym_eigs(mk, H, d, e, evl, evc, at<double>(ws, L.eigscr), st);
    if (err == cudaSuccess) err = launch_scale_columns(evl, evc, H, d, e, wk, st);
    if (err == cudaSuccess)
      err = launch_zproj(k, c.bf16, H, N, Nv, d, e, wk, z, zproj_planes ? zp : nullptr, zps,
                         zproj_planes ? at<float>(ws, L.xnk) : nullptr, st);
    const cudaError_t ej = join_side(ss, side, st);
    SPR_TRY(err);
    SPR_TRY(ej);
  }
  const long long hs_z = static_cast<long long>(Nv) * e;
  SPR_TRY(launch_gather_init(z, kXf64, hs_z, e, e, init_k, Ck, H, mu, mun, st));
  const int sms = sm_count();
  AssignTC ak;
  if (tc_keys) {
    if (!zproj_planes)
      SPR_TRY(launch_split_rows(z, kXf64, hs_z, e, Nv, e, L.Dpk, 3, H, zp, zps,
                                at<float>(ws, L.xnk), st));
    ak = assign_common(c, ws, lab_k, flags, 0, sms);
    ak.a_planes = zp;
    ak.a_plane_stride = zps;
    ak.a_rows_total = static_cast<size_t>(H) * Nv;
    ak.a_head = Nv;
    ak.nA = 3;
    ak.b_planes = at<__nv_bfloat16>(ws, L.muplanes);
    ak.b_plane_stride = static_cast<long long>(H) * L.CpadK * L.Dpk;
    ak.nB = 3;
    ak.Dp = L.Dpk;
    ak.Cpad = L.CpadK;
    ak.npairs = 6;
    const int pk[6] = {0 * 4 + 0, 0 * 4 + 1, 1 * 4 + 0, 0 * 4 + 2, 1 * 4 + 1, 2 * 4 + 0};
    for (int i = 0; i < 6; ++i) ak.pairs[i] = pk[i];
    ak.cvals = at<float>(ws, L.cfk);
    ak.xnorm = at<float>(ws, L.xnk);
    ak.hmax = at<float>(ws, L.hmk);
    ak.x_exact = z;
    ak.x_kind = kXf64;
    ak.x_hs = hs_z;
    ak.x_ld = e;
    ak.D = e;
    ak.y_tr = at<double>(ws, L.ytr);
    ak.c_exact = mun;
    ak.m = Ck;
    ak.direct = 1;
    ak.metric = nullptr;
  }
  for (int t = 0; t < iters; ++t) {
    if (tc_keys) {
      SPR_TRY(launch_prep_centroids(mu, mun, Ck, e, L.Dpk, L.CpadK, 3, H,
                                    at<__nv_bfloat16>(ws, L.muplanes),
                                    static_cast<long long>(H) * L.CpadK * L.Dpk,
                                    at<float>(ws, L.cfk), at<float>(ws, L.hmk),
                                    at<double>(ws, L.ytr), flags, 0, st));
      SPR_TRY(launch_argmin_tc(ak, st));
    } else {
      SPR_TRY(launch_argmin(z, kXf64, hs_z, e, Nv, e, mu, mun, Ck, H, lab_k, flags, 0, nullptr,
                            c.stats, st));
    }
    SPR_TRY(launch_finalize_pass(H, t, flags, 0, c.stats->key_passes, st));
    if (t + 1 < iters) {
      SPR_TRY(launch_counting_sort(lab_k, H, Nv, Ck, L.nchunk, hist, sperm, soff, flags + 1, 4,
                                   nullptr, st));
      SPR_TRY(launch_group_mean(z, kXf64, hs_z, e, e, sperm, Nv, soff, Ck + 1, Ck, H, true, mu,
                                mun, flags + 1, 4, st));
    }
  }
  // K/V group centroids in the original space, query metric G = s^2 C_K^T C_K
  SPR_TRY(launch_counting_sort(lab_k, H, Nv, Ck, L.nchunk, hist, sperm, soff, nullptr, 0, nullptr,
                               st));
  SPR_TRY(launch_group_mean(k, c.kind, hs_in, d, d, sperm, Nv, soff, Ck + 1, Ck, H, false, ck,
                            nullptr, nullptr, 0, st));
  SPR_TRY(launch_gram_f64(ck, ck, nullptr, nullptr, static_cast<long long>(Ck) * d,
                          static_cast<long long>(Ck) * d, d, Ck, H, d, c.scale * c.scale, 0.0, G,
                          static_cast<long long>(d) * d, 0, at<double>(ws, L.gpart), st));
  // queries: Lloyd passes on logit profiles in the d-space form (on the
  // tensor cores for bf16 inputs, exact in one bf16 plane)
  for (int t = 0; t < iters; ++t) {
    SPR_TRY(launch_query_metric_apply(G, qbar, Cq, H, d, wg, cg, flags + 3, 4, st));
    SPR_TRY(dpass_run(c, ws, pq, wg, cg));
    SPR_TRY(launch_finalize_pass(H, t, flags, 2, c.stats->query_passes, st));
    if (t + 1 < iters) {
      SPR_TRY(launch_counting_sort(lab_q, H, Nv, Cq, L.nchunk, hist, sperm, soff, flags + 3, 4,
                                   nullptr, st));
      SPR_TRY(launch_group_mean(q, c.kind, hs_in, d, d, sperm, Nv, soff, Cq + 1, Cq, H, true,
                                qbar, nullptr, flags + 3, 4, st));
    }
  }
  SPR_TRY(launch_write_labels(lab_q, H, N, Nv, Cq, label_q, st));
  SPR_TRY(launch_write_labels(lab_k, H, N, Nv, Ck, label_k, st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_permute(const void* q, const void* k, const void* v, sparsepr_dtype dt,
                                 const sparsepr_params* p, const int32_t* label_q,
                                 const int32_t* label_k, int32_t* perm_q, int32_t* perm_k,
                                 int32_t* off_q, int32_t* off_k, void* qp, void* kp, void* vp,
                                 void* ws, size_t ws_bytes, void* stream) {
  Ctx c;
  sparsepr_status s = setup(&c, p, dt, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  s = check_permute_args(q, k, v, label_q, label_k, perm_q, perm_k, off_q, off_k, qp, kp, vp);
  if (s != SPARSEPR_OK) return s;
  return permute_rows(c, q, k, v, label_q, label_k, perm_q, perm_k, off_q, off_k, qp, kp, vp, true,
                      ws);
}

sparsepr_status sparsepr_route(const void* qp, const void* kp, sparsepr_dtype dt,
                               const sparsepr_params* p, const int32_t* off_q,
                               const int32_t* off_k, int32_t* csr, int32_t* k_per_head, void* ws,
                               size_t ws_bytes, void* stream) {
  Ctx c;
  sparsepr_status s = setup(&c, p, dt, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  if (!qp || !kp || !off_q || !off_k || !csr || !k_per_head) return SPARSEPR_ERR_INVALID_ARG;
  if (!al16(qp, kp)) return SPARSEPR_ERR_INVALID_ARG;
  const int H = c.p.H, N = c.p.N, d = c.p.d, Ck = c.p.Ck, Cq = c.p.Cq;
  double* cq = at<double>(ws, c.L.cq);
  double* ckr = at<double>(ws, c.L.ckr);
  // block scores of the video groups (the text groups are kept outside the budget)
  SPR_TRY(launch_range_mean(qp, c.kind, H, N, d, off_q, Cq, c.L.Cqt + 1, cq, c.st));
  SPR_TRY(launch_range_mean(kp, c.kind, H, N, d, off_k, Ck, c.L.Ckt + 1, ckr, c.st));
  int32_t kh[SPARSEPR_MAX_HEADS];
  for (int h = 0; h < H; ++h) kh[h] = keep_budget(c.p.keep[h], Ck);
  SPR_TRY(launch_write_k(kh, H, k_per_head, c.st));
  SPR_TRY(launch_route_gemm(cq, ckr, H, Cq, Ck, d, c.scale, k_per_head, c.L.kmax,
                            at<double>(ws, c.L.scores), c.L.scores_bytes, csr, c.st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_block_sparse_attn(const void* qp, const void* kp, const void* vp,
                                           sparsepr_dtype dt, const sparsepr_params* p,
                                           const int32_t* off_q, const int32_t* off_k,
                                           const int32_t* csr, const int32_t* k_per_head,
                                           float* o_sparse, int64_t* pairs_sparse, void* ws,
                                           size_t ws_bytes, void* stream) {
  Ctx c;
  sparsepr_status s = setup(&c, p, dt, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  if (!qp || !kp || !vp || !off_q || !off_k || !csr || !k_per_head || !o_sparse || !pairs_sparse)
    return SPARSEPR_ERR_INVALID_ARG;
  if (!al16(qp, kp, vp, o_sparse)) return SPARSEPR_ERR_INVALID_ARG;
  Bf16Qkv t;
  SPR_TRY(bf16_inputs(c, ws, qp, kp, vp, true, &t));
  SPR_TRY(launch_block_sparse_attn(
      main_attn_args(c, ws, t, off_q, off_k, csr, k_per_head, o_sparse, pairs_sparse), c.st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_probe_correct(const void* qp, const void* kp, const void* vp,
                                       sparsepr_dtype dt, const sparsepr_params* p,
                                       const int32_t* off_q, const int32_t* perm_q,
                                       const float* o_sparse, const int64_t* pairs_sparse,
                                       void* out, int32_t* probes, int64_t* pairs_exec,
                                       double* fit, void* ws, size_t ws_bytes, void* stream) {
  Ctx c;
  sparsepr_status s = setup(&c, p, dt, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  if (!qp || !kp || !vp || !off_q || !perm_q || !o_sparse || !pairs_sparse || !out ||
      !pairs_exec || (c.p.M > 0 && !probes))
    return SPARSEPR_ERR_INVALID_ARG;
  if (!al16(qp, kp, vp, o_sparse, out)) return SPARSEPR_ERR_INVALID_ARG;
  if (c.p.M > 0) {
    Bf16Qkv t;
    SPR_TRY(bf16_inputs(c, ws, qp, kp, vp, false, &t));
    sparsepr_status fs = probe_pass(c, ws, t, qp, off_q, probes, false, c.st);
    if (fs != SPARSEPR_OK) return fs;
    std::lock_guard<std::mutex> lk(g_side_mu);
    fs = probe_solve(c, ws, probes, o_sparse, fit, c.st, side_stream(0));
    if (fs != SPARSEPR_OK) return fs;
  } else {
    SPR_TRY(zero_fit(c, ws, fit, c.st));
  }
  SPR_TRY(probe_apply(c, ws, o_sparse, probes, perm_q, pairs_sparse, out, pairs_exec, c.st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_attention(const void* q, const void* k, const void* v, sparsepr_dtype dt,
                                   const sparsepr_params* p, const sparsepr_call_buffers* b,
                                   void* out, void* ws, size_t ws_bytes, void* stream) {
  if (!b || !out) return SPARSEPR_ERR_INVALID_ARG;
  sparsepr_status s = sparsepr_partition(q, k, dt, p, b->label_q, b->label_k, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  {
    Ctx c;
    s = setup(&c, p, dt, ws, ws_bytes, stream);
    if (s != SPARSEPR_OK) return s;
    s = check_permute_args(q, k, v, b->label_q, b->label_k, b->perm_q, b->perm_k, b->off_q,
                           b->off_k, b->qp, b->kp, b->vp);
    if (s != SPARSEPR_OK) return s;
    s = permute_rows(c, q, k, v, b->label_q, b->label_k, b->perm_q, b->perm_k, b->off_q, b->off_k,
                     b->qp, b->kp, b->vp, false, ws);
    if (s != SPARSEPR_OK) return s;
    // V is read first by the attention: its gather runs beside the routing
    // (joined on every path)
    std::lock_guard<std::mutex> lk(g_side_mu);
    SideStream* ss = side_stream(0);
    const cudaStream_t side = fork_side(ss, c.st);
    const cudaError_t ev = launch_gather_rows(v, b->vp, nullptr, nullptr, b->perm_k, c.p.H, c.p.N,
                                              c.p.d, c.bf16 ? 2 : 4, side);
    s = sparsepr_route(b->qp, b->kp, dt, p, b->off_q, b->off_k, b->csr, b->k_per_head, ws,
                       ws_bytes, stream);
    const cudaError_t ej = join_side(ss, side, c.st);
    if (s != SPARSEPR_OK) return s;
    SPR_TRY(ev);
    SPR_TRY(ej);
  }
  Ctx c;
  s = setup(&c, p, dt, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  if (!b->o_sparse || !b->pairs_sparse || !b->pairs_exec || (c.p.M > 0 && !b->probes))
    return SPARSEPR_ERR_INVALID_ARG;
  if (!al16(b->o_sparse, out)) return SPARSEPR_ERR_INVALID_ARG;
  Bf16Qkv t;
  SPR_TRY(bf16_inputs(c, ws, b->qp, b->kp, b->vp, true, &t));
  const AttnArgs a = main_attn_args(c, ws, t, b->off_q, b->off_k, b->csr, b->k_per_head,
                                    b->o_sparse, b->pairs_sparse);
  SPR_TRY(launch_attn_meta(a, c.st));  // the runs the dual probe pass reads
  // The overlap pays while the dual pass's extra work (the probe rows' masked
  // pass over all keys, 4 d H M N flop) costs less than the fit latency it
  // hides (about 0.6 ms, latency-bound on H CTAs): below 4e11 flop (the 720p
  // 12-head layer: 2.4e11). Wider calls keep the five-call order.
  const double dual_flop = 4.0 * c.p.d * c.p.H * static_cast<double>(c.p.M) * c.p.N;
  if (c.p.M > 0 && dual_flop >= kDualFlopMax) {
    SPR_TRY(launch_attn_kernel(a, c.st));
    sparsepr_status fs = probe_pass(c, ws, t, b->qp, b->off_q, b->probes, false, c.st);
    if (fs != SPARSEPR_OK) return fs;
    std::lock_guard<std::mutex> lk(g_side_mu);
    fs = probe_solve(c, ws, b->probes, b->o_sparse, b->fit, c.st, side_stream(0));
    if (fs != SPARSEPR_OK) return fs;
  } else if (c.p.M > 0) {
    // the probe rows' dense and sparse outputs in one pass (work for every
    // SM, so in order before the attention), then the fit, latency-bound on
    // few SMs, on a side stream beside the attention of all rows; joined on
    // every path
    sparsepr_status fs = probe_pass(c, ws, t, b->qp, b->off_q, b->probes, true, c.st);
    if (fs != SPARSEPR_OK) return fs;
    std::lock_guard<std::mutex> lk(g_side_mu);
    SideStream* ss = side_stream(0);
    const cudaStream_t side = fork_side(ss, c.st);
    fs = probe_solve(c, ws, b->probes, nullptr, b->fit, side, side_stream(1));
    const cudaError_t ea = launch_attn_kernel(a, c.st);
    const cudaError_t ej = join_side(ss, side, c.st);
    if (fs != SPARSEPR_OK) return fs;
    SPR_TRY(ea);
    SPR_TRY(ej);
  } else {
    SPR_TRY(launch_attn_kernel(a, c.st));
    SPR_TRY(zero_fit(c, ws, b->fit, c.st));
  }
  SPR_TRY(probe_apply(c, ws, b->o_sparse, b->probes, b->perm_q, b->pairs_sparse, out,
                      b->pairs_exec, c.st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_probe_diagnostics(const sparsepr_params* p, const int32_t* probes,
                                           double* mass, double* error, double* energy,
                                           void* ws, size_t ws_bytes, void* stream) {
  Ctx c;
  sparsepr_status s = setup(&c, p, SPARSEPR_BF16, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  if (!probes || !mass || !error || !energy || c.p.M < 1) return SPARSEPR_ERR_INVALID_ARG;
  if (c.p.r > 64) return SPARSEPR_ERR_UNSUPPORTED;
  const Layout& L = c.L;
  // the leading right singular vectors of R as sparsepr_probe_correct left
  // them: the eigen solver's output for r <= kTriEigMax, the projector's selection in
  // the Gram region otherwise
  const double* vr = at<double>(ws, c.p.r <= kTriEigMax ? L.evec : L.gram);
  SPR_TRY(launch_probe_diagnostics(probes, at<float>(ws, L.lse_s), at<float>(ws, L.lse_d),
                                   at<double>(ws, L.xr), at<double>(ws, L.bmat),
                                   at<double>(ws, L.bvec), vr, c.p.H, c.p.N, c.p.M, c.p.d, c.p.r,
                                   mass, error, at<double>(ws, L.diag), energy, c.st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_support_expansion(const void* qp, const void* kp, sparsepr_dtype dt,
                                           const sparsepr_params* p, const int32_t* off_q,
                                           const int32_t* off_k, double tau, int32_t group_stride,
                                           double* individual, double* aggregate, void* ws,
                                           size_t ws_bytes, void* stream) {
  Ctx c;
  sparsepr_status s = setup(&c, p, dt, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  if (!qp || !kp || !off_q || !off_k || !individual || !aggregate || group_stride < 1 ||
      !(tau > 0.0 && tau <= 1.0))
    return SPARSEPR_ERR_INVALID_ARG;
  if (!al16(qp, kp)) return SPARSEPR_ERR_INVALID_ARG;
  int R = 0, P = 0;
  if (support_smem_bytes(c.L.Ckt, c.p.d, &R, &P) == 0) return SPARSEPR_ERR_UNSUPPORTED;
  const int H = c.p.H, Cq = c.p.Cq;
  const size_t words = (static_cast<size_t>(c.L.Ckt) + 31) / 32;
  uint32_t* bits = at<uint32_t>(ws, c.L.dscr);
  auto* sums = at<unsigned long long>(ws, c.L.dscr + align256(static_cast<size_t>(H) * Cq * words * 4));
  SPR_TRY(launch_support_expansion(qp, kp, c.bf16, off_q, c.L.Cqt + 1, off_k, c.L.Ckt, H, c.p.N,
                                   c.p.d, Cq, group_stride, c.scale, tau, bits, sums, individual,
                                   aggregate, c.st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_density_profile(const void* q, const void* k, sparsepr_dtype dt,
                                         const sparsepr_params* p, double tau, int32_t row_stride,
                                         double* density, void* ws, size_t ws_bytes,
                                         void* stream) {
  Ctx c;
  sparsepr_status s = setup(&c, p, dt, ws, ws_bytes, stream);
  if (s != SPARSEPR_OK) return s;
  if (!q || !k || !density || row_stride < 1 || !(tau > 0.0 && tau <= 1.0))
    return SPARSEPR_ERR_INVALID_ARG;
  if (!al16(q, k)) return SPARSEPR_ERR_INVALID_ARG;
  const int H = c.p.H, N = c.p.N;
  double* scr = at<double>(ws, c.L.dscr);
  auto* cnt = at<unsigned long long>(ws, c.L.dscr + align256(static_cast<size_t>(kDiagRows) * N * 8));
  SPR_TRY(launch_density(q, k, c.bf16, H, N, c.L.Nv, c.p.d, row_stride, c.scale, tau, scr, cnt,
                         density, c.st));
  return SPARSEPR_OK;
}

}  // extern "C"
