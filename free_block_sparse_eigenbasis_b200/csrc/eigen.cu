// Leading eigenpairs (up to 64) of the small symmetric PSD matrices of the path, in fp64:
// the sampled-query metric M_K ("Partition the Support, Reconstruct the
// Residual", 2.A: k-means on the eigenvectors of M_K) and the probe residual
// Gram R^T R (2.B: leading singular vectors of the probe residuals).
//
// Textbook dense symmetric eigensolver, specialised to "top ne of d":
//   1. Householder reduction to tridiagonal form, A = Q T Q^T with
//      Q = H_0 H_1 ... H_{d-3}, H_k = I - tau_k v_k v_k^T (Golub & Van Loan,
//      Matrix Computations, sec. 8.3.1), one CTA per matrix held in its
//      threads' registers;
//   2. the ne largest eigenvalues of T by multisection on Sturm-sequence
//      counts (sec. 8.4.1): 8 to 32 threads per eigenvalue, one point each;
//   3. their eigenvectors by inverse iteration on T - lambda I with one
//      partial-pivoting tridiagonal LU per eigenvalue reused by every step
//      (sec. 8.2.2 / 7.6.1), and classical Gram-Schmidt applied twice inside
//      clusters of close eigenvalues after each step;
//   4. back-transformation u = Q y, each warp applying every reflection to
//      its (up to two) vectors at once.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kTriThreads = 512;
constexpr int kInvIters = 3;

// Scratch per matrix (fp64): hv [D][D] Householder vectors (row k holds v_k
// at columns k+1.., v_k[0] = 1), tau [D], dg [D], od [D].
//
// The matrix lives in registers: warp w holds rows w, w + 16, .. (kRpw of
// them) and lane l columns l, l + 32, .. (kCpl), so row k (= column k by
// symmetry) sits in one warp, which forms v_k, tau_k and beta_k from it
// alone. Per column k:
//   1. the warp holding row k publishes v_k and tau_k (alternating buffers,
//      so that it can run ahead while other warps still read the last v);
//   2. every warp forms its rows of p = tau A v: per-lane partial dots, then
//      a transposed butterfly over the lanes that leaves each row's sum in a
//      group of lanes; the block sums v^T p from per-warp partials (one
//      fixed order, identical in every thread);
//   3. every thread updates its entries, A -= v w^T + w v^T with
//      w = p - (tau / 2)(v^T p) v (Golub & Van Loan, sec. 8.3.1).
// Every thread updates all its entries without branches (v and w are zero
// at indices <= k, which leaves those entries unchanged): a skip test per
// entry costs more than the two FMAs it saves. Two barriers per column.
constexpr int kTriWarps = kTriThreads / 32;

template <int D>
__global__ void __launch_bounds__(kTriThreads, 1)
    tridiag_kernel(const double* A_in, double* scratch) {
  constexpr int kRpw = D / kTriWarps;  // rows per warp
  constexpr int kCpl = D / 32;         // columns per lane
  constexpr int kLgR = kRpw == 8 ? 3 : (kRpw == 4 ? 2 : (kRpw == 2 ? 1 : 0));
  static_assert((1 << kLgR) == kRpw, "rows per warp must be a power of two up to 8");
  constexpr int kGroup = 32 >> kLgR;  // lanes that share one row's sum
  __shared__ double vb[2][D + 1];     // v (and tau at [D]), two buffers
  __shared__ double pb[D];            // p = tau A v (zero at rows <= k)
  __shared__ double part[kTriWarps];  // per-warp partials of v^T p
  const int h = blockIdx.x;
  const double* Ah = A_in + static_cast<size_t>(h) * D * D;
  double* hv = scratch + static_cast<size_t>(h) * (D * D + 3 * D);
  double* tau = hv + D * D;
  double* dg = tau + D;
  double* od = dg + D;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  double a[kRpw][kCpl];
#pragma unroll
  for (int r = 0; r < kRpw; ++r)
#pragma unroll
    for (int c = 0; c < kCpl; ++c) a[r][c] = Ah[(wid + kTriWarps * r) * D + lane + 32 * c];
  const int rho = lane >> (5 - kLgR);  // the row slot whose sum this lane ends with
  for (int k = 0; k < D - 2; ++k) {
    double* vv = vb[k & 1];
    if (wid == (k % kTriWarps)) {
      const int rk = k / kTriWarps;
      double x[kCpl];
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        x[c] = 0.0;
#pragma unroll
        for (int r = 0; r < kRpw; ++r) x[c] = (r == rk) ? a[r][c] : x[c];
      }
      double x2 = 0.0, al = 0.0;
      const int ca = (k + 1) >> 5;
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        const int j = lane + 32 * c;
        if (j > k + 1) x2 = fma(x[c], x[c], x2);
        al = (c == ca) ? x[c] : al;
      }
      x2 = warp_sum_f64(x2);
      const double alpha = __shfl_sync(0xffffffffu, al, (k + 1) & 31);
      double tk = 0.0, beta = alpha, scl = 0.0;
      if (x2 != 0.0) {  // else the column is already reduced: H_k = I
        beta = -copysign(sqrt(alpha * alpha + x2), alpha);
        tk = (beta - alpha) / beta;
        scl = 1.0 / (alpha - beta);
      }
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        const int j = lane + 32 * c;
        const double vj = (j == k + 1) ? 1.0 : (j > k + 1 ? x[c] * scl : 0.0);
        vv[j] = vj;
        hv[k * D + j] = vj;
      }
      if (lane == 0) {
        vv[D] = tk;
        tau[k] = tk;
        od[k] = beta;
      }
    }
    __syncthreads();
    const double tk = vv[D];
    double vc[kCpl];
#pragma unroll
    for (int c = 0; c < kCpl; ++c) vc[c] = vv[lane + 32 * c];
    {
      // every entry, without branches: v is zero at indices <= k, and the
      // rows <= k are masked below
      double t[kRpw];
#pragma unroll
      for (int r = 0; r < kRpw; ++r) t[r] = 0.0;
#pragma unroll
      for (int c = 0; c < kCpl; ++c)
#pragma unroll
        for (int r = 0; r < kRpw; ++r) t[r] = fma(a[r][c], vc[c], t[r]);
      // transposed butterfly: halve the rows held per lane at each step
#pragma unroll
      for (int st = 0; st < kLgR; ++st) {
        const int half = kRpw >> (st + 1);
        const int m = 16 >> st;
        const bool hi = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const double send = hi ? t[i] : t[i + half];
          const double keep = hi ? t[i + half] : t[i];
          t[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
#pragma unroll
      for (int o = kGroup >> 1; o > 0; o >>= 1) t[0] += __shfl_xor_sync(0xffffffffu, t[0], o);
      const int row = wid + kTriWarps * rho;
      const double pr = (row > k) ? tk * t[0] : 0.0;
      const bool leader = (lane & (kGroup - 1)) == 0;
      if (leader) pb[row] = pr;
      const double pv = warp_sum_f64(leader ? pr * vv[row] : 0.0);
      if (lane == 0) part[wid] = pv;
    }
    __syncthreads();
    double pv = 0.0;
#pragma unroll
    for (int i = 0; i < kTriWarps; ++i) pv += part[i];
    const double hc = 0.5 * tk * pv;
    double wc[kCpl];
#pragma unroll
    for (int c = 0; c < kCpl; ++c) {
      const int j = lane + 32 * c;
      wc[c] = (j > k) ? fma(-hc, vc[c], pb[j]) : 0.0;
    }
    // every entry, without branches: v and w are zero at indices <= k, so
    // those entries are left unchanged
#pragma unroll
    for (int r = 0; r < kRpw; ++r) {
      const int i = wid + kTriWarps * r;
      const double vr = vv[i];
      const double wr = (i > k) ? fma(-hc, vr, pb[i]) : 0.0;
#pragma unroll
      for (int c = 0; c < kCpl; ++c) a[r][c] = fma(-wr, vc[c], fma(-vr, wc[c], a[r][c]));
    }
  }
#pragma unroll
  for (int r = 0; r < kRpw; ++r)
#pragma unroll
    for (int c = 0; c < kCpl; ++c) {
      const int i = wid + kTriWarps * r, j = lane + 32 * c;
      if (i == j) dg[i] = a[r][c];
      if (i == D - 1 && j == D - 2) od[D - 2] = a[r][c];
    }
  if (tid == 0) {
    od[D - 1] = 0.0;
    tau[D - 2] = 0.0;
    tau[D - 1] = 0.0;
  }
}

// Gershgorin bound max_i |d_i| + |e_{i-1}| + |e_i| of T and the largest
// squared off-diagonal entry, by the calling warp (lanes over the rows, then
// a max over the lanes: the result does not depend on the order).
template <int D>
__device__ __forceinline__ void tri_bounds(const double* dg, const double* od, int lane,
                                           double* tnorm, double* emax2) {
  double m = 0.0, e = 0.0;
  for (int i = lane; i < D; i += 32) {
    m = fmax(m, fabs(dg[i]) + (i > 0 ? fabs(od[i - 1]) : 0.0) + (i < D - 1 ? fabs(od[i]) : 0.0));
    if (i < D - 1) e = fmax(e, od[i] * od[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    e = fmax(e, __shfl_xor_sync(0xffffffffu, e, o));
  }
  if (lane == 0) {
    *tnorm = m;
    if (emax2) *emax2 = e;
  }
}

// Number of eigenvalues of T below each of P points x (Sturm sequences of
// the LDL^T pivots), the P recurrences interleaved.
template <int D, int P>
__device__ void sturm_counts(const double* dg, const double* e2, const double (&x)[P],
                             double pivmin, int (&cnt)[P]) {
  double q[P];
#pragma unroll
  for (int p = 0; p < P; ++p) {
    q[p] = dg[0] - x[p];
    if (fabs(q[p]) < pivmin) q[p] = -pivmin;
    cnt[p] = (q[p] < 0.0);
  }
#pragma unroll 1
  for (int i = 1; i < D; ++i) {
    const double d = dg[i], e = e2[i - 1];
#pragma unroll
    for (int p = 0; p < P; ++p) {
      q[p] = d - x[p] - e * rcp_newton(q[p]);
      if (fabs(q[p]) < pivmin) q[p] = -pivmin;
      cnt[p] += (q[p] < 0.0);
    }
  }
}

// Partial-pivoting LU of the tridiagonal T - lam I (LAPACK dgttrf layout):
// multipliers dl, pivots pv, U's diagonal (stored as its reciprocal in a),
// first and second superdiagonals du, du2. The arrays are the calling
// thread's work arrays in shared memory, element i at [i * S] (S threads
// interleaved).
template <int D, int S>
__device__ void tri_factor(const double* dg, const double* od, double lam, double tiny, double* a,
                           double* dl, double* du, double* du2, int* pv) {
  // the current diagonal entry and superdiagonal entry (as the previous
  // step's elimination left them) are carried in registers, and each step
  // picks its pivot row by selects, so that the chain from one step to the
  // next holds no shared-memory round trip and no divergent branch
  double a_cur = dg[0] - lam;
  double du_cur = od[0];
#pragma unroll 2
  for (int i = 0; i < D - 1; ++i) {
    const double li = od[i];
    const double a_nx = dg[i + 1] - lam;
    const double du_nx = (i < D - 2) ? od[i + 1] : 0.0;
    const bool sw = !(fabs(a_cur) >= fabs(li));  // pivot on the subdiagonal row
    const double piv = sw ? li : (a_cur == 0.0 ? tiny : a_cur);
    const double f = (sw ? a_cur : li) / piv;
    a[i * S] = piv;
    dl[i * S] = f;
    pv[i * S] = sw ? 1 : 0;
    du[i * S] = sw ? a_nx : du_cur;
    if (i < D - 2) du2[i * S] = sw ? du_nx : 0.0;
    a_cur = sw ? fma(-f, a_nx, du_cur) : fma(-f, du_cur, a_nx);
    du_cur = sw ? -f * du_nx : du_nx;
  }
  a[(D - 1) * S] = (a_cur == 0.0) ? tiny : a_cur;
#pragma unroll 8
  for (int i = 0; i < D; ++i) a[i * S] = 1.0 / a[i * S];  // independent: unrolled to overlap
}

// b <- (T - lam I)^-1 b with the factors of tri_factor; returns |b|^2 of the
// result. The element that the next step updates is carried in registers.
template <int D, int S>
__device__ double tri_apply(const double* ra, const double* dl, const double* du,
                            const double* du2, const int* pv, double* b) {
  double cur = b[0];
#pragma unroll 4
  for (int i = 0; i < D - 1; ++i) {
    const double nx = b[i + 1];
    const bool sw = pv[i * S] != 0;
    const double top = sw ? nx : cur;
    const double bot = sw ? cur : nx;
    b[i] = top;
    cur = fma(-dl[i * S], top, bot);
  }
  double x1 = cur * ra[(D - 1) * S];                               // x_{i+2}
  double x0 = (b[D - 2] - du[(D - 2) * S] * x1) * ra[(D - 2) * S];  // x_{i+1}
  b[D - 1] = x1;
  b[D - 2] = x0;
  double nn = fma(x1, x1, x0 * x0);
#pragma unroll 4
  for (int i = D - 3; i >= 0; --i) {
    const double xi = (b[i] - du[i * S] * x0 - du2[i * S] * x1) * ra[i * S];
    b[i] = xi;
    nn = fma(xi, xi, nn);
    x1 = x0;
    x0 = xi;
  }
  return nn;
}

// Fixed start vector of inverse iteration: components in [0.5, 1.5) from an
// integer hash of (index, eigenvalue rank), so that no start vector is
// orthogonal to an eigenvector by construction and none costs a
// transcendental per component.
__device__ __forceinline__ double start_component(int i, int v) {
  uint32_t x = static_cast<uint32_t>(i) * 0x9E3779B1u ^ (static_cast<uint32_t>(v) + 0x7F4A7C15u) * 0x85EBCA77u;
  x ^= x >> 15;
  x *= 0x2C1B3C6Du;
  x ^= x >> 12;
  return 0.5 + static_cast<double>(x) * (1.0 / 4294967296.0);
}

constexpr int kEigThreads = 512;
constexpr int kEigWarps = kEigThreads / 32;
constexpr int kEigMax = kTriEigMax;  // eigenpairs per matrix
constexpr int kInvBatch = 32;  // eigenvalues in inverse iteration at a time

// The ne largest eigenvalues of the tridiagonal T of each matrix by
// multisection on Sturm-sequence counts (Golub & Van Loan, sec. 8.4.1): one
// warp per eigenvalue (rank e_i, ascending index D-1-e_i), each lane
// evaluating the count at one of 32 interior points of the current interval,
// which shrinks 33-fold per round, to 4 eps |lambda| + pivmin. A few warps per
// CTA and several CTAs per matrix, so that the fp64 recurrences of the
// eigenvalues spread over the SMs instead of sharing one. Writes
// evals[h, e_i].
constexpr int kBisWarps = 2;

template <int D>
__global__ void __launch_bounds__(kBisWarps * 32) multisect_kernel(const double* scratch, int ne,
                                                                  double* evals) {
  __shared__ double dg[D], od[D], e2[D];
  __shared__ double tnorm, emax2_s;
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const double* tau = scratch + static_cast<size_t>(h) * (D * D + 3 * D) + D * D;
  for (int i = tid; i < D; i += blockDim.x) {
    dg[i] = tau[D + i];
    od[i] = tau[2 * D + i];
    e2[i] = (i < D - 1) ? od[i] * od[i] : 0.0;
  }
  __syncthreads();
  if (tid < 32) tri_bounds<D>(dg, od, lane, &tnorm, &emax2_s);  // the same bound as tri_eig_kernel's
  __syncthreads();
  const int e_i = blockIdx.y * kBisWarps + (tid >> 5);
  if (e_i >= ne) return;  // the whole warp
  const double eps = 1.1102230246251565e-16;
  const double emax2 = emax2_s;
  const double pivmin = 2.2250738585072014e-308 * fmax(1.0, emax2);
  const int m = D - 1 - e_i;
  const double inv_parts = 1.0 / 33.0;
  double lo = -tnorm - 1.0, hi = tnorm + 1.0;
  for (int it = 0; it < 200; ++it) {
    const double w = hi - lo;
    if (!(w > 4.0 * eps * fmax(fabs(lo), fabs(hi)) + pivmin)) break;  // warp-uniform
    double x[1] = {lo + w * (lane + 1) * inv_parts};
    int cnt[1] = {D};
    sturm_counts<D, 1>(dg, e2, x, pivmin, cnt);
    const int nt = __popc(__ballot_sync(0xffffffffu, cnt[0] <= m));  // points below lambda
    const double nlo = nt > 0 ? lo + w * nt * inv_parts : lo;
    const double nhi = nt < 32 ? lo + w * (nt + 1) * inv_parts : hi;
    lo = nlo;
    hi = nhi;
  }
  if (lane == 0) evals[static_cast<size_t>(h) * ne + e_i] = 0.5 * (lo + hi);
}

// One CTA of 512 threads per matrix, ne <= 64 eigenpairs (largest first),
// from the eigenvalues multisect_kernel left in evals: inverse iteration by
// thread t (one LU, three solves) for batches of 32 eigenvalues, Gram-Schmidt
// inside clusters by all warps, then the back-transformation with warp w
// owning vectors w, w + 16, ... Writes evals [H, ne] and evecs [H, D, ne].
// Dynamic shared memory: the inverse-iteration work arrays of one batch (32
// threads interleaved; later the staged Householder vectors), then the
// vectors Y [kEigMax][D + 1].
template <int D>
constexpr size_t eig_work_bytes() {
  return static_cast<size_t>(4) * D * kInvBatch * 8 + static_cast<size_t>(D) * kInvBatch * 4;
}
template <int D>
constexpr size_t eig_smem_bytes() {
  return eig_work_bytes<D>() + static_cast<size_t>(kEigMax) * (D + 1) * 8;
}
static_assert(eig_work_bytes<128>() >= (128 * 128 + 128) * 8 &&
                  eig_work_bytes<64>() >= (64 * 64 + 64) * 8,
              "the back-transformation reuses the work space for the Householder vectors");
static_assert(eig_smem_bytes<128>() <= 232448 - 4096, "shared memory");

template <int D>
__global__ void __launch_bounds__(kEigThreads, 1) tri_eig_kernel(const double* scratch, int ne,
                                                       double* evals, double* evecs) {
  extern __shared__ double eig_work[];  // inverse-iteration work arrays, then Y
  double (*Y)[D + 1] = reinterpret_cast<double (*)[D + 1]>(eig_work + eig_work_bytes<D>() / 8);
  __shared__ double dg[D], od[D];
  __shared__ double lam[kEigMax];
  __shared__ double tnorm;
  __shared__ double gdot[kEigMax], gred[kEigWarps];
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const double* hv = scratch + static_cast<size_t>(h) * (D * D + 3 * D);
  const double* tau = hv + D * D;
  for (int i = tid; i < D; i += blockDim.x) {
    dg[i] = tau[D + i];
    od[i] = tau[2 * D + i];
  }
  __syncthreads();
  if (tid < 32) tri_bounds<D>(dg, od, lane, &tnorm, nullptr);
  __syncthreads();
  const double eps = 1.1102230246251565e-16;
  // the eigenvalues, from multisect_kernel
  for (int i = tid; i < ne; i += blockDim.x) lam[i] = evals[static_cast<size_t>(h) * ne + i];
  __syncthreads();
  // inverse iteration from a fixed, index-dependent start vector, 32
  // eigenvalues at a time; Gram-Schmidt against the earlier vectors of the
  // same cluster (rank order; classical Gram-Schmidt applied twice), all warps
  double* wk = eig_work + (tid & 31);
  int* pv = reinterpret_cast<int*>(eig_work + 4 * D * kInvBatch) + (tid & 31);
  const double tiny = eps * fmax(tnorm, 1e-300);
  const double ortol = 1e-3 * tnorm;
  double* wa = wk;
  double* wdl = wk + D * kInvBatch;
  double* wdu = wk + 2 * D * kInvBatch;
  double* wdu2 = wk + 3 * D * kInvBatch;
  for (int b0 = 0; b0 < ne; b0 += kInvBatch) {
    const int nb = min(kInvBatch, ne - b0);
    const int vi = b0 + tid;  // this thread's eigenvalue (tid < nb)
    if (tid < nb) {
#pragma unroll 4
      for (int i = 0; i < D; ++i) Y[vi][i] = start_component(i, vi);
      tri_factor<D, kInvBatch>(dg, od, lam[vi], tiny, wa, wdl, wdu, wdu2, pv);
    }
    for (int it = 0; it < kInvIters; ++it) {
      if (tid < nb) {
        double* bvec = Y[vi];
        const double sacc = tri_apply<D, kInvBatch>(wa, wdl, wdu, wdu2, pv, bvec);
        const double inv = 1.0 / sqrt(sacc);
#pragma unroll 4
        for (int i = 0; i < D; ++i) bvec[i] *= inv;
      }
      __syncthreads();
      for (int t = (b0 > 0 ? b0 : 1); t < b0 + nb; ++t) {
        int s0 = t;
        while (s0 > 0 && fabs(lam[s0 - 1] - lam[s0]) <= ortol) --s0;
        if (s0 == t) continue;  // the same for every thread
        for (int pass = 0; pass < 2; ++pass) {
          for (int sv = s0 + wid; sv < t; sv += kEigWarps) {
            double dot = 0.0;
            for (int i = lane; i < D; i += 32) dot = fma(Y[sv][i], Y[t][i], dot);
            dot = warp_sum_f64(dot);
            if (lane == 0) gdot[sv] = dot;
          }
          __syncthreads();
          if (tid < D) {
            double yv = Y[t][tid];
            for (int sv = s0; sv < t; ++sv) yv -= gdot[sv] * Y[sv][tid];
            Y[t][tid] = yv;
          }
          __syncthreads();
        }
        double nn = (tid < D) ? Y[t][tid] * Y[t][tid] : 0.0;
        nn = warp_sum_f64(nn);
        if (lane == 0) gred[wid] = nn;
        __syncthreads();
        double tot = 0.0;
#pragma unroll
        for (int w = 0; w < kEigWarps; ++w) tot += gred[w];
        if (tid < D) Y[t][tid] *= 1.0 / sqrt(tot);
        __syncthreads();
      }
    }
    __syncthreads();  // the work arrays are reused by the next batch
  }
  // back-transformation: u = H_0 (H_1 (... H_{D-3} y)); the Householder
  // vectors (row k holds v_k, zero at columns <= k) and tau are first staged
  // in the (now free) work space
  double* hs = eig_work;          // [D][D]
  double* ts = eig_work + D * D;  // [D]
  for (int i = tid; i < D * D; i += blockDim.x) hs[i] = hv[i];
  for (int i = tid; i < D; i += blockDim.x) ts[i] = tau[i];
  __syncthreads();
  // warp w owns vectors w, w + 16, w + 32, w + 48, held in registers (lane l:
  // components l, l + 32, ..), and applies each reflection to all of them at
  // once; the warps run independently
  constexpr int kVpw = kEigMax / kEigWarps;
  constexpr int kCpl = D / 32;
  const int nv = ne > wid ? (ne - wid + kEigWarps - 1) / kEigWarps : 0;
  double y[kVpw][kCpl];
#pragma unroll
  for (int v = 0; v < kVpw; ++v)
#pragma unroll
    for (int j = 0; j < kCpl; ++j) y[v][j] = (v < nv) ? Y[wid + kEigWarps * v][lane + 32 * j] : 0.0;
  for (int k = D - 3; k >= 0; --k) {
    const double tk = ts[k];
    if (tk == 0.0) continue;
    const double* hk = hs + k * D;
    double hj[kCpl];
#pragma unroll
    for (int j = 0; j < kCpl; ++j) hj[j] = hk[lane + 32 * j];
    double dot[kVpw];
#pragma unroll
    for (int v = 0; v < kVpw; ++v) {
      dot[v] = 0.0;
#pragma unroll
      for (int j = 0; j < kCpl; ++j) dot[v] = fma(hj[j], y[v][j], dot[v]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int v = 0; v < kVpw; ++v) dot[v] += __shfl_xor_sync(0xffffffffu, dot[v], o);
#pragma unroll
    for (int v = 0; v < kVpw; ++v) {
      const double f = dot[v] * tk;
#pragma unroll
      for (int j = 0; j < kCpl; ++j) y[v][j] = fma(-f, hj[j], y[v][j]);
    }
  }
  for (int v = 0; v < nv; ++v) {
    const int t = wid + kEigWarps * v;
#pragma unroll
    for (int j = 0; j < kCpl; ++j) {
      double yv = 0.0;
#pragma unroll
      for (int u = 0; u < kVpw; ++u) yv = (u == v) ? y[u][j] : yv;
      evecs[(static_cast<size_t>(h) * D + lane + 32 * j) * ne + t] = yv;
    }
    if (lane == 0) evals[static_cast<size_t>(h) * ne + t] = lam[t];
  }
}

template <int D>
cudaError_t launch_d(const double* A, int H, int ne, double* evals, double* evecs,
                     double* scratch, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tri_eig_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(eig_smem_bytes<D>()));
  if (e != cudaSuccess) return e;
  tridiag_kernel<D><<<H, kTriThreads, 0, st>>>(A, scratch);
  multisect_kernel<D><<<dim3(H, (ne + kBisWarps - 1) / kBisWarps), kBisWarps * 32, 0, st>>>(
      scratch, ne, evals);
  tri_eig_kernel<D><<<H, kEigThreads, eig_smem_bytes<D>(), st>>>(scratch, ne, evals, evecs);
  return cudaGetLastError();
}

}  // namespace

size_t sym_eigs_scratch_doubles(int H, int d) {
  return static_cast<size_t>(H) * (static_cast<size_t>(d) * d + 3 * d);
}

cudaError_t launch_sym_eigs(const double* A, int H, int d, int ne, double* evals, double* evecs,
                            double* scratch, cudaStream_t st) {
  if (ne < 1 || ne > kEigMax || ne > d) return cudaErrorInvalidValue;
  if (d == 128) return launch_d<128>(A, H, ne, evals, evecs, scratch, st);
  if (d == 64) return launch_d<64>(A, H, ne, evals, evecs, scratch, st);
  return cudaErrorInvalidValue;
}

namespace {
// err[i] = |rcp_newton(x[i]) - 1/x[i]| in units of the last place of the
// correctly rounded 1/x[i] (__drcp_rn)
__global__ void check_reciprocal_kernel(const double* x, long long n, double* err) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const double r = __drcp_rn(x[i]);
  const double y = rcp_newton(x[i]);
  int ex = 0;
  frexp(r, &ex);
  err[i] = fabs(y - r) / ldexp(1.0, ex - 53);
}
}  // namespace

cudaError_t launch_check_reciprocal(const double* x, long long n, double* err, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  check_reciprocal_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(x, n, err);
  return cudaGetLastError();
}

}  // namespace spr
