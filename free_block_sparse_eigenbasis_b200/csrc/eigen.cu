// Leading eigenpairs of the small symmetric PSD matrices of the path, in fp64:
// the sampled-query metric M_K ("Partition the Support, Reconstruct the
// Residual", 2.A: k-means on the eigenvectors of M_K) and the probe residual
// Gram R^T R (2.B: leading singular vectors of the probe residuals).
//
// Textbook dense symmetric eigensolver, specialised to "top ne of d":
//   1. Householder reduction to tridiagonal form, A = Q T Q^T with
//      Q = H_0 H_1 ... H_{d-3}, H_k = I - tau_k v_k v_k^T (Golub & Van Loan,
//      Matrix Computations, sec. 8.3.1), one CTA per matrix in shared memory;
//   2. the ne largest eigenvalues of T by bisection on Sturm-sequence counts
//      (sec. 8.4.1), one thread per eigenvalue;
//   3. their eigenvectors by inverse iteration on T - lambda I with
//      partial-pivoting tridiagonal LU (sec. 8.2.2 / 7.6.1), with
//      Gram-Schmidt inside clusters of close eigenvalues after each step;
//   4. back-transformation u = Q y, one warp per vector.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kTriThreads = 512;
constexpr int kInvIters = 3;

// Scratch per matrix (fp64): hv [D][D] Householder vectors (row k holds v_k
// at columns k+1.., v_k[0] = 1), tau [D], dg [D], od [D].
template <int D>
__global__ void __launch_bounds__(kTriThreads) tridiag_kernel(const double* A_in, double* scratch) {
  extern __shared__ double tsm[];
  double* A = tsm;              // [D*D] full symmetric (rows are read instead of columns)
  double* v = A + D * D;        // [D]
  double* w = v + D;            // [D]
  __shared__ double red[2][kTriThreads / 32];
  __shared__ double pw[kTriThreads / D][D];
  const int h = blockIdx.x;
  const double* Ah = A_in + static_cast<size_t>(h) * D * D;
  double* hv = scratch + static_cast<size_t>(h) * (D * D + 3 * D);
  double* tau = hv + D * D;
  double* dg = tau + D;
  double* od = dg + D;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int t = tid; t < D * D; t += blockDim.x) A[t] = Ah[t];
  __syncthreads();
  int nsum = 0;
  // sum over the block with one barrier (alternating buffers; every thread
  // adds the warp partials in the same order)
  auto block_sum = [&](double x) -> double {
    x = warp_sum_f64(x);
    double* rb = red[nsum++ & 1];
    if (lane == 0) rb[wid] = x;
    __syncthreads();
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < kTriThreads / 32; ++i) s += rb[i];
    return s;
  };
  constexpr int kParts = kTriThreads / D;  // row parts of the matrix-vector product
  for (int k = 0; k < D - 2; ++k) {
    const int n1 = D - k - 1;  // length of v (rows k+1 .. D-1)
    const double* Ak = A + k * D;  // row k = column k (symmetry)
    double x2 = 0.0;
    for (int i = k + 2 + tid; i < D; i += blockDim.x) x2 = fma(Ak[i], Ak[i], x2);
    x2 = block_sum(x2);
    const double alpha = Ak[k + 1];
    if (x2 == 0.0) {  // column already reduced: H_k = I
      if (tid == 0) {
        tau[k] = 0.0;
        od[k] = alpha;
      }
      for (int i = tid; i < n1; i += blockDim.x) hv[k * D + (k + 1 + i)] = (i == 0) ? 1.0 : 0.0;
      __syncthreads();
      continue;
    }
    const double beta = -copysign(sqrt(alpha * alpha + x2), alpha);
    const double tk = (beta - alpha) / beta;
    const double scl = 1.0 / (alpha - beta);
    for (int i = tid; i < n1; i += blockDim.x) {
      const double vi = (i == 0) ? 1.0 : Ak[k + 1 + i] * scl;
      v[i] = vi;
      hv[k * D + (k + 1 + i)] = vi;
    }
    if (tid == 0) {
      tau[k] = tk;
      od[k] = beta;
    }
    __syncthreads();
    // p = tau A22 v by columns (A22 symmetric): thread (column c, part) sums
    // the rows r = part, part + kParts, ...
    {
      const int c = tid % D, part = tid / D;
      double sacc = 0.0;
      if (c < n1) {
        const double* col = A + (k + 1) * D + (k + 1) + c;
        for (int r = part; r < n1; r += kParts) sacc = fma(col[r * D], v[r], sacc);
      }
      pw[part][c] = sacc;
    }
    __syncthreads();
    double pv = 0.0;
    if (tid < n1) {
      double sacc = pw[0][tid];
#pragma unroll
      for (int q = 1; q < kParts; ++q) sacc += pw[q][tid];
      const double wi = tk * sacc;
      w[tid] = wi;
      pv = wi * v[tid];
    }
    pv = block_sum(pv);
    const double kk = -0.5 * tk * pv;
    if (tid < n1) w[tid] += kk * v[tid];
    __syncthreads();
    // A22 -= v w^T + w v^T (warp = row stripe, lane = column stripe)
    for (int r = wid; r < n1; r += kTriThreads / 32) {
      const double vr = v[r], wr = w[r];
      double* Ar = A + (k + 1 + r) * D + (k + 1);
      for (int c = lane; c < n1; c += 32) Ar[c] -= vr * w[c] + wr * v[c];
    }
    __syncthreads();
  }
  for (int i = tid; i < D; i += blockDim.x) dg[i] = A[i * D + i];
  if (tid == 0) {
    od[D - 2] = A[(D - 1) * D + (D - 2)];
    od[D - 1] = 0.0;
    tau[D - 2] = 0.0;
    tau[D - 1] = 0.0;
  }
}

// Number of eigenvalues of T below x (Sturm sequence of the LDL^T pivots).
template <int D>
__device__ int sturm_count(const double* dg, const double* e2, double x, double pivmin) {
  int cnt = 0;
  double q = dg[0] - x;
  if (fabs(q) < pivmin) q = -pivmin;
  cnt += (q < 0.0);
#pragma unroll 1
  for (int i = 1; i < D; ++i) {
    q = dg[i] - x - e2[i - 1] * __drcp_rn(q);
    if (fabs(q) < pivmin) q = -pivmin;
    cnt += (q < 0.0);
  }
  return cnt;
}

// Solve (T - lam I) y = b in place (b <- y) with a partial-pivoting LU of
// the tridiagonal system. a, dl, du, du2, pv are the calling thread's work
// arrays in shared memory, element i at [i * S] (S threads interleaved).
template <int D, int S>
__device__ void tri_solve(const double* dg, const double* od, double lam, double tiny, double* a,
                          double* dl, double* du, double* du2, int* pv, double* b) {
  for (int i = 0; i < D; ++i) a[i * S] = dg[i] - lam;
  for (int i = 0; i < D - 1; ++i) {
    dl[i * S] = od[i];
    du[i * S] = od[i];
    du2[i * S] = 0.0;
  }
#pragma unroll 1
  for (int i = 0; i < D - 1; ++i) {
    const double ai = a[i * S], li = dl[i * S];
    if (fabs(ai) >= fabs(li)) {
      const double piv = (ai == 0.0) ? tiny : ai;
      a[i * S] = piv;
      const double f = li / piv;
      dl[i * S] = f;
      a[(i + 1) * S] -= f * du[i * S];
      pv[i * S] = 0;
    } else {
      const double f = ai / li;
      a[i * S] = li;
      dl[i * S] = f;
      const double t = du[i * S];
      const double an = a[(i + 1) * S];
      du[i * S] = an;
      a[(i + 1) * S] = t - f * an;
      if (i < D - 2) {
        du2[i * S] = du[(i + 1) * S];
        du[(i + 1) * S] = -f * du[(i + 1) * S];
      }
      pv[i * S] = 1;
    }
  }
  if (a[(D - 1) * S] == 0.0) a[(D - 1) * S] = tiny;
  // L solve
#pragma unroll 1
  for (int i = 0; i < D - 1; ++i) {
    if (pv[i * S] == 0) {
      b[i + 1] -= dl[i * S] * b[i];
    } else {
      const double t = b[i];
      b[i] = b[i + 1];
      b[i + 1] = t - dl[i * S] * b[i];
    }
  }
  // U solve
  b[D - 1] /= a[(D - 1) * S];
  b[D - 2] = (b[D - 2] - du[(D - 2) * S] * b[D - 1]) / a[(D - 2) * S];
#pragma unroll 1
  for (int i = D - 3; i >= 0; --i)
    b[i] = (b[i] - du[i * S] * b[i + 1] - du2[i * S] * b[i + 2]) / a[i * S];
}

constexpr int kEigThreads = 256;

// One CTA per matrix, ne <= 32 eigenpairs (largest first): bisection and
// inverse iteration by thread t, clustered Gram-Schmidt by warp 0, then
// back-transformation by warp t % 8. Writes evals [H, ne] and evecs [H, D, ne].
template <int D>
constexpr size_t eig_work_bytes() {
  return static_cast<size_t>(4) * D * 32 * 8 + static_cast<size_t>(D) * 32 * 4;
}
static_assert(eig_work_bytes<128>() >= (128 * 128 + 128) * 8 &&
                  eig_work_bytes<64>() >= (64 * 64 + 64) * 8,
              "the back-transformation reuses the work space for the Householder vectors");

template <int D>
__global__ void __launch_bounds__(kEigThreads) tri_eig_kernel(const double* scratch, int ne,
                                                       double* evals, double* evecs) {
  extern __shared__ double eig_work[];  // inverse-iteration work arrays, 32 threads interleaved
  __shared__ double dg[D], od[D], e2[D];
  __shared__ double lam[32];
  __shared__ double Y[32][D + 1];  // padded: thread t walks row t
  __shared__ double tnorm;
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const double* hv = scratch + static_cast<size_t>(h) * (D * D + 3 * D);
  const double* tau = hv + D * D;
  for (int i = tid; i < D; i += blockDim.x) {
    dg[i] = tau[D + i];
    od[i] = tau[2 * D + i];
  }
  __syncthreads();
  for (int i = tid; i < D; i += blockDim.x) e2[i] = (i < D - 1) ? od[i] * od[i] : 0.0;
  if (tid == 0) {
    double m = 0.0;
    for (int i = 0; i < D; ++i)
      m = fmax(m, fabs(dg[i]) + (i > 0 ? fabs(od[i - 1]) : 0.0) + (i < D - 1 ? fabs(od[i]) : 0.0));
    tnorm = m;
  }
  __syncthreads();
  const double eps = 1.1102230246251565e-16;
  double emax2 = 0.0;
  for (int i = 0; i < D - 1; ++i) emax2 = fmax(emax2, e2[i]);
  const double pivmin = 2.2250738585072014e-308 * fmax(1.0, emax2);
  // multisection: eight threads per wanted eigenvalue (rank e_i = tid / 8,
  // ascending index D-1-e_i) evaluate the Sturm count at eight interior
  // points of the current interval, which shrinks nine-fold per round
  {
    const int e_i = tid >> 3, q = tid & 7;
    const bool act = e_i < ne;
    const int m = D - 1 - e_i;
    double lo = -tnorm - 1.0, hi = tnorm + 1.0;
    for (int it = 0; it < 100; ++it) {
      const double w = hi - lo;
      const bool done = !(w > 4.0 * eps * fmax(fabs(lo), fabs(hi)) + pivmin);
      if (__all_sync(0xffffffffu, done || !act)) break;
      bool pred = false;
      if (act && !done) pred = sturm_count<D>(dg, e2, lo + w * (q + 1) * (1.0 / 9.0), pivmin) <= m;
      const unsigned bal = __ballot_sync(0xffffffffu, pred);
      const int nt = __popc((bal >> ((lane >> 3) * 8)) & 0xFFu);  // points below lambda
      if (act && !done) {
        const double nlo = nt > 0 ? lo + w * nt * (1.0 / 9.0) : lo;
        const double nhi = nt < 8 ? lo + w * (nt + 1) * (1.0 / 9.0) : hi;
        lo = nlo;
        hi = nhi;
      }
    }
    if (act && q == 0) lam[e_i] = 0.5 * (lo + hi);
  }
  __syncthreads();
  // inverse iteration from a fixed, index-dependent start vector
  double* wk = eig_work + (tid & 31);
  int* pv = reinterpret_cast<int*>(eig_work + 4 * D * 32) + (tid & 31);
  const double tiny = eps * fmax(tnorm, 1e-300);
  if (tid < ne)
    for (int i = 0; i < D; ++i) Y[tid][i] = 1.0 + 0.5 * sin(0.7 * (i + 1) * (tid + 1));
  const double ortol = 1e-3 * tnorm;
  for (int it = 0; it < kInvIters; ++it) {
    if (tid < ne) {
      double* b = Y[tid];
      tri_solve<D, 32>(dg, od, lam[tid], tiny, wk, wk + D * 32, wk + 2 * D * 32, wk + 3 * D * 32, pv, b);
      double s = 0.0;
      for (int i = 0; i < D; ++i) s = fma(b[i], b[i], s);
      const double inv = 1.0 / sqrt(s);
      for (int i = 0; i < D; ++i) b[i] *= inv;
    }
    __syncthreads();
    // Gram-Schmidt against earlier vectors of the same cluster, in rank order
    if (wid == 0) {
      for (int t = 1; t < ne; ++t) {
        for (int s = t - 1; s >= 0; --s) {
          if (fabs(lam[s] - lam[s + 1]) > ortol) break;  // cluster boundary
          double dot = 0.0;
          for (int i = lane; i < D; i += 32) dot = fma(Y[s][i], Y[t][i], dot);
          dot = warp_sum_f64(dot);
          for (int i = lane; i < D; i += 32) Y[t][i] -= dot * Y[s][i];
          __syncwarp();
        }
        double nn = 0.0;
        for (int i = lane; i < D; i += 32) nn = fma(Y[t][i], Y[t][i], nn);
        nn = warp_sum_f64(nn);
        const double inv = 1.0 / sqrt(nn);
        for (int i = lane; i < D; i += 32) Y[t][i] *= inv;
        __syncwarp();
      }
    }
    __syncthreads();
  }
  // back-transformation: u = H_0 (H_1 (... H_{D-3} y)), warp w owns vectors
  // w, w + 8, ...; the Householder vectors and tau are first staged in the
  // (now free) inverse-iteration work space
  double* hs = eig_work;          // [D][D]
  double* ts = eig_work + D * D;  // [D]
  for (int i = tid; i < D * D; i += blockDim.x) hs[i] = hv[i];
  for (int i = tid; i < D; i += blockDim.x) ts[i] = tau[i];
  __syncthreads();
  for (int t = wid; t < ne; t += kEigThreads / 32) {
    double* y = Y[t];
    for (int k = D - 3; k >= 0; --k) {
      const double tk = ts[k];
      if (tk == 0.0) continue;
      const double* hk = hs + k * D;
      double dot = 0.0;
      for (int i = k + 1 + lane; i < D; i += 32) dot = fma(hk[i], y[i], dot);
      dot = warp_sum_f64(dot) * tk;
      for (int i = k + 1 + lane; i < D; i += 32) y[i] -= dot * hk[i];
      __syncwarp();
    }
    for (int i = lane; i < D; i += 32)
      evecs[(static_cast<size_t>(h) * D + i) * ne + t] = y[i];
    if (lane == 0) evals[static_cast<size_t>(h) * ne + t] = lam[t];
  }
}

template <int D>
cudaError_t launch_d(const double* A, int H, int ne, double* evals, double* evecs,
                     double* scratch, cudaStream_t st) {
  const size_t shb = (static_cast<size_t>(D) * D + 2 * D) * 8;
  cudaError_t e = cudaFuncSetAttribute(tridiag_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(shb));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(tri_eig_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(eig_work_bytes<D>()));
  if (e != cudaSuccess) return e;
  tridiag_kernel<D><<<H, kTriThreads, shb, st>>>(A, scratch);
  tri_eig_kernel<D><<<H, kEigThreads, eig_work_bytes<D>(), st>>>(scratch, ne, evals, evecs);
  return cudaGetLastError();
}

}  // namespace

size_t sym_eigs_scratch_doubles(int H, int d) {
  return static_cast<size_t>(H) * (static_cast<size_t>(d) * d + 3 * d);
}

cudaError_t launch_sym_eigs(const double* A, int H, int d, int ne, double* evals, double* evecs,
                            double* scratch, cudaStream_t st) {
  if (ne < 1 || ne > 32 || ne > d) return cudaErrorInvalidValue;
  if (d == 128) return launch_d<128>(A, H, ne, evals, evecs, scratch, st);
  if (d == 64) return launch_d<64>(A, H, ne, evals, evecs, scratch, st);
  return cudaErrorInvalidValue;
}

}  // namespace spr
