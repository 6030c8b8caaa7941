// Small dense fp64 eigen-solver for the d x d symmetric matrices of the path:
// the sampled-query metric M_K ("Partition the Support, Reconstruct the
// Residual", 2.A: k-means on the eigenvectors of M_K) and the probe residual
// Gram R^T R (2.B: leading singular vectors of the probe residuals).
//
// Cyclic two-sided Jacobi in round-robin ("tournament") order: each step
// rotates d/2 disjoint index pairs at once, d-1 steps visit every pair once
// per sweep. Rotation angles follow the symmetric 2x2 Schur decomposition
// (Golub & Van Loan, Matrix Computations, sec. 8.5). One CTA per matrix; the
// upper triangle of A (packed) and the full eigenvector matrix live in
// shared memory. Blocks whose two rotations are both the identity are
// skipped, so late sweeps cost little.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kJacobiThreads = 1024;
constexpr int kMaxSweeps = 30;

template <int D>
__device__ __forceinline__ int tri(int i, int j) {
  // packed upper triangle, i <= j
  return i * D - ((i * (i - 1)) >> 1) + (j - i);
}
template <int D>
__device__ __forceinline__ int sym(int i, int j) {
  return i <= j ? tri<D>(i, j) : tri<D>(j, i);
}

template <int D>
__global__ void __launch_bounds__(kJacobiThreads) jacobi_kernel(const double* A_in, double* eval,
                                                                double* evec, DeviceStats* stats,
                                                                int which) {
  constexpr int P = D / 2;
  constexpr int NT = D * (D + 1) / 2;
  extern __shared__ double jsm[];
  double* A = jsm;           // [NT]
  double* V = A + NT;        // [D*D], V[i*D + j]
  double* cs = V + D * D;    // [P] cos
  double* sn = cs + P;       // [P] sin
  int* pp = reinterpret_cast<int*>(sn + P);  // [P]
  int* qq = pp + P;                          // [P]
  __shared__ double red[kJacobiThreads / 32][2];
  __shared__ int stop;
  const int h = blockIdx.x;
  const double* Ah = A_in + static_cast<size_t>(h) * D * D;
  for (int t = threadIdx.x; t < D * D; t += blockDim.x) {
    const int i = t / D, j = t % D;
    if (i <= j) A[tri<D>(i, j)] = Ah[t];
    V[t] = (i == j) ? 1.0 : 0.0;
  }
  __syncthreads();
  int sweep = 0;
  for (; sweep < kMaxSweeps; ++sweep) {
    // convergence: off-diagonal Frobenius mass relative to the diagonal
    double off = 0.0, dia = 0.0;
    for (int t = threadIdx.x; t < NT; t += blockDim.x) {
      const double v = A[t];
      // t is the packed index of (i, j); diagonal entries sit at tri(i, i)
      int i = 0;
      // find the row of packed index t (rows have D, D-1, ... entries)
      int lo = 0, hi = D - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tri<D>(mid, mid) <= t) lo = mid; else hi = mid - 1;
      }
      i = lo;
      if (t == tri<D>(i, i))
        dia += v * v;
      else
        off += v * v;
    }
    off = warp_sum_f64(off);
    dia = warp_sum_f64(dia);
    if ((threadIdx.x & 31) == 0) {
      red[threadIdx.x >> 5][0] = off;
      red[threadIdx.x >> 5][1] = dia;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double o = 0.0, g = 0.0;
      for (int w = 0; w < kJacobiThreads / 32; ++w) {
        o += red[w][0];
        g += red[w][1];
      }
      stop = (o <= 1e-28 * g) || (o == 0.0);
    }
    __syncthreads();
    if (stop) break;
    for (int step = 0; step < D - 1; ++step) {
      // pairs of this step and their rotations
      if (threadIdx.x < P) {
        const int k = threadIdx.x;
        // players 0..D-1: player 0 fixed, the others rotate by `step`
        const int a = (k == 0) ? 0 : 1 + ((k - 1 + step) % (D - 1));
        const int b = 1 + ((D - 2 - k + step) % (D - 1));
        const int p0 = min(a, b), q0 = max(a, b);
        const double app = A[tri<D>(p0, p0)], aqq = A[tri<D>(q0, q0)], apq = A[tri<D>(p0, q0)];
        double c = 1.0, s = 0.0;
        if (apq != 0.0 && fabs(apq) > 1e-300 && fabs(apq) >= 1e-18 * sqrt(fabs(app * aqq))) {
          const double tau = (aqq - app) / (2.0 * apq);
          double t;
          if (fabs(tau) > 1e15)
            t = 0.5 / tau;
          else
            t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        pp[k] = p0;
        qq[k] = q0;
        cs[k] = c;
        sn[k] = s;
      }
      __syncthreads();
      // A <- J^T A J over the 2x2 blocks (a, b), a <= b
      for (int idx = threadIdx.x; idx < P * P; idx += blockDim.x) {
        const int a = idx / P, b = idx % P;
        if (a > b) continue;
        const double sa = sn[a], sb = sn[b];
        if (sa == 0.0 && sb == 0.0) continue;  // both rotations are the identity
        const int pa = pp[a], qa = qq[a];
        const double ca = cs[a];
        if (a == b) {
          const double app = A[tri<D>(pa, pa)], aqq = A[tri<D>(qa, qa)], apq = A[tri<D>(pa, qa)];
          const double t = sa / ca;
          A[tri<D>(pa, pa)] = app - t * apq;
          A[tri<D>(qa, qa)] = aqq + t * apq;
          A[tri<D>(pa, qa)] = 0.0;
        } else {
          const int pb = pp[b], qb = qq[b];
          const double cb = cs[b];
          const int i00 = sym<D>(pa, pb), i01 = sym<D>(pa, qb), i10 = sym<D>(qa, pb),
                    i11 = sym<D>(qa, qb);
          const double x00 = A[i00], x01 = A[i01], x10 = A[i10], x11 = A[i11];
          // Y = R_a^T X, R = [[c, s], [-s, c]]
          const double y00 = ca * x00 - sa * x10, y01 = ca * x01 - sa * x11;
          const double y10 = sa * x00 + ca * x10, y11 = sa * x01 + ca * x11;
          // X' = Y R_b
          A[i00] = cb * y00 - sb * y01;
          A[i01] = sb * y00 + cb * y01;
          A[i10] = cb * y10 - sb * y11;
          A[i11] = sb * y10 + cb * y11;
        }
      }
      // V <- V J
      for (int idx = threadIdx.x; idx < D * P; idx += blockDim.x) {
        const int i = idx / P, k = idx % P;
        const double s = sn[k];
        if (s == 0.0) continue;
        const double c = cs[k];
        double* vr = V + i * D;
        const int p0 = pp[k], q0 = qq[k];
        const double vp = vr[p0], vq = vr[q0];
        vr[p0] = c * vp - s * vq;
        vr[q0] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }
  for (int t = threadIdx.x; t < D * D; t += blockDim.x)
    evec[static_cast<size_t>(h) * D * D + t] = V[t];
  for (int j = threadIdx.x; j < D; j += blockDim.x)
    eval[static_cast<size_t>(h) * D + j] = A[tri<D>(j, j)];
  if (threadIdx.x == 0 && stats) atomicMax(&stats->eig_sweeps[which], sweep);
}

// wk[h, a, t] = evec[h, a, j] (* sqrt(max(lambda_j, 0))) where j has rank t
// in descending eigenvalue order (ties to the lower index), t < e.
__global__ void top_eig_projector_kernel(const double* eval, const double* evec, int d, int e,
                                         double* wk, int sqrt_scale) {
  const int h = blockIdx.x, j = threadIdx.x;
  if (j >= d) return;
  const double* ev = eval + static_cast<size_t>(h) * d;
  const double lj = ev[j];
  int rank = 0;
  for (int i = 0; i < d; ++i) {
    const double li = ev[i];
    rank += (li > lj) || (li == lj && i < j);
  }
  if (rank >= e) return;
  const double sc = sqrt_scale ? sqrt(fmax(lj, 0.0)) : 1.0;
  const double* V = evec + static_cast<size_t>(h) * d * d;
  for (int a = 0; a < d; ++a)
    wk[(static_cast<size_t>(h) * d + a) * e + rank] = V[static_cast<size_t>(a) * d + j] * sc;
}

__global__ void scale_columns_kernel(const double* vals, const double* vecs, int d, int e,
                                     double* wk) {
  const int h = blockIdx.x;
  for (int t = threadIdx.x; t < d * e; t += blockDim.x) {
    const int c = t % e;
    wk[static_cast<size_t>(h) * d * e + t] =
        vecs[static_cast<size_t>(h) * d * e + t] * sqrt(fmax(vals[static_cast<size_t>(h) * e + c], 0.0));
  }
}

template <int D>
cudaError_t launch_jacobi_d(const double* A, int H, double* eval, double* evec,
                            DeviceStats* stats, int which, cudaStream_t st) {
  constexpr int P = D / 2;
  const size_t shb = (static_cast<size_t>(D) * (D + 1) / 2 + static_cast<size_t>(D) * D + 2 * P) * 8 +
                     2 * P * 4;
  cudaError_t e = cudaFuncSetAttribute(jacobi_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(shb));
  if (e != cudaSuccess) return e;
  jacobi_kernel<D><<<H, kJacobiThreads, shb, st>>>(A, eval, evec, stats, which);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_jacobi(const double* A, int H, int d, double* eval, double* evec,
                          DeviceStats* stats, int which, cudaStream_t st) {
  if (d == 128) return launch_jacobi_d<128>(A, H, eval, evec, stats, which, st);
  if (d == 64) return launch_jacobi_d<64>(A, H, eval, evec, stats, which, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_top_eig_projector(const double* eval, const double* evec, int H, int d, int e,
                                     double* wk, bool sqrt_scale, cudaStream_t st) {
  top_eig_projector_kernel<<<H, 128, 0, st>>>(eval, evec, d, e, wk, sqrt_scale ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_scale_columns(const double* vals, const double* vecs, int H, int d, int e,
                                 double* wk, cudaStream_t st) {
  scale_columns_kernel<<<H, 256, 0, st>>>(vals, vecs, d, e, wk);
  return cudaGetLastError();
}

}  // namespace spr
