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
// shared memory.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kJacobiThreads = 512;
constexpr int kMaxSweeps = 24;

__device__ __forceinline__ int tri(int i, int j, int d) {
  // packed upper triangle, i <= j
  return i * d - (i * (i - 1)) / 2 + (j - i);
}
__device__ __forceinline__ int sym(int i, int j, int d) {
  return i <= j ? tri(i, j, d) : tri(j, i, d);
}

__global__ void __launch_bounds__(kJacobiThreads) jacobi_kernel(const double* A_in, int d,
                                                                double* eval, double* evec,
                                                                DeviceStats* stats) {
  extern __shared__ double jsm[];
  const int P = d / 2;
  const int ntri = d * (d + 1) / 2;
  double* A = jsm;              // [ntri]
  double* V = A + ntri;         // [d*d], V[i*d + j]
  double* cs = V + d * d;       // [P] cos
  double* sn = cs + P;          // [P] sin
  int* pp = reinterpret_cast<int*>(sn + P);  // [P]
  int* qq = pp + P;                          // [P]
  __shared__ double red[kJacobiThreads / 32];
  __shared__ int stop;
  const int h = blockIdx.x;
  const double* Ah = A_in + static_cast<size_t>(h) * d * d;
  for (int t = threadIdx.x; t < d * d; t += blockDim.x) {
    const int i = t / d, j = t % d;
    if (i <= j) A[tri(i, j, d)] = Ah[t];
    V[t] = (i == j) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
    // convergence: off-diagonal Frobenius mass relative to the diagonal
    double off = 0.0, dia = 0.0;
    for (int t = threadIdx.x; t < d * d; t += blockDim.x) {
      const int i = t / d, j = t % d;
      if (i < j) {
        const double v = A[tri(i, j, d)];
        off += v * v;
      } else if (i == j) {
        const double v = A[tri(i, i, d)];
        dia += v * v;
      }
    }
    off = warp_sum_f64(off);
    dia = warp_sum_f64(dia);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = off;
    __syncthreads();
    if (threadIdx.x == 0) {
      double o = 0.0;
      for (int w = 0; w < kJacobiThreads / 32; ++w) o += red[w];
      red[0] = o;
    }
    __syncthreads();
    const double off_tot = red[0];
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dia;
    __syncthreads();
    if (threadIdx.x == 0) {
      double o = 0.0;
      for (int w = 0; w < kJacobiThreads / 32; ++w) o += red[w];
      stop = (off_tot <= 1e-28 * o) || (off_tot == 0.0);
    }
    __syncthreads();
    if (stop) break;
    for (int step = 0; step < d - 1; ++step) {
      // pairs of this step and their rotations
      for (int k = threadIdx.x; k < P; k += blockDim.x) {
        // players 0..d-1: player 0 fixed, the others rotate by `step`
        const int a = (k == 0) ? 0 : 1 + ((k - 1 + step) % (d - 1));
        const int b = 1 + ((d - 2 - k + step) % (d - 1));
        const int p0 = min(a, b), q0 = max(a, b);
        const double app = A[tri(p0, p0, d)], aqq = A[tri(q0, q0, d)], apq = A[tri(p0, q0, d)];
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
        const int pa = pp[a], qa = qq[a];
        const double ca = cs[a], sa = sn[a];
        if (a == b) {
          const double app = A[tri(pa, pa, d)], aqq = A[tri(qa, qa, d)], apq = A[tri(pa, qa, d)];
          if (sa != 0.0) {
            const double t = sa / ca;
            A[tri(pa, pa, d)] = app - t * apq;
            A[tri(qa, qa, d)] = aqq + t * apq;
            A[tri(pa, qa, d)] = 0.0;
          }
        } else {
          const int pb = pp[b], qb = qq[b];
          const double cb = cs[b], sb = sn[b];
          const int i00 = sym(pa, pb, d), i01 = sym(pa, qb, d), i10 = sym(qa, pb, d),
                    i11 = sym(qa, qb, d);
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
      for (int idx = threadIdx.x; idx < d * P; idx += blockDim.x) {
        const int i = idx / P, k = idx % P;
        const double c = cs[k], s = sn[k];
        if (s == 0.0) continue;
        double* vr = V + static_cast<size_t>(i) * d;
        const double vp = vr[pp[k]], vq = vr[qq[k]];
        vr[pp[k]] = c * vp - s * vq;
        vr[qq[k]] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }
  for (int t = threadIdx.x; t < d * d; t += blockDim.x)
    evec[static_cast<size_t>(h) * d * d + t] = V[t];
  for (int j = threadIdx.x; j < d; j += blockDim.x)
    eval[static_cast<size_t>(h) * d + j] = A[tri(j, j, d)];
}

// wk[h, a, t] = evec[h, a, j] * sqrt(max(lambda_j, 0)) where j has rank t in
// descending eigenvalue order (ties to the lower index), t < e.
__global__ void top_eig_projector_kernel(const double* eval, const double* evec, int d, int e,
                                         double* wk) {
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
  const double sc = sqrt(fmax(lj, 0.0));
  const double* V = evec + static_cast<size_t>(h) * d * d;
  for (int a = 0; a < d; ++a)
    wk[(static_cast<size_t>(h) * d + a) * e + rank] = V[static_cast<size_t>(a) * d + j] * sc;
}

}  // namespace

cudaError_t launch_jacobi(const double* A, int H, int d, double* eval, double* evec,
                          DeviceStats* stats, cudaStream_t st) {
  const int P = d / 2;
  const size_t shb = (static_cast<size_t>(d) * (d + 1) / 2 + static_cast<size_t>(d) * d + 2 * P) * 8 +
                     2 * P * 4;
  cudaError_t e = cudaFuncSetAttribute(jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(shb));
  if (e != cudaSuccess) return e;
  jacobi_kernel<<<H, kJacobiThreads, shb, st>>>(A, d, eval, evec, stats);
  return cudaGetLastError();
}

cudaError_t launch_top_eig_projector(const double* eval, const double* evec, int H, int d, int e,
                                     double* wk, cudaStream_t st) {
  top_eig_projector_kernel<<<H, 128, 0, st>>>(eval, evec, d, e, wk);
  return cudaGetLastError();
}

}  // namespace spr
