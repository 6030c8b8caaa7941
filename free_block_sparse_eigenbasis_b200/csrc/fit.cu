// Stage 4 of "Partition the Support, Reconstruct the Residual" (2.B,
// probe-fitted residual reconstruction): stratified probe rows, their exact
// dense outputs (computed by the attention kernel in dense mode), the ridge
// fit of R ~ b + x B in fp64, its restriction to the leading residual
// subspace, and the fused correction + unpermute of every unprobed row.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

// Probes per query group by largest remainder (ties to the lower group),
// rows at offsets floor((t + 1/2) n_g / m_g) inside each group.
__global__ void probe_select_kernel(const int32_t* off_q, int off_stride, int Cq, int M,
                                    int32_t* probes) {
  extern __shared__ int64_t psm[];
  int64_t* rem = psm;                                  // [Cq]
  int32_t* m = reinterpret_cast<int32_t*>(rem + Cq);   // [Cq]
  int32_t* start = m + Cq;                             // [Cq]
  __shared__ int32_t left;
  const int h = blockIdx.x;
  const int32_t* oq = off_q + static_cast<size_t>(h) * off_stride;
  const int64_t Nt = oq[Cq] - oq[0];
  for (int g = threadIdx.x; g < Cq; g += blockDim.x) {
    const int64_t n = oq[g + 1] - oq[g];
    const int64_t num = static_cast<int64_t>(M) * n;
    m[g] = static_cast<int32_t>(Nt > 0 ? num / Nt : 0);
    rem[g] = Nt > 0 ? num % Nt : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t s = 0;
    for (int g = 0; g < Cq; ++g) s += m[g];
    left = static_cast<int32_t>(M - s);
  }
  __syncthreads();
  // rank of each remainder (larger first, lower group on ties)
  for (int g = threadIdx.x; g < Cq; g += blockDim.x) {
    const int64_t rg = rem[g];
    int rank = 0;
    for (int o = 0; o < Cq; ++o) rank += (rem[o] > rg) || (rem[o] == rg && o < g);
    start[g] = rank;  // temporary
  }
  __syncthreads();
  for (int g = threadIdx.x; g < Cq; g += blockDim.x)
    if (start[g] < left) m[g] += 1;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t s = 0;
    for (int g = 0; g < Cq; ++g) {
      start[g] = s;
      s += m[g];
    }
  }
  __syncthreads();
  int32_t* out = probes + static_cast<size_t>(h) * M;
  for (int g = threadIdx.x; g < Cq; g += blockDim.x) {
    const int64_t n = oq[g + 1] - oq[g];
    const int mg = m[g];
    for (int t = 0; t < mg; ++t)
      out[start[g] + t] = oq[g] + static_cast<int32_t>(((2LL * t + 1) * n) / (2LL * mg));
  }
}

// dst[h, t, :] = bf16(qp[h, probes[h, t], :]); rows M..M+127 of each head's
// slot region are zero.
__global__ void gather_probe_rows_kernel(const void* qp, int bf16, const int32_t* probes, int N,
                                         int M, int d, __nv_bfloat16* dst) {
  const int h = blockIdx.y;
  const int t = blockIdx.x;
  __nv_bfloat16* o = dst + (static_cast<size_t>(h) * M + t) * d;
  if (t >= M) return;
  const size_t src_row = static_cast<size_t>(h) * N + probes[static_cast<size_t>(h) * M + t];
  for (int a = threadIdx.x; a < d; a += blockDim.x) {
    if (bf16)
      o[a] = static_cast<const __nv_bfloat16*>(qp)[src_row * d + a];
    else
      o[a] = __float2bfloat16_rn(static_cast<const float*>(qp)[src_row * d + a]);
  }
}

// X = O_sparse[probes], R = O_dense - X (fp64), column means xbar, rbar.
// X = O_sparse[probes], R = O_dense - X (fp64) for a block of probe rows
// per CTA (thread = column), with the block's column sums of X and R in
// part [H, nblk, 2, d]; probe_means_kernel adds the blocks in order.
__global__ void probe_residuals_kernel(const float* o_sparse, const float* od,
                                       const int32_t* probes, int N, int M, int d, int rows_blk,
                                       double* xr, double* part) {
  const int h = blockIdx.y, blk = blockIdx.x, a = threadIdx.x;
  if (a >= d) return;
  double* X = xr + static_cast<size_t>(h) * 2 * M * d;
  double* R = X + static_cast<size_t>(M) * d;
  double sx = 0.0, sr = 0.0;
  const int t0 = blk * rows_blk, t1 = min(M, t0 + rows_blk);
#pragma unroll 4
  for (int t = t0; t < t1; ++t) {
    const size_t row = static_cast<size_t>(h) * N + probes[static_cast<size_t>(h) * M + t];
    const double x = o_sparse[row * d + a];
    const double r = static_cast<double>(od[(static_cast<size_t>(h) * M + t) * d + a]) - x;
    X[static_cast<size_t>(t) * d + a] = x;
    R[static_cast<size_t>(t) * d + a] = r;
    sx += x;
    sr += r;
  }
  double* pp = part + ((static_cast<size_t>(h) * gridDim.x + blk) * 2) * d;
  pp[a] = sx;
  pp[d + a] = sr;
}

__global__ void probe_means_kernel(const double* part, int nblk, int M, int d, double* means) {
  const int h = blockIdx.x, a = threadIdx.x;
  if (a >= d) return;
  double sx = 0.0, sr = 0.0;
  for (int b = 0; b < nblk; ++b) {
    const double* pp = part + ((static_cast<size_t>(h) * nblk + b) * 2) * d;
    sx += pp[a];
    sr += pp[d + a];
  }
  means[(static_cast<size_t>(h) * 2 + 0) * d + a] = M > 0 ? sx / M : 0.0;
  means[(static_cast<size_t>(h) * 2 + 1) * d + a] = M > 0 ? sr / M : 0.0;
}

// Ridge solve per head: L L^T = A (right-looking Cholesky on the packed
// lower triangle in shared memory), then L Y = C and L^T B = Y with all d
// right-hand sides at once (row-by-row elimination, parallel over the rows
// below and the columns), and b = rbar - xbar B.
constexpr int kRidgeThreads = 512;

template <int d>
__global__ void __launch_bounds__(kRidgeThreads)
    ridge_solve_kernel(const double* gram, double* bmat, double* bvec, const double* means,
                       DeviceStats* stats) {
  extern __shared__ double rsm[];
  const int ntri = d * (d + 1) / 2;
  double* Lp = rsm;          // packed lower triangle, L[i][k] at i*(i+1)/2 + k
  double* Cm = rsm + ntri;   // [d][d] right-hand sides (row-major), solved in place
  __shared__ int bad;
  const int h = blockIdx.x, tid = threadIdx.x;
  const double* A = gram + static_cast<size_t>(h) * 2 * d * d;
  const double* C = A + static_cast<size_t>(d) * d;
  for (int t = tid; t < d * d; t += blockDim.x) {
    const int i = t / d, k = t % d;
    if (k <= i) Lp[i * (i + 1) / 2 + k] = A[t];
    Cm[t] = C[t];
  }
  if (tid == 0) bad = 0;
  __syncthreads();
  auto L = [&](int i, int k) -> double& { return Lp[i * (i + 1) / 2 + k]; };
  // Cholesky: column j, then the trailing triangle (4 threads per row)
  for (int j = 0; j < d; ++j) {
    if (tid == 0) {
      double s = L(j, j);
      if (!(s > 0.0)) {
        bad = 1;
        s = 1.0;
      }
      L(j, j) = sqrt(s);
    }
    __syncthreads();
    const double ljj = L(j, j);
    for (int i = j + 1 + tid; i < d; i += blockDim.x) L(i, j) /= ljj;
    __syncthreads();
    for (int q = tid; q < (d - j - 1) * 4; q += blockDim.x) {
      const int i = j + 1 + (q >> 2);
      const double lij = L(i, j);
      for (int k = j + 1 + (q & 3); k <= i; k += 4) L(i, k) -= lij * L(k, j);
    }
    __syncthreads();
  }
  // forward: L Y = C
  for (int i = 0; i < d; ++i) {
    const double lii = L(i, i);
    for (int c = tid; c < d; c += blockDim.x) Cm[i * d + c] /= lii;
    __syncthreads();
    for (int t = tid; t < (d - i - 1) * d; t += blockDim.x) {
      const int r = i + 1 + t / d, c = t % d;
      Cm[r * d + c] -= L(r, i) * Cm[i * d + c];
    }
    __syncthreads();
  }
  // backward: L^T B = Y
  for (int i = d - 1; i >= 0; --i) {
    const double lii = L(i, i);
    for (int c = tid; c < d; c += blockDim.x) Cm[i * d + c] /= lii;
    __syncthreads();
    for (int t = tid; t < i * d; t += blockDim.x) {
      const int r = t / d, c = t % d;
      Cm[r * d + c] -= L(i, r) * Cm[i * d + c];
    }
    __syncthreads();
  }
  if (bad) {
    for (int t = tid; t < d * d; t += blockDim.x) Cm[t] = 0.0;
    if (tid == 0) raise_status(stats, SPARSEPR_ERR_NUMERIC);
    __syncthreads();
  }
  double* Bo = bmat + static_cast<size_t>(h) * d * d;
  for (int t = tid; t < d * d; t += blockDim.x) Bo[t] = Cm[t];
  if (tid < d) {
    const int col = tid;
    const double* xbar = means + static_cast<size_t>(h) * 2 * d;
    const double* rbar = xbar + d;
    double s = rbar[col];
    for (int a2 = 0; a2 < d; ++a2) s -= xbar[a2] * Cm[a2 * d + col];
    bvec[static_cast<size_t>(h) * d + col] = bad ? 0.0 : s;
  }
}

// Restriction to the residual subspace: with V_r [d, r] the leading right
// singular vectors of R, B' = (B V_r) V_r^T and b' = (b V_r) V_r^T (fp64),
// stored fp32 for the correction (and fp64 if asked). One CTA per row of B'
// (row d is the intercept).
__global__ void project_map_kernel(const double* bmat, const double* bvec, const double* vr,
                                   int d, int r, float* bp32, float* bv32, double* fit_out) {
  __shared__ double rw[128], T[128];
  const int a = blockIdx.x, h = blockIdx.y;
  const double* row = (a < d) ? bmat + (static_cast<size_t>(h) * d + a) * d
                              : bvec + static_cast<size_t>(h) * d;
  const double* V = vr + static_cast<size_t>(h) * d * r;
  for (int k = threadIdx.x; k < d; k += blockDim.x) rw[k] = row[k];
  __syncthreads();
  for (int t = threadIdx.x; t < r; t += blockDim.x) {
    double s = 0.0;
    for (int k = 0; k < d; ++k) s = fma(rw[k], V[static_cast<size_t>(k) * r + t], s);
    T[t] = s;
  }
  __syncthreads();
  const int col = threadIdx.x;
  if (col < d) {
    double s = 0.0;
    for (int t = 0; t < r; ++t) s = fma(T[t], V[static_cast<size_t>(col) * r + t], s);
    if (a < d) {
      bp32[(static_cast<size_t>(h) * d + col) * d + a] = static_cast<float>(s);  // B'^T
      if (fit_out) fit_out[static_cast<size_t>(h) * (d * d + d) + a * d + col] = s;
    } else {
      bv32[static_cast<size_t>(h) * d + col] = static_cast<float>(s);
      if (fit_out) fit_out[static_cast<size_t>(h) * (d * d + d) + d * d + col] = s;
    }
  }
}

// out[perm_q[i]] = O_dense(probe) for probe rows, else x + b' + x B'
// (x = o_sparse row, fp32); 32 group-major rows per CTA, B' in shared memory.
// CUDA-core form for inputs too small for the tensor-core kernel.
constexpr int kCorrRows = 32;

template <bool OUT_BF16>
__global__ void __launch_bounds__(256) correct_kernel(const float* o_sparse, const float* od,
                                                      const int32_t* probes,
                                                      const int32_t* perm_q, const float* bp32,
                                                      const float* bv32, int N, int n_corr, int M,
                                                      int d, void* out) {
  extern __shared__ float csm[];
  float* Bs = csm;                 // [d][d]
  float* xs = Bs + d * d;          // [kCorrRows][d]
  __shared__ int prow[kCorrRows];  // probe index or -1
  const int h = blockIdx.y;
  const int i0 = blockIdx.x * kCorrRows;
  const float* Bh = bp32 + static_cast<size_t>(h) * d * d;
  for (int t = threadIdx.x; t < d * d; t += blockDim.x) Bs[(t % d) * d + t / d] = Bh[t];  // B' from B'^T
  for (int t = threadIdx.x; t < kCorrRows * d; t += blockDim.x) {
    const int r = t / d, a = t % d;
    const int i = i0 + r;
    xs[t] = (i < N) ? o_sparse[(static_cast<size_t>(h) * N + i) * d + a] : 0.f;
  }
  if (threadIdx.x < kCorrRows) {
    const int i = i0 + threadIdx.x;
    const int32_t* pr = probes + static_cast<size_t>(h) * M;
    int lo = 0, hi = M;  // first probe >= i
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pr[mid] < i) lo = mid + 1; else hi = mid;
    }
    prow[threadIdx.x] = (lo < M && pr[lo] == i) ? lo : -1;
  }
  __syncthreads();
  const float* bv = bv32 + static_cast<size_t>(h) * d;
  for (int t = threadIdx.x; t < kCorrRows * d; t += blockDim.x) {
    const int r = t / d, col = t % d;
    const int i = i0 + r;
    if (i >= N) continue;
    float y;
    if (i >= n_corr) {
      y = xs[r * d + col];  // text rows: exact already, not corrected
    } else if (prow[r] >= 0) {
      y = od[(static_cast<size_t>(h) * M + prow[r]) * d + col];
    } else {
      const float* xr = xs + r * d;
      float acc = 0.f;
      for (int a = 0; a < d; ++a) acc = fmaf(xr[a], Bs[a * d + col], acc);
      y = xr[col] + bv[col] + acc;
    }
    const size_t dst = (static_cast<size_t>(h) * N + perm_q[static_cast<size_t>(h) * N + i]) * d + col;
    if (OUT_BF16)
      static_cast<__nv_bfloat16*>(out)[dst] = __float2bfloat16_rn(y);
    else
      static_cast<float*>(out)[dst] = y;
  }
}

__global__ void pairs_exec_kernel(const int64_t* ps, int H, int64_t add, int64_t* pe,
                                  DeviceStats* stats) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  const int64_t v = ps[h] + add;
  pe[h] = v;
  stats->pairs_exec[h] = v;
}

}  // namespace

cudaError_t launch_probe_select(const int32_t* off_q, int off_stride, int H, int Cq, int M,
                                int32_t* probes, cudaStream_t st) {
  const size_t shb = static_cast<size_t>(Cq) * 16;
  probe_select_kernel<<<H, 256, shb, st>>>(off_q, off_stride, Cq, M, probes);
  return cudaGetLastError();
}

cudaError_t launch_gather_probe_rows(const void* qp, bool bf16, const int32_t* probes, int H,
                                     int N, int M, int d, __nv_bfloat16* dst, cudaStream_t st) {
  gather_probe_rows_kernel<<<dim3(M, H), 128, 0, st>>>(qp, bf16 ? 1 : 0, probes, N, M, d, dst);
  return cudaGetLastError();
}

cudaError_t launch_probe_residuals(const float* o_sparse, const float* od, const int32_t* probes,
                                   int H, int N, int M, int d, double* xr, double* means,
                                   double* part, size_t part_doubles, cudaStream_t st) {
  // blocks of >= 16 rows, at most part_doubles / (2 d H) of them
  int nblk = (M + 15) / 16;
  const int cap = static_cast<int>(part_doubles / (2 * static_cast<size_t>(d) * H));
  if (nblk > cap) nblk = cap;
  if (nblk < 1) return cudaErrorInvalidValue;
  const int rows_blk = (M + nblk - 1) / nblk;
  nblk = (M + rows_blk - 1) / rows_blk;
  if (nblk < 1) nblk = 1;
  probe_residuals_kernel<<<dim3(nblk, H), d, 0, st>>>(o_sparse, od, probes, N, M, d, rows_blk, xr,
                                                      part);
  probe_means_kernel<<<H, d, 0, st>>>(part, nblk, M, d, means);
  return cudaGetLastError();
}

cudaError_t launch_ridge_solve(double* gram, int H, int d, double* bmat, double* bvec,
                               const double* means, DeviceStats* stats, cudaStream_t st) {
  const size_t shb = (static_cast<size_t>(d) * (d + 1) / 2 + static_cast<size_t>(d) * d) * 8;
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  auto kern = (d == 128) ? ridge_solve_kernel<128> : ridge_solve_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(shb));
  if (e != cudaSuccess) return e;
  kern<<<H, kRidgeThreads, shb, st>>>(gram, bmat, bvec, means, stats);
  return cudaGetLastError();
}

cudaError_t launch_project_map(const double* bmat, const double* bvec, const double* vr, int H,
                               int d, int r, float* bp32, float* bv32, double* fit_out,
                               cudaStream_t st) {
  project_map_kernel<<<dim3(d + 1, H), 128, 0, st>>>(bmat, bvec, vr, d, r, bp32, bv32, fit_out);
  return cudaGetLastError();
}

cudaError_t launch_correct(const float* o_sparse, const float* od, const int32_t* probes,
                           const int32_t* perm_q, const float* bp32, const float* bv32, int H,
                           int N, int n_corr, int M, int d, void* out, bool out_bf16,
                           cudaStream_t st) {
  const size_t shb = (static_cast<size_t>(d) * d + static_cast<size_t>(kCorrRows) * d) * 4;
  dim3 grid((N + kCorrRows - 1) / kCorrRows, H);
  cudaError_t e;
  if (out_bf16) {
    e = cudaFuncSetAttribute(correct_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(shb));
    if (e != cudaSuccess) return e;
    correct_kernel<true><<<grid, 256, shb, st>>>(o_sparse, od, probes, perm_q, bp32, bv32, N,
                                                 n_corr, M, d, out);
  } else {
    e = cudaFuncSetAttribute(correct_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(shb));
    if (e != cudaSuccess) return e;
    correct_kernel<false><<<grid, 256, shb, st>>>(o_sparse, od, probes, perm_q, bp32, bv32, N,
                                                  n_corr, M, d, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_pairs_exec(const int64_t* pairs_sparse, int H, int64_t add, int64_t* pairs_exec,
                              DeviceStats* stats, cudaStream_t st) {
  pairs_exec_kernel<<<(H + 127) / 128, 128, 0, st>>>(pairs_sparse, H, add, pairs_exec, stats);
  return cudaGetLastError();
}

}  // namespace spr
