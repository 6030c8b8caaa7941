// Stage 4 of "Partition the Support, Reconstruct the Residual" (2.B,
// probe-fitted residual reconstruction): stratified probe rows, their exact
// dense outputs (computed by the attention kernel in dense mode), the ridge
// fit of R ~ b + x B in fp64, its restriction to the leading residual
// subspace, and the fused correction + unpermute of every unprobed row.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

// Exclusive prefix sums of v[0..n) into out (out may be v), and the total,
// by the whole block (blockDim.x a multiple of 32): chunks of blockDim.x
// values, a warp scan by shuffles, then the warp totals. Integer sums, so
// the result does not depend on the order. Every thread reads the total from
// shared memory on return, so two calls must be separated by a barrier.
__device__ int32_t block_exclusive_scan(const int32_t* v, int32_t* out, int n) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int c = base + threadIdx.x;
    const int32_t x0 = (c < n) ? v[c] : 0;
    int32_t x = x0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int32_t t = (lane < nw) ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      if (lane < nw) warp_tot[lane] = t;
    }
    __syncthreads();
    const int32_t before = carry + (wid > 0 ? warp_tot[wid - 1] : 0) + (x - x0);
    __syncthreads();  // every thread has read carry and warp_tot
    if (c < n) out[c] = before;
    if (threadIdx.x == blockDim.x - 1) carry = before + x0;
    __syncthreads();
  }
  return carry;
}

// Probes per query group by largest remainder (ties to the lower group),
// rows at offsets floor((t + 1/2) n_g / m_g) inside each group.
__global__ void probe_select_kernel(const int32_t* off_q, int off_stride, int Cq, int M,
                                    int32_t* probes, int32_t* pgrp) {
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
  {
    // the floors' total (start is free here); each m[g] <= M, so it fits
    const int32_t s = block_exclusive_scan(m, start, Cq);
    if (threadIdx.x == 0) left = M - s;
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
  block_exclusive_scan(m, start, Cq);
  __syncthreads();
  int32_t* out = probes + static_cast<size_t>(h) * M;
  int32_t* grp = pgrp ? pgrp + static_cast<size_t>(h) * M : nullptr;
  for (int g = threadIdx.x; g < Cq; g += blockDim.x) {
    const int64_t n = oq[g + 1] - oq[g];
    const int mg = m[g];
    for (int t = 0; t < mg; ++t) {
      out[start[g] + t] = oq[g] + static_cast<int32_t>(((2LL * t + 1) * n) / (2LL * mg));
      if (grp) grp[start[g] + t] = g;
    }
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

// X = O_sparse[probes] (or the probe rows' sparse outputs x_rows [H, M, d]
// when given), R = O_dense - X (fp64) for a block of probe rows
// per CTA (thread = column), with the block's column sums of X and R in
// part [H, nblk, 2, d]; probe_means_kernel adds the blocks in order.
__global__ void probe_residuals_kernel(const float* o_sparse, const float* x_rows,
                                       const float* od, const int32_t* probes, int N, int M,
                                       int d, int rows_blk, double* xr, double* part) {
  const int h = blockIdx.y, blk = blockIdx.x, a = threadIdx.x;
  if (a >= d) return;
  double* X = xr + static_cast<size_t>(h) * 2 * M * d;
  double* R = X + static_cast<size_t>(M) * d;
  double sx = 0.0, sr = 0.0;
  const int t0 = blk * rows_blk, t1 = min(M, t0 + rows_blk);
#pragma unroll 4
  for (int t = t0; t < t1; ++t) {
    const double x =
        x_rows ? x_rows[(static_cast<size_t>(h) * M + t) * d + a]
               : o_sparse[(static_cast<size_t>(h) * N + probes[static_cast<size_t>(h) * M + t]) * d + a];
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

// Ridge solve per head, A B = C with A = X^T X + lambda I (SPD) and C = X^T R,
// then b = rbar - xbar B. One CTA per head; the d x d matrices live in the
// threads' registers: warp w holds rows w, w + 16, .. and lane l columns l,
// l + 32, .. (Golub & Van Loan, sec. 4.2, right-looking outer-product
// Cholesky, then substitution by rows):
//   1. Cholesky, column j: the warp holding row j of the (symmetric) trailing
//      matrix forms l_jj = sqrt(a_jj) and l_kj = a_jk / l_jj (k > j) and
//      publishes them as row j of Lt = L^T in shared memory; every thread
//      then updates a_ik -= l_ij l_kj on its entries with i, k > j;
//   2. L Y = C: the warp holding row j of C forms y_j = c_j / l_jj and
//      publishes it; every thread updates c_i -= l_ij y_j for its rows i > j;
//   3. L^T B = Y the same way from the last row up (y_i -= l_ji b_j, i < j).
// One barrier per step; the published rows of Y and B alternate between two
// buffers so that the next row's warp can run ahead. A pivot that is not
// positive (A not SPD) is replaced by 1 for the rest of the solve and the
// head gets B = 0, b = 0 and SPARSEPR_ERR_NUMERIC.
constexpr int kRidgeThreads = 512;
constexpr int kRidgeWarps = kRidgeThreads / 32;

template <int d>
constexpr size_t ridge_smem_bytes() {
  return (static_cast<size_t>(d) * (d + 1) + 2 * d + static_cast<size_t>(kRidgeWarps) * d) * 8;
}

template <int d>
__global__ void __launch_bounds__(kRidgeThreads, 1)
    ridge_solve_kernel(const double* gram, double* bmat, double* bvec, const double* means,
                       DeviceStats* stats) {
  constexpr int kRpw = d / kRidgeWarps, kCpl = d / 32;
  extern __shared__ double rsm[];
  double* Lt = rsm;                                 // [d][d + 1]: row j = column j of L
  double* rowb = Lt + static_cast<size_t>(d) * (d + 1);  // [2][d] published rows
  double* part = rowb + 2 * d;                      // [warps][d] partial sums of xbar B
  __shared__ int bad;
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const double* A = gram + static_cast<size_t>(h) * 2 * d * d;
  const double* C = A + static_cast<size_t>(d) * d;
  if (tid == 0) bad = 0;
  double m[kRpw][kCpl];
#pragma unroll
  for (int r = 0; r < kRpw; ++r)
#pragma unroll
    for (int c = 0; c < kCpl; ++c) m[r][c] = A[(wid + kRidgeWarps * r) * d + lane + 32 * c];
  __syncthreads();
  // 1. Cholesky
  for (int j = 0; j < d; ++j) {
    double* lrow = Lt + static_cast<size_t>(j) * (d + 1);
    if (wid == j % kRidgeWarps) {
      const int rj = j / kRidgeWarps;
      double x[kCpl];
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        x[c] = 0.0;
#pragma unroll
        for (int r = 0; r < kRpw; ++r) x[c] = (r == rj) ? m[r][c] : x[c];
      }
      // a_jj (a select here would become an indexed local-memory load; a
      // non-finite row makes a_jj non-finite and fails the pivot test)
      double ajj = 0.0;
#pragma unroll
      for (int c = 0; c < kCpl; ++c) ajj = fma((c == (j >> 5)) ? 1.0 : 0.0, x[c], ajj);
      ajj = __shfl_sync(0xffffffffu, ajj, j & 31);
      if (!(ajj > 0.0)) {
        if (lane == 0) bad = 1;
        ajj = 1.0;
      }
      const double ljj = sqrt(ajj);
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        const int k = lane + 32 * c;
        lrow[k] = (k > j) ? x[c] / ljj : (k == j ? ljj : 0.0);
      }
    }
    __syncthreads();
    double lc[kCpl];
#pragma unroll
    for (int c = 0; c < kCpl; ++c) lc[c] = lrow[lane + 32 * c];
    // every entry, without branches: l_ij is zero for i < j and l_kj for
    // k < j; row j and column j are not read again by the factorisation
#pragma unroll
    for (int r = 0; r < kRpw; ++r) {
      const double li = lrow[wid + kRidgeWarps * r];
#pragma unroll
      for (int c = 0; c < kCpl; ++c) m[r][c] = fma(-li, lc[c], m[r][c]);
    }
  }
  // 2. L Y = C (the registers now hold C)
#pragma unroll
  for (int r = 0; r < kRpw; ++r)
#pragma unroll
    for (int c = 0; c < kCpl; ++c) m[r][c] = C[(wid + kRidgeWarps * r) * d + lane + 32 * c];
  for (int j = 0; j < d; ++j) {
    double* yrow = rowb + (j & 1) * d;
    if (wid == j % kRidgeWarps) {
      const double ljj = Lt[static_cast<size_t>(j) * (d + 1) + j];
      const int rj = j / kRidgeWarps;
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        double x = 0.0;
#pragma unroll
        for (int r = 0; r < kRpw; ++r) x = (r == rj) ? m[r][c] : x;
        yrow[lane + 32 * c] = x / ljj;
      }
    }
    __syncthreads();
    double yc[kCpl];
#pragma unroll
    for (int c = 0; c < kCpl; ++c) yc[c] = yrow[lane + 32 * c];
    const double* lrow = Lt + static_cast<size_t>(j) * (d + 1);
#pragma unroll
    for (int r = 0; r < kRpw; ++r) {
      const int i = wid + kRidgeWarps * r;
      if (i > j) {
        const double li = lrow[i];
#pragma unroll
        for (int c = 0; c < kCpl; ++c) m[r][c] = fma(-li, yc[c], m[r][c]);
      } else if (i == j) {
#pragma unroll
        for (int c = 0; c < kCpl; ++c) m[r][c] = yc[c];
      }
    }
  }
  // 3. L^T B = Y
  for (int j = d - 1; j >= 0; --j) {
    double* brow = rowb + (j & 1) * d;
    if (wid == j % kRidgeWarps) {
      const double ljj = Lt[static_cast<size_t>(j) * (d + 1) + j];
      const int rj = j / kRidgeWarps;
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        double x = 0.0;
#pragma unroll
        for (int r = 0; r < kRpw; ++r) x = (r == rj) ? m[r][c] : x;
        brow[lane + 32 * c] = x / ljj;
      }
    }
    __syncthreads();
    double bc[kCpl];
#pragma unroll
    for (int c = 0; c < kCpl; ++c) bc[c] = brow[lane + 32 * c];
#pragma unroll
    for (int r = 0; r < kRpw; ++r) {
      const int i = wid + kRidgeWarps * r;
      if (i < j) {
        const double lji = Lt[static_cast<size_t>(i) * (d + 1) + j];
#pragma unroll
        for (int c = 0; c < kCpl; ++c) m[r][c] = fma(-lji, bc[c], m[r][c]);
      } else if (i == j) {
#pragma unroll
        for (int c = 0; c < kCpl; ++c) m[r][c] = bc[c];
      }
    }
  }
  const bool failed = bad != 0;  // set before the first barrier after the Cholesky
  double* Bo = bmat + static_cast<size_t>(h) * d * d;
  const double* xbar = means + static_cast<size_t>(h) * 2 * d;
  const double* rbar = xbar + d;
  double pc[kCpl];
#pragma unroll
  for (int c = 0; c < kCpl; ++c) pc[c] = 0.0;
#pragma unroll
  for (int r = 0; r < kRpw; ++r) {
    const int i = wid + kRidgeWarps * r;
    const double xi = xbar[i];
#pragma unroll
    for (int c = 0; c < kCpl; ++c) {
      const double v = failed ? 0.0 : m[r][c];
      Bo[static_cast<size_t>(i) * d + lane + 32 * c] = v;
      pc[c] = fma(xi, v, pc[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < kCpl; ++c) part[wid * d + lane + 32 * c] = pc[c];
  __syncthreads();
  if (tid < d) {
    double sx = 0.0;
#pragma unroll
    for (int w = 0; w < kRidgeWarps; ++w) sx += part[w * d + tid];
    bvec[static_cast<size_t>(h) * d + tid] = failed ? 0.0 : rbar[tid] - sx;
  }
  if (failed && tid == 0) raise_status(stats, SPARSEPR_ERR_NUMERIC);
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
                                int32_t* probes, int32_t* pgrp, cudaStream_t st) {
  const size_t shb = static_cast<size_t>(Cq) * 16;
  probe_select_kernel<<<H, 256, shb, st>>>(off_q, off_stride, Cq, M, probes, pgrp);
  return cudaGetLastError();
}

cudaError_t launch_gather_probe_rows(const void* qp, bool bf16, const int32_t* probes, int H,
                                     int N, int M, int d, __nv_bfloat16* dst, cudaStream_t st) {
  gather_probe_rows_kernel<<<dim3(M, H), 128, 0, st>>>(qp, bf16 ? 1 : 0, probes, N, M, d, dst);
  return cudaGetLastError();
}

cudaError_t launch_probe_residuals(const float* o_sparse, const float* x_rows, const float* od,
                                   const int32_t* probes, int H, int N, int M, int d, double* xr,
                                   double* means, double* part, size_t part_doubles,
                                   cudaStream_t st) {
  // blocks of >= 16 rows, at most part_doubles / (2 d H) of them
  int nblk = (M + 15) / 16;
  const int cap = static_cast<int>(part_doubles / (2 * static_cast<size_t>(d) * H));
  if (nblk > cap) nblk = cap;
  if (nblk < 1) return cudaErrorInvalidValue;
  const int rows_blk = (M + nblk - 1) / nblk;
  nblk = (M + rows_blk - 1) / rows_blk;
  if (nblk < 1) nblk = 1;
  probe_residuals_kernel<<<dim3(nblk, H), d, 0, st>>>(o_sparse, x_rows, od, probes, N, M, d,
                                                      rows_blk, xr, part);
  probe_means_kernel<<<H, d, 0, st>>>(part, nblk, M, d, means);
  return cudaGetLastError();
}

cudaError_t launch_ridge_solve(double* gram, int H, int d, double* bmat, double* bvec,
                               const double* means, DeviceStats* stats, cudaStream_t st) {
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  const size_t shb = (d == 128) ? ridge_smem_bytes<128>() : ridge_smem_bytes<64>();
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
