// Structural diagnostics of one call, from "Partition the Support, Reconstruct
// the Residual" (section 3, structural analysis; section 4, ablations):
//   * on the probe rows: the dense softmax mass that a row's route keeps, the
//     row's sparse-vs-dense error, and how the probe residual's energy splits
//     between the fitted affine map, its subspace restriction and the rest;
// computed on the device from what sparsepr_probe_correct leaves in the
// workspace. All sums are fp64 in a fixed order.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kPdRows = 8;      // probe rows per CTA
constexpr int kPdThreads = 128;

__device__ __forceinline__ double block_sum128(double v, double* red) {
  // 128 threads: four warps, added in warp order
  v = warp_sum_f64(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  return (red[0] + red[1]) + (red[2] + red[3]);
}

// Per probe row t: retained mass 2^(lse_sparse - lse_dense), ||R_t||, and the
// four energies |R_t|^2, |R_t V_r|^2, |R_t - F_t|^2, |R_t - F_t P_r|^2 with
// F_t = b + X_t B the fitted map and P_r = V_r V_r^T.
__global__ void __launch_bounds__(kPdThreads)
    probe_diag_kernel(const int32_t* probes, const float* lse_s, const float* lse_d,
                      const double* xr, const double* bmat, const double* bvec, const double* vr,
                      int N, int M, int d, int r, double* mass, double* err, double* energy_rows) {
  __shared__ double xs[128], rs[128], fs[128], cv[128], red[4];
  const int h = blockIdx.y, a = threadIdx.x;
  const double* X = xr + static_cast<size_t>(h) * 2 * M * d;
  const double* R = X + static_cast<size_t>(M) * d;
  const double* B = bmat + static_cast<size_t>(h) * d * d;
  const double* bv = bvec + static_cast<size_t>(h) * d;
  const double* V = vr + static_cast<size_t>(h) * d * r;
  for (int k = 0; k < kPdRows; ++k) {
    const int t = blockIdx.x * kPdRows + k;
    if (t >= M) break;  // uniform over the block
    __syncthreads();
    if (a < d) {
      xs[a] = X[static_cast<size_t>(t) * d + a];
      rs[a] = R[static_cast<size_t>(t) * d + a];
    }
    __syncthreads();
    // F_t = b + X_t B (thread a: column a)
    double f = 0.0;
    if (a < d) {
      f = bv[a];
      for (int b = 0; b < d; ++b) f = fma(xs[b], B[static_cast<size_t>(b) * d + a], f);
      fs[a] = f;
    }
    __syncthreads();
    // (F_t V_r)_j and (R_t V_r)_j by threads j < r, j - r < r
    double rv = 0.0;
    if (a < r) {
      double c = 0.0;
      for (int b = 0; b < d; ++b) c = fma(fs[b], V[static_cast<size_t>(b) * r + a], c);
      cv[a] = c;
    }
    if (a >= 64 && a - 64 < r) {
      const int j = a - 64;
      for (int b = 0; b < d; ++b) rv = fma(rs[b], V[static_cast<size_t>(b) * r + j], rv);
    }
    __syncthreads();
    double e0 = 0.0, e2 = 0.0, e3 = 0.0;
    if (a < d) {
      double fp = 0.0;  // (F_t P_r)_a
      for (int j = 0; j < r; ++j) fp = fma(cv[j], V[static_cast<size_t>(a) * r + j], fp);
      const double ra = rs[a];
      e0 = ra * ra;
      e2 = (ra - fs[a]) * (ra - fs[a]);
      e3 = (ra - fp) * (ra - fp);
    }
    const double s0 = block_sum128(e0, red);
    const double s1 = block_sum128(rv * rv, red);
    const double s2 = block_sum128(e2, red);
    const double s3 = block_sum128(e3, red);
    if (a == 0) {
      const size_t i = static_cast<size_t>(h) * M + t;
      const int row = probes[i];
      mass[i] = exp2(static_cast<double>(lse_s[static_cast<size_t>(h) * N + row]) -
                     static_cast<double>(lse_d[static_cast<size_t>(h) * M + t]));
      err[i] = sqrt(s0);
      double* er = energy_rows + i * 4;
      er[0] = s0;
      er[1] = s1;
      er[2] = s2;
      er[3] = s3;
    }
  }
}

// energy[h] = { sum |R|^2, sum |R V_r|^2 / tot, sum |R - F|^2 / tot,
// sum |R - F P_r|^2 / tot } over the probe rows, summed in row order.
__global__ void probe_energy_kernel(const double* energy_rows, int H, int M, double* energy) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  double s[4] = {0.0, 0.0, 0.0, 0.0};
  for (int t = 0; t < M; ++t)
    for (int c = 0; c < 4; ++c) s[c] += energy_rows[(static_cast<size_t>(h) * M + t) * 4 + c];
  double* e = energy + static_cast<size_t>(h) * 4;
  e[0] = s[0];
  if (s[0] > 0.0) {
    e[1] = s[1] / s[0];
    e[2] = s[2] / s[0];
    e[3] = s[3] / s[0];
  } else {  // no residual: everything is explained
    e[1] = 1.0;
    e[2] = 0.0;
    e[3] = 0.0;
  }
}

// ---------------------------------------------------------------------------
// Support expansion of a shared route (section 3: a query group's rows need
// far more key groups together than each needs alone). For the rows of the
// sampled video query groups: the dense softmax mass of every key group (the
// row's logits over all N keys in fp64, exact for bf16 / fp32 inputs up to the
// last additions), the row's individual support at mass tau = the fewest key
// groups, largest mass first (ties to the lower index), whose running sum
// reaches tau (within 1e-15), and the union of the rows' supports.
// One CTA takes R rows of one group at a time (the key rows are read once per
// R rows); the union is an OR-ed bit set per group, the sizes an integer sum.
// ---------------------------------------------------------------------------
constexpr int kSeThreads = 256;
constexpr int kSeCtas = 16;  // CTAs per sampled group

template <typename T>
__global__ void __launch_bounds__(kSeThreads)
    support_kernel(const T* qp, const T* kp, const int32_t* off_q, int oq_stride,
                   const int32_t* off_k, int Ckt, int N, int d, int Cqv, int stride, int R, int P,
                   double scale, double tau, uint32_t* union_bits, unsigned long long* size_sum) {
  extern __shared__ double se_sm[];
  double* qs = se_sm;                                  // [R][d]
  double* mass = qs + static_cast<size_t>(R) * d;      // [R][Ckt]
  double* skey = mass + static_cast<size_t>(R) * Ckt;  // [P] sort keys
  int* sidx = reinterpret_cast<int*>(skey + P);        // [P]
  __shared__ double rmax[8], rtot[8], red[kSeThreads / 32][8];
  __shared__ int nsel;
  const int h = blockIdx.z, gs = blockIdx.y, g = gs * stride;
  if (g >= Cqv) return;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int32_t* oq = off_q + static_cast<size_t>(h) * oq_stride;
  const int32_t* ok = off_k + static_cast<size_t>(h) * (Ckt + 1);
  const int lo = oq[g], hi = oq[g + 1];
  const int words = (Ckt + 31) / 32;
  uint32_t* ub = union_bits + (static_cast<size_t>(h) * Cqv + g) * words;
  const T* Kh = kp + static_cast<size_t>(h) * N * d;
  unsigned long long sizes = 0;
  for (int r0 = lo + blockIdx.x * R; r0 < hi; r0 += kSeCtas * R) {
    const int nr = min(R, hi - r0);
    __syncthreads();
    for (int i = tid; i < R * d; i += kSeThreads) {
      const int r = i / d, t = i % d;
      qs[i] = (r < nr) ? to_f64(qp, (static_cast<size_t>(h) * N + r0 + r) * d + t) : 0.0;
    }
    __syncthreads();
    // pass 1: scaled row maxima
    double m[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) m[r] = -INFINITY;
    for (int j = tid; j < N; j += kSeThreads) {
      double sv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int t = 0; t < d; ++t) {
        const double kv = to_f64(Kh, static_cast<size_t>(j) * d + t);
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < nr) sv[r] = fma(qs[r * d + t], kv, sv[r]);
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) m[r] = fmax(m[r], scale * sv[r]);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      for (int o = 16; o > 0; o >>= 1) m[r] = fmax(m[r], __shfl_xor_sync(0xffffffffu, m[r], o));
      if (lane == 0) red[w][r] = m[r];
    }
    __syncthreads();
    if (tid < 8) {
      double v = red[0][tid];
      for (int q = 1; q < kSeThreads / 32; ++q) v = fmax(v, red[q][tid]);
      rmax[tid] = v;
    }
    __syncthreads();
    // pass 2: per key group, the sum of exp(scale s - max) over its keys (in key order)
    for (int c = tid; c < Ckt; c += kSeThreads) {
      double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int j = ok[c]; j < ok[c + 1]; ++j) {
        double sv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int t = 0; t < d; ++t) {
          const double kv = to_f64(Kh, static_cast<size_t>(j) * d + t);
#pragma unroll
          for (int r = 0; r < 8; ++r)
            if (r < nr) sv[r] = fma(qs[r * d + t], kv, sv[r]);
        }
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < nr) acc[r] += exp(scale * sv[r] - rmax[r]);
      }
      for (int r = 0; r < nr; ++r) mass[static_cast<size_t>(r) * Ckt + c] = acc[r];
    }
    __syncthreads();
    // row totals, in a fixed order
    for (int r = 0; r < nr; ++r) {
      double v = 0.0;
      for (int c = tid; c < Ckt; c += kSeThreads) v += mass[static_cast<size_t>(r) * Ckt + c];
      v = warp_sum_f64(v);
      if (lane == 0) red[w][r] = v;
    }
    __syncthreads();
    if (tid < nr) {
      double v = 0.0;
      for (int q = 0; q < kSeThreads / 32; ++q) v += red[q][tid];
      rtot[tid] = v;
    }
    __syncthreads();
    // each row: sort the groups by mass (descending, ties to the lower index),
    // count the prefix that reaches tau, mark those groups
    for (int r = 0; r < nr; ++r) {
      for (int i = tid; i < P; i += kSeThreads) {
        skey[i] = (i < Ckt) ? mass[static_cast<size_t>(r) * Ckt + i] / rtot[r] : -1.0;
        sidx[i] = i;
      }
      __syncthreads();
      for (int size = 2; size <= P; size <<= 1) {
        for (int strd = size >> 1; strd > 0; strd >>= 1) {
          for (int t = tid; t < (P >> 1); t += kSeThreads) {
            const int a = 2 * strd * (t / strd) + (t % strd), b = a + strd;
            const double ka = skey[a], kb = skey[b];
            const int ia = sidx[a], ib = sidx[b];
            const bool a_first = ka > kb || (ka == kb && ia < ib);
            if (((a & size) == 0) != a_first) {
              skey[a] = kb;
              skey[b] = ka;
              sidx[a] = ib;
              sidx[b] = ia;
            }
          }
          __syncthreads();
        }
      }
      if (tid == 0) {
        double run = 0.0;
        int n = 0;
        while (n < Ckt) {
          run += skey[n];
          ++n;
          if (run >= tau - 1e-15) break;
        }
        nsel = n;
        sizes += static_cast<unsigned long long>(n);
      }
      __syncthreads();
      for (int i = tid; i < nsel; i += kSeThreads) atomicOr(&ub[sidx[i] >> 5], 1u << (sidx[i] & 31));
      __syncthreads();
    }
  }
  if (tid == 0 && sizes) atomicAdd(&size_sum[static_cast<size_t>(h) * Cqv + g], sizes);
}

// indiv[h, g] = mean support size of the group's rows, aggregate = |union|
// (sampled groups; the others NaN)
__global__ void support_finalize_kernel(const uint32_t* union_bits,
                                        const unsigned long long* size_sum, const int32_t* off_q,
                                        int oq_stride, int H, int Cqv, int Ckt, int stride,
                                        double* indiv, double* aggregate) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * Cqv) return;
  const int h = i / Cqv, g = i % Cqv;
  if (g % stride) {
    indiv[i] = NAN;
    aggregate[i] = NAN;
    return;
  }
  const int n = off_q[static_cast<size_t>(h) * oq_stride + g + 1] - off_q[static_cast<size_t>(h) * oq_stride + g];
  const int words = (Ckt + 31) / 32;
  int u = 0;
  for (int k = 0; k < words; ++k) u += __popc(union_bits[static_cast<size_t>(i) * words + k]);
  indiv[i] = n > 0 ? static_cast<double>(size_sum[i]) / n : 0.0;
  aggregate[i] = static_cast<double>(u);
}

}  // namespace

cudaError_t launch_probe_diagnostics(const int32_t* probes, const float* lse_s, const float* lse_d,
                                     const double* xr, const double* bmat, const double* bvec,
                                     const double* vr, int H, int N, int M, int d, int r,
                                     double* mass, double* err, double* energy_rows,
                                     double* energy, cudaStream_t st) {
  if (d > 128 || r > 64 || M < 1) return cudaErrorInvalidValue;
  probe_diag_kernel<<<dim3((M + kPdRows - 1) / kPdRows, H), kPdThreads, 0, st>>>(
      probes, lse_s, lse_d, xr, bmat, bvec, vr, N, M, d, r, mass, err, energy_rows);
  probe_energy_kernel<<<(H + 63) / 64, 64, 0, st>>>(energy_rows, H, M, energy);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Density profile ("Attention Sparsity is Input-Stable", offline layer-wise
// sparsity profiling): for a sampled row, the smallest number n of its N
// softmax weights, largest first, whose sum reaches tau (within 1e-15 of the
// total); the head's density is the mean of n / N over the sampled rows.
// Per row: the scaled logits over all N keys in fp64 go to a scratch row,
// become weights w = exp(s - max) in place, and an MSB-first radix select
// over the weights' bit patterns (positive doubles order like their bits,
// eight 8-bit digits) finds the weight at which the running sum from the
// top crosses tau * sum(w); the weights equal to it are then counted one by
// one. Bucket sums are fp64 shared-memory atomics, so the crossing is decided
// to within their rounding, far inside the 1e-15 slack.
// ---------------------------------------------------------------------------
constexpr int kDnThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kDnThreads)
    density_kernel(const T* q, const T* k, int N, int Nv, int d, int row_stride,
                   int rows_per_head, int H, double scale, double tau, double* scratch,
                   unsigned long long* count_sum) {
  __shared__ double qs[128];
  __shared__ unsigned int hcnt[256];
  __shared__ double hsum[256];
  __shared__ double red[kDnThreads / 32];
  __shared__ double s_bcast[2];
  __shared__ unsigned long long prefix_s, mask_s;
  __shared__ int done_s;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  double* sc = scratch + static_cast<size_t>(blockIdx.x) * N;
  const int items = H * rows_per_head;
  for (int it = blockIdx.x; it < items; it += gridDim.x) {
    const int h = it / rows_per_head, row = (it % rows_per_head) * row_stride;
    const T* Kh = k + static_cast<size_t>(h) * N * d;
    __syncthreads();
    for (int t = tid; t < d; t += kDnThreads) qs[t] = to_f64(q, (static_cast<size_t>(h) * N + row) * d + t);
    __syncthreads();
    double m = -INFINITY;
    for (int j = tid; j < N; j += kDnThreads) {
      double s = 0.0;
      for (int t = 0; t < d; ++t) s = fma(qs[t], to_f64(Kh, static_cast<size_t>(j) * d + t), s);
      s *= scale;
      sc[j] = s;
      m = fmax(m, s);
    }
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[w] = m;
    __syncthreads();
    if (tid == 0) {
      double v = red[0];
      for (int q2 = 1; q2 < kDnThreads / 32; ++q2) v = fmax(v, red[q2]);
      s_bcast[0] = v;
    }
    __syncthreads();
    const double mx = s_bcast[0];
    double z = 0.0;
    for (int j = tid; j < N; j += kDnThreads) {
      const double wv = exp(sc[j] - mx);
      sc[j] = wv;
      z += wv;
    }
    z = warp_sum_f64(z);
    __syncthreads();
    if (lane == 0) red[w] = z;
    __syncthreads();
    if (tid == 0) {
      double v = 0.0;
      for (int q2 = 0; q2 < kDnThreads / 32; ++q2) v += red[q2];
      s_bcast[1] = (tau - 1e-15) * v;  // target mass
      prefix_s = 0;
      mask_s = 0;
      done_s = 0;
    }
    __syncthreads();
    const double target = s_bcast[1];
    double above = 0.0;  // sum of the weights above the current bucket (thread 0)
    unsigned long long n_above = 0;
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int i = tid; i < 256; i += kDnThreads) {
        hcnt[i] = 0;
        hsum[i] = 0.0;
      }
      __syncthreads();
      const unsigned long long pre = prefix_s, msk = mask_s;
      for (int j = tid; j < N; j += kDnThreads) {
        const double wv = sc[j];
        const unsigned long long key = static_cast<unsigned long long>(__double_as_longlong(wv));
        if ((key & msk) == pre) {
          const int dg = static_cast<int>((key >> shift) & 255ull);
          atomicAdd(&hcnt[dg], 1u);
          atomicAdd(&hsum[dg], wv);
        }
      }
      __syncthreads();
      if (tid == 0) {
        int dsel = 0;
        for (int dg = 255; dg >= 0; --dg) {
          if (above + hsum[dg] >= target || dg == 0) {
            dsel = dg;
            break;
          }
          above += hsum[dg];
          n_above += hcnt[dg];
        }
        prefix_s = pre | (static_cast<unsigned long long>(dsel) << shift);
        mask_s = msk | (255ull << shift);
        if (pass == 7) {
          // every weight of the final bucket equals w*: take them one by one
          const double ws = __longlong_as_double(static_cast<long long>(prefix_s));
          unsigned long long mcount = 1;
          while (mcount < hcnt[dsel] && above + ws * static_cast<double>(mcount) < target) ++mcount;
          atomicAdd(&count_sum[h], n_above + mcount);
        }
      }
      __syncthreads();
    }
  }
}

__global__ void density_finalize_kernel(const unsigned long long* count_sum, int H,
                                        int rows_per_head, int N, double* density) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  density[h] = static_cast<double>(count_sum[h]) / (static_cast<double>(rows_per_head) * N);
}

constexpr int kDnCtas = kDiagRows;

cudaError_t launch_density(const void* q, const void* k, bool bf16, int H, int N, int Nv, int d,
                           int row_stride, double scale, double tau, double* scratch,
                           unsigned long long* count_sum, double* density, cudaStream_t st) {
  const int rows_per_head = (Nv + row_stride - 1) / row_stride;
  cudaError_t e = cudaMemsetAsync(count_sum, 0, static_cast<size_t>(H) * 8, st);
  if (e != cudaSuccess) return e;
  const int items = H * rows_per_head;
  const int grid = items < kDnCtas ? items : kDnCtas;
  if (bf16)
    density_kernel<<<grid, kDnThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                static_cast<const __nv_bfloat16*>(k), N, Nv, d,
                                                row_stride, rows_per_head, H, scale, tau, scratch,
                                                count_sum);
  else
    density_kernel<<<grid, kDnThreads, 0, st>>>(static_cast<const float*>(q),
                                                static_cast<const float*>(k), N, Nv, d, row_stride,
                                                rows_per_head, H, scale, tau, scratch, count_sum);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  density_finalize_kernel<<<(H + 63) / 64, 64, 0, st>>>(count_sum, H, rows_per_head, N, density);
  return cudaGetLastError();
}

size_t support_smem_bytes(int Ckt, int d, int* R, int* P) {
  int pw = 1;
  while (pw < Ckt) pw <<= 1;
  *P = pw;
  const size_t fixed = static_cast<size_t>(pw) * 12;
  for (int r = 8; r >= 1; --r) {
    const size_t b = static_cast<size_t>(r) * (d + Ckt) * 8 + fixed;
    if (b <= kMaxDynSmem - 4096) {
      *R = r;
      return b;
    }
  }
  *R = 0;
  return 0;
}

cudaError_t launch_support_expansion(const void* qp, const void* kp, bool bf16,
                                     const int32_t* off_q, int oq_stride, const int32_t* off_k,
                                     int Ckt, int H, int N, int d, int Cqv, int stride,
                                     double scale, double tau, uint32_t* union_bits,
                                     unsigned long long* size_sum, double* indiv,
                                     double* aggregate, cudaStream_t st) {
  int R = 0, P = 0;
  const size_t shb = support_smem_bytes(Ckt, d, &R, &P);
  if (R < 1) return cudaErrorInvalidValue;
  const int words = (Ckt + 31) / 32;
  cudaError_t e = cudaMemsetAsync(union_bits, 0, static_cast<size_t>(H) * Cqv * words * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(size_sum, 0, static_cast<size_t>(H) * Cqv * 8, st);
  if (e != cudaSuccess) return e;
  const dim3 grid(kSeCtas, (Cqv + stride - 1) / stride, H);
  if (bf16) {
    e = cudaFuncSetAttribute(support_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(shb));
    if (e != cudaSuccess) return e;
    support_kernel<<<grid, kSeThreads, shb, st>>>(static_cast<const __nv_bfloat16*>(qp),
                                                  static_cast<const __nv_bfloat16*>(kp), off_q,
                                                  oq_stride, off_k, Ckt, N, d, Cqv, stride, R, P,
                                                  scale, tau, union_bits, size_sum);
  } else {
    e = cudaFuncSetAttribute(support_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(shb));
    if (e != cudaSuccess) return e;
    support_kernel<<<grid, kSeThreads, shb, st>>>(static_cast<const float*>(qp),
                                                  static_cast<const float*>(kp), off_q, oq_stride,
                                                  off_k, Ckt, N, d, Cqv, stride, R, P, scale, tau,
                                                  union_bits, size_sum);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  support_finalize_kernel<<<(H * Cqv + 127) / 128, 128, 0, st>>>(
      union_bits, size_sum, off_q, oq_stride, H, Cqv, Ckt, stride, indiv, aggregate);
  return cudaGetLastError();
}

}  // namespace spr
