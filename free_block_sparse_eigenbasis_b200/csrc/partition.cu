// Stage 1 of "Partition the Support, Reconstruct the Residual" (2.A,
// response-coupled partitioning): sampled-query metric M_K, key response
// coordinates in its eigenbasis, key k-means, K/V group centroids, query
// k-means on logit profiles (in the exact d-space form with
// G = scale^2 C_K^T C_K).
//
// All distance, centroid and metric arithmetic is fp64; sums run in a fixed
// order, so labels do not depend on scheduling.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

// ---------------------------------------------------------------------------
// Initial centroids: partial Fisher-Yates shuffle driven by SplitMix64
// (Steele, Lea & Flood 2014). Draw i uses the generator's (i + 1)-th state,
// so every swap target j_i = i + z_i mod (Nv - i) is formed in parallel
// first; the swaps then run in order on one thread. The virtual array
// a[i] = i is kept as a small open-addressing map of the positions that
// moved; position i is never read after step i (later targets are > i), so
// only the swap target j_i is written back.
// ---------------------------------------------------------------------------
constexpr int kFyTable = 16384;  // >= 2 * kMaxGroups, power of two

__device__ __forceinline__ int fy_find(const int32_t* keys, int32_t pos) {
  unsigned s = (static_cast<unsigned>(pos) * 2654435761u) & (kFyTable - 1);
  while (keys[s] != -1 && keys[s] != pos) s = (s + 1) & (kFyTable - 1);
  return static_cast<int>(s);
}

__global__ void fy_init_kernel(int Nv, int Ck, int Cq, uint64_t seed, int32_t* init_k,
                               int32_t* init_q) {
  extern __shared__ int32_t tab[];
  int32_t* keys = tab;
  int32_t* vals = tab + kFyTable;
  int32_t* tgt = vals + kFyTable;  // [C] swap targets
  const int h = blockIdx.x, which = blockIdx.y;
  const int C = which ? Cq : Ck;
  int32_t* out = which ? init_q + static_cast<size_t>(h) * Cq : init_k + static_cast<size_t>(h) * Ck;
  for (int i = threadIdx.x; i < kFyTable; i += blockDim.x) keys[i] = -1;
  const uint64_t base = seed ^ static_cast<uint64_t>(2 * h + which);
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    uint64_t z = base + static_cast<uint64_t>(i + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    tgt[i] = i + static_cast<int>(z % static_cast<uint64_t>(Nv - i));
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  for (int i = 0; i < C; ++i) {
    const int j = tgt[i];
    const int si = fy_find(keys, i);
    const int32_t vi = (keys[si] == i) ? vals[si] : i;
    const int sj = fy_find(keys, j);
    const int32_t vj = (keys[sj] == j) ? vals[sj] : j;
    keys[sj] = j;  // a match or the empty slot that ends j's probe
    vals[sj] = vi;
    out[i] = vj;
  }
}

// e = 16 (the workloads' eigenbasis size): thread = two key rows with all 16
// coordinates of each in registers; the rows of k are streamed with 16-byte
// loads and W [d][16] is read from shared memory as 16-byte broadcasts, so
// every value of W read serves two rows. Same ascending-column sums as
// above. With `zp` given it also writes what the tensor-core assignment
// reads of each row: its three bf16 planes (hi, mid, lo: each the bf16
// rounding of what the planes before it leave) and its norm rounded up, with
// the squares summed in the order of split_rows_vec_kernel (pairs of
// columns, then a butterfly over eight of them), so both give the same bits.
constexpr int kZRowThreads = 128;
constexpr int kZ16Rows = 2;  // rows per thread

template <typename T>
__global__ void __launch_bounds__(kZRowThreads, 4)
    zproj_row16_kernel(const T* k, int N, int Nv, int d, const double* wk, double* z,
                       __nv_bfloat16* zp, long long zps, float* xnorm) {
  constexpr int E = 16, EPT = 16 / sizeof(T);
  extern __shared__ double w16[];  // [d][16]
  const int h = blockIdx.y;
  const int j0 = blockIdx.x * kZRowThreads * kZ16Rows + threadIdx.x;
  const double* W = wk + static_cast<size_t>(h) * d * E;
  for (int t = threadIdx.x; t < d * E; t += kZRowThreads) w16[t] = W[t];
  __syncthreads();
  if (j0 >= Nv) return;
  const bool two = j0 + kZRowThreads < Nv;
  const T* kr0 = k + (static_cast<size_t>(h) * N + j0) * d;
  const T* kr1 = two ? kr0 + static_cast<size_t>(kZRowThreads) * d : kr0;
  double acc[kZ16Rows][E];
#pragma unroll
  for (int r = 0; r < kZ16Rows; ++r)
#pragma unroll
    for (int c = 0; c < E; ++c) acc[r][c] = 0.0;
  // the next 16-byte pieces of both rows are loaded while the current ones
  // are multiplied
  uint4 u0 = *reinterpret_cast<const uint4*>(kr0), u1 = *reinterpret_cast<const uint4*>(kr1);
#pragma unroll 1
  for (int a0 = 0; a0 < d; a0 += EPT) {
    uint4 n0 = u0, n1 = u1;
    if (a0 + EPT < d) {
      n0 = *reinterpret_cast<const uint4*>(kr0 + a0 + EPT);
      n1 = *reinterpret_cast<const uint4*>(kr1 + a0 + EPT);
    }
    double kv[kZ16Rows][EPT];
    vwiden16<T>(u0, kv[0]);
    vwiden16<T>(u1, kv[1]);
    u0 = n0;
    u1 = n1;
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      const double2* wa = reinterpret_cast<const double2*>(w16 + (a0 + i) * E);
#pragma unroll
      for (int c2 = 0; c2 < E / 2; ++c2) {
        const double2 wv = wa[c2];
#pragma unroll
        for (int r = 0; r < kZ16Rows; ++r) {
          acc[r][2 * c2] = fma(kv[r][i], wv.x, acc[r][2 * c2]);
          acc[r][2 * c2 + 1] = fma(kv[r][i], wv.y, acc[r][2 * c2 + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kZ16Rows; ++r) {
    if (r == 1 && !two) break;
    double2* zr = reinterpret_cast<double2*>(
        z + (static_cast<size_t>(h) * Nv + j0 + r * kZRowThreads) * E);
#pragma unroll
    for (int c2 = 0; c2 < E / 2; ++c2) zr[c2] = make_double2(acc[r][2 * c2], acc[r][2 * c2 + 1]);
    if (zp) {
      const size_t row = static_cast<size_t>(h) * Nv + j0 + r * kZRowThreads;
      double s8[E / 2];
#pragma unroll
      for (int t = 0; t < E / 2; ++t)
        s8[t] = fma(acc[r][2 * t + 1], acc[r][2 * t + 1], acc[r][2 * t] * acc[r][2 * t]);
      const double ss = ((s8[0] + s8[4]) + (s8[2] + s8[6])) + ((s8[1] + s8[5]) + (s8[3] + s8[7]));
      xnorm[row] = static_cast<float>(sqrt(ss) * (1.0 + 1e-6));
#pragma unroll
      for (int pl = 0; pl < 3; ++pl) {
        __align__(16) __nv_bfloat16 b[E];
#pragma unroll
        for (int i = 0; i < E; ++i) {
          b[i] = __double2bfloat16(acc[r][i]);
          acc[r][i] -= static_cast<double>(__bfloat162float(b[i]));
        }
        uint4* dst = reinterpret_cast<uint4*>(zp + pl * zps + row * E);
        dst[0] = *reinterpret_cast<const uint4*>(b);
        dst[1] = *reinterpret_cast<const uint4*>(b + 8);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Gram kernels: out = factor * sum_s x_s y_s^T (+ diag I), on the fp64 tensor
// cores (mma.sync m8n8k4, fp64 products and sums). A CTA of 4 warps forms a
// 32x32 output tile over one range of the rows s (ascending), each warp a
// 16x16 quarter (2x2 accumulators of 8x8); the rows stream through shared
// memory 32 at a time, the next chunk's loads issued before the current
// chunk's MMAs. With several ranges per Gram (more CTAs, so more loads in
// flight) each range writes its partial sums and gram_reduce_kernel adds the
// ranges in order.
// ---------------------------------------------------------------------------
constexpr int kGT = 32;   // output tile edge
constexpr int kGS = 32;   // samples per chunk
constexpr int kGPad = 40; // shared row stride (doubles): fragment loads take two wavefronts
constexpr int kGThreads = 128;
constexpr int kGLoads = kGS * kGT / kGThreads;  // elements of x (and of y) per thread per chunk

__device__ __forceinline__ void mma_f64_8x8x4(double (&c)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(c[0]), "+d"(c[1])
               : "d"(a), "d"(b));
}

template <typename Loader>
__device__ void gram_tile(Loader ld, int s_beg, int S, int d, double factor, double diag,
                          double* out) {
  __shared__ double xs[kGS][kGPad];
  __shared__ double ys[kGS][kGPad];
  __shared__ long long rows[2][kGS];  // source rows of a chunk's samples, two chunks
  const int a0 = blockIdx.x * kGT, b0 = blockIdx.y * kGT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wa = (warp >> 1) * 16, wb = (warp & 1) * 16;  // this warp's quarter
  // fragments: A (8x4, row) a[r = lane / 4][k = lane % 4] = x_{s+k}[row r];
  // B (4x8, col) b[k = lane % 4][n = lane / 4] = y_{s+k}[col n];
  // C (8x8) c[r = lane / 4][n = 2 (lane % 4) + {0, 1}]
  const int fr = lane >> 2, fk = lane & 3;
  double acc[2][2][2];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
  // element e of this thread's share of a chunk: sample ss = t / kGT, column cc = t % kGT
  double px[kGLoads], py[kGLoads];
  auto fetch = [&](int s0, const long long* rw) {
#pragma unroll
    for (int e = 0; e < kGLoads; ++e) {
      const int t = threadIdx.x + e * kGThreads;
      const int ss = t / kGT, cc = t % kGT;
      const bool in = s0 + ss < S;
      px[e] = (in && a0 + cc < d) ? ld.x(rw[ss], a0 + cc) : 0.0;
      py[e] = (in && b0 + cc < d) ? ld.y(rw[ss], b0 + cc) : 0.0;
    }
  };
  if (threadIdx.x < kGS && s_beg + static_cast<int>(threadIdx.x) < S)
    rows[0][threadIdx.x] = ld.row(s_beg + threadIdx.x);
  __syncthreads();
  fetch(s_beg, rows[0]);
  for (int c = 0, s0 = s_beg; s0 < S; ++c, s0 += kGS) {
    __syncthreads();  // the previous chunk has been read
#pragma unroll
    for (int e = 0; e < kGLoads; ++e) {
      const int t = threadIdx.x + e * kGThreads;
      xs[t / kGT][t % kGT] = px[e];
      ys[t / kGT][t % kGT] = py[e];
    }
    const int s1 = s0 + kGS;
    if (threadIdx.x < kGS && s1 + static_cast<int>(threadIdx.x) < S)
      rows[(c + 1) & 1][threadIdx.x] = ld.row(s1 + threadIdx.x);
    __syncthreads();
    if (s1 < S) fetch(s1, rows[(c + 1) & 1]);
#pragma unroll
    for (int k0 = 0; k0 < kGS; k0 += 4) {
      double fa[2], fb[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) fa[i] = xs[k0 + fk][wa + 8 * i + fr];
#pragma unroll
      for (int j = 0; j < 2; ++j) fb[j] = ys[k0 + fk][wb + 8 * j + fr];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) mma_f64_8x8x4(acc[i][j], fa[i], fb[j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int a = a0 + wa + 8 * i + fr, b = b0 + wb + 8 * j + 2 * fk + t;
        if (a < d && b < d)
          out[static_cast<size_t>(a) * d + b] = factor * acc[i][j][t] + (a == b ? diag : 0.0);
      }
}

// x(row, a) / y(row, b): element a (b) of source row `row`; row(s): the
// source row of sample s (computed once per chunk of samples)
template <typename T>
struct SampledQueryLoader {
  const T* q;
  int Nv, Ms, d;
  __device__ long long row(int s) const { return ((2LL * s + 1) * Nv) / (2LL * Ms); }
  __device__ double x(long long row, int a) const { return to_f64(q, static_cast<size_t>(row) * d + a); }
  __device__ double y(long long row, int b) const { return x(row, b); }
};

// range sp of `splits` equal ranges of S rows
__device__ __forceinline__ void gram_range(int S, int splits, int sp, int* beg, int* end) {
  *beg = static_cast<int>((static_cast<long long>(S) * sp) / splits);
  *end = static_cast<int>((static_cast<long long>(S) * (sp + 1)) / splits);
}

template <typename T>
__global__ void __launch_bounds__(kGThreads)
    metric_mk_kernel(const T* q, int N, int Nv, int d, int Ms, int splits, double* out,
                     double* part) {
  const int h = blockIdx.z / splits, sp = blockIdx.z % splits;
  SampledQueryLoader<T> ld{q + static_cast<size_t>(h) * N * d, Nv, Ms, d};
  int b, e;
  gram_range(Ms, splits, sp, &b, &e);
  if (splits == 1)
    gram_tile(ld, b, e, d, 1.0 / Ms, 0.0, out + static_cast<size_t>(h) * d * d);
  else
    gram_tile(ld, b, e, d, 1.0, 0.0, part + (static_cast<size_t>(h) * splits + sp) * d * d);
}

struct F64Loader {
  const double *X, *Y, *xm, *ym;
  int ld;
  __device__ long long row(int s) const { return s; }
  __device__ double x(long long s, int a) const {
    return X[static_cast<size_t>(s) * ld + a] - (xm ? xm[a] : 0.0);
  }
  __device__ double y(long long s, int b) const {
    return Y[static_cast<size_t>(s) * ld + b] - (ym ? ym[b] : 0.0);
  }
};

__global__ void __launch_bounds__(kGThreads) gram_f64_kernel(const __grid_constant__ GramJobs g) {
  const int jh = blockIdx.z / g.splits, sp = blockIdx.z % g.splits;  // jh = job * H + head
  const int job = jh / g.H, h = jh % g.H;
  const GramJob& J = g.job[job];
  F64Loader l{J.X + h * J.hsx, J.Y + h * J.hsy, J.xm ? J.xm + h * J.ms : nullptr,
              J.ym ? J.ym + h * J.ms : nullptr, g.ld};
  int b, e;
  gram_range(g.S, g.splits, sp, &b, &e);
  if (g.splits == 1)
    gram_tile(l, b, e, g.d, J.factor, J.diag, J.out + h * J.os);
  else
    gram_tile(l, b, e, g.d, 1.0, 0.0,
              g.part + (static_cast<size_t>(jh) * g.splits + sp) * g.d * g.d);
}

// out = factor * (sum of the ranges' partial sums, in range order) + diag I
__global__ void gram_reduce_kernel(const __grid_constant__ GramJobs g) {
  const int jh = blockIdx.y, job = jh / g.H, h = jh % g.H;
  const GramJob& J = g.job[job];
  const int dd = g.d * g.d;
  const double* P = g.part + static_cast<size_t>(jh) * g.splits * dd;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < dd; i += gridDim.x * blockDim.x) {
    double sum = P[i];
    for (int sp = 1; sp < g.splits; ++sp) sum += P[static_cast<size_t>(sp) * dd + i];
    const int a = i / g.d, b = i % g.d;
    J.out[h * J.os + i] = J.factor * sum + (a == b ? J.diag : 0.0);
  }
}

// ranges per Gram: about 256 rows each, at most kGramSplits
int gram_splits(int S) {
  int sp = S / 256;
  if (sp > kGramSplits) sp = kGramSplits;
  return sp < 1 ? 1 : sp;
}

// ---------------------------------------------------------------------------
// Key response coordinates z = W^T k, W = U_e L_e^{1/2} ([d, e] fp64).
// ---------------------------------------------------------------------------
constexpr int kZRows = 128;
constexpr int kZThreads = 256;

// 16-byte vector of k widened to float
__device__ __forceinline__ int zvec_elems(const __nv_bfloat16*) { return 8; }
__device__ __forceinline__ int zvec_elems(const float*) { return 4; }
__device__ __forceinline__ void zvec_store(const __nv_bfloat16* src, float* dst) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    dst[2 * i] = __uint_as_float(w[i] << 16);
    dst[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void zvec_store(const float* src, float* dst) {
  const float4 v = *reinterpret_cast<const float4*>(src);
  dst[0] = v.x;
  dst[1] = v.y;
  dst[2] = v.z;
  dst[3] = v.w;
}

// Block = 128 key rows: the rows are staged in shared memory (as fp32, exact
// for bf16 / fp32 inputs) with 16-byte loads; thread t computes 8 of the e
// coordinates of row t % 128 (per column of k: one shared load of k and four
// 16-byte broadcast loads of w serve 8 fma), summing over the d columns in
// ascending order in fp64.
template <typename T>
__global__ void __launch_bounds__(kZThreads) zproj_kernel(const T* k, int N, int Nv, int d, int e,
                                                          const double* wk, double* z) {
  extern __shared__ double zsm[];
  double* w = zsm;                                    // [d][e]
  float* ks = reinterpret_cast<float*>(zsm + d * e);  // [kZRows][d+1]
  const int h = blockIdx.y;
  const int j0 = blockIdx.x * kZRows;
  const double* W = wk + static_cast<size_t>(h) * d * e;
  for (int t = threadIdx.x; t < d * e; t += blockDim.x) w[t] = W[t];
  const T* kh = k + static_cast<size_t>(h) * N * d;
  const int ve = zvec_elems(kh), vpr = d / ve;  // elements per vector, vectors per row
  for (int t = threadIdx.x; t < kZRows * vpr; t += blockDim.x) {
    const int r = t / vpr, a = (t % vpr) * ve;
    const int j = j0 + r;
    float tmp[8];
    if (j < Nv) {
      zvec_store(kh + static_cast<size_t>(j) * d + a, tmp);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) tmp[i] = 0.f;
    }
    for (int i = 0; i < ve; ++i) ks[r * (d + 1) + a + i] = tmp[i];
  }
  __syncthreads();
  const int r = threadIdx.x % kZRows;
  const int j = j0 + r;
  if (j >= Nv) return;
  const float* kr = ks + r * (d + 1);
  double* zr = z + (static_cast<size_t>(h) * Nv + j) * e;
  for (int c0 = (threadIdx.x / kZRows) * 8; c0 < e; c0 += (kZThreads / kZRows) * 8) {
    const int ne = min(8, e - c0);
    double acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.0;
    if (ne == 8 && (e % 2) == 0) {
      for (int a = 0; a < d; ++a) {
        const double kv = static_cast<double>(kr[a]);
        const double2* wa = reinterpret_cast<const double2*>(w + a * e + c0);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const double2 wv = wa[c];
          acc[2 * c] = fma(kv, wv.x, acc[2 * c]);
          acc[2 * c + 1] = fma(kv, wv.y, acc[2 * c + 1]);
        }
      }
    } else {
      for (int a = 0; a < d; ++a) {
        const double kv = static_cast<double>(kr[a]);
        const double* wa = w + a * e + c0;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (c < ne) acc[c] = fma(kv, wa[c], acc[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < ne) zr[c0 + c] = acc[c];
  }
}

// ---------------------------------------------------------------------------
// Gather initial centroids (rows idx of src) as fp64, with squared norms.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double load_x(const void* X, int kind, size_t i) {
  if (kind == kXf64) return static_cast<const double*>(X)[i];
  if (kind == kXbf16) return to_f64(static_cast<const __nv_bfloat16*>(X), i);
  return to_f64(static_cast<const float*>(X), i);
}

__global__ void gather_init_kernel(const void* src, int kind, long long hs, int ld, int D,
                                   const int32_t* idx, int C, double* dst, double* norms) {
  const int h = blockIdx.y;
  const int c = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= C) return;
  const size_t row = static_cast<size_t>(idx[static_cast<size_t>(h) * C + c]);
  double ss = 0.0;
  for (int t = lane; t < D; t += 32) {
    const double v = load_x(src, kind, h * hs + row * ld + t);
    dst[(static_cast<size_t>(h) * C + c) * D + t] = v;
    ss = fma(v, v, ss);
  }
  ss = warp_sum_f64(ss);
  if (norms && lane == 0) norms[static_cast<size_t>(h) * C + c] = ss;
}

// ---------------------------------------------------------------------------
// Nearest centroid: labels[i] = argmin_j (c_j - 2 x_i . y_j), lowest j on
// ties, fp64. 64 rows x 64 centroids per tile step, 16x16 threads, 4x4
// register block per thread, D in chunks of 32.
// The value c_j - 2 x.y_j is the squared distance minus x^T G x, with G = I
// (keys: y = mu, c = |mu|^2) or the query metric G (queries: y = G qbar,
// c = qbar^T G qbar); near ties (see kNearTieRel) are counted from the two
// smallest values plus x^T G x (a null stats pointer counts none). For
// G != I the quadratic form is only
// formed for candidate rows, whose gap lies within 1e-11 of
// |second value| + trace(G) |x|^2 (an upper bound of the second distance,
// G being positive semidefinite).
// ---------------------------------------------------------------------------
constexpr int kAR = 64, kAC = 64, kAK = 32;

__device__ double quad_form_row(const void* X, int kind, size_t xb, int D, const double* G) {
  double acc = 0.0;
  for (int a = 0; a < D; ++a) {
    double ga = 0.0;
    for (int b = 0; b < D; ++b) ga = fma(G[static_cast<size_t>(a) * D + b], load_x(X, kind, xb + b), ga);
    acc = fma(load_x(X, kind, xb + a), ga, acc);
  }
  return acc;
}

__global__ void __launch_bounds__(256) argmin_kernel(const void* X, int kind, long long hsx,
                                                     int ldx, int n, int D, const double* Y,
                                                     const double* c, int m, int32_t* labels,
                                                     int32_t* flags, int flag_base,
                                                     const double* G, DeviceStats* stats) {
  __shared__ double xs[kAK][kAR + 2];
  __shared__ double ys[kAK][kAC + 2];
  __shared__ double gtr;
  const int h = blockIdx.y;
  int32_t* fl = flags + h * 4;
  if (fl[flag_base + 1]) return;  // this head's k-means already converged
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int r0 = blockIdx.x * kAR;
  const double* Yh = Y + static_cast<size_t>(h) * m * D;
  const double* ch = c + static_cast<size_t>(h) * m;
  const double* Gh = G ? G + static_cast<size_t>(h) * D * D : nullptr;
  if (threadIdx.x == 0) {
    double t = 0.0;
    if (Gh)
      for (int a = 0; a < D; ++a) t += Gh[static_cast<size_t>(a) * D + a];
    gtr = t;
  }
  Top2 best[4];
  double xx[4] = {0.0, 0.0, 0.0, 0.0};  // |x|^2 of this thread's rows
#pragma unroll
  for (int i = 0; i < 4; ++i) best[i] = top2_empty();
  for (int c0 = 0; c0 < m; c0 += kAC) {
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int k0 = 0; k0 < D; k0 += kAK) {
      for (int t = threadIdx.x; t < kAK * kAR; t += blockDim.x) {
        const int rr = t / kAK, kk = t % kAK;
        const int row = r0 + rr, col = k0 + kk;
        xs[kk][rr] = (row < n && col < D)
                         ? load_x(X, kind, h * hsx + static_cast<size_t>(row) * ldx + col)
                         : 0.0;
        const int cc = c0 + rr;
        ys[kk][rr] = (cc < m && col < D) ? Yh[static_cast<size_t>(cc) * D + col] : 0.0;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kAK; ++kk) {
        double xv[4], yv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[i] = xs[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) yv[j] = ys[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fma(xv[i], yv[j], acc[i][j]);
        if (c0 == 0)
#pragma unroll
          for (int i = 0; i < 4; ++i) xx[i] = fma(xv[i], xv[i], xx[i]);
      }
      __syncthreads();
    }
    // epilogue: nearest and second nearest of this centroid chunk
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      Top2 t = top2_empty();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = c0 + tx * 4 + j;
        if (cc < m) top2_push(t, ch[cc] - 2.0 * acc[i][j], cc);
      }
      // reduce over the 16 lanes sharing these rows (lowest index on ties)
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) {
        const double o1 = __shfl_xor_sync(0xffffffffu, t.b1, o);
        const int oi = __shfl_xor_sync(0xffffffffu, t.i1, o);
        const double o2 = __shfl_xor_sync(0xffffffffu, t.b2, o);
        top2_merge(t, o1, oi, o2);
      }
      top2_merge(best[i], t.b1, t.i1, t.b2);
    }
  }
  if (tx == 0) {
    int changed = 0, ties = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = r0 + ty * 4 + i;
      if (row < n) {
        int32_t* lp = labels + static_cast<size_t>(h) * n + row;
        if (*lp != best[i].i1) changed++;
        *lp = best[i].i1;
        const double gap = best[i].b2 - best[i].b1;
        if (m > 1) {
          if (!Gh) {
            ties += (gap <= kNearTieRel * (best[i].b2 + xx[i]));
          } else if (gap <= 1e-11 * (fabs(best[i].b2) + gtr * xx[i])) {
            const double xgx =
                quad_form_row(X, kind, h * hsx + static_cast<size_t>(row) * ldx, D, Gh);
            ties += (gap <= kNearTieRel * (best[i].b2 + xgx));
          }
        }
      }
    }
    if (changed) atomicAdd(&fl[flag_base + 0], changed);
    if (ties && stats)
      atomicAdd(reinterpret_cast<unsigned long long*>(&stats->near_ties[flag_base >> 1]),
                static_cast<unsigned long long>(ties));
  }
}

// After a pass: count it; a pass after the first that changed no label ends
// that head's k-means (labels repeat).
__global__ void finalize_pass_kernel(int H, int pass, int32_t* flags, int flag_base,
                                     int32_t* passes_out) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  int32_t* fl = flags + h * 4;
  if (fl[flag_base + 1]) return;
  passes_out[h] = pass + 1;
  if (pass > 0 && fl[flag_base + 0] == 0) fl[flag_base + 1] = 1;
  fl[flag_base + 0] = 0;
}

// ---------------------------------------------------------------------------
// Group means in a fixed order over the members in the stable sort's order
// (so repeated calls give the same bits).
// ---------------------------------------------------------------------------
constexpr int kMeanThreads = 256;
constexpr int kMeanMaxD = 128;

// One CTA per (group, head). Thread t sums column t % D over the rows
// lo + t / D, lo + t / D + 256 / D, ... of the group (consecutive threads
// read consecutive columns of one row), then the row lanes' partial sums
// are added in shared memory in a fixed order.
template <typename T>
__device__ __forceinline__ double mean_ld(const T* X, size_t i) { return to_f64(X, i); }
template <>
__device__ __forceinline__ double mean_ld<double>(const double* X, size_t i) { return X[i]; }

template <typename T>
__global__ void __launch_bounds__(kMeanThreads) group_mean_kernel(
    const T* X, long long hsx, int ldx, int D, const int32_t* perm, int perm_stride,
    const int32_t* off, int off_stride, int C, bool keep_prev, double* out, double* norms,
    const int32_t* skip, int skip_stride) {
  __shared__ double part[kMeanThreads];
  __shared__ double red[kMeanThreads / 32];
  const int h = blockIdx.y, c = blockIdx.x;
  if (skip && skip[h * skip_stride]) return;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int32_t* oo = off + static_cast<size_t>(h) * off_stride;
  const int32_t* pp = perm ? perm + static_cast<size_t>(h) * perm_stride : nullptr;
  const int lo = oo[c], hi = oo[c + 1], n = hi - lo;
  const int RL = kMeanThreads / D;  // row lanes
  const int col = threadIdx.x % D, rl = threadIdx.x / D;
  const T* Xh = X + h * hsx;
  double acc = 0.0;
  if (rl < RL) {
    int p = lo + rl;
#pragma unroll 1
    for (; p + 3 * RL < hi; p += 4 * RL) {
      size_t r0, r1, r2, r3;
      if (pp) {
        r0 = pp[p];
        r1 = pp[p + RL];
        r2 = pp[p + 2 * RL];
        r3 = pp[p + 3 * RL];
      } else {
        r0 = p;
        r1 = p + RL;
        r2 = p + 2 * RL;
        r3 = p + 3 * RL;
      }
      const double v0 = mean_ld(Xh, r0 * ldx + col), v1 = mean_ld(Xh, r1 * ldx + col);
      const double v2 = mean_ld(Xh, r2 * ldx + col), v3 = mean_ld(Xh, r3 * ldx + col);
      acc += v0;
      acc += v1;
      acc += v2;
      acc += v3;
    }
    for (; p < hi; p += RL) {
      const size_t r = pp ? static_cast<size_t>(pp[p]) : static_cast<size_t>(p);
      acc += mean_ld(Xh, r * ldx + col);
    }
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  double* dst = out + (static_cast<size_t>(h) * C + c) * D;
  double ss = 0.0;
  for (int t = threadIdx.x; t < D; t += blockDim.x) {
    double v;
    if (n > 0) {
      double sum = part[t];
      for (int q = 1; q < RL; ++q) sum += part[q * D + t];
      v = sum / static_cast<double>(n);
    } else {
      v = keep_prev ? dst[t] : 0.0;
    }
    dst[t] = v;
    ss = fma(v, v, ss);
  }
  if (norms) {
    ss = warp_sum_f64(ss);
    if (lane == 0) red[w] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      double sum = red[0];
      for (int q = 1; q < kMeanThreads / 32; ++q) sum += red[q];
      norms[static_cast<size_t>(h) * C + c] = sum;
    }
  }
}

// 16-byte pieces in flight per thread in the vector and warp forms of the
// group mean, and the row positions staged in shared memory at a time.
constexpr int kMeanDepth = 8;
constexpr int kMeanChunk = 1024;     // per CTA (vector form)
constexpr int kMeanWarpChunk = 128;  // per warp (warp form)

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Adds to acc, in ascending order, this thread's 16-byte pieces of the rows
// rows_s[q], q = q0, q0 + RL, ... < nq (row stride ldx, Xh already at the
// thread's columns). The pieces come through the thread's own kMeanDepth
// shared-memory slots (slot s at slot0[s * kMeanThreads]), kMeanDepth copies
// in flight; a slot is refilled only after its piece was added, so the
// thread reads and writes no other thread's slots.
template <typename T, int EPT>
__device__ __forceinline__ void sum_pieces(const T* Xh, int ldx, const int32_t* rows_s, int q0,
                                           int nq, int RL, uint4* slot0, double (&acc)[EPT]) {
  const int K = q0 < nq ? (nq - q0 + RL - 1) / RL : 0;
#pragma unroll
  for (int s = 0; s < kMeanDepth; ++s) {
    if (s < K) cp_async16(slot0 + s * kMeanThreads, Xh + static_cast<size_t>(rows_s[q0 + s * RL]) * ldx);
    cp_async_commit();
  }
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    cp_async_wait<kMeanDepth - 1>();  // the piece k has landed
    uint4* sl = slot0 + (k & (kMeanDepth - 1)) * kMeanThreads;
    double v[EPT];
    vwiden16<T>(*sl, v);
#pragma unroll
    for (int i = 0; i < EPT; ++i) acc[i] += v[i];
    if (k + kMeanDepth < K)
      cp_async16(sl, Xh + static_cast<size_t>(rows_s[q0 + (k + kMeanDepth) * RL]) * ldx);
    cp_async_commit();
  }
  cp_async_wait<0>();
}

// Vector form of the group mean for rows of D * sizeof(T) bytes that split
// into 16-byte pieces: TPR = D * sizeof(T) / 16 threads per row, each summing
// EPT = 16 / sizeof(T) columns over the rows lo + rl, lo + rl + RL, ...
// (RL = 256 / TPR row lanes, kMeanDepth pieces in flight), then the row lanes' sums
// are combined in a fixed order (within a warp by shuffles, across warps in
// shared memory).
template <typename T>
__global__ void __launch_bounds__(kMeanThreads) group_mean_vec_kernel(
    const T* X, long long hsx, int ldx, int D, const int32_t* perm, int perm_stride,
    const int32_t* off, int off_stride, int C, bool keep_prev, double* out, double* norms,
    const int32_t* skip, int skip_stride) {
  constexpr int EPT = 16 / sizeof(T);
  static_assert(sizeof(double) * EPT <= sizeof(uint4) * kMeanDepth, "partial sums fit in the slots");
  __shared__ __align__(16) uint4 slots[kMeanDepth * kMeanThreads];
  __shared__ int32_t rows_s[kMeanChunk];
  __shared__ double red[kMeanThreads / 32];
  double* part = reinterpret_cast<double*>(slots);  // after the sums
  const int h = blockIdx.y, c = blockIdx.x;
  if (skip && skip[h * skip_stride]) return;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int32_t* oo = off + static_cast<size_t>(h) * off_stride;
  const int32_t* pp = perm ? perm + static_cast<size_t>(h) * perm_stride : nullptr;
  const int lo = oo[c], hi = oo[c + 1], n = hi - lo;
  const int TPR = D / EPT, RL = kMeanThreads / TPR;
  const int col = (threadIdx.x % TPR) * EPT, rl = threadIdx.x / TPR;
  const T* Xh = X + h * hsx + col;
  double acc[EPT];
#pragma unroll
  for (int i = 0; i < EPT; ++i) acc[i] = 0.0;
  // the group's rows in chunks of kMeanChunk positions (a multiple of RL, so
  // that row lane rl sums the rows lo + rl, lo + rl + RL, ... in ascending
  // order), their row indices staged in shared memory
#pragma unroll 1
  for (int cb = lo; cb < hi; cb += kMeanChunk) {
    const int nq = min(kMeanChunk, hi - cb);
    __syncthreads();  // the previous chunk's positions are no longer read
    for (int i = threadIdx.x; i < nq; i += kMeanThreads) rows_s[i] = pp ? pp[cb + i] : cb + i;
    __syncthreads();
    sum_pieces<T, EPT>(Xh, ldx, rows_s, rl, nq, RL, slots + threadIdx.x, acc);
  }
  __syncthreads();  // every slot read before the partial sums overwrite them
  // the row lanes of a warp that share columns (lanes TPR apart) first, by
  // shuffles; then the warps' partial rows in shared memory, in warp order
  int prow = rl, npart = RL;
  if (TPR <= 32) {
    for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < EPT; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    prow = w;
    npart = kMeanThreads / 32;
  }
  if (TPR > 32 || lane < TPR)
#pragma unroll
    for (int i = 0; i < EPT; ++i) part[prow * D + col + i] = acc[i];
  __syncthreads();
  double* dst = out + (static_cast<size_t>(h) * C + c) * D;
  double ss = 0.0;
  for (int t = threadIdx.x; t < D; t += blockDim.x) {
    double v;
    if (n > 0) {
      double sum = part[t];
      for (int q = 1; q < npart; ++q) sum += part[q * D + t];
      v = sum / static_cast<double>(n);
    } else {
      v = keep_prev ? dst[t] : 0.0;
    }
    dst[t] = v;
    ss = fma(v, v, ss);
  }
  if (norms) {
    ss = warp_sum_f64(ss);
    if (lane == 0) red[w] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      double sum = red[0];
      for (int q = 1; q < kMeanThreads / 32; ++q) sum += red[q];
      norms[static_cast<size_t>(h) * C + c] = sum;
    }
  }
}

// Warp form of the group mean (TPR = D * sizeof(T) / 16 <= 32 threads per
// row): one warp per group, eight groups per CTA; lane l sums the 16-byte
// piece l % TPR of the rows lo + l / TPR, lo + l / TPR + 32 / TPR, ...
// (kMeanDepth pieces in flight), then the lanes that share a piece are added
// by shuffles in a fixed order.
constexpr int kMeanWarpGroups = 8;

template <typename T>
__global__ void __launch_bounds__(kMeanWarpGroups * 32) group_mean_warp_kernel(
    const T* X, long long hsx, int ldx, int D, const int32_t* perm, int perm_stride,
    const int32_t* off, int off_stride, int C, bool keep_prev, double* out, double* norms,
    const int32_t* skip, int skip_stride) {
  constexpr int EPT = 16 / sizeof(T);
  static_assert(kMeanWarpGroups * 32 == kMeanThreads, "slot stride");
  __shared__ __align__(16) uint4 slots[kMeanDepth * kMeanThreads];
  __shared__ int32_t rows_s[kMeanWarpGroups][kMeanWarpChunk];
  const int h = blockIdx.y;
  const int c = blockIdx.x * kMeanWarpGroups + static_cast<int>(threadIdx.x >> 5);
  if (c >= C) return;  // the whole warp
  if (skip && skip[h * skip_stride]) return;
  const int lane = threadIdx.x & 31;
  const int32_t* oo = off + static_cast<size_t>(h) * off_stride;
  const int32_t* pp = perm ? perm + static_cast<size_t>(h) * perm_stride : nullptr;
  const int lo = oo[c], hi = oo[c + 1], n = hi - lo;
  const int TPR = D / EPT, RL = 32 / TPR;  // row lanes
  const int col = (lane % TPR) * EPT, rl = lane / TPR;
  const T* Xh = X + h * hsx + col;
  double acc[EPT];
#pragma unroll
  for (int i = 0; i < EPT; ++i) acc[i] = 0.0;
  // the group's rows in chunks of kMeanWarpChunk positions (a multiple of
  // RL: lane row rl sums the rows lo + rl, lo + rl + RL, ... in ascending
  // order), their row indices staged in the warp's shared memory
  int32_t* rw = rows_s[threadIdx.x >> 5];
#pragma unroll 1
  for (int cb = lo; cb < hi; cb += kMeanWarpChunk) {
    const int nq = min(kMeanWarpChunk, hi - cb);
    __syncwarp();  // the previous chunk's positions are no longer read
    for (int i = lane; i < nq; i += 32) rw[i] = pp ? pp[cb + i] : cb + i;
    __syncwarp();
    sum_pieces<T, EPT>(Xh, ldx, rw, rl, nq, RL, slots + threadIdx.x, acc);
  }
  for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < EPT; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  double* dst = out + (static_cast<size_t>(h) * C + c) * D;
  double ss = 0.0;
  if (lane < TPR) {
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      const double v = (n > 0) ? acc[i] / static_cast<double>(n) : (keep_prev ? dst[col + i] : 0.0);
      dst[col + i] = v;
      ss = fma(v, v, ss);
    }
  }
  if (norms) {
    ss = warp_sum_f64(ss);
    if (lane == 0) norms[static_cast<size_t>(h) * C + c] = ss;
  }
}

// W_g = G qbar_g, c_g = qbar_g^T G qbar_g (fp64, fixed-order reduction).
// One CTA per (8 query centroids, head), 512 threads: thread (a, part) sums
// the quarter `part` of the columns b of row a of W for the CTA's centroids
// (G is symmetric, so column a is read, coalesced across a); the four
// quarters are then added in part order. Every element of G is read once per
// CTA; four times the warps of a thread-per-column form, each with a quarter
// of the dependent loads.
constexpr int kQmaG = 8;
constexpr int kQmaParts = 4;

__global__ void __launch_bounds__(128 * kQmaParts)
    query_metric_apply_kernel(const double* G, const double* qbar, int Cq, int d, double* wg,
                              double* cg, const int32_t* skip, int skip_stride) {
  __shared__ double qs[kQmaG][128];
  __shared__ double part_w[kQmaParts - 1][kQmaG][128];
  __shared__ double red[kQmaG][4];
  const int h = blockIdx.y, g0 = blockIdx.x * kQmaG;
  if (skip && skip[h * skip_stride]) return;
  const int ng = min(kQmaG, Cq - g0);
  const double* Gh = G + static_cast<size_t>(h) * d * d;
  const int a = threadIdx.x & 127, part = threadIdx.x >> 7;
  for (int i = threadIdx.x; i < kQmaG * 128; i += blockDim.x) {
    const int g = i >> 7, b = i & 127;
    qs[g][b] = (g < ng && b < d) ? qbar[(static_cast<size_t>(h) * Cq + g0 + g) * d + b] : 0.0;
  }
  __syncthreads();
  double w[kQmaG];
#pragma unroll
  for (int g = 0; g < kQmaG; ++g) w[g] = 0.0;
  const int span = d / kQmaParts, b0 = part * span;
  if (a < d) {
#pragma unroll 1
    for (int b = b0; b < b0 + span; b += 16) {  // 16 loads of G in flight
      double gb[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) gb[i] = Gh[static_cast<size_t>(b + i) * d + a];
#pragma unroll
      for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int g = 0; g < kQmaG; ++g) w[g] = fma(gb[i], qs[g][b + i], w[g]);
    }
  }
  if (part > 0)
#pragma unroll
    for (int g = 0; g < kQmaG; ++g) part_w[part - 1][g][a] = w[g];
  __syncthreads();
  if (part == 0) {
    const int lane = a & 31, wp = a >> 5;
#pragma unroll
    for (int g = 0; g < kQmaG; ++g) {
      double v = w[g];
#pragma unroll
      for (int pp = 0; pp < kQmaParts - 1; ++pp) v += part_w[pp][g][a];
      if (a < d && g < ng) wg[(static_cast<size_t>(h) * Cq + g0 + g) * d + a] = v;
      const double cv = warp_sum_f64((a < d) ? qs[g][a] * v : 0.0);
      if (lane == 0) red[g][wp] = cv;
    }
  }
  __syncthreads();
  if (threadIdx.x < ng)
    cg[static_cast<size_t>(h) * Cq + g0 + threadIdx.x] =
        (red[threadIdx.x][0] + red[threadIdx.x][1]) + (red[threadIdx.x][2] + red[threadIdx.x][3]);
}

// ---------------------------------------------------------------------------
// Alternative partitions (the ablations' semantic k-means, the co-clustering
// page's bidirectional rounds): helpers around the d-space assignment.
// ---------------------------------------------------------------------------
// G = I (semantic k-means is the d-space form with the identity metric)
__global__ void identity_kernel(double* G, int d) {
  const int h = blockIdx.y;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < d * d; t += gridDim.x * blockDim.x)
    G[static_cast<size_t>(h) * d * d + t] = (t / d == t % d) ? 1.0 : 0.0;
}

// members per group from the counting sort's offsets
__global__ void group_counts_kernel(const int32_t* off, int off_stride, int C, int H,
                                    int32_t* cnt) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * C) return;
  const int h = i / C, c = i % C;
  cnt[i] = off[static_cast<size_t>(h) * off_stride + c + 1] - off[static_cast<size_t>(h) * off_stride + c];
}

// Mean affinity vectors of the blocks: pbar[j] = scale * C xbar_j (C: [m2, d]
// centres of the other side), for blocks j whose mean xbar_j is current:
// every block in the first round, afterwards the blocks with members (an
// empty block keeps its vector). One warp per (8 blocks, centre g): lanes
// over d, then shuffles.
constexpr int kAcRows = 8;

__global__ void __launch_bounds__(256)
    affinity_centres_kernel(const double* xbar, const double* C, int m1, int m2, int d,
                            double scale, const int32_t* cnt, int first, double* pbar) {
  __shared__ double xs[kAcRows][128];
  const int h = blockIdx.y, j0 = blockIdx.x * kAcRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kAcRows * 128; i += blockDim.x) {
    const int r = i >> 7, a = i & 127;
    xs[r][a] = (j0 + r < m1 && a < d) ? xbar[(static_cast<size_t>(h) * m1 + j0 + r) * d + a] : 0.0;
  }
  __syncthreads();
  bool upd[kAcRows];
#pragma unroll
  for (int r = 0; r < kAcRows; ++r)
    upd[r] = j0 + r < m1 && (first || cnt[static_cast<size_t>(h) * m1 + j0 + r] > 0);
  const double* Ch = C + static_cast<size_t>(h) * m2 * d;
  for (int g = warp; g < m2; g += blockDim.x / 32) {
    double acc[kAcRows];
#pragma unroll
    for (int r = 0; r < kAcRows; ++r) acc[r] = 0.0;
    for (int a = lane; a < d; a += 32) {
      const double cv = Ch[static_cast<size_t>(g) * d + a];
#pragma unroll
      for (int r = 0; r < kAcRows; ++r) acc[r] = fma(xs[r][a], cv, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kAcRows; ++r) {
      const double v = warp_sum_f64(acc[r]);
      if (lane == 0 && upd[r]) pbar[(static_cast<size_t>(h) * m1 + j0 + r) * m2 + g] = scale * v;
    }
  }
}

// The d-space form of the affinity distance: for pbar_j (in the space of the
// other side's m2 centres C), |scale C x - pbar_j|^2 = x^T G x + c_j - 2 x . y_j
// with y_j = scale C^T pbar_j and c_j = |pbar_j|^2 (G = scale^2 C^T C is the
// same for every j, so it does not change the nearest block). Thread a
// forms y_j[a]; eight blocks per CTA.
__global__ void __launch_bounds__(128)
    dspace_centres_kernel(const double* pbar, const double* C, int m1, int m2, int d,
                          double scale, double* y, double* c) {
  extern __shared__ double ps[];  // [kAcRows][m2]
  __shared__ double red[kAcRows][4];
  const int h = blockIdx.y, j0 = blockIdx.x * kAcRows, a = threadIdx.x;
  const int lane = a & 31, wp = a >> 5;
  for (int i = a; i < kAcRows * m2; i += blockDim.x) {
    const int r = i / m2, g = i % m2;
    ps[i] = (j0 + r < m1) ? pbar[(static_cast<size_t>(h) * m1 + j0 + r) * m2 + g] : 0.0;
  }
  __syncthreads();
  const double* Ch = C + static_cast<size_t>(h) * m2 * d;
  double acc[kAcRows];
#pragma unroll
  for (int r = 0; r < kAcRows; ++r) acc[r] = 0.0;
  if (a < d)
    for (int g = 0; g < m2; ++g) {
      const double cv = Ch[static_cast<size_t>(g) * d + a];
#pragma unroll
      for (int r = 0; r < kAcRows; ++r) acc[r] = fma(ps[r * m2 + g], cv, acc[r]);
    }
#pragma unroll
  for (int r = 0; r < kAcRows; ++r)
    if (a < d && j0 + r < m1) y[(static_cast<size_t>(h) * m1 + j0 + r) * d + a] = scale * acc[r];
  // c_j = |pbar_j|^2, fixed order: thread a sums g = a, a + 128, ...; then warps
#pragma unroll
  for (int r = 0; r < kAcRows; ++r) {
    double v = 0.0;
    for (int g = a; g < m2; g += blockDim.x) v = fma(ps[r * m2 + g], ps[r * m2 + g], v);
    v = warp_sum_f64(v);
    if (lane == 0) red[r][wp] = v;
  }
  __syncthreads();
  if (a < kAcRows && j0 + a < m1)
    c[static_cast<size_t>(h) * m1 + j0 + a] = (red[a][0] + red[a][1]) + (red[a][2] + red[a][3]);
}

// One co-clustering round ends when both sides' passes are counted: a round
// after the first in which neither keys nor queries changed label ends the
// head's rounds (both sides' done flags).
__global__ void finalize_round_kernel(int H, int round, int32_t* flags, int32_t* passes_k,
                                      int32_t* passes_q) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  int32_t* fl = flags + h * 4;
  if (fl[1]) return;
  passes_k[h] = round + 1;
  passes_q[h] = round + 1;
  if (round > 0 && fl[0] == 0 && fl[2] == 0) {
    fl[1] = 1;
    fl[3] = 1;
  }
  fl[0] = 0;
  fl[2] = 0;
}

__global__ void write_labels_kernel(const int32_t* lab, int H, int N, int Nv, int C_text,
                                    int32_t* out) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<size_t>(H) * N) return;
  const int h = static_cast<int>(i / N), j = static_cast<int>(i % N);
  out[i] = (j < Nv) ? lab[static_cast<size_t>(h) * Nv + j] : C_text;
}

}  // namespace

cudaError_t launch_fy_init(int H, int Nv, int Ck, int Cq, uint64_t seed, int32_t* init_k,
                           int32_t* init_q, cudaStream_t st) {
  if (Ck > kMaxGroups || Cq > kMaxGroups) return cudaErrorInvalidValue;
  const int shb = (2 * kFyTable + kMaxGroups) * 4;
  const cudaError_t e =
      cudaFuncSetAttribute(fy_init_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, shb);
  if (e != cudaSuccess) return e;
  fy_init_kernel<<<dim3(H, 2), 256, shb, st>>>(Nv, Ck, Cq, seed, init_k, init_q);
  return cudaGetLastError();
}

cudaError_t launch_metric_mk(const void* q, bool bf16, int H, int N, int Nv, int d, int Ms,
                             double* out, double* part, cudaStream_t st) {
  const int splits = gram_splits(Ms);
  dim3 grid((d + kGT - 1) / kGT, (d + kGT - 1) / kGT, H * splits);
  if (bf16)
    metric_mk_kernel<<<grid, kGThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(q), N, Nv, d,
                                                 Ms, splits, out, part);
  else
    metric_mk_kernel<<<grid, kGThreads, 0, st>>>(static_cast<const float*>(q), N, Nv, d, Ms,
                                                 splits, out, part);
  if (splits > 1) {
    GramJobs g = {};
    g.job[0] = GramJob{nullptr, nullptr, nullptr, nullptr, 0, 0, 0, out,
                       static_cast<long long>(d) * d, 1.0 / Ms, 0.0};
    g.njobs = 1;
    g.d = d;
    g.H = H;
    g.part = part;
    g.splits = splits;
    gram_reduce_kernel<<<dim3((d * d + 255) / 256, H), 256, 0, st>>>(g);
  }
  return cudaGetLastError();
}

cudaError_t launch_gram_f64(GramJobs g, cudaStream_t st) {
  if (g.njobs < 1 || g.njobs > kGramJobs) return cudaErrorInvalidValue;
  g.splits = gram_splits(g.S);
  dim3 grid((g.d + kGT - 1) / kGT, (g.d + kGT - 1) / kGT, g.H * g.njobs * g.splits);
  gram_f64_kernel<<<grid, kGThreads, 0, st>>>(g);
  if (g.splits > 1)
    gram_reduce_kernel<<<dim3((g.d * g.d + 255) / 256, g.H * g.njobs), 256, 0, st>>>(g);
  return cudaGetLastError();
}

cudaError_t launch_gram_f64(const double* X, const double* Y, const double* xm,
                            const double* ym, long long hsx, long long hsy, int ld, int S, int H,
                            int d, double factor, double diag, double* out, long long os,
                            long long ms, double* part, cudaStream_t st) {
  GramJobs g = {};
  g.job[0] = GramJob{X, Y, xm, ym, hsx, hsy, ms, out, os, factor, diag};
  g.njobs = 1;
  g.ld = ld;
  g.S = S;
  g.d = d;
  g.H = H;
  g.part = part;
  return launch_gram_f64(g, st);
}

cudaError_t launch_zproj(const void* k, bool bf16, int H, int N, int Nv, int d, int e,
                         const double* wk, double* z, __nv_bfloat16* zp, long long zps,
                         float* xnorm, cudaStream_t st) {
  const bool row16 = e == 16 && d % 8 == 0 && reinterpret_cast<uintptr_t>(k) % 16 == 0;
  // the planes only with the two-row form
  if (zp && (!row16 || !xnorm || reinterpret_cast<uintptr_t>(zp) % 16 != 0 || zps % 8 != 0))
    return cudaErrorInvalidValue;
  if (row16) {
    const size_t shb16 = static_cast<size_t>(d) * 16 * 8;
    dim3 g16((Nv + kZRowThreads * kZ16Rows - 1) / (kZRowThreads * kZ16Rows), H);
    if (bf16)
      zproj_row16_kernel<<<g16, kZRowThreads, shb16, st>>>(static_cast<const __nv_bfloat16*>(k), N, Nv,
                                                           d, wk, z, zp, zps, xnorm);
    else
      zproj_row16_kernel<<<g16, kZRowThreads, shb16, st>>>(static_cast<const float*>(k), N, Nv, d,
                                                           wk, z, zp, zps, xnorm);
    return cudaGetLastError();
  }
  const size_t shb = static_cast<size_t>(d) * e * 8 + static_cast<size_t>(kZRows) * (d + 1) * 4;
  dim3 grid((Nv + kZRows - 1) / kZRows, H);
  if (bf16) {
    const cudaError_t err = cudaFuncSetAttribute(
        zproj_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(shb));
    if (err != cudaSuccess) return err;
    zproj_kernel<<<grid, kZThreads, shb, st>>>(static_cast<const __nv_bfloat16*>(k), N, Nv, d, e, wk, z);
  } else {
    const cudaError_t err = cudaFuncSetAttribute(
        zproj_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(shb));
    if (err != cudaSuccess) return err;
    zproj_kernel<<<grid, kZThreads, shb, st>>>(static_cast<const float*>(k), N, Nv, d, e, wk, z);
  }
  return cudaGetLastError();
}

cudaError_t launch_gather_init(const void* src, int src_kind, long long head_stride, int ld,
                               int D, const int32_t* idx, int C, int H, double* dst,
                               double* norms, cudaStream_t st) {
  dim3 grid((C + 3) / 4, H);
  gather_init_kernel<<<grid, 128, 0, st>>>(src, src_kind, head_stride, ld, D, idx, C, dst, norms);
  return cudaGetLastError();
}

cudaError_t launch_argmin(const void* X, int x_kind, long long hsx, int ldx, int n, int D,
                          const double* Y, const double* c, int m, int H, int32_t* labels,
                          int32_t* flags, int flag_base, const double* G, DeviceStats* stats,
                          cudaStream_t st) {
  dim3 grid((n + kAR - 1) / kAR, H);
  argmin_kernel<<<grid, 256, 0, st>>>(X, x_kind, hsx, ldx, n, D, Y, c, m, labels, flags,
                                      flag_base, G, stats);
  return cudaGetLastError();
}

cudaError_t launch_finalize_pass(int H, int pass, int32_t* flags, int flag_base,
                                 int32_t* passes_out, cudaStream_t st) {
  finalize_pass_kernel<<<(H + 127) / 128, 128, 0, st>>>(H, pass, flags, flag_base, passes_out);
  return cudaGetLastError();
}

cudaError_t launch_group_mean(const void* X, int x_kind, long long hsx, int ldx, int D,
                              const int32_t* perm, int perm_stride, const int32_t* off,
                              int off_stride, int C, int H, bool keep_prev, double* out,
                              double* norms, const int32_t* skip, int skip_stride,
                              cudaStream_t st) {
  if (D > kMeanMaxD || D < 1) return cudaErrorInvalidValue;
  dim3 grid(C, H);
  const int es = (x_kind == kXf64) ? 8 : (x_kind == kXbf16 ? 2 : 4);
  const bool vec = (D * es) % 16 == 0 && kMeanThreads % (D * es / 16) == 0 && (ldx * es) % 16 == 0 &&
                   (hsx * es) % 16 == 0 && (reinterpret_cast<uintptr_t>(X) & 15) == 0;
  // the warp form (one warp per group) for short rows, and for rows of up to
  // 32 pieces when the groups are small on average (at most 256 rows), where
  // a CTA per group would spend more time on its start and its reduction
  // than on its rows
  const int tpr = D * es / 16;
  const bool small_groups = hsx / ldx <= 256LL * C;
  if (vec && 32 % tpr == 0 && (D * es <= 128 || small_groups)) {
    const dim3 wgrid((C + kMeanWarpGroups - 1) / kMeanWarpGroups, H);
    if (x_kind == kXf64)
      group_mean_warp_kernel<<<wgrid, kMeanWarpGroups * 32, 0, st>>>(
          static_cast<const double*>(X), hsx, ldx, D, perm, perm_stride, off, off_stride, C,
          keep_prev, out, norms, skip, skip_stride);
    else if (x_kind == kXbf16)
      group_mean_warp_kernel<<<wgrid, kMeanWarpGroups * 32, 0, st>>>(
          static_cast<const __nv_bfloat16*>(X), hsx, ldx, D, perm, perm_stride, off, off_stride, C,
          keep_prev, out, norms, skip, skip_stride);
    else
      group_mean_warp_kernel<<<wgrid, kMeanWarpGroups * 32, 0, st>>>(
          static_cast<const float*>(X), hsx, ldx, D, perm, perm_stride, off, off_stride, C,
          keep_prev, out, norms, skip, skip_stride);
    return cudaGetLastError();
  }
  if (vec) {
    if (x_kind == kXf64)
      group_mean_vec_kernel<<<grid, kMeanThreads, 0, st>>>(static_cast<const double*>(X), hsx, ldx,
                                                           D, perm, perm_stride, off, off_stride, C,
                                                           keep_prev, out, norms, skip, skip_stride);
    else if (x_kind == kXbf16)
      group_mean_vec_kernel<<<grid, kMeanThreads, 0, st>>>(
          static_cast<const __nv_bfloat16*>(X), hsx, ldx, D, perm, perm_stride, off, off_stride, C,
          keep_prev, out, norms, skip, skip_stride);
    else
      group_mean_vec_kernel<<<grid, kMeanThreads, 0, st>>>(static_cast<const float*>(X), hsx, ldx,
                                                           D, perm, perm_stride, off, off_stride, C,
                                                           keep_prev, out, norms, skip, skip_stride);
    return cudaGetLastError();
  }
  if (x_kind == kXf64)
    group_mean_kernel<<<grid, kMeanThreads, 0, st>>>(static_cast<const double*>(X), hsx, ldx, D,
                                                     perm, perm_stride, off, off_stride, C,
                                                     keep_prev, out, norms, skip, skip_stride);
  else if (x_kind == kXbf16)
    group_mean_kernel<<<grid, kMeanThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(X), hsx,
                                                     ldx, D, perm, perm_stride, off, off_stride,
                                                     C, keep_prev, out, norms, skip, skip_stride);
  else
    group_mean_kernel<<<grid, kMeanThreads, 0, st>>>(static_cast<const float*>(X), hsx, ldx, D,
                                                     perm, perm_stride, off, off_stride, C,
                                                     keep_prev, out, norms, skip, skip_stride);
  return cudaGetLastError();
}

cudaError_t launch_query_metric_apply(const double* G, const double* qbar, int Cq, int H, int d,
                                      double* wg, double* cg, const int32_t* skip,
                                      int skip_stride, cudaStream_t st) {
  if (d % (16 * kQmaParts) != 0 || d > 128) return cudaErrorInvalidValue;
  query_metric_apply_kernel<<<dim3((Cq + kQmaG - 1) / kQmaG, H), 128 * kQmaParts, 0, st>>>(
      G, qbar, Cq, d, wg, cg, skip, skip_stride);
  return cudaGetLastError();
}

cudaError_t launch_identity(double* G, int H, int d, cudaStream_t st) {
  identity_kernel<<<dim3((d * d + 255) / 256, H), 256, 0, st>>>(G, d);
  return cudaGetLastError();
}

cudaError_t launch_group_counts(const int32_t* off, int off_stride, int C, int H, int32_t* cnt,
                                cudaStream_t st) {
  group_counts_kernel<<<(H * C + 255) / 256, 256, 0, st>>>(off, off_stride, C, H, cnt);
  return cudaGetLastError();
}

cudaError_t launch_affinity_centres(const double* xbar, const double* C, int m1, int m2, int d,
                                    int H, double scale, const int32_t* cnt, bool first,
                                    double* pbar, cudaStream_t st) {
  if (d > 128) return cudaErrorInvalidValue;
  affinity_centres_kernel<<<dim3((m1 + kAcRows - 1) / kAcRows, H), 256, 0, st>>>(
      xbar, C, m1, m2, d, scale, cnt, first ? 1 : 0, pbar);
  return cudaGetLastError();
}

cudaError_t launch_dspace_centres(const double* pbar, const double* C, int m1, int m2, int d,
                                  int H, double scale, double* y, double* c, cudaStream_t st) {
  const size_t shb = static_cast<size_t>(kAcRows) * m2 * 8;
  if (d > 128 || shb > kMaxDynSmem) return cudaErrorInvalidValue;
  const cudaError_t e = cudaFuncSetAttribute(dspace_centres_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(shb));
  if (e != cudaSuccess) return e;
  dspace_centres_kernel<<<dim3((m1 + kAcRows - 1) / kAcRows, H), 128, shb, st>>>(pbar, C, m1, m2,
                                                                                  d, scale, y, c);
  return cudaGetLastError();
}

cudaError_t launch_finalize_round(int H, int round, int32_t* flags, int32_t* passes_k,
                                  int32_t* passes_q, cudaStream_t st) {
  finalize_round_kernel<<<(H + 127) / 128, 128, 0, st>>>(H, round, flags, passes_k, passes_q);
  return cudaGetLastError();
}

cudaError_t launch_write_labels(const int32_t* lab, int H, int N, int Nv, int C_text,
                                int32_t* out, cudaStream_t st) {
  const size_t tot = static_cast<size_t>(H) * N;
  write_labels_kernel<<<static_cast<unsigned>((tot + 255) / 256), 256, 0, st>>>(lab, H, N, Nv,
                                                                              C_text, out);
  return cudaGetLastError();
}

}  // namespace spr
