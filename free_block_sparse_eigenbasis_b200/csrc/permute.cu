// Stage 2 (group-major gather) and stage 3a (centroid block scores + top-k
// routing) of the path: "Partition the Support, Reconstruct the Residual",
// 2.C (contiguous group-major layouts), and "Attention Sparsity is
// Input-Stable", block selection (scores C_q[i] . C_k[j] from block centres,
// top-k key blocks per query block).
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

// dst[h, i, :] = src[h, perm[h, i], :]; rows are copied with 16-byte vectors.
__global__ void gather_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                   const int32_t* __restrict__ perm, int N, int vec_per_row,
                                   size_t total_vec) {
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total_vec) return;
  const size_t row = t / vec_per_row;
  const int v = static_cast<int>(t % vec_per_row);
  const size_t h = row / N;
  const size_t srow = h * N + static_cast<size_t>(perm[row]);
  dst[t] = __ldg(src + srow * vec_per_row + v);
}

// One CTA per (query group g, head h): fp64 scores of all key groups in
// shared memory, top-k by rank (greater score first, lower index on ties),
// kept ids written in ascending order.
constexpr int kRouteThreads = 256;

__global__ void __launch_bounds__(kRouteThreads) route_kernel(const double* __restrict__ cq,
                                                              const double* __restrict__ ckr,
                                                              int Cq, int Ck, int d, double scale,
                                                              const int32_t* __restrict__ kh,
                                                              int kmax, int32_t* __restrict__ csr) {
  extern __shared__ double rsm[];
  double* score = rsm;                                       // [Ck]
  double* qv = rsm + Ck;                                     // [d]
  int* kept = reinterpret_cast<int*>(qv + d);                // [Ck]
  __shared__ int wsum[kRouteThreads / 32];
  __shared__ int carry;
  const int g = blockIdx.x, h = blockIdx.y;
  const double* qrow = cq + (static_cast<size_t>(h) * Cq + g) * d;
  for (int a = threadIdx.x; a < d; a += blockDim.x) qv[a] = qrow[a];
  __syncthreads();
  const double* ckh = ckr + static_cast<size_t>(h) * Ck * d;
  for (int c = threadIdx.x; c < Ck; c += blockDim.x) {
    const double* kr = ckh + static_cast<size_t>(c) * d;
    double acc = 0.0;
    for (int a = 0; a < d; ++a) acc = fma(qv[a], kr[a], acc);
    score[c] = scale * acc;
  }
  __syncthreads();
  const int k = kh[h];
  for (int c = threadIdx.x; c < Ck; c += blockDim.x) {
    const double sc = score[c];
    int rank = 0;
    for (int o = 0; o < Ck; ++o) {
      const double so = score[o];
      rank += (so > sc) || (so == sc && o < c);
    }
    kept[c] = rank < k ? 1 : 0;
  }
  __syncthreads();
  // ascending compaction of the kept ids (block-wide exclusive scan)
  int32_t* out = csr + (static_cast<size_t>(h) * Cq + g) * kmax;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < Ck; base += blockDim.x) {
    const int c = base + threadIdx.x;
    const int f = (c < Ck) ? kept[c] : 0;
    int x = f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[wid] = x;
    __syncthreads();
    int before = carry;
    for (int w = 0; w < wid; ++w) before += wsum[w];
    before += x - f;
    if (f) out[before] = c;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = before + f;
    __syncthreads();
  }
  for (int i = k + threadIdx.x; i < kmax; i += blockDim.x) out[i] = -1;
}

struct KhParam {
  int32_t v[SPARSEPR_MAX_HEADS];
};

__global__ void write_k_kernel(KhParam kp, int H, int32_t* out) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) out[h] = kp.v[h];
}

}  // namespace

cudaError_t launch_gather_rows(const void* src, void* dst, const int32_t* perm, int H, int N,
                               int d, int elem_bytes, cudaStream_t st) {
  const int vec = d * elem_bytes / 16;
  const size_t total = static_cast<size_t>(H) * N * vec;
  gather_rows_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), perm, N, vec, total);
  return cudaGetLastError();
}

cudaError_t launch_route(const double* cq, const double* ckr, int H, int Cq, int Ck, int d,
                         double scale, const int32_t* kh, int kmax, int32_t* csr,
                         cudaStream_t st) {
  const size_t shb = static_cast<size_t>(Ck) * 8 + static_cast<size_t>(d) * 8 +
                     static_cast<size_t>(Ck) * 4;
  cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(shb));
  if (e != cudaSuccess) return e;
  route_kernel<<<dim3(Cq, H), kRouteThreads, shb, st>>>(cq, ckr, Cq, Ck, d, scale, kh, kmax, csr);
  return cudaGetLastError();
}

cudaError_t launch_range_mean(const void* X, int x_kind, int H, int N, int d, const int32_t* off,
                              int C, double* out, cudaStream_t st) {
  return launch_group_mean(X, x_kind, static_cast<long long>(N) * d, d, d, nullptr, 0, off, C + 1,
                           C, H, false, out, nullptr, nullptr, 0, st);
}

cudaError_t launch_write_k(const int32_t* kh_host_vals, int H, int32_t* k_per_head,
                           cudaStream_t st) {
  KhParam kp;
  for (int h = 0; h < SPARSEPR_MAX_HEADS; ++h) kp.v[h] = (h < H) ? kh_host_vals[h] : 0;
  write_k_kernel<<<(H + 127) / 128, 128, 0, st>>>(kp, H, k_per_head);
  return cudaGetLastError();
}

}  // namespace spr
