// Stage 2 (group-major gather) and stage 3a (centroid block scores + top-k
// routing) of the path: "Partition the Support, Reconstruct the Residual",
// 2.C (contiguous group-major layouts), and "Attention Sparsity is
// Input-Stable", block selection (scores C_q[i] . C_k[j] from block centres,
// top-k key blocks per query block).
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

// dst[h, i, :] = src[h, perm[h, i], :] for one or two (src, dst) pairs that
// share the permutation (K and V), rows copied in 16-byte pieces. Grid: x over
// the rows of a head in blocks of kGatherDepth passes, y over heads, so that
// no index needs a 64-bit division. A thread moves piece v of the rows
// rr, rr + R, ..., rr + (kGatherDepth - 1) R of its block (R = rows per pass,
// 256 / pieces per row); all its loads, of both pairs, are issued before its
// first store, so several are in flight together.
constexpr int kGatherThreads = 256, kGatherDepth = 4;

__global__ void __launch_bounds__(kGatherThreads) gather_rows_kernel(
    const uint4* __restrict__ s0, uint4* __restrict__ d0, const uint4* __restrict__ s1,
    uint4* __restrict__ d1, const int32_t* __restrict__ perm, int N, int vpr) {
  const int rpp = kGatherThreads / vpr;
  const int rr = static_cast<int>(threadIdx.x) / vpr;
  const int v = static_cast<int>(threadIdx.x) - rr * vpr;
  if (rr >= rpp) return;
  const size_t hb = static_cast<size_t>(blockIdx.y) * N;
  const int r0 = static_cast<int>(blockIdx.x) * rpp * kGatherDepth + rr;
  int sr[kGatherDepth];
#pragma unroll
  for (int j = 0; j < kGatherDepth; ++j) {
    const int r = r0 + j * rpp;
    sr[j] = r < N ? __ldg(perm + hb + r) : -1;
  }
  uint4 u[kGatherDepth], w[kGatherDepth];
#pragma unroll
  for (int j = 0; j < kGatherDepth; ++j)
    if (sr[j] >= 0) u[j] = __ldcs(s0 + (hb + sr[j]) * vpr + v);
  if (s1) {
#pragma unroll
    for (int j = 0; j < kGatherDepth; ++j)
      if (sr[j] >= 0) w[j] = __ldcs(s1 + (hb + sr[j]) * vpr + v);
  }
#pragma unroll
  for (int j = 0; j < kGatherDepth; ++j)
    if (sr[j] >= 0) d0[(hb + r0 + j * rpp) * vpr + v] = u[j];
  if (s1) {
#pragma unroll
    for (int j = 0; j < kGatherDepth; ++j)
      if (sr[j] >= 0) d1[(hb + r0 + j * rpp) * vpr + v] = w[j];
  }
}

// ---------------------------------------------------------------------------
// Routing in two kernels: the block-score matrix
// S_h = scale * C_Q C_K^T of a group of heads as one fp64 GEMM (64 x 64 tiles,
// 4 x 4 outputs per thread, dot products summed in ascending column order),
// then one warp per query group selects the top-k key groups by a radix
// select on the scores' order-preserving bit patterns (greater score first,
// lower id on ties) and writes their ids in ascending order.
// ---------------------------------------------------------------------------
constexpr int kSgT = 64, kSgK = 16;

__global__ void __launch_bounds__(256) score_gemm_kernel(const double* __restrict__ A,
                                                         const double* __restrict__ B, int M,
                                                         int Nn, int d, double scale,
                                                         double* __restrict__ S) {
  __shared__ double As[kSgK][kSgT + 1], Bs[kSgK][kSgT + 1];
  const int h = blockIdx.z, i0 = blockIdx.y * kSgT, j0 = blockIdx.x * kSgT;
  const double* Ah = A + static_cast<size_t>(h) * M * d;
  const double* Bh = B + static_cast<size_t>(h) * Nn * d;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.0;
  for (int k0 = 0; k0 < d; k0 += kSgK) {
    for (int t = threadIdx.x; t < kSgT * kSgK; t += blockDim.x) {
      const int row = t / kSgK, kk = t % kSgK;
      const int k = k0 + kk;
      As[kk][row] = (i0 + row < M && k < d) ? Ah[static_cast<size_t>(i0 + row) * d + k] : 0.0;
      Bs[kk][row] = (j0 + row < Nn && k < d) ? Bh[static_cast<size_t>(j0 + row) * d + k] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSgK; ++kk) {
      double a[4], b[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = As[kk][ty * 4 + r];
#pragma unroll
      for (int c = 0; c < 4; ++c) b[c] = Bs[kk][tx * 4 + c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fma(a[r], b[c], acc[r][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty * 4 + r;
    if (i >= M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + tx * 4 + c;
      if (j < Nn) S[(static_cast<size_t>(h) * M + i) * Nn + j] = scale * acc[r][c];
    }
  }
}

// order-preserving bit pattern of a finite double (-0 taken as +0)
__device__ __forceinline__ uint64_t score_key(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x + 0.0));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

constexpr int kTopkWarps = 8;

__global__ void __launch_bounds__(kTopkWarps * 32) topk_route_kernel(
    const double* __restrict__ S, int H, int Cq, int Ck, const int32_t* __restrict__ kh, int h0,
    int kmax, int32_t* __restrict__ csr) {
  __shared__ int hist[kTopkWarps][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gi = blockIdx.x * kTopkWarps + w;  // (head within the chunk, query group)
  if (gi >= H * Cq) return;
  const int hl = gi / Cq;  // (the query group is gi % Cq)
  const double* row = S + static_cast<size_t>(gi) * Ck;
  const int k = kh[h0 + hl];
  int* hs = hist[w];
  // radix select of the k-th largest key, eight bits at a time
  uint64_t prefix = 0;
  int want = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hs[b] = 0;
    __syncwarp();
    for (int c = lane; c < Ck; c += 32) {
      const uint64_t u = score_key(row[c]);
      const bool match = (shift == 56) || ((u >> (shift + 8)) == (prefix >> (shift + 8)));
      if (match) atomicAdd(&hs[(u >> shift) & 255], 1);
    }
    __syncwarp();
    // lane l owns bins 255 - 8l - 7 .. 255 - 8l (from the top); suffix counts
    int cnt[8], tot = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      cnt[q] = hs[255 - 8 * lane - q];
      tot += cnt[q];
    }
    int incl = tot;  // inclusive prefix over lanes = count of bins above this lane's last bin
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int before = incl - tot;  // keys in higher bins than this lane's
    // the lane whose range holds the want-th key finds the bin
    int bin = -1, above = 0;
    if (before < want && want <= incl) {
      int run = before;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (bin < 0 && run + cnt[q] >= want) {
          bin = 255 - 8 * lane - q;
          above = run;
        }
        run += cnt[q];
      }
    }
    const unsigned who = __ballot_sync(0xffffffffu, bin >= 0);
    const int src = __ffs(who) - 1;
    bin = __shfl_sync(0xffffffffu, bin, src);
    above = __shfl_sync(0xffffffffu, above, src);
    want -= above;
    prefix |= static_cast<uint64_t>(bin) << shift;
    __syncwarp();
  }
  // prefix = key of the k-th largest score; take every larger key and the
  // `want` lowest ids among the equal ones, in ascending id order
  int32_t* out = csr + static_cast<size_t>(gi) * kmax;
  int n_out = 0, n_eq = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int c0 = 0; c0 < Ck; c0 += 32) {
    const int c = c0 + lane;
    uint64_t u = 0;
    if (c < Ck) u = score_key(row[c]);
    const bool gt = c < Ck && u > prefix, eq = c < Ck && u == prefix;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && n_eq + __popc(beq & lt) < want);
    const unsigned bk = __ballot_sync(0xffffffffu, take);
    if (take) out[n_out + __popc(bk & lt)] = c;
    n_out += __popc(bk);
    n_eq += __popc(beq);
  }
  for (int i = k + lane; i < kmax; i += 32) out[i] = -1;
}

struct KhParam {
  int32_t v[SPARSEPR_MAX_HEADS];
};

__global__ void write_k_kernel(KhParam kp, int H, int32_t* out) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) out[h] = kp.v[h];
}

}  // namespace

cudaError_t launch_gather_rows(const void* src, void* dst, const void* src2, void* dst2,
                               const int32_t* perm, int H, int N, int d, int elem_bytes,
                               cudaStream_t st) {
  const int vpr = d * elem_bytes / 16;
  if (vpr < 1 || vpr > kGatherThreads || vpr * 16 != d * elem_bytes || (src2 == nullptr) != (dst2 == nullptr))
    return cudaErrorInvalidValue;
  if (H < 1 || N < 1) return cudaSuccess;
  const int rows_per_block = (kGatherThreads / vpr) * kGatherDepth;
  const dim3 grid(static_cast<unsigned>((N + rows_per_block - 1) / rows_per_block),
                  static_cast<unsigned>(H));
  gather_rows_kernel<<<grid, kGatherThreads, 0, st>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), static_cast<const uint4*>(src2),
      static_cast<uint4*>(dst2), perm, N, vpr);
  return cudaGetLastError();
}

size_t route_scores_bytes(int H, int Cq, int Ck) {
  const size_t per_head = static_cast<size_t>(Cq) * Ck * 8;
  size_t heads = (static_cast<size_t>(64) << 20) / per_head;
  if (heads < 1) heads = 1;
  if (heads > static_cast<size_t>(H)) heads = H;
  return heads * per_head;
}

cudaError_t launch_route_gemm(const double* cq, const double* ckr, int H, int Cq, int Ck, int d,
                              double scale, const int32_t* kh, int kmax, double* scores,
                              size_t scores_bytes, int32_t* csr, cudaStream_t st) {
  const size_t per_head = static_cast<size_t>(Cq) * Ck * 8;
  const int hc = static_cast<int>(scores_bytes / per_head);
  if (hc < 1) return cudaErrorInvalidValue;
  for (int h0 = 0; h0 < H; h0 += hc) {
    const int nh = min(hc, H - h0);
    dim3 g1((Ck + kSgT - 1) / kSgT, (Cq + kSgT - 1) / kSgT, nh);
    score_gemm_kernel<<<g1, 256, 0, st>>>(cq + static_cast<size_t>(h0) * Cq * d,
                                          ckr + static_cast<size_t>(h0) * Ck * d, Cq, Ck, d, scale,
                                          scores);
    const int rows = nh * Cq;
    topk_route_kernel<<<(rows + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, 0, st>>>(
        scores, nh, Cq, Ck, kh, h0, kmax, csr + static_cast<size_t>(h0) * Cq * kmax);
  }
  return cudaGetLastError();
}

cudaError_t launch_range_mean(const void* X, int x_kind, int H, int N, int d, const int32_t* off,
                              int C, int off_stride, double* out, cudaStream_t st) {
  return launch_group_mean(X, x_kind, static_cast<long long>(N) * d, d, d, nullptr, 0, off,
                           off_stride, C, H, false, out, nullptr, nullptr, 0, st);
}

cudaError_t launch_write_k(const int32_t* kh_host_vals, int H, int32_t* k_per_head,
                           cudaStream_t st) {
  KhParam kp;
  for (int h = 0; h < SPARSEPR_MAX_HEADS; ++h) kp.v[h] = (h < H) ? kh_host_vals[h] : 0;
  write_k_kernel<<<(H + 127) / 128, 128, 0, st>>>(kp, H, k_per_head);
  return cudaGetLastError();
}

}  // namespace spr
