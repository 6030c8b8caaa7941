// Stable counting sort of per-head group labels: the group-major order of
// "Partition the Support, Reconstruct the Residual" (2.C, contiguous
// group-major layouts), also used to form the k-means group sums in a fixed
// (ascending token) order.
//
// Per head: per-chunk histograms, an exclusive scan in (group, chunk) order
// (down the chunks of every group, then over the group totals), and a stable
// scatter in which the warps of a chunk claim positions one after another.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kSortThreads = 256;

__global__ void sort_hist_kernel(const int32_t* __restrict__ labels, int n, int C, int nchunk,
                                 int32_t* __restrict__ hist, const int32_t* skip,
                                 int skip_stride, DeviceStats* stats) {
  extern __shared__ int32_t sh[];
  const int h = blockIdx.y, chunk = blockIdx.x;
  if (skip && skip[h * skip_stride]) return;
  for (int c = threadIdx.x; c < C; c += blockDim.x) sh[c] = 0;
  __syncthreads();
  const int32_t* lab = labels + static_cast<size_t>(h) * n;
  const int lo = chunk * kSortChunk, hi = min(n, lo + kSortChunk);
  for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    const int32_t g = lab[i];
    if (g >= 0 && g < C)
      atomicAdd(&sh[g], 1);
    else if (stats)
      raise_status(stats, SPARSEPR_ERR_INVALID_ARG);  // label out of range: token dropped
  }
  __syncthreads();
  int32_t* out = hist + (static_cast<size_t>(h) * nchunk + chunk) * C;
  for (int c = threadIdx.x; c < C; c += blockDim.x) out[c] = sh[c];
}

// hist[h][chunk][c] becomes the position of chunk's first element of group c
// relative to the start of group c, and off[h][c] the size of group c: one
// thread per (group, head) walks the chunks with 16 loads in flight.
constexpr int kColThreads = 128;

__global__ void __launch_bounds__(kColThreads)
    sort_colscan_kernel(int C, int nchunk, int32_t* __restrict__ hist, int32_t* __restrict__ off,
                        const int32_t* skip, int skip_stride) {
  const int h = blockIdx.y, c = blockIdx.x * kColThreads + threadIdx.x;
  if (skip && skip[h * skip_stride]) return;
  if (c >= C) return;
  int32_t* col = hist + static_cast<size_t>(h) * nchunk * C + c;
  int32_t run = 0;
  int k = 0;
  for (; k + 16 <= nchunk; k += 16) {
    int32_t v[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = col[static_cast<size_t>(k + q) * C];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      col[static_cast<size_t>(k + q) * C] = run;
      run += v[q];
    }
  }
  for (; k < nchunk; ++k) {
    const int32_t v = col[static_cast<size_t>(k) * C];
    col[static_cast<size_t>(k) * C] = run;
    run += v;
  }
  off[static_cast<size_t>(h) * (C + 1) + c] = run;  // total for now
}

// One CTA per head: the group sizes in off[h] become the groups' first
// positions (exclusive scan), off[h][C] = n.
__global__ void __launch_bounds__(1024) sort_scan_kernel(int n, int C, int32_t* __restrict__ off,
                                                         const int32_t* skip, int skip_stride) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  const int h = blockIdx.x;
  if (skip && skip[h * skip_stride]) return;
  int32_t* oo = off + static_cast<size_t>(h) * (C + 1);
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int base = 0; base < C; base += blockDim.x) {
    const int c = base + threadIdx.x;
    int32_t v = (c < C) ? oo[c] : 0;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int32_t t = (lane < nw) ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      if (lane < nw) warp_tot[lane] = t;  // inclusive warp prefix
    }
    __syncthreads();
    const int32_t before = carry + (wid > 0 ? warp_tot[wid - 1] : 0) + (x - v);
    __syncthreads();
    if (c < C) oo[c] = before;
    if (threadIdx.x == blockDim.x - 1) carry = before + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) oo[C] = n;
}

__global__ void sort_scatter_kernel(const int32_t* __restrict__ labels, int n, int C, int nchunk,
                                    const int32_t* __restrict__ hist,
                                    const int32_t* __restrict__ off, int32_t* __restrict__ perm,
                                    const int32_t* skip, int skip_stride) {
  extern __shared__ int32_t cnt[];
  const int h = blockIdx.y, chunk = blockIdx.x;
  if (skip && skip[h * skip_stride]) return;
  const int32_t* start = hist + (static_cast<size_t>(h) * nchunk + chunk) * C;
  const int32_t* oo = off + static_cast<size_t>(h) * (C + 1);
  for (int c = threadIdx.x; c < C; c += blockDim.x) cnt[c] = oo[c] + start[c];
  __syncthreads();
  const int32_t* lab = labels + static_cast<size_t>(h) * n;
  int32_t* pp = perm + static_cast<size_t>(h) * n;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int lo = chunk * kSortChunk, hi = min(n, lo + kSortChunk);
  for (int r0 = lo; r0 < hi; r0 += blockDim.x) {
    const int i = r0 + threadIdx.x;
    int32_t g = (i < hi) ? lab[i] : -1;
    if (g >= C) g = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, g);
    const int leader = __ffs(peers) - 1;
    int32_t base = 0;
    for (int w = 0; w < nw; ++w) {
      if (wid == w && g >= 0 && lane == leader) {
        base = cnt[g];
        cnt[g] = base + __popc(peers);
      }
      __syncthreads();
    }
    base = __shfl_sync(0xffffffffu, base, leader);
    if (g >= 0) pp[base + __popc(peers & lt)] = i;
  }
}

}  // namespace

cudaError_t launch_counting_sort(const int32_t* labels, int H, int n, int C, int nchunk,
                                 int32_t* hist, int32_t* perm, int32_t* off,
                                 const int32_t* skip, int skip_stride, DeviceStats* stats,
                                 cudaStream_t st) {
  const size_t shb = static_cast<size_t>(C) * 4;
  dim3 g2(nchunk, H);
  sort_hist_kernel<<<g2, kSortThreads, shb, st>>>(labels, n, C, nchunk, hist, skip, skip_stride,
                                                  stats);
  sort_colscan_kernel<<<dim3((C + kColThreads - 1) / kColThreads, H), kColThreads, 0, st>>>(
      C, nchunk, hist, off, skip, skip_stride);
  sort_scan_kernel<<<H, 1024, 0, st>>>(n, C, off, skip, skip_stride);
  sort_scatter_kernel<<<g2, kSortThreads, shb, st>>>(labels, n, C, nchunk, hist, off, perm, skip,
                                                       skip_stride);
  return cudaGetLastError();
}

}  // namespace spr
