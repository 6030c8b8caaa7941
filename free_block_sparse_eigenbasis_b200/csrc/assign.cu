// Nearest-centroid assignment of the k-means passes of "Partition the Support,
// Reconstruct the Residual" (2.A) on the 5th-generation tensor cores, with a
// certified error bound so that the labels equal those of exact fp64
// arithmetic.
//
// For rows x_i and centroid-side vectors y_j with offsets c_j, the label is
// argmin_j d_ij, d_ij = c_j - 2 x_i . y_j (lowest j on ties):
//   keys:    x = z (response coordinates), y = mu, c = |mu|^2
//   queries: x = q, y = G qbar, c = qbar^T G qbar   (d-space profile form)
// x and y are split into bf16 planes (x = x1 + x2 + x3 + r, |r| <= 2^-24 |x|);
// the plane products x_a . y_b with a + b <= 4 (planes counted from 0) are
// summed by tcgen05.mma in fp32. With K_t accumulated terms per dot product
// the computed d'_ij satisfies
//   |d'_ij - d_ij| <= E_i = (K_t 2^-22 + 2^-20) |x_i| Y + 2^-22 (C + 2 |x_i| Y),
// Y = max_j |y_j|, C = max_j |c_j| (a generous bound: products of bf16 values
// are exact in fp32, each accumulation step loses at most 2^-23 relative).
// The epilogue reduces values whose three low mantissa bits are replaced by
// the column's position within its piece (at most 7 ulp, < 2^-20 |d'|), so
// the bound it uses adds 2^-20 (C + 2 |x_i| Y). A row whose best and
// second-best packed d' differ by more than 2 E_i has a certain label; every
// other row is appended to a list and decided again in fp64 by
// recheck_kernel.
//
// Persistent CTAs (at most one per SM) each take a contiguous range of the
// row tiles of all heads, ordered head-major; the centroid planes of the
// current head stay in shared memory and are reloaded when the range crosses
// into the next head. One warp issues the TMA loads and another the MMAs
// (each on its own, so neither waits behind the other's barrier polls).
// Row tiles of 128 stream through a TMA ring of 2 to 4 stages (as many as
// shared memory holds beside the centroid planes); the 128 x (<=256)
// accumulator of each centroid chunk alternates between two TMEM buffers, so
// the epilogue of one chunk overlaps the MMAs of the next.
// The epilogue is four groups of four warps: every group sees all 128 rows
// (warp w reads TMEM lanes 32 (w % 4) ..) and a quarter of each chunk's
// columns; each thread keeps four chains (columns k mod 4) of best, second
// best and the piece of the best, takes two columns of a chain per step
// (min / max of the pair, then a three-input min for the second best), and
// the groups' partial results meet in shared memory at the end of a tile.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kAsGroups = 4;                 // epilogue column groups
constexpr int kAsEpi = kAsGroups * kTileM;   // epilogue threads (thread = row within a group)
constexpr int kAsThreads = kAsEpi + 64;      // + a TMA producer warp and an MMA warp
constexpr int kAsChunk = 256;                // centroids per accumulator chunk
constexpr uint32_t kAsTmemCols = 512;
constexpr size_t kAsMinSmem = 120 * 1024;    // keeps one CTA (and one TMEM owner) per SM
constexpr int kAsMaxStages = 4;              // row-tile ring depth (as shared memory allows)
// named barriers of the epilogue threads (0 is __syncthreads)
constexpr int kBarXchFull = 1, kBarXchFree = 2, kBarHead = 3;

struct AsBars {
  uint64_t b_full, b_empty;
  uint64_t a_full[kAsMaxStages], a_empty[kAsMaxStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_idle;
  uint32_t tmem_base;
  int abort;
};

struct AsMaps {
  CUtensorMap a[3];  // row planes, box (inner, 128 rows)
  CUtensorMap b[3];  // centroid planes, box (inner, 16 rows)
};

struct AsParams {
  int n;          // rows per head
  int a_head;     // row offset between heads in the A maps
  int b_head;     // row offset between heads in the B maps (= Cpad)
  int Cpad;       // centroids per head, padded to a multiple of 16
  int nA, nB;     // planes
  int npairs;
  int pairs[6];   // (plane of x) * 4 + (plane of y)
  int sw32;       // 1: 32-byte rows (D = 16), 0: 128-byte swizzle atoms (D = 64 * atoms)
  int atoms;      // 64-column atoms (sw32: 1)
  int Kt;         // accumulated terms per dot product
  float res;      // bound on the plane-split residual and dropped plane products, relative
  int tiles_per_head;
  int H;
  int stages;          // row-tile ring depth, 2 .. kAsMaxStages
  uint32_t pos_clear;  // ~7: clears the three low mantissa bits that carry a column position
  const float* cvals;  // [H, Cpad] fp32 offsets (+inf on padding)
  const float* xnorm;  // [H, n] |x_i| (rounded up)
  const float* hmax;   // [H, 2] Y, C (rounded up)
  int32_t* labels;     // [H, n]
  int32_t* flags;      // [H, 4]; changes counter at flag_base, done flag at flag_base + 1
  int flag_base;
  int32_t* recheck;    // [H, n] rows to decide in fp64
  int32_t* nrecheck;   // [H]
  DeviceStats* stats;
};

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, bool sw32) {
  // K-major canonical layouts: LBO = 16 bytes (unused), SBO = stride of 8-row groups
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>((sw32 ? 256u : 1024u) >> 4) << 32;
  d |= 1ull << 46;
  d |= (sw32 ? 6ull : 2ull) << 61;
  return d;
}

// Walks the head segments of a CTA's tile range [g, g1): calls f(h, t0, t1)
// for every head that has not converged, with its tiles t0..t1-1.
template <typename F>
__device__ __forceinline__ void for_segments(const AsParams& p, int g, int g1, F&& f) {
  while (g < g1) {
    const int h = g / p.tiles_per_head;
    const int ge = min(g1, (h + 1) * p.tiles_per_head);
    if (!p.flags[h * 4 + p.flag_base + 1]) f(h, g - h * p.tiles_per_head, ge - h * p.tiles_per_head);
    g = ge;
  }
}

// value with its position (0..7) within a chain piece in the low three
// mantissa bits: changes the value by at most 7 ulp, and the minimum of
// packed values carries the position of its column
// (clear = ~7 comes in as a runtime value so that the compiler emits one
// three-input logic op with the position as its immediate)
__device__ __forceinline__ float pack_pos(float v, int pos, uint32_t clear) {
  return __uint_as_float((__float_as_uint(v) & clear) | static_cast<uint32_t>(pos));
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// orders later reads of the registers after the preceding tcgen05.wait::ld
__device__ __forceinline__ void reg_fence32(uint32_t (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 8)
    asm volatile("" : "+r"(v[i]), "+r"(v[i + 1]), "+r"(v[i + 2]), "+r"(v[i + 3]), "+r"(v[i + 4]),
                 "+r"(v[i + 5]), "+r"(v[i + 6]), "+r"(v[i + 7]));
}

__global__ void __launch_bounds__(kAsThreads, 1)
    argmin_tc_kernel(const __grid_constant__ AsMaps maps, const AsParams p) {
  const int row_bytes = p.sw32 ? 32 : 128;
  const int slab_a = kTileM * row_bytes;                // one atom of a 128-row tile
  const int a_stage = p.nA * p.atoms * slab_a;
  const int slab_b = p.Cpad * row_bytes;                // one atom of all centroids
  const int b_bytes = p.nB * p.atoms * slab_b;
  const int nchunks = (p.Cpad + kAsChunk - 1) / kAsChunk;
  const int T = p.H * p.tiles_per_head;
  const int g0 = static_cast<int>(static_cast<long long>(blockIdx.x) * T / gridDim.x);
  const int g1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * T / gridDim.x);

  extern __shared__ uint8_t as_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(as_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* Bs = sm;
  uint8_t* As = sm + ((b_bytes + 1023) & ~1023);
  float* cs = reinterpret_cast<float*>(As + p.stages * a_stage);
  float* xd1 = cs + p.Cpad;                 // [kAsGroups - 1][128]
  float* xd2 = xd1 + (kAsGroups - 1) * kTileM;
  int* xi1 = reinterpret_cast<int*>(xd2 + (kAsGroups - 1) * kTileM);
  AsBars* bars = reinterpret_cast<AsBars*>(xi1 + (kAsGroups - 1) * kTileM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->b_full, 1);
    mbar_init(&bars->b_empty, 1);
    for (int s = 0; s < kAsMaxStages; ++s) {
      mbar_init(&bars->a_full[s], 1);
      mbar_init(&bars->a_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->acc_full[s], 1);
      mbar_init(&bars->acc_empty[s], kAsEpi);
    }
    mbar_init(&bars->mma_idle, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kAsTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const int inner = p.sw32 ? 16 : 64;
  volatile int never = 0;

  if (warp == kAsEpi / 32) {
    if (lane == 0) {
      // ----------------------------- TMA producer -----------------------------
      int u = 0, seg = 0;
      bool ok = true;
      for_segments(p, g0, g1, [&](int h, int t0, int t1) {
        if (!ok) return;
        if (seg > 0 && !mbar_wait(&bars->b_empty, (seg - 1) & 1, abort)) { ok = false; return; }
        mbar_arrive_expect_tx(&bars->b_full, b_bytes);
        for (int pl = 0; pl < p.nB; ++pl)
          for (int a = 0; a < p.atoms; ++a)
            for (int r = 0; r < p.Cpad; r += 16)
              tma_load_2d(Bs + (pl * p.atoms + a) * slab_b + r * row_bytes, &maps.b[pl],
                          &bars->b_full, a * inner, h * p.b_head + r);
        ++seg;
        for (int t = t0; t < t1; ++t) {
          const int s = u % p.stages;
          if (u >= p.stages && !mbar_wait(&bars->a_empty[s], ((u - p.stages) / p.stages) & 1, abort)) {
            ok = false;
            return;
          }
          mbar_arrive_expect_tx(&bars->a_full[s], a_stage);
          for (int pl = 0; pl < p.nA; ++pl)
            for (int a = 0; a < p.atoms; ++a)
              tma_load_2d(As + s * a_stage + (pl * p.atoms + a) * slab_a, &maps.a[pl],
                          &bars->a_full[s], a * inner, h * p.a_head + t * kTileM);
          ++u;
        }
      });
      // let every load this thread issued land before the CTA exits
      for (int x = max(0, u - p.stages); x < u; ++x)
        mbar_wait(&bars->a_full[x % p.stages], (x / p.stages) & 1, &never);
      if (seg > 0) mbar_wait(&bars->b_full, (seg - 1) & 1, &never);
    }
  } else if (warp == kAsEpi / 32 + 1) {
    if (lane == 0) {
      // ------------------------------ MMA issuer ------------------------------
      // Descriptors are the base descriptors of the A ring and the B planes
      // plus 16-byte offsets (the start-address field; shared memory < 256 KB),
      // precomputed per plane pair and per K step.
      const uint64_t da0 = smem_desc(smem_u32(As), p.sw32), db0 = smem_desc(smem_u32(Bs), p.sw32);
      const int ksteps = p.sw32 ? 1 : p.atoms * 4;  // 16-column K steps
      uint32_t pa_off[6], pb_off[6], ka_off[8], kb_off[8];
#pragma unroll
      for (int pi = 0; pi < 6; ++pi) {
        pa_off[pi] = static_cast<uint32_t>(((p.pairs[pi] >> 2) * p.atoms * slab_a) >> 4);
        pb_off[pi] = static_cast<uint32_t>(((p.pairs[pi] & 3) * p.atoms * slab_b) >> 4);
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int atom = p.sw32 ? 0 : (ks >> 2), koff = p.sw32 ? 0 : (ks & 3) * 32;
        ka_off[ks] = static_cast<uint32_t>((atom * slab_a + koff) >> 4);
        kb_off[ks] = static_cast<uint32_t>((atom * slab_b + koff) >> 4);
      }
      int u = 0, gc = 0, seg = 0;
      bool ok = true;
      for_segments(p, g0, g1, [&](int h, int t0, int t1) {
        if (!ok) return;
        if (!mbar_wait(&bars->b_full, seg & 1, abort)) { ok = false; return; }
        ++seg;
        for (int t = t0; t < t1; ++t, ++u) {
          const int s = u % p.stages;
          if (!mbar_wait(&bars->a_full[s], (u / p.stages) & 1, abort)) { ok = false; return; }
          tc_fence_after();
          const uint64_t abase = da0 + static_cast<uint64_t>((s * a_stage) >> 4);
          for (int c = 0; c < nchunks; ++c, ++gc) {
            const int buf = gc & 1;
            if (gc >= 2 && !mbar_wait(&bars->acc_empty[buf], ((gc - 2) >> 1) & 1, abort)) {
              ok = false;
              return;
            }
            tc_fence_after();
            const int N = min(kAsChunk, p.Cpad - c * kAsChunk);
            const uint32_t idesc = idesc_bf16(kTileM, N, 0);
            const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * kAsChunk);
            const uint64_t bbase = db0 + static_cast<uint64_t>((c * kAsChunk * row_bytes) >> 4);
#pragma unroll
            for (int pi = 0; pi < 6; ++pi) {
              if (pi < p.npairs) {
                const uint64_t ap = abase + pa_off[pi], bp = bbase + pb_off[pi];
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                  if (ks < ksteps)
                    mma_bf16_ss(d_tmem, ap + ka_off[ks], bp + kb_off[ks], idesc,
                                (pi > 0 || ks > 0) ? 1u : 0u);
              }
            }
            mma_commit(&bars->acc_full[buf]);
          }
          mma_commit(&bars->a_empty[s]);
        }
        mma_commit(&bars->b_empty);  // the head's centroid planes may be replaced
      });
      // all MMAs issued by this thread complete before tensor memory is freed
      mma_commit(&bars->mma_idle);
      mbar_wait(&bars->mma_idle, 0, &never);
    }
  } else {
    // ------------------- epilogue: group q, row r of the tile -------------------
    // Every epilogue thread passes the same sequence of named barriers, also
    // after a failed wait (it then skips the work), so none is left behind.
    // Group q reads its columns of a chunk in pieces of at most 32.
    const int q = warp / 4;
    const int r = (warp & 3) * 32 + lane;
    const int et = threadIdx.x;  // 0 .. kAsEpi - 1
    const uint32_t lane_base = static_cast<uint32_t>(((warp & 3) * 32) << 16);
    // E bound: MMA terms, fp32 offsets and rounding, and the index bits
    // packed into the low three mantissa bits of each value (<= 7 ulp)
    const float kt_term = static_cast<float>(p.Kt) * 2.384185791015625e-07f + p.res;
    const uint32_t clear = p.pos_clear;
    int gc = 0, nx = 0;
    bool ok = true;
    uint32_t va[32];
    for_segments(p, g0, g1, [&](int h, int t0, int t1) {
      named_barrier_sync(kBarHead, kAsEpi);  // the previous head's offsets are no longer read
      for (int j = et; j < p.Cpad; j += kAsEpi) cs[j] = p.cvals[static_cast<size_t>(h) * p.Cpad + j];
      named_barrier_sync(kBarHead, kAsEpi);
      const float Y = p.hmax[h * 2 + 0], C = p.hmax[h * 2 + 1];
      int32_t* fl = p.flags + h * 4;
      float b1[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
      float b2[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
      int blk[4] = {0, 0, 0, 0};
      // reduce one piece of w (16 or 32) columns starting at column jb:
      // values packed with their position within the chain, then a pair at
      // a time into the chain's best and second best
      auto reduce = [&](const uint32_t (&v)[32], int w, int jb) {
        const float4* c4 = reinterpret_cast<const float4*>(cs + jb);
        const float ob[4] = {b1[0], b1[1], b1[2], b1[3]};
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
          if (pr < 2 || w >= 32) {
            const float4 ca = c4[2 * pr], cb = c4[2 * pr + 1];
            const float ea[4] = {ca.x, ca.y, ca.z, ca.w}, eb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float x = pack_pos(fmaf(-2.f, __uint_as_float(v[8 * pr + k]), ea[k]), 2 * pr, clear);
              const float y = pack_pos(fmaf(-2.f, __uint_as_float(v[8 * pr + 4 + k]), eb[k]), 2 * pr + 1, clear);
              const float m = fminf(x, y), M = fmaxf(x, y);
              b2[k] = min3f(b2[k], fmaxf(b1[k], m), M);
              b1[k] = fminf(b1[k], m);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) blk[k] = (b1[k] < ob[k]) ? jb : blk[k];
      };
      const int U = (t1 - t0) * nchunks;  // (tile, chunk) steps of this head
      float xn_pf = 0.f;  // |x| and the current label of group 0's row, loaded at
      int lab_pf = -1;    // the start of the tile so the latency overlaps its chunks
      for (int u = 0; u < U; ++u) {
        const int c = u % nchunks;
        const int t = t0 + u / nchunks;
        if (c == 0) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            b1[k] = INFINITY;
            b2[k] = INFINITY;
            blk[k] = 0;
          }
          const int row = t * kTileM + r;
          if (q == 0 && row < p.n) {
            const size_t li = static_cast<size_t>(h) * p.n + row;
            xn_pf = p.xnorm[li];
            lab_pf = p.labels[li];
          }
        }
        ok = ok && mbar_wait(&bars->acc_full[gc & 1], (gc >> 1) & 1, abort);
        ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
        tc_fence_after();
        // this group's columns [a0, a1) of chunk c
        const int N = min(kAsChunk, p.Cpad - c * kAsChunk);
        const int nb = N >> 4;
        const int a0 = 16 * ((q * nb) / kAsGroups), a1 = 16 * (((q + 1) * nb) / kAsGroups);
        const uint32_t base = tmem + lane_base + static_cast<uint32_t>((gc & 1) * kAsChunk);
        for (int col = a0; col < a1; col += 32) {
          const int w = min(32, a1 - col);  // warp-uniform
          if (ok) {
            if (w >= 32)
              tmem_ld32(base + col, va);
            else
              tmem_ld16(base + col, *reinterpret_cast<uint32_t(*)[16]>(va));
          }
          tmem_wait_ld();
          reg_fence32(va);
          if (ok) reduce(va, w, c * kAsChunk + col);
        }
        tc_fence_before();
        mbar_arrive(&bars->acc_empty[gc & 1]);
        ++gc;
        if (c + 1 < nchunks) continue;
        // ---- end of tile t: merge the chains, then the groups ----
        // a chain's best sits at column blk + 4 * (packed position) + k
        float d1 = b1[0], d2 = b2[0];
        int i1 = blk[0] + 4 * static_cast<int>(__float_as_uint(b1[0]) & 7u);
#pragma unroll
        for (int k = 1; k < 4; ++k) {
          const int ik = blk[k] + 4 * static_cast<int>(__float_as_uint(b1[k]) & 7u) + k;
          if (b1[k] < d1 || (b1[k] == d1 && ik < i1)) {
            d2 = fminf(d1, b2[k]);
            d1 = b1[k];
            i1 = ik;
          } else {
            d2 = fminf(d2, b1[k]);
          }
        }
        if (q > 0) {
          if (nx > 0) named_barrier_sync(kBarXchFree, kAsEpi);  // group 0 has read the last tile
          xd1[(q - 1) * kTileM + r] = d1;
          xd2[(q - 1) * kTileM + r] = d2;
          xi1[(q - 1) * kTileM + r] = i1;
          named_barrier_arrive(kBarXchFull, kAsEpi);
        } else {
          named_barrier_sync(kBarXchFull, kAsEpi);
#pragma unroll
          for (int g = 0; g < kAsGroups - 1; ++g) {
            const float od1 = xd1[g * kTileM + r], od2 = xd2[g * kTileM + r];
            const int oi1 = xi1[g * kTileM + r];
            if (od1 < d1 || (od1 == d1 && oi1 < i1)) {
              d2 = fminf(d1, od2);
              d1 = od1;
              i1 = oi1;
            } else {
              d2 = fminf(d2, od1);
            }
          }
          named_barrier_arrive(kBarXchFree, kAsEpi);
          const int row = t * kTileM + r;
          bool changed = false, flag = false;
          if (ok && row < p.n) {
            const size_t li = static_cast<size_t>(h) * p.n + row;
            const float xy = xn_pf * Y;
            const float E = kt_term * xy + 1.25e-06f * (C + 2.f * xy);
            if (d2 - d1 > 2.f * E) {
              changed = lab_pf != i1;
              if (changed) p.labels[li] = i1;
            } else {
              flag = true;
            }
          }
          // rows to decide in fp64: one list append per warp
          const unsigned fb = __ballot_sync(0xffffffffu, flag);
          if (fb) {
            int base = 0;
            if (lane == 0) {
              base = atomicAdd(&p.nrecheck[h], __popc(fb));
              atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats->recheck_rows[p.flag_base >> 1]),
                        static_cast<unsigned long long>(__popc(fb)));
            }
            base = __shfl_sync(0xffffffffu, base, 0);
            if (flag) p.recheck[static_cast<size_t>(h) * p.n + base + __popc(fb & ((1u << lane) - 1u))] = row;
          }
          // one atomic per warp for the label-change counter
          const unsigned cb = __ballot_sync(0xffffffffu, changed);
          if (lane == 0 && cb) atomicAdd(&fl[p.flag_base], __popc(cb));
        }
        ++nx;
      }
    });
    if (q > 0 && nx > 0) named_barrier_sync(kBarXchFree, kAsEpi);  // balance the last arrival
  }
  __syncthreads();
  if (*abort && threadIdx.x == 0) raise_status(p.stats, SPARSEPR_ERR_TIMEOUT);
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kAsTmemCols);
  }
}

// ---------------------------------------------------------------------------
// fp64 decision of the flagged rows, R rows per block at a time (grid stride
// over the head's list): thread j scores centroids j, j + 256, ... in
// ascending order from the transposed centroid side yT [D, m], each load of
// yT (contiguous across the warp) serving the R rows of the batch, so the
// centroid table streams from L2 once per batch instead of once per row
// (R = 8 for rows of 64 or more columns; R = 1 for the short key rows, whose
// few flagged rows are best spread over all blocks). Then per row the nearest
// and second-nearest value (lowest index on ties) over the block.
// direct = 1: d = sum_t (x_t - y_jt)^2; else d = c_j - 2 x . y_j.
// ---------------------------------------------------------------------------
constexpr int kRcThreads = 256, kRcMaxD = 128, kRcRows = 8;
constexpr int kRcWarps = kRcThreads / 32;

__device__ __forceinline__ double ldx(const void* X, int kind, size_t i) {
  if (kind == kXf64) return static_cast<const double*>(X)[i];
  if (kind == kXbf16) return static_cast<double>(__bfloat162float(static_cast<const __nv_bfloat16*>(X)[i]));
  return static_cast<double>(static_cast<const float*>(X)[i]);
}

template <int DT, bool DIRECT, int R>
__global__ void __launch_bounds__(kRcThreads)
    recheck_kernel(const void* X, int kind, long long hsx, int ldx_, int n, int Drt,
                   const double* yT, const double* c, int m, int32_t* labels, int32_t* flags,
                   int flag_base, const int32_t* recheck, const int32_t* nrecheck,
                   const double* G, DeviceStats* stats) {
  __shared__ __align__(16) double xs[R][kRcMaxD];
  __shared__ double wb1[R][kRcWarps], wb2[R][kRcWarps];
  __shared__ int wbi[R][kRcWarps];
  __shared__ int rows_s[R], cand_s[R];
  __shared__ double gap_s[R], sec_s[R], xpart[kRcWarps];
  __shared__ double gtr;
  const int D = DT > 0 ? DT : Drt;
  const int h = blockIdx.y;
  int32_t* fl = flags + h * 4;
  if (fl[flag_base + 1]) return;
  const int cnt = nrecheck[h];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double* Yh = yT + static_cast<size_t>(h) * D * m;
  const double* ch = DIRECT ? nullptr : c + static_cast<size_t>(h) * m;
  const double* Gh = (!DIRECT && G) ? G + static_cast<size_t>(h) * D * D : nullptr;
  if (threadIdx.x == 0) {  // trace of G, for the near-tie test (blocks with rows)
    double t = 0.0;
    if (Gh && static_cast<long long>(blockIdx.x) * R < cnt) {
#pragma unroll 1
      for (int a0 = 0; a0 < D; a0 += 8) {  // eight loads in flight, summed in order
        double g[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) g[q] = (a0 + q < D) ? Gh[static_cast<size_t>(a0 + q) * (D + 1)] : 0.0;
#pragma unroll
        for (int q = 0; q < 8; ++q) t += g[q];
      }
    }
    gtr = t;
  }
  int ties = 0;
  for (int k0 = blockIdx.x * R; k0 < cnt; k0 += gridDim.x * R) {
    const int nb = min(R, cnt - k0);
    __syncthreads();  // the previous batch's rows and results are consumed
    if (threadIdx.x < R)
      rows_s[threadIdx.x] = threadIdx.x < nb ? recheck[static_cast<size_t>(h) * n + k0 + threadIdx.x] : 0;
    __syncthreads();
    for (int i = threadIdx.x; i < R * D; i += kRcThreads) {
      const int r = i / D, t = i % D;
      xs[r][t] = (r < nb) ? ldx(X, kind, h * hsx + static_cast<size_t>(rows_s[r]) * ldx_ + t) : 0.0;
    }
    __syncthreads();
    Top2 t2[R];
#pragma unroll
    for (int r = 0; r < R; ++r) t2[r] = top2_empty();
    // scores of centroid j for the batch's rows: with the row length fixed at
    // compile time the column loop is unrolled, so loads run ahead of the FMAs
    auto score = [&](int j, double (&acc)[R]) {
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = 0.0;
      auto step = [&](int t, double y) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (DIRECT) {
            const double e = xs[r][t] - y;
            acc[r] = fma(e, e, acc[r]);
          } else {
            acc[r] = fma(xs[r][t], y, acc[r]);
          }
        }
      };
      // columns t and t + 1 (t even) with one 16-byte shared load per row:
      // the same FMAs in the same order as two steps
      auto step2 = [&](int t, double y0, double y1) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const double2 xv = *reinterpret_cast<const double2*>(&xs[r][t]);
          if (DIRECT) {
            const double e0 = xv.x - y0;
            acc[r] = fma(e0, e0, acc[r]);
            const double e1 = xv.y - y1;
            acc[r] = fma(e1, e1, acc[r]);
          } else {
            acc[r] = fma(xv.x, y0, acc[r]);
            acc[r] = fma(xv.y, y1, acc[r]);
          }
        }
      };
      if (DT > 0 && DT <= 16 && DT % 2 == 0) {
        double y[DT > 0 ? DT : 1];
#pragma unroll
        for (int t = 0; t < DT; ++t) y[t] = Yh[static_cast<size_t>(t) * m + j];
#pragma unroll
        for (int t = 0; t < DT; t += 2) step2(t, y[t], y[t + 1]);
      } else if (DT > 0 && DT <= 16) {
#pragma unroll
        for (int t = 0; t < DT; ++t) step(t, Yh[static_cast<size_t>(t) * m + j]);
      } else if (DT > 0) {
        // chunks of 8 columns, the next chunk's loads issued before this
        // chunk's FMAs
        double ya[8], yb[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) ya[q] = Yh[static_cast<size_t>(q) * m + j];
#pragma unroll 1
        for (int t = 0; t < DT; t += 16) {
#pragma unroll
          for (int q = 0; q < 8; ++q) yb[q] = Yh[static_cast<size_t>(t + 8 + q) * m + j];
#pragma unroll
          for (int q = 0; q < 8; q += 2) step2(t + q, ya[q], ya[q + 1]);
          if (t + 16 < DT)
#pragma unroll
            for (int q = 0; q < 8; ++q) ya[q] = Yh[static_cast<size_t>(t + 16 + q) * m + j];
#pragma unroll
          for (int q = 0; q < 8; q += 2) step2(t + 8 + q, yb[q], yb[q + 1]);
        }
      } else {
        int t = 0;
#pragma unroll 1
        for (; t + 8 <= D; t += 8) {
          double y[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) y[q] = Yh[static_cast<size_t>(t + q) * m + j];
#pragma unroll
          for (int q = 0; q < 8; ++q) step(t + q, y[q]);
        }
        for (; t < D; ++t) step(t, Yh[static_cast<size_t>(t) * m + j]);
      }
    };
    constexpr int kJU = (R == 1) ? 2 : 1;  // short rows: two centroids in flight
#pragma unroll kJU
    for (int j = threadIdx.x; j < m; j += kRcThreads) {  // ascending within the thread
      double acc[R];
      score(j, acc);
#pragma unroll
      for (int r = 0; r < R; ++r) top2_push(t2[r], DIRECT ? acc[r] : ch[j] - 2.0 * acc[r], j);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double o1 = __shfl_xor_sync(0xffffffffu, t2[r].b1, o);
        const int oi = __shfl_xor_sync(0xffffffffu, t2[r].i1, o);
        const double o2 = __shfl_xor_sync(0xffffffffu, t2[r].b2, o);
        top2_merge(t2[r], o1, oi, o2);
      }
      if (lane == 0) {
        wb1[r][w] = t2[r].b1;
        wb2[r][w] = t2[r].b2;
        wbi[r][w] = t2[r].i1;
      }
    }
    __syncthreads();
    if (threadIdx.x < nb) {
      const int r = threadIdx.x;
      Top2 b = Top2{wb1[r][0], wb2[r][0], wbi[r][0]};
      for (int q = 1; q < kRcWarps; ++q) top2_merge(b, wb1[r][q], wbi[r][q], wb2[r][q]);
      const size_t li = static_cast<size_t>(h) * n + rows_s[r];
      if (labels[li] != b.i1) atomicAdd(&fl[flag_base], 1);
      labels[li] = b.i1;
      // near tie: DIRECT values are squared distances; otherwise they lack
      // x^T G x, formed below (by the whole block) for candidate rows only
      const double gap = b.b2 - b.b1;
      int cd = 0;
      if (m > 1) {
        if (DIRECT) {
          ties += (gap <= kNearTieRel * b.b2);
        } else if (Gh) {
          double xx = 0.0;
          for (int a = 0; a < D; ++a) xx = fma(xs[r][a], xs[r][a], xx);
          cd = gap <= 1e-11 * (fabs(b.b2) + gtr * xx);
        }
      }
      cand_s[r] = cd;
      gap_s[r] = gap;
      sec_s[r] = b.b2;
    }
    if (!DIRECT) {
      __syncthreads();  // cand_s, gap_s, sec_s are visible
      for (int r = 0; r < nb; ++r) {
        if (!cand_s[r]) continue;  // block-uniform
        double part = 0.0;
        for (int bcol = threadIdx.x; bcol < D; bcol += kRcThreads) {
          double gb = 0.0;
          for (int a = 0; a < D; ++a) gb = fma(xs[r][a], Gh[static_cast<size_t>(a) * D + bcol], gb);
          part = fma(gb, xs[r][bcol], part);
        }
        part = warp_sum_f64(part);
        if (lane == 0) xpart[w] = part;
        __syncthreads();
        if (threadIdx.x == 0) {
          double xgx = 0.0;
          for (int q = 0; q < kRcWarps; ++q) xgx += xpart[q];
          ties += (gap_s[r] <= kNearTieRel * (sec_s[r] + xgx));
        }
        __syncthreads();  // xpart is free again
      }
    }
  }
  if (ties)
    atomicAdd(reinterpret_cast<unsigned long long*>(&stats->near_ties[flag_base >> 1]),
              static_cast<unsigned long long>(ties));
}

template <bool DIRECT>
void launch_recheck_d(const AssignTC& a, cudaStream_t st) {
  // short rows (D <= 16): one row per block at a time over at most 128
  // blocks per head; longer rows: batches of kRcRows over at most 64 blocks
  // per head. In all no more blocks than two per SM (one wave at two
  // resident blocks of 256 threads at up to 128 registers), so that the
  // blocks with rows do not wait behind waves of blocks without.
  const int nb_all = 2 * (a.sm_count > 0 ? a.sm_count : 148) / (a.H > 0 ? a.H : 1);
  const int nb1 = nb_all > 128 ? 128 : (nb_all < 1 ? 1 : nb_all);
  const int nb8 = nb_all > 64 ? 64 : (nb_all < 1 ? 1 : nb_all);
#define SPR_RC(DT, R, NB)                                                                       \
  recheck_kernel<DT, DIRECT, R><<<dim3(NB, a.H), kRcThreads, 0, st>>>(                        \
      a.x_exact, a.x_kind, a.x_hs, a.x_ld, a.n, a.D, a.y_tr, a.c_exact, a.m, a.labels, a.flags, \
      a.flag_base, a.recheck, a.nrecheck, a.metric, a.stats)
  if (a.D == 16)
    SPR_RC(16, 1, nb1);
  else if (a.D == 64)
    SPR_RC(64, kRcRows, nb8);
  else if (a.D == 128)
    SPR_RC(128, kRcRows, nb8);
  else if (a.D < 16)
    SPR_RC(0, 1, nb1);
  else
    SPR_RC(0, kRcRows, nb8);
#undef SPR_RC
}

// ---------------------------------------------------------------------------
// Operand preparation.
// ---------------------------------------------------------------------------
// Split rows of fp64 X (or widen bf16 / fp32 X) into P bf16 planes of Dp
// columns (zero padded); norm[row] = |x| rounded up.
__global__ void split_rows_kernel(const void* X, int kind, long long hsx, int ldx_, int n, int D,
                                  int Dp, int P, __nv_bfloat16* planes, long long plane_stride,
                                  float* norms) {
  const int h = blockIdx.y;
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n) return;
  const size_t xb = h * hsx + static_cast<size_t>(row) * ldx_;
  const size_t ob = (static_cast<size_t>(h) * n + row) * Dp;
  double ss = 0.0;
  for (int t = lane; t < Dp; t += 32) {
    double v = (t < D) ? ldx(X, kind, xb + t) : 0.0;
    ss = fma(v, v, ss);
    for (int pl = 0; pl < P; ++pl) {
      const __nv_bfloat16 b = __double2bfloat16(v);
      planes[pl * plane_stride + ob + t] = b;
      v -= static_cast<double>(__bfloat162float(b));
    }
  }
  ss = warp_sum_f64(ss);
  if (norms && lane == 0)
    norms[static_cast<size_t>(h) * n + row] = static_cast<float>(sqrt(ss) * (1.0 + 1e-6));
}

// The same for rows that split into 16-byte pieces (D = Dp, TPR = D / EPT
// threads per row dividing 32, 16-byte aligned rows): each thread widens one
// piece, writes its plane values, and the row's lanes sum the squares.
template <typename T>
__global__ void __launch_bounds__(256)
    split_rows_vec_kernel(const T* X, long long hsx, int ldx_, int n, int D, int P,
                          __nv_bfloat16* planes, long long plane_stride, float* norms) {
  constexpr int EPT = 16 / sizeof(T);
  const int TPR = D / EPT;
  const int h = blockIdx.y;
  const int row = blockIdx.x * (256 / TPR) + static_cast<int>(threadIdx.x) / TPR;
  const int col = (static_cast<int>(threadIdx.x) % TPR) * EPT;
  double ss = 0.0;
  if (row < n) {
    double v[EPT];
    vload16(X + h * hsx + static_cast<size_t>(row) * ldx_ + col, v);
#pragma unroll
    for (int i = 0; i < EPT; ++i) ss = fma(v[i], v[i], ss);
    const size_t ob = (static_cast<size_t>(h) * n + row) * D + col;
    for (int pl = 0; pl < P; ++pl) {
      __align__(16) __nv_bfloat16 b[EPT];
#pragma unroll
      for (int i = 0; i < EPT; ++i) {
        b[i] = __double2bfloat16(v[i]);
        v[i] -= static_cast<double>(__bfloat162float(b[i]));
      }
      if (EPT == 8)
        *reinterpret_cast<uint4*>(planes + pl * plane_stride + ob) = *reinterpret_cast<const uint4*>(b);
      else if (EPT == 4)
        *reinterpret_cast<uint2*>(planes + pl * plane_stride + ob) = *reinterpret_cast<const uint2*>(b);
      else
        *reinterpret_cast<uint32_t*>(planes + pl * plane_stride + ob) = *reinterpret_cast<const uint32_t*>(b);
    }
  }
  for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (norms && row < n && col == 0)
    norms[static_cast<size_t>(h) * n + row] = static_cast<float>(sqrt(ss) * (1.0 + 1e-6));
}

// Centroid side: planes of y (padded to Cpad rows with zeros), fp32 offsets
// (a large finite value on padding, so that values with index bits packed
// into their low mantissa bits stay ordered numbers), the per-head maxima
// Y = max |y_j|, C = max |c_j| (rounded up; merged across CTAs with an
// integer max on the bits of the non-negative floats, after hmax was zeroed)
// and the transposed fp64 copy yT [D, m] read by the fp64 decisions. One warp
// per centroid row.
constexpr int kPrepWarps = 16;
constexpr float kPadOffset = 1.0e38f;

__global__ void __launch_bounds__(kPrepWarps * 32)
    prep_centroids_kernel(const double* Yv, const double* cv, int m, int D, int Dp, int Cpad,
                          int P, __nv_bfloat16* planes, long long plane_stride, float* cf,
                          float* hmax, double* ytr, const int32_t* flags, int flag_base) {
  __shared__ float ym[kPrepWarps], cm[kPrepWarps];
  const int h = blockIdx.y;
  if (flags && flags[h * 4 + flag_base + 1]) return;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int j = blockIdx.x * kPrepWarps + wid;
  float yv = 0.f, cvv = 0.f;
  if (j < Cpad) {
    const size_t ob = (static_cast<size_t>(h) * Cpad + j) * Dp;
    double ss = 0.0;
    for (int t = lane; t < Dp; t += 32) {
      double v = (j < m && t < D) ? Yv[(static_cast<size_t>(h) * m + j) * D + t] : 0.0;
      if (j < m && t < D) ytr[(static_cast<size_t>(h) * D + t) * m + j] = v;
      ss = fma(v, v, ss);
      for (int pl = 0; pl < P; ++pl) {
        const __nv_bfloat16 b = __double2bfloat16(v);
        planes[pl * plane_stride + ob + t] = b;
        v -= static_cast<double>(__bfloat162float(b));
      }
    }
    ss = warp_sum_f64(ss);
    if (lane == 0) {
      if (j < m) {
        const double cj = cv[static_cast<size_t>(h) * m + j];
        cf[static_cast<size_t>(h) * Cpad + j] = static_cast<float>(cj);
        yv = static_cast<float>(sqrt(ss) * (1.0 + 1e-6));
        cvv = static_cast<float>(fabs(cj) * (1.0 + 1e-6));
      } else {
        cf[static_cast<size_t>(h) * Cpad + j] = kPadOffset;
      }
    }
  }
  if (lane == 0) {
    ym[wid] = yv;
    cm[wid] = cvv;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = ym[0], c = cm[0];
    for (int w = 1; w < kPrepWarps; ++w) {
      a = fmaxf(a, ym[w]);
      c = fmaxf(c, cm[w]);
    }
    atomicMax(reinterpret_cast<int*>(&hmax[h * 2 + 0]), __float_as_int(a));
    atomicMax(reinterpret_cast<int*>(&hmax[h * 2 + 1]), __float_as_int(c));
  }
}

__global__ void zero_counts_kernel(int32_t* p, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = 0;
}

bool plane_map(CUtensorMap* m, const void* base, size_t rows, int Dp, bool sw32, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(Dp), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(Dp) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(sw32 ? 16 : 64),
                       static_cast<cuuint32_t>(rows < static_cast<size_t>(box_rows) ? rows : box_rows)};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             sw32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t assign_tc_smem_bytes(int nA, int nB, int Dp, int Cpad) {
  const bool sw32 = (Dp == 16);
  const int row_bytes = sw32 ? 32 : 128;
  const int atoms = sw32 ? 1 : Dp / 64;
  const size_t b = static_cast<size_t>(nB) * atoms * Cpad * row_bytes;
  const size_t a = static_cast<size_t>(nA) * atoms * kTileM * row_bytes;
  return 1024 + ((b + 1023) & ~static_cast<size_t>(1023)) + 2 * a + static_cast<size_t>(Cpad) * 4 +
         static_cast<size_t>(kAsGroups - 1) * kTileM * 12 + sizeof(AsBars);
}

cudaError_t launch_split_rows(const void* X, int kind, long long hsx, int ldx, int n, int D,
                              int Dp, int P, int H, __nv_bfloat16* planes, long long plane_stride,
                              float* norms, cudaStream_t st) {
  const int es = kind == kXf64 ? 8 : (kind == kXbf16 ? 2 : 4);
  const int ept = 16 / es;
  const int tpr = D / ept;
  const bool vec = D == Dp && D % ept == 0 && tpr >= 1 && tpr <= 32 && (tpr & (tpr - 1)) == 0 &&
                   reinterpret_cast<uintptr_t>(X) % 16 == 0 && (static_cast<long long>(ldx) * es) % 16 == 0 &&
                   (hsx * es) % 16 == 0;
  if (vec) {
    dim3 grid((n + 256 / tpr - 1) / (256 / tpr), H);
    if (kind == kXf64)
      split_rows_vec_kernel<<<grid, 256, 0, st>>>(static_cast<const double*>(X), hsx, ldx, n, D, P,
                                                  planes, plane_stride, norms);
    else if (kind == kXbf16)
      split_rows_vec_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), hsx, ldx, n,
                                                  D, P, planes, plane_stride, norms);
    else
      split_rows_vec_kernel<<<grid, 256, 0, st>>>(static_cast<const float*>(X), hsx, ldx, n, D, P,
                                                  planes, plane_stride, norms);
    return cudaGetLastError();
  }
  dim3 grid((n + 7) / 8, H);
  split_rows_kernel<<<grid, 256, 0, st>>>(X, kind, hsx, ldx, n, D, Dp, P, planes, plane_stride,
                                          norms);
  return cudaGetLastError();
}

cudaError_t launch_prep_centroids(const double* Y, const double* c, int m, int D, int Dp,
                                  int Cpad, int P, int H, __nv_bfloat16* planes,
                                  long long plane_stride, float* cf, float* hmax, double* ytr,
                                  const int32_t* flags, int flag_base, cudaStream_t st) {
  zero_counts_kernel<<<(2 * H + 127) / 128, 128, 0, st>>>(reinterpret_cast<int32_t*>(hmax), 2 * H);
  dim3 grid((Cpad + kPrepWarps - 1) / kPrepWarps, H);
  prep_centroids_kernel<<<grid, kPrepWarps * 32, 0, st>>>(Y, c, m, D, Dp, Cpad, P, planes,
                                                          plane_stride, cf, hmax, ytr, flags,
                                                          flag_base);
  return cudaGetLastError();
}

cudaError_t launch_argmin_tc(const AssignTC& a, cudaStream_t st) {
  const bool sw32 = (a.Dp == 16);
  AsMaps maps;
  for (int pl = 0; pl < 3; ++pl) {
    const int ia = pl < a.nA ? pl : 0, ib = pl < a.nB ? pl : 0;
    if (!plane_map(&maps.a[pl], a.a_planes + ia * a.a_plane_stride, a.a_rows_total, a.Dp, sw32,
                   kTileM) ||
        !plane_map(&maps.b[pl], a.b_planes + ib * a.b_plane_stride,
                   static_cast<size_t>(a.H) * a.Cpad, a.Dp, sw32, 16))
      return cudaErrorInvalidValue;
  }
  AsParams p;
  p.n = a.n;
  p.a_head = a.a_head;
  p.b_head = a.Cpad;
  p.Cpad = a.Cpad;
  p.nA = a.nA;
  p.nB = a.nB;
  p.npairs = a.npairs;
  for (int i = 0; i < 6; ++i) p.pairs[i] = a.pairs[i];
  p.sw32 = sw32 ? 1 : 0;
  p.atoms = sw32 ? 1 : a.Dp / 64;
  p.Kt = a.npairs * a.Dp;
  // 3 planes: residual <= 2^-24 per side, dropped products <= 2^-23 (bound 2^-20);
  // 2 planes of y: residual <= 2^-16 (bound 2^-14)
  p.res = (a.nB >= 3) ? 9.5367431640625e-07f : 6.103515625e-05f;
  p.tiles_per_head = (a.n + kTileM - 1) / kTileM;
  p.pos_clear = ~7u;
  p.H = a.H;
  p.cvals = a.cvals;
  p.xnorm = a.xnorm;
  p.hmax = a.hmax;
  p.labels = a.labels;
  p.flags = a.flags;
  p.flag_base = a.flag_base;
  p.recheck = a.recheck;
  p.nrecheck = a.nrecheck;
  p.stats = a.stats;
  zero_counts_kernel<<<(a.H + 127) / 128, 128, 0, st>>>(a.nrecheck, a.H);
  // as many row-tile stages as shared memory holds (at least the two that
  // assign_tc_smem_bytes counts)
  size_t shb = assign_tc_smem_bytes(a.nA, a.nB, a.Dp, a.Cpad);
  const size_t a_stage = static_cast<size_t>(a.nA) * p.atoms * kTileM * (sw32 ? 32 : 128);
  p.stages = 2;
  while (p.stages < kAsMaxStages && shb + a_stage <= static_cast<size_t>(kMaxDynSmem)) {
    shb += a_stage;
    ++p.stages;
  }
  if (shb < kAsMinSmem) shb = kAsMinSmem;
  cudaError_t e = cudaFuncSetAttribute(argmin_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(shb));
  if (e != cudaSuccess) return e;
  const long long tiles = static_cast<long long>(a.H) * p.tiles_per_head;
  int ctas = a.sm_count;
  if (ctas > tiles) ctas = static_cast<int>(tiles);
  if (ctas < 1) ctas = 1;
  argmin_tc_kernel<<<ctas, kAsThreads, shb, st>>>(maps, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.direct)
    launch_recheck_d<true>(a, st);
  else
    launch_recheck_d<false>(a, st);
  return cudaGetLastError();
}

}  // namespace spr
