// Residual correction of "Partition the Support, Reconstruct the Residual"
// (2.B): every query row that is not a probe gets
//   y = x + x B' + b',   x = its sparse-attention output (fp32),
// and probe rows take their dense output. The map B' = B P_r is d x d per
// head, so x B' is a [rows x d] x [d x d] product per head: it runs on the
// tensor cores (kind::tf32, fp32 accumulation); x itself and b' are added in
// fp32, so only the correction term carries tf32 rounding (relative 2^-11).
//
// Persistent CTAs (at most one per SM) take contiguous ranges of the
// 128-row tiles of all heads; B'^T of the current head stays in shared
// memory. Row tiles stream through a 2-stage TMA ring, accumulators
// alternate between two TMEM buffers, and eight epilogue warps (warp w: TMEM
// lanes 32 (w % 4) .., columns half w / 4) add x and b', pick the dense rows
// of the probes and scatter rows back to the original token order.
#include "common.cuh"
#include "internal.h"

namespace spr {

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

namespace {

constexpr int kCtEpi = 256;               // epilogue threads
constexpr int kCtThreads = kCtEpi + 32;   // + one warp: lane 0 TMA, lane 1 MMA
constexpr uint32_t kCtTmemCols = 256;     // two accumulators of up to 128 columns
constexpr int kCtBarHead = 1;

struct CtBars {
  uint64_t b_full, b_empty;
  uint64_t a_full[2], a_empty[2];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_idle;
  uint32_t tmem_base;
  int abort;
};

struct CtMaps {
  CUtensorMap a;  // o_sparse [H*N, d] fp32, box (32 columns, 128 rows)
  CUtensorMap b;  // B'^T [H*d, d] fp32, box (32 columns, d rows)
};

struct CtParams {
  int H, N, M, tiles_per_head;
  int n_corr;             // rows >= n_corr (text tokens) are copied, not corrected
  const float* od;        // [H, M, d] dense outputs of the probes
  const int32_t* probes;  // [H, M] ascending group-major positions
  const int32_t* perm_q;  // [H, N] group-major position -> token
  const float* bv;        // [H, d] b'
  void* out;              // [H, N, d] bf16 or fp32, token order
  DeviceStats* stats;
};

template <int D>
struct CtSmem {
  static constexpr int kAtoms = D / 32;           // 128-byte swizzle atoms of fp32
  static constexpr int kSlabA = kTileM * 128;     // one atom of a 128-row tile
  static constexpr int kAStage = kAtoms * kSlabA;
  static constexpr int kSlabB = D * 128;
  static constexpr int kBBytes = kAtoms * kSlabB;
  static constexpr int b_off = 0;
  static constexpr int a_off = kBBytes;
  static constexpr int bv_off = a_off + 2 * kAStage;
  static constexpr int bar_off = bv_off + D * 4;
  static constexpr int total = bar_off + static_cast<int>(sizeof(CtBars)) + 1024;
};

template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(kCtThreads, 1)
    correct_tc_kernel(const __grid_constant__ CtMaps maps, const CtParams p) {
  using S = CtSmem<D>;
  const int T = p.H * p.tiles_per_head;
  const int g0 = static_cast<int>(static_cast<long long>(blockIdx.x) * T / gridDim.x);
  const int g1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * T / gridDim.x);
  extern __shared__ uint8_t ct_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ct_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* Bs = sm + S::b_off;
  uint8_t* As = sm + S::a_off;
  float* bvs = reinterpret_cast<float*>(sm + S::bv_off);
  CtBars* bars = reinterpret_cast<CtBars*>(sm + S::bar_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->b_full, 1);
    mbar_init(&bars->b_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->a_full[s], 1);
      mbar_init(&bars->a_empty[s], kCtEpi);
      mbar_init(&bars->acc_full[s], 1);
      mbar_init(&bars->acc_empty[s], kCtEpi);
    }
    mbar_init(&bars->mma_idle, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kCtTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  volatile int never = 0;
  // head segments of this CTA's tile range: f(h, t0, t1)
  auto segments = [&](auto&& f) {
    int g = g0;
    while (g < g1) {
      const int h = g / p.tiles_per_head;
      const int ge = min(g1, (h + 1) * p.tiles_per_head);
      f(h, g - h * p.tiles_per_head, ge - h * p.tiles_per_head);
      g = ge;
    }
  };

  if (warp == kCtEpi / 32) {
    if (lane == 0) {
      // ----------------------------- TMA producer -----------------------------
      int u = 0, seg = 0;
      bool ok = true;
      segments([&](int h, int t0, int t1) {
        if (!ok) return;
        if (seg > 0 && !mbar_wait(&bars->b_empty, (seg - 1) & 1, abort)) { ok = false; return; }
        mbar_arrive_expect_tx(&bars->b_full, S::kBBytes);
        for (int a = 0; a < S::kAtoms; ++a)
          tma_load_2d(Bs + a * S::kSlabB, &maps.b, &bars->b_full, a * 32, h * D);
        ++seg;
        for (int t = t0; t < t1; ++t) {
          const int s = u & 1;
          if (u >= 2 && !mbar_wait(&bars->a_empty[s], ((u - 2) >> 1) & 1, abort)) { ok = false; return; }
          mbar_arrive_expect_tx(&bars->a_full[s], S::kAStage);
          for (int a = 0; a < S::kAtoms; ++a)
            tma_load_2d(As + s * S::kAStage + a * S::kSlabA, &maps.a, &bars->a_full[s], a * 32,
                        h * p.N + t * kTileM);
          ++u;
        }
      });
      for (int x = max(0, u - 2); x < u; ++x) mbar_wait(&bars->a_full[x & 1], (x >> 1) & 1, &never);
      if (seg > 0) mbar_wait(&bars->b_full, (seg - 1) & 1, &never);
    } else if (lane == 1) {
      // ------------------------------ MMA issuer ------------------------------
      constexpr uint32_t idesc = idesc_tf32(kTileM, D);
      const uint32_t a_addr = smem_u32(As), b_addr = smem_u32(Bs);
      int u = 0, seg = 0;
      bool ok = true;
      segments([&](int h, int t0, int t1) {
        if (!ok) return;
        if (!mbar_wait(&bars->b_full, seg & 1, abort)) { ok = false; return; }
        ++seg;
        for (int t = t0; t < t1; ++t, ++u) {
          const int s = u & 1;
          if (!mbar_wait(&bars->a_full[s], (u >> 1) & 1, abort)) { ok = false; return; }
          if (u >= 2 && !mbar_wait(&bars->acc_empty[s], ((u - 2) >> 1) & 1, abort)) {
            ok = false;
            return;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(s * D);
#pragma unroll
          for (int ks = 0; ks < D / 8; ++ks) {
            const uint32_t off = static_cast<uint32_t>((ks >> 2) * S::kSlabA + (ks & 3) * 32);
            const uint32_t boff = static_cast<uint32_t>((ks >> 2) * S::kSlabB + (ks & 3) * 32);
            mma_tf32_ss(d_tmem, smem_desc_sw128(a_addr + s * S::kAStage + off, 16, 1024),
                        smem_desc_sw128(b_addr + boff, 16, 1024), idesc, ks > 0 ? 1u : 0u);
          }
          mma_commit(&bars->acc_full[s]);
        }
        mma_commit(&bars->b_empty);  // the head's B'^T may be replaced
      });
      mma_commit(&bars->mma_idle);
      mbar_wait(&bars->mma_idle, 0, &never);
    }
  } else {
    // ------------- epilogue: row r of the tile, half hf of the columns -------------
    const int r = (warp & 3) * 32 + lane, hf = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(((warp & 3) * 32) << 16);
    int u = 0;
    bool ok = true;
    segments([&](int h, int t0, int t1) {
      named_barrier_sync(kCtBarHead, kCtEpi);  // the previous head's b' is no longer read
      for (int j = threadIdx.x; j < D; j += kCtEpi) bvs[j] = p.bv[static_cast<size_t>(h) * D + j];
      named_barrier_sync(kCtBarHead, kCtEpi);
      const int32_t* pr = p.probes + static_cast<size_t>(h) * p.M;
      const int32_t* pq = p.perm_q + static_cast<size_t>(h) * p.N;
      int lo = 0;  // first probe >= the row's position (ascending over the tiles)
      // the row's token index, read one tile ahead so that the load overlaps
      // the waits of the tile before
      int tok = (t0 * kTileM + r < p.N) ? pq[t0 * kTileM + r] : 0;
      for (int t = t0; t < t1; ++t, ++u) {
        const int s = u & 1;
        const int i = t * kTileM + r;  // group-major position in head h
        const int in = i + kTileM;
        const int tok_next = (t + 1 < t1 && in < p.N) ? pq[in] : 0;
        const bool valid = i < p.N;
        if (valid) {  // probe rows: before the waits too
          if (t == t0) {  // a binary search at the segment's first tile
            int hi = p.M;
            while (lo < hi) {
              const int mid = (lo + hi) >> 1;
              if (pr[mid] < i) lo = mid + 1; else hi = mid;
            }
          } else {  // then a forward scan (about M * 128 / N probes per tile)
            while (lo < p.M && pr[lo] < i) ++lo;
          }
        }
        const bool is_probe = valid && lo < p.M && pr[lo] == i;
        ok = ok && mbar_wait(&bars->acc_full[s], (u >> 1) & 1, abort);
        ok = ok && mbar_wait(&bars->a_full[s], (u >> 1) & 1, abort);  // x tile visible here too
        // tcgen05.ld is warp-collective: the whole warp loads or none of it does
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          const bool plain = i >= p.n_corr;  // text row: x itself
          const size_t dst = valid ? (static_cast<size_t>(h) * p.N + tok) * D : 0;
          const float* odr = p.od + (static_cast<size_t>(h) * p.M + lo) * D;
          const uint8_t* xa = As + s * S::kAStage + r * 128;
          // the half row's accumulators in one round trip
          uint32_t accs[D / 64][32];
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tmem_ld32(tmem + lane_base + static_cast<uint32_t>(s * D + hf * (D / 2) + c * 32), accs[c]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            const int col0 = hf * (D / 2) + c * 32;  // 32 columns = one swizzle atom
            const uint32_t (&acc)[32] = accs[c];
            if (!valid) continue;
            float y[32];
            const uint8_t* xrow = xa + (col0 / 32) * S::kSlabA;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 xv = *reinterpret_cast<const float4*>(xrow + ((q ^ (r & 7)) << 4));
              if (plain) {
                y[4 * q + 0] = xv.x;
                y[4 * q + 1] = xv.y;
                y[4 * q + 2] = xv.z;
                y[4 * q + 3] = xv.w;
              } else {
                y[4 * q + 0] = xv.x + __uint_as_float(acc[4 * q + 0]) + bvs[col0 + 4 * q + 0];
                y[4 * q + 1] = xv.y + __uint_as_float(acc[4 * q + 1]) + bvs[col0 + 4 * q + 1];
                y[4 * q + 2] = xv.z + __uint_as_float(acc[4 * q + 2]) + bvs[col0 + 4 * q + 2];
                y[4 * q + 3] = xv.w + __uint_as_float(acc[4 * q + 3]) + bvs[col0 + 4 * q + 3];
              }
            }
            if (is_probe) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 v = *reinterpret_cast<const float4*>(odr + col0 + 4 * q);
                y[4 * q + 0] = v.x;
                y[4 * q + 1] = v.y;
                y[4 * q + 2] = v.z;
                y[4 * q + 3] = v.w;
              }
            }
            if (OUT_BF16) {
              uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + dst + col0);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                o[q] = make_uint4(pack_bf16x2(y[8 * q + 0], y[8 * q + 1]),
                                  pack_bf16x2(y[8 * q + 2], y[8 * q + 3]),
                                  pack_bf16x2(y[8 * q + 4], y[8 * q + 5]),
                                  pack_bf16x2(y[8 * q + 6], y[8 * q + 7]));
            } else {
              float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + dst + col0);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                o[q] = make_float4(y[4 * q + 0], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bars->acc_empty[s]);
        mbar_arrive(&bars->a_empty[s]);
        tok = tok_next;
      }
    });
  }
  __syncthreads();
  if (*abort && threadIdx.x == 0) raise_status(p.stats, SPARSEPR_ERR_TIMEOUT);
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kCtTmemCols);
  }
}

bool map_f32(CUtensorMap* m, const void* base, size_t rows, int cols, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
  cuuint32_t box[2] = {32, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool OUT_BF16>
cudaError_t launch_ct(const CtMaps& maps, const CtParams& p, int sm_count, cudaStream_t st) {
  const int shb = CtSmem<D>::total;
  cudaError_t e = cudaFuncSetAttribute(correct_tc_kernel<D, OUT_BF16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, shb);
  if (e != cudaSuccess) return e;
  const long long tiles = static_cast<long long>(p.H) * p.tiles_per_head;
  int ctas = sm_count;
  if (ctas > tiles) ctas = static_cast<int>(tiles);
  if (ctas < 1) ctas = 1;
  correct_tc_kernel<D, OUT_BF16><<<ctas, kCtThreads, shb, st>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace

bool correct_tc_supported(int H, int N, int d) {
  return (d == 64 || d == 128) && static_cast<long long>(H) * N >= kTileM &&
         CtSmem<128>::total <= 232448;
}

cudaError_t launch_correct_tc(const float* o_sparse, const float* od, const int32_t* probes,
                              const int32_t* perm_q, const float* bpT, const float* bv32, int H,
                              int N, int n_corr, int M, int d, void* out, bool out_bf16,
                              int sm_count, DeviceStats* stats, cudaStream_t st) {
  CtMaps maps;
  if (!map_f32(&maps.a, o_sparse, static_cast<size_t>(H) * N, d, kTileM) ||
      !map_f32(&maps.b, bpT, static_cast<size_t>(H) * d, d, d))
    return cudaErrorInvalidValue;
  CtParams p;
  p.H = H;
  p.N = N;
  p.M = M;
  p.n_corr = n_corr;
  p.tiles_per_head = (N + kTileM - 1) / kTileM;
  p.od = od;
  p.probes = probes;
  p.perm_q = perm_q;
  p.bv = bv32;
  p.out = out;
  p.stats = stats;
  if (d == 128)
    return out_bf16 ? launch_ct<128, true>(maps, p, sm_count, st)
                    : launch_ct<128, false>(maps, p, sm_count, st);
  if (d == 64)
    return out_bf16 ? launch_ct<64, true>(maps, p, sm_count, st)
                    : launch_ct<64, false>(maps, p, sm_count, st);
  return cudaErrorInvalidValue;
}

}  // namespace spr
