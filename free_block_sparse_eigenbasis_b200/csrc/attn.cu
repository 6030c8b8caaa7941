// Variable-block sparse attention on the 5th-generation tensor cores
// ("Partition the Support, Reconstruct the Residual", 2.C sparse execution;
// "Attention Sparsity is Input-Stable", block selection: the softmax is
// normalised over the kept logits only).
//
// One CTA computes one 128-row query tile of one query group. The key side
// is the union of the kept key groups' contiguous ranges in the group-major
// K/V; runs of adjacent kept groups are merged and cut into 8-row slots,
// 16 slots per 128-key tile, each slot fetched by TMA at an arbitrary row.
// Rows of a slot past its run's end are masked to -inf, so skipped key
// groups are never multiplied (only the tail padding of a run is).
//
// Roles (192 threads): warps 0-3 own one query row per thread (TMEM lane =
// row) and run the online softmax and the epilogue; warp 4 lane 0 issues TMA
// loads; warp 5 lane 0 issues tcgen05.mma. S = Q K^T goes to one of two TMEM
// buffers (S(j+1) runs while the softmax of tile j works), P is written bf16
// to shared memory in the 128B-swizzled K-major layout, and O += P V
// accumulates in TMEM. O is rescaled only when a row maximum grows by more
// than 2^8; O and the row sum always share one reference maximum, so the
// result is exact.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kStages = 2;
constexpr int kSlotsPerTile = kTileN / kSlotRows;  // 16
constexpr int kAttnThreads = 192;
constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O [256, 256+d)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int HD>
struct Smem {
  static constexpr int kAtoms = HD / 64;           // 128-byte swizzle atoms along d
  static constexpr int kSlab = kTileM * 128;       // one 64-column slab of 128 rows (16 KB)
  static constexpr int kQBytes = kAtoms * kSlab;
  static constexpr int kKVBytes = kAtoms * kSlab;  // kTileN == kTileM
  static constexpr int kPBytes = (kTileN / 64) * kSlab;
  static constexpr int q_off = 0;
  static constexpr int k_off = q_off + kQBytes;
  static constexpr int v_off = k_off + kStages * kKVBytes;
  static constexpr int p_off = v_off + kStages * kKVBytes;
  static constexpr int bar_off = p_off + kPBytes;
};
// Dynamic shared memory requested: the d=128 footprint for both head dims, so
// that one CTA holds an SM (each CTA allocates 512 TMEM columns), plus
// 1024 bytes of alignment slack.
constexpr int kAttnSmemBytes = Smem<128>::bar_off + 256 + 1024;
static_assert(kAttnSmemBytes <= 232448, "shared memory");

struct Bars {
  uint64_t q_full;
  uint64_t kfull[kStages], vfull[kStages], kempty[kStages], vempty[kStages];
  uint64_t s_full[2];
  uint64_t p_full, pv_done, mma_idle;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Walks the kept key groups of one query group in ascending order, merging
// adjacent ranges, and hands out 8-row slots (start row, valid rows).
struct SlotIter {
  const int32_t* csr;
  const int32_t* offk;
  int k, ci, pos, end;
  __device__ void init(const int32_t* c, const int32_t* o, int kk) {
    csr = c;
    offk = o;
    k = kk;
    ci = -1;
    pos = 0;
    end = 0;
  }
  __device__ bool next(int& start, int& valid) {
    while (pos >= end) {
      ++ci;
      if (ci >= k) return false;
      const int c = csr[ci];
      pos = offk[c];
      end = offk[c + 1];
      while (ci + 1 < k && offk[csr[ci + 1]] == end) {
        ++ci;
        end = offk[csr[ci] + 1];
      }
    }
    start = pos;
    valid = min(kSlotRows, end - pos);
    pos += kSlotRows;
    return true;
  }
};

struct AttnParams {
  int H, N, q_rows, Cq, Ck, kmax;
  const int32_t* off_q;   // [H, Cq+1]
  const int32_t* off_k;   // [H, Ck+1]
  const int32_t* csr;     // [H, Cq, kmax]
  const int32_t* kh;      // [H]
  const int32_t* work;    // [H, tiles_per_head]
  const int32_t* nwork;   // [H]
  const int32_t* nslots;  // [H, Cq]
  int tiles_per_head;
  int q_box_rows;  // rows of one Q TMA box (128, fewer for tiny tensors)
  float sc;  // scale * log2(e)
  float* out;
  DeviceStats* stats;
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  // byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128B-swizzled slab
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = Smem<HD>;
  constexpr int kAtoms = HD / 64;
  const int h = blockIdx.y;
  if (static_cast<int>(blockIdx.x) >= p.nwork[h]) return;
  const int wcode = p.work[static_cast<size_t>(h) * p.tiles_per_head + blockIdx.x];
  const int g = wcode >> 16, tq = wcode & 0xFFFF;
  const int32_t* offq = p.off_q + static_cast<size_t>(h) * (p.Cq + 1);
  const int32_t* offk = p.off_k + static_cast<size_t>(h) * (p.Ck + 1);
  const int row0 = offq[g] + tq * kTileM;
  const int rows_valid = min(kTileM, offq[g + 1] - row0);
  const int ns = p.nslots[static_cast<size_t>(h) * p.Cq + g];
  const int T = (ns + kSlotsPerTile - 1) / kSlotsPerTile;
  const int kk = p.kh[h];
  const int32_t* csr_row = p.csr + (static_cast<size_t>(h) * p.Cq + g) * p.kmax;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (T == 0) {
    // empty kept set (reported by the slot-count kernel): rows are zero
    if (static_cast<int>(threadIdx.x) < rows_valid) {
      float* o = p.out + (static_cast<size_t>(h) * p.q_rows + row0 + threadIdx.x) * HD;
      for (int c = 0; c < HD; c += 4) *reinterpret_cast<float4*>(o + c) = make_float4(0, 0, 0, 0);
    }
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* Qs = smem + L::q_off;
  uint8_t* Ks = smem + L::k_off;
  uint8_t* Vs = smem + L::v_off;
  uint8_t* Ps = smem + L::p_off;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::bar_off);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    mbar_init(&bars->s_full[0], 1);
    mbar_init(&bars->s_full[1], 1);
    mbar_init(&bars->p_full, kTileM);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->mma_idle, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 4) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      const int krow_base = h * p.N;
      mbar_arrive_expect_tx(&bars->q_full, kAtoms * p.q_box_rows * 128);
      for (int a = 0; a < kAtoms; ++a)
        tma_load_2d(Qs + a * L::kSlab, &tmQ, &bars->q_full, a * 64, h * p.q_rows + row0);
      SlotIter it;
      it.init(csr_row, offk, kk);
      int issued_k = -1, issued_v = -1;
      bool ok = true;
      for (int j = 0; j < T && ok; ++j) {
        const int st = j % kStages;
        const uint32_t par = ((j / kStages) + 1) & 1;  // phase of tile j - kStages
        int starts[kSlotsPerTile];
#pragma unroll
        for (int s = 0; s < kSlotsPerTile; ++s) {
          int st0 = 0, vv = 0;
          if (!it.next(st0, vv)) st0 = 0;
          starts[s] = st0;
        }
        if (j >= kStages && !mbar_wait(&bars->kempty[st], par, abort)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->kfull[st], L::kKVBytes);
        uint8_t* kd = Ks + st * L::kKVBytes;
        for (int s = 0; s < kSlotsPerTile; ++s)
          for (int a = 0; a < kAtoms; ++a)
            tma_load_2d(kd + a * L::kSlab + s * 1024, &tmK, &bars->kfull[st], a * 64,
                        krow_base + starts[s]);
        issued_k = j;
        if (j >= kStages && !mbar_wait(&bars->vempty[st], par, abort)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->vfull[st], L::kKVBytes);
        uint8_t* vd = Vs + st * L::kKVBytes;
        for (int s = 0; s < kSlotsPerTile; ++s)
          for (int a = 0; a < kAtoms; ++a)
            tma_load_2d(vd + a * L::kSlab + s * 1024, &tmV, &bars->vfull[st], a * 64,
                        krow_base + starts[s]);
        issued_v = j;
      }
      if (!ok) {
        // let the loads already in flight land before the CTA exits
        volatile int never = 0;
        for (int j = max(0, issued_k - kStages + 1); j <= issued_k; ++j)
          mbar_wait(&bars->kfull[j % kStages], (j / kStages) & 1, &never);
        for (int j = max(0, issued_v - kStages + 1); j <= issued_v; ++j)
          mbar_wait(&bars->vfull[j % kStages], (j / kStages) & 1, &never);
        volatile int never2 = 0;
        mbar_wait(&bars->q_full, 0, &never2);
      }
    }
  } else if (warp == 5) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kTileM, kTileN, 0);
      constexpr uint32_t idO = idesc_bf16(kTileM, HD, 1);
      const uint32_t q_addr = smem_u32(Qs), k_addr = smem_u32(Ks), v_addr = smem_u32(Vs),
                     p_addr = smem_u32(Ps);
      auto issue_s = [&](int j) {
        const int st = j % kStages;
        const uint32_t d_tmem = tmem + static_cast<uint32_t>((j & 1) * kTileN);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint32_t off = static_cast<uint32_t>((ks >> 2) * L::kSlab + (ks & 3) * 32);
          const uint64_t ad = smem_desc_sw128(q_addr + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + st * L::kKVBytes + off, 16, 1024);
          mma_bf16_ss(d_tmem, ad, bd, idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->kempty[st]);
        mma_commit(&bars->s_full[j & 1]);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort);
      if (ok) ok = mbar_wait(&bars->kfull[0], 0, abort);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; j < T && ok; ++j) {
        if (j + 1 < T) {
          const int st1 = (j + 1) % kStages;
          if (!mbar_wait(&bars->kfull[st1], ((j + 1) / kStages) & 1, abort)) { ok = false; break; }
          tc_fence_after();
          issue_s(j + 1);
        }
        const int st = j % kStages;
        if (!mbar_wait(&bars->p_full, j & 1, abort)) { ok = false; break; }
        if (!mbar_wait(&bars->vfull[st], (j / kStages) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t o_tmem = tmem + 2u * kTileN;
#pragma unroll
        for (int ks = 0; ks < kTileN / 16; ++ks) {
          const uint32_t aoff = static_cast<uint32_t>((ks >> 2) * L::kSlab + (ks & 3) * 32);
          const uint64_t ad = smem_desc_sw128(p_addr + aoff, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(v_addr + st * L::kKVBytes + ks * 16 * 128, L::kSlab, 1024);
          mma_bf16_ss(o_tmem, ad, bd, idO, (j > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bars->vempty[st]);
        mma_commit(&bars->pv_done);
      }
      // all issued MMAs complete before the CTA releases tensor memory
      mma_commit(&bars->mma_idle);
      volatile int never = 0;
      mbar_wait(&bars->mma_idle, 0, &never);
    }
  } else {
    // --------------------- softmax (warps 0-3, one row per thread) -------------
    const int row = threadIdx.x;  // 0..127 == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp * 32) << 16);
    const float sc = p.sc;
    float m_ref = -INFINITY, l_sum = 0.f;
    SlotIter it;
    it.init(csr_row, offk, kk);
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      // which of the 128 key columns are real keys
      uint32_t vmask[4] = {0, 0, 0, 0};
#pragma unroll
      for (int s = 0; s < kSlotsPerTile; ++s) {
        int st0 = 0, vv = 0;
        if (!it.next(st0, vv)) vv = 0;
        const uint32_t bits = (vv >= 8) ? 0xFFu : ((1u << vv) - 1u);
        vmask[s >> 2] |= bits << ((s & 3) * 8);
      }
      if (!mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort)) { ok = false; break; }
      tc_fence_after();
      float sv[kTileN];
      const uint32_t s_tmem = tmem + lane_base + static_cast<uint32_t>((j & 1) * kTileN);
#pragma unroll
      for (int c = 0; c < kTileN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(s_tmem + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const bool valid = (vmask[c] >> i) & 1u;
          sv[c * 32 + i] = valid ? __uint_as_float(r[i]) * sc : -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kTileN; ++i) mx = fmaxf(mx, sv[i]);
      // P_{j-1} V_{j-1} must be complete before P is overwritten or O rescaled
      if (j > 0 && !mbar_wait(&bars->pv_done, (j - 1) & 1, abort)) { ok = false; break; }
      tc_fence_after();
      if (j == 0) {
        m_ref = mx;
      } else {
        const bool need = mx > m_ref + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m_ref - mx) : 1.f;
          if (need) {
            l_sum *= alpha;
            m_ref = mx;
          }
          const uint32_t o_tmem = tmem + lane_base + 2u * kTileN;
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(o_tmem + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(o_tmem + c * 32, r);
          }
          tmem_wait_st();
        }
      }
      // P = 2^(s - m_ref) in bf16, row sum in fp32
      float rs = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < kTileN / 8; ++c8) {
        float pv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pv[i] = ex2_approx(sv[c8 * 8 + i] - m_ref);
          rs += pv[i];
        }
        uint4 pk;
        pk.x = pack_bf16x2(pv[0], pv[1]);
        pk.y = pack_bf16x2(pv[2], pv[3]);
        pk.z = pack_bf16x2(pv[4], pv[5]);
        pk.w = pack_bf16x2(pv[6], pv[7]);
        const uint32_t off = static_cast<uint32_t>((c8 >> 3) * L::kSlab) + swz(row, c8 & 7);
        *reinterpret_cast<uint4*>(Ps + off) = pk;
      }
      l_sum += rs;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
    }
    // ---------------- epilogue: O / l -> global (fp32, group-major rows) ------
    if (ok && mbar_wait(&bars->pv_done, (T - 1) & 1, abort)) {
      tc_fence_after();
      const float inv = 1.f / l_sum;
      const uint32_t o_tmem = tmem + lane_base + 2u * kTileN;
      float* orow = p.out + (static_cast<size_t>(h) * p.q_rows + row0 + row) * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(o_tmem + c * 32, r);
        tmem_wait_ld();
        if (row < rows_valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(orow + c * 32 + i) =
                make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                            __uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
        }
      }
    }
  }
  __syncthreads();
  if (*abort && threadIdx.x == 0) raise_status(p.stats, SPARSEPR_ERR_TIMEOUT);
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Work list: one entry per 128-row tile of each query group, (g << 16) | t.
// ---------------------------------------------------------------------------
__global__ void work_list_kernel(const int32_t* off_q, int Cq, int tiles_per_head, int32_t* work,
                                 int32_t* nwork) {
  const int h = blockIdx.x;
  const int32_t* oq = off_q + static_cast<size_t>(h) * (Cq + 1);
  __shared__ int32_t total;
  if (threadIdx.x == 0) {
    int32_t pos = 0;
    for (int g = 0; g < Cq; ++g) {
      const int n = oq[g + 1] - oq[g];
      const int t = (n + kTileM - 1) / kTileM;
      for (int i = 0; i < t && pos < tiles_per_head; ++i)
        work[static_cast<size_t>(h) * tiles_per_head + pos++] = (g << 16) | i;
    }
    total = pos;
    nwork[h] = pos;
  }
}

// KV slot counts per query group (same merge rule as the attention kernel's
// walk) and the exact routed pair count per head.
__global__ void slots_pairs_kernel(const int32_t* off_q, const int32_t* off_k, const int32_t* csr,
                                   const int32_t* kh, int H, int N, int Cq, int Ck, int kmax,
                                   int32_t* nslots, int64_t* pairs, DeviceStats* stats) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * Cq) return;
  const int h = i / Cq, g = i % Cq;
  const int32_t* oq = off_q + static_cast<size_t>(h) * (Cq + 1);
  const int32_t* ok = off_k + static_cast<size_t>(h) * (Ck + 1);
  const int32_t* row = csr + static_cast<size_t>(i) * kmax;
  const int k = kh[h];
  const int64_t nq = oq[g + 1] - oq[g];
  // reject malformed routes before the attention kernel walks them
  bool valid = (k >= 0 && k <= kmax && ok[0] >= 0 && ok[Ck] <= N && nq >= 0);
  for (int ci = 0; valid && ci < k; ++ci) {
    const int c = row[ci];
    valid = (c >= 0 && c < Ck && ok[c] >= 0 && ok[c] <= ok[c + 1]);
  }
  if (!valid) {
    nslots[i] = 0;
    raise_status(stats, SPARSEPR_ERR_INVALID_ARG);
    return;
  }
  int64_t keys = 0;
  int slots = 0;
  int ci = 0;
  while (ci < k) {
    int c = row[ci];
    int lo = ok[c], hi = ok[c + 1];
    while (ci + 1 < k && ok[row[ci + 1]] == hi) {
      ++ci;
      hi = ok[row[ci] + 1];
    }
    keys += hi - lo;
    slots += (hi - lo + kSlotRows - 1) / kSlotRows;
    ++ci;
  }
  nslots[i] = slots;
  if (pairs && nq > 0) atomicAdd(reinterpret_cast<unsigned long long*>(&pairs[h]),
                                 static_cast<unsigned long long>(nq * keys));
  if (nq > 0 && keys == 0) raise_status(stats, SPARSEPR_ERR_NUMERIC);
}

__global__ void zero_i64_kernel(int64_t* p, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = 0;
}

__global__ void pairs_to_stats_kernel(const int64_t* pairs, int H, DeviceStats* stats) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < H) stats->pairs_sparse[i] = pairs[i];
}

__global__ void cast_bf16_kernel(const float* src, __nv_bfloat16* dst, size_t n) {
  const size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    const float4 v = *reinterpret_cast<const float4*>(src + i);
    reinterpret_cast<__nv_bfloat162*>(dst + i)[0] = __floats2bfloat162_rn(v.x, v.y);
    reinterpret_cast<__nv_bfloat162*>(dst + i)[1] = __floats2bfloat162_rn(v.z, v.w);
  } else {
    for (size_t t = i; t < n; ++t) dst[t] = __float2bfloat16_rn(src[t]);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps (driver entry point fetched through the runtime).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
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

// 2D bf16 map over [rows, d] with a box of 64 columns x box_rows rows,
// 128-byte swizzle; rows past the end read as zero.
bool make_map(CUtensorMap* m, const void* base, size_t rows, int d, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int HD>
cudaError_t launch_attn_hd(const AttnArgs& a, AttnParams prm, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  const size_t qrows_total = static_cast<size_t>(a.H) * a.q_rows;
  prm.q_box_rows = qrows_total < static_cast<size_t>(kTileM) ? static_cast<int>(qrows_total) : kTileM;
  if (!make_map(&tq, a.qp, qrows_total, HD, prm.q_box_rows) ||
      !make_map(&tk, a.kp, static_cast<size_t>(a.H) * a.N, HD, kSlotRows) ||
      !make_map(&tv, a.vp, static_cast<size_t>(a.H) * a.N, HD, kSlotRows))
    return cudaErrorInvalidValue;
  const int shb = kAttnSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<HD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, shb);
  if (e != cudaSuccess) return e;
  dim3 grid(a.tiles_per_head, a.H);
  sparse_attn_kernel<HD><<<grid, kAttnThreads, shb, st>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_sparse_attn(const AttnArgs& a, cudaStream_t st) {
  work_list_kernel<<<a.H, 32, 0, st>>>(a.off_q, a.Cq, a.tiles_per_head, a.work, a.nwork);
  if (a.pairs) zero_i64_kernel<<<(a.H + 127) / 128, 128, 0, st>>>(a.pairs, a.H);
  const int n = a.H * a.Cq;
  slots_pairs_kernel<<<(n + 127) / 128, 128, 0, st>>>(a.off_q, a.off_k, a.csr, a.kh, a.H, a.N,
                                                     a.Cq, a.Ck, a.kmax, a.nslots, a.pairs,
                                                     a.stats);
  if (a.pairs) pairs_to_stats_kernel<<<(a.H + 127) / 128, 128, 0, st>>>(a.pairs, a.H, a.stats);
  AttnParams prm;
  prm.H = a.H;
  prm.N = a.N;
  prm.q_rows = a.q_rows;
  prm.Cq = a.Cq;
  prm.Ck = a.Ck;
  prm.kmax = a.kmax;
  prm.off_q = a.off_q;
  prm.off_k = a.off_k;
  prm.csr = a.csr;
  prm.kh = a.kh;
  prm.work = a.work;
  prm.nwork = a.nwork;
  prm.nslots = a.nslots;
  prm.tiles_per_head = a.tiles_per_head;
  prm.sc = a.scale * kLog2e;
  prm.out = a.out;
  prm.stats = a.stats;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.d == 128) return launch_attn_hd<128>(a, prm, st);
  if (a.d == 64) return launch_attn_hd<64>(a, prm, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_cast_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t st) {
  const size_t threads = (n + 3) / 4;
  cast_bf16_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(src, dst, n);
  return cudaGetLastError();
}

}  // namespace spr
