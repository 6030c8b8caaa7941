// Variable-block sparse attention on the 5th-generation tensor cores
// ("Partition the Support, Reconstruct the Residual", 2.C sparse execution;
// "Attention Sparsity is Input-Stable", block selection: the softmax is
// normalised over the kept logits only).
//
// One CTA computes one 128-row query tile of one query group. The key side
// is the union of the kept key groups' contiguous ranges in the group-major
// K/V; runs of adjacent kept groups are merged (once per query group, by the
// slot-count kernel) and cut into 8-row slots, 16 slots per 128-key tile,
// each slot fetched by TMA at an arbitrary row. Rows of a slot past its
// run's end are masked to -inf, so skipped key groups are never multiplied
// (only the tail padding of a run is).
//
// Roles (192 threads): warps 0-3 own one query row per thread (TMEM lane =
// row) and run the online softmax and the epilogue; warp 4 lanes 0 and 1
// stream Q+K and V with TMA (each contiguous piece of slots as power-of-two
// boxes of 8..128 rows); warp 5 lane 0 issues tcgen05.mma.
//   * S = Q K^T goes to one of two TMEM buffers, so S(j+1) runs on the
//     tensor cores while the softmax of tile j works;
//   * P is written bf16 to one of two shared-memory buffers (128B-swizzled,
//     K-major), so the softmax of tile j+1 overlaps P(j) V(j);
//   * O += P V accumulates in TMEM. O is rescaled only when a row maximum
//     grows by more than 2^8; O and the row sum always share one reference
//     maximum, so the result is exact.
// Every mbarrier wait is bounded; a wait that runs out marks the status word
// and the CTA drains its in-flight copies and MMAs, frees tensor memory and
// returns.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kStages = 2;
constexpr int kSlotsPerTile = kTileN / kSlotRows;  // 16
constexpr int kAttnThreads = 320;  // 8 softmax warps, 1 TMA warp, 1 MMA warp
constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O [256, 256+d), exchange [480,512)
constexpr uint32_t kXchCol = 480;    // row-max / row-sum exchange between the two halves of a row
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
  static constexpr int p_off = v_off + kStages * kKVBytes;  // two P buffers
  static constexpr int bar_off = p_off + 2 * kPBytes;
  static constexpr int runs_off = bar_off + 256;
};
// Dynamic shared memory: the d=128 footprint for both head dims (one CTA per
// SM; each CTA allocates 512 TMEM columns), the barrier block, a run list of
// up to kSmemRuns entries, and 1024 bytes of alignment slack.
// The whole per-block maximum is requested; what the 1024-byte alignment of
// the tile region leaves after the barriers holds the run list (>= 226 runs).
constexpr int kAttnSmemBytes = 232448;
static_assert(Smem<128>::runs_off + 226 * 8 + 1008 <= kAttnSmemBytes, "shared memory");

struct Bars {
  uint64_t q_full;
  uint64_t kfull[kStages], vfull[kStages], kempty[kStages], vempty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2], pv_done[2];
  uint64_t mma_idle;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Walks the merged key runs of one query group in ascending order and hands
// out 8-row slots (start row, valid rows).
struct SlotIter {
  const int2* runs;
  int nruns, ri, pos, end;
  __device__ void init(const int2* r, int n) {
    runs = r;
    nruns = n;
    ri = -1;
    pos = 0;
    end = 0;
  }
  __device__ bool next(int& start, int& valid) {
    while (pos >= end) {
      ++ri;
      if (ri >= nruns) return false;
      const int2 rr = runs[ri];
      pos = rr.x;
      end = rr.x + rr.y;
    }
    start = pos;
    valid = min(kSlotRows, end - pos);
    pos += kSlotRows;
    return true;
  }
};

// TMA maps: Q (64-column x 128-row boxes) and K / V with boxes of 8, 16, 32,
// 64 and 128 rows (index = log2(rows / 8)).
struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[5];
  CUtensorMap v[5];
};

struct AttnParams {
  int H, N, q_rows, Cq, kmax;
  const int32_t* off_q;   // [H, Cq+1]
  const int32_t* work;    // [H, tiles_per_head]
  const int32_t* nwork;   // [H]
  const int32_t* nslots;  // [H, Cq]
  const int2* runs;       // [H, Cq, kmax] merged key runs (start, length)
  const int32_t* nruns;   // [H, Cq]
  int tiles_per_head;
  int q_box_rows;  // rows of one Q TMA box (128, fewer for tiny tensors)
  int max_lg;      // largest K/V box used: 8 << max_lg rows (<= rows of the tensor)
  float sc;        // scale * log2(e)
  float* out;
  DeviceStats* stats;
};

// The two warps that share a lane quarter (w and w+4) swap one float per
// row: each stores its value in tensor-memory column base + half, then reads
// the partner's column. Buffers alternate between calls, so one barrier per
// call suffices (a column is rewritten only after the partner passed the
// next barrier, i.e. after it read the old value).
__device__ __forceinline__ float exchange_pair(uint32_t col_base, int half, int quarter, float v) {
  tmem_st1(col_base + half, __float_as_uint(v));
  tmem_wait_st();
  tc_fence_before();
  named_barrier_sync(1 + quarter, 64);
  tc_fence_after();
  const uint32_t o = tmem_ld1(col_base + (half ^ 1));
  tmem_wait_ld();
  return __uint_as_float(o);
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  // byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128B-swizzled slab
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  using L = Smem<HD>;
  constexpr int kAtoms = HD / 64;
  const int h = blockIdx.y;
  if (static_cast<int>(blockIdx.x) >= p.nwork[h]) return;
  const int wcode = p.work[static_cast<size_t>(h) * p.tiles_per_head + blockIdx.x];
  const int g = wcode >> 16, tq = wcode & 0xFFFF;
  const int32_t* offq = p.off_q + static_cast<size_t>(h) * (p.Cq + 1);
  const int row0 = offq[g] + tq * kTileM;
  const int rows_valid = min(kTileM, offq[g + 1] - row0);
  const size_t gi = static_cast<size_t>(h) * p.Cq + g;
  const int ns = p.nslots[gi];
  const int T = (ns + kSlotsPerTile - 1) / kSlotsPerTile;
  const int nr = p.nruns[gi];
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
  int2* runs_s = reinterpret_cast<int2*>(smem + L::runs_off);
  // run-list capacity left in the dynamic allocation after alignment
  const int cap = (kAttnSmemBytes - static_cast<int>(smem - smem_raw) - L::runs_off) / 8;
  const int2* runs_g = p.runs + gi * p.kmax;
  const bool runs_in_smem = nr <= cap;
  const int2* runs = runs_in_smem ? runs_s : runs_g;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], 2 * kTileM);
      mbar_init(&bars->pv_done[b], 1);
    }
    mbar_init(&bars->mma_idle, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (runs_in_smem)
    for (int i = threadIdx.x; i < nr; i += blockDim.x) runs_s[i] = runs_g[i];
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 8) {
    // --------------- TMA producers: lane 0 streams Q and K, lane 1 V ---------------
    if (lane < 2) {
      const bool is_k = (lane == 0);
      const int krow_base = h * p.N;
      if (is_k) {
        mbar_arrive_expect_tx(&bars->q_full, kAtoms * p.q_box_rows * 128);
        for (int a = 0; a < kAtoms; ++a)
          tma_load_2d(Qs + a * L::kSlab, &maps.q, &bars->q_full, a * 64, h * p.q_rows + row0);
      }
      const CUtensorMap* bm = is_k ? maps.k : maps.v;
      uint8_t* base = is_k ? Ks : Vs;
      uint64_t* full = is_k ? bars->kfull : bars->vfull;
      uint64_t* empty = is_k ? bars->kempty : bars->vempty;
      SlotIter it;
      it.init(runs, nr);
      int issued = -1;
      bool ok = true;
      for (int j = 0; j < T; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(&empty[st], ((j / kStages) + 1) & 1, abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[st], L::kKVBytes);
        uint8_t* dst = base + st * L::kKVBytes;
        // contiguous pieces of consecutive slots, each loaded as power-of-two boxes
        int s = 0;
        while (s < kSlotsPerTile) {
          int r0 = 0, vv = 0;
          if (!it.next(r0, vv)) r0 = 0;  // past the last run: any valid rows (masked)
          int n = 1;
          int la = r0, lv = 0;
          while (s + n < kSlotsPerTile) {
            SlotIter peek = it;
            if (!peek.next(la, lv)) la = -1;
            if (la != r0 + kSlotRows * n) break;
            it = peek;
            ++n;
          }
          int t = s, r = r0, m = n;
#pragma unroll 1
          for (int lg = p.max_lg; lg >= 0; --lg) {
            const int sz = 1 << lg;
            while (m >= sz) {
#pragma unroll
              for (int a = 0; a < kAtoms; ++a)
                tma_load_2d(dst + a * L::kSlab + t * 1024, &bm[lg], &full[st], a * 64,
                            krow_base + r);
              t += sz;
              r += sz * kSlotRows;
              m -= sz;
            }
          }
          s += n;
        }
        issued = j;
      }
      if (!ok) {
        // let the loads already in flight land before the CTA exits
        volatile int never = 0;
        for (int j = max(0, issued - kStages + 1); j <= issued; ++j)
          mbar_wait(&full[j % kStages], (j / kStages) & 1, &never);
        if (is_k) mbar_wait(&bars->q_full, 0, &never);
      }
    }
  } else if (warp == 9) {
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
        if (!mbar_wait(&bars->p_full[j & 1], (j >> 1) & 1, abort)) { ok = false; break; }
        if (!mbar_wait(&bars->vfull[st], (j / kStages) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t o_tmem = tmem + 2u * kTileN;
        const uint32_t pb = p_addr + static_cast<uint32_t>((j & 1) * L::kPBytes);
#pragma unroll
        for (int ks = 0; ks < kTileN / 16; ++ks) {
          const uint32_t aoff = static_cast<uint32_t>((ks >> 2) * L::kSlab + (ks & 3) * 32);
          const uint64_t ad = smem_desc_sw128(pb + aoff, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(v_addr + st * L::kKVBytes + ks * 16 * 128, L::kSlab, 1024);
          mma_bf16_ss(o_tmem, ad, bd, idO, (j > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bars->vempty[st]);
        mma_commit(&bars->pv_done[j & 1]);
      }
      // all issued MMAs complete before the CTA releases tensor memory
      mma_commit(&bars->mma_idle);
      volatile int never = 0;
      mbar_wait(&bars->mma_idle, 0, &never);
    }
  } else {
    // ------------- softmax (warps 0-7): two threads per query row -------------
    // warp w owns TMEM lanes 32*(w%4).. (rows) and key columns 64*(w/4)..+63;
    // the two halves of a row agree on the row maximum through shared memory
    constexpr int kHalf = kTileN / 2;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;  // 0..127 == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((quarter * 32) << 16);
    const uint32_t o_tmem = tmem + lane_base + 2u * kTileN + half * (HD / 2);
    const uint32_t xch = tmem + lane_base + kXchCol;  // columns: 2 buffers x 2 halves
    const float sc = p.sc;
    float m_ref = -INFINITY, l_sum = 0.f;
    SlotIter it;
    it.init(runs, nr);
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      // which of this half's 64 key columns are real keys
      uint32_t vmask[2] = {0, 0};
#pragma unroll
      for (int s = 0; s < kSlotsPerTile; ++s) {
        int st0 = 0, vv = 0;
        if (!it.next(st0, vv)) vv = 0;
        const uint32_t bits = (vv >= 8) ? 0xFFu : ((1u << vv) - 1u);
        if ((s >> 3) == half) vmask[(s >> 2) & 1] |= bits << ((s & 3) * 8);
      }
      if (!mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort)) { ok = false; break; }
      tc_fence_after();
      float sv[kHalf];
      {
        uint32_t r[kHalf];
        const uint32_t s_tmem =
            tmem + lane_base + static_cast<uint32_t>((j & 1) * kTileN + half * kHalf);
        tmem_ld32(s_tmem + 0, *reinterpret_cast<uint32_t(*)[32]>(r + 0));
        tmem_ld32(s_tmem + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kHalf; ++i)
          sv[i] = ((vmask[i >> 5] >> (i & 31)) & 1u) ? __uint_as_float(r[i]) * sc : -INFINITY;
      }
      // row maximum of this half: eight independent chains, then a tree
      float m8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) m8[k] = sv[k];
#pragma unroll
      for (int i = 8; i < kHalf; ++i) m8[i & 7] = fmaxf(m8[i & 7], sv[i]);
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      // row maximum over both halves (through tensor memory)
      mx = fmaxf(mx, exchange_pair(xch + (j & 1) * 2, half, quarter, mx));
      // reference maximum for this tile (moves only when it grows by > 2^8)
      float alpha = 1.f;
      bool need = false;
      if (j == 0) {
        m_ref = mx;
      } else if (mx > m_ref + kRescaleThreshold) {
        need = true;
        alpha = ex2_approx(m_ref - mx);
        m_ref = mx;
      }
      // P = 2^(s - m_ref): bf16 pairs in registers, partial row sum in fp32
      uint32_t pk[kHalf / 2];
      float r8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kHalf; i += 2) {
        const float a = ex2_approx(sv[i] - m_ref), b = ex2_approx(sv[i + 1] - m_ref);
        r8[(i >> 1) & 7] += a + b;
        pk[i >> 1] = pack_bf16x2(a, b);
      }
      const float rs = ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
      // P buffer (j & 1) is free once P(j-2) V(j-2) has completed
      if (j >= 2 && !mbar_wait(&bars->pv_done[j & 1], ((j - 2) >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      if (__any_sync(0xffffffffu, need)) {
        // O must hold P(j-1) V(j-1) before it is rescaled (this half's columns)
        if (!mbar_wait(&bars->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HD / 64; ++c) {
          uint32_t r[32];
          tmem_ld32(o_tmem + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(o_tmem + c * 32, r);
        }
        tmem_wait_st();
      }
      l_sum = l_sum * alpha + rs;
      uint8_t* pbuf = Ps + (j & 1) * L::kPBytes + half * L::kSlab;
#pragma unroll
      for (int c8 = 0; c8 < kHalf / 8; ++c8) {
        const uint4 v4 = make_uint4(pk[c8 * 4 + 0], pk[c8 * 4 + 1], pk[c8 * 4 + 2], pk[c8 * 4 + 3]);
        *reinterpret_cast<uint4*>(pbuf + swz(row, c8)) = v4;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full[j & 1]);
    }
    // ---------------- epilogue: O / l -> global (fp32, group-major rows) ------
    // both halves of a row combine their partial sums (buffer T & 1 is free:
    // the partner read buffer (T-1) & 1 last)
    l_sum += exchange_pair(xch + (T & 1) * 2, half, quarter, l_sum);
    if (ok && mbar_wait(&bars->pv_done[(T - 1) & 1], ((T - 1) >> 1) & 1, abort)) {
      tc_fence_after();
      const float inv = 1.f / l_sum;
      float* orow = p.out + (static_cast<size_t>(h) * p.q_rows + row0 + row) * HD + half * (HD / 2);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) {
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
// One warp per head: tile counts are prefix-summed 32 groups at a time.
// ---------------------------------------------------------------------------
__global__ void work_list_kernel(const int32_t* off_q, int Cq, int tiles_per_head, int32_t* work,
                                 int32_t* nwork) {
  const int h = blockIdx.x, lane = threadIdx.x;
  const int32_t* oq = off_q + static_cast<size_t>(h) * (Cq + 1);
  int32_t* wl = work + static_cast<size_t>(h) * tiles_per_head;
  int32_t base = 0;
  for (int g0 = 0; g0 < Cq; g0 += 32) {
    const int g = g0 + lane;
    const int n = (g < Cq) ? oq[g + 1] - oq[g] : 0;
    const int t = n > 0 ? (n + kTileM - 1) / kTileM : 0;
    int x = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const int start = base + x - t;
    for (int i = 0; i < t && start + i < tiles_per_head; ++i) wl[start + i] = (g << 16) | i;
    base += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) nwork[h] = min(base, tiles_per_head);
}

// Merged key runs and KV slot counts per query group (same rule the attention
// kernel walks), and the exact routed pair count per head.
__global__ void slots_pairs_kernel(const int32_t* off_q, const int32_t* off_k, const int32_t* csr,
                                   const int32_t* kh, int H, int N, int Cq, int Ck, int kmax,
                                   int32_t* nslots, int2* runs, int32_t* nruns, int64_t* pairs,
                                   DeviceStats* stats) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * Cq) return;
  const int h = i / Cq, g = i % Cq;
  const int32_t* oq = off_q + static_cast<size_t>(h) * (Cq + 1);
  const int32_t* ok = off_k + static_cast<size_t>(h) * (Ck + 1);
  const int32_t* row = csr + static_cast<size_t>(i) * kmax;
  int2* rout = runs + static_cast<size_t>(i) * kmax;
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
    nruns[i] = 0;
    raise_status(stats, SPARSEPR_ERR_INVALID_ARG);
    return;
  }
  int64_t keys = 0;
  int slots = 0, nr = 0;
  int ci = 0;
  while (ci < k) {
    const int c = row[ci];
    const int lo = ok[c];
    int hi = ok[c + 1];
    while (ci + 1 < k && ok[row[ci + 1]] == hi) {
      ++ci;
      hi = ok[row[ci] + 1];
    }
    if (hi > lo) {
      rout[nr++] = make_int2(lo, hi - lo);
      keys += hi - lo;
      slots += (hi - lo + kSlotRows - 1) / kSlotRows;
    }
    ++ci;
  }
  nslots[i] = slots;
  nruns[i] = nr;
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
  AttnMaps maps;
  const size_t qrows_total = static_cast<size_t>(a.H) * a.q_rows;
  const size_t krows_total = static_cast<size_t>(a.H) * a.N;
  prm.q_box_rows = qrows_total < static_cast<size_t>(kTileM) ? static_cast<int>(qrows_total) : kTileM;
  if (!make_map(&maps.q, a.qp, qrows_total, HD, prm.q_box_rows)) return cudaErrorInvalidValue;
  prm.max_lg = 0;
  for (int lg = 0; lg < 5; ++lg) {
    // boxes larger than the tensor (tiny inputs) are never used
    const int rows = kSlotRows << lg;
    const bool fits = static_cast<size_t>(rows) <= krows_total;
    if (fits) prm.max_lg = lg;
    const int box = fits ? rows : kSlotRows;
    if (!make_map(&maps.k[lg], a.kp, krows_total, HD, box) ||
        !make_map(&maps.v[lg], a.vp, krows_total, HD, box))
      return cudaErrorInvalidValue;
  }
  const int shb = kAttnSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<HD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, shb);
  if (e != cudaSuccess) return e;
  dim3 grid(a.tiles_per_head, a.H);
  sparse_attn_kernel<HD><<<grid, kAttnThreads, shb, st>>>(maps, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_sparse_attn(const AttnArgs& a, cudaStream_t st) {
  work_list_kernel<<<a.H, 32, 0, st>>>(a.off_q, a.Cq, a.tiles_per_head, a.work, a.nwork);
  if (a.pairs) zero_i64_kernel<<<(a.H + 127) / 128, 128, 0, st>>>(a.pairs, a.H);
  const int n = a.H * a.Cq;
  slots_pairs_kernel<<<(n + 127) / 128, 128, 0, st>>>(a.off_q, a.off_k, a.csr, a.kh, a.H, a.N,
                                                     a.Cq, a.Ck, a.kmax, a.nslots, a.runs,
                                                     a.nruns, a.pairs, a.stats);
  if (a.pairs) pairs_to_stats_kernel<<<(a.H + 127) / 128, 128, 0, st>>>(a.pairs, a.H, a.stats);
  AttnParams prm;
  prm.H = a.H;
  prm.N = a.N;
  prm.q_rows = a.q_rows;
  prm.Cq = a.Cq;
  prm.kmax = a.kmax;
  prm.off_q = a.off_q;
  prm.work = a.work;
  prm.nwork = a.nwork;
  prm.nslots = a.nslots;
  prm.runs = a.runs;
  prm.nruns = a.nruns;
  prm.tiles_per_head = a.tiles_per_head;
  prm.q_box_rows = kTileM;
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
