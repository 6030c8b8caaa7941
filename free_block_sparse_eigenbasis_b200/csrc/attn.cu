// Variable-block sparse attention on the 5th-generation tensor cores
// ("Partition the Support, Reconstruct the Residual", 2.C sparse execution;
// "Attention Sparsity is Input-Stable", block selection: the softmax is
// normalised over the kept logits only).
//
// One CTA computes one unit of up to 256 query rows of one query group. The
// key side is the union of the kept key groups' contiguous ranges in the
// group-major K/V; runs of adjacent kept groups are merged (once per query
// group, by the slot-count kernel) and cut into 8-row slots, 16 slots per
// 128-key tile, each contiguous piece fetched by TMA at an arbitrary row.
// Rows of a slot past its run's end are masked to -inf, so skipped key groups
// are never multiplied (only the tail padding of a run is).
//
// Roles (352 threads): two softmax warpgroups (warps 0-3 and 4-7, thread =
// query row = TMEM lane) each own one TMEM slot (S_i, O_i, with P_i written
// as packed bf16 over the first 64 columns of S_i); warp 8 streams Q and the
// K tiles and warp 10 the V tiles with TMA, each through its own ring; warp 9
// lane 0 issues tcgen05.mma.
//   * a unit of two 128-row query tiles gives tile i to warpgroup i: both
//     see every key tile, and the tensor cores alternate between them
//     (P_0 V, S_0 of the next tile, P_1 V, S_1 of the next tile), so one
//     warpgroup's softmax overlaps the other's MMAs;
//   * a unit of one query tile splits the key tiles instead (even ones to
//     warpgroup 0, odd ones to warpgroup 1) with separate running maxima
//     and accumulators, merged at the end;
//   * P V reads P from tensor memory (no shared-memory round trip). The
//     softmax streams each row in two halves of 64 columns against a
//     reference maximum taken from the first key tile, with no maximum pass
//     afterwards; a half whose sum exceeds 2^32 is formed again against a
//     reference raised by a whole number of log2 units, and O, the row sum
//     and the stored half are scaled by that power of two. O and the row
//     sum always share one reference, so the result is exact.
// Every mbarrier wait is bounded; a wait that runs out marks the status word
// and the CTA drains its in-flight copies and MMAs, frees tensor memory and
// returns.
#include "common.cuh"
#include "internal.h"

namespace spr {
namespace {

constexpr int kStages = 2;                         // K and V ring depth
constexpr int kSlotsPerTile = kTileN / kSlotRows;  // 16
constexpr int kUnitRows = 2 * kTileM;              // query rows per CTA
constexpr int kAttnThreads = 352;  // 8 softmax warps, K TMA warp (8), MMA warp (9), V TMA warp (10)
constexpr uint32_t kTmemCols = 512;  // S_0 [0,128), S_1 [128,256), O_0 [256,256+d), O_1 after
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kOverflowSum = 4294967296.0f;  // 2^32: a larger half sum moves the reference

template <int HD>
struct Smem {
  static constexpr int kAtoms = HD / 64;           // 128-byte swizzle atoms along d
  static constexpr int kSlab = kTileM * 128;       // one 64-column slab of 128 rows (16 KB)
  static constexpr int kQBytes = kAtoms * kSlab;   // one query tile
  static constexpr int kKVBytes = kAtoms * kSlab;  // kTileN == kTileM
  static constexpr int q_off = 0;                  // two query tiles
  static constexpr int k_off = q_off + 2 * kQBytes;
  static constexpr int v_off = k_off + kStages * kKVBytes;
  static constexpr int bar_off = v_off + kStages * kKVBytes;
  static constexpr int ml_off = bar_off + 256;     // [2][2][128] f32 row maxima and sums
  static constexpr int runs_off = ml_off + 2048;
};
// Dynamic shared memory: the d=128 footprint for both head dims (one CTA per
// SM; each CTA allocates 512 TMEM columns), the barrier block, the final
// merge buffer, a run list, and 1024 bytes of alignment slack. What the
// 1024-byte alignment of the tile region leaves holds the run list (>= 4000
// runs); longer lists are read from global memory.
constexpr int kAttnSmemBytes = 232448;
static_assert(Smem<128>::runs_off + 4000 * 8 + 1008 <= kAttnSmemBytes, "shared memory");

struct Bars {
  uint64_t q_full;
  uint64_t kfull[kStages], vfull[kStages], kempty[kStages], vempty[kStages];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t mma_idle;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

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
  int splits, units;  // split-KV (splits > 1): partial outputs per (unit, split)
  float* opart;
  float* lpart;
  float* lse;  // [H, q_rows] log2-sum-exp of each row's scaled logits (may be null)
  int unit_rows;  // query rows per unit: 256 (two tiles), 128 in the dual probe pass
  // dual probe pass: the second warpgroup takes the same rows and key tiles
  // with each row's keys limited to the kept runs of its query group
  float* out2;            // [H, q_rows, d] its outputs (splits == 1)
  float* opart2;          // its split-KV partial outputs / log2-sum-exps
  float* lpart2;
  float* lse2;            // [H, q_rows] (may be null)
  const int32_t* pgrp;    // [H, q_rows] query group of each row
  const int2* gruns;      // [H, gCq, gkmax + 1] kept runs of the query groups (ascending)
  const int32_t* gnruns;  // [H, gCq]
  int gCq, gkmax;
};

// Key-column validity of the key tiles of one query group, walked in
// ascending tile order: every run contributes ceil(len / 8) slots, of which
// only the last may be partial; slots past the last run are padding.
struct MaskWalk {
  const int2* runs;
  int nr, ns, ri, rend;  // rend: slots up to and including run ri
  __device__ void init(const int2* r, int n, int nslots) {
    runs = r;
    nr = n;
    ns = nslots;
    ri = 0;
    rend = (n > 0) ? (r[0].y + kSlotRows - 1) / kSlotRows : 0;
  }
  // consume the runs that end before tile j (start of a key-tile range)
  __device__ void advance_to(int j) {
    while (ri < nr && rend <= j * kSlotsPerTile) {
      ++ri;
      if (ri < nr) rend += (runs[ri].y + kSlotRows - 1) / kSlotRows;
    }
  }
  // bit c of m[c / 32] = key column c of tile j is a real key
  __device__ void tile(int j, uint32_t (&m)[4]) {
    m[0] = m[1] = m[2] = m[3] = 0xFFFFFFFFu;
    const int lo = j * kSlotsPerTile, hi = lo + kSlotsPerTile;
    while (ri < nr && rend <= hi) {
      const int rem = runs[ri].y & (kSlotRows - 1);
      const int last = rend - 1;
      if (rem && last >= lo) {
        const int s = last - lo;
        m[s >> 2] &= ~((0xFFu & ~((1u << rem) - 1u)) << ((s & 3) * 8));
      }
      ++ri;
      if (ri < nr) rend += (runs[ri].y + kSlotRows - 1) / kSlotRows;
    }
    for (int s = max(ns, lo) - lo; s < kSlotsPerTile; ++s) m[s >> 2] &= ~(0xFFu << ((s & 3) * 8));
  }
};

// Packed fp32x2 fma (one instruction for two columns) and the three-input
// maximum of sm_100, used by the softmax.
__device__ __forceinline__ void fma2(float& x0, float& x1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(x0), "=f"(x1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
// packed fp32x2 add: (x.x, x.y) += (a, b)
__device__ __forceinline__ void add2(float2& x, float a, float b) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(x.x), "=f"(x.y)
      : "f"(x.x), "f"(x.y), "f"(a), "f"(b));
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// DUAL: the dual probe pass (units of one 128-row tile, see AttnParams).
template <int HD, bool DUAL>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  using L = Smem<HD>;
  constexpr int kAtoms = HD / 64;
  const int h = blockIdx.y;
  const int wi = static_cast<int>(blockIdx.x) / p.splits, split = static_cast<int>(blockIdx.x) % p.splits;
  if (wi >= p.nwork[h]) return;
  const int wcode = p.work[static_cast<size_t>(h) * p.tiles_per_head + wi];
  const int g = wcode >> 16, tu = wcode & 0xFFFF;
  const int32_t* offq = p.off_q + static_cast<size_t>(h) * (p.Cq + 1);
  const int row0 = offq[g] + tu * p.unit_rows;
  const int rows_unit = min(p.unit_rows, offq[g + 1] - row0);
  const int nq = (!DUAL && rows_unit > kTileM) ? 2 : 1;  // query tiles in this unit
  const size_t gi = static_cast<size_t>(h) * p.Cq + g;
  const int ns = p.nslots[gi];
  const int T_all = (ns + kSlotsPerTile - 1) / kSlotsPerTile;
  // this CTA's key tiles [j0, j0 + T)
  const int j0 = static_cast<int>(static_cast<long long>(T_all) * split / p.splits);
  const int T = static_cast<int>(static_cast<long long>(T_all) * (split + 1) / p.splits) - j0;
  const int nr = p.nruns[gi];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool partial = p.splits > 1;
  const size_t pbase = ((static_cast<size_t>(h) * p.units + wi) * p.splits + split) * p.unit_rows;

  if (T == 0) {
    // empty kept set (reported by the slot-count kernel) or an empty split:
    // rows are zero (partials: zero with log-sum -inf)
    if (static_cast<int>(threadIdx.x) < rows_unit) {
      for (int o2 = 0; o2 < (DUAL ? 2 : 1); ++o2) {
        float* op = o2 ? p.opart2 : p.opart;
        float* lp = o2 ? p.lpart2 : p.lpart;
        float* ls = o2 ? p.lse2 : p.lse;
        float* o = partial ? op + (pbase + threadIdx.x) * HD
                           : (o2 ? p.out2 : p.out) + (static_cast<size_t>(h) * p.q_rows + row0 + threadIdx.x) * HD;
        for (int c = 0; c < HD; c += 4) *reinterpret_cast<float4*>(o + c) = make_float4(0, 0, 0, 0);
        if (partial) lp[pbase + threadIdx.x] = -INFINITY;
        else if (ls) ls[static_cast<size_t>(h) * p.q_rows + row0 + threadIdx.x] = -INFINITY;
      }
    }
    return;
  }
  // tasks (query tile, key tile) of warpgroup i: two tiles -> (i, t) for every
  // key tile t; one tile -> (0, 2t + i)
  const bool two = DUAL || (nq == 2);  // both warpgroups take every key tile
  const int ntask[2] = {two ? T : (T + 1) / 2, two ? T : T / 2};

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* Qs = smem + L::q_off;
  uint8_t* Ks = smem + L::k_off;
  uint8_t* Vs = smem + L::v_off;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::bar_off);
  float* ml = reinterpret_cast<float*>(smem + L::ml_off);
  int2* runs_s = reinterpret_cast<int2*>(smem + L::runs_off);
  // run-list capacity left in the dynamic allocation after alignment
  const int cap = (kAttnSmemBytes - static_cast<int>(smem - smem_raw) - L::runs_off) / 8;
  const int2* runs_g = p.runs + gi * (p.kmax + 1);
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
      mbar_init(&bars->p_full[b], kTileM);
      mbar_init(&bars->o_done[b], 1);
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

  if (warp == 8 || warp == 10) {
    // ------- TMA producers: warp 8 streams Q once and the K tiles, warp 10
    // the V tiles, each through its own ring. Lane s (and s + 16) finds the
    // first row of slot s of a tile; a tile whose slots are all contiguous is
    // fetched as one 128-row box, any other tile slot by slot (8-row boxes,
    // lanes 0-15 in parallel). -------
    const bool is_k = (warp == 8);
    const int krow_base = h * p.N;
    if (is_k && lane == 0) {
      mbar_arrive_expect_tx(&bars->q_full, nq * kAtoms * p.q_box_rows * 128);
      for (int qt = 0; qt < nq; ++qt)
        for (int a = 0; a < kAtoms; ++a)
          tma_load_2d(Qs + qt * L::kQBytes + a * L::kSlab, &maps.q, &bars->q_full, a * 64,
                      h * p.q_rows + row0 + qt * kTileM);
    }
    const int sl = lane & (kSlotsPerTile - 1);
    auto run_slots = [&](int r) { return (runs[r].y + kSlotRows - 1) / kSlotRows; };
    // run holding the first slot of this CTA's key range, and that run's first slot
    int rb = 0, cb = 0;
    {
      const int t0 = j0 * kSlotsPerTile;
      while (rb < nr && t0 >= cb + run_slots(rb)) {
        cb += run_slots(rb);
        ++rb;
      }
    }
    uint8_t* ring = is_k ? Ks : Vs;
    uint64_t* full = is_k ? bars->kfull : bars->vfull;
    uint64_t* empty = is_k ? bars->kempty : bars->vempty;
    const CUtensorMap* map_slot = is_k ? &maps.k[0] : &maps.v[0];
    const CUtensorMap* map_tile = is_k ? &maps.k[4] : &maps.v[4];
    int issued = -1;
    const bool big_box = p.max_lg == 4;  // the tensor holds at least one 128-row box
    for (int j = 0; j < T; ++j) {
      const int t = (j0 + j) * kSlotsPerTile + sl;
      int r = rb, c = cb;
      while (r < nr && t >= c + run_slots(r)) {
        c += run_slots(r);
        ++r;
      }
      // past the last run: any rows of the head (masked)
      const int row = (r < nr) ? runs[r].x + (t - c) * kSlotRows : 0;
      rb = __shfl_sync(0xffffffffu, r, kSlotsPerTile - 1);  // runs ascend: the next tile starts here
      cb = __shfl_sync(0xffffffffu, c, kSlotsPerTile - 1);
      const int prev = __shfl_up_sync(0xffffffffu, row, 1);
      const bool follows = lane == 0 || lane >= kSlotsPerTile || row == prev + kSlotRows;
      const bool whole = big_box && __all_sync(0xffffffffu, follows);
      const int row_first = __shfl_sync(0xffffffffu, row, 0);
      const int st = j % kStages;
      bool w = true;
      if (lane == 0 && j >= kStages) w = mbar_wait(&empty[st], ((j / kStages) + 1) & 1, abort);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      if (lane == 0) mbar_arrive_expect_tx(&full[st], L::kKVBytes);
      __syncwarp();
      if (whole) {
        if (lane == 0)
          for (int a = 0; a < kAtoms; ++a)
            tma_load_2d(ring + st * L::kKVBytes + a * L::kSlab, map_tile, &full[st], a * 64,
                        krow_base + row_first);
      } else if (lane < kSlotsPerTile) {
        for (int a = 0; a < kAtoms; ++a)
          tma_load_2d(ring + st * L::kKVBytes + a * L::kSlab + sl * 1024, map_slot, &full[st],
                      a * 64, krow_base + row);
      }
      issued = j;
    }
    // let the loads already in flight land before the CTA exits
    if (lane == 0) {
      volatile int never = 0;
      for (int j = max(0, issued - kStages + 1); j <= issued; ++j)
        mbar_wait(&full[j % kStages], (j / kStages) & 1, &never);
      if (is_k) mbar_wait(&bars->q_full, 0, &never);
    }
  } else if (warp == 9) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kTileM, kTileN, 0);
      constexpr uint32_t idO = idesc_bf16(kTileM, HD, 1);
      const uint32_t q_addr = smem_u32(Qs), k_addr = smem_u32(Ks), v_addr = smem_u32(Vs);
      bool ok = mbar_wait(&bars->q_full, 0, abort);
      auto kv_of = [&](int i, int t) { return two ? t : 2 * t + i; };
      // S_i = Q_(tile of i) K(kv)^T
      auto issue_s = [&](int i, int t) -> bool {
        const int kv = kv_of(i, t), st = kv % kStages;
        if (!mbar_wait(&bars->kfull[st], (kv / kStages) & 1, abort)) return false;
        tc_fence_after();
        const uint32_t qa = q_addr + ((two && !DUAL) ? i : 0) * L::kQBytes;  // dual: one Q tile
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(i * kTileN);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint32_t off = static_cast<uint32_t>((ks >> 2) * L::kSlab + (ks & 3) * 32);
          const uint64_t ad = smem_desc_sw128(qa + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + st * L::kKVBytes + off, 16, 1024);
          mma_bf16_ss(d_tmem, ad, bd, idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[i]);
        if (!two || i == 1) mma_commit(&bars->kempty[st]);  // last reader of K(kv)
        return true;
      };
      // O_i += P_i V(kv), P_i from tensor memory
      auto issue_pv = [&](int i, int t) -> bool {
        const int kv = kv_of(i, t), st = kv % kStages;
        if (!mbar_wait(&bars->p_full[i], t & 1, abort)) return false;
        if (!mbar_wait(&bars->vfull[st], (kv / kStages) & 1, abort)) return false;
        tc_fence_after();
        const uint32_t o_tmem = tmem + 2u * kTileN + static_cast<uint32_t>(i * HD);
        const uint32_t p_tmem = tmem + static_cast<uint32_t>(i * kTileN);
#pragma unroll
        for (int ks = 0; ks < kTileN / 16; ++ks) {
          const uint64_t bd =
              smem_desc_sw128(v_addr + st * L::kKVBytes + ks * 16 * 128, L::kSlab, 1024);
          mma_bf16_ts(o_tmem, p_tmem + static_cast<uint32_t>(ks * 8), bd, idO,
                      (t > 0 || ks > 0) ? 1u : 0u);
        }
        if (!two || i == 1) mma_commit(&bars->vempty[st]);  // last reader of V(kv)
        if (t == ntask[i] - 1) mma_commit(&bars->o_done[i]);
        return true;
      };
      for (int i = 0; i < 2 && ok; ++i)
        if (ntask[i] > 0) ok = issue_s(i, 0);
      const int nt = max(ntask[0], ntask[1]);
      for (int t = 0; t < nt && ok; ++t)
        for (int i = 0; i < 2 && ok; ++i) {
          if (t >= ntask[i]) continue;
          ok = issue_pv(i, t);
          if (ok && t + 1 < ntask[i]) ok = issue_s(i, t + 1);
        }
      // all issued MMAs complete before the CTA releases tensor memory
      mma_commit(&bars->mma_idle);
      volatile int never = 0;
      mbar_wait(&bars->mma_idle, 0, &never);
    }
  } else {
    // ------------- softmax: warpgroup i = warp / 4, thread = row -------------
    const int i = warp >> 2;
    const int row = (warp & 3) * 32 + lane;  // 0..127 == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(((warp & 3) * 32) << 16);
    const uint32_t s_tmem = tmem + lane_base + static_cast<uint32_t>(i * kTileN);
    const uint32_t o_base = tmem + lane_base + 2u * kTileN;
    const float sc = p.sc;
    float m_ref = -INFINITY, l_sum = 0.f;
    MaskWalk mw;
    mw.init(runs, nr, ns);
    mw.advance_to(j0);
    // dual pass, warpgroup 1: this row's keys are its query group's kept runs
    // (key tile j covers keys [128 j, 128 j + 128) in the dense pass)
    const bool kmask = DUAL && i == 1;
    const int2* gr = nullptr;
    int gnr = 0, gri = 0;
    if (kmask && row < rows_unit) {
      const size_t gg = static_cast<size_t>(h) * p.gCq + p.pgrp[static_cast<size_t>(h) * p.q_rows + row0 + row];
      gr = p.gruns + gg * (p.gkmax + 1);
      gnr = p.gnruns[gg];
    }
    bool ok = true;
    for (int t = 0; t < ntask[i]; ++t) {
      const int kv = two ? t : 2 * t + i;  // local key tile; global tile j0 + kv
      uint32_t vm[4];
      if (!two && i == 1) {
        uint32_t skip[4];
        mw.tile(j0 + kv - 1, skip);  // advance past the other warpgroup's tile
      }
      mw.tile(j0 + kv, vm);
      if (!two && i == 0 && kv + 1 < T) {
        uint32_t skip[4];
        mw.tile(j0 + kv + 1, skip);
      }
      uint32_t km[4] = {0u, 0u, 0u, 0u};  // dual: bit c = key column c is kept for this row
      if (kmask) {
        const int k0 = (j0 + kv) * kTileN, k1 = k0 + kTileN;
        while (gri < gnr && gr[gri].x + gr[gri].y <= k0) ++gri;
        for (int r2 = gri; r2 < gnr && gr[r2].x < k1; ++r2) {
          const int a = max(gr[r2].x, k0) - k0, b = min(gr[r2].x + gr[r2].y, k1) - k0;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int lo = max(a, 32 * w) - 32 * w, hi = min(b, 32 * w + 32) - 32 * w;
            if (lo < hi) km[w] |= (hi == 32 ? 0xFFFFFFFFu : ((1u << hi) - 1u)) & ~((1u << lo) - 1u);
          }
        }
      }
      // tcgen05.ld / st below are warp-collective: the warp proceeds or stops as one
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[i], t & 1, abort))) { ok = false; break; }
      tc_fence_after();
      // The row is processed in two halves of 64 key columns: S half hf is
      // loaded, exponentiated and packed, and its P stored over columns
      // [32 hf, 32 hf + 32) of S_i, columns that hold S values already read.
      uint32_t r[kTileN / 2];
      auto load_half = [&](int hf) {
        tmem_ld32(s_tmem + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(r));
        tmem_ld32(s_tmem + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
        tmem_wait_ld();
        if (kmask) {
#pragma unroll
          for (int c = 0; c < kTileN / 2; ++c)
            if (!((km[2 * hf + (c >> 5)] >> (c & 31)) & 1u)) r[c] = __float_as_uint(-INFINITY);
        }
        if ((vm[2 * hf] & vm[2 * hf + 1]) != 0xFFFFFFFFu) {
          // only partial or padding slots (the same for every row) are touched
#pragma unroll
          for (int sl = 0; sl < kSlotsPerTile / 2; ++sl) {
            const uint32_t b = (vm[2 * hf + (sl >> 2)] >> ((sl & 3) * 8)) & 0xFFu;
            if (b != 0xFFu) {
#pragma unroll
              for (int q = 0; q < kSlotRows; ++q)
                if (!((b >> q) & 1u)) r[sl * kSlotRows + q] = __float_as_uint(-INFINITY);
            }
          }
        }
      };
      // scaled maximum of the loaded half: eight chains of three-input maxima
      auto half_max = [&]() -> float {
        float m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = __uint_as_float(r[k]);
#pragma unroll
        for (int c = 8; c < kTileN / 2; c += 2)
          m8[(c >> 1) & 7] = max3f(m8[(c >> 1) & 7], __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
        return sc * fmaxf(max3f(m8[0], m8[1], m8[2]),
                          fmaxf(max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      };
      // P = 2^(s sc - m_ref) of the loaded half as bf16 pairs; returns its sum
      uint32_t pk[32];
      auto exp_half = [&](float mref) -> float {
        float2 r4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        const float nm = (mref == -INFINITY) ? 0.f : -mref;  // no kept key yet: P = 0
#pragma unroll
        for (int c = 0; c < kTileN / 2; c += 2) {
          float xa, xb;
          fma2(xa, xb, __uint_as_float(r[c]), __uint_as_float(r[c + 1]), sc, nm);
          const float a = ex2_approx(xa), b = ex2_approx(xb);
          add2(r4[(c >> 1) & 3], a, b);
          pk[c >> 1] = pack_bf16x2(a, b);
        }
        return (r4[0].x + r4[0].y + r4[1].x + r4[1].y) + (r4[2].x + r4[2].y + r4[3].x + r4[3].y);
      };
      // Reference maximum m_ref: the first tile's row maximum; later tiles
      // are exponentiated against it with no maximum pass. A half whose sum
      // exceeds 2^32 (some value may exceed 2^32, or overflowed) moves the
      // reference up by the whole number k of log2 units that brings its
      // largest value to at most 1: its S is reloaded (P not yet stored over
      // it) and its values formed again, and the P half already stored, the
      // row sum and O are scaled by 2^-k, exactly. O and the row sum always
      // share one reference, so the result is exact.
      // (dual, masked rows: the first tile that holds one of the row's keys;
      // nothing has been accumulated before it)
      if (t == 0 || (kmask && __any_sync(0xffffffffu, m_ref == -INFINITY))) {
        load_half(0);
        const float m0 = half_max();
        load_half(1);
        const float mt = fmaxf(m0, half_max());
        if (m_ref == -INFINITY) m_ref = mt;
      }
      float alpha = 1.f, rs = 0.f;
      bool need = false;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        load_half(hf);
        float rh = exp_half(m_ref);
        if (__any_sync(0xffffffffu, !(rh <= kOverflowSum))) {
          const bool over = !(rh <= kOverflowSum);
          load_half(hf);
          float sh = 1.f;  // 2^-k, formed from its bits (0 when k >= 127)
          if (over) {
            const float k = ceilf(half_max() - m_ref);
            sh = (k < 127.f) ? __int_as_float((127 - static_cast<int>(k)) << 23) : 0.f;
            m_ref += k;
            need = true;
          }
          alpha *= sh;
          rs *= sh;
          if (hf == 1 && __any_sync(0xffffffffu, sh != 1.f)) {
            // the stored P half 0 follows the new reference (exact: a power of two)
            uint32_t q[32];
            tmem_ld32(s_tmem, q);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c)
              q[c] = pack_bf16x2(__uint_as_float(q[c] << 16) * sh, __uint_as_float(q[c] & 0xFFFF0000u) * sh);
            tmem_st32(s_tmem, q);
          }
          rh = exp_half(m_ref);
        }
        tmem_st32(s_tmem + hf * 32, pk);
        rs += rh;
      }
      if (__any_sync(0xffffffffu, need)) {
        // P_i(t-1) V has completed (it precedes S_i(t)); O_i is not read again
        // before P_i(t) is published below
        const uint32_t o_tmem = o_base + static_cast<uint32_t>(i * HD);
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_tmem + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(o_tmem + c * 32, o);
        }
      }
      l_sum = l_sum * alpha + rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[i]);
    }
    // ---------------- epilogue: O / l -> global (fp32, group-major rows) ------
    if (two) {
      if (__all_sync(0xffffffffu, ok && mbar_wait(&bars->o_done[i], 0, abort))) {
        tc_fence_after();
        // a row with no kept key in this range (dual pass) gets 0 and -inf
        const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
        const float lsev = l_sum > 0.f ? m_ref + __log2f(l_sum) : -INFINITY;
        const uint32_t o_tmem = o_base + static_cast<uint32_t>(i * HD);
        const int ur = DUAL ? row : i * kTileM + row;  // row within the unit
        const bool valid = ur < rows_unit;
        const bool second = DUAL && i == 1;
        float* orow = partial ? (second ? p.opart2 : p.opart) + (pbase + ur) * HD
                              : (second ? p.out2 : p.out) + (static_cast<size_t>(h) * p.q_rows + row0 + ur) * HD;
        if (partial && valid) (second ? p.lpart2 : p.lpart)[pbase + ur] = lsev;
        float* lsep = second ? p.lse2 : p.lse;
        if (!partial && valid && lsep) lsep[static_cast<size_t>(h) * p.q_rows + row0 + ur] = lsev;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_tmem + c * 32, o);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<float4*>(orow + c * 32 + k) =
                  make_float4(__uint_as_float(o[k]) * inv, __uint_as_float(o[k + 1]) * inv,
                              __uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
          }
        }
      }
    } else {
      // merge the two halves of the key tiles: each warpgroup writes half of
      // the columns of every row
      ml[i * 2 * kTileM + row] = m_ref;
      ml[i * 2 * kTileM + kTileM + row] = l_sum;
      named_barrier_sync(1, 2 * kTileM);
      const float m0 = ml[row], l0 = ml[kTileM + row];
      const float m1 = ml[2 * kTileM + row], l1 = ml[3 * kTileM + row];
      const bool has1 = ntask[1] > 0;
      const float mm = has1 ? fmaxf(m0, m1) : m0;
      const float a0 = ex2_approx(m0 - mm), a1 = has1 ? ex2_approx(m1 - mm) : 0.f;
      const float inv = 1.f / (l0 * a0 + l1 * a1);
      const float f0 = a0 * inv, f1 = a1 * inv;
      ok = ok && mbar_wait(&bars->o_done[0], 0, abort);
      if (has1) ok = ok && mbar_wait(&bars->o_done[1], 0, abort);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const bool valid = row < rows_unit;
        float* orow = partial ? p.opart + (pbase + row) * HD
                              : p.out + (static_cast<size_t>(h) * p.q_rows + row0 + row) * HD;
        if (partial && valid && i == 0) p.lpart[pbase + row] = mm + __log2f(l0 * a0 + l1 * a1);
        if (!partial && valid && i == 0 && p.lse)
          p.lse[static_cast<size_t>(h) * p.q_rows + row0 + row] = mm + __log2f(l0 * a0 + l1 * a1);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c) {
          const int col = i * (HD / 2) + c * 32;
          uint32_t o0[32], o1[32];
          tmem_ld32(o_base + col, o0);
          if (has1) tmem_ld32(o_base + HD + col, o1);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int k = 0; k < 32; k += 4) {
              float4 v;
              v.x = __uint_as_float(o0[k]) * f0 + (has1 ? __uint_as_float(o1[k]) * f1 : 0.f);
              v.y = __uint_as_float(o0[k + 1]) * f0 + (has1 ? __uint_as_float(o1[k + 1]) * f1 : 0.f);
              v.z = __uint_as_float(o0[k + 2]) * f0 + (has1 ? __uint_as_float(o1[k + 2]) * f1 : 0.f);
              v.w = __uint_as_float(o0[k + 3]) * f0 + (has1 ? __uint_as_float(o1[k + 3]) * f1 : 0.f);
              *reinterpret_cast<float4*>(orow + col + k) = v;
            }
          }
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
// Work list: one entry per unit (256 rows; 128 in the dual probe pass) of
// each query group, (g << 16) | u.
// One warp per head: tile counts are prefix-summed 32 groups at a time.
// ---------------------------------------------------------------------------
__global__ void work_list_kernel(const int32_t* off_q, int Cq, int tiles_per_head, int unit_rows,
                                 int32_t* work, int32_t* nwork) {
  const int h = blockIdx.x, lane = threadIdx.x;
  const int32_t* oq = off_q + static_cast<size_t>(h) * (Cq + 1);
  int32_t* wl = work + static_cast<size_t>(h) * tiles_per_head;
  int32_t base = 0;
  for (int g0 = 0; g0 < Cq; g0 += 32) {
    const int g = g0 + lane;
    const int n = (g < Cq) ? oq[g + 1] - oq[g] : 0;
    const int t = n > 0 ? (n + unit_rows - 1) / unit_rows : 0;
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
// kernel walks), and the exact routed pair count per head. With text tokens
// (text = 1) the last query group keeps every key and every other group
// also keeps the last key group (the text tokens), outside its budget.
// One warp per (head, query group), lanes over the kept key groups: a kept
// group starts a run unless its keys begin where the previous kept group's
// end, and ends it unless the next one begins where it ends; runs of no
// keys are then dropped in order.
constexpr int kSpWarps = 8;

__global__ void __launch_bounds__(kSpWarps * 32)
    slots_pairs_kernel(const int32_t* off_q, const int32_t* off_k, const int32_t* csr,
                       const int32_t* kh, int H, int N, int Cq, int Ck, int kmax, int text,
                       int32_t* nslots, int2* runs, int32_t* nruns, int64_t* pairs,
                       DeviceStats* stats) {
  const int i = blockIdx.x * kSpWarps + static_cast<int>(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= H * Cq) return;  // the whole warp
  const int h = i / Cq, g = i % Cq;
  const int Cqv = Cq - text, Ckv = Ck - text;  // routed (video) groups
  const int32_t* oq = off_q + static_cast<size_t>(h) * (Cq + 1);
  const int32_t* ok = off_k + static_cast<size_t>(h) * (Ck + 1);
  int2* rout = runs + static_cast<size_t>(i) * (kmax + 1);
  const int64_t nq = oq[g + 1] - oq[g];
  bool valid = (ok[0] >= 0 && ok[Ck] <= N && nq >= 0);
  long long keys = 0;
  int slots = 0, nr = 0;
  if (text && g == Cqv) {
    if (valid && N > 0) {  // the text query group: every key
      if (lane == 0) rout[0] = make_int2(0, N);
      nr = 1;
      slots = (N + kSlotRows - 1) / kSlotRows;
      keys = N;
    }
  } else {
    const int32_t* row = csr + (static_cast<size_t>(h) * Cqv + g) * kmax;
    const int k = kh[h];
    valid = valid && k >= 0 && k <= kmax;
    // reject malformed routes before the attention kernel walks them
    if (valid)
      for (int ci = lane; ci < k; ci += 32) {
        const int c = row[ci];
        valid = valid && (c >= 0 && c < Ckv && ok[c] >= 0 && ok[c] <= ok[c + 1]);
      }
    valid = __all_sync(0xffffffffu, valid);
    if (valid) {
      for (int b0 = 0; b0 < k; b0 += 32) {
        const int ci = b0 + lane;
        bool start = false, last = false;
        int lo = 0, hi = 0;
        if (ci < k) {
          const int c = row[ci];
          lo = ok[c];
          hi = ok[c + 1];
          start = ci == 0 || ok[row[ci - 1] + 1] != lo;
          last = ci == k - 1 || ok[row[ci + 1]] != hi;
          keys += hi - lo;
        }
        const unsigned sb = __ballot_sync(0xffffffffu, start);
        const int r = nr + __popc(sb & ((2u << lane) - 1u)) - 1;  // this group's run
        if (start) rout[r].x = lo;
        if (last) rout[r].y = hi;  // the run's end, for now
        nr += __popc(sb);
      }
      __syncwarp();
      int kept = 0;  // lengths; runs without keys dropped in order
      for (int b0 = 0; b0 < nr; b0 += 32) {
        const int r = b0 + lane;
        int2 v = make_int2(0, 0);
        if (r < nr) {
          v = rout[r];
          v.y -= v.x;
        }
        const bool keep = r < nr && v.y > 0;
        const unsigned kb = __ballot_sync(0xffffffffu, keep);
        __syncwarp();  // the chunk is read before any of it is rewritten
        if (keep) {
          rout[kept + __popc(kb & ((1u << lane) - 1u))] = v;
          slots += (v.y + kSlotRows - 1) / kSlotRows;
        }
        kept += __popc(kb);
      }
      nr = kept;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        slots += __shfl_xor_sync(0xffffffffu, slots, o);
        keys += __shfl_xor_sync(0xffffffffu, keys, o);
      }
      __syncwarp();
      if (text && lane == 0) {  // the text key group, merged into the last run when adjacent
        const int lo = ok[Ckv], hi = ok[Ckv + 1];
        if (hi > lo) {
          if (nr > 0 && rout[nr - 1].x + rout[nr - 1].y == lo) {
            const int plen = rout[nr - 1].y;
            slots -= (plen + kSlotRows - 1) / kSlotRows;
            rout[nr - 1].y = plen + (hi - lo);
            slots += (rout[nr - 1].y + kSlotRows - 1) / kSlotRows;
          } else {
            rout[nr++] = make_int2(lo, hi - lo);
            slots += (hi - lo + kSlotRows - 1) / kSlotRows;
          }
          keys += hi - lo;
        }
      }
    }
  }
  if (lane != 0) return;
  if (!valid) {
    nslots[i] = 0;
    nruns[i] = 0;
    raise_status(stats, SPARSEPR_ERR_INVALID_ARG);
    return;
  }
  nslots[i] = slots;
  nruns[i] = nr;
  if (pairs && nq > 0) atomicAdd(reinterpret_cast<unsigned long long*>(&pairs[h]),
                                 static_cast<unsigned long long>(nq * keys));
  if (nq > 0 && keys == 0) raise_status(stats, SPARSEPR_ERR_NUMERIC);
}

// Split-KV combine: out = sum_s 2^(l_s - L) O_s / sum_s 2^(l_s - L),
// L = max_s l_s, over the splits' normalised partial outputs O_s and
// log2-sum-exps l_s (fixed order over the splits). Block = 8 rows of one
// unit, thread = (row, 4 columns).
__global__ void split_combine_kernel(const float* opart, const float* lpart, const int32_t* off_q,
                                     const int32_t* work, const int32_t* nwork, int Cq,
                                     int tiles_per_head, int units, int splits, int unit_rows,
                                     int q_rows, int d, float* out, float* lse) {
  const int h = blockIdx.z, wi = blockIdx.y;
  if (wi >= nwork[h]) return;
  const int wcode = work[static_cast<size_t>(h) * tiles_per_head + wi];
  const int g = wcode >> 16, tu = wcode & 0xFFFF;
  const int32_t* offq = off_q + static_cast<size_t>(h) * (Cq + 1);
  const int row0 = offq[g] + tu * unit_rows;
  const int rows = min(unit_rows, offq[g + 1] - row0);
  const int cpr = d / 4;  // threads per row
  const int r = blockIdx.x * (blockDim.x / cpr) + threadIdx.x / cpr;
  const int c = (threadIdx.x % cpr) * 4;
  if (r >= rows) return;
  const size_t ub = (static_cast<size_t>(h) * units + wi) * splits;
  float L = -INFINITY;
  for (int s = 0; s < splits; ++s) L = fmaxf(L, lpart[(ub + s) * unit_rows + r]);
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ls = lpart[(ub + s) * unit_rows + r];
    if (ls == -INFINITY) continue;
    const float wgt = exp2f(ls - L);
    const float4 o = *reinterpret_cast<const float4*>(opart + ((ub + s) * unit_rows + r) * d + c);
    num.x = fmaf(wgt, o.x, num.x);
    num.y = fmaf(wgt, o.y, num.y);
    num.z = fmaf(wgt, o.z, num.z);
    num.w = fmaf(wgt, o.w, num.w);
    den += wgt;
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  *reinterpret_cast<float4*>(out + (static_cast<size_t>(h) * q_rows + row0 + r) * d + c) =
      make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
  if (lse && c == 0)
    lse[static_cast<size_t>(h) * q_rows + row0 + r] = den > 0.f ? L + __log2f(den) : -INFINITY;
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
// 2D bf16 map over [rows, d] with a box of 64 columns x box_rows rows,
// 128-byte swizzle; rows past the end read as zero.
bool make_map(CUtensorMap* m, const void* base, size_t rows, int d, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
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

template <int HD, bool DUAL>
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
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<HD, DUAL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, shb);
  if (e != cudaSuccess) return e;
  dim3 grid(a.tiles_per_head * prm.splits, a.H);
  sparse_attn_kernel<HD, DUAL><<<grid, kAttnThreads, shb, st>>>(maps, prm);
  if (prm.splits > 1) {
    const dim3 cg(prm.unit_rows / (256 / (HD / 4)), a.units, a.H);
    split_combine_kernel<<<cg, 256, 0, st>>>(a.opart, a.lpart, a.off_q, a.work, a.nwork, a.Cq,
                                             a.tiles_per_head, a.units, prm.splits, prm.unit_rows,
                                             a.q_rows, HD, a.out, a.lse);
    if (DUAL)
      split_combine_kernel<<<cg, 256, 0, st>>>(a.opart2, a.lpart2, a.off_q, a.work, a.nwork, a.Cq,
                                               a.tiles_per_head, a.units, prm.splits,
                                               prm.unit_rows, a.q_rows, HD, a.out2, a.lse2);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_meta(const AttnArgs& a, cudaStream_t st) {
  const int unit_rows = a.dual ? kTileM : kUnitRows;
  work_list_kernel<<<a.H, 32, 0, st>>>(a.off_q, a.Cq, a.tiles_per_head, unit_rows, a.work, a.nwork);
  if (a.pairs) zero_i64_kernel<<<(a.H + 127) / 128, 128, 0, st>>>(a.pairs, a.H);
  const int n = a.H * a.Cq;
  slots_pairs_kernel<<<(n + kSpWarps - 1) / kSpWarps, kSpWarps * 32, 0, st>>>(
      a.off_q, a.off_k, a.csr, a.kh, a.H, a.N, a.Cq, a.Ck, a.kmax, a.text, a.nslots, a.runs,
      a.nruns, a.pairs, a.stats);
  if (a.pairs) pairs_to_stats_kernel<<<(a.H + 127) / 128, 128, 0, st>>>(a.pairs, a.H, a.stats);
  return cudaGetLastError();
}

cudaError_t launch_attn_kernel(const AttnArgs& a, cudaStream_t st) {
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
  prm.splits = a.splits > 1 ? a.splits : 1;
  prm.units = a.units;
  prm.opart = a.opart;
  prm.lpart = a.lpart;
  prm.lse = a.lse;
  prm.unit_rows = a.dual ? kTileM : kUnitRows;
  prm.out2 = a.out2;
  prm.opart2 = a.opart2;
  prm.lpart2 = a.lpart2;
  prm.lse2 = a.lse2;
  prm.pgrp = a.pgrp;
  prm.gruns = a.gruns;
  prm.gnruns = a.gnruns;
  prm.gCq = a.gCq;
  prm.gkmax = a.gkmax;
  if (prm.splits > 1 && (!a.opart || !a.lpart || a.units < 1)) return cudaErrorInvalidValue;
  if (a.dual && (!a.out2 || !a.pgrp || !a.gruns || !a.gnruns || a.gCq < 1 ||
                 (prm.splits > 1 && (!a.opart2 || !a.lpart2))))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.d == 128) return a.dual ? launch_attn_hd<128, true>(a, prm, st) : launch_attn_hd<128, false>(a, prm, st);
  if (a.d == 64) return a.dual ? launch_attn_hd<64, true>(a, prm, st) : launch_attn_hd<64, false>(a, prm, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_block_sparse_attn(const AttnArgs& a, cudaStream_t st) {
  const cudaError_t e = launch_attn_meta(a, st);
  if (e != cudaSuccess) return e;
  return launch_attn_kernel(a, st);
}

cudaError_t launch_cast_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t st) {
  const size_t threads = (n + 3) / 4;
  cast_bf16_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(src, dst, n);
  return cudaGetLastError();
}

}  // namespace spr
