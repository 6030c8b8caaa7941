// Workspace layout of the SparsePR library. The caller passes one device
// buffer `ws`; every call carves the same regions out of it, at offsets that
// depend only on the parameters. Regions are 256-byte aligned.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/sparsepr.h"

namespace spr {

using DeviceStats = sparsepr_stats;

constexpr int kTileM = 128;     // query rows per attention tile
constexpr int kTileN = 128;     // keys per attention KV tile
constexpr int kSlotRows = 8;    // keys per TMA row-slot of a KV tile
constexpr int kSortChunk = 1024;  // tokens per counting-sort chunk
constexpr int kMaxGroups = 4096;
constexpr int kMaxSplits = 8;   // split-KV ranges of the dense probe pass
constexpr size_t kMaxDynSmem = 232448;  // dynamic shared memory per block on sm_100
constexpr int kDiagRows = 64;   // density-profile rows processed at once (one CTA each)
constexpr int kTriEigMax = 64;  // eigenpairs of the tridiagonal solver (more: cyclic Jacobi)
constexpr int kGramJobs = 3;    // Grams of one launch (the probe fit forms three)
constexpr int kGramSplits = 4;  // sample ranges of a Gram, summed in order afterwards

struct Layout {
  // statistics / status (always at offset 0)
  size_t stats;
  // stage 1
  size_t fy;       // [H, Nv] int32 Fisher-Yates scratch
  size_t init_k;   // [H, Ck] int32
  size_t init_q;   // [H, Cq] int32
  size_t mk;       // [H, d, d] f64 (M_K, later the probe residual Gram R^T R)
  size_t evec;     // [H, d, d] f64 Jacobi eigenvectors (columns)
  size_t eval;     // [H, d] f64 Jacobi eigenvalues
  size_t eigscr;   // tridiagonal eigensolver scratch: [H, d*d + 3d] f64
  size_t wk;       // [H, d, e] f64 key projector U_e L_e^{1/2}
  size_t z;        // [H, Nv, e] f64 key coordinates
  size_t mu;       // [H, Ck, e] f64 key centroids
  size_t munorm;   // [H, Ck] f64 squared centroid norms
  size_t lab_k;    // [H, Nv] int32
  size_t lab_q;    // [H, Nv] int32
  size_t flags;    // [H, 4] int32: changes_k, done_k, changes_q, done_q
  size_t hist;     // [H, nchunk, Cmax] int32 counting-sort chunk histograms
  size_t sortoff;  // [H, Cmax + 1] int32
  size_t sortperm; // [H, Nv] int32
  size_t ck;       // [H, Ck, d] f64 K/V group centroids
  size_t g;        // [H, d, d] f64 query metric G
  size_t qbar;     // [H, Cq, d] f64 query centroids
  size_t wg;       // [H, Cq, d] f64 G * qbar
  size_t cg;       // [H, Cq] f64 qbar^T G qbar
  // tensor-core assignment operands
  size_t zplanes;  // [3][H * Nv][Dpk] bf16 planes of z
  size_t xnk;      // [H, Nv] f32 |z|
  size_t xnq;      // [H, Nv] f32 |q|
  size_t muplanes; // [3][H * CpadK][Dpk] bf16
  size_t cfk;      // [H, CpadK] f32
  size_t hmk;      // [H, 2] f32
  size_t wplanes;  // [3][H * CpadQ][d] bf16
  size_t cfq;      // [H, CpadQ] f32
  size_t hmq;      // [H, 2] f32
  size_t recheck;  // [H, Nv] int32
  size_t nrecheck; // [H] int32
  size_t ytr;      // [H, D, m] f64 centroid side, transposed, for the fp64 decisions
                   // (keys: D = e, m = Ck; queries: D = d, m = Cq)
  // stage 3
  size_t cq;       // [H, Cq, d] f64 query-group means (route)
  size_t ckr;      // [H, Ck, d] f64 key-group means (route)
  size_t scores;   // [heads per pass, Cq, Ck] f64 block scores (route)
  size_t bf16_qkv; // [3, H, N, d] bf16 copies (fp32 inputs only)
  size_t work;     // [H, tiles_per_head] int32 attention work list
  size_t nwork;    // [H] int32
  size_t nslots;   // [H, Cqt] int32 KV row-slots per query group
  size_t runs;     // [H, Cqt, kmax + 1] int2 merged kept key runs (start, length)
  size_t nruns;    // [H, Cqt] int32
  // stage 4
  size_t probe_q;  // [H, M, d] bf16 gathered probe rows (group-major)
  size_t od;       // [H, M, d] f32 dense outputs of the probes
  size_t xr;       // [H, 2, M, d] f64: X = O_sparse[probes], R = O_dense - X
  size_t means;    // [H, 2, d] f64: xbar, rbar
  size_t gram;     // [H, 2, d, d] f64: Xc^T Xc + lam I, Xc^T Rc
  size_t gpart;    // [kGramJobs, H, kGramSplits, d, d] f64: partial Gram sums
  size_t bmat;     // [H, d, d] f64 ridge solution B
  size_t bvec;     // [H, d] f64 intercept b
  size_t bp32;     // [H, d, d] f32 projected B'
  size_t bv32;     // [H, d] f32 projected b'
  size_t pwork;    // [H, M/128 + 1] int32 probe attention work list
  size_t pnwork;   // [H] int32
  size_t pmeta;    // [H, 12] int32: dense-mode off_q(2), off_k(2), csr(1), k(1), nslots(1),
                   // nruns(1), runs(2 int2: run-list stride kmax + 1 = 2)
  size_t opart;    // [H, punits, kMaxSplits, 256, d] f32 split-KV partial outputs (probes)
  size_t lpart;    // [H, punits, kMaxSplits, 256] f32 split-KV log2-sum-exps
  size_t opart2;   // [H, punits, kMaxSplits, 256, d] f32: partial sparse outputs of the dual pass
  size_t lpart2;   // [H, punits, kMaxSplits, 256] f32
  size_t xp;       // [H, M + 1, d] f32 sparse outputs of the probe rows (dual pass)
  size_t pgrp;     // [H, M + 1] int32 query group of each probe row
  size_t lse_s;    // [H, N] f32 log2-sum-exp of each row's kept logits (sparse pass, group-major)
  size_t lse_d;    // [H, M + 1] f32 log2-sum-exp of each probe row over all keys (dense pass)
  size_t diag;     // [H, M + 1, 4] f64 per-probe-row residual energies (diagnostics)
  size_t pkbar;    // co-clustering: [H, Ck, Cq] f64 mean affinity vector of each key block
  size_t pqbar;    // co-clustering: [H, Cq, Ck] f64 mean affinity vector of each query block
  size_t cnt;      // [H, Ck + Cq] int32 members per key / query block (alternative partitions)
  size_t dscr;     // diagnostics scratch: support union bits [H, Cq, ceil(Ckt/32)] u32 and
                   // size sums [H, Cq] u64; or density weights [kDiagRows, N] f64 and counts [H]
  size_t total;

  int Nv, e, Cmax, nchunk, tiles_per_head, kmax;
  int Ckt, Cqt;    // groups including the text group (n_text > 0: Ck + 1, Cq + 1)
  int Dpk, CpadK, CpadQ;
  size_t scores_bytes;
  int punits;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline int keep_budget(double keep, int Ck) {
  // k = max(1, min(Ck, ceil(keep * Ck - 1e-9))) evaluated in fp64
  double v = keep * static_cast<double>(Ck) - 1e-9;
  long long k = static_cast<long long>(v);
  if (static_cast<double>(k) < v) k += 1;  // ceil for positive v
  if (v <= 0) k = 0;
  if (k < 1) k = 1;
  if (k > Ck) k = Ck;
  return static_cast<int>(k);
}

inline void compute_layout(const sparsepr_params& p, Layout* L) {
  const size_t H = p.H, N = p.N, d = p.d;
  const int Nv = p.N - p.n_text;
  const size_t e = p.n_eig, Ck = p.Ck, Cq = p.Cq, M = p.M;
  L->Nv = Nv;
  L->e = p.n_eig;
  const int text = p.n_text > 0 ? 1 : 0;
  L->Ckt = p.Ck + text;
  L->Cqt = p.Cq + text;
  L->Cmax = (L->Ckt > L->Cqt ? L->Ckt : L->Cqt);
  L->nchunk = (p.N + kSortChunk - 1) / kSortChunk;
  L->tiles_per_head = (p.N + kTileM - 1) / kTileM + L->Cqt;
  int kmax = 1;
  if (p.keep)
    for (int h = 0; h < p.H; ++h) {
      int k = keep_budget(p.keep[h], p.Ck);
      if (k > kmax) kmax = k;
    }
  L->kmax = kmax;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L->stats = take(sizeof(DeviceStats));
  L->fy = take(H * Nv * 4);
  L->init_k = take(H * Ck * 4);
  L->init_q = take(H * Cq * 4);
  L->mk = take(H * d * d * 8);
  L->evec = take(H * d * d * 8);
  L->eval = take(H * d * 8);
  L->eigscr = take(H * (d * d + 3 * d) * 8);
  L->wk = take(H * d * e * 8);
  L->z = take(H * Nv * e * 8);
  L->mu = take(H * Ck * e * 8);
  L->munorm = take(H * Ck * 8);
  L->lab_k = take(H * Nv * 4);
  L->lab_q = take(H * Nv * 4);
  L->flags = take(H * 4 * 4);
  L->hist = take(H * static_cast<size_t>(L->nchunk) * L->Cmax * 4);
  L->sortoff = take(H * (L->Cmax + 1) * 4);
  L->sortperm = take(H * Nv * 4);
  L->ck = take(H * Ck * d * 8);
  L->g = take(H * d * d * 8);
  L->qbar = take(H * Cq * d * 8);
  L->Dpk = (p.n_eig <= 16) ? 16 : 64;
  L->CpadK = (p.Ck + 15) / 16 * 16;
  L->CpadQ = (p.Cq + 15) / 16 * 16;
  // the alternative partitions run the d-space assignment on both sides:
  // its centroid-side regions hold max(Ck, Cq) rows
  const bool alt = p.partition != 0;
  const size_t Cm = alt ? (Ck > Cq ? Ck : Cq) : Cq;
  const size_t Cpm = alt ? (L->CpadK > L->CpadQ ? L->CpadK : L->CpadQ) : L->CpadQ;
  L->wg = take(H * Cm * d * 8);
  L->cg = take(H * Cm * 8);
  L->zplanes = take(3 * H * Nv * static_cast<size_t>(L->Dpk) * 2);
  L->xnk = take(H * Nv * 4);
  L->xnq = take(H * Nv * 4);
  L->muplanes = take(3 * H * static_cast<size_t>(L->CpadK) * L->Dpk * 2);
  L->cfk = take(H * static_cast<size_t>(L->CpadK) * 4);
  L->hmk = take(H * 8);
  L->wplanes = take(3 * H * Cpm * d * 2);
  L->cfq = take(H * Cpm * 4);
  L->hmq = take(H * 8);
  L->recheck = take(H * Nv * 4);
  L->nrecheck = take(H * 4);
  {
    size_t yt = Ck * e > Cq * d ? Ck * e : Cq * d;
    if (alt && Cm * d > yt) yt = Cm * d;
    L->ytr = take(H * yt * 8);
  }
  L->cq = take(H * Cq * d * 8);
  L->ckr = take(H * Ck * d * 8);
  {
    const size_t per_head = Cq * Ck * 8;
    size_t heads = (static_cast<size_t>(64) << 20) / per_head;
    if (heads < 1) heads = 1;
    if (heads > H) heads = H;
    L->scores_bytes = heads * per_head;
    L->scores = take(L->scores_bytes);
  }
  L->bf16_qkv = take(3 * H * N * d * 2);
  L->work = take(H * static_cast<size_t>(L->tiles_per_head) * 4);
  L->nwork = take(H * 4);
  L->nslots = take(H * static_cast<size_t>(L->Cqt) * 4);
  L->runs = take(H * static_cast<size_t>(L->Cqt) * (kmax + 1) * 8);
  L->nruns = take(H * static_cast<size_t>(L->Cqt) * 4);
  L->probe_q = take(H * (M + kTileM) * d * 2);
  L->od = take(H * (M + 1) * d * 4);
  L->xr = take(H * 2 * (M + 1) * d * 8);
  L->means = take(H * 2 * d * 8);
  L->gram = take(H * 2 * d * d * 8);
  L->gpart = take(static_cast<size_t>(kGramJobs) * kGramSplits * H * d * d * 8);
  L->bmat = take(H * d * d * 8);
  L->bvec = take(H * d * 8);
  L->bp32 = take(H * d * d * 4);
  L->bv32 = take(H * d * 4);
  L->pwork = take(H * (M / kTileM + 2) * 4);
  L->pnwork = take(H * 4);
  L->pmeta = take(H * 12 * 4);
  L->punits = static_cast<int>(M / 256 + 1);
  L->opart = take(H * static_cast<size_t>(L->punits) * kMaxSplits * 256 * d * 4);
  L->lpart = take(H * static_cast<size_t>(L->punits) * kMaxSplits * 256 * 4);
  L->opart2 = take(H * static_cast<size_t>(L->punits) * kMaxSplits * 256 * d * 4);
  L->lpart2 = take(H * static_cast<size_t>(L->punits) * kMaxSplits * 256 * 4);
  L->xp = take(H * (M + 1) * d * 4);
  L->pgrp = take(H * (M + 1) * 4);
  L->lse_s = take(H * N * 4);
  L->lse_d = take(H * (M + 1) * 4);
  L->diag = take(H * (M + 1) * 4 * 8);
  const bool cocl = p.partition == 2;
  L->pkbar = take(cocl ? H * Ck * Cq * 8 : 0);
  L->pqbar = take(cocl ? H * Cq * Ck * 8 : 0);
  L->cnt = take(alt ? H * (Ck + Cq) * 4 : 0);
  {
    const size_t words = (static_cast<size_t>(L->Ckt) + 31) / 32;
    const size_t se = align256(H * Cq * words * 4) + H * Cq * 8;
    const size_t dn = align256(static_cast<size_t>(kDiagRows) * N * 8) + H * 8;
    L->dscr = take(se > dn ? se : dn);
  }
  L->total = o;
}

// Offset and size of a named region that holds a stage's intermediate
// results (the read-out of sparsepr_workspace_region); false for an unknown
// name.
inline bool named_region(const sparsepr_params& p, const Layout& L, const char* name, size_t* off,
                         size_t* bytes) {
  const size_t H = p.H, d = p.d, e = p.n_eig, Ck = p.Ck, Cq = p.Cq, Nv = L.Nv, M = p.M;
  struct R {
    const char* n;
    size_t o, b;
  } const tab[] = {
      {"init_k", L.init_k, H * Ck * 4}, {"init_q", L.init_q, H * Cq * 4},
      {"mk", L.mk, H * d * d * 8},      {"eval", L.eval, H * e * 8},
      {"evec", L.evec, H * d * e * 8},  {"wk", L.wk, H * d * e * 8},
      {"z", L.z, H * Nv * e * 8},       {"ck", L.ck, H * Ck * d * 8},
      {"g", L.g, H * d * d * 8},        {"bmat", L.bmat, H * d * d * 8},
      {"bvec", L.bvec, H * d * 8},      {"xr", L.xr, H * 2 * M * d * 8},
      {"vr", p.r <= kTriEigMax ? L.evec : L.gram, H * d * static_cast<size_t>(p.r) * 8},
      {"zplanes", L.zplanes, 3 * H * Nv * static_cast<size_t>(L.Dpk) * 2},
      {"xnk", L.xnk, H * Nv * 4},
  };
  for (const R& r : tab) {
    const char* a = r.n;
    const char* b = name;
    while (*a && *a == *b) {
      ++a;
      ++b;
    }
    if (*a == 0 && *b == 0) {
      *off = r.o;
      *bytes = r.b;
      return true;
    }
  }
  return false;
}

template <typename T>
inline T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

}  // namespace spr
