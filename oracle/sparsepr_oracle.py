"""Plain fp64 CPU oracle of the SparsePR per-call sparse attention path.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
CPU-baseline / reference leg may import this module. The product (the CUDA
library and its Python binding) never imports, calls or links it, and this
module imports nothing from the product.

Sources (pages, cited by title and section):
  [SPR]  "Partition the Support, Reconstruct the Residual: Training-Free Sparse
         Attention for Video Generation and World Models" (gist.science
         summary), section 2 "Methodology" -- A. response-coupled
         partitioning, B. probe-fitted residual reconstruction, C. sparse
         execution.
  [SVOO] "Attention Sparsity is Input-Stable: Training-Free Sparse Attention
         for Video Generation via Offline Sparsity Profiling and Online QK
         Co-Clustering" (papernotes.org note), "method details" -- block
         selection + sparse attention assembly.
  [EXP]  cloud.baidu.com sparse-attention explainer, "principle" section --
         the masked-score pseudo-code (mask, masked score, softmax, @ V).

Every function works on ONE head in float64 numpy. Library primitives
(matmul, eigh, svd, solve, stable argsort) are used as steps; no blocking,
fusion or reordering beyond the definitions. Readings taken where the pages
are silent are listed in each docstring (and collected in the design notes).

Parity pins: each function is pinned by tests/test_oracle_*.py against
closed forms, invariants, brute force and library re-derivations that do not
share its formula. End-to-end output values beyond those invariants are
"parity unpinned" (the pages print no per-call outputs).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

MASK64 = (1 << 64) - 1


# ---------------------------------------------------------------------------
# Random draws of the method: k-means initial token indices.
# ---------------------------------------------------------------------------

def splitmix64_stream(seed: int):
    """SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): state advances by the golden-gamma constant,
    output is the variant-13 mix of the state."""
    state = seed & MASK64
    while True:
        state = (state + 0x9E3779B97F4A7C15) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        yield z ^ (z >> 31)


def init_indices(n: int, C: int, seed: int, head: int, which: int) -> np.ndarray:
    """C distinct token indices out of range(n): the first C slots of a
    partial Fisher-Yates shuffle driven by SplitMix64 seeded with
    seed XOR (2*head + which); which = 0 for keys, 1 for queries.

    Reading (the pages give no initialisation): index-based seeding, so the
    result does not depend on the sign or rotation of the eigenbasis."""
    if not 0 < C <= n:
        raise ValueError("need 0 < C <= n")
    gen = splitmix64_stream(seed ^ (2 * head + which))
    a = list(range(n))
    for i in range(C):
        j = i + next(gen) % (n - i)
        a[i], a[j] = a[j], a[i]
    return np.array(a[:C], dtype=np.int64)


# ---------------------------------------------------------------------------
# Stage 1: response-coupled partitioning  [SPR 2.A]
# ---------------------------------------------------------------------------

def sample_rows(Nv: int, Ms: int) -> np.ndarray:
    """Indices of the sampled queries Q_s. Reading: deterministic strides
    floor((s + 1/2) * Nv / Ms), s = 0..Ms-1, over the video tokens."""
    s = np.arange(Ms, dtype=np.int64)
    return ((2 * s + 1) * Nv) // (2 * Ms)


def metric_MK(q_video: np.ndarray, Ms: int) -> np.ndarray:
    """M_K = Q_s^T Q_s / M_s from the sampled queries [SPR 2.A, "Key-response
    coordinates"]."""
    Qs = q_video[sample_rows(q_video.shape[0], Ms)]
    return Qs.T @ Qs / Ms


def eigenbasis(MK: np.ndarray, e: int):
    """Top-e eigenpairs of the symmetric PSD metric M_K, eigenvalues in
    descending order [SPR 2.A: k-means on the eigenvectors of M_K].
    Tiny negative eigenvalues from rounding are clamped to 0."""
    w, U = np.linalg.eigh(MK)
    order = np.argsort(-w, kind="stable")[:e]
    return np.maximum(w[order], 0.0), U[:, order]


def key_coordinates(k_video: np.ndarray, lam_e: np.ndarray, U_e: np.ndarray) -> np.ndarray:
    """Response coordinates of the keys, z = Lambda_e^{1/2} U_e^T k.

    Reading: ||Q_s (k1 - k2)||^2 / M_s = (k1-k2)^T M_K (k1-k2), so with this
    scaling the distance between coordinates is the distance between the
    keys' response profiles restricted to the top-e eigen-subspace."""
    return k_video @ (U_e * np.sqrt(lam_e)[None, :])


def sqdist(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """Squared Euclidean distances ||x_i - c_j||^2, [n, m], via the expansion
    ||x||^2 - 2 x.c + ||c||^2 (fp64)."""
    return ((X * X).sum(1)[:, None] - 2.0 * (X @ C.T)
            + (C * C).sum(1)[None, :])


def group_means(X: np.ndarray, labels: np.ndarray, C: int, prev: Optional[np.ndarray] = None):
    """Mean of the rows of X in each group; an empty group keeps ``prev``
    (k-means update) or is the zero vector (prev None). Rows are summed in
    ascending row order."""
    sums = np.zeros((C, X.shape[1]))
    np.add.at(sums, labels, X)
    cnt = np.bincount(labels, minlength=C).astype(np.float64)
    out = np.zeros_like(sums) if prev is None else prev.copy()
    nz = cnt > 0
    out[nz] = sums[nz] / cnt[nz][:, None]
    return out


NEAR_TIE_REL = 1e-12


def count_near_ties(D: np.ndarray) -> int:
    """Rows of a distance matrix whose two smallest squared distances
    d1 <= d2 satisfy d2 - d1 <= 1e-12 d2: rows whose nearest centroid is
    decided by rounding rather than by the data (reading: such a row has
    more than one correct label, so it is counted and reported rather than
    compared; exact ties, e.g. two identical centroids, count, and the
    lowest index wins them)."""
    if D.shape[1] < 2:
        return 0
    two = np.partition(D, 1, axis=1)[:, :2]
    return int(np.count_nonzero(two[:, 1] - two[:, 0] <= NEAR_TIE_REL * two[:, 1]))


def nearest(X: np.ndarray, C: np.ndarray, chunk: int = 8192, ties: Optional[list] = None):
    """Index of the nearest centroid of every row (lowest index on ties).
    Rows are independent; they are evaluated in chunks to bound memory.
    ``ties``: if a list, the count of near-tie rows is appended to it."""
    out = np.empty(X.shape[0], dtype=np.int64)
    nt = 0
    for s in range(0, X.shape[0], chunk):
        D = sqdist(X[s:s + chunk], C)
        out[s:s + chunk] = np.argmin(D, axis=1)
        if ties is not None:
            nt += count_near_ties(D)
    if ties is not None:
        ties.append(nt)
    return out


def lloyd(X: np.ndarray, init: np.ndarray, iters: int, ties: Optional[list] = None):
    """Lloyd k-means: assign every row to its nearest centroid (lowest index
    on ties), stop when no label changes, else move each centroid to its
    group mean (an empty group keeps its centroid). At most ``iters``
    assignment passes. Returns (labels, centroids, passes); ``ties``, if a
    list, receives the near-tie count of every pass.

    Reading: the pages fix neither init, stopping nor empty groups; SVOO's
    note says single-digit iteration counts suffice."""
    mu = X[init].copy()
    labels = None
    passes = 0
    for _ in range(iters):
        new = nearest(X, mu, ties=ties)  # first minimum = lowest index
        passes += 1
        if labels is not None and np.array_equal(new, labels):
            break
        labels = new
        mu = group_means(X, labels, mu.shape[0], prev=mu)
    return labels, mu, passes


def key_partition(k_video, q_video, Ck, Ms, e, iters, seed, head):
    """Keys clustered by k-means on their response coordinates in the
    eigenbasis of M_K; gives the paired K/V groups [SPR 2.A]."""
    MK = metric_MK(q_video, Ms)
    lam_e, U_e = eigenbasis(MK, e)
    Z = key_coordinates(k_video, lam_e, U_e)
    init = init_indices(k_video.shape[0], Ck, seed, head, 0)
    ties = []
    labels, _, passes = lloyd(Z, init, iters, ties)
    return labels, dict(MK=MK, lam=lam_e, U=U_e, Z=Z, passes=passes, near_ties=sum(ties))


def query_profiles(q_video: np.ndarray, CK: np.ndarray, scale: float) -> np.ndarray:
    """Pre-softmax logit profile of each query against the K/V group
    centroids, p_i = scale * C_K q_i, in R^{Ck} [SPR 2.A,
    "Query-response coordinates"]."""
    return scale * (q_video @ CK.T)


def query_partition(q_video, CK, Cq, iters, seed, head, scale):
    """Queries clustered by k-means on their logit profiles (literal Ck-dim
    profile space) [SPR 2.A]. One asymmetric pass: keys first, then
    queries, no alternation."""
    P = query_profiles(q_video, CK, scale)
    init = init_indices(q_video.shape[0], Cq, seed, head, 1)
    ties = []
    labels, _, passes = lloyd(P, init, iters, ties)
    return labels, dict(passes=passes, near_ties=sum(ties))


def semantic_partition(q_video, k_video, Ck, Cq, iters, seed, head):
    """The comparison partition of the ablations [SPR 2.A results; SPR 4,
    ablations]: keys and queries clustered separately by plain Euclidean
    k-means on their own rows, no response coupling. Reading: same
    initialisation draws and pass cap as the response-coupled partition.
    Returns (key labels, query labels, key info, query info)."""
    init_k = init_indices(k_video.shape[0], Ck, seed, head, 0)
    lab_k, _, kp = lloyd(k_video, init_k, iters)
    init_q = init_indices(q_video.shape[0], Cq, seed, head, 1)
    lab_q, _, qp = lloyd(q_video, init_q, iters)
    nan = np.full((q_video.shape[1], q_video.shape[1]), np.nan)
    return lab_k, lab_q, dict(passes=kp, MK=nan, lam=np.zeros(0), U=np.zeros((0, 0))), \
        dict(passes=qp)


def coclustering_partition(q_video, k_video, Ck, Cq, iters, seed, head, scale):
    """Bidirectional QK co-clustering ["Attention Sparsity is Input-Stable"
    (papernotes.org note), "key designs", online bidirectional
    co-clustering], offered as an alternative partition. Each round: (A) each
    key's affinity vector to the current query centres, P_k = scale * K C_q^T,
    is assigned to the nearest key-block centre in that space (the mean
    affinity vector of the block's current members), then the key centres
    C_k are the blocks' mean K rows; (B) symmetrically for the queries with
    P_q = scale * Q C_k^T against the just-updated C_k. Readings: C_q starts
    at the query rows of the Fisher-Yates draws (which = 1) and the first key
    blocks are the singletons of the key draws (which = 0), the first query
    blocks those of the query draws; an empty block keeps its previous centre;
    at most ``iters`` rounds, stopping after a round that changes no label.
    Returns (key labels, query labels, rounds)."""
    seeds_k = init_indices(k_video.shape[0], Ck, seed, head, 0)
    seeds_q = init_indices(q_video.shape[0], Cq, seed, head, 1)
    Cq_c = q_video[seeds_q].copy()
    lab_k = lab_q = None
    Pk_bar = Pq_bar = None
    rounds = 0
    for _ in range(iters):
        rounds += 1
        Pk = scale * (k_video @ Cq_c.T)
        Pk_bar = Pk[seeds_k] if lab_k is None else group_means(Pk, lab_k, Ck, prev=Pk_bar)
        new_k = nearest(Pk, Pk_bar)
        Ck_c = group_means(k_video, new_k, Ck)
        Pq = scale * (q_video @ Ck_c.T)
        Pq_bar = Pq[seeds_q] if lab_q is None else group_means(Pq, lab_q, Cq, prev=Pq_bar)
        new_q = nearest(Pq, Pq_bar)
        done = (lab_k is not None and np.array_equal(new_k, lab_k)
                and np.array_equal(new_q, lab_q))
        lab_k, lab_q = new_k, new_q
        Cq_c = group_means(q_video, lab_q, Cq, prev=Cq_c)
        if done:
            break
    return lab_k, lab_q, rounds


# ---------------------------------------------------------------------------
# Stage 2: group-major layout  [SPR 2.C]
# ---------------------------------------------------------------------------

def group_major(labels: np.ndarray, C: int):
    """Stable permutation into contiguous group-major order. perm[i] is the
    original token of group-major row i (ascending token order inside a
    group), inv is its inverse, off[c]..off[c+1] is group c's row range."""
    perm = np.argsort(labels, kind="stable").astype(np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    off = np.zeros(C + 1, dtype=np.int64)
    off[1:] = np.cumsum(np.bincount(labels, minlength=C))
    return perm, inv, off


# ---------------------------------------------------------------------------
# Stage 3: routing and variable-block sparse attention  [SVOO, SPR 2.C, EXP]
# ---------------------------------------------------------------------------

def keep_budget(keep: float, Ck: int) -> int:
    """Kept key groups per query group, k = max(1, ceil(keep * Ck - 1e-9)),
    at most Ck [SVOO: top-ceil((1-s) K_k)]. The 1e-9 guard keeps products
    such as 0.22*1000 from rounding up; k >= 1 keeps at least one key per
    row."""
    return int(min(Ck, max(1, math.ceil(keep * Ck - 1e-9))))


def range_means(Xp: np.ndarray, off: np.ndarray) -> np.ndarray:
    """Mean row of each group-major range (zero vector for an empty range)."""
    C = off.size - 1
    out = np.zeros((C, Xp.shape[1]))
    for c in range(C):
        if off[c + 1] > off[c]:
            out[c] = Xp[off[c]:off[c + 1]].mean(axis=0)
    return out


def route(CQ: np.ndarray, CK: np.ndarray, k: int, scale: float) -> np.ndarray:
    """Block scores A[g, c] = scale * C_Q[g] . C_K[c] from the group centroids;
    each query group keeps its top-k key groups (ties: lowest index), listed
    in ascending order [SVOO, block selection]."""
    A = scale * (CQ @ CK.T)
    csr = np.empty((CQ.shape[0], k), dtype=np.int64)
    for g in range(CQ.shape[0]):
        top = np.argsort(-A[g], kind="stable")[:k]
        csr[g] = np.sort(top)
    return csr


def kept_key_mask(csr_row, off_k: np.ndarray, N: int, extra_groups=()) -> np.ndarray:
    """Boolean mask over the N group-major keys: the union of the kept key
    groups' ranges."""
    m = np.zeros(N, dtype=bool)
    for c in list(csr_row) + list(extra_groups):
        m[off_k[c]:off_k[c + 1]] = True
    return m


def masked_attention_rows(Qp, Kp, Vp, rows, group_of_row, mask_of_group, scale):
    """Masked-softmax attention of the listed rows [EXP pseudo-code: mask,
    masked scores, softmax, weights @ V]: logits outside the row's mask are
    -inf, so the softmax is taken over the kept logits only [SVOO]. Rows that
    share a group share a mask and are evaluated together.
    Returns O [len(rows), d]."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, Vp.shape[1]))
    groups = np.array([group_of_row(int(i)) for i in rows], dtype=np.int64)
    for g in np.unique(groups):
        sel = np.nonzero(groups == g)[0]
        m = mask_of_group(int(g))
        if not m.any():
            raise FloatingPointError("empty kept set for query group %d" % g)
        S = scale * (Qp[rows[sel]] @ Kp.T)
        S = np.where(m[None, :], S, -np.inf)
        W = np.exp(S - S.max(axis=1, keepdims=True))
        W /= W.sum(axis=1, keepdims=True)
        out[sel] = W @ Vp
    return out


def dense_attention(Q, K, V, scale):
    """Plain softmax attention softmax(scale * Q K^T) V (textbook form)."""
    S = scale * (Q @ K.T)
    S = S - S.max(axis=1, keepdims=True)
    W = np.exp(S)
    W /= W.sum(axis=1, keepdims=True)
    return W @ V


# ---------------------------------------------------------------------------
# Stage 4: probe-fitted residual reconstruction  [SPR 2.B]
# ---------------------------------------------------------------------------

def probe_counts(n: np.ndarray, M: int) -> np.ndarray:
    """Probes per query group, m_g proportional to the group size n_g by the
    largest-remainder method (remainder ties go to the lower group), sum M.
    Reading of "stratified across query groups" [SPR 2.B]."""
    n = np.asarray(n, dtype=np.int64)
    Nt = int(n.sum())
    if not 0 <= M <= Nt:
        raise ValueError("need 0 <= M <= number of rows")
    m = (M * n) // Nt
    rem = (M * n) % Nt
    left = M - int(m.sum())
    order = sorted(range(n.size), key=lambda g: (-int(rem[g]), g))
    for g in order[:left]:
        m[g] += 1
    return m


def probe_rows(off_q: np.ndarray, M: int) -> np.ndarray:
    """Group-major row indices of the probes: m_g rows of group g at offsets
    floor((t + 1/2) n_g / m_g), t = 0..m_g-1, groups in ascending order."""
    n = np.diff(off_q)
    m = probe_counts(n, M)
    rows = []
    for g in range(n.size):
        for t in range(int(m[g])):
            rows.append(int(off_q[g]) + ((2 * t + 1) * int(n[g])) // (2 * int(m[g])))
    return np.array(rows, dtype=np.int64)


def ridge_fit(X: np.ndarray, R: np.ndarray, lam: float):
    """Affine residual model R ~ b + x B by ridge regression [SPR 2.B,
    "affine calibration"]. Reading: the intercept b is not penalised
    (implemented by centring), lam is not scaled by M, normal equations in
    fp64: B = (Xc^T Xc + lam I)^{-1} Xc^T Rc, b = rbar - xbar B."""
    xbar = X.mean(axis=0)
    rbar = R.mean(axis=0)
    Xc = X - xbar
    Rc = R - rbar
    A = Xc.T @ Xc + lam * np.eye(X.shape[1])
    B = np.linalg.solve(A, Xc.T @ Rc)
    b = rbar - xbar @ B
    return B, b


def residual_subspace(R: np.ndarray, r: int) -> np.ndarray:
    """Leading-r right singular vectors of the (uncentred) probe residual
    matrix R, as columns [d, r] [SPR 2.B, "subspace restriction"]."""
    _, _, Vt = np.linalg.svd(R, full_matrices=True)
    return Vt[:r].T


def project_map(B: np.ndarray, b: np.ndarray, Vr: np.ndarray):
    """Restrict the affine map to the residual subspace: B' = B P_r,
    b' = b P_r with P_r = V_r V_r^T."""
    P = Vr @ Vr.T
    return B @ P, b @ P


# ---------------------------------------------------------------------------
# One attention call on one head
# ---------------------------------------------------------------------------

@dataclass
class HeadResult:
    label_q: np.ndarray
    label_k: np.ndarray
    perm_q: np.ndarray
    perm_k: np.ndarray
    off_q: np.ndarray
    off_k: np.ndarray
    k: int
    csr: np.ndarray
    probes: np.ndarray
    pairs_sparse: int
    pairs_exec: int
    rows: np.ndarray  # group-major rows whose outputs were computed
    o_sparse: np.ndarray  # [len(rows), d]
    out: np.ndarray  # [len(rows), d] corrected output of those rows
    o_dense_probe: np.ndarray
    o_sparse_probe: np.ndarray
    B: np.ndarray
    b: np.ndarray
    Bp: np.ndarray
    bp: np.ndarray
    Vr: np.ndarray
    info: dict = field(default_factory=dict)


def resolve_scale(scale: float, d: int) -> float:
    return scale if scale > 0 else 1.0 / math.sqrt(d)


def run_head(q, k, v, p: dict, head: int, rows=None, partition_only=False) -> HeadResult:
    """The whole per-call path on one head (q, k, v: [N, d] float64).

    ``p`` holds the method parameters (Ck, Cq, Ms, n_eig, kmeans_iters, keep
    [per head], M, r, lam, scale, seed, n_text; optionally partition =
    "response" (default), "semantic" (the ablations' uncoupled k-means on
    raw Q and K rows) or "coclustering" (the co-clustering page's
    alternating QK partition)). ``rows`` restricts the
    sparse-attention and corrected outputs to those group-major rows
    (default: all rows); partition, routing, probes and the fit are always
    computed in full.

    Text tokens (n_text > 0, the trailing indices). Reading: they take part
    in neither k-means nor Q_s; they form one extra key group (index Ck) that
    every query group keeps outside the budget, and one extra query group
    (index Cq) that keeps every key group; text rows are never probes and
    never corrected.
    """
    N, d = q.shape
    nt = int(p.get("n_text", 0))
    Nv = N - nt
    Ck, Cq = int(p["Ck"]), int(p["Cq"])
    scale = resolve_scale(float(p.get("scale", 0.0)), d)
    seed = int(p["seed"])
    iters = int(p["kmeans_iters"])
    qv, kv = q[:Nv], k[:Nv]

    # Stage 1 [SPR 2.A]
    mode = p.get("partition", "response")
    if mode == "semantic":
        lab_k_v, lab_q_v, kinfo, qinfo = semantic_partition(qv, kv, Ck, Cq, iters, seed, head)
    elif mode == "coclustering":
        lab_k_v, lab_q_v, rounds = coclustering_partition(qv, kv, Ck, Cq, iters, seed, head, scale)
        kinfo = dict(passes=rounds, MK=np.full((d, d), np.nan), lam=np.zeros(0),
                     U=np.zeros((0, 0)))
        qinfo = dict(passes=rounds)
    else:
        lab_k_v, kinfo = key_partition(kv, qv, Ck, int(p["Ms"]), int(p["n_eig"]),
                                       iters, seed, head)
        CK_part = group_means(kv, lab_k_v, Ck)  # original-space K/V group centroids
        lab_q_v, qinfo = query_partition(qv, CK_part, Cq, iters, seed, head, scale)
    label_k = np.concatenate([lab_k_v, np.full(nt, Ck, dtype=np.int64)])
    label_q = np.concatenate([lab_q_v, np.full(nt, Cq, dtype=np.int64)])
    Ckt, Cqt = Ck + (1 if nt else 0), Cq + (1 if nt else 0)

    # Stage 2 [SPR 2.C]
    perm_q, inv_q, off_q = group_major(label_q, Cqt)
    perm_k, inv_k, off_k = group_major(label_k, Ckt)
    info = dict(key_passes=kinfo["passes"], query_passes=qinfo["passes"],
                MK=kinfo["MK"], eig_lam=kinfo["lam"], eig_U=kinfo["U"],
                key_near_ties=kinfo.get("near_ties"), query_near_ties=qinfo.get("near_ties"))
    kk = keep_budget(float(p["keep"][head] if isinstance(p["keep"], (list, tuple)) else p["keep"]), Ck)
    if partition_only:
        return HeadResult(label_q, label_k, perm_q, perm_k, off_q, off_k, kk,
                          None, None, 0, 0, None, None, None, None, None,
                          None, None, None, None, None, info)
    Qp, Kp, Vp = q[perm_q], k[perm_k], v[perm_k]

    # Stage 3 [SVOO block selection; SPR 2.C]
    CQ = range_means(Qp, off_q)[:Cq]
    CK = range_means(Kp, off_k)[:Ck]
    csr = route(CQ, CK, kk, scale)
    text_group = (Ck,) if nt else ()

    def row_group(i):
        return int(np.searchsorted(off_q, i, side="right") - 1)

    masks = {}

    def mask_of_group(g):
        if g not in masks:
            if g == Cq:  # text query group: every key
                masks[g] = np.ones(N, dtype=bool)
            else:
                masks[g] = kept_key_mask(csr[g], off_k, N, text_group)
        return masks[g]

    n_q = np.diff(off_q)
    n_k = np.diff(off_k)
    pairs_sparse = 0
    for g in range(Cq):
        pairs_sparse += int(n_q[g]) * (int(n_k[csr[g]].sum()) + (int(n_k[Ck]) if nt else 0))
    if nt:
        pairs_sparse += int(n_q[Cq]) * N

    # Stage 4 [SPR 2.B]
    M = int(p["M"])
    probes = probe_rows(off_q[:Cq + 1], M)
    pairs_exec = pairs_sparse + M * N
    if M > 0:
        Xs = masked_attention_rows(Qp, Kp, Vp, probes, row_group, mask_of_group, scale)
        Od = dense_attention(Qp[probes], Kp, Vp, scale)
        R = Od - Xs
        B, b = ridge_fit(Xs, R, float(p["lam"]))
        Vr = residual_subspace(R, int(p["r"]))
        Bp, bp = project_map(B, b, Vr)
    else:
        # no probes: the hard-drop variant (sparse output, no reconstruction)
        Xs = Od = np.zeros((0, d))
        B = Bp = np.zeros((d, d))
        b = bp = np.zeros(d)
        Vr = np.zeros((d, 0))

    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    Os = masked_attention_rows(Qp, Kp, Vp, rows, row_group, mask_of_group, scale)
    out = Os + bp[None, :] + Os @ Bp
    probe_pos = {int(r_): j for j, r_ in enumerate(probes)}
    for t, i in enumerate(rows):
        if int(i) in probe_pos:
            out[t] = Od[probe_pos[int(i)]]
        elif nt and row_group(int(i)) == Cq:
            out[t] = Os[t]  # text rows are not corrected
    return HeadResult(label_q, label_k, perm_q, perm_k, off_q, off_k, kk, csr,
                      probes, pairs_sparse, pairs_exec, rows, Os, out, Od, Xs,
                      B, b, Bp, bp, Vr, info)


def run(q, k, v, p: dict, heads=None, rows=None):
    """run_head over heads (q, k, v: [H, N, d] float64). Returns a list of
    HeadResult, one per head in ``heads`` (default: all)."""
    hs = range(q.shape[0]) if heads is None else heads
    return [run_head(q[i], k[i], v[i], p, h, rows=rows)
            for i, h in enumerate(hs)]


def output_original_order(res: HeadResult, N: int, d: int) -> np.ndarray:
    """Corrected output of all rows scattered back to the original token
    order (requires res.rows == all rows)."""
    out = np.zeros((N, d))
    out[res.perm_q[res.rows]] = res.out
    return out
