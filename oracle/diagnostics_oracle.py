"""Plain fp64 CPU oracle of the structural diagnostics that SparsePR's
analysis reports, computed from one head's call.

TEST INFRASTRUCTURE, like sparsepr_oracle: only the tests may import it; the
product never imports, calls or links it.

Source: "Partition the Support, Reconstruct the Residual: Training-Free
Sparse Attention for Video Generation and World Models" (gist.science
summary), section 3 "Core contributions", structural analysis: (i) the
sparsity of single queries does not fix the support a shared route needs
(aggregate support several times larger), (ii) retained attention mass does
not bound the post-softmax error, (iii) the partition's geometry changes the
"affine-explainable" part of the residual; and section 4, ablations
(response-coupled partitioning lowers the orthogonal residual energy).

The pages name the quantities but give no formulas; the readings taken:
  * individual support of a row at mass tau: the fewest key groups whose
    dense softmax mass reaches tau (largest mass first, ties to the lower
    group index); aggregate support of a query group: the union of its rows'
    individual supports; expansion = |union| / mean individual size;
  * retained mass of a row: dense softmax mass on the keys its route keeps;
    error: Euclidean norm of O_dense - O_sparse for that row;
  * affine-explainable fraction of the probe residual R: ||R P_r||_F^2 /
    ||R||_F^2 with P_r the projector of the fitted subspace; orthogonal
    energy: the share of ||R||_F^2 that the fitted (projected) map leaves,
    ||R - (b' + X B')||_F^2 / ||R||_F^2, on the probe rows.
"""
from __future__ import annotations

import numpy as np

from oracle import sparsepr_oracle as O


def dense_weights(Qp: np.ndarray, Kp: np.ndarray, rows: np.ndarray, scale: float) -> np.ndarray:
    """Full softmax weights of the listed group-major rows over all N keys."""
    S = scale * (Qp[rows] @ Kp.T)
    W = np.exp(S - S.max(axis=1, keepdims=True))
    return W / W.sum(axis=1, keepdims=True)


def group_mass(W: np.ndarray, off_k: np.ndarray) -> np.ndarray:
    """Dense softmax mass of each row on each key group's range [rows, C]."""
    C = off_k.size - 1
    out = np.zeros((W.shape[0], C))
    for c in range(C):
        out[:, c] = W[:, off_k[c]:off_k[c + 1]].sum(axis=1)
    return out


def individual_support(mass_row: np.ndarray, tau: float) -> np.ndarray:
    """Fewest key groups whose mass reaches tau: groups by decreasing mass
    (ties to the lower index) until the running sum is >= tau."""
    order = np.argsort(-mass_row, kind="stable")
    run = np.cumsum(mass_row[order])
    n = int(np.searchsorted(run, tau - 1e-15, side="left")) + 1
    return np.sort(order[:min(n, order.size)])


def support_expansion(res: O.HeadResult, Qp, Kp, p: dict, tau: float) -> dict:
    """Per video query group: mean individual support size, aggregate
    (union) size, and their ratio; counted in key groups (a text key group,
    when present, counts as one more group)."""
    Cq = int(p["Cq"])
    scale = O.resolve_scale(float(p.get("scale", 0.0)), Qp.shape[1])
    Ck = res.off_k.size - 1
    indiv, union, ratio = np.zeros(Cq), np.zeros(Cq), np.full(Cq, np.nan)
    for g in range(Cq):
        rows = np.arange(res.off_q[g], res.off_q[g + 1])
        if rows.size == 0:
            continue
        gm = group_mass(dense_weights(Qp, Kp, rows, scale), res.off_k)
        sets = [individual_support(gm[t], tau) for t in range(rows.size)]
        indiv[g] = np.mean([s.size for s in sets])
        u = np.zeros(Ck, dtype=bool)
        for s in sets:
            u[s] = True
        union[g] = u.sum()
        ratio[g] = union[g] / indiv[g]
    return dict(individual=indiv, aggregate=union, expansion=ratio)


def kept_keys(res: O.HeadResult, p: dict, g: int, N: int) -> np.ndarray:
    """The keys query group g attends to, as in the call: its routed key
    groups plus the text key group; the text query group keeps every key."""
    Ck, Cq, nt = int(p["Ck"]), int(p["Cq"]), int(p.get("n_text", 0))
    if nt and g == Cq:
        return np.ones(N, dtype=bool)
    return O.kept_key_mask(res.csr[g], res.off_k, N, (Ck,) if nt else ())


def retained_mass_and_error(res: O.HeadResult, Qp, Kp, Vp, p: dict) -> dict:
    """For each computed row of ``res`` (res.rows): retained dense mass on
    the routed keys, the sparse-vs-dense error norm, and the dropped keys'
    weighted mean value (so that O_dense = m O_sparse + (1 - m) O_drop)."""
    rows = res.rows
    scale = O.resolve_scale(float(p.get("scale", 0.0)), Qp.shape[1])
    W = dense_weights(Qp, Kp, rows, scale)
    Od = W @ Vp
    m = np.zeros(rows.size)
    drop = np.zeros_like(Od)
    for t, i in enumerate(rows):
        g = int(np.searchsorted(res.off_q, i, side="right") - 1)
        keep = kept_keys(res, p, g, Kp.shape[0])
        m[t] = W[t, keep].sum()
        wd = np.where(keep, 0.0, W[t])
        if wd.sum() > 0:
            drop[t] = (wd @ Vp) / wd.sum()
    err = np.linalg.norm(Od - res.o_sparse, axis=1)
    return dict(mass=m, error=err, o_dense=Od, o_drop=drop)


def residual_energy(res: O.HeadResult) -> dict:
    """Energy split of the probe residual R = O_dense - O_sparse (probe
    rows): explainable fraction ||R P_r||^2 / ||R||^2, and the shares left
    by the fitted map before (b + X B) and after (b' + X B') the subspace
    restriction."""
    R = res.o_dense_probe - res.o_sparse_probe
    X = res.o_sparse_probe
    tot = float((R * R).sum())
    if tot == 0.0:
        return dict(total=0.0, explainable=1.0, orthogonal_fit=0.0, orthogonal_projected=0.0)
    P = res.Vr @ res.Vr.T
    RP = R @ P
    F = R - (res.b[None, :] + X @ res.B)
    Fp = R - (res.bp[None, :] + X @ res.Bp)
    return dict(total=tot, explainable=float((RP * RP).sum()) / tot,
                orthogonal_fit=float((F * F).sum()) / tot,
                orthogonal_projected=float((Fp * Fp).sum()) / tot)


# ---------------------------------------------------------------------------
# Per-head density profile  ["Attention Sparsity is Input-Stable: Training-Free
# Sparse Attention for Video Generation via Offline Sparsity Profiling and
# Online QK Co-Clustering" (papernotes.org note), "key designs", offline
# layer-wise sparsity profiling]
#
# Readings: a row's density is the smallest fraction of its N attention
# weights whose sum reaches tau (weights taken largest first); a head's
# density on one input is the mean of its rows' densities over the rows
# examined; the Gaussian over the calibration inputs is the maximum-
# likelihood fit (population standard deviation); its upper alpha quantile is
# the conservative density, clipped to [0, 1], and the sparsity is 1 minus it.
# ---------------------------------------------------------------------------

def row_density(weights: np.ndarray, tau: float) -> float:
    """Smallest fraction of the row's weights (largest first) whose sum
    reaches tau."""
    w = np.sort(np.asarray(weights, dtype=np.float64))[::-1]
    run = np.cumsum(w)
    n = int(np.searchsorted(run, tau - 1e-15, side="left")) + 1
    return min(n, w.size) / w.size


def head_density(Q: np.ndarray, K: np.ndarray, rows: np.ndarray, scale: float,
                 tau: float) -> float:
    """Mean row density of the listed query rows' full softmax over K."""
    W = dense_weights(Q, K, np.asarray(rows, dtype=np.int64), scale)
    return float(np.mean([row_density(W[t], tau) for t in range(W.shape[0])]))


def conservative_density(samples, alpha: float) -> dict:
    """Gaussian fit of one head's densities over calibration inputs and its
    upper alpha quantile mu + z_alpha sigma; sparsity = 1 - that density."""
    from scipy.stats import norm
    x = np.asarray(samples, dtype=np.float64)
    mu, sigma = float(x.mean()), float(x.std())
    d_hat = min(1.0, max(0.0, mu + float(norm.ppf(alpha)) * sigma))
    return dict(mu=mu, sigma=sigma, density=d_hat, sparsity=1.0 - d_hat)
