"""Pins of the diagnostics oracle (structural analysis of SparsePR, section 3)
against hand examples, brute force and exact identities. CPU only."""
import itertools
import math

import numpy as np

from oracle import diagnostics_oracle as D
from oracle import sparsepr_oracle as O
from free_block_sparse_eigenbasis_b200 import synth


def _tiny(keep=0.25, **kw):
    w = synth.custom("diag", 1, (4, 8, 8), 64, "f32", n_comp=8, sigma=0.3, noise_var=0.0, Ck=16,
                     Cq=8, Ms=64, n_eig=2, M=16, r=8, lam=1e-3, seed=0, keep=keep, **kw)
    q, k, v = synth.generate(w)
    q, k, v = synth.as_f64(q[0]), synth.as_f64(k[0]), synth.as_f64(v[0])
    p = w.params()
    res = O.run_head(q, k, v, p, 0)
    return w, p, res, q[res.perm_q], k[res.perm_k], v[res.perm_k]


def test_individual_support_hand_example():
    m = np.array([0.1, 0.5, 0.2, 0.2])
    assert D.individual_support(m, 0.5).tolist() == [1]
    assert D.individual_support(m, 0.7).tolist() == [1, 2]  # tie 2/3 to the lower index
    assert D.individual_support(m, 0.71).tolist() == [1, 2, 3]
    assert D.individual_support(m, 1.0).tolist() == [0, 1, 2, 3]


def test_individual_support_is_a_smallest_covering_set():
    rng = np.random.default_rng(3)
    for _ in range(40):
        m = rng.dirichlet(np.full(8, 0.4))
        tau = float(rng.uniform(0.2, 0.95))
        got = D.individual_support(m, tau)
        assert m[got].sum() >= tau - 1e-12
        best = min(s for s in range(1, 9)
                   if any(m[list(c)].sum() >= tau - 1e-12
                          for c in itertools.combinations(range(8), s)))
        assert got.size == best


def test_support_expansion_brute_force_and_identical_rows():
    w, p, res, Qp, Kp, Vp = _tiny()
    tau = 0.6
    ex = D.support_expansion(res, Qp, Kp, p, tau)
    scale = 1.0 / math.sqrt(w.d)
    for g in range(w.Cq):
        rows = range(res.off_q[g], res.off_q[g + 1])
        sets = []
        for i in rows:
            s = [scale * float(Qp[i] @ Kp[j]) for j in range(w.N)]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            z = sum(e)
            gm = [sum(e[j] for j in range(res.off_k[c], res.off_k[c + 1])) / z
                  for c in range(w.Ck)]
            order = sorted(range(w.Ck), key=lambda c: (-gm[c], c))
            acc, chosen = 0.0, []
            for c in order:
                chosen.append(c)
                acc += gm[c]
                if acc >= tau - 1e-15:
                    break
            sets.append(set(chosen))
        if not sets:
            continue
        assert ex["individual"][g] == np.mean([len(s) for s in sets])
        assert ex["aggregate"][g] == len(set().union(*sets))
        assert ex["expansion"][g] >= 1.0
    # a query group whose rows are one vector needs no more than one row's support
    Q1 = Qp.copy()
    g0 = int(np.argmax(np.diff(res.off_q)[:w.Cq]))
    Q1[res.off_q[g0]:res.off_q[g0 + 1]] = Qp[res.off_q[g0]]
    assert D.support_expansion(res, Q1, Kp, p, tau)["expansion"][g0] == 1.0


def test_retained_mass_decomposes_the_dense_output():
    """O_dense = m O_sparse + (1 - m) O_drop row by row, with O_sparse from the
    call's own masked attention; keep = 1 retains all mass with zero error."""
    w, p, res, Qp, Kp, Vp = _tiny()
    rm = D.retained_mass_and_error(res, Qp, Kp, Vp, p)
    m = rm["mass"][:, None]
    assert np.all((rm["mass"] > 0) & (rm["mass"] <= 1 + 1e-12))
    assert np.abs(rm["o_dense"] - (m * res.o_sparse + (1 - m) * rm["o_drop"])).max() < 1e-12
    assert np.allclose(rm["error"], np.linalg.norm(rm["o_dense"] - res.o_sparse, axis=1))
    w1, p1, r1, Q1, K1, V1 = _tiny(keep=1.0)
    rm1 = D.retained_mass_and_error(r1, Q1, K1, V1, p1)
    assert np.abs(rm1["mass"] - 1).max() < 1e-12 and rm1["error"].max() < 1e-12


def _fit_result(X, R, lam, r):
    B, b = O.ridge_fit(X, R, lam)
    Vr = O.residual_subspace(R, r)
    Bp, bp = O.project_map(B, b, Vr)
    z = np.zeros(0)
    return O.HeadResult(z, z, z, z, z, z, 0, z, z, 0, 0, z, z, z, X + R, X, B, b, Bp, bp, Vr)


def test_residual_energy_closed_forms():
    rng = np.random.default_rng(5)
    M, d = 40, 6
    X = rng.standard_normal((M, d))
    # generic residual: explainable share = top-r eigenvalues of R^T R over the trace
    R = rng.standard_normal((M, d)) @ np.diag([3, 2, 1, 0.5, 0.2, 0.1])
    for r in (1, 3, 6):
        e = D.residual_energy(_fit_result(X, R, 1e-2, r))
        ev = np.sort(np.linalg.eigvalsh(R.T @ R))[::-1]
        assert abs(e["explainable"] - ev[:r].sum() / ev.sum()) < 1e-12
        # the projected map leaves the energy outside the subspace plus the
        # unprojected fit's leftover inside it (orthogonal split)
        hr = _fit_result(X, R, 1e-2, r)
        F = R - (hr.b[None, :] + X @ hr.B)
        vals, vecs = np.linalg.eigh(R.T @ R)
        U = vecs[:, np.argsort(vals)[::-1][:r]]
        FP = F @ U @ U.T
        tot = (R * R).sum()
        assert abs(e["orthogonal_projected"] - (1 - e["explainable"] + (FP * FP).sum() / tot)) < 1e-12
        assert abs(e["orthogonal_fit"] - (F * F).sum() / tot) < 1e-12
    # an exactly affine residual, no ridge, full rank: the fit leaves nothing
    B0 = rng.standard_normal((d, d))
    b0 = rng.standard_normal(d)
    Ra = b0[None, :] + X @ B0
    e = D.residual_energy(_fit_result(X, Ra, 0.0, d))
    assert e["explainable"] > 1 - 1e-12
    assert e["orthogonal_fit"] < 1e-20 and e["orthogonal_projected"] < 1e-20
    # rank-deficient affine residual at its rank: the projection loses nothing
    B1 = rng.standard_normal((d, 2)) @ rng.standard_normal((2, d))
    Rb = X @ B1
    e = D.residual_energy(_fit_result(X, Rb, 0.0, 2))
    assert e["explainable"] > 1 - 1e-12 and e["orthogonal_projected"] < 1e-20


def test_semantic_partition_is_plain_lloyd_on_raw_rows_and_expands_support():
    """The ablations' semantic partition: keys and queries each a Lloyd fixed
    point of plain Euclidean distance on their own rows (checked with loops
    from the labels alone); the rest of the call is unchanged, so its
    invariants still hold."""
    w = synth.custom("sem", 1, (2, 4, 8), 16, "f32", n_comp=6, sigma=0.4, noise_var=0.05, Ck=6,
                     Cq=4, Ms=32, n_eig=16, kmeans_iters=200, M=8, r=4, seed=3, keep=0.5)
    q, k, v = synth.generate(w)
    q, k, v = synth.as_f64(q[0]), synth.as_f64(k[0]), synth.as_f64(v[0])
    p = dict(w.params(), partition="semantic")
    res = O.run_head(q, k, v, p, 0)
    assert res.info["key_passes"] < w.kmeans_iters and res.info["query_passes"] < w.kmeans_iters
    for X, lab, C in ((k, res.label_k, w.Ck), (q, res.label_q, w.Cq)):
        assert len(set(lab.tolist())) == C
        means = [[sum(X[i, a] for i in range(w.N) if lab[i] == c) / int((lab == c).sum())
                  for a in range(w.d)] for c in range(C)]
        for i in range(w.N):
            dist = [sum((X[i, a] - means[c][a]) ** 2 for a in range(w.d)) for c in range(C)]
            assert dist[lab[i]] <= min(dist) + 1e-9 * max(1.0, min(dist))
    assert np.all(np.isfinite(res.out)) and res.pairs_exec == res.pairs_sparse + w.M * w.N
    assert np.array_equal(np.sort(res.perm_q), np.arange(w.N))


def test_row_density_closed_forms_and_brute_force():
    N = 40
    # equal weights: ceil(tau N) of N are needed
    for tau in (0.95, 0.5, 0.025, 1.0):
        assert D.row_density(np.full(N, 1.0 / N), tau) == math.ceil(tau * N - 1e-9) / N
    one_hot = np.zeros(N)
    one_hot[17] = 1.0
    assert D.row_density(one_hot, 0.95) == 1.0 / N
    rng = np.random.default_rng(9)
    for _ in range(30):
        w = rng.dirichlet(np.full(9, 0.3))
        tau = float(rng.uniform(0.3, 0.99))
        best = min(s for s in range(1, 10)
                   if any(w[list(c)].sum() >= tau - 1e-12
                          for c in itertools.combinations(range(9), s)))
        assert D.row_density(w, tau) == best / 9


def test_head_density_two_levels_of_logits():
    """Keys in two blocks of logits a (n1 keys) and 0 (n2 keys): the row's
    weights are e^a/Z and 1/Z, so the covering count has a closed form."""
    n1, n2, a = 5, 35, 3.0
    K = np.zeros((n1 + n2, 2))
    K[:n1, 0] = a
    Q = np.array([[1.0, 0.0]])
    Z = n1 * math.exp(a) + n2
    hi = math.exp(a) / Z
    for tau in (0.3, 0.8, 0.95):
        if tau <= n1 * hi:
            n = math.ceil(tau / hi - 1e-12)
        else:
            n = n1 + math.ceil((tau - n1 * hi) * Z - 1e-9)
        assert D.head_density(Q, K, [0], 1.0, tau) == n / (n1 + n2)


def test_conservative_density_quantile():
    # z at 0.95 is 1.6448536...; at alpha = 0.5 the quantile is the mean
    s = [0.2, 0.3, 0.25, 0.35]
    mu = sum(s) / 4
    sd = math.sqrt(sum((x - mu) ** 2 for x in s) / 4)
    r = D.conservative_density(s, 0.95)
    assert abs(r["density"] - (mu + 1.6448536269514722 * sd)) < 1e-12
    assert abs(r["sparsity"] - (1 - r["density"])) < 1e-15
    assert abs(D.conservative_density(s, 0.5)["density"] - mu) < 1e-15
    assert D.conservative_density([0.99, 0.5], 0.999)["density"] == 1.0  # clipped


def test_coclustering_partition_is_a_joint_fixed_point():
    """The co-clustering partition at convergence: key labels are the nearest
    key-block centres in the space of affinities to the query blocks' mean
    rows, and query labels the nearest query-block centres in the space of
    affinities to the key blocks' mean rows; recomputed with loops from the
    labels alone."""
    w = synth.custom("cocl", 1, (2, 4, 8), 16, "f32", n_comp=6, sigma=0.4, noise_var=0.05, Ck=6,
                     Cq=4, Ms=32, n_eig=16, kmeans_iters=200, M=8, r=4, seed=3, keep=0.5)
    q, k, v = synth.generate(w)
    q, k, v = synth.as_f64(q[0]), synth.as_f64(k[0]), synth.as_f64(v[0])
    p = dict(w.params(), partition="coclustering")
    res = O.run_head(q, k, v, p, 0)
    assert res.info["key_passes"] < w.kmeans_iters
    lk, lq = res.label_k, res.label_q
    assert len(set(lk.tolist())) == w.Ck and len(set(lq.tolist())) == w.Cq
    s = 1.0 / math.sqrt(w.d)

    def means(X, lab, C):
        return [[sum(X[i][a] for i in range(len(X)) if lab[i] == c) / int((lab == c).sum())
                 for a in range(len(X[0]))] for c in range(C)]

    def check(X, lab, C, anchors):
        P = [[s * sum(X[i, a] * anchors[c][a] for a in range(w.d)) for c in range(len(anchors))]
             for i in range(w.N)]
        Pb = means(P, lab, C)
        for i in range(w.N):
            dist = [sum((P[i][j] - Pb[c][j]) ** 2 for j in range(len(anchors))) for c in range(C)]
            assert dist[lab[i]] <= min(dist) + 1e-9 * max(1.0, min(dist)), i

    check(k, lk, w.Ck, means(q, lq, w.Cq))
    check(q, lq, w.Cq, means(k, lk, w.Ck))
    assert np.all(np.isfinite(res.out))
