"""GPU parity of the structural diagnostics ("Partition the Support,
Reconstruct the Residual", section 3 structural analysis, section 4
ablations) against the diagnostics oracle.

sparsepr_probe_diagnostics: retained dense mass and sparse-vs-dense error of
every probe row, and the probe residual's energy split. Two checks:
  * the kernel's arithmetic, on the very inputs it read (X, R, B, b, V_r from
    the workspace), against the oracle's residual_energy to 1e-10;
  * the whole chain against the oracle run on the same seeded inputs, within
    tolerances derived from the output tolerance (element max-abs 2e-2,
    mean-abs 2e-3): a probe row's error norm to sqrt(d) * 3 * 2e-3, retained
    mass to 1e-3 (it comes from fp32 log-sum-exps of the two passes)."""
import math
import types

import numpy as np
import pytest
import torch

from free_block_sparse_eigenbasis_b200 import synth
from oracle import diagnostics_oracle as D
from oracle import sparsepr_oracle as O
from tests.parity import gpu_run, np_, oracle_head

pytestmark = pytest.mark.gpu

CASES = [
    synth.custom("small_bf16_d128", 2, (4, 16, 32), 128, "bf16", Ck=64, Cq=16, Ms=256,
                 n_eig=8, M=64, r=16, keep=(0.25, 0.4), seed=11),
    synth.custom("text_bf16_d128", 2, (3, 8, 16), 128, "bf16", n_text=40, Ck=24, Cq=6, Ms=128,
                 n_eig=8, M=32, r=8, keep=(0.2, 0.3), seed=21),
    synth.custom("bf16_d64_r40", 1, (3, 8, 16), 64, "bf16", Ck=40, Cq=10, Ms=128, n_eig=8,
                 M=96, r=40, keep=0.3, seed=31),
    synth.workload("tiny"),
]


def _S():
    from free_block_sparse_eigenbasis_b200 import sparsepr as S
    return S


@pytest.mark.parametrize("w", CASES, ids=[x.name for x in CASES])
def test_probe_diagnostics_match_oracle(w):
    S = _S()
    b, (q, k, v) = gpu_run(w)
    p = w.params()
    H, M, d, r = w.H, w.M, w.d, w.r
    mass = torch.empty(H, M, dtype=torch.float64, device="cuda")
    err = torch.empty_like(mass)
    energy = torch.empty(H, 4, dtype=torch.float64, device="cuda")
    S.sparsepr_probe_diagnostics(p, b.probes, mass, err, energy, b.ws)
    torch.cuda.synchronize()
    assert S.sparsepr_read_stats(b.ws)["status"] == 0
    xr = np_(S.workspace_view(b.ws, p, "xr")).reshape(H, 2, M, d)
    vr = np_(S.workspace_view(b.ws, p, "vr")).reshape(H, d, r)
    bm = np_(S.workspace_view(b.ws, p, "bmat")).reshape(H, d, d)
    bb = np_(S.workspace_view(b.ws, p, "bvec")).reshape(H, d)
    for h in range(H):
        # (1) the kernel's arithmetic on its own inputs
        X, R = xr[h, 0], xr[h, 1]
        P = vr[h] @ vr[h].T
        fake = types.SimpleNamespace(o_sparse_probe=X, o_dense_probe=X + R, Vr=vr[h], B=bm[h],
                                     b=bb[h], Bp=bm[h] @ P, bp=bb[h] @ P)
        e = D.residual_energy(fake)
        got = np_(energy[h])
        want = [e["total"], e["explainable"], e["orthogonal_fit"], e["orthogonal_projected"]]
        assert np.allclose(got, want, rtol=1e-10, atol=1e-12), (h, got, want)
        assert np.allclose(np_(err[h]), np.linalg.norm(R, axis=1), rtol=1e-12, atol=1e-14)
        # (2) against the oracle on the same inputs
        res = oracle_head(w, q, k, v, h)
        probes = res.probes
        assert np.array_equal(np_(b.probes[h]), probes)
        res_p = oracle_head(w, q, k, v, h, rows=probes)
        Qp = synth.as_f64(q[h])[res.perm_q]
        Kp = synth.as_f64(k[h])[res.perm_k]
        Vp = synth.as_f64(v[h])[res.perm_k]
        rm = D.retained_mass_and_error(res_p, Qp, Kp, Vp, p)
        assert np.abs(np_(mass[h]) - rm["mass"]).max() <= 1e-3, "retained mass head %d" % h
        assert np.abs(np_(err[h]) - rm["error"]).max() <= math.sqrt(d) * 3 * 2e-3
        # the diagnostic's message: retained mass does not bound the error
        assert np.all((np_(mass[h]) > 0) & (np_(mass[h]) <= 1 + 1e-6))


@pytest.mark.parametrize("tau", [0.9, 0.5])
@pytest.mark.parametrize("w", CASES, ids=[x.name for x in CASES])
def test_support_expansion_matches_oracle(w, tau):
    """Individual support sizes (their mean per group) and the union size of
    every video query group, bit for bit: both sides decide with fp64 masses
    from exact logits."""
    S = _S()
    b, (q, k, v) = gpu_run(w)
    p = w.params()
    H, Cq = w.H, w.Cq
    indiv = torch.empty(H, Cq, dtype=torch.float64, device="cuda")
    agg = torch.empty_like(indiv)
    S.sparsepr_support_expansion(b.qp, b.kp, p, b.off_q, b.off_k, tau, 1, indiv, agg, b.ws)
    torch.cuda.synchronize()
    for h in range(H):
        res = oracle_head(w, q, k, v, h, rows=np.zeros(0, dtype=np.int64))
        Qp = synth.as_f64(q[h])[res.perm_q]
        Kp = synth.as_f64(k[h])[res.perm_k]
        se = D.support_expansion(res, Qp, Kp, p, tau)
        assert np.array_equal(np_(agg[h]), se["aggregate"]), "aggregate head %d" % h
        assert np.array_equal(np_(indiv[h]), se["individual"]), "individual head %d" % h
    # sampling every 3rd group leaves the others NaN and the sampled ones equal
    indiv3 = torch.empty_like(indiv)
    agg3 = torch.empty_like(indiv)
    S.sparsepr_support_expansion(b.qp, b.kp, p, b.off_q, b.off_k, tau, 3, indiv3, agg3, b.ws)
    torch.cuda.synchronize()
    g = np.arange(Cq)
    assert np.all(np.isnan(np_(agg3)[:, g % 3 != 0]))
    assert np.array_equal(np_(agg3)[:, g % 3 == 0], np_(agg)[:, g % 3 == 0])


@pytest.mark.parametrize("w", CASES, ids=[x.name for x in CASES])
def test_density_profile_matches_oracle(w):
    """Mean tau-mass density of sampled rows per head: the count of weights
    summed over the rows equals the oracle's exactly."""
    S = _S()
    q, k, v = synth.generate(w)
    p = w.params()
    ws = torch.empty(S.workspace_bytes(p), dtype=torch.uint8, device="cuda")
    dens = torch.empty(w.H, dtype=torch.float64, device="cuda")
    stride = 3
    for tau in (0.95, 0.5):
        S.sparsepr_density_profile(q.cuda(), k.cuda(), p, tau, stride, dens, ws)
        torch.cuda.synchronize()
        rows = np.arange(0, w.Nv, stride)
        for h in range(w.H):
            Q, K = synth.as_f64(q[h]), synth.as_f64(k[h])
            want = D.head_density(Q, K, rows, 1 / math.sqrt(w.d), tau)
            got = float(dens[h])
            assert round(got * rows.size * w.N) == round(want * rows.size * w.N), (h, tau, got, want)
            assert abs(got - want) <= 1e-12
