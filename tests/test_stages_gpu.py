"""GPU stage-level parity of the partition ("Partition the Support, Reconstruct
the Residual", 2.A, response-coupled partitioning): each intermediate result
the library leaves in its workspace after sparsepr_partition, read through
sparsepr_workspace_region, against the fp64 oracle's value of the same step on
the same seeded inputs. A mismatch in the end-to-end labels then points at one
kernel: the sampled-query metric M_K, its leading eigenpairs (eigenvectors up
to sign), the key projector, the key response coordinates z, the K group
means C_K over the final key labels and the query metric G = scale^2 C_K^T C_K.

Tolerances follow the fp64 arithmetic: sums over at most a few thousand terms
(relative 1e-12), eigenvalues to 1e-12 of the largest, eigenvectors to
1e-13 * lambda_max / gap (the perturbation bound of an eigenvector whose
eigenvalue lies `gap` away from the rest of the spectrum). Each comparison is
also shown to reject the oracle's value with a planted relative error of
1e-9, so a wrong scale or a dropped term cannot pass."""
import math

import numpy as np
import pytest
import torch

from free_block_sparse_eigenbasis_b200 import synth
from oracle import sparsepr_oracle as O

pytestmark = pytest.mark.gpu

CASES = [
    synth.workload("tiny"),
    synth.custom("small_f32_d64", 1, (3, 7, 11), 64, "f32", Ck=12, Cq=5, Ms=64, n_eig=4,
                 M=20, r=8, keep=0.3, seed=5),
    synth.custom("small_bf16_d128", 2, (4, 16, 32), 128, "bf16", Ck=64, Cq=16, Ms=256,
                 n_eig=8, M=64, r=16, keep=(0.25, 0.4), seed=11),
    synth.custom("bf16_d64_e24", 1, (3, 8, 16), 64, "bf16", Ck=40, Cq=10, Ms=128, n_eig=24,
                 M=24, r=8, keep=0.3, seed=31),
    synth.custom("text_bf16_d128", 2, (3, 8, 16), 128, "bf16", n_text=40, Ck=24, Cq=6, Ms=128,
                 n_eig=8, M=32, r=8, keep=(0.2, 0.3), seed=21),
    synth.workload("wan13b_480p"),
]


def _S():
    from free_block_sparse_eigenbasis_b200 import sparsepr as S
    return S


def rel(got, want):
    return float(np.abs(got - want).max() / max(np.abs(want).max(), 1e-300))


def check_rel(got, want, tol, what):
    err = rel(got, want)
    assert err <= tol, "%s: relative error %.3e > %.1e" % (what, err, tol)
    planted = rel(got, want * (1 + 1e-9))
    assert planted > tol, "%s: a planted 1e-9 scale error passes (%.3e)" % (what, planted)


def run_partition(w):
    S = _S()
    q, k, v = synth.generate(w)
    p = w.params()
    b = S.allocate(p, q.dtype)
    b.ws.fill_(0xFF)  # nothing the stages read may come from before the call
    S.sparsepr_partition(q.cuda(), k.cuda(), p, b.label_q, b.label_k, b.ws)
    torch.cuda.synchronize()
    assert S.sparsepr_read_stats(b.ws)["status"] == 0
    regions = {n: S.workspace_view(b.ws, p, n).cpu().numpy()
               for n in ("mk", "eval", "evec", "wk", "z", "ck", "g", "init_k", "init_q")}
    return b, q, k, p, regions


@pytest.mark.parametrize("w", CASES, ids=[x.name for x in CASES])
def test_partition_stages_match_oracle(w):
    b, q, k, p, R = run_partition(w)
    H, d, e, Nv, Ck, Cq = w.H, w.d, w.n_eig, w.Nv, w.Ck, w.Cq
    scale = 1.0 / math.sqrt(d)
    heads = [0, H - 1] if H > 2 else range(H)
    for h in heads:
        qv = synth.as_f64(q[h])[:Nv]
        kv = synth.as_f64(k[h])[:Nv]
        # initial centroid rows: the partial Fisher-Yates draws, bit-exact
        assert np.array_equal(R["init_k"].reshape(H, Ck)[h], O.init_indices(Nv, Ck, w.seed, h, 0))
        assert np.array_equal(R["init_q"].reshape(H, Cq)[h], O.init_indices(Nv, Cq, w.seed, h, 1))
        # M_K from the sampled queries
        MK = O.metric_MK(qv, w.Ms)
        check_rel(R["mk"].reshape(H, d, d)[h], MK, 1e-12, "M_K head %d" % h)
        # leading eigenpairs
        lam, U = O.eigenbasis(MK, e)
        spec = np.sort(np.linalg.eigvalsh(MK))[::-1]
        ev = R["eval"].reshape(H, e)[h]
        assert np.abs(ev - lam).max() <= 1e-12 * spec[0], ("eigenvalues", h, ev - lam)
        assert np.abs(ev - lam * (1 + 1e-9)).max() > 1e-12 * spec[0]
        evec = R["evec"].reshape(H, d, e)[h]
        sgn = np.sign((evec * U).sum(axis=0))
        assert np.all(sgn != 0)
        for j in range(e):
            gap = min(abs(spec[j] - spec[i]) for i in range(d) if i != j)
            tol = 1e-13 * spec[0] / max(gap, 1e-300) + 1e-14
            err = np.abs(evec[:, j] * sgn[j] - U[:, j]).max()
            assert err <= tol, ("eigenvector", h, j, err, tol)
            assert abs(np.linalg.norm(evec[:, j]) - 1.0) < 1e-13
        # key projector W_K = U_e Lambda_e^{1/2} (the GPU's own eigenvectors)
        wk = R["wk"].reshape(H, d, e)[h]
        check_rel(wk, evec * np.sqrt(np.maximum(ev, 0.0))[None, :], 1e-14, "W_K head %d" % h)
        # key response coordinates z = W_K^T k: against the GPU's projector
        # exactly, and against the oracle's coordinates up to the column signs
        z = R["z"].reshape(H, Nv, e)[h]
        check_rel(z, kv @ wk, 1e-13, "z head %d" % h)
        Z = O.key_coordinates(kv, lam, U)
        zt = max(1e-13 * spec[0] / min(abs(spec[j] - spec[i]) for j in range(e)
                                      for i in range(d) if i != j), 1e-12)
        assert rel(z * sgn[None, :], Z) <= zt * math.sqrt(d), ("z vs oracle", h)
        # final key labels, K group means in the original space and G
        labels, _ = O.key_partition(kv, qv, Ck, w.Ms, e, w.kmeans_iters, w.seed, h)
        assert np.array_equal(b.label_k[h, :Nv].cpu().numpy(), labels), "key labels head %d" % h
        CK = O.group_means(kv, labels, Ck)
        check_rel(R["ck"].reshape(H, Ck, d)[h], CK, 1e-12, "C_K head %d" % h)
        check_rel(R["g"].reshape(H, d, d)[h], scale * scale * (CK.T @ CK), 1e-12, "G head %d" % h)


def _bf16_rne(x):
    """fp64 -> nearest bf16 value (ties to even), as fp64; normal range."""
    b = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    half = np.uint64((1 << 44) - 1) + ((b >> np.uint64(45)) & np.uint64(1))
    r = (b + half) & ~np.uint64((1 << 45) - 1)
    return r.view(np.float64)


PLANE_CASES = [
    synth.custom("planes_bf16_d128_e16", 2, (4, 16, 32), 128, "bf16", Ck=64, Cq=16, Ms=256,
                 n_eig=16, M=64, r=16, keep=0.3, seed=13),
    synth.workload("wan13b_480p"),
]


@pytest.mark.parametrize("w", PLANE_CASES, ids=[x.name for x in PLANE_CASES])
def test_key_planes_and_norms_from_z(w):
    """The bf16 planes of the key coordinates (written by the projection
    itself for e = 16) are z split exactly: plane 1 is the nearest bf16 of
    z, plane 2 of what it leaves, plane 3 of what both leave; the stored row
    norms bound |z| from above by at most 1e-6 relative plus float rounding."""
    S = _S()
    b, q, k, p, R = run_partition(w)
    H, Nv, e = w.H, w.Nv, w.n_eig
    assert e == 16
    z = R["z"].reshape(H * Nv, e)
    planes = S.workspace_view(b.ws, p, "zplanes").float().cpu().numpy().astype(np.float64)
    planes = planes.reshape(3, H * Nv, 16)
    rest = z.copy()
    for pl in range(3):
        want = _bf16_rne(rest)
        assert np.array_equal(planes[pl], want), ("plane", pl, np.abs(planes[pl] - want).max())
        rest = rest - want
    # a planted one-ulp change of one element in the first plane is seen
    bad = planes[0].copy()
    bad[0, 0] = np.nextafter(np.float32(bad[0, 0]), np.float32(np.inf))
    assert not np.array_equal(bad, _bf16_rne(z))
    xn = S.workspace_view(b.ws, p, "xnk").cpu().numpy().astype(np.float64)
    nz = np.sqrt((z * z).sum(axis=1))
    assert (xn >= nz * (1 - 1e-12)).all()
    assert (xn <= nz * (1 + 1e-6) * (1 + 2.0 ** -23) + 1e-300).all()
