"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs. Integer outputs (labels, permutations, offsets, routes,
probes, pair counts) must match bit for bit; float outputs must lie within
max-abs 2e-2 and mean-abs 2e-3."""
import math

import numpy as np
import pytest
import torch

from free_block_sparse_eigenbasis_b200 import synth
from oracle import sparsepr_oracle as O
from tests.parity import (MAX_ABS, MEAN_ABS, assert_close, compare_head, gpu_run, np_,
                          oracle_head)

pytestmark = pytest.mark.gpu


def _S():
    from free_block_sparse_eigenbasis_b200 import sparsepr as S
    return S


def test_tiny_full_pipeline():
    w = synth.workload("tiny")
    b, (q, k, v) = gpu_run(w)
    res = oracle_head(w, q, k, v, 0)
    compare_head(b, res, w, 0, None)
    st = _S().sparsepr_read_stats(b.ws)
    assert st["status"] == 0
    assert st["key_passes"][0] == res.info["key_passes"]
    assert st["query_passes"][0] == res.info["query_passes"]
    assert st["near_ties"] == [res.info["key_near_ties"], res.info["query_near_ties"]]
    # the fitted map
    fit = np_(b.fit[0])
    d = w.d
    assert np.abs(fit[:d * d].reshape(d, d) - res.Bp).max() < 5e-2 * max(1.0, np.abs(res.Bp).max())


@pytest.mark.parametrize("fill", [0x00, 0xFF, 0x5A])
def test_tiny_result_independent_of_prior_memory(fill):
    """The whole call on buffers pre-filled with one byte pattern (0xFF makes
    every double a NaN, 0x5A a huge finite value): integer outputs and
    outputs must equal the oracle's whatever the memory held before."""
    w = synth.workload("tiny")
    b, (q, k, v) = gpu_run(w, fill=fill)
    res = oracle_head(w, q, k, v, 0)
    compare_head(b, res, w, 0, None)
    assert _S().sparsepr_read_stats(b.ws)["status"] == 0


SMALL = [
    # several query tiles per group, ragged tails, two heads with different budgets
    synth.custom("small_bf16_d128", 2, (4, 16, 32), 128, "bf16", Ck=64, Cq=16, Ms=256,
                 n_eig=8, M=64, r=16, keep=(0.25, 0.4), seed=11),
    # fp32 input, d=64, N not a multiple of 8 or 128
    synth.custom("small_f32_d64", 1, (3, 7, 11), 64, "f32", Ck=12, Cq=5, Ms=64, n_eig=4,
                 M=20, r=8, keep=0.3, seed=5),
    # keep = 1: the sparse path is dense attention
    synth.custom("keep_one", 1, (2, 8, 16), 128, "bf16", Ck=16, Cq=4, Ms=64, n_eig=4, M=16,
                 r=8, keep=1.0, seed=3),
    # one key group kept, no probes (hard-drop: output = sparse output)
    synth.custom("hard_drop", 1, (2, 8, 16), 128, "bf16", Ck=16, Cq=4, Ms=64, n_eig=4, M=0,
                 r=8, keep=0.05, seed=4),
    # trailing text tokens: an always-kept key group and a dense query group,
    # never probed or corrected (HunyuanVideo-shaped joint attention)
    synth.custom("text_bf16_d128", 2, (3, 8, 16), 128, "bf16", n_text=40, Ck=24, Cq=6, Ms=128,
                 n_eig=8, M=32, r=8, keep=(0.2, 0.3), seed=21),
    synth.custom("text_f32_d64_hard_drop", 1, (2, 5, 13), 64, "f32", n_text=9, Ck=10, Cq=4,
                 Ms=64, n_eig=4, M=0, r=4, keep=0.25, seed=22),
    # bf16 d=64 with e=24: 64-column operand rows on both tensor-core assignment passes
    synth.custom("bf16_d64_e24", 1, (3, 8, 16), 64, "bf16", Ck=40, Cq=10, Ms=128, n_eig=24,
                 M=24, r=8, keep=0.3, seed=31),
    # residual subspace ranks past one inverse-iteration batch (r = 48) and past
    # the tridiagonal solver (r = 96: cyclic Jacobi)
    synth.custom("rank48", 1, (4, 8, 16), 128, "bf16", Ck=32, Cq=8, Ms=128, n_eig=8, M=128,
                 r=48, keep=0.3, seed=41),
    synth.custom("rank96", 1, (4, 8, 16), 128, "bf16", Ck=32, Cq=8, Ms=128, n_eig=8, M=128,
                 r=96, keep=0.3, seed=42),
]


@pytest.mark.parametrize("w", SMALL, ids=[x.name for x in SMALL])
def test_small_full_pipeline(w):
    b, (q, k, v) = gpu_run(w, fill=0xFF)
    ties = [0, 0]
    for h in range(w.H):
        res = oracle_head(w, q, k, v, h)
        compare_head(b, res, w, h, None)
        ties[0] += res.info["key_near_ties"]
        ties[1] += res.info["query_near_ties"]
    st = _S().sparsepr_read_stats(b.ws)
    assert st["status"] == 0
    assert st["near_ties"] == ties


def test_keep_one_matches_dense_attention():
    w = SMALL[2]
    b, (q, k, v) = gpu_run(w)
    D = O.dense_attention(synth.as_f64(q[0]), synth.as_f64(k[0]), synth.as_f64(v[0]),
                          1 / math.sqrt(w.d))
    assert_close(np_(b.out[0].float()), D, "keep=1 vs dense")


def test_attention_kernel_on_oracle_routes():
    """The attention call alone, fed the oracle's permutation and routes."""
    S = _S()
    w = SMALL[0]
    q, k, v = synth.generate(w)
    p = w.params()
    b = S.allocate(p, q.dtype)
    for h in range(w.H):
        res = oracle_head(w, q, k, v, h)
        b.qp[h].copy_(q[h][torch.from_numpy(res.perm_q)].cuda())
        b.kp[h].copy_(k[h][torch.from_numpy(res.perm_k)].cuda())
        b.vp[h].copy_(v[h][torch.from_numpy(res.perm_k)].cuda())
        b.off_q[h].copy_(torch.from_numpy(res.off_q).int())
        b.off_k[h].copy_(torch.from_numpy(res.off_k).int())
        b.csr[h].fill_(-1)
        b.csr[h][:, :res.k].copy_(torch.from_numpy(res.csr).int())
        b.k_per_head[h] = res.k
    S.sparsepr_block_sparse_attn(b.qp, b.kp, b.vp, p, b.off_q, b.off_k, b.csr, b.k_per_head,
                                 b.o_sparse, b.pairs_sparse, b.ws)
    torch.cuda.synchronize()
    for h in range(w.H):
        res = oracle_head(w, q, k, v, h)
        assert int(b.pairs_sparse[h]) == res.pairs_sparse
        assert_close(np_(b.o_sparse[h]), res.o_sparse, "o_sparse head %d" % h)


@pytest.mark.parametrize("N", [16, 130, 1000, 4096 + 40])
def test_dense_mode_against_textbook_attention(N):
    S = _S()
    g = torch.Generator().manual_seed(N)
    q = torch.randn(2, N, 128, generator=g).bfloat16()
    k = torch.randn(2, N, 128, generator=g).bfloat16()
    v = torch.randn(2, N, 128, generator=g).bfloat16()
    out = torch.empty(2, N, 128, device="cuda")
    S.dense_attention(q.cuda(), k.cuda(), v.cuda(), out)
    torch.cuda.synchronize()
    for h in range(2):
        D = O.dense_attention(q[h].double().numpy(), k[h].double().numpy(), v[h].double().numpy(),
                              1 / math.sqrt(128))
        assert_close(np_(out[h]), D, "dense N=%d head %d" % (N, h))


@pytest.mark.parametrize("N", [1024, 1124])
def test_dense_mode_logit_jumps_move_the_reference(N):
    """Keys whose logits exceed those of the first key tile by far more than
    2^32 in probability (in the first and in the second half of later tiles,
    and again further on): the online softmax moves its reference maximum
    and rescales the stored values, O and the row sum; the result must still
    be the textbook softmax attention. N = 1124 ends with a unit of one query
    tile, whose two warpgroups split the key tiles and merge at the end."""
    S = _S()
    d = 128
    g = torch.Generator().manual_seed(7)
    q = torch.randn(2, N, d, generator=g)
    k = torch.randn(2, N, d, generator=g)
    v = torch.randn(2, N, d, generator=g)
    q[:, :, 0] += 6.0
    k[:, 128 + 70, 0] += 120.0  # tile 1, second half of its columns
    k[:, 256 + 10, 0] += 120.0  # tile 2, first half
    k[:, 640 + 100, 0] += 240.0  # tile 5: a further jump
    k[1, 900, 0] -= 200.0  # a logit far below the reference
    q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
    out = torch.empty(2, N, d, device="cuda")
    S.dense_attention(q.cuda(), k.cuda(), v.cuda(), out)
    torch.cuda.synchronize()
    for h in range(2):
        D = O.dense_attention(q[h].double().numpy(), k[h].double().numpy(), v[h].double().numpy(),
                              1 / math.sqrt(d))
        assert_close(np_(out[h]), D, "logit jumps head %d" % h)


def test_wan13b_480p_first_and_last_head():
    w = synth.workload("wan13b_480p")
    b, (q, k, v) = gpu_run(w)
    rows = np.arange(0, w.N, 61)
    for h in (0, w.H - 1):
        res = oracle_head(w, q, k, v, h, rows=rows)
        compare_head(b, res, w, h, rows)
    assert _S().sparsepr_read_stats(b.ws)["status"] == 0


def test_wan13b_720p_head0_sampled():
    """The benchmark's workload and launch configuration: all 12 heads on the
    GPU, head 0 checked against the oracle on sampled rows."""
    w = synth.workload("wan13b_720p")
    b, (q, k, v) = gpu_run(w)
    rows = np.arange(7, w.N, 149)
    res = oracle_head(w, q, k, v, 0, rows=rows)
    compare_head(b, res, w, 0, rows)
    st = _S().sparsepr_read_stats(b.ws)
    assert st["status"] == 0
    # every head: a valid partition and exact pair accounting from its own routes
    for h in range(w.H):
        off_q, off_k = np_(b.off_q[h]), np_(b.off_k[h])
        assert off_q[-1] == w.N and off_k[-1] == w.N
        lab = np_(b.label_q[h])
        assert np.array_equal(np.diff(off_q), np.bincount(lab, minlength=w.Cq))
        csr = np_(b.csr[h])[:, :int(b.k_per_head[h])]
        nk = np.diff(off_k)
        pairs = int((np.diff(off_q) * nk[csr].sum(axis=1)).sum())
        assert pairs == int(b.pairs_sparse[h]) == st["pairs_sparse"][h]
        assert int(b.pairs_exec[h]) == pairs + w.M * w.N


def _check_partition_and_pairs(b, w, st, heads):
    """A valid partition per head and, for video-only layers, exact pair
    accounting from the head's own routes."""
    for h in heads:
        off_q, off_k = np_(b.off_q[h]), np_(b.off_k[h])
        assert off_q[-1] == w.N and off_k[-1] == w.N
        lab = np_(b.label_q[h])
        assert np.array_equal(np.diff(off_q), np.bincount(lab, minlength=len(off_q) - 1))
        if w.n_text == 0:
            csr = np_(b.csr[h])[:, :int(b.k_per_head[h])]
            nk = np.diff(off_k)
            pairs = int((np.diff(off_q) * nk[csr].sum(axis=1)).sum())
            assert pairs == int(b.pairs_sparse[h]) == st["pairs_sparse"][h]
            assert int(b.pairs_exec[h]) == pairs + w.M * w.N


def test_wan14b_720p_all_heads_in_one_call():
    """Wan2.1-14B-shaped layer: all 40 heads in one call, with their per-head
    keep fractions drawn from [0.15, 0.35]; the first and last heads and the
    heads with the smallest and the largest budget checked against the
    oracle on sampled rows, every head for a valid partition and exact pair
    accounting."""
    w = synth.workload("wan14b_720p")
    assert w.H == 40
    b, (q, k, v) = gpu_run(w)
    st = _S().sparsepr_read_stats(b.ws)
    assert st["status"] == 0
    rows = np.arange(11, w.N, 997)
    keep = np.asarray(w.keep)
    for h in sorted({0, w.H - 1, int(keep.argmin()), int(keep.argmax())}):
        res = oracle_head(w, q, k, v, h, rows=rows)
        compare_head(b, res, w, h, rows)
    _check_partition_and_pairs(b, w, st, range(w.H))


def test_hunyuan13b_720p_text_sampled():
    """HunyuanVideo-shaped joint attention (its first 4 of 24 heads): 118,800
    video tokens and 256 always-kept text tokens, 1500 key and 300 query
    groups; head 0 checked against the oracle on sampled video rows and text
    rows (the text query group is last in group-major order)."""
    w = synth.workload("hunyuan13b_720p", heads=4)
    b, (q, k, v) = gpu_run(w)
    st = _S().sparsepr_read_stats(b.ws)
    assert st["status"] == 0
    rows = np.concatenate([np.arange(5, w.Nv, 601), np.arange(w.N - w.n_text, w.N, 17)])
    res = oracle_head(w, q, k, v, 0, rows=rows)
    compare_head(b, res, w, 0, rows)
    _check_partition_and_pairs(b, w, st, range(w.H))


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    """A wait on a barrier that nothing completes gives up after the limit and
    sets the TIMEOUT bit; the next call on the same context runs normally."""
    S = _S()
    w = SMALL[0]
    p = w.params()
    ws = torch.zeros(S.workspace_bytes(p), dtype=torch.uint8, device="cuda")
    S.sparsepr_reset_stats(ws)
    S.sparsepr_check_wait_limit(ws)
    torch.cuda.synchronize()
    st = S.sparsepr_read_stats(ws)
    assert st["status"] & (1 << S.ERR_TIMEOUT)
    b, (q, k, v) = gpu_run(w)  # partition resets the status word at the start of its call
    assert S.sparsepr_read_stats(b.ws)["status"] == 0
    res = oracle_head(w, q, k, v, 0)
    compare_head(b, res, w, 0, None)


def test_multisection_reciprocal_within_two_ulp():
    """The reciprocal in the eigenvalue multisection's Sturm counts (an
    approximate reciprocal refined by two Newton-Raphson steps, not correctly
    rounded) against CUDA's correctly rounded one: within 2 ulp over random
    mantissas across the normal range, both signs, powers of two and the
    magnitudes the counts meet (pivots down to the safe minimum times the
    largest squared off-diagonal)."""
    S = _S()
    g = torch.Generator().manual_seed(7)
    n = 1 << 20
    mant = 1.0 + torch.rand(n, generator=g, dtype=torch.float64)
    expo = torch.randint(-1020, 1020, (n,), generator=g)
    sign = torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0).double()
    x = sign * torch.ldexp(mant, expo)
    special = torch.tensor([1.0, -1.0, 2.0, 0.5, 3.0, 1.0 / 3.0, 2.2250738585072014e-308,
                            -2.2250738585072014e-308, 4.0 * 2.2250738585072014e-308,
                            1.7976931348623157e+308 / 4.0, 0.1, -7.0, 1e-300, 1e300],
                           dtype=torch.float64)
    xd = torch.cat([x, special]).cuda()
    err = S.sparsepr_check_reciprocal(xd)
    torch.cuda.synchronize()
    e = err.cpu()
    assert torch.isfinite(e).all()
    assert e.max().item() <= 2.0, e.max().item()
