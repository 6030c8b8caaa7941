"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and compare."""
import math

import numpy as np
import torch

from free_block_sparse_eigenbasis_b200 import synth
from oracle import sparsepr_oracle as O

# Output tolerances for unit-variance bf16 inputs with fp32 accumulation.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def gpu_run(w, q=None, k=None, v=None, with_fit=True, fill=None):
    """Full path on the GPU; returns (buffers, q, k, v) with q/k/v on CPU.
    fill: a byte written over every buffer of the call (workspace and
    outputs) before it, so that a read of memory the call did not write
    shows up as a mismatch."""
    from free_block_sparse_eigenbasis_b200 import sparsepr as S
    if q is None:
        q, k, v = synth.generate(w)
    p = w.params()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    b = S.allocate(p, qd.dtype, with_fit=with_fit)
    if fill is not None:
        for t in vars(b).values():
            if isinstance(t, torch.Tensor):
                t.view(torch.uint8).fill_(fill)
    S.attention(qd, kd, vd, p, b)
    torch.cuda.synchronize()
    return b, (q, k, v)


def np_(t):
    return t.detach().cpu().numpy()


def oracle_head(w, q, k, v, h, rows=None):
    return O.run_head(synth.as_f64(q[h]), synth.as_f64(k[h]), synth.as_f64(v[h]), w.params(), h,
                      rows=rows)


def assert_close(got, want, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), what + ": non-finite values"
    err = np.abs(got - want)
    assert err.max() <= max_abs, "%s: max-abs %.3e > %.1e" % (what, err.max(), max_abs)
    assert err.mean() <= mean_abs, "%s: mean-abs %.3e > %.1e" % (what, err.mean(), mean_abs)
    return float(err.max()), float(err.mean())


def compare_head(b, res, w, h, check_rows):
    """Bit-exact integer outputs and tolerance-checked float outputs of head h."""
    Nv = w.Nv
    assert np.array_equal(np_(b.label_k[h]), res.label_k), "label_k head %d" % h
    assert np.array_equal(np_(b.label_q[h]), res.label_q), "label_q head %d" % h
    assert np.array_equal(np_(b.perm_q[h]), res.perm_q)
    assert np.array_equal(np_(b.perm_k[h]), res.perm_k)
    assert np.array_equal(np_(b.off_q[h]), res.off_q)
    assert np.array_equal(np_(b.off_k[h]), res.off_k)
    assert int(b.k_per_head[h]) == res.k
    csr = np_(b.csr[h])
    assert np.array_equal(csr[:, :res.k], res.csr), "csr head %d" % h
    assert np.all(csr[:, res.k:] == -1)
    if w.M > 0:
        assert np.array_equal(np_(b.probes[h]), res.probes), "probes head %d" % h
    assert int(b.pairs_sparse[h]) == res.pairs_sparse
    assert int(b.pairs_exec[h]) == res.pairs_exec
    rows = res.rows
    os_gpu = np_(b.o_sparse[h])[rows]
    e1 = assert_close(os_gpu, res.o_sparse, "o_sparse head %d" % h)
    out_gpu = np_(b.out[h].float())[res.perm_q[rows]]
    e2 = assert_close(out_gpu, res.out, "out head %d" % h)
    return e1, e2
