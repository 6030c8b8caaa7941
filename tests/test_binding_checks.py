"""The Python binding checks every tensor argument (shape, dtype, row-major
layout, device) before the C ABI sees a bare pointer. CPU only: the library's
compute entry points are replaced by a recorder, and the buffers that
`allocate` makes must pass every check of every call."""
import ctypes

import pytest
import torch

from free_block_sparse_eigenbasis_b200 import sparsepr as S
from free_block_sparse_eigenbasis_b200 import synth


class _Stream:
    cuda_stream = 0


class _Recorder:
    """Stands in for the library's enqueueing calls; sizing calls go to the
    real library."""

    def __init__(self, real):
        self.real, self.calls = real, []

    def __getattr__(self, name):
        if name in ("sparsepr_workspace_bytes", "sparsepr_route_width", "sparsepr_status_string"):
            return getattr(self.real, name)

        def rec(*args):
            self.calls.append((name, args))
            return S.OK
        return rec


@pytest.fixture
def host_lib(monkeypatch):
    rec = _Recorder(S.lib)
    monkeypatch.setattr(S, "lib", rec)
    monkeypatch.setattr(S, "_DEVICE_TYPE", "cpu")
    return rec


@pytest.mark.parametrize("name,dtype", [("tiny", torch.float32), ("small_text", torch.bfloat16)])
def test_allocated_buffers_pass_every_check(host_lib, name, dtype):
    if name == "tiny":
        w = synth.workload("tiny")
    else:
        w = synth.custom("small_text", 2, (2, 8, 8), 128, "bf16", n_text=16, Ck=12, Cq=6, Ms=32,
                         n_eig=4, M=0, r=4, keep=(0.25, 0.5))
    p = w.params()
    q = torch.zeros((w.H, w.N, w.d), dtype=dtype)
    b = S.allocate(p, dtype, "cpu", with_fit=True)
    S.attention(q, q.clone(), q.clone(), p, b, stream=_Stream())
    names = [c[0] for c in host_lib.calls]
    assert names == ["sparsepr_partition", "sparsepr_permute", "sparsepr_route",
                     "sparsepr_block_sparse_attn", "sparsepr_probe_correct"]
    # the byte count handed over is the workspace's size
    assert host_lib.calls[0][1][-2] == b.ws.numel()
    S.sparsepr_route_noalloc(b.qp, b.kp, p, b.off_q, b.off_k, b.csr, b.k_per_head, _Stream())
    S.sparsepr_reset_stats(b.ws, _Stream())
    S.sparsepr_check_wait_limit(b.ws, _Stream())


def test_dense_mode_buffers_pass_every_check(host_lib):
    q = torch.zeros((2, 100, 64), dtype=torch.bfloat16)
    out = torch.empty((2, 100, 64), dtype=torch.float32)
    S.dense_attention(q, q.clone(), q.clone(), out, stream=_Stream())
    assert [c[0] for c in host_lib.calls] == ["sparsepr_block_sparse_attn"]


def _tiny_bufs():
    w = synth.workload("tiny")
    p = w.params()
    q = torch.zeros((w.H, w.N, w.d), dtype=torch.float32)
    return p, q, S.allocate(p, torch.float32, "cpu")


def test_bad_arguments_raise_before_the_library(host_lib):
    p, q, b = _tiny_bufs()
    st = _Stream()
    with pytest.raises(ValueError, match="label_q has shape"):
        S.sparsepr_partition(q, q, p, b.label_q[:, :-1], b.label_k, b.ws, st)
    with pytest.raises(TypeError, match="label_k has dtype"):
        S.sparsepr_partition(q, q, p, b.label_q, b.label_k.long(), b.ws, st)
    with pytest.raises(TypeError, match="k has dtype"):
        S.sparsepr_partition(q, q.bfloat16(), p, b.label_q, b.label_k, b.ws, st)
    with pytest.raises(ValueError, match="contiguous"):
        S.sparsepr_partition(q.transpose(1, 2).contiguous().transpose(1, 2), q, p, b.label_q,
                             b.label_k, b.ws, st)
    with pytest.raises(TypeError, match="ws has dtype"):
        S.sparsepr_partition(q, q, p, b.label_q, b.label_k, b.ws.view(torch.int32), st)
    with pytest.raises(ValueError, match="off_k has shape"):
        S.sparsepr_permute(q, q, q, p, b.label_q, b.label_k, b.perm_q, b.perm_k, b.off_q,
                           b.off_k[:, :-1], b.qp, b.kp, b.vp, b.ws, st)
    with pytest.raises(ValueError, match="csr has shape"):
        S.sparsepr_route(b.qp, b.kp, p, b.off_q, b.off_k, b.csr[:, :, :-1], b.k_per_head, b.ws,
                         st)
    with pytest.raises(TypeError, match="o_sparse has dtype"):
        S.sparsepr_block_sparse_attn(b.qp, b.kp, b.vp, p, b.off_q, b.off_k, b.csr, b.k_per_head,
                                     b.o_sparse.double(), b.pairs_sparse, b.ws, st)
    with pytest.raises(ValueError, match="probes has shape"):
        S.sparsepr_probe_correct(b.qp, b.kp, b.vp, p, b.off_q, b.perm_q, b.o_sparse,
                                 b.pairs_sparse, b.out, b.probes[:, :-1], b.pairs_exec, b.ws,
                                 stream=st)
    with pytest.raises(ValueError, match="fit has shape"):
        S.sparsepr_probe_correct(b.qp, b.kp, b.vp, p, b.off_q, b.perm_q, b.o_sparse,
                                 b.pairs_sparse, b.out, b.probes, b.pairs_exec, b.ws,
                                 fit=torch.empty(1, dtype=torch.float64), stream=st)
    assert host_lib.calls == []


def test_host_tensors_are_rejected():
    # the real device check: CPU tensors never reach the library
    p, q, b = _tiny_bufs()
    with pytest.raises(ValueError, match="CUDA tensor"):
        S.sparsepr_partition(q, q, p, b.label_q, b.label_k, b.ws, _Stream())
    with pytest.raises(ValueError, match="CUDA tensor"):
        S.sparsepr_read_stats(b.ws)


def test_reciprocal_check_rejects_tensors_it_cannot_pass():
    """The reciprocal self-check takes a contiguous 1-D fp64 CUDA tensor only;
    anything else is refused in the binding, before the library is called."""
    for bad in (torch.zeros(4, dtype=torch.float64),                 # host memory
                torch.zeros(4, dtype=torch.float32),
                torch.zeros((2, 2), dtype=torch.float64)):
        with pytest.raises(ValueError):
            S.sparsepr_check_reciprocal(bad)
