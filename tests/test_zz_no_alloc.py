"""GPU test of sparsepr_route_noalloc, the routing call for callers that
cannot allocate device memory or pass a workspace (code that must not
trigger cudaMalloc's implicit device synchronisation, or that lives in a
memory pool reserved up front). Its scratch is a fixed device array inside
the library and it runs the same kernels as sparsepr_route (which uses the
caller's workspace), so its routes must equal those of sparsepr_route bit
for bit on every call, including repeated calls that reuse the array.
Collected last on purpose: it runs after every other test."""
import ctypes

import pytest
import torch

from free_block_sparse_eigenbasis_b200 import synth

pytestmark = pytest.mark.gpu


def _routes_both_ways(w):
    from free_block_sparse_eigenbasis_b200 import sparsepr as S
    q, k, v = synth.generate(w)
    p = w.params()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    b = S.allocate(p, qd.dtype)
    S.sparsepr_partition(qd, kd, p, b.label_q, b.label_k, b.ws)
    S.sparsepr_permute(qd, kd, vd, p, b.label_q, b.label_k, b.perm_q, b.perm_k, b.off_q, b.off_k,
                       b.qp, b.kp, b.vp, b.ws)
    S.sparsepr_route(b.qp, b.kp, p, b.off_q, b.off_k, b.csr, b.k_per_head, b.ws)
    torch.cuda.synchronize()
    ref_csr, ref_k = b.csr.clone(), b.k_per_head.clone()
    outs = []
    for _ in range(2):  # two calls in a row share the library's scratch array
        csr = torch.full_like(b.csr, -7)
        kk = torch.full_like(b.k_per_head, -7)
        S.sparsepr_route_noalloc(b.qp, b.kp, p, b.off_q, b.off_k, csr, kk)
        torch.cuda.synchronize()
        outs.append((csr, kk))
    return ref_csr, ref_k, outs


@pytest.mark.parametrize("name", ["small", "text", "wan13b_480p"])
def test_route_noalloc_matches_route(name):
    if name == "small":
        w = synth.custom("noalloc_small", 2, (4, 16, 32), 128, "bf16", Ck=64, Cq=16, Ms=256,
                         n_eig=8, M=64, r=16, keep=(0.25, 0.4), seed=11)
    elif name == "text":
        # trailing text tokens: offsets carry one extra group per side
        w = synth.custom("noalloc_text", 2, (3, 8, 16), 128, "bf16", n_text=40, Ck=24, Cq=6,
                         Ms=128, n_eig=8, M=32, r=8, keep=(0.2, 0.3), seed=21)
    else:
        # 12 heads of ((100 + 500) * 128 + 100 * 500) * 8 bytes: several head
        # chunks of the array
        w = synth.workload("wan13b_480p")
    ref_csr, ref_k, outs = _routes_both_ways(w)
    for csr, kk in outs:  # integer outputs: bit-exact
        assert torch.equal(csr, ref_csr)
        assert torch.equal(kk, ref_k)


def test_route_noalloc_rejects_oversized_heads():
    from free_block_sparse_eigenbasis_b200 import sparsepr as S
    # one head needs ((4096 + 4096) * 128 + 4096 * 4096) * 8 bytes > the 8 MiB array
    w = synth.custom("too_big", 1, (4, 32, 64), 128, "bf16", Ck=4096, Cq=4096, Ms=64, n_eig=4,
                     M=16, r=8, keep=0.1, seed=1)
    prm, keep = S.make_params(w.params())
    fake = ctypes.c_void_p(1 << 40)  # rejected before anything touches it
    code = S.lib.sparsepr_route_noalloc(fake, fake, S.BF16, ctypes.byref(prm), fake, fake, fake,
                                        fake, None)
    assert code == S.ERR_WORKSPACE
