"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/sparsepr.h declares, sizes its workspace, and
rejects bad arguments before anything is enqueued."""
import ctypes
import os
import re

import pytest

from free_block_sparse_eigenbasis_b200 import sparsepr as S
from free_block_sparse_eigenbasis_b200 import synth
from oracle import sparsepr_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "sparsepr.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sparsepr_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_five_calls():
    names = declared_functions()
    for n in ("sparsepr_partition", "sparsepr_permute", "sparsepr_route",
              "sparsepr_block_sparse_attn", "sparsepr_probe_correct"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(S._LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(declared_functions()) == set(S.EXPORTED)


def test_workspace_regions_lie_inside_the_workspace_and_do_not_overlap():
    w = synth.workload("wan13b_480p")
    p = w.params()
    total = S.workspace_bytes(p)
    d, e, H = w.d, w.n_eig, w.H
    want = dict(init_k=H * w.Ck * 4, init_q=H * w.Cq * 4, mk=H * d * d * 8, eval=H * e * 8,
                evec=H * d * e * 8, wk=H * d * e * 8, z=H * w.Nv * e * 8, ck=H * w.Ck * d * 8,
                g=H * d * d * 8, bmat=H * d * d * 8, bvec=H * d * 8)
    spans = []
    for name, nb in want.items():
        off, got = S.sparsepr_workspace_region(p, name)
        assert got == nb, name
        assert off % 256 == 0 and off + nb <= total, name
        spans.append((off, off + nb, name))
    spans.sort()
    for (a0, a1, n0), (b0, b1, n1) in zip(spans, spans[1:]):
        assert a1 <= b0, (n0, n1)
    for bad in ("", "Z", "mk ", "nope"):
        with pytest.raises(S.SparsePRError) as ei:
            S.sparsepr_workspace_region(p, bad)
        assert ei.value.code == S.ERR_INVALID_ARG


def test_params_struct_layout():
    # 12 int32 + lambda + scale + seed + keep pointer
    assert ctypes.sizeof(S.Params) == 48 + 8 + 8 + 8 + 8
    assert S.Params.lam.offset == 48 and S.Params.keep.offset == 72


def test_workspace_and_route_width():
    for name in ("tiny", "wan13b_480p", "wan13b_720p", "wan14b_720p"):
        w = synth.workload(name)
        p = w.params()
        assert S.workspace_bytes(p) > 0
        assert S.route_width(p) == max(O.keep_budget(k, w.Ck) for k in w.keep)


def test_keep_budget_matches_oracle_on_edge_values():
    base = synth.workload("tiny").params()
    for keep, Ck in [(0.22, 1000), (0.2201, 1000), (1e-6, 1000), (1.0, 16), (0.3333333, 3)]:
        p = dict(base, Ck=Ck, N=4096, keep=[keep])
        assert S.route_width(p) == O.keep_budget(keep, Ck)


@pytest.mark.parametrize("bad", [
    dict(d=96), dict(H=0), dict(H=300), dict(Ck=0), dict(Cq=5000), dict(Ms=0),
    dict(n_eig=0), dict(n_eig=40), dict(M=-1), dict(r=0), dict(r=65), dict(lam=-1.0),
    dict(keep=[0.0]), dict(keep=[1.5]), dict(n_text=-1), dict(n_text=256), dict(kmeans_iters=0),
    dict(N=8),
])
def test_invalid_params_rejected_on_host(bad):
    p = dict(synth.workload("tiny").params(), **bad)
    assert S.workspace_bytes(p) == 0
    prm, keep = S.make_params(p)
    fake = ctypes.c_void_p(1 << 40)  # never dereferenced: the call must fail first
    code = S.lib.sparsepr_partition(fake, fake, S.BF16, ctypes.byref(prm), fake, fake, fake,
                                    1 << 30, None)
    assert code in (S.ERR_INVALID_ARG, S.ERR_UNSUPPORTED)


def test_text_tokens_accepted_and_sized():
    # trailing text tokens add one key group and one query group per head
    p = dict(synth.workload("tiny").params(), n_text=8)
    assert S.workspace_bytes(p) > 0
    assert S.route_width(p) == S.route_width(dict(p, n_text=0))  # routes cover video groups


def test_null_pointers_and_small_workspace_rejected():
    p = synth.workload("tiny").params()
    prm, keep = S.make_params(p)
    fake = ctypes.c_void_p(1 << 40)
    need = S.workspace_bytes(p)
    lib = S.lib
    assert lib.sparsepr_partition(None, fake, S.F32, ctypes.byref(prm), fake, fake, fake, need,
                                  None) == S.ERR_INVALID_ARG
    assert lib.sparsepr_partition(fake, fake, S.F32, ctypes.byref(prm), fake, fake, fake,
                                  need - 1, None) == S.ERR_WORKSPACE
    # misaligned workspace
    assert lib.sparsepr_partition(fake, fake, S.F32, ctypes.byref(prm), fake, fake,
                                  ctypes.c_void_p((1 << 40) + 8), need, None) == S.ERR_WORKSPACE
    assert lib.sparsepr_partition(fake, fake, 7, ctypes.byref(prm), fake, fake, fake, need,
                                  None) == S.ERR_UNSUPPORTED
    assert lib.sparsepr_route(fake, fake, S.F32, ctypes.byref(prm), fake, fake, None, fake, fake,
                              need, None) == S.ERR_INVALID_ARG
    assert lib.sparsepr_block_sparse_attn(fake, fake, fake, S.F32, ctypes.byref(prm), fake, fake,
                                          fake, fake, fake, None, fake, need,
                                          None) == S.ERR_INVALID_ARG
    assert lib.sparsepr_probe_correct(fake, fake, fake, S.F32, ctypes.byref(prm), fake, fake, fake,
                                      fake, fake, None, fake, None, fake, need,
                                      None) == S.ERR_INVALID_ARG
    # permuted outputs may not alias the inputs
    assert lib.sparsepr_permute(fake, fake, fake, S.F32, ctypes.byref(prm), fake, fake, fake, fake,
                                fake, fake, fake, fake, fake, fake, need,
                                None) == S.ERR_INVALID_ARG


def test_status_strings():
    for c in range(7):
        assert S.status_string(c)


def test_header_is_plain_c_and_a_c_program_links_and_runs(tmp_path):
    """The boundary is a C ABI: the header compiles as pedantic C99, and a C
    program links against the library and gets the same host-side answers
    as the Python binding (no GPU needed for these calls)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "abi.c"
    src.write_text(
        '#include <stdio.h>\n#include "sparsepr.h"\n'
        "int main(void) {\n"
        "  double keep[2] = {0.25, 0.4};\n"
        "  sparsepr_params p = {0};\n"
        "  p.H = 2; p.N = 2048; p.d = 128; p.n_text = 0; p.Ck = 64; p.Cq = 16; p.Ms = 256;\n"
        "  p.n_eig = 8; p.kmeans_iters = 10; p.M = 64; p.r = 16; p.lambda = 1e-2; p.scale = 0.0;\n"
        "  p.seed = 11; p.keep = keep;\n"
        '  printf("%zu %d %s\\n", sparsepr_workspace_bytes(&p), (int)sparsepr_route_width(&p),\n'
        "         sparsepr_status_string(SPARSEPR_ERR_TIMEOUT));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "abi"
    pkg = os.path.join(root, "free_block_sparse_eigenbasis_b200")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(root, "include"), str(src), "-L", pkg, "-lsparsepr",
                    "-Wl,-rpath," + pkg, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    p = dict(H=2, N=2048, d=128, n_text=0, Ck=64, Cq=16, Ms=256, n_eig=8, kmeans_iters=10,
             keep=[0.25, 0.4], M=64, r=16, lam=1e-2, scale=0.0, seed=11)
    assert int(out[0]) == S.workspace_bytes(p)
    assert int(out[1]) == S.route_width(p)
    assert " ".join(out[2:]) == S.status_string(S.ERR_TIMEOUT)


def test_route_noalloc_rejects_misaligned_and_oversized_before_any_launch():
    w = synth.custom("noalloc_cpu", 1, (4, 16, 32), 128, "bf16", Ck=64, Cq=16, Ms=256, n_eig=8,
                     M=64, r=16, keep=0.25, seed=11)
    prm, keep = S.make_params(w.params())
    fake = ctypes.c_void_p(1 << 40)  # never touched: every case fails on the host
    odd = ctypes.c_void_p((1 << 40) + 4)
    f = S.lib.sparsepr_route_noalloc
    assert f(odd, fake, S.BF16, ctypes.byref(prm), fake, fake, fake, fake, None) == S.ERR_INVALID_ARG
    assert f(fake, odd, S.BF16, ctypes.byref(prm), fake, fake, fake, fake, None) == S.ERR_INVALID_ARG
    assert f(fake, fake, 7, ctypes.byref(prm), fake, fake, fake, fake, None) == S.ERR_UNSUPPORTED
    assert f(fake, fake, S.BF16, ctypes.byref(prm), None, fake, fake, fake, None) == S.ERR_INVALID_ARG
    big = synth.custom("noalloc_big", 1, (4, 32, 64), 128, "bf16", Ck=1100, Cq=900, Ms=64,
                       n_eig=4, M=16, r=8, keep=0.1, seed=1)  # (2000*128 + 990000)*8 > 8 MiB
    prm2, keep2 = S.make_params(big.params())
    assert f(fake, fake, S.BF16, ctypes.byref(prm2), fake, fake, fake, fake, None) == S.ERR_WORKSPACE
