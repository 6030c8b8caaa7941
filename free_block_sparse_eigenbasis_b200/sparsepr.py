"""Thin Python binding of libsparsepr.so (the C ABI in include/sparsepr.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. torch is used for device memory and streams. Importing this module
loads the in-tree library and raises if it has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsparsepr.so")
MAX_HEADS = 256

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_NUMERIC = range(7)
BF16, F32 = 0, 1
# sparsepr_params.partition; the parameter dicts name the mode as the oracle does
PARTITION_MODES = dict(response=0, semantic=1, coclustering=2)

EXPORTED = ("sparsepr_workspace_bytes", "sparsepr_status_string", "sparsepr_partition",
            "sparsepr_permute", "sparsepr_route", "sparsepr_route_width",
            "sparsepr_block_sparse_attn", "sparsepr_probe_correct", "sparsepr_read_stats",
            "sparsepr_reset_stats", "sparsepr_check_wait_limit", "sparsepr_route_noalloc",
            "sparsepr_workspace_region", "sparsepr_probe_diagnostics",
            "sparsepr_support_expansion", "sparsepr_density_profile", "sparsepr_attention",
            "sparsepr_check_reciprocal")


class Params(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
                ("n_text", ctypes.c_int32), ("Ck", ctypes.c_int32), ("Cq", ctypes.c_int32),
                ("Ms", ctypes.c_int32), ("n_eig", ctypes.c_int32),
                ("kmeans_iters", ctypes.c_int32), ("M", ctypes.c_int32), ("r", ctypes.c_int32),
                ("partition", ctypes.c_int32), ("lam", ctypes.c_double), ("scale", ctypes.c_double),
                ("seed", ctypes.c_uint64), ("keep", ctypes.POINTER(ctypes.c_double))]


class CallBuffers(ctypes.Structure):
    """sparsepr_call_buffers: device pointers of every output of one call."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "label_q", "label_k", "perm_q", "perm_k", "off_q", "off_k", "qp", "kp", "vp", "csr",
        "k_per_head", "o_sparse", "pairs_sparse", "probes", "pairs_exec", "fit")]


class Stats(ctypes.Structure):
    _fields_ = [("status", ctypes.c_uint32), ("H", ctypes.c_int32),
                ("key_passes", ctypes.c_int32 * MAX_HEADS),
                ("query_passes", ctypes.c_int32 * MAX_HEADS),
                ("pairs_sparse", ctypes.c_int64 * MAX_HEADS),
                ("pairs_exec", ctypes.c_int64 * MAX_HEADS),
                ("recheck_rows", ctypes.c_int64 * 2),
                ("eig_sweeps", ctypes.c_int32 * 2), ("near_ties", ctypes.c_int64 * 2)]


class SparsePRError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__("%s: %s (status %d)" % (where, status_string(code), code))
        self.code = code


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError("libsparsepr.so is not built; run "
                          "`python -m free_block_sparse_eigenbasis_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, V, I32P, I64P = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    PP = ctypes.POINTER(Params)
    st = ctypes.c_int
    sz = ctypes.c_size_t
    lib.sparsepr_workspace_bytes.argtypes = [PP]
    lib.sparsepr_workspace_bytes.restype = sz
    lib.sparsepr_status_string.argtypes = [st]
    lib.sparsepr_status_string.restype = ctypes.c_char_p
    lib.sparsepr_route_width.argtypes = [PP]
    lib.sparsepr_route_width.restype = ctypes.c_int32
    lib.sparsepr_partition.argtypes = [P, P, st, PP, I32P, I32P, V, sz, V]
    lib.sparsepr_permute.argtypes = [P, P, P, st, PP, I32P, I32P, I32P, I32P, I32P, I32P, P, P, P,
                                     V, sz, V]
    lib.sparsepr_route.argtypes = [P, P, st, PP, I32P, I32P, I32P, I32P, V, sz, V]
    lib.sparsepr_block_sparse_attn.argtypes = [P, P, P, st, PP, I32P, I32P, I32P, I32P, P, I64P,
                                               V, sz, V]
    lib.sparsepr_probe_correct.argtypes = [P, P, P, st, PP, I32P, I32P, P, I64P, P, I32P, I64P, P,
                                           V, sz, V]
    lib.sparsepr_route_noalloc.argtypes = [P, P, st, PP, I32P, I32P, I32P, I32P, V]
    lib.sparsepr_route_noalloc.restype = st
    lib.sparsepr_workspace_region.argtypes = [PP, ctypes.c_char_p, ctypes.POINTER(sz),
                                              ctypes.POINTER(sz)]
    lib.sparsepr_workspace_region.restype = st
    lib.sparsepr_probe_diagnostics.argtypes = [PP, I32P, P, P, P, V, sz, V]
    lib.sparsepr_probe_diagnostics.restype = st
    lib.sparsepr_support_expansion.argtypes = [P, P, st, PP, I32P, I32P, ctypes.c_double,
                                               ctypes.c_int32, P, P, V, sz, V]
    lib.sparsepr_support_expansion.restype = st
    lib.sparsepr_density_profile.argtypes = [P, P, st, PP, ctypes.c_double, ctypes.c_int32, P, V,
                                             sz, V]
    lib.sparsepr_density_profile.restype = st
    lib.sparsepr_attention.argtypes = [P, P, P, st, PP, ctypes.POINTER(CallBuffers), P, V, sz, V]
    lib.sparsepr_attention.restype = st
    lib.sparsepr_read_stats.argtypes = [V, ctypes.POINTER(Stats)]
    lib.sparsepr_reset_stats.argtypes = [V, V]
    lib.sparsepr_check_wait_limit.argtypes = [V, V]
    lib.sparsepr_check_reciprocal.argtypes = [P, ctypes.c_int64, P, V]
    lib.sparsepr_check_reciprocal.restype = st
    for name in ("sparsepr_partition", "sparsepr_permute", "sparsepr_route",
                 "sparsepr_block_sparse_attn", "sparsepr_probe_correct", "sparsepr_read_stats",
                 "sparsepr_reset_stats", "sparsepr_check_wait_limit"):
        getattr(lib, name).restype = st
    return lib


lib = _load()


def status_string(code: int) -> str:
    return lib.sparsepr_status_string(code).decode()


def make_params(p: dict):
    """ctypes Params from a plain parameter dict; returns (params, keep array)
    -- keep the second value alive for as long as the first is used."""
    H = int(p["H"])
    keep = p["keep"]
    if not isinstance(keep, (list, tuple)):
        keep = [keep] * H
    arr = (ctypes.c_double * max(1, H))(*[float(x) for x in keep[:H]])
    prm = Params(H=H, N=int(p["N"]), d=int(p["d"]), n_text=int(p.get("n_text", 0)),
                 Ck=int(p["Ck"]), Cq=int(p["Cq"]), Ms=int(p["Ms"]), n_eig=int(p["n_eig"]),
                 kmeans_iters=int(p["kmeans_iters"]), M=int(p["M"]), r=int(p["r"]),
                 partition=PARTITION_MODES[p.get("partition", "response")],
                 lam=float(p["lam"]), scale=float(p.get("scale", 0.0)),
                 seed=int(p["seed"]) & ((1 << 64) - 1),
                 keep=ctypes.cast(arr, ctypes.POINTER(ctypes.c_double)))
    return prm, arr


_DEVICE_TYPE = "cuda"  # tensors handed to the library live on this device type


def _arg(t, name: str, shape=None, dtype=None):
    """Device pointer of a tensor argument after the checks the C ABI cannot
    make from a bare pointer: shape, dtype, dense row-major layout and a CUDA
    device. Raises ValueError / TypeError before anything is enqueued."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous (row-major)" % name)
    if t.device.type != _DEVICE_TYPE:
        raise ValueError("%s must be a CUDA tensor" % name)
    return ctypes.c_void_p(t.data_ptr())


def _ws(ws, name: str = "ws"):
    """(pointer, bytes) of the workspace: a contiguous CUDA byte buffer."""
    return _arg(ws, name, (ws.numel(),) if isinstance(ws, torch.Tensor) else None,
                torch.uint8), ws.numel()


def _dims(p: dict):
    """H, N, d and the group-offset widths (text tokens add one group per side)."""
    H, N, d = int(p["H"]), int(p["N"]), int(p["d"])
    text = 1 if int(p.get("n_text", 0)) > 0 else 0
    return H, N, d, int(p["Cq"]) + text + 1, int(p["Ck"]) + text + 1


def _qkv(p: dict, names_tensors):
    """Checks the [H, N, d] inputs of one dtype (bf16 or fp32, set by the first)."""
    H, N, d = int(p["H"]), int(p["N"]), int(p["d"])
    dt = names_tensors[0][1].dtype if isinstance(names_tensors[0][1], torch.Tensor) else None
    ptrs = [_arg(t, n, (H, N, d), dt) for n, t in names_tensors]
    return ptrs, _dtype_code(names_tensors[0][1])


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return BF16
    if x.dtype == torch.float32:
        return F32
    raise TypeError("Q/K/V must be bf16 or fp32")


def _check(code: int, where: str):
    if code != OK:
        raise SparsePRError(code, where)


def workspace_bytes(p: dict) -> int:
    prm, keep = make_params(p)
    return int(lib.sparsepr_workspace_bytes(ctypes.byref(prm)))


def route_width(p: dict) -> int:
    prm, keep = make_params(p)
    return int(lib.sparsepr_route_width(ctypes.byref(prm)))


# ---- the five calls, same names as the C ABI --------------------------------

I32, I64 = torch.int32, torch.int64


def sparsepr_partition(q, k, p, label_q, label_k, ws, stream=None):
    prm, keep = make_params(p)
    H, N, d, _, _ = _dims(p)
    (pq, pk), dt = _qkv(p, [("q", q), ("k", k)])
    wp, wb = _ws(ws)
    _check(lib.sparsepr_partition(pq, pk, dt, ctypes.byref(prm),
                                  _arg(label_q, "label_q", (H, N), I32),
                                  _arg(label_k, "label_k", (H, N), I32), wp, wb,
                                  _stream(stream)), "sparsepr_partition")


def sparsepr_permute(q, k, v, p, label_q, label_k, perm_q, perm_k, off_q, off_k, qp, kp, vp, ws,
                     stream=None):
    prm, keep = make_params(p)
    H, N, d, wq, wk = _dims(p)
    (pq, pk, pv, pqp, pkp, pvp), dt = _qkv(p, [("q", q), ("k", k), ("v", v), ("qp", qp),
                                              ("kp", kp), ("vp", vp)])
    wp, wb = _ws(ws)
    _check(lib.sparsepr_permute(pq, pk, pv, dt, ctypes.byref(prm),
                                _arg(label_q, "label_q", (H, N), I32),
                                _arg(label_k, "label_k", (H, N), I32),
                                _arg(perm_q, "perm_q", (H, N), I32),
                                _arg(perm_k, "perm_k", (H, N), I32),
                                _arg(off_q, "off_q", (H, wq), I32),
                                _arg(off_k, "off_k", (H, wk), I32), pqp, pkp, pvp, wp, wb,
                                _stream(stream)), "sparsepr_permute")


def _route_args(qp, kp, p, off_q, off_k, csr, k_per_head):
    H, N, d, wq, wk = _dims(p)
    (pq, pk), dt = _qkv(p, [("qp", qp), ("kp", kp)])
    return (pq, pk, dt, _arg(off_q, "off_q", (H, wq), I32), _arg(off_k, "off_k", (H, wk), I32),
            _arg(csr, "csr", (H, int(p["Cq"]), route_width(p)), I32),
            _arg(k_per_head, "k_per_head", (H,), I32))


def sparsepr_route(qp, kp, p, off_q, off_k, csr, k_per_head, ws, stream=None):
    prm, keep = make_params(p)
    pq, pk, dt, poq, pok, pcsr, pkh = _route_args(qp, kp, p, off_q, off_k, csr, k_per_head)
    wp, wb = _ws(ws)
    _check(lib.sparsepr_route(pq, pk, dt, ctypes.byref(prm), poq, pok, pcsr, pkh, wp, wb,
                              _stream(stream)), "sparsepr_route")


def sparsepr_route_noalloc(qp, kp, p, off_q, off_k, csr, k_per_head, stream=None):
    """sparsepr_route without a workspace (its scratch is a fixed device array
    inside the library); for callers that cannot allocate device memory."""
    prm, keep = make_params(p)
    pq, pk, dt, poq, pok, pcsr, pkh = _route_args(qp, kp, p, off_q, off_k, csr, k_per_head)
    _check(lib.sparsepr_route_noalloc(pq, pk, dt, ctypes.byref(prm), poq, pok, pcsr, pkh,
                                      _stream(stream)), "sparsepr_route_noalloc")


def sparsepr_block_sparse_attn(qp, kp, vp, p, off_q, off_k, csr, k_per_head, o_sparse,
                               pairs_sparse, ws, stream=None):
    prm, keep = make_params(p)
    H, N, d, _, _ = _dims(p)
    pq, pk, dt, poq, pok, pcsr, pkh = _route_args(qp, kp, p, off_q, off_k, csr, k_per_head)
    (pv,), _ = _qkv(p, [("vp", vp)])
    if vp.dtype != qp.dtype:
        raise TypeError("vp has dtype %s, expected %s" % (vp.dtype, qp.dtype))
    wp, wb = _ws(ws)
    _check(lib.sparsepr_block_sparse_attn(pq, pk, pv, dt, ctypes.byref(prm), poq, pok, pcsr, pkh,
                                          _arg(o_sparse, "o_sparse", (H, N, d), torch.float32),
                                          _arg(pairs_sparse, "pairs_sparse", (H,), I64), wp, wb,
                                          _stream(stream)), "sparsepr_block_sparse_attn")


def sparsepr_probe_correct(qp, kp, vp, p, off_q, perm_q, o_sparse, pairs_sparse, out, probes,
                           pairs_exec, ws, fit=None, stream=None):
    prm, keep = make_params(p)
    H, N, d, wq, _ = _dims(p)
    M = int(p["M"])
    (pq, pk, pv, pout), dt = _qkv(p, [("qp", qp), ("kp", kp), ("vp", vp), ("out", out)])
    wp, wb = _ws(ws)
    _check(lib.sparsepr_probe_correct(pq, pk, pv, dt, ctypes.byref(prm),
                                      _arg(off_q, "off_q", (H, wq), I32),
                                      _arg(perm_q, "perm_q", (H, N), I32),
                                      _arg(o_sparse, "o_sparse", (H, N, d), torch.float32),
                                      _arg(pairs_sparse, "pairs_sparse", (H,), I64), pout,
                                      _arg(probes, "probes", (H, M) if M > 0 else None, I32),
                                      _arg(pairs_exec, "pairs_exec", (H,), I64),
                                      None if fit is None else
                                      _arg(fit, "fit", (H, d * d + d), torch.float64),
                                      wp, wb, _stream(stream)), "sparsepr_probe_correct")


def sparsepr_probe_diagnostics(p, probes, mass, error, energy, ws, stream=None):
    """Retained mass and error of every probe row, and the residual energy
    split per head (see include/sparsepr.h)."""
    prm, keep = make_params(p)
    H, M = int(p["H"]), int(p["M"])
    f64 = torch.float64
    _check(lib.sparsepr_probe_diagnostics(ctypes.byref(prm), _arg(probes, "probes", (H, M), I32),
                                          _arg(mass, "mass", (H, M), f64),
                                          _arg(error, "error", (H, M), f64),
                                          _arg(energy, "energy", (H, 4), f64), *_ws(ws),
                                          _stream(stream)), "sparsepr_probe_diagnostics")


def sparsepr_support_expansion(qp, kp, p, off_q, off_k, tau, group_stride, individual,
                               aggregate, ws, stream=None):
    """Mean individual and aggregate (union) support size, in key groups, of
    every group_stride-th video query group (see include/sparsepr.h)."""
    prm, keep = make_params(p)
    H, N, d, wq, wk = _dims(p)
    Cq = int(p["Cq"])
    (pq, pk), dt = _qkv(p, [("qp", qp), ("kp", kp)])
    f64 = torch.float64
    _check(lib.sparsepr_support_expansion(pq, pk, dt, ctypes.byref(prm),
                                          _arg(off_q, "off_q", (H, wq), I32),
                                          _arg(off_k, "off_k", (H, wk), I32), float(tau),
                                          int(group_stride),
                                          _arg(individual, "individual", (H, Cq), f64),
                                          _arg(aggregate, "aggregate", (H, Cq), f64), *_ws(ws),
                                          _stream(stream)), "sparsepr_support_expansion")


def sparsepr_density_profile(q, k, p, tau, row_stride, density, ws, stream=None):
    """Mean tau-mass density of every row_stride-th video row, per head."""
    prm, keep = make_params(p)
    H = int(p["H"])
    (pq, pk), dt = _qkv(p, [("q", q), ("k", k)])
    _check(lib.sparsepr_density_profile(pq, pk, dt, ctypes.byref(prm), float(tau), int(row_stride),
                                        _arg(density, "density", (H,), torch.float64), *_ws(ws),
                                        _stream(stream)), "sparsepr_density_profile")


def sparsepr_reset_stats(ws, stream=None):
    _check(lib.sparsepr_reset_stats(_ws(ws)[0], _stream(stream)), "sparsepr_reset_stats")


def sparsepr_check_wait_limit(ws, stream=None):
    _check(lib.sparsepr_check_wait_limit(_ws(ws)[0], _stream(stream)), "sparsepr_check_wait_limit")


def sparsepr_check_reciprocal(x, stream=None):
    """Distance in ulp of the multisection's reciprocal from the correctly
    rounded 1/x, for a 1-D fp64 device tensor x; returns a tensor like x."""
    if x.dtype != torch.float64 or x.dim() != 1 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x: a contiguous 1-D float64 CUDA tensor")
    err = torch.empty_like(x)
    _check(lib.sparsepr_check_reciprocal(x.data_ptr(), x.numel(), err.data_ptr(), _stream(stream)),
           "sparsepr_check_reciprocal")
    return err


_REGION_DTYPES = dict(init_k=torch.int32, init_q=torch.int32, zplanes=torch.bfloat16,
                      xnk=torch.float32)


def sparsepr_workspace_region(p: dict, name: str):
    """(byte offset, bytes) of a named intermediate-result region of the
    workspace for these parameters."""
    prm, keep = make_params(p)
    off, nb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib.sparsepr_workspace_region(ctypes.byref(prm), name.encode(), ctypes.byref(off),
                                         ctypes.byref(nb)), "sparsepr_workspace_region")
    return int(off.value), int(nb.value)


def workspace_view(ws, p: dict, name: str) -> torch.Tensor:
    """The named region of `ws` as a flat tensor of its element type (fp64;
    int32 for the initial centroid rows, bf16 for the key planes, fp32 for
    the key row norms); a view, no copy."""
    off, nb = sparsepr_workspace_region(p, name)
    return ws[off:off + nb].view(_REGION_DTYPES.get(name, torch.float64))


def sparsepr_read_stats(ws) -> dict:
    s = Stats()
    _check(lib.sparsepr_read_stats(_ws(ws)[0], ctypes.byref(s)), "sparsepr_read_stats")
    H = max(0, min(s.H, MAX_HEADS))
    return dict(status=int(s.status), H=H, key_passes=list(s.key_passes[:H]),
                query_passes=list(s.query_passes[:H]), pairs_sparse=list(s.pairs_sparse[:H]),
                pairs_exec=list(s.pairs_exec[:H]), recheck_rows=list(s.recheck_rows),
                eig_sweeps=list(s.eig_sweeps), near_ties=list(s.near_ties))


# ---- buffers + the whole call ----------------------------------------------

@dataclass
class Buffers:
    """Device buffers of one attention call (all owned by torch)."""
    ws: torch.Tensor
    label_q: torch.Tensor
    label_k: torch.Tensor
    perm_q: torch.Tensor
    perm_k: torch.Tensor
    off_q: torch.Tensor
    off_k: torch.Tensor
    qp: torch.Tensor
    kp: torch.Tensor
    vp: torch.Tensor
    csr: torch.Tensor
    k_per_head: torch.Tensor
    o_sparse: torch.Tensor
    pairs_sparse: torch.Tensor
    out: torch.Tensor
    probes: torch.Tensor
    pairs_exec: torch.Tensor
    fit: Optional[torch.Tensor]


def allocate(p: dict, dtype: torch.dtype, device="cuda", with_fit=False) -> Buffers:
    H, N, d = int(p["H"]), int(p["N"]), int(p["d"])
    Ck, Cq, M = int(p["Ck"]), int(p["Cq"]), int(p["M"])
    text = 1 if int(p.get("n_text", 0)) > 0 else 0  # text tokens form one extra group per side
    wsb = workspace_bytes(p)
    if wsb == 0:
        raise SparsePRError(ERR_INVALID_ARG, "workspace_bytes")
    kmax = route_width(p)
    i32 = dict(dtype=torch.int32, device=device)
    return Buffers(
        ws=torch.empty(wsb, dtype=torch.uint8, device=device),
        label_q=torch.empty((H, N), **i32), label_k=torch.empty((H, N), **i32),
        perm_q=torch.empty((H, N), **i32), perm_k=torch.empty((H, N), **i32),
        off_q=torch.empty((H, Cq + text + 1), **i32), off_k=torch.empty((H, Ck + text + 1), **i32),
        qp=torch.empty((H, N, d), dtype=dtype, device=device),
        kp=torch.empty((H, N, d), dtype=dtype, device=device),
        vp=torch.empty((H, N, d), dtype=dtype, device=device),
        csr=torch.empty((H, Cq, kmax), **i32), k_per_head=torch.empty(H, **i32),
        o_sparse=torch.empty((H, N, d), dtype=torch.float32, device=device),
        pairs_sparse=torch.empty(H, dtype=torch.int64, device=device),
        out=torch.empty((H, N, d), dtype=dtype, device=device),
        probes=torch.empty((H, max(M, 1)), **i32),
        pairs_exec=torch.empty(H, dtype=torch.int64, device=device),
        fit=torch.empty((H, d * d + d), dtype=torch.float64, device=device) if with_fit else None)


def attention(q, k, v, p: dict, bufs: Optional[Buffers] = None, stream=None) -> Buffers:
    """One SparsePR attention call on [H, N, d] device tensors: the five
    library calls in order on one stream. Returns the buffers (bufs.out is
    the corrected output in the original token order)."""
    if bufs is None:
        bufs = allocate(p, q.dtype, q.device)
    b = bufs
    sparsepr_partition(q, k, p, b.label_q, b.label_k, b.ws, stream)
    sparsepr_permute(q, k, v, p, b.label_q, b.label_k, b.perm_q, b.perm_k, b.off_q, b.off_k, b.qp,
                     b.kp, b.vp, b.ws, stream)
    sparsepr_route(b.qp, b.kp, p, b.off_q, b.off_k, b.csr, b.k_per_head, b.ws, stream)
    sparsepr_block_sparse_attn(b.qp, b.kp, b.vp, p, b.off_q, b.off_k, b.csr, b.k_per_head,
                               b.o_sparse, b.pairs_sparse, b.ws, stream)
    sparsepr_probe_correct(b.qp, b.kp, b.vp, p, b.off_q, b.perm_q, b.o_sparse, b.pairs_sparse,
                           b.out, b.probes, b.pairs_exec, b.ws, b.fit, stream)
    return b


def sparsepr_attention(q, k, v, p: dict, bufs: Buffers, stream=None) -> Buffers:
    """The whole call in one library entry point (sparsepr_attention): the
    probe fit runs on a side stream beside the attention of all rows. Fills
    the same buffers as attention(); bufs.out is the output."""
    prm, keep = make_params(p)
    H, N, d, oq, ok = _dims(p)
    (pq, pk, pv), dt = _qkv(p, [("q", q), ("k", k), ("v", v)])
    b = bufs
    I32T = torch.int32
    ptr = lambda t, n, shape, dtype: _arg(t, n, shape, dtype).value  # noqa: E731
    kmax = route_width(p)
    M = int(p["M"])
    cb = CallBuffers(
        label_q=ptr(b.label_q, "label_q", (H, N), I32T), label_k=ptr(b.label_k, "label_k", (H, N), I32T),
        perm_q=ptr(b.perm_q, "perm_q", (H, N), I32T), perm_k=ptr(b.perm_k, "perm_k", (H, N), I32T),
        off_q=ptr(b.off_q, "off_q", (H, oq), I32T), off_k=ptr(b.off_k, "off_k", (H, ok), I32T),
        qp=ptr(b.qp, "qp", (H, N, d), q.dtype), kp=ptr(b.kp, "kp", (H, N, d), q.dtype),
        vp=ptr(b.vp, "vp", (H, N, d), q.dtype),
        csr=ptr(b.csr, "csr", (H, int(p["Cq"]), kmax), I32T),
        k_per_head=ptr(b.k_per_head, "k_per_head", (H,), I32T),
        o_sparse=ptr(b.o_sparse, "o_sparse", (H, N, d), torch.float32),
        pairs_sparse=ptr(b.pairs_sparse, "pairs_sparse", (H,), I64),
        probes=ptr(b.probes, "probes", (H, max(M, 1)), I32T),
        pairs_exec=ptr(b.pairs_exec, "pairs_exec", (H,), I64),
        fit=None if b.fit is None else ptr(b.fit, "fit", (H, d * d + d), torch.float64))
    out = _arg(b.out, "out", (H, N, d), q.dtype)
    wp, wb = _ws(b.ws)
    _check(lib.sparsepr_attention(pq, pk, pv, dt, ctypes.byref(prm), ctypes.byref(cb), out, wp, wb,
                                  _stream(stream)), "sparsepr_attention")
    return b


def dense_params(H: int, N: int, d: int, scale: float = 0.0) -> dict:
    """Parameters of the same attention kernel run densely: one query group
    and one key group covering all N tokens, keep = 1."""
    return dict(H=H, N=N, d=d, n_text=0, Ck=1, Cq=1, Ms=1, n_eig=1, kmeans_iters=1,
                keep=[1.0] * H, M=0, r=1, lam=0.0, scale=scale, seed=0)


def dense_attention(q, k, v, out, ws=None, stream=None, meta=None):
    """Dense softmax attention through the same block-sparse kernel (the
    baseline of the same design): identity order, one group, full route.
    ``meta`` caches the small routing tensors between calls."""
    H, N, d = q.shape
    p = dense_params(H, N, d)
    if meta is None:
        meta = dict(
            off=torch.tensor([[0, N]] * H, dtype=torch.int32, device=q.device),
            csr=torch.zeros((H, 1, 1), dtype=torch.int32, device=q.device),
            kh=torch.ones(H, dtype=torch.int32, device=q.device),
            pairs=torch.empty(H, dtype=torch.int64, device=q.device))
    if ws is None:
        ws = torch.empty(workspace_bytes(p), dtype=torch.uint8, device=q.device)
    sparsepr_block_sparse_attn(q, k, v, p, meta["off"], meta["off"], meta["csr"], meta["kh"], out,
                               meta["pairs"], ws, stream)
    return meta, ws
