"""The certification bound of the tensor-core k-means assignment, checked on
the CPU with an emulation of its arithmetic: x and y split into three bf16
planes, the six plane products with a + b <= 2 summed in fp32 (products of
bf16 values are exact in fp32), the offset applied with one fp32 fma, and the
column position written into the three low mantissa bits. Every emulated
distance must lie within the bound E of the exact fp64 distance, so a row
whose best and second-best emulated distances differ by more than 2 E has the
same nearest centroid as exact arithmetic."""
import numpy as np
import pytest


def bf16(a):
    """Round fp64 values to bf16 (nearest, ties to even), returned as fp64."""
    f = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (f >> 16) & 1
    r = ((f + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def planes(a, n=3):
    out, rest = [], np.asarray(a, dtype=np.float64)
    for _ in range(n):
        p = bf16(rest)
        out.append(p)
        rest = rest - p
    return out


PAIRS = [(0, 0), (0, 1), (1, 0), (0, 2), (1, 1), (2, 0)]
RES_3PLANES = 9.5367431640625e-07  # plane-split residual and dropped products, relative


def emulate(x, Y, c, rng):
    """d'_j for one row x against centroid rows Y[j] with offsets c[j]."""
    xp, yp = planes(x), [planes(Y[:, t]) for t in range(Y.shape[1])]
    D = x.shape[0]
    v = np.zeros(Y.shape[0], dtype=np.float32)
    for a, b in PAIRS:  # accumulate in fp32, one product at a time
        for t in range(D):
            prod = (xp[a][t] * yp[t][b]).astype(np.float32)  # exact
            v = (v + prod).astype(np.float32)
    # fma(-2, v, c) in fp32: exact in fp64, then one rounding
    dd = (np.float64(-2.0) * v.astype(np.float64) + c.astype(np.float32).astype(np.float64))
    dd = dd.astype(np.float32)
    bits = dd.view(np.uint32)
    pos = rng.integers(0, 8, size=bits.shape).astype(np.uint32)
    return ((bits & np.uint32(~7 & 0xFFFFFFFF)) | pos).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("D,scale", [(16, 1.0), (16, 30.0), (8, 0.01)])
def test_emulated_distances_within_bound(D, scale):
    rng = np.random.default_rng(D + int(scale * 100))
    m = 48
    Y = rng.standard_normal((m, D)) * scale
    c = (Y * Y).sum(1)  # keys: c_j = |y_j|^2, d = |y|^2 - 2 x.y
    Ymax = float(np.sqrt((Y * Y).sum(1)).max() * (1 + 1e-6))
    C = float(np.abs(c).max() * (1 + 1e-6))
    Kt = len(PAIRS) * D
    kt_term = Kt * 2.0 ** -22 + RES_3PLANES
    for _ in range(40):
        x = rng.standard_normal(D) * scale * rng.uniform(0.2, 3.0)
        d = c - 2.0 * (Y @ x)  # exact enough in fp64
        dp = emulate(x, Y, c, rng)
        xy = float(np.sqrt((x * x).sum()) * (1 + 1e-6)) * Ymax
        E = kt_term * xy + 1.25e-06 * (C + 2.0 * xy)
        assert np.all(np.abs(dp - d) <= E), (np.abs(dp - d).max(), E)


def test_certified_rows_have_the_exact_label():
    rng = np.random.default_rng(5)
    D, m = 16, 64
    Y = rng.standard_normal((m, D))
    c = (Y * Y).sum(1)
    Ymax = float(np.sqrt((Y * Y).sum(1)).max() * (1 + 1e-6))
    C = float(np.abs(c).max() * (1 + 1e-6))
    kt_term = len(PAIRS) * D * 2.0 ** -22 + RES_3PLANES
    certified = 0
    for _ in range(200):
        x = rng.standard_normal(D)
        d = c - 2.0 * (Y @ x)
        dp = emulate(x, Y, c, rng)
        xy = float(np.sqrt((x * x).sum()) * (1 + 1e-6)) * Ymax
        E = kt_term * xy + 1.25e-06 * (C + 2.0 * xy)
        order = np.argsort(dp, kind="stable")
        if dp[order[1]] - dp[order[0]] > 2 * E:
            certified += 1
            assert order[0] == int(np.argmin(d))
    assert certified > 150  # the bound certifies almost every row


def emulate_query(x, Y, c, nB, rng):
    """The query pass: x is a bf16 row (one exact plane), the centroid side
    G qbar is split into nB bf16 planes, products (0, b) for b < nB summed in
    fp32, then the same fp32 fma with the offset and position packing."""
    yp = [planes(Y[:, t], nB) for t in range(Y.shape[1])]
    v = np.zeros(Y.shape[0], dtype=np.float32)
    for b in range(nB):
        for t in range(x.shape[0]):
            v = (v + (x[t] * yp[t][b]).astype(np.float32)).astype(np.float32)
    dd = (np.float64(-2.0) * v.astype(np.float64) + c.astype(np.float32).astype(np.float64))
    bits = dd.astype(np.float32).view(np.uint32)
    pos = rng.integers(0, 8, size=bits.shape).astype(np.uint32)
    return ((bits & np.uint32(~7 & 0xFFFFFFFF)) | pos).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("nB,res", [(3, 9.5367431640625e-07), (2, 6.103515625e-05)])
def test_query_pass_distances_within_bound(nB, res):
    """d = 128, as in the query pass: the bound with Kt = nB * d and the
    residual term of nB centroid planes covers every emulated distance."""
    rng = np.random.default_rng(40 + nB)
    D, m = 128, 24
    Y = rng.standard_normal((m, D)) * rng.uniform(0.1, 4.0, size=(m, 1))  # G qbar rows
    c = np.abs(rng.standard_normal(m)) * 50.0  # qbar^T G qbar >= 0
    Ymax = float(np.sqrt((Y * Y).sum(1)).max() * (1 + 1e-6))
    C = float(np.abs(c).max() * (1 + 1e-6))
    kt_term = nB * D * 2.0 ** -22 + res
    for _ in range(30):
        x = bf16(rng.standard_normal(D) * rng.uniform(0.2, 3.0))
        d = c - 2.0 * (Y @ x)
        dp = emulate_query(x, Y, c, nB, rng)
        xy = float(np.sqrt((x * x).sum()) * (1 + 1e-6)) * Ymax
        E = kt_term * xy + 1.25e-06 * (C + 2.0 * xy)
        assert np.all(np.abs(dp - d) <= E), (np.abs(dp - d).max(), E)
