"""Pins of the oracle's multi-dimensional Lorenzo path (orc_compress_lorenzo
and its inverse), each against something other than the oracle itself:

* the block stencil against NumPy's first differences along x, y, z with a
  zero pad (the reset at the block faces), modulo 2^32, and its inverse
  against NumPy cumulative sums;
* closed forms: a constant block leaves one residual at the block origin, a
  linear one its gradient on the three edges, a trilinear i*j*k term one
  interior constant;
* every stream re-decoded independently: payload codes through a bit matrix,
  the block order through a NumPy reshape/transpose of the brick grid (not
  the oracle's index arithmetic), residuals summed back with NumPy, compared
  with the quantiser's codes; the outlier list is the flagged set in C
  order within each brick; every element within eb.
CPU only."""
import numpy as np
import pytest

from error_bounded_lossy_encode_b200 import workloads as WL
from tests import streamcheck as SC

EDGES = {(3, 64): (4, 4, 4), (3, 256): (4, 8, 8), (2, 64): (1, 8, 8), (2, 256): (1, 16, 16)}
BRICK = {3: (16, 16, 16), 2: (1, 64, 64)}


def _np_lorenzo(q, be):
    a = q.astype(np.int64).reshape(be)
    for ax in (2, 1, 0):
        a = np.diff(a, axis=ax, prepend=0)
    return (a & 0xFFFFFFFF).astype(np.uint32).view(np.int32).reshape(-1)


def _np_unlorenzo(d, be):
    a = d.astype(np.int64).reshape(be)
    for ax in (2, 1, 0):
        a = np.cumsum(a, axis=ax) & 0xFFFFFFFF
    return a.astype(np.uint32).view(np.int32).reshape(-1)


@pytest.mark.parametrize("key", sorted(EDGES))
def test_edges(orc, key):
    rank, block = key
    be, ce = orc.nd_edges(rank, block)
    assert be == EDGES[key] and ce == BRICK[rank] and np.prod(be) == block and np.prod(ce) == 4096
    assert orc.nd_edges(rank, 32) is None and orc.nd_edges(rank, 128) is None and orc.nd_edges(1, 64) is None


@pytest.mark.parametrize("be", sorted(set(EDGES.values())))
def test_block_stencil_vs_numpy(orc, be):
    rng = np.random.default_rng(sum(be))
    for scale in (3, 1000, 1 << 29, 1 << 31):
        q = rng.integers(-scale, scale, size=int(np.prod(be)), dtype=np.int64).astype(np.int32)
        d = orc.lorenzo_block(q, be)
        assert np.array_equal(d, _np_lorenzo(q, be))
        assert np.array_equal(orc.unlorenzo_block(d, be), q)
        assert np.array_equal(_np_unlorenzo(d, be), q)


@pytest.mark.parametrize("be", sorted(set(EDGES.values())))
def test_block_stencil_closed_forms(orc, be):
    Z, Y, X = be
    i, j, k = np.meshgrid(np.arange(Z), np.arange(Y), np.arange(X), indexing="ij")
    # constant: the block origin keeps the value, everything else predicts it exactly
    d = orc.lorenzo_block(np.full(Z * Y * X, 7, np.int32), be).reshape(be)
    assert d[0, 0, 0] == 7 and np.count_nonzero(d) == 1
    # linear: origin a, then the gradient once along each axis' first edge
    q = (5 + 3 * i - 2 * j + 4 * k).astype(np.int32)
    d = orc.lorenzo_block(q.reshape(-1), be).reshape(be)
    want = np.zeros(be, np.int64)
    want[0, 0, 0] = 5
    want[1:, 0, 0] = 3
    want[0, 1:, 0] = -2
    want[0, 0, 1:] = 4
    assert np.array_equal(d, want)
    # trilinear i*j*k: a constant 1 where all three are >= 1 (3-D blocks only)
    if Z > 1:
        d = orc.lorenzo_block((i * j * k).astype(np.int32).reshape(-1), be).reshape(be)
        assert np.array_equal(d, ((i >= 1) & (j >= 1) & (k >= 1)).astype(np.int64))


def _stream_order(dims, be, ce):
    """C-order element index of every code in stream order (brick, block, element)."""
    Z, Y, X = dims
    g = (Z // ce[0], Y // ce[1], X // ce[2])
    k = (ce[0] // be[0], ce[1] // be[1], ce[2] // be[2])
    idx = np.arange(Z * Y * X).reshape(g[0], k[0], be[0], g[1], k[1], be[1], g[2], k[2], be[2])
    return idx.transpose(0, 3, 6, 1, 4, 7, 2, 5, 8).reshape(-1)


def _check_nd_stream(orc, x, s, block, rank):
    dims = (1,) + x.shape if x.ndim == 2 else x.shape
    be, ce = EDGES[(rank, block)], BRICK[rank]
    P = SC.parts(s)  # header, widths, chunk index, payload, outliers (1-D layout rules hold per chunk)
    h = P["h"]
    assert h["flags"] & 2 and h["n"] == x.size and h["nb"] == x.size // block and h["nc"] == x.size // 4096
    assert SC.header(s)["reserved"][:24] == np.array(dims, "<u8").tobytes() and not any(SC.header(s)["reserved"][24:])
    b = orc.Bound(h["eb"], np.float32(h["inv2eb"]), np.float32(h["step"]))
    flat = x.reshape(-1)
    q, flag = orc.quantize(flat, b)
    # payload -> codes (bit matrix), block-local prefix sums (NumPy), stream order -> C order
    bits = np.unpackbits(P["payload"], bitorder="little")
    words = -(-(P["widths"] * block) // 32)
    starts = np.concatenate([[0], np.cumsum(words)])
    order = _stream_order(dims, be, ce)
    got = np.zeros(x.size, np.int64)
    for bi in range(h["nb"]):
        w = int(P["widths"][bi])
        z = np.zeros(block, np.uint64)
        if w:
            m = bits[32 * starts[bi]: 32 * starts[bi] + w * block].reshape(block, w).astype(np.uint64)
            z = (m << np.arange(w, dtype=np.uint64)).sum(axis=1)
        d = np.where(z % 2 == 0, z // 2, -((z + 1) // 2).astype(np.int64)).astype(np.int64)
        got[order[bi * block:(bi + 1) * block]] = _np_unlorenzo(d, be)
        # the width is the smallest that holds every zigzag code of the block
        assert w == (int(z.max()).bit_length() if block else 0)
    assert np.array_equal(got, q.astype(np.int64))
    # outliers: per brick, the flagged elements in ascending C order
    brick_of = np.empty(x.size, np.int64)
    brick_of[order] = np.arange(x.size) // 4096
    want_idx = np.concatenate([np.flatnonzero(flag & (brick_of == c)) for c in range(h["nc"])]) \
        if h["nc"] else np.zeros(0, np.int64)
    assert h["m"] == int(flag.sum()) and np.array_equal(P["idx"], want_idx.astype(np.uint32))
    assert np.array_equal(P["val"], flat.view(np.uint32)[want_idx])
    y = orc.decompress(s, x.size)
    keep = ~flag
    assert np.all(np.abs(flat[keep].astype(np.float64) - y[keep].astype(np.float64)) <= h["eb"])
    assert np.array_equal(y.view(np.uint32)[flag], flat.view(np.uint32)[flag])
    return h


@pytest.mark.parametrize("key", sorted(EDGES))
@pytest.mark.parametrize("bound", [("rel", 1e-3), ("rel", 1e-6), ("abs", 1e-7), ("abs", 0.0)])
def test_nd_stream_independent_decode(orc, key, bound):
    rank, block = key
    shape = (32, 48, 16) if rank == 3 else (128, 192)
    x = WL.with_spikes((1, 1, int(np.prod(shape))), 3, p_nonfinite=2e-3).reshape(shape)
    x[0, ..., :5] = [np.nan, np.inf, -np.inf, -0.0, 1e-40][:5]
    s = orc.compress_lorenzo(x, block, **{bound[0]: bound[1]})
    _check_nd_stream(orc, x, s, block, rank)


@pytest.mark.parametrize("key", sorted(EDGES))
def test_nd_smooth_field_and_constant(orc, key):
    rank, block = key
    shape = (16, 32, 64) if rank == 3 else (64, 128)
    x = WL.kfield((1, 1, int(np.prod(shape))), 5).reshape(shape)
    _check_nd_stream(orc, x, orc.compress_lorenzo(x, block, rel=1e-4), block, rank)
    c = np.full(shape, -3.25, np.float32)  # (a relative bound of a constant is 0: all outliers)
    h = _check_nd_stream(orc, c, orc.compress_lorenzo(c, block, abs=1e-3), block, rank)
    q0 = int(np.rint(np.float32(-3.25) * np.float32(h["inv2eb"])))  # every block: one residual, at its origin
    w = (2 * q0 if q0 >= 0 else -2 * q0 - 1).bit_length()
    assert h["m"] == 0 and np.all(SC.parts(orc.compress_lorenzo(c, block, abs=1e-3))["widths"] == w)
    assert h["W"] == (c.size // block) * (w * block // 32)


def test_nd_rejects_unsupported_shapes(orc):
    with pytest.raises(orc.OracleError):
        orc.compress_lorenzo(np.zeros((16, 16, 17), np.float32), 64, rel=1e-3)
    with pytest.raises(orc.OracleError):
        orc.compress_lorenzo(np.zeros((16, 16, 16), np.float32), 128, rel=1e-3)
    with pytest.raises(orc.OracleError):
        orc.compress_lorenzo(np.zeros((64, 60), np.float32), 64, rel=1e-3)
