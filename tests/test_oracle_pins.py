"""Pins of the CPU oracle against things other than itself.

Each test names the oracle step it pins and what it is pinned to: a
hand-derived worked example, exact rational arithmetic, a library routine
(NumPy min/max, bit matrices, cumsum), closed forms, invariants of the method
(the error bound, lossless outliers), or brute force over tiny inputs.
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from error_bounded_lossy_encode_b200 import workloads as WL
from tests import streamcheck as SC

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BLOCKS = (32, 64, 128, 256)


# --------------------------------------------------------------------------------------
# Worked example derived by hand (no program involved)
# --------------------------------------------------------------------------------------

def test_worked_example_by_hand(orc):
    """x = [0, 2, 4, 3, -1], absolute bound 0.5, block 32.

    By hand: 2*eb = 1.0 so step = 1.0 and inv2eb = 1.0; q = x; Lorenzo deltas
    with predecessor 0 at the block start: [0, 2, 2, -1, -4]; zigzag:
    [0, 4, 4, 1, 7]; OR = 7 so w = 3; bits (LSB first) 0 | 4<<3 | 4<<6 | 1<<9
    | 7<<12 = 32 + 256 + 512 + 28672 = 29472 = 0x00007320: one word.
    Layout: header 128 B, width byte at 128 padded to 144, one chunk index
    pair (0, 0) at 144 padded to 160, the chunk record (one payload word, no
    outliers) at 160: total 164 bytes."""
    x = np.array([0, 2, 4, 3, -1], np.float32)
    s = orc.compress(x, 32, abs=0.5)
    assert s.size == 164
    h = SC.header(s)
    assert (h["magic"], h["version"], h["flags"], h["n"], h["block"], h["chunk"]) == (0x434C4245, 1, 1, 5, 32, 4096)
    assert (h["eb"], h["inv2eb"], h["step"], h["vmin"], h["vmax"]) == (0.5, 1.0, 1.0, 0.0, 0.0)
    assert (h["nb"], h["nc"], h["W"], h["m"], h["total"], h["bound"]) == (1, 1, 1, 0, 164, 0.5)
    assert h["reserved"] == bytes(32)
    assert list(s[128:144]) == [3] + [0] * 15
    assert list(s[144:160]) == [0] * 16
    assert list(s[160:164]) == [0x20, 0x73, 0, 0]
    assert orc.decompress(s, 5).tolist() == [0, 2, 4, 3, -1]


def test_worked_example_relative_and_outlier(orc):
    """x = [-1, 3, 1.25, nan], relative bound 0.25, block 32, by hand.

    Finite range [-1, 3] so eb = 0.25*4 = 1.0, 2eb = 2 -> step 2.0, inv2eb
    0.5.  y = [-0.5, 1.5, 0.625, nan] -> q = [-0 (=0, tie to even), 2 (tie to
    even), 1, 0 (non-finite)].  x' = [0, 4, 2, 0]: errors 1, 1, 0.75 <= eb,
    nan is an outlier.  deltas [0, 2, -1, -1] -> zigzag [0, 4, 1, 1], w = 3,
    word = 0 | 4<<3 | 1<<6 | 1<<9 = 32 + 64 + 512 = 608 = 0x260.  One outlier
    (3, nan bits): the record at 160 holds the payload word, then idx 3 at
    164, then the nan bits at 168: total 172."""
    x = np.array([-1.0, 3.0, 1.25, np.nan], np.float32)
    s = orc.compress(x, 32, rel=0.25)
    h = SC.header(s)
    assert (h["eb"], h["inv2eb"], h["step"], h["vmin"], h["vmax"]) == (1.0, 0.5, 2.0, -1.0, 3.0)
    assert (h["W"], h["m"], h["total"]) == (1, 1, 172)
    assert s[128] == 3
    assert list(s[160:164]) == [0x60, 0x02, 0, 0]
    assert list(s[144:160]) == [0] * 16
    assert s[164:168].view(np.uint32)[0] == 3
    assert s[168:172].view(np.uint32)[0] == np.float32(np.nan).view(np.uint32)
    y = orc.decompress(s, 4)
    assert y[:3].tolist() == [0.0, 4.0, 2.0] and np.isnan(y[3])


# --------------------------------------------------------------------------------------
# Step 1: value range -- pinned to NumPy min/max over the finite elements
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(6))
def test_value_range_vs_numpy(orc, seed):
    x = WL.edge_mix(5000 + seed * 37, seed)
    lo, hi, anyf = orc.value_range(x)
    f = x[np.isfinite(x)]
    assert anyf == (f.size > 0)
    assert np.float32(lo) == f.min() and np.float32(hi) == f.max()
    assert np.float32(lo).view(np.uint32) == (f.min() + np.float32(0)).view(np.uint32)


def test_value_range_special(orc):
    assert orc.value_range(np.array([np.nan, np.inf, -np.inf], np.float32)) == (0.0, 0.0, False)
    assert orc.value_range(np.array([], np.float32)) == (0.0, 0.0, False)
    lo, hi, _ = orc.value_range(np.array([-0.0, -0.0], np.float32))
    assert np.float32(lo).view(np.uint32) == 0 and np.float32(hi).view(np.uint32) == 0  # canonical +0


# --------------------------------------------------------------------------------------
# Step 2: bound resolution -- exact rationals with the stated roundings
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("rel,vmin,vmax", [(0.25, -1.0, 3.0), (1e-3, 0.0, 1.0), (1e-4, -3.7, 4.1),
                                           (1e-6, -1e3, 999.5), (0.1, 5.0, 5.0), (1e-2, -1e-38, 1e-38)])
def test_resolve_bound_exact(orc, rel, vmin, vmax):
    b = orc.resolve_bound(False, rel, vmin, vmax)
    vmin32, vmax32 = np.float32(vmin), np.float32(vmax)
    diff = float(Fraction(float(vmax32)) - Fraction(float(vmin32)))       # one double rounding
    eb = float(Fraction(rel) * Fraction(diff))                            # one double rounding
    assert b.eb == eb
    if eb == 0:
        assert np.isinf(b.inv2eb) and b.step == 0
    else:
        with np.errstate(over="ignore"):
            assert b.inv2eb == np.float32(float(Fraction(1) / (2 * Fraction(eb))))
        assert b.step == np.float32(2 * eb)


def test_resolve_bound_absolute(orc):
    b = orc.resolve_bound(True, 1e-7)
    assert b.eb == 1e-7
    assert b.step == np.float32(2e-7)
    assert b.inv2eb == np.float32(float(Fraction(1) / (2 * Fraction(1e-7))))
    assert abs(float(b.step) * float(b.inv2eb) - 1.0) < 2.0 ** -22


# --------------------------------------------------------------------------------------
# Step 3: quantisation and outlier test -- exact rational arithmetic
# --------------------------------------------------------------------------------------

def _quant_cases():
    rng = np.random.default_rng(11)
    out = []
    for eb in (0.5, 1.0 / 16, 1e-3, 1.0 / 6, 1e-7, 2.0, 3.1e-5):
        x = np.concatenate([rng.standard_normal(400) * s for s in (1e-6, 1e-3, 1.0, 1e3)]).astype(np.float32)
        out.append((eb, x))
    # exact ties of x*inv2eb: inv2eb = 8 (eb = 1/16), x = (k + 0.5)/8
    k = np.arange(-300, 300)
    out.append((1.0 / 16, ((k + 0.5) / 8).astype(np.float32)))
    # near the int range limit: |y| around 2^30
    inv = float(np.float32(1 / (2 * 1e-3)))
    ys = np.array([2 ** 30 - 64, 2 ** 30 - 1, 2 ** 30, 2 ** 30 + 128, -2 ** 30, -(2 ** 30) + 64], np.float64)
    out.append((1e-3, (ys / inv).astype(np.float32)))
    out.append((1e-3, WL.edge_mix(600, 3)))
    return out


@pytest.mark.parametrize("case", range(len(_quant_cases())))
def test_quantize_exact(orc, case):
    eb, x = _quant_cases()[case]
    b = orc.resolve_bound(True, eb)
    q, flag = orc.quantize(x, b)
    qe, fe, amb = SC.exact_codes_and_flags(x, b.inv2eb, b.step, b.eb)
    assert np.array_equal(q.astype(np.int64), qe)
    ok = (flag == fe) | amb
    assert ok.all(), np.flatnonzero(~ok)[:10]
    for i in np.flatnonzero(amb):  # fp64 test decides where the exact error is within an ulp of eb
        xr = float(np.float32(q[i]) * b.step)
        assert flag[i] == (not (abs(float(x[i]) - xr) <= b.eb))


def test_quantize_special_values(orc):
    b = orc.resolve_bound(True, 1.0 / 16)  # inv2eb = 8, step = 0.125
    x = np.array([0.0, -0.0, 1.0 / 16, 3.0 / 16, -1.0 / 16, 2.0 ** 28, np.inf, -np.inf, np.nan], np.float32)
    q, flag = orc.quantize(x, b)
    # 1/16*8 = 0.5 -> 0 (even); 3/16*8 = 1.5 -> 2; -0.5 -> -0 -> 0; 2^28*8 = 2^31 out of range
    assert q.tolist() == [0, 0, 0, 2, 0, 0, 0, 0, 0]
    assert flag.tolist() == [False, False, False, False, False, True, True, True, True]


def test_zero_bound_is_lossless_via_outliers(orc):
    x = WL.edge_mix(3000, 5)
    s = orc.compress(x, 64, abs=0.0)
    y = orc.decompress(s, x.size)
    nz = x.view(np.uint32) & np.uint32(0x7FFFFFFF) != 0
    assert np.array_equal(y.view(np.uint32)[nz], x.view(np.uint32)[nz])
    assert np.all(y.view(np.uint32)[~nz] == 0)  # +-0 reconstruct as +0
    assert SC.header(s)["m"] == int(nz.sum())


# --------------------------------------------------------------------------------------
# Steps 4-5: delta and zigzag -- closed forms, bijection
# --------------------------------------------------------------------------------------

def test_zigzag_order_and_bijection(orc):
    # the textbook zigzag enumerates 0, -1, 1, -2, 2, ... as 0, 1, 2, 3, 4, ...
    seq = [0] + [v for k in range(1, 2000) for v in (-k, k)]
    assert [orc.zigzag(d) for d in seq] == list(range(len(seq)))
    edges = [0, 1, -1, 2 ** 30 - 1, -(2 ** 30), 2 ** 31 - 2, -(2 ** 31) + 2, 2 ** 31 - 1, -(2 ** 31)]
    for d in edges:
        assert orc.unzigzag(orc.zigzag(d)) == d
        assert orc.zigzag(d) == (2 * d if d >= 0 else -2 * d - 1)
    rng = np.random.default_rng(3)
    for z in rng.integers(0, 2 ** 32, size=2000, dtype=np.uint64):
        assert orc.zigzag(orc.unzigzag(int(z))) == int(z)


def test_codes_and_widths_vs_numpy_diff(orc):
    rng = np.random.default_rng(5)
    for B in BLOCKS:
        x = (np.cumsum(rng.standard_normal(3 * B + 17)) * 3).astype(np.float32)
        b = orc.resolve_bound(True, 0.01)
        q, _ = orc.quantize(x, b)
        z, w = orc.block_codes(x, B, b.inv2eb)
        assert np.array_equal(w.astype(np.int64), SC.widths_from_codes(q, B))
        for s in range(0, x.size, B):
            d = np.diff(np.concatenate([[0], q[s:s + B].astype(np.int64)]))
            assert np.array_equal(z[s:s + B].astype(np.int64), np.where(d >= 0, 2 * d, -2 * d - 1))


# --------------------------------------------------------------------------------------
# Step 6: width and bitpack -- bit matrices, exhaustive over widths and counts
# --------------------------------------------------------------------------------------

def test_width_is_minimal(orc):
    rng = np.random.default_rng(1)
    assert orc.block_width(np.zeros(7, np.uint32)) == 0
    for w in range(33):
        for _ in range(5):
            z = rng.integers(0, 2 ** w, size=rng.integers(1, 257), dtype=np.uint64).astype(np.uint32) if w else \
                np.zeros(5, np.uint32)
            expect = max(int(v).bit_length() for v in z)
            assert orc.block_width(z) == expect


def test_pack_layout_bitmatrix_exhaustive(orc):
    rng = np.random.default_rng(2)
    for w in range(33):
        for cnt in range(1, 257):
            z = rng.integers(0, 2 ** w, size=cnt, dtype=np.uint64).astype(np.uint32) if w else \
                np.zeros(cnt, np.uint32)
            words = orc.pack_block(z, w)
            assert words.size == (w * cnt + 31) // 32
            bits = np.unpackbits(words.view(np.uint8), bitorder="little")
            want = ((z[:, None].astype(np.uint64) >> np.arange(w, dtype=np.uint64)) & 1).astype(np.uint8)
            assert np.array_equal(bits[: w * cnt], want.reshape(-1))
            assert not bits[w * cnt:].any()
            assert np.array_equal(orc.unpack_block(words, cnt, w), z)


# --------------------------------------------------------------------------------------
# Whole streams: bound invariant, lossless outliers, layout closed forms,
# independent bit-matrix decode of the codes
# --------------------------------------------------------------------------------------

def _check_stream(orc, x, s, block, eb_expected=None):
    P = SC.parts(s)
    h, off = P["h"], P["off"]
    n = x.size
    assert h["magic"] == SC.MAGIC and h["n"] == n and h["block"] == block and h["chunk"] == SC.CHUNK
    assert h["reserved"] == bytes(32)
    cnt = SC.block_counts(n, block)
    assert h["nb"] == cnt.size and h["nc"] == -(-n // SC.CHUNK)
    words = -(-(P["widths"] * cnt) // 32)
    assert h["W"] == int(words.sum())
    assert off["total"] == h["total"] == s.size
    if eb_expected is not None:
        assert h["eb"] == eb_expected
    b = orc.Bound(h["eb"], np.float32(h["inv2eb"]), np.float32(h["step"]))
    q, flag = orc.quantize(x, b)
    # codes recovered from the payload with a bit matrix equal the quantiser's codes
    assert np.array_equal(SC.decode_codes_bitmatrix(s), q.astype(np.int64))
    assert np.array_equal(P["widths"], SC.widths_from_codes(q, block))
    # outlier list: ascending, exactly the flagged elements, raw bits
    assert h["m"] == int(flag.sum())
    assert np.array_equal(P["idx"], np.flatnonzero(flag).astype(np.uint32))
    assert np.array_equal(P["val"], x.view(np.uint32)[flag])
    # chunk index: record word offset and outliers before each chunk
    per_chunk_m = np.add.reduceat(flag.astype(np.int64), np.arange(0, n, SC.CHUNK)) if n else np.zeros(0, np.int64)
    bpc = SC.CHUNK // block
    chunk_words = np.add.reduceat(words, np.arange(0, cnt.size, bpc)) if cnt.size else np.zeros(0, np.int64)
    rec_sizes = chunk_words + 2 * per_chunk_m
    assert np.array_equal(P["index"][:, 0], np.concatenate([[0], np.cumsum(rec_sizes)])[:-1])
    assert np.array_equal(P["index"][:, 1], np.concatenate([[0], np.cumsum(per_chunk_m)])[:-1])
    assert np.array_equal(P["chunk_m"], per_chunk_m)
    # padding bytes are zero
    raw = P["raw"]
    assert not raw[off["width"] + h["nb"]:off["index"]].any()
    assert not raw[off["index"] + 8 * h["nc"]:off["record"]].any()
    # reconstruction: within eb in fp64 for non-outliers, outliers bit-exact
    y = orc.decompress(s, n)
    keep = ~flag
    err = np.abs(x[keep].astype(np.float64) - y[keep].astype(np.float64))
    assert np.all(err <= h["eb"])
    assert np.array_equal(y.view(np.uint32)[flag], x.view(np.uint32)[flag])
    assert np.all(np.isfinite(x[keep]))
    return h


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("n", [0, 1, 31, 32, 33, 255, 257, 4095, 4096, 4097, 3 * 4096 + 7, 20011])
def test_stream_invariants_sizes(orc, block, n):
    x = WL.edge_mix(n, n + block)
    s = orc.compress(x, block, rel=1e-3)
    lo, hi, _ = orc.value_range(x)
    _check_stream(orc, x, s, block, orc.resolve_bound(False, 1e-3, lo, hi).eb)


@pytest.mark.parametrize("mode,bound", [("rel", 1e-2), ("rel", 1e-5), ("abs", 1e-7), ("abs", 0.3), ("abs", 0.0),
                                        ("rel", 0.0)])
@pytest.mark.parametrize("gen", ["sine", "field", "spikes", "noise"])
def test_stream_invariants_workloads(orc, mode, bound, gen):
    rng = np.random.default_rng(7)
    n = 50000
    if gen == "sine":
        x = WL.sine_noise(n, 0)
    elif gen == "field":
        x = WL.kfield((40, 50, 25), 1)
    elif gen == "spikes":
        x = WL.with_spikes((32, 40, 40), 2, p_nonfinite=1e-3)
    else:
        x = rng.uniform(-1, 1, n).astype(np.float32)
    for block in (32, 256):
        s = orc.compress(x, block, **{mode: bound})
        _check_stream(orc, x, s, block)


def test_noise_zero_ramp_small(orc):
    x = WL.noise_zero_ramp(1 << 16, 4)
    s = orc.compress(x, 128, abs=1e-7)
    h = _check_stream(orc, x, s, 128)
    P = SC.parts(s)
    assert (P["widths"][(1 << 15) // 128:(3 << 14) // 128] == 0).all()  # the zero quarter costs no payload
    assert h["m"] > 0


def test_constant_and_nonfinite_inputs(orc):
    x = np.full(1000, 3.25, np.float32)  # range 0 -> eb 0 -> every nonzero element is an outlier
    s = orc.compress(x, 64, rel=1e-3)
    h = _check_stream(orc, x, s, 64, 0.0)
    assert h["m"] == 1000
    x = np.full(300, np.nan, np.float32)
    x.view(np.uint32)[::3] = 0x7FC00001
    s = orc.compress(x, 32, rel=1e-3)
    h = _check_stream(orc, x, s, 32, 0.0)
    assert h["m"] == 300 and (h["vmin"], h["vmax"]) == (0.0, 0.0)
    x = np.zeros(5000, np.float32)
    s = orc.compress(x, 128, rel=1e-3)
    h = _check_stream(orc, x, s, 128, 0.0)
    assert h["m"] == 0 and h["W"] == 0


def test_errors(orc):
    x = WL.edge_mix(5000, 9)
    s = orc.compress(x, 64, abs=1e-3)
    m = SC.header(s)["m"]
    assert m > 0
    with pytest.raises(orc.OracleError) as e:
        orc.compress(x, 64, abs=1e-3, outlier_cap=m - 1)
    assert e.value.code == orc.ERR_OUTLIER_CAP
    assert orc.compress(x, 64, abs=1e-3, outlier_cap=m).size == s.size
    with pytest.raises(orc.OracleError) as e:
        orc.compress(x, 64, abs=1e-3, out_cap=s.size - 1)
    assert e.value.code == orc.ERR_CAPACITY
    for bad in (48, 512, 0):
        with pytest.raises(orc.OracleError):
            orc.compress(x, bad, abs=1e-3)
    with pytest.raises(orc.OracleError):
        orc.compress(x, 64, abs=-1.0)
    # corrupt streams are rejected
    t = s.copy(); t[0] ^= 1
    with pytest.raises(orc.OracleError):
        orc.decompress(t, x.size)
    t = s.copy(); t[128] = 33
    with pytest.raises(orc.OracleError):
        orc.decompress(t, x.size)
    with pytest.raises(orc.OracleError):
        orc.decompress(s[:-4], x.size)


# --------------------------------------------------------------------------------------
# Brute force over tiny inputs
# --------------------------------------------------------------------------------------

def _grid(eb):
    inv = float(np.float32(1.0 / (2 * eb)))
    vals = [0.0, -0.0, eb / 2, -eb / 2, eb, -eb, 3 * eb, -3 * eb, 2 ** 30 / inv, -(2 ** 31) / inv,
            1e-42, np.nan, np.inf, -np.inf]
    return np.array(vals, np.float32)


@pytest.mark.parametrize("eb", [0.25, 1e-3, 1e-7])
def test_bruteforce_tiny(orc, eb):
    g = _grid(eb)
    for n in (1, 2, 3):
        for combo in itertools.product(range(g.size), repeat=n):
            x = g[list(combo)]
            s = orc.compress(x, 32, abs=eb)
            h = SC.header(s)
            assert h["total"] == s.size == SC.sections(h)["total"]
            y = orc.decompress(s, n)
            b = orc.resolve_bound(True, eb)
            _, fe, amb = SC.exact_codes_and_flags(x, b.inv2eb, b.step, b.eb)
            q, flag = orc.quantize(x, b)
            assert (np.array_equal(flag, fe) or amb.any())
            for i in range(n):
                if flag[i]:
                    assert y.view(np.uint32)[i] == x.view(np.uint32)[i]
                else:
                    assert abs(float(x[i]) - float(y[i])) <= eb
            assert h["m"] == int(flag.sum())
    # relative mode over the same grid (n = 3): eb follows the finite range
    for combo in itertools.product(range(g.size), repeat=3):
        x = g[list(combo)]
        s = orc.compress(x, 32, rel=0.01)
        y = orc.decompress(s, 3)
        h = SC.header(s)
        f = x[np.isfinite(x)]
        rng_ = (float(f.max()) - float(f.min())) if f.size else 0.0
        assert h["eb"] == 0.01 * rng_
        for i in range(3):
            assert (y.view(np.uint32)[i] == x.view(np.uint32)[i]) or abs(float(x[i]) - float(y[i])) <= h["eb"]


# --------------------------------------------------------------------------------------
# Golden fixtures written by tests/golden/make_golden.py (which calls only the oracle)
# --------------------------------------------------------------------------------------

def test_golden_fixtures(orc):
    path = os.path.join(GOLDEN, "oracle_streams.json")
    with open(path) as f:
        cases = json.load(f)["cases"]
    from tests.golden.make_golden import case_input

    for c in cases:
        x = case_input(c)
        assert WL.sha256(x) == c["input_sha256"]
        s = orc.compress(x, c["block"], **{c["mode"]: c["bound"]})
        assert s.size == c["total"]
        assert WL.sha256(s) == c["stream_sha256"], c["name"]


# --------------------------------------------------------------------------------------
# Property-based: random small arrays mixing ordinary values, huge and tiny magnitudes,
# ties, signed zeros and non-finite values, over both bound modes and every block size
# --------------------------------------------------------------------------------------

def _fuzz_settings():
    from hypothesis import HealthCheck, settings

    return settings(max_examples=120, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])


def test_stream_invariants_fuzz(orc):
    from hypothesis import given
    from hypothesis import strategies as st

    finite = st.floats(width=32, allow_nan=False, allow_infinity=False)
    special = st.sampled_from([0.0, -0.0, float("nan"), float("inf"), float("-inf"), 1e-45, -1e-45, 2.0 ** 30,
                               -(2.0 ** 31), 0.5, 1.5, 2.5, 1e38])
    values = st.lists(st.one_of(finite, special, st.floats(-10, 10, width=32)), min_size=0, max_size=600)

    @_fuzz_settings()
    @given(values, st.sampled_from([32, 64, 128, 256]), st.sampled_from(["rel", "abs"]),
           st.sampled_from([0.0, 1e-7, 1e-4, 1e-2, 0.25, 3.0, 1e30]))
    def check(vals, block, mode, bound):
        x = np.array(vals, dtype=np.float32)
        s = orc.compress(x, block, **{mode: bound})
        _check_stream(orc, x, s, block)

    check()


def test_stream_invariants_fuzz_multichunk(orc):
    """Sizes across several 4096-element chunks and ragged tails, values from a
    seeded mixture (smooth, noisy, spikes, specials), random bound and block."""
    from hypothesis import given
    from hypothesis import strategies as st

    @_fuzz_settings()
    @given(st.integers(0, 2 ** 32 - 1), st.sampled_from([1, 4095, 4096, 4097, 8191, 3 * 4096 + 17, 5 * 4096]),
           st.sampled_from([32, 64, 128, 256]), st.sampled_from(["rel", "abs"]),
           st.sampled_from([0.0, 1e-6, 1e-3, 0.1, 10.0]))
    def check(seed, n, block, mode, bound):
        rng = np.random.default_rng(seed)
        t = np.arange(n)
        x = np.sin(t / rng.uniform(5, 500)) * rng.uniform(0.1, 1e3) + rng.normal(0, rng.uniform(0, 1), n)
        spikes = rng.random(n) < rng.uniform(0, 0.05)
        x[spikes] = rng.uniform(-1e6, 1e6, int(spikes.sum()))
        bad = rng.random(n) < 1e-3
        x[bad] = rng.choice([np.nan, np.inf, -np.inf, 0.0, -0.0], int(bad.sum()))
        x = x.astype(np.float32)
        s = orc.compress(x, block, **{mode: bound})
        _check_stream(orc, x, s, block)

    check()


# ---------------------------------------------------------------------------
# compress_range: one part of a larger array under the whole array's bound.

def _chunk_records(s):
    """Per chunk: (width bytes of its blocks, its record words) of a stream."""
    P = SC.parts(s)
    h = P["h"]
    rec = P["raw"][P["off"]["record"]:P["off"]["total"]].view(np.uint32)
    R = h["W"] + 2 * h["m"]
    starts = list(P["index"][:, 0]) + [R]
    bpc = SC.CHUNK // h["block"]
    return [(P["widths"][c * bpc:(c + 1) * bpc].copy(), rec[starts[c]:starts[c + 1]].copy())
            for c in range(h["nc"])]


@pytest.mark.parametrize("block", BLOCKS)
def test_compress_range_with_own_range_is_compress(orc, block):
    for x in (WL.with_spikes((12, 32, 48), 2, p_nonfinite=1e-3), WL.edge_mix(9001, block), WL.sine_noise(5000, 1)):
        lo, hi, _ = orc.value_range(x)
        assert np.array_equal(orc.compress_range(x, block, 1e-3, lo, hi), orc.compress(x, block, rel=1e-3))


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("parts", [2, 3, 5])
def test_compress_range_shards_match_the_whole_stream(orc, block, parts):
    """Chunk-aligned parts coded under the whole array's range: each part's
    stream passes every independent stream check with eb = rel * (vmax - vmin)
    of the whole (exact rationals), and its width bytes, payload words and
    outlier values are byte for byte those of the whole array's stream for
    the same chunks (outlier indices count from the part's first element)."""
    rel = 1e-3
    x = np.concatenate([WL.kfield((8, 32, 64), 3), WL.with_spikes((8, 16, 64), 4, p_nonfinite=2e-3),
                        WL.edge_mix(3 * 4096 + 77, 5)])
    lo, hi, _ = orc.value_range(x)
    eb = float(Fraction(rel) * Fraction(float(Fraction(float(np.float32(hi))) - Fraction(float(np.float32(lo))))))
    whole = _chunk_records(orc.compress(x, block, rel=rel))
    nc = -(-x.size // SC.CHUNK)
    cuts = [0] + [(nc * k // parts) * SC.CHUNK for k in range(1, parts)] + [x.size]
    c0 = 0
    for a, b in zip(cuts[:-1], cuts[1:]):
        s = orc.compress_range(x[a:b], block, rel, lo, hi)
        h = _check_stream(orc, x[a:b], s, block, eb_expected=eb)
        assert h["vmin"] == np.float32(lo) and h["vmax"] == np.float32(hi) and h["flags"] == 0
        mine = _chunk_records(s)
        for k, (w, r) in enumerate(mine):
            W, Rw = whole[c0 + k]
            assert np.array_equal(w, W[:w.size]) and not W[w.size:].any()
            # same payload words and outlier values; outlier indices are the
            # part's own (element index within the part)
            pw = int((-(-(w.astype(np.int64) * SC.block_counts(b - a, block)[
                k * (SC.CHUNK // block):(k + 1) * (SC.CHUNK // block)]) // 32)).sum())
            mc = (r.size - pw) // 2
            assert r.size == Rw.size and pw + 2 * mc == r.size
            assert np.array_equal(r[:pw], Rw[:pw]), (a, k)
            assert np.array_equal(r[pw:pw + mc].astype(np.int64) + a, Rw[pw:pw + mc].astype(np.int64)), (a, k)
            assert np.array_equal(r[pw + mc:], Rw[pw + mc:]), (a, k)
        c0 += len(mine)
    assert c0 == nc


def test_compress_range_rejects_bad_ranges(orc):
    x = WL.edge_mix(100, 1)
    for lo, hi in ((1.0, 0.0), (np.nan, 1.0), (0.0, np.inf)):
        with pytest.raises(orc.OracleError):
            orc.compress_range(x, 64, 1e-3, lo, hi)
