"""Pins of the oracle's chunk-cooperative codec (Quant -> Diff -> Bitshuffle
-> RZE, orc_compress_chunked), each against an independent restatement:

* Bitshuffle against a NumPy bit matrix (np.unpackbits / np.packbits, little
  bit order) and single-bit placements; the inverse round-trips;
* RZE against a NumPy nonzero mask (bitmap packed little-endian, then the
  nonzero words); the inverse round-trips and rejects a short payload;
* RRE against a NumPy "differs from the word before" mask and a hand-worked
  example; its inverse against a NumPy forward fill of the kept words;
* every stream decoded end to end in NumPy (record words, zero elimination,
  the bit matrix, zigzag, cumulative sum per chunk), compared with the
  quantiser's codes, with the outlier list and the bound on every element;
  chunks that keep their shuffled words verbatim and ragged final chunks.
CPU only."""
import struct

import numpy as np
import pytest

from error_bounded_lossy_encode_b200 import workloads as WL

CHUNK_BYTES = (4096, 8192, 16384)


def _np_bitshuffle(words):
    mp = words.size
    bits = np.unpackbits(words.astype("<u4").view(np.uint8), bitorder="little").reshape(mp // 32, 32, 32)
    planes = bits.transpose(2, 0, 1)  # (bit b, group g, lane l)
    return np.packbits(planes.reshape(-1), bitorder="little").view("<u4").astype(np.uint32)


def _np_rze(words):
    bm = np.packbits((words != 0).astype(np.uint8), bitorder="little").view("<u4").astype(np.uint32)
    return np.concatenate([bm, words[words != 0]])


@pytest.mark.parametrize("mp", [32, 64, 96, 1024, 4096])
def test_bitshuffle_vs_numpy_bit_matrix(orc, mp):
    rng = np.random.default_rng(mp)
    for scale in (2, 1 << 10, 1 << 32):
        w = rng.integers(0, scale, size=mp, dtype=np.uint64).astype(np.uint32)
        sh = orc.bitshuffle(w)
        assert np.array_equal(sh, _np_bitshuffle(w))
        assert np.array_equal(orc.unbitshuffle(sh), w)


def test_bitshuffle_single_bits(orc):
    for G in (1, 2, 3):
        for g in range(G):
            for l in (0, 5, 31):
                for b in (0, 7, 31):
                    w = np.zeros(32 * G, np.uint32)
                    w[32 * g + l] = np.uint32(1 << b)
                    sh = orc.bitshuffle(w)
                    want = np.zeros(32 * G, np.uint32)
                    want[b * G + g] = np.uint32(1 << l)
                    assert np.array_equal(sh, want), (G, g, l, b)


@pytest.mark.parametrize("density", [0.0, 0.05, 0.5, 1.0])
def test_rze_vs_numpy(orc, density):
    rng = np.random.default_rng(int(density * 100))
    w = rng.integers(1, 1 << 32, size=1024, dtype=np.uint64).astype(np.uint32)
    w[rng.random(1024) >= density] = 0
    r = orc.rze(w)
    assert np.array_equal(r, _np_rze(w))
    back, used = orc.unrze(r, 1024)
    assert used == r.size and np.array_equal(back, w)
    if r.size > 32:
        with pytest.raises(orc.OracleError):
            orc.unrze(r[:-1], 1024)


def _np_rre(words):
    pred = np.concatenate([np.zeros(1, np.uint32), words[:-1]])
    keep = words != pred
    bm = np.packbits(keep.astype(np.uint8), bitorder="little").view("<u4").astype(np.uint32)
    return np.concatenate([bm, words[keep]])


def _np_unrre(pay, mp):
    """Each word is the last kept word at or before it (0 before the first)."""
    keep = np.unpackbits(pay[:mp // 32].view(np.uint8), bitorder="little")[:mp].astype(bool)
    vals = np.concatenate([np.zeros(1, np.uint32), pay[mp // 32:]])
    return vals[np.cumsum(keep)], int(keep.sum())


def test_rre_hand_worked(orc):
    # words 0 0 5 5 5 7 0 0 (then zeros): 5, 7 and 0 differ from their predecessors at 2, 5, 6
    w = np.zeros(32, np.uint32)
    w[2:5], w[5] = 5, 7
    r = orc.rre(w)
    assert list(r) == [(1 << 2) | (1 << 5) | (1 << 6), 5, 7, 0]
    back, used = orc.unrre(r, 32)
    assert used == 4 and np.array_equal(back, w)
    # a run of one nonzero value costs one word, where zero elimination keeps all of them
    v = np.full(64, 9, np.uint32)
    assert list(orc.rre(v)) == [1, 0, 9] and orc.rze(v).size == 2 + 64


@pytest.mark.parametrize("density", [0.0, 0.05, 0.5, 1.0])
def test_rre_vs_numpy(orc, density):
    rng = np.random.default_rng(7 + int(density * 100))
    w = rng.integers(0, 4, size=1024, dtype=np.uint32)  # few distinct values: runs and repeats
    w[rng.random(1024) >= density] = 0
    r = orc.rre(w)
    assert np.array_equal(r, _np_rre(w))
    back, used = orc.unrre(r, 1024)
    want, kept = _np_unrre(r, 1024)
    assert used == r.size == 32 + kept and np.array_equal(back, w) and np.array_equal(want, w)
    if r.size > 32:
        with pytest.raises(orc.OracleError):
            orc.unrre(r[:-1], 1024)


def _np_decode(stream):
    """Independent decode of a chunked stream: codes (int64) and the outlier
    (index, bits) pairs."""
    s = np.asarray(stream, np.uint8)
    (magic, version, flags, n, block, chunk, eb, inv2eb, step, vmin, vmax, nb, nc, W, m, total, bound) = \
        struct.unpack_from("<IHHQIIdffffQQQQQd", bytes(s[:128]))
    assert magic == 0x434C4245 and flags & 4 and block == 0 and nb == 0 and total == s.size
    rre = bool(flags & 8)
    index_off = 128
    record_off = index_off + -(-8 * nc // 16) * 16
    index = s[index_off:index_off + 8 * nc].view("<u4").reshape(-1, 2).astype(np.int64)
    rec = s[record_off:].view("<u4").astype(np.int64)
    codes = np.zeros(n, np.int64)
    oidx, oval, words_seen, raws = [], [], 0, []
    for c in range(nc):
        r0 = int(index[c, 0])
        r1 = int(index[c + 1, 0]) if c + 1 < nc else W + 2 * m
        mc = (int(index[c + 1, 1]) if c + 1 < nc else m) - int(index[c, 1])
        e0, e1 = c * chunk, min(n, (c + 1) * chunk)
        mp = -(-(e1 - e0) // 32) * 32
        head = int(rec[r0])
        P, raw = head & 0x7FFFFFFF, head >> 31
        raws.append(raw)
        assert r1 - r0 == 1 + P + 2 * mc
        pay = rec[r0 + 1:r0 + 1 + P].astype(np.uint32)
        if raw:
            assert P == mp
            sh = pay
        elif rre:
            sh, kept = _np_unrre(pay, mp)
            assert P == mp // 32 + kept and P < mp  # verbatim only when repetition elimination would not shrink
        else:
            bits = np.unpackbits(pay[:mp // 32].view(np.uint8), bitorder="little")[:mp].astype(bool)
            sh = np.zeros(mp, np.uint32)
            sh[bits] = pay[mp // 32:]
            assert P == mp // 32 + int(bits.sum()) and P < mp  # verbatim only when zero elimination would not shrink
        bitsm = np.unpackbits(sh.view(np.uint8), bitorder="little").reshape(32, mp // 32, 32)  # (b, g, l)
        z = np.packbits(bitsm.transpose(1, 2, 0).reshape(-1), bitorder="little").view("<u4").astype(np.int64)
        d = np.where(z % 2 == 0, z // 2, -(z + 1) // 2)
        codes[e0:e1] = np.cumsum(d[:e1 - e0])
        oidx.append(rec[r0 + 1 + P:r0 + 1 + P + mc])
        oval.append(rec[r0 + 1 + P + mc:r0 + 1 + P + 2 * mc])
        words_seen += 1 + P
    assert words_seen == W
    cat = lambda a: np.concatenate(a) if a else np.zeros(0, np.int64)
    return codes, cat(oidx), cat(oval), dict(eb=eb, inv2eb=inv2eb, step=step, n=n, m=m, raw=raws, rre=rre)


def _check(orc, x, s):
    codes, oidx, oval, h = _np_decode(s)
    b = orc.Bound(h["eb"], np.float32(h["inv2eb"]), np.float32(h["step"]))
    q, flag = orc.quantize(x, b)
    wrap = lambda v: ((v + (1 << 31)) % (1 << 32)) - (1 << 31)
    assert np.array_equal(wrap(codes), q.astype(np.int64))
    assert np.array_equal(oidx, np.flatnonzero(flag)) and np.array_equal(oval, x.view(np.uint32)[flag].astype(np.int64))
    y = orc.decompress(s, x.size)
    keep = ~flag
    assert np.all(np.abs(x[keep].astype(np.float64) - y[keep].astype(np.float64)) <= h["eb"])
    assert np.array_equal(y.view(np.uint32)[flag], x.view(np.uint32)[flag])
    return h


@pytest.mark.parametrize("coder", ["rze", "rre"])
@pytest.mark.parametrize("cb", CHUNK_BYTES)
@pytest.mark.parametrize("bound", [("rel", 1e-3), ("rel", 1e-6), ("abs", 1e-7), ("abs", 0.0)])
def test_chunked_stream_independent_decode(orc, cb, bound, coder):
    x = np.concatenate([WL.with_spikes((8, 32, 64), 3, p_nonfinite=2e-3), WL.edge_mix(cb // 4 * 2 + 77, 5),
                        WL.sine_noise(5000, 2)])
    h = _check(orc, x, orc.compress_chunked(x, cb, coder=coder, **{bound[0]: bound[1]}))
    assert h["rre"] == (coder == "rre")


def test_rre_stream_shrinks_repeated_words(orc):
    """A ramp with a constant step per element quantizes to codes with one
    constant first difference: every group's plane words repeat the group
    before, so RRE keeps a word per plane change where RZE keeps every
    nonzero plane word.  On sparse differences (a ramp that steps every 64
    elements) a nonzero word is followed by zeros and RRE keeps both, so
    there RZE is the smaller one."""
    ramp = (np.arange(1 << 14, dtype=np.float64) * 0.004).astype(np.float32)
    a = orc.compress_chunked(ramp, 16384, abs=1e-3, coder="rze")
    b = orc.compress_chunked(ramp, 16384, abs=1e-3, coder="rre")
    _check(orc, ramp, a)
    _check(orc, ramp, b)
    assert b.size < a.size
    steps = (np.arange(1 << 14, dtype=np.float64) // 64 * 0.01).astype(np.float32)
    a = orc.compress_chunked(steps, 16384, abs=1e-3, coder="rze")
    b = orc.compress_chunked(steps, 16384, abs=1e-3, coder="rre")
    _check(orc, steps, a)
    _check(orc, steps, b)
    assert a.size < b.size


@pytest.mark.parametrize("cb", CHUNK_BYTES)
def test_chunked_verbatim_and_sizes(orc, cb):
    rng = np.random.default_rng(cb)
    # differences of codes up to 2^29 fill every bit plane: zero elimination cannot shrink, the chunk stays verbatim
    noise = rng.uniform(-1e9, 1e9, 3 * cb // 4).astype(np.float32)
    for coder in ("rze", "rre"):
        s = orc.compress_chunked(noise, cb, abs=1.0, coder=coder)
        h = _check(orc, noise, s)
        assert any(h["raw"]) and s.size <= orc.max_chunked_bytes(noise.size, cb)
    smooth = orc.compress_chunked(WL.sine_noise(3 * cb // 4, 1), cb, rel=1e-3)
    assert not any(_check(orc, WL.sine_noise(3 * cb // 4, 1), smooth)["raw"])
    for n in (0, 1, 31, 33, cb // 4 - 1, cb // 4, cb // 4 + 1):
        _check(orc, WL.edge_mix(n, n + cb), orc.compress_chunked(WL.edge_mix(n, n + cb), cb, rel=1e-3))
    with pytest.raises(orc.OracleError):
        orc.compress_chunked(noise, 2048, rel=1e-3)
