"""Independent checks of a compressed stream, written with different
primitives from the oracle (struct for the header, NumPy bit matrices for the
payload, closed forms for zigzag and the prefix sum, exact rationals for the
rounding steps).  Used to pin the oracle and to validate GPU streams.
"""
from __future__ import annotations

import struct
from fractions import Fraction

import numpy as np

HEADER_FMT = "<IHHQIIdffffQQQQQd"
HEADER_KEYS = ("magic", "version", "flags", "n", "block", "chunk", "eb", "inv2eb", "step", "vmin", "vmax",
               "nb", "nc", "W", "m", "total", "bound")
MAGIC = 0x434C4245
CHUNK = 4096


def pad16(v: int) -> int:
    return -(-v // 16) * 16


def header(stream) -> dict:
    b = bytes(np.asarray(stream, dtype=np.uint8)[:128])
    vals = struct.unpack_from(HEADER_FMT, b, 0)
    h = dict(zip(HEADER_KEYS, vals))
    h["reserved"] = b[96:128]
    return h


def sections(h: dict) -> dict:
    w_off = 128
    i_off = w_off + pad16(h["nb"])
    r_off = i_off + pad16(8 * h["nc"])
    return dict(width=w_off, index=i_off, record=r_off, total=r_off + 4 * (h["W"] + 2 * h["m"]))


def block_counts(n: int, block: int) -> np.ndarray:
    nb = -(-n // block)
    cnt = np.full(nb, block, np.int64)
    if nb and n % block:
        cnt[-1] = n % block
    return cnt


def parts(stream) -> dict:
    """Split a stream into its sections.  Records are walked chunk by chunk
    with the widths (payload words of each block) and the chunk index
    (outliers per chunk); payload words of all chunks are concatenated, and so
    are the outlier index and value arrays."""
    s = np.asarray(stream, dtype=np.uint8)
    h = header(s)
    off = sections(h)
    widths = s[off["width"]:off["width"] + h["nb"]].astype(np.int64)
    index = s[off["index"]:off["index"] + 8 * h["nc"]].view(np.uint32).reshape(-1, 2).astype(np.int64) \
        if h["nc"] else np.zeros((0, 2), np.int64)
    rec = s[off["record"]:off["total"]].view(np.uint32)
    cnt = block_counts(h["n"], h["block"])
    bwords = -(-(widths * cnt) // 32)
    bpc = CHUNK // h["block"]
    payload, idx, val, chunk_m, chunk_words = [], [], [], [], []
    for c in range(h["nc"]):
        r0 = int(index[c, 0])
        m_c = (int(index[c + 1, 1]) if c + 1 < h["nc"] else h["m"]) - int(index[c, 1])
        pw = int(bwords[c * bpc:(c + 1) * bpc].sum())
        payload.append(rec[r0:r0 + pw])
        idx.append(rec[r0 + pw:r0 + pw + m_c])
        val.append(rec[r0 + pw + m_c:r0 + pw + 2 * m_c])
        chunk_m.append(m_c)
        chunk_words.append(pw)
    cat = lambda a: np.concatenate(a).astype(np.uint32) if a else np.zeros(0, np.uint32)
    return dict(h=h, off=off, widths=widths, index=index, payload=cat(payload).view(np.uint8),
                idx=cat(idx), val=cat(val), raw=s, chunk_m=np.array(chunk_m, np.int64),
                chunk_words=np.array(chunk_words, np.int64), block_words=bwords)


def decode_codes_bitmatrix(stream) -> np.ndarray:
    """Recover the quantisation codes q from a stream with a bit matrix:
    block payload bits (LSB-first over little-endian words) -> rows of w bits
    -> z -> closed-form inverse zigzag -> per-block cumulative sum."""
    P = parts(stream)
    h = P["h"]
    n, B = h["n"], h["block"]
    cnt = block_counts(n, B)
    words = -(-(P["widths"] * cnt) // 32)
    starts = np.concatenate([[0], np.cumsum(words)])
    bits = np.unpackbits(P["payload"], bitorder="little")
    q = np.zeros(n, np.int64)
    for b in range(h["nb"]):
        w, c = int(P["widths"][b]), int(cnt[b])
        if w == 0:
            continue
        blk = bits[32 * starts[b]: 32 * starts[b] + w * c].reshape(c, w).astype(np.uint64)
        z = (blk << np.arange(w, dtype=np.uint64)).sum(axis=1)
        d = np.where(z % 2 == 0, z // 2, -((z + 1) // 2).astype(np.int64)).astype(np.int64)
        q[b * B: b * B + c] = np.cumsum(d)
    return q


def widths_from_codes(q: np.ndarray, block: int) -> np.ndarray:
    """Block widths from codes with np.diff (reset per block) and bit lengths."""
    n = q.size
    out = []
    for s in range(0, n, block):
        blk = q[s:s + block].astype(np.int64)
        d = np.diff(np.concatenate([[0], blk]))
        z = np.where(d >= 0, 2 * d, -2 * d - 1)
        out.append(int(z.max()).bit_length() if z.size else 0)
    return np.array(out, np.int64)


# exact rounding ------------------------------------------------------------------------

_F32_MAX = Fraction(float(np.finfo(np.float32).max))
_F32_HALF_ULP_MAX = Fraction(2) ** 103  # half an ulp at the top binade


def f32_round(F: Fraction) -> np.float32:
    """Round an exact rational to the nearest float32, ties to even."""
    if F == 0:
        return np.float32(0.0)
    if abs(F) >= _F32_MAX + _F32_HALF_ULP_MAX:
        return np.float32(np.inf if F > 0 else -np.inf)
    c = np.float32(float(F))
    best, best_err = None, None
    for cand in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
        if not np.isfinite(cand):
            continue
        err = abs(F - Fraction(float(cand)))
        if best is None or err < best_err or (err == best_err and (int(cand.view(np.uint32)) & 1) == 0):
            best, best_err = cand, err
    return np.float32(best)


def exact_codes_and_flags(x: np.ndarray, inv2eb: np.float32, step: np.float32, eb: float):
    """q and the outlier flag of every element by exact rational arithmetic.

    Returns (q, flag, ambiguous) where ambiguous marks elements whose exact
    error lies within one double ulp of eb (there the method's fp64 test is the
    definition and the exact comparison may differ by rounding)."""
    q = np.zeros(x.size, np.int64)
    flag = np.zeros(x.size, bool)
    amb = np.zeros(x.size, bool)
    Finv = Fraction(float(inv2eb)) if np.isfinite(inv2eb) else None
    Feb = Fraction(eb) if np.isfinite(eb) else None
    for i, v in enumerate(x.astype(np.float32)):
        if not np.isfinite(v):
            flag[i] = True
            continue
        if Finv is None:  # inv2eb = +inf: y is +-inf (or NaN for 0)
            qi = 0
        else:
            y = f32_round(Fraction(float(v)) * Finv)
            qi = round(Fraction(float(y))) if abs(float(y)) < 2.0 ** 30 else 0
        q[i] = qi
        if not np.isfinite(step):
            xr = np.float32(np.nan) if qi == 0 else np.float32(np.inf if qi > 0 else -np.inf)
        else:
            xr = f32_round(Fraction(qi) * Fraction(float(step)))
        if not np.isfinite(xr):
            flag[i] = True
            continue
        err = abs(Fraction(float(v)) - Fraction(float(xr)))
        if Feb is None:
            flag[i] = False
            continue
        flag[i] = err > Feb
        if abs(err - Feb) <= Feb * Fraction(1, 1 << 50):
            amb[i] = True
    return q, flag, amb
