"""CPU oracle of the error-bounded lossy encoding -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product library
(``error_bounded_lossy_encode_b200``) never imports it and shares no code with
it: the oracle is plain scalar C (``eblc_oracle.c``) built with gcc, wrapped
here with ctypes and numpy for marshalling only.

What each function computes, with its source (page title, section), is stated
in ``eblc_oracle.c``.  Every function here has at least one pin in
``tests/test_oracle_pins.py`` that checks it against something other than
itself (exact rational arithmetic, library routines, closed forms, a
hand-derived worked example, brute force over tiny inputs).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# EBLC_ORACLE_SRC points the tests at another copy of the source (the
# planted-mistake tests build mutated copies in a temporary directory).
_SRC = os.environ.get("EBLC_ORACLE_SRC") or os.path.join(_HERE, "eblc_oracle.c")
_LIB = (_SRC[:-2] + ".so") if os.environ.get("EBLC_ORACLE_SRC") else os.path.join(_HERE, "liboracle.so")

ERR_ARG, ERR_CAPACITY, ERR_OUTLIER_CAP, ERR_CORRUPT, ERR_NOMEM = -1, -2, -3, -4, -5
CHUNK = 4096
HEADER_BYTES = 128


def build(force: bool = False) -> str:
    """Compile the oracle with IEEE semantics (no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_OMP_SRC = os.path.join(_HERE, "eblc_oracle_omp.c")
_OMP_LIB = os.path.join(_HERE, "liboracle_omp.so")


def build_omp(force: bool = False) -> str:
    """Compile the all-core build (eblc_oracle_omp.c: the oracle's own steps,
    run over chunks with OpenMP; the benchmark's all-core CPU baseline)."""
    newest = max(os.path.getmtime(_OMP_SRC), os.path.getmtime(_SRC))
    if force or not os.path.exists(_OMP_LIB) or os.path.getmtime(_OMP_LIB) < newest:
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-I", os.path.dirname(_SRC), "-o", _OMP_LIB, _OMP_SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _OMP_LIB


class _Header(ctypes.Structure):
    _fields_ = [(k, ctypes.c_uint32) for k in ("magic", "version", "flags", "block", "chunk", "pad")] + \
               [(k, ctypes.c_uint64) for k in ("n", "nb", "nc", "W", "m", "total")] + \
               [("eb", ctypes.c_double), ("bound", ctypes.c_double)] + \
               [(k, ctypes.c_float) for k in ("inv2eb", "step", "vmin", "vmax")] + \
               [(k, ctypes.c_uint64) for k in ("width_off", "index_off", "record_off")] + \
               [("dims", ctypes.c_uint64 * 3)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        u64, u32, i32, dbl, flt = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int32, ctypes.c_double, ctypes.c_float
        L.orc_value_range.argtypes = [P, u64, P, P]
        L.orc_value_range.restype = ctypes.c_int
        L.orc_resolve_bound.argtypes = [ctypes.c_int, dbl, flt, flt, P, P, P]
        L.orc_resolve_bound.restype = None
        L.orc_quantize.argtypes = [P, u64, flt, flt, dbl, P, P]
        L.orc_quantize.restype = None
        L.orc_zigzag.argtypes = [i32]
        L.orc_zigzag.restype = u32
        L.orc_unzigzag.argtypes = [u32]
        L.orc_unzigzag.restype = i32
        L.orc_block_width.argtypes = [P, u32]
        L.orc_block_width.restype = u32
        L.orc_block_words.argtypes = [u32, u32]
        L.orc_block_words.restype = u32
        L.orc_pack_block.argtypes = [P, u32, u32, P]
        L.orc_pack_block.restype = None
        L.orc_unpack_block.argtypes = [P, u32, u32, P]
        L.orc_unpack_block.restype = None
        L.orc_max_compressed_bytes.argtypes = [u64, u32, u64]
        L.orc_max_compressed_bytes.restype = u64
        L.orc_compress.argtypes = [P, u64, u32, ctypes.c_int, dbl, u64, P, u64]
        L.orc_compress.restype = ctypes.c_int64
        L.orc_compress_range.argtypes = [P, u64, u32, dbl, flt, flt, u64, P, u64]
        L.orc_compress_range.restype = ctypes.c_int64
        L.orc_parse_header.argtypes = [P, u64, ctypes.POINTER(_Header)]
        L.orc_parse_header.restype = ctypes.c_int
        L.orc_compress_lorenzo.argtypes = [P, ctypes.c_int, P, u32, ctypes.c_int, dbl, u64, P, u64]
        L.orc_compress_lorenzo.restype = ctypes.c_int64
        L.orc_nd_edges.argtypes = [ctypes.c_int, u32, P, P]
        L.orc_nd_edges.restype = ctypes.c_int
        L.orc_lorenzo_block.argtypes = [P, P, P]
        L.orc_lorenzo_block.restype = None
        L.orc_unlorenzo_block.argtypes = [P, P, P]
        L.orc_unlorenzo_block.restype = None
        L.orc_bitshuffle.argtypes = [P, u32, P]
        L.orc_bitshuffle.restype = None
        L.orc_unbitshuffle.argtypes = [P, u32, P]
        L.orc_unbitshuffle.restype = None
        L.orc_rze.argtypes = [P, u32, P]
        L.orc_rze.restype = u32
        L.orc_unrze.argtypes = [P, u64, u32, P]
        L.orc_unrze.restype = ctypes.c_int64
        L.orc_max_chunked_bytes.argtypes = [u64, u32, u64]
        L.orc_max_chunked_bytes.restype = u64
        L.orc_compress_chunked.argtypes = [P, u64, u32, ctypes.c_int, dbl, u64, P, u64]
        L.orc_compress_chunked.restype = ctypes.c_int64
        L.orc_compress_chunked_coder.argtypes = [P, u64, u32, ctypes.c_int, ctypes.c_int, dbl, u64, P, u64]
        L.orc_compress_chunked_coder.restype = ctypes.c_int64
        L.orc_rre.argtypes = [P, u32, P]
        L.orc_rre.restype = u32
        L.orc_unrre.argtypes = [P, u64, u32, P]
        L.orc_unrre.restype = ctypes.c_int64
        L.orc_decompress.argtypes = [P, u64, P, u64]
        L.orc_decompress.restype = ctypes.c_int
        L.orc_block_codes.argtypes = [P, u64, u32, flt, P, P]
        L.orc_block_codes.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


def value_range(x):
    x = _f32(x)
    lo, hi = np.zeros(1, np.float32), np.zeros(1, np.float32)
    any_finite = lib().orc_value_range(_ptr(x), x.size, _ptr(lo), _ptr(hi))
    return float(lo[0]), float(hi[0]), bool(any_finite)


@dataclass
class Bound:
    eb: float
    inv2eb: np.float32
    step: np.float32


def resolve_bound(abs_mode: bool, bound: float, vmin: float = 0.0, vmax: float = 0.0) -> Bound:
    eb, inv, st = np.zeros(1, np.float64), np.zeros(1, np.float32), np.zeros(1, np.float32)
    lib().orc_resolve_bound(int(abs_mode), float(bound), float(np.float32(vmin)), float(np.float32(vmax)),
                            _ptr(eb), _ptr(inv), _ptr(st))
    return Bound(float(eb[0]), inv[0], st[0])


def quantize(x, bnd: Bound):
    x = _f32(x)
    q = np.zeros(x.size, np.int32)
    flag = np.zeros(x.size, np.uint8)
    lib().orc_quantize(_ptr(x), x.size, float(bnd.inv2eb), float(bnd.step), float(bnd.eb), _ptr(q), _ptr(flag))
    return q, flag.astype(bool)


def zigzag(d: int) -> int:
    return int(lib().orc_zigzag(int(d)))


def unzigzag(z: int) -> int:
    return int(lib().orc_unzigzag(int(z)))


def block_width(z) -> int:
    z = np.ascontiguousarray(z, dtype=np.uint32)
    return int(lib().orc_block_width(_ptr(z), z.size))


def block_words(w: int, cnt: int) -> int:
    return int(lib().orc_block_words(w, cnt))


def pack_block(z, w: int) -> np.ndarray:
    z = np.ascontiguousarray(z, dtype=np.uint32)
    out = np.zeros(max(1, block_words(w, z.size)), np.uint32)
    lib().orc_pack_block(_ptr(z), z.size, w, _ptr(out))
    return out[: block_words(w, z.size)]


def unpack_block(words, cnt: int, w: int) -> np.ndarray:
    words = np.ascontiguousarray(words, dtype=np.uint32)
    if words.size == 0:
        words = np.zeros(1, np.uint32)
    z = np.zeros(max(1, cnt), np.uint32)
    lib().orc_unpack_block(_ptr(words), cnt, w, _ptr(z))
    return z[:cnt]


def max_compressed_bytes(n: int, block: int, outlier_cap: int | None = None) -> int:
    return int(lib().orc_max_compressed_bytes(n, block, n if outlier_cap is None else outlier_cap))


def compress(x, block: int = 128, *, rel: float | None = None, abs: float | None = None,
             outlier_cap: int | None = None, out_cap: int | None = None):
    """Return the stream as a uint8 array, or raise OracleError(code)."""
    x = _f32(x).reshape(-1)
    if (rel is None) == (abs is None):
        raise ValueError("exactly one of rel / abs")
    abs_mode = abs is not None
    bound = float(abs if abs_mode else rel)
    cap = x.size if outlier_cap is None else int(outlier_cap)
    need = max_compressed_bytes(x.size, block, cap) if out_cap is None else int(out_cap)
    out = np.zeros(max(need, 1), np.uint8)
    rc = lib().orc_compress(_ptr(x), x.size, block, int(abs_mode), bound, cap, _ptr(out), need)
    if rc < 0:
        raise OracleError(int(rc))
    return out[:rc].copy()


def compress_range(x, block: int, rel: float, vmin: float, vmax: float, *, outlier_cap: int | None = None):
    """compress() of one part of a larger array under the relative bound of
    the whole: eb = rel * (vmax - vmin) with the given range (see
    orc_compress_range)."""
    x = _f32(x).reshape(-1)
    cap = x.size if outlier_cap is None else int(outlier_cap)
    need = max_compressed_bytes(x.size, block, cap)
    out = np.zeros(max(need, 1), np.uint8)
    rc = lib().orc_compress_range(_ptr(x), x.size, block, float(rel), float(np.float32(vmin)),
                                  float(np.float32(vmax)), cap, _ptr(out), need)
    if rc < 0:
        raise OracleError(int(rc))
    return out[:rc].copy()


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle error {code}")
        self.code = code


def parse_header(stream) -> dict:
    s = np.ascontiguousarray(stream, dtype=np.uint8)
    h = _Header()
    rc = lib().orc_parse_header(_ptr(s) if s.size else 0, s.size, ctypes.byref(h))
    if rc != 0:
        raise OracleError(rc)
    d = {k: getattr(h, k) for k, _ in _Header._fields_}
    d["dims"] = tuple(int(v) for v in h.dims)
    return d


def nd_edges(rank: int, block: int):
    """(block edges, brick edges), each (z, y, x), of the multi-dimensional
    Lorenzo layout, or None when rank / block is not supported."""
    be, ce = np.zeros(3, np.uint32), np.zeros(3, np.uint32)
    if not lib().orc_nd_edges(rank, block, _ptr(be), _ptr(ce)):
        return None
    return tuple(int(v) for v in be), tuple(int(v) for v in ce)


def lorenzo_block(q, be) -> np.ndarray:
    """Lorenzo residuals of one block (codes in C order, edges be), int32 modulo 2^32."""
    q = np.ascontiguousarray(q, dtype=np.int32).reshape(-1)
    e = np.ascontiguousarray(be, dtype=np.uint32)
    d = np.zeros(q.size, np.int32)
    lib().orc_lorenzo_block(_ptr(q), _ptr(e), _ptr(d))
    return d


def unlorenzo_block(d, be) -> np.ndarray:
    d = np.ascontiguousarray(d, dtype=np.int32).reshape(-1)
    e = np.ascontiguousarray(be, dtype=np.uint32)
    q = np.zeros(d.size, np.int32)
    lib().orc_unlorenzo_block(_ptr(d), _ptr(e), _ptr(q))
    return q


def compress_lorenzo(x, block: int = 64, *, rel: float | None = None, abs: float | None = None,
                     outlier_cap: int | None = None):
    """compress() with the multi-dimensional Lorenzo predictor over x's own
    dims (x of shape (Z, Y, X) or (Y, X); see orc_compress_lorenzo)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim not in (2, 3):
        raise ValueError("x must be 2-D or 3-D")
    if (rel is None) == (abs is None):
        raise ValueError("exactly one of rel / abs")
    dims = np.array((1,) + x.shape if x.ndim == 2 else x.shape, np.uint64)
    abs_mode = abs is not None
    cap = x.size if outlier_cap is None else int(outlier_cap)
    need = max_compressed_bytes(x.size, block, cap)
    out = np.zeros(max(need, 1), np.uint8)
    rc = lib().orc_compress_lorenzo(_ptr(x), x.ndim, _ptr(dims), block, int(abs_mode),
                                    float(abs if abs_mode else rel), cap, _ptr(out), need)
    if rc < 0:
        raise OracleError(int(rc))
    return out[:rc].copy()


def decompress(stream, n: int) -> np.ndarray:
    s = np.ascontiguousarray(stream, dtype=np.uint8)
    out = np.zeros(max(n, 1), np.float32)
    rc = lib().orc_decompress(_ptr(s), s.size, _ptr(out), n)
    if rc != 0:
        raise OracleError(rc)
    return out[:n]


def block_codes(x, block: int, inv2eb) -> tuple[np.ndarray, np.ndarray]:
    x = _f32(x).reshape(-1)
    nb = (x.size + block - 1) // block
    z = np.zeros(max(1, x.size), np.uint32)
    w = np.zeros(max(1, nb), np.uint8)
    lib().orc_block_codes(_ptr(x), x.size, block, float(np.float32(inv2eb)), _ptr(z), _ptr(w))
    return z[: x.size], w[:nb]


_omp = None


def _omp_lib():
    global _omp
    if _omp is None:
        L = ctypes.CDLL(build_omp())
        P, u64, u32, dbl = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_double
        L.orc_compress_omp.argtypes = [P, u64, u32, ctypes.c_int, dbl, u64, P, u64]
        L.orc_compress_omp.restype = ctypes.c_int64
        L.orc_decompress_omp.argtypes = [P, u64, P, u64]
        L.orc_decompress_omp.restype = ctypes.c_int
        L.orc_omp_threads.argtypes = []
        L.orc_omp_threads.restype = ctypes.c_int
        _omp = L
    return _omp


def omp_threads() -> int:
    """Threads the all-core build uses (OpenMP's default: the cores this
    process may run on, or OMP_NUM_THREADS)."""
    return int(_omp_lib().orc_omp_threads())


def compress_omp(x, block: int = 128, *, rel: float | None = None, abs: float | None = None):
    """compress() on all host cores; the stream is byte-identical."""
    x = _f32(x).reshape(-1)
    if (rel is None) == (abs is None):
        raise ValueError("exactly one of rel / abs")
    abs_mode = abs is not None
    need = max_compressed_bytes(x.size, block)
    out = np.zeros(max(need, 1), np.uint8)
    rc = _omp_lib().orc_compress_omp(_ptr(x), x.size, block, int(abs_mode), float(abs if abs_mode else rel),
                                     x.size, _ptr(out), need)
    if rc < 0:
        raise OracleError(int(rc))
    return out[:rc].copy()


def decompress_omp(stream, n: int) -> np.ndarray:
    """decompress() on all host cores."""
    s = np.ascontiguousarray(stream, dtype=np.uint8)
    out = np.zeros(max(n, 1), np.float32)
    rc = _omp_lib().orc_decompress_omp(_ptr(s), s.size, _ptr(out), n)
    if rc != 0:
        raise OracleError(rc)
    return out[:n]


def bitshuffle(words) -> np.ndarray:
    """Bit-plane transpose of a multiple of 32 codes (see orc_bitshuffle)."""
    w = np.ascontiguousarray(words, dtype=np.uint32)
    out = np.zeros(max(w.size, 1), np.uint32)
    lib().orc_bitshuffle(_ptr(w), w.size, _ptr(out))
    return out[: w.size]


def unbitshuffle(words) -> np.ndarray:
    w = np.ascontiguousarray(words, dtype=np.uint32)
    out = np.zeros(max(w.size, 1), np.uint32)
    lib().orc_unbitshuffle(_ptr(w), w.size, _ptr(out))
    return out[: w.size]


def rze(words) -> np.ndarray:
    """Zero elimination: bitmap words, then the nonzero words."""
    w = np.ascontiguousarray(words, dtype=np.uint32)
    out = np.zeros(max(w.size + w.size // 32, 1), np.uint32)
    k = lib().orc_rze(_ptr(w), w.size, _ptr(out))
    return out[:k]


def unrze(words, mp: int):
    """Inverse of rze for mp words; returns (words, consumed) or raises."""
    w = np.ascontiguousarray(words, dtype=np.uint32)
    src = w if w.size else np.zeros(1, np.uint32)
    out = np.zeros(max(mp, 1), np.uint32)
    k = lib().orc_unrze(_ptr(src), w.size, mp, _ptr(out))
    if k < 0:
        raise OracleError(int(k))
    return out[:mp], int(k)


def rre(words) -> np.ndarray:
    """Repetition elimination: bitmap words (bit j: word j differs from word
    j - 1, word -1 being 0), then the words that differ."""
    w = np.ascontiguousarray(words, dtype=np.uint32)
    out = np.zeros(max(w.size + w.size // 32, 1), np.uint32)
    k = lib().orc_rre(_ptr(w), w.size, _ptr(out))
    return out[:k]


def unrre(words, mp: int):
    """Inverse of rre for mp words; returns (words, consumed) or raises."""
    w = np.ascontiguousarray(words, dtype=np.uint32)
    src = w if w.size else np.zeros(1, np.uint32)
    out = np.zeros(max(mp, 1), np.uint32)
    k = lib().orc_unrre(_ptr(src), w.size, mp, _ptr(out))
    if k < 0:
        raise OracleError(int(k))
    return out[:mp], int(k)


def max_chunked_bytes(n: int, chunk_bytes: int, outlier_cap: int | None = None) -> int:
    return int(lib().orc_max_chunked_bytes(n, chunk_bytes, n if outlier_cap is None else outlier_cap))


def compress_chunked(x, chunk_bytes: int = 16384, *, rel: float | None = None, abs: float | None = None,
                     outlier_cap: int | None = None, coder: str = "rze"):
    """The chunk-cooperative codec (Quant -> Diff -> Bitshuffle -> RZE, or
    RRE with coder="rre"; see orc_compress_chunked_coder): the stream as a
    uint8 array."""
    if coder not in ("rze", "rre"):
        raise ValueError("coder is rze or rre")
    x = _f32(x).reshape(-1)
    if (rel is None) == (abs is None):
        raise ValueError("exactly one of rel / abs")
    abs_mode = abs is not None
    cap = x.size if outlier_cap is None else int(outlier_cap)
    need = max(max_chunked_bytes(x.size, chunk_bytes, cap), 1)
    out = np.zeros(need, np.uint8)
    rc = lib().orc_compress_chunked_coder(_ptr(x), x.size, chunk_bytes, int(coder == "rre"), int(abs_mode),
                                          float(abs if abs_mode else rel), cap, _ptr(out), need)
    if rc < 0:
        raise OracleError(int(rc))
    return out[:rc].copy()
