"""Seeded synthetic float32 workloads.

This module only draws inputs.  It holds none of the compressor's arithmetic
and imports neither the CUDA library nor the CPU oracle, so both sides of
every parity test consume exactly the same bytes.

All arrays are computed in float64 with NumPy's PCG64 generator
(``np.random.default_rng(seed)``) and cast to float32 once at the end.

Workloads (sizes and seeds of the five standard configurations):

* ``sine_noise``   x_i = sin(2*pi*i/4096) + 0.01*N(0,1), n = 2^20, seed 0.
* ``kfield``       zero-mean, unit-variance Gaussian random field with an
                   isotropic power spectrum |k|^-3 (amplitude |k|^-1.5),
                   synthesised by FFT from white noise: rfftn -> multiply by
                   |k|^-1.5 with k in cycles/sample from fftfreq/rfftfreq on
                   each axis, DC zeroed -> irfftn -> standardise.  Used for
                   the 256x384x384 field (seed 1), the 512^3 field (seed 2)
                   and the 1-D 2^28 series (seed 3).
* ``with_spikes``  1 % of positions (Bernoulli 0.01) replaced by U(-1e3, 1e3),
                   then Bernoulli 1e-6 positions set to NaN, +Inf or -Inf with
                   equal probability (drawn from the same generator, after
                   the field).
* ``noise_zero_ramp``  2^30 elements: [0, 2^29) U[-1, 1]; then 2^28 zeros;
                   then a ramp i/(2^28-1), i = 0..2^28-1 (seed 4).  Built for
                   any n divisible by 4 with the same proportions.

``standard(name)`` returns one of the five configurations by name:
``sine1m``, ``field256x384x384``, ``field512cube_spikes``, ``series2p28``,
``noise_zero_ramp2p30``.  ``EBLC_DATA_CACHE=<dir>`` caches generated arrays
as ``.npy`` files keyed by name and parameters.
"""
from __future__ import annotations

import hashlib
import os

import numpy as np


def _rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def _fft_workers() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def sine_noise(n: int = 1 << 20, seed: int = 0) -> np.ndarray:
    rng = _rng(seed)
    i = np.arange(n, dtype=np.float64)
    x = np.sin(2.0 * np.pi * i / 4096.0) + 0.01 * rng.standard_normal(n)
    return x.astype(np.float32)


def _kfield_f64(shape: tuple[int, ...], rng: np.random.Generator) -> np.ndarray:
    import scipy.fft as sfft

    white = rng.standard_normal(shape)
    spec = sfft.rfftn(white, workers=_fft_workers())
    del white
    k2 = None
    for ax, size in enumerate(shape):
        f = np.fft.rfftfreq(size) if ax == len(shape) - 1 else np.fft.fftfreq(size)
        view = [1] * len(shape)
        view[ax] = f.size
        term = (f * f).reshape(view)
        k2 = term if k2 is None else k2 + term
    with np.errstate(divide="ignore"):
        amp = np.where(k2 > 0.0, k2 ** (-0.75), 0.0)  # |k|^-1.5 = (k^2)^-0.75
    spec *= amp
    del amp, k2
    field = sfft.irfftn(spec, s=shape, workers=_fft_workers())
    del spec
    field -= field.mean()
    field /= field.std()
    return field


def kfield(shape: tuple[int, ...], seed: int) -> np.ndarray:
    return _kfield_f64(tuple(shape), _rng(seed)).astype(np.float32).reshape(-1)


def with_spikes(shape: tuple[int, ...], seed: int, p_spike: float = 0.01, spike_amp: float = 1e3,
                p_nonfinite: float = 1e-6) -> np.ndarray:
    rng = _rng(seed)
    x = _kfield_f64(tuple(shape), rng).reshape(-1)
    n = x.size
    spike = rng.random(n) < p_spike
    x[spike] = rng.uniform(-spike_amp, spike_amp, size=int(spike.sum()))
    bad = np.flatnonzero(rng.random(n) < p_nonfinite)
    kinds = rng.integers(0, 3, size=bad.size)
    x[bad] = np.where(kinds == 0, np.nan, np.where(kinds == 1, np.inf, -np.inf))
    return x.astype(np.float32)


def noise_zero_ramp(n: int = 1 << 30, seed: int = 4) -> np.ndarray:
    if n % 4:
        raise ValueError("n must be divisible by 4")
    rng = _rng(seed)
    half, quarter = n // 2, n // 4
    out = np.empty(n, np.float32)
    step = 1 << 24
    for s in range(0, half, step):  # chunked so the float64 temporary stays small
        e = min(half, s + step)
        out[s:e] = rng.uniform(-1.0, 1.0, size=e - s)
    out[half:half + quarter] = 0.0
    denom = float(quarter - 1) if quarter > 1 else 1.0
    for s in range(0, quarter, step):
        e = min(quarter, s + step)
        out[half + quarter + s:half + quarter + e] = np.arange(s, e, dtype=np.float64) / denom
    return out


# name -> (builder, kwargs, compressor options used with it, description)
STANDARD = {
    "sine1m": (sine_noise, dict(n=1 << 20, seed=0), dict(rel=1e-3, block=128),
               "1-D sine + 0.01 N(0,1), n=2^20"),
    "field256x384x384": (kfield, dict(shape=(256, 384, 384), seed=1), dict(rel=1e-4, block=256),
                         "3-D k^-3 Gaussian field 256x384x384"),
    "field512cube_spikes": (with_spikes, dict(shape=(512, 512, 512), seed=2), dict(rel=1e-3, block=64),
                            "3-D k^-3 field 512^3 + 1% spikes U(-1e3,1e3) + 1e-6 NaN/+-Inf"),
    "series2p28": (kfield, dict(shape=(1 << 28,), seed=3), dict(rel=1e-4, block=128),
                   "1-D k^-3 series, n=2^28 (sweep rel 1e-2..1e-6 x block 32..256)"),
    "noise_zero_ramp2p30": (noise_zero_ramp, dict(n=1 << 30, seed=4), dict(abs=1e-7, block=128),
                            "U[-1,1] | zeros | ramp, n=2^30"),
}

SWEEP_REL = (1e-2, 1e-3, 1e-4, 1e-5, 1e-6)
SWEEP_BLOCK = (32, 64, 128, 256)


def _key(name: str, kwargs: dict) -> str:
    return name + "_" + hashlib.sha1(repr(sorted(kwargs.items())).encode()).hexdigest()[:10]


def standard(name: str) -> np.ndarray:
    builder, kwargs, _, _ = STANDARD[name]
    cache = os.environ.get("EBLC_DATA_CACHE")
    if cache:
        path = os.path.join(cache, _key(name, kwargs) + ".npy")
        if os.path.exists(path):
            return np.load(path, mmap_mode=None)
        arr = builder(**kwargs)
        os.makedirs(cache, exist_ok=True)
        tmp = path[:-4] + f".tmp{os.getpid()}.npy"
        np.save(tmp, arr)
        os.replace(tmp, path)
        return arr
    return builder(**kwargs)


def options_of(name: str) -> dict:
    return dict(STANDARD[name][2])


def dims_of(name: str) -> tuple[int, ...]:
    """The workload's array shape, slowest axis first ((n,) for 1-D ones)."""
    kw = STANDARD[name][1]
    return tuple(kw["shape"]) if "shape" in kw else (int(kw["n"]),)


def sha256(x: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(x).view(np.uint8)).hexdigest()


# Small structured inputs for edge cases --------------------------------------------------

def edge_mix(n: int, seed: int) -> np.ndarray:
    """A mixture with every kind of element the method must handle: smooth
    values, exact ties of x*inv2eb when inv2eb is a power of two, zeros of both
    signs, denormals, huge values, NaN (with payloads) and +-Inf."""
    rng = _rng(seed)
    x = np.cumsum(rng.standard_normal(n) * 0.05)
    kind = rng.integers(0, 16, size=n)
    x = np.where(kind == 1, np.round(x * 8.0) / 8.0 + 1.0 / 16.0, x)  # ties at step 1/8
    x = np.where(kind == 2, 0.0, x)
    x = np.where(kind == 3, -0.0, x)
    x = np.where(kind == 4, rng.uniform(-1e6, 1e6, size=n), x)
    x = x.astype(np.float32)
    bits = x.view(np.uint32)
    den = rng.integers(1, 1 << 23, size=n, dtype=np.uint32)
    bits = np.where(kind == 5, den, bits)                                  # +denormal
    bits = np.where(kind == 6, den | np.uint32(0x80000000), bits)          # -denormal
    bits = np.where(kind == 7, np.uint32(0x7FC00000) | (den & np.uint32(0x3FFFFF)), bits)  # NaN payloads
    bits = np.where(kind == 8, np.uint32(0x7F800000), bits)                # +Inf
    bits = np.where(kind == 9, np.uint32(0xFF800000), bits)                # -Inf
    bits = np.where(kind == 10, np.uint32(0x7F7FFFFF), bits)               # FLT_MAX
    return bits.view(np.float32).copy()
