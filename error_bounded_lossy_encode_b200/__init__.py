"""B200-native error-bounded lossy compressor for float32 arrays.

Thin ctypes binding of ``libeblc.so`` (C ABI declared in ``include/eblc.h``):
argument marshalling only.  Every step of compression and decompression runs
in the library's CUDA kernels; there is no CPU code path here, and every
entry point raises ``RuntimeError`` when the library has not been built.

Functions keep the C names::

    st, plan = eblc_plan_create(dims, strides=None, options="rel=1e-3,block=64")
    st, lim  = eblc_plan_get_limits(plan)
    st, nbytes = eblc_compress(plan, cuda_exec(stream), d_in, d_out, capacity, sidecar)
    st = eblc_compress_async(plan, cuda_exec(stream), d_in, d_out, capacity, d_result)   # no host sync
    st = eblc_value_range(plan, cuda_exec(stream), d_in, d_range)                       # device float[2]
    st, nbytes = eblc_compress_range(plan, cuda_exec(stream), d_in, d_range, d_out, capacity, sidecar)
    st = eblc_decompress(plan, cuda_exec(stream), d_stream, nbytes, sidecar, d_out)
    st = eblc_check(plan, cuda_exec(stream))
    eblc_plan_destroy(plan)

Pointers are plain integers (``tensor.data_ptr()``), streams are integer
``cudaStream_t`` handles (``torch.cuda.current_stream().cuda_stream``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libeblc.so")

EBLC_OK, EBLC_UNSUPPORTED, EBLC_INVALID_ARG, EBLC_CAPACITY, EBLC_CORRUPT, EBLC_CUDA_ERROR, EBLC_TIMEOUT, \
    EBLC_NOMEM = range(8)
STATUS_NAMES = {0: "OK", 1: "UNSUPPORTED", 2: "INVALID_ARG", 3: "CAPACITY", 4: "CORRUPT", 5: "CUDA_ERROR",
                6: "TIMEOUT", 7: "NOMEM"}
EBLC_EXECUTION_HOST, EBLC_EXECUTION_CUDA, EBLC_EXECUTION_HIP = 0, 1, 2


class eblc_execution_t(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("num_threads", ctypes.c_int32), ("stream", ctypes.c_void_p)]


class eblc_limits_t(ctypes.Structure):
    _fields_ = [("n", ctypes.c_uint64), ("block", ctypes.c_uint32), ("chunk", ctypes.c_uint32),
                ("max_compressed_bytes", ctypes.c_uint64), ("payload_alignment", ctypes.c_uint64),
                ("sidecar_bytes", ctypes.c_uint64), ("sidecar_alignment", ctypes.c_uint64),
                ("outlier_capacity", ctypes.c_uint64), ("bound", ctypes.c_double), ("abs_mode", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class eblc_sidecar_t(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32), ("version", ctypes.c_uint16), ("flags", ctypes.c_uint16),
                ("block", ctypes.c_uint32), ("chunk", ctypes.c_uint32), ("n", ctypes.c_uint64),
                ("total_bytes", ctypes.c_uint64), ("payload_words", ctypes.c_uint64),
                ("n_outliers", ctypes.c_uint64), ("eb", ctypes.c_double), ("step", ctypes.c_float),
                ("inv2eb", ctypes.c_float)]


class eblc_async_result_t(ctypes.Structure):
    _fields_ = [("compressed_bytes", ctypes.c_uint64), ("payload_words", ctypes.c_uint64),
                ("n_outliers", ctypes.c_uint64), ("status", ctypes.c_uint32), ("reserved", ctypes.c_uint32)]


class eblc_kernel_time_t(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 24), ("ms", ctypes.c_float), ("launches", ctypes.c_uint32)]


assert ctypes.sizeof(eblc_sidecar_t) == 64
assert ctypes.sizeof(eblc_async_result_t) == 32


def _fields(s: ctypes.Structure) -> dict:
    return {k: getattr(s, k) for k, _ in s._fields_}


_lib = None


def lib() -> ctypes.CDLL:
    """Load libeblc.so; fail loudly if it is missing (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libeblc.so is not built ({LIB_PATH}); run `python -m error_bounded_lossy_encode_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, u64, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int
    L.eblc_abi_version.argtypes = []
    L.eblc_abi_version.restype = ctypes.c_uint32
    L.eblc_status_string.argtypes = [i32]
    L.eblc_status_string.restype = ctypes.c_char_p
    L.eblc_plan_create.argtypes = [ctypes.POINTER(P), i32, ctypes.POINTER(ctypes.c_int64),
                                   ctypes.POINTER(ctypes.c_int64), ctypes.c_char_p]
    L.eblc_plan_create.restype = i32
    L.eblc_plan_get_limits.argtypes = [P, ctypes.POINTER(eblc_limits_t)]
    L.eblc_plan_get_limits.restype = i32
    L.eblc_compress.argtypes = [P, ctypes.POINTER(eblc_execution_t), P, P, ctypes.c_size_t,
                                ctypes.POINTER(ctypes.c_size_t), P]
    L.eblc_compress.restype = i32
    L.eblc_compress_async.argtypes = [P, ctypes.POINTER(eblc_execution_t), P, P, ctypes.c_size_t, P]
    L.eblc_compress_async.restype = i32
    L.eblc_value_range.argtypes = [P, ctypes.POINTER(eblc_execution_t), P, P]
    L.eblc_value_range.restype = i32
    L.eblc_compress_range.argtypes = [P, ctypes.POINTER(eblc_execution_t), P, P, P, ctypes.c_size_t,
                                      ctypes.POINTER(ctypes.c_size_t), P]
    L.eblc_compress_range.restype = i32
    L.eblc_decompress.argtypes = [P, ctypes.POINTER(eblc_execution_t), P, ctypes.c_size_t, P, P]
    L.eblc_decompress.restype = i32
    L.eblc_check.argtypes = [P, ctypes.POINTER(eblc_execution_t)]
    L.eblc_check.restype = i32
    L.eblc_plan_kernel_times.argtypes = [P, ctypes.POINTER(eblc_kernel_time_t), i32, ctypes.POINTER(i32)]
    L.eblc_plan_kernel_times.restype = i32
    L.eblc_plan_destroy.argtypes = [P]
    L.eblc_plan_destroy.restype = None
    L.eblc_compress_noalloc.argtypes = [P, u64, ctypes.c_uint32, i32, ctypes.c_double, P, ctypes.c_size_t, P,
                                        ctypes.POINTER(ctypes.c_size_t), P]
    L.eblc_compress_noalloc.restype = i32
    _lib = L
    return L


def cuda_exec(stream: int = 0) -> eblc_execution_t:
    return eblc_execution_t(EBLC_EXECUTION_CUDA, 0, ctypes.c_void_p(stream or None))


def host_exec() -> eblc_execution_t:
    return eblc_execution_t(EBLC_EXECUTION_HOST, 0, None)


def eblc_abi_version() -> int:
    return int(lib().eblc_abi_version())


def eblc_status_string(status: int) -> str:
    return lib().eblc_status_string(int(status)).decode()


def eblc_plan_create(dims, strides=None, options: str | None = None):
    dims = [int(d) for d in dims]
    d = (ctypes.c_int64 * max(1, len(dims)))(*dims)
    s = None if strides is None else (ctypes.c_int64 * max(1, len(dims)))(*[int(x) for x in strides])
    plan = ctypes.c_void_p()
    st = lib().eblc_plan_create(ctypes.byref(plan), len(dims), d, s,
                                None if options is None else options.encode())
    return st, (plan if st == EBLC_OK else None)


def eblc_plan_get_limits(plan):
    lim = eblc_limits_t()
    st = lib().eblc_plan_get_limits(plan, ctypes.byref(lim))
    return st, _fields(lim)


def eblc_compress(plan, exec_: eblc_execution_t, d_in: int, d_out: int, out_capacity: int, sidecar=None):
    """Returns (status, compressed_bytes).  `sidecar`: an eblc_sidecar_t or None."""
    nbytes = ctypes.c_size_t(0)
    st = lib().eblc_compress(plan, ctypes.byref(exec_), ctypes.c_void_p(d_in or None),
                             ctypes.c_void_p(d_out or None), out_capacity, ctypes.byref(nbytes),
                             None if sidecar is None else ctypes.byref(sidecar))
    return st, int(nbytes.value)


def eblc_compress_async(plan, exec_: eblc_execution_t, d_in: int, d_out: int, out_capacity: int,
                        d_result: int) -> int:
    """Queue a compress on exec_'s stream; the device writes an
    eblc_async_result_t (32 bytes) at d_result.  Returns the queueing status."""
    return lib().eblc_compress_async(plan, ctypes.byref(exec_), ctypes.c_void_p(d_in or None),
                                     ctypes.c_void_p(d_out or None), out_capacity, ctypes.c_void_p(d_result or None))


def eblc_value_range(plan, exec_: eblc_execution_t, d_in: int, d_range: int) -> int:
    """Queue the value range of d_in into the device float[2] at d_range."""
    return lib().eblc_value_range(plan, ctypes.byref(exec_), ctypes.c_void_p(d_in or None),
                                  ctypes.c_void_p(d_range or None))


def eblc_compress_range(plan, exec_: eblc_execution_t, d_in: int, d_range: int, d_out: int, out_capacity: int,
                        sidecar: eblc_sidecar_t | None = None):
    """Compress under the value range in the device float[2] at d_range.
    Returns (status, compressed_bytes)."""
    nbytes = ctypes.c_size_t(0)
    st = lib().eblc_compress_range(plan, ctypes.byref(exec_), ctypes.c_void_p(d_in or None),
                                   ctypes.c_void_p(d_range or None), ctypes.c_void_p(d_out or None), out_capacity,
                                   ctypes.byref(nbytes), None if sidecar is None else ctypes.byref(sidecar))
    return st, int(nbytes.value)


def async_result(raw) -> dict:
    """Decode the 32 bytes of an eblc_async_result_t (e.g. a uint8 tensor copied to the host)."""
    r = eblc_async_result_t.from_buffer_copy(bytes(raw))
    return _fields(r)


def eblc_decompress(plan, exec_: eblc_execution_t, d_in: int, compressed_bytes: int, sidecar, d_out: int) -> int:
    return lib().eblc_decompress(plan, ctypes.byref(exec_), ctypes.c_void_p(d_in or None), compressed_bytes,
                                 None if sidecar is None else ctypes.byref(sidecar), ctypes.c_void_p(d_out or None))


def eblc_check(plan, exec_: eblc_execution_t | None = None) -> int:
    return lib().eblc_check(plan, None if exec_ is None else ctypes.byref(exec_))


def eblc_plan_kernel_times(plan, cap: int = 8):
    arr = (eblc_kernel_time_t * cap)()
    cnt = ctypes.c_int(0)
    st = lib().eblc_plan_kernel_times(plan, arr, cap, ctypes.byref(cnt))
    return st, [(arr[i].name.decode(), float(arr[i].ms), int(arr[i].launches)) for i in range(cnt.value)]


def eblc_plan_destroy(plan) -> None:
    if plan is not None:
        lib().eblc_plan_destroy(plan)


EBLC_NOALLOC_MAX_N = 1 << 26


def eblc_compress_noalloc(d_in: int, n: int, block: int, abs_mode: bool, bound: float, d_out: int,
                          out_capacity: int, stream: int = 0, sidecar=None):
    """Plan-free compress that allocates no device memory (see include/eblc.h).
    Returns (status, compressed_bytes)."""
    nbytes = ctypes.c_size_t(0)
    st = lib().eblc_compress_noalloc(ctypes.c_void_p(d_in or None), n, block, int(bool(abs_mode)), float(bound),
                                     ctypes.c_void_p(d_out or None), out_capacity, ctypes.c_void_p(stream or None),
                                     ctypes.byref(nbytes), None if sidecar is None else ctypes.byref(sidecar))
    return st, int(nbytes.value)


def sidecar_dict(sc: eblc_sidecar_t) -> dict:
    return _fields(sc)
