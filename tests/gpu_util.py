"""Torch-based helpers for GPU tests: device buffers and streams around the
C-ABI binding.  Nothing here computes any part of the method."""
from __future__ import annotations

import numpy as np
import torch

import error_bounded_lossy_encode_b200 as E


def opts(block: int, rel=None, abs=None, extra: str = "") -> str:
    s = f"{'abs' if abs is not None else 'rel'}={abs if abs is not None else rel!r},block={block}"
    return s + ("," + extra if extra else "")


class GpuCodec:
    def __init__(self, n: int, block: int, rel=None, abs=None, extra: str = "", dims=None, strides=None):
        st, self.plan = E.eblc_plan_create(dims if dims is not None else [n], strides, opts(block, rel, abs, extra))
        assert st == E.EBLC_OK, E.STATUS_NAMES[st]
        st, self.lim = E.eblc_plan_get_limits(self.plan)
        assert st == E.EBLC_OK
        self.n = n

    def compress(self, x: torch.Tensor, cap: int | None = None, stream: torch.cuda.Stream | None = None):
        cap = self.lim["max_compressed_bytes"] if cap is None else cap
        out = torch.empty(max(cap, 16), dtype=torch.uint8, device="cuda")
        sc = E.eblc_sidecar_t()
        s = stream or torch.cuda.current_stream()
        st, nbytes = E.eblc_compress(self.plan, E.cuda_exec(s.cuda_stream), x.data_ptr(), out.data_ptr(), cap, sc)
        return st, out, nbytes, sc

    def compress_np(self, x_np: np.ndarray, **kw):
        x = torch.from_numpy(np.ascontiguousarray(x_np, dtype=np.float32)).cuda()
        st, out, nbytes, sc = self.compress(x, **kw)
        torch.cuda.synchronize()
        return st, out[:nbytes].cpu().numpy(), sc

    def decompress(self, s_dev: torch.Tensor, nbytes: int, sc=None, stream: torch.cuda.Stream | None = None):
        out = torch.empty(max(self.n, 4), dtype=torch.float32, device="cuda")
        s = stream or torch.cuda.current_stream()
        st = E.eblc_decompress(self.plan, E.cuda_exec(s.cuda_stream), s_dev.data_ptr(), nbytes, sc, out.data_ptr())
        return st, out[: self.n]

    def decompress_np(self, stream_np: np.ndarray, sc=None):
        buf = torch.zeros(max(16, stream_np.size), dtype=torch.uint8)
        buf[: stream_np.size] = torch.from_numpy(np.ascontiguousarray(stream_np))
        d = buf.cuda()
        st, out = self.decompress(d, stream_np.size, sc)
        chk = E.eblc_check(self.plan, E.cuda_exec(torch.cuda.current_stream().cuda_stream))
        return st, chk, out.cpu().numpy()

    def check(self) -> int:
        return E.eblc_check(self.plan, E.cuda_exec(torch.cuda.current_stream().cuda_stream))

    def close(self):
        E.eblc_plan_destroy(self.plan)
        self.plan = None

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()


def bits_equal(a: np.ndarray, b: np.ndarray) -> bool:
    return a.shape == b.shape and np.array_equal(a.view(np.uint32), b.view(np.uint32))


def first_diff(a: np.ndarray, b: np.ndarray):
    n = min(a.size, b.size)
    d = np.flatnonzero(a[:n] != b[:n])
    return (int(d[0]) if d.size else None), a.size, b.size
