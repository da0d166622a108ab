"""GPU parity with the CPU oracle through the C ABI: streams byte-identical
(outliers are stored in index order on both sides), reconstructions
bit-identical, and cross-decoding (GPU decodes the oracle's stream and vice
versa).  Sizes span several 4096-element tiles and ragged tails."""
import numpy as np
import pytest

from error_bounded_lossy_encode_b200 import workloads as WL
from tests import streamcheck as SC

pytestmark = pytest.mark.gpu

BLOCKS = (32, 64, 128, 256)


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _run_parity(orc, x, block, rel=None, abs=None):
    from tests.gpu_util import GpuCodec, bits_equal, first_diff

    want = orc.compress(x, block, rel=rel, abs=abs)
    with GpuCodec(x.size, block, rel=rel, abs=abs) as g:
        st, got, sc = g.compress_np(x)
        assert st == 0, st
        assert got.size == want.size and np.array_equal(got, want), first_diff(got, want)
        assert sc.total_bytes == want.size and sc.n_outliers == SC.header(want)["m"]
        y_ref = orc.decompress(want, x.size)
        st, chk, y = g.decompress_np(got, sc)
        assert st == 0 and chk == 0, (st, chk)
        assert bits_equal(y, y_ref)
        st, chk, y2 = g.decompress_np(want, None)  # no sidecar: header read back from the device
        assert st == 0 and chk == 0 and bits_equal(y2, y_ref)
    return want


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("n", [1, 31, 32, 33, 255, 4095, 4096, 4097, 3 * 4096 + 7, 65537])
def test_parity_sizes_edge_mix(torch_cuda, orc, block, n):
    _run_parity(orc, WL.edge_mix(n, n * 7 + block), block, rel=1e-3)


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("mode,bound", [("rel", 1e-2), ("rel", 1e-5), ("abs", 1e-7), ("abs", 0.05), ("abs", 0.0)])
def test_parity_modes(torch_cuda, orc, block, mode, bound):
    x = np.concatenate([WL.sine_noise(50000, 0), WL.edge_mix(9000, 3), WL.noise_zero_ramp(40000, 4)])
    _run_parity(orc, x, block, **{mode: bound})


@pytest.mark.parametrize("block", BLOCKS)
def test_parity_fields(torch_cuda, orc, block):
    _run_parity(orc, WL.kfield((40, 48, 64), 1), block, rel=1e-4)
    _run_parity(orc, WL.with_spikes((32, 32, 40), 2, p_nonfinite=1e-3), block, rel=1e-3)


def test_parity_empty(torch_cuda, orc):
    from tests.gpu_util import GpuCodec

    want = orc.compress(np.zeros(0, np.float32), 64, rel=1e-3)
    with GpuCodec(0, 64, rel=1e-3) as g:
        st, got, sc = g.compress_np(np.zeros(4, np.float32)[:0])
        assert st == 0 and np.array_equal(got, want)
        st, chk, y = g.decompress_np(got, sc)
        assert st == 0 and chk == 0 and y.size == 0


@pytest.mark.parametrize("case", ["zeros", "constant", "all_nan", "huge", "denormal", "ties", "neg_zero", "inf_mix"])
def test_parity_special_inputs(torch_cuda, orc, case):
    n = 3 * 4096 + 100
    rng = np.random.default_rng(5)
    if case == "zeros":
        x = np.zeros(n, np.float32)
    elif case == "constant":
        x = np.full(n, -7.25, np.float32)
    elif case == "all_nan":
        x = np.full(n, np.nan, np.float32)
        x.view(np.uint32)[::5] = 0x7FA00001
    elif case == "huge":
        x = (rng.standard_normal(n) * 1e30).astype(np.float32)
    elif case == "denormal":
        x = (rng.integers(1, 1 << 23, n).astype(np.uint32)).view(np.float32)
    elif case == "ties":
        x = ((rng.integers(-1000, 1000, n) + 0.5) / 8).astype(np.float32)
    elif case == "neg_zero":
        x = np.where(rng.random(n) < 0.5, -0.0, 1e-9).astype(np.float32)
    else:
        x = rng.standard_normal(n).astype(np.float32)
        x[rng.random(n) < 0.01] = np.inf
        x[rng.random(n) < 0.01] = -np.inf
    for block in (32, 256):
        for kw in (dict(rel=1e-3), dict(abs=1.0 / 16), dict(abs=1e-30), dict(rel=0.5)):
            _run_parity(orc, x, block, **kw)


def test_repeated_calls_identical(torch_cuda, orc):
    """Two look-back status sets alternate between calls; every call must
    produce the same stream."""
    from tests.gpu_util import GpuCodec

    x = WL.with_spikes((24, 64, 64), 2, p_nonfinite=1e-3)
    want = orc.compress(x, 64, rel=1e-3)
    with GpuCodec(x.size, 64, rel=1e-3) as g:
        for _ in range(5):
            st, got, _ = g.compress_np(x)
            assert st == 0 and np.array_equal(got, want)


def test_nondefault_stream_and_dims(torch_cuda, orc):
    import torch
    from tests.gpu_util import GpuCodec

    x = WL.kfield((16, 24, 32), 1)
    want = orc.compress(x, 128, rel=1e-4)
    with GpuCodec(x.size, 128, rel=1e-4, dims=[16, 24, 32], strides=[24 * 32, 32, 1]) as g:
        s = torch.cuda.Stream()
        xd = torch.from_numpy(x).cuda()
        torch.cuda.synchronize()
        st, out, nbytes, sc = g.compress(xd, stream=s)
        assert st == 0
        torch.cuda.synchronize()
        assert np.array_equal(out[:nbytes].cpu().numpy(), want)
        st, y = g.decompress(out, nbytes, sc, stream=s)
        s.synchronize()
        assert st == 0 and np.array_equal(y.cpu().numpy().view(np.uint32), orc.decompress(want, x.size).view(np.uint32))


def test_host_execution(torch_cuda, orc):
    """HOST kind: host pointers, the same GPU kernels behind plan staging."""
    import ctypes

    import error_bounded_lossy_encode_b200 as E

    x = WL.edge_mix(20000, 11)
    want = orc.compress(x, 64, rel=1e-3)
    st, plan = E.eblc_plan_create([x.size], None, "rel=1e-3,block=64")
    assert st == 0
    try:
        _, lim = E.eblc_plan_get_limits(plan)
        out = np.zeros(lim["max_compressed_bytes"] + 16, np.uint8)
        base = out.ctypes.data
        off = (-base) % 16
        sc = E.eblc_sidecar_t()
        st, nbytes = E.eblc_compress(plan, E.host_exec(), x.ctypes.data, base + off, lim["max_compressed_bytes"], sc)
        assert st == 0 and nbytes == want.size
        got = out[off:off + nbytes]
        assert np.array_equal(got, want)
        y = np.zeros(x.size + 4, np.float32)
        yo = (-y.ctypes.data) % 16 // 4
        st = E.eblc_decompress(plan, E.host_exec(), base + off, nbytes, sc, y.ctypes.data + 4 * yo)
        assert st == 0
        assert np.array_equal(y[yo:yo + x.size].view(np.uint32), orc.decompress(want, x.size).view(np.uint32))
        del ctypes
    finally:
        E.eblc_plan_destroy(plan)


def test_cross_decode_oracle_stream(torch_cuda, orc):
    from tests.gpu_util import GpuCodec, bits_equal

    for block in BLOCKS:
        x = np.concatenate([WL.edge_mix(30000, block), WL.sine_noise(12345, 1)])
        s = orc.compress(x, block, abs=1e-3)
        with GpuCodec(x.size, block, abs=1e-3) as g:
            st, chk, y = g.decompress_np(s, None)
            assert st == 0 and chk == 0
            assert bits_equal(y, orc.decompress(s, x.size))


@pytest.mark.parametrize("block", BLOCKS)
def test_parity_many_tiles_per_cta(torch_cuda, orc, block):
    """Enough 4096-element chunks (about 5 per CTA) that every CTA cycles its
    shared-memory rings and barrier phases several times, in both kernels."""
    rng = np.random.default_rng(block)
    n = 1500 * 4096 + 123
    x = np.cumsum(rng.standard_normal(n) * 0.02).astype(np.float32)
    x[rng.random(n) < 1e-4] = np.nan
    x[rng.random(n) < 1e-3] *= 1e3
    _run_parity(orc, x, block, rel=1e-3)
    _run_parity(orc, x, block, abs=1e-4)


@pytest.mark.parametrize("block", (32, 256))
def test_parity_full_width_slices(torch_cuda, orc, block):
    """Every block at width 32 (codes alternate between +-(2^30 - 64), abs
    bound 0.5, so x' = x and there are no outliers): each compute warp's
    part of a tile is the largest it can be, and several tiles per CTA
    cycle its packed-word buffer through every wrap-around position."""
    n = 4096 * 148 * 2 * 6 + 4096 - 3
    x = np.where(np.arange(n) % 2 == 0, 1.0, -1.0) * float(2 ** 30 - 64)
    want = _run_parity(orc, x.astype(np.float32), block, abs=0.5)
    h = SC.header(want)
    assert h["m"] == 0 and h["W"] == n  # 32-bit codes: one word per element
