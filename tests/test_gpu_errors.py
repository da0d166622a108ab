"""Error paths through the C ABI on the GPU.  Nothing here faults, traps or
hangs a GPU: capacity and corruption are detected by bounds checks, and the
look-back timeout is forced with the plan's test hook (a tile that never
publishes, with a 100 ms wait limit) so a bounded wait runs out and the
kernel returns normally."""
import numpy as np
import pytest

import error_bounded_lossy_encode_b200 as E
from error_bounded_lossy_encode_b200 import workloads as WL
from tests import streamcheck as SC

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available()
    return torch


def test_output_capacity(torch_cuda, orc):
    from tests.gpu_util import GpuCodec

    x = WL.sine_noise(100000, 0)
    want = orc.compress(x, 128, rel=1e-3)
    with GpuCodec(x.size, 128, rel=1e-3) as g:
        st, _, nbytes, _ = g.compress(torch_cuda.from_numpy(x).cuda(), cap=want.size - 4)
        assert st == E.EBLC_CAPACITY and nbytes == want.size  # the size it would need
        st, got, _ = g.compress_np(x)
        assert st == 0 and np.array_equal(got, want)  # plan still usable
        st, _, _, _ = g.compress(torch_cuda.from_numpy(x).cuda(), cap=64)
        assert st == E.EBLC_CAPACITY


def test_outlier_capacity(torch_cuda, orc):
    from tests.gpu_util import GpuCodec

    x = WL.edge_mix(50000, 2)
    m = SC.header(orc.compress(x, 64, abs=1e-3))["m"]
    with GpuCodec(x.size, 64, abs=1e-3, extra=f"outlier_cap={m - 1}") as g:
        st, _, _ = g.compress_np(x)
        assert st == E.EBLC_CAPACITY
    with GpuCodec(x.size, 64, abs=1e-3, extra=f"outlier_cap={m}") as g:
        st, got, _ = g.compress_np(x)
        assert st == 0 and np.array_equal(got, orc.compress(x, 64, abs=1e-3))


def test_corrupt_streams(torch_cuda, orc):
    from tests.gpu_util import GpuCodec

    x = WL.edge_mix(40000, 4)
    s = orc.compress(x, 64, rel=1e-3)
    h = SC.header(s)
    with GpuCodec(x.size, 64, rel=1e-3) as g:
        bad = s.copy()
        bad[0] ^= 0xFF  # magic
        st, _, _ = g.decompress_np(bad, None)
        assert st == E.EBLC_CORRUPT
        bad = s.copy()
        bad[128 + 3] = 40  # a width above 32: detected on the device
        st, chk, _ = g.decompress_np(bad, None)
        assert st == 0 and chk == E.EBLC_CORRUPT
        nb = -(-x.size // 64)
        for blk in (nb - 1, 64 * 3 + 17):  # the last block of the stream; one inside a later chunk
            bad = s.copy()
            bad[128 + blk] = 33
            st, chk, _ = g.decompress_np(bad, None)
            assert st == 0 and chk == E.EBLC_CORRUPT, blk
        bad = s.copy()
        off = SC.sections(h)
        bad[off["index"] + 8: off["index"] + 12] = np.frombuffer(np.uint32(0xFFFFFF).tobytes(), np.uint8)
        st, chk, _ = g.decompress_np(bad, None)
        assert st == 0 and chk == E.EBLC_CORRUPT
        st, _, _ = g.decompress_np(s[:-8], None)  # truncated
        assert st == E.EBLC_CORRUPT
        st, chk, y = g.decompress_np(s, None)  # the plan still works
        assert st == 0 and chk == 0
        assert np.array_equal(y.view(np.uint32), orc.decompress(s, x.size).view(np.uint32))


def test_lookback_timeout_is_reported(torch_cuda, orc):
    from tests.gpu_util import GpuCodec

    x = WL.sine_noise(40 * 4096, 0)
    with GpuCodec(x.size, 128, rel=1e-3, extra="stall_tile=1,wait_ms=100") as g:
        st, _, _ = g.compress_np(x)
        assert st == E.EBLC_TIMEOUT
    torch_cuda.cuda.synchronize()  # the context is still usable
    with GpuCodec(x.size, 128, rel=1e-3) as g:
        st, got, _ = g.compress_np(x)
        assert st == 0 and np.array_equal(got, orc.compress(x, 128, rel=1e-3))


def test_plan_recovers_after_timeout(torch_cuda, orc):
    """Call 0 succeeds, call 1 times out (tile 5 never publishes; later waits
    give up, so some look-back words of the array call 2 will use are never
    cleared), and calls 2 and 3 on the same plan, on other inputs, must again
    produce the oracle's streams: a failed call's leftovers are cleared
    before the next call."""
    from tests.gpu_util import GpuCodec

    xs = [WL.sine_noise(60 * 4096, k) for k in range(4)]
    wants = [orc.compress(x, 128, rel=1e-3) for x in xs]
    with GpuCodec(xs[0].size, 128, rel=1e-3, extra="stall_tile=5,stall_call=1,wait_ms=100") as g:
        st, got, _ = g.compress_np(xs[0])
        assert st == 0 and np.array_equal(got, wants[0])
        st, _, _ = g.compress_np(xs[1])
        assert st == E.EBLC_TIMEOUT
        for k in (2, 3):
            st, got, _ = g.compress_np(xs[k])
            assert st == 0 and np.array_equal(got, wants[k]), k


def test_async_timeout_reported_on_device(torch_cuda, orc):
    import torch

    from tests.gpu_util import GpuCodec

    x_np = WL.sine_noise(60 * 4096, 7)
    want = orc.compress(x_np, 128, rel=1e-3)
    with GpuCodec(x_np.size, 128, rel=1e-3, extra="stall_tile=3,wait_ms=100") as g:
        x = torch.from_numpy(x_np).cuda()
        cap = g.lim["max_compressed_bytes"]
        out = torch.zeros(cap, dtype=torch.uint8, device="cuda")
        d_result = torch.zeros(32, dtype=torch.uint8, device="cuda")
        ex = E.cuda_exec(torch.cuda.current_stream().cuda_stream)
        for k, expect in enumerate((E.EBLC_TIMEOUT, E.EBLC_OK)):
            assert E.eblc_compress_async(g.plan, ex, x.data_ptr(), out.data_ptr(), cap, d_result.data_ptr()) == 0
            torch.cuda.synchronize()
            r = E.async_result(d_result.cpu().numpy().tobytes())
            assert r["status"] == expect, (k, r)
        assert np.array_equal(out[: want.size].cpu().numpy(), want)


def test_argument_errors(torch_cuda):
    st, plan = E.eblc_plan_create([1000], None, "rel=1e-3,block=64")
    assert st == 0
    try:
        x = torch_cuda.zeros(1004, device="cuda")
        out = torch_cuda.zeros(1 << 16, dtype=torch_cuda.uint8, device="cuda")
        hip = E.eblc_execution_t(E.EBLC_EXECUTION_HIP, 0, None)
        assert E.eblc_compress(plan, hip, x.data_ptr(), out.data_ptr(), out.numel())[0] == E.EBLC_UNSUPPORTED
        ex = E.cuda_exec(0)
        assert E.eblc_compress(plan, ex, x.data_ptr() + 4, out.data_ptr(), out.numel())[0] == E.EBLC_INVALID_ARG
        assert E.eblc_compress(plan, ex, x.data_ptr(), out.data_ptr() + 8, out.numel() - 8)[0] == E.EBLC_INVALID_ARG
        assert E.eblc_compress(plan, ex, 0, out.data_ptr(), out.numel())[0] == E.EBLC_INVALID_ARG
    finally:
        E.eblc_plan_destroy(plan)
    assert E.eblc_plan_create([4, 5], [1, 4], "rel=1e-3")[0] == E.EBLC_UNSUPPORTED  # not C-contiguous
    assert E.eblc_plan_create([(1 << 30) + 1], None, None)[0] == E.EBLC_UNSUPPORTED
