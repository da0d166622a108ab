"""The host-sync-free compress (eblc_compress_async): the same stream as the
oracle and as the synchronous call, the device-written result record, the
capacity report, interleaving with synchronous calls on one plan, and
capture into a CUDA graph that is then replayed on new inputs."""
import numpy as np
import pytest

import error_bounded_lossy_encode_b200 as E
from error_bounded_lossy_encode_b200 import workloads as WL
from tests import streamcheck as SC

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _result(torch, d_result):
    torch.cuda.synchronize()
    return E.async_result(d_result.cpu().numpy().tobytes())


def _async(torch, g, x, out, d_result, cap=None):
    cap = g.lim["max_compressed_bytes"] if cap is None else cap
    st = E.eblc_compress_async(g.plan, E.cuda_exec(torch.cuda.current_stream().cuda_stream), x.data_ptr(),
                               out.data_ptr(), cap, d_result.data_ptr())
    assert st == E.EBLC_OK, E.STATUS_NAMES[st]
    return _result(torch, d_result)


@pytest.mark.parametrize("block,n,mode", [(64, 4096 * 300 + 17, dict(rel=1e-3)), (128, 100_003, dict(abs=1e-2)),
                                          (32, 4096, dict(rel=1e-4)), (256, 1, dict(rel=1e-3))])
def test_async_matches_oracle(torch_cuda, orc, block, n, mode):
    from tests.gpu_util import GpuCodec

    torch = torch_cuda
    x_np = WL.edge_mix(n, n + block)
    want = orc.compress(x_np, block, **mode)
    h = SC.header(want)
    with GpuCodec(n, block, **mode) as g:
        x = torch.from_numpy(x_np).cuda()
        out = torch.zeros(g.lim["max_compressed_bytes"], dtype=torch.uint8, device="cuda")
        d_result = torch.zeros(32, dtype=torch.uint8, device="cuda")
        r = _async(torch, g, x, out, d_result)
        assert r["status"] == E.EBLC_OK
        assert r["compressed_bytes"] == want.size and r["n_outliers"] == h["m"] and r["payload_words"] == h["W"]
        assert np.array_equal(out[: want.size].cpu().numpy(), want)


def test_async_interleaved_with_sync_calls(torch_cuda, orc):
    """Calls alternate between the plan's two look-back arrays on the device;
    synchronous and asynchronous calls may follow each other in any order."""
    from tests.gpu_util import GpuCodec

    torch = torch_cuda
    n, block = 4096 * 37 + 5, 64
    xs = [WL.edge_mix(n, 100 + k) for k in range(5)]
    wants = [orc.compress(x, block, rel=1e-3) for x in xs]
    with GpuCodec(n, block, rel=1e-3) as g:
        d_result = torch.zeros(32, dtype=torch.uint8, device="cuda")
        for k, kind in enumerate(["async", "sync", "sync", "async", "async"]):
            x = torch.from_numpy(xs[k]).cuda()
            if kind == "async":
                out = torch.zeros(g.lim["max_compressed_bytes"], dtype=torch.uint8, device="cuda")
                r = _async(torch, g, x, out, d_result)
                assert r["status"] == E.EBLC_OK and r["compressed_bytes"] == wants[k].size
                got = out[: wants[k].size].cpu().numpy()
            else:
                st, out, nbytes, _ = g.compress(x)
                assert st == E.EBLC_OK and nbytes == wants[k].size
                got = out[:nbytes].cpu().numpy()
            assert np.array_equal(got, wants[k]), (k, kind)


def test_async_capacity_reported_on_device(torch_cuda, orc):
    from tests.gpu_util import GpuCodec

    torch = torch_cuda
    n, block = 4096 * 20, 128
    x_np = WL.edge_mix(n, 9)
    want = orc.compress(x_np, block, rel=1e-4)
    with GpuCodec(n, block, rel=1e-4) as g:
        x = torch.from_numpy(x_np).cuda()
        cap = want.size - 64
        out = torch.zeros(g.lim["max_compressed_bytes"], dtype=torch.uint8, device="cuda")
        d_result = torch.zeros(32, dtype=torch.uint8, device="cuda")
        r = _async(torch, g, x, out, d_result, cap=cap)
        assert r["status"] == E.EBLC_CAPACITY and r["compressed_bytes"] == want.size
        assert not out[cap:].any().item()  # nothing written beyond the capacity
        # the plan is still good afterwards
        r = _async(torch, g, x, out, d_result)
        assert r["status"] == E.EBLC_OK and np.array_equal(out[: want.size].cpu().numpy(), want)


def test_async_argument_errors(torch_cuda):
    from tests.gpu_util import GpuCodec

    torch = torch_cuda
    with GpuCodec(4096, 64, rel=1e-3) as g:
        x = torch.zeros(4096, device="cuda")
        out = torch.zeros(g.lim["max_compressed_bytes"], dtype=torch.uint8, device="cuda")
        d_result = torch.zeros(32, dtype=torch.uint8, device="cuda")
        cap = g.lim["max_compressed_bytes"]
        ex = E.cuda_exec(torch.cuda.current_stream().cuda_stream)
        assert E.eblc_compress_async(g.plan, ex, x.data_ptr(), out.data_ptr(), cap, 0) == E.EBLC_INVALID_ARG
        assert E.eblc_compress_async(g.plan, E.host_exec(), x.data_ptr(), out.data_ptr(), cap,
                                     d_result.data_ptr()) == E.EBLC_INVALID_ARG
        assert E.eblc_compress_async(g.plan, ex, x.data_ptr(), out.data_ptr() + 4, cap - 16,
                                     d_result.data_ptr()) == E.EBLC_INVALID_ARG
        assert E.eblc_compress_async(g.plan, ex, x.data_ptr(), out.data_ptr(), 64,
                                     d_result.data_ptr()) == E.EBLC_CAPACITY


@pytest.mark.parametrize("mode", [dict(rel=1e-3), dict(abs=1e-3)])
def test_graph_capture_and_replay(torch_cuda, orc, mode):
    """Capture one compress into a CUDA graph, then replay it on four new
    inputs copied into the captured input buffer: every replay's stream and
    result record match the oracle for that input."""
    from tests.gpu_util import GpuCodec

    torch = torch_cuda
    n, block = 4096 * 296 * 2 + 1234, 64
    xs = [WL.with_spikes((n,), seed=20 + k) for k in range(4)]
    wants = [orc.compress(x, block, **mode) for x in xs]
    with GpuCodec(n, block, **mode) as g:
        cap = g.lim["max_compressed_bytes"]
        x_static = torch.zeros(n, dtype=torch.float32, device="cuda")
        out = torch.zeros(cap, dtype=torch.uint8, device="cuda")
        d_result = torch.zeros(32, dtype=torch.uint8, device="cuda")
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):  # warm-up outside capture (first-launch setup)
            st = E.eblc_compress_async(g.plan, E.cuda_exec(s.cuda_stream), x_static.data_ptr(), out.data_ptr(), cap,
                                       d_result.data_ptr())
            assert st == E.EBLC_OK
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            st = E.eblc_compress_async(g.plan, E.cuda_exec(torch.cuda.current_stream().cuda_stream),
                                       x_static.data_ptr(), out.data_ptr(), cap, d_result.data_ptr())
        assert st == E.EBLC_OK
        for k in range(4):
            x_static.copy_(torch.from_numpy(xs[k]).cuda())
            d_result.zero_()
            graph.replay()
            r = _result(torch, d_result)
            assert r["status"] == E.EBLC_OK and r["compressed_bytes"] == wants[k].size, k
            assert np.array_equal(out[: wants[k].size].cpu().numpy(), wants[k]), k
        del graph
