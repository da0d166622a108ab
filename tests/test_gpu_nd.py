"""The 2-D / 3-D Lorenzo path (plan option lorenzo=nd) on the GPU, through
the C ABI: streams byte-identical to the oracle's orc_compress_lorenzo and
reconstructions bit-identical to the oracle's decode, over several bricks,
both block sizes, both bound modes, with spikes and non-finite values;
unsupported shapes and predictor mismatches are reported."""
import numpy as np
import pytest

import error_bounded_lossy_encode_b200 as E
from error_bounded_lossy_encode_b200 import workloads as WL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _ex(torch):
    return E.cuda_exec(torch.cuda.current_stream().cuda_stream)


def _field(shape, seed, specials=True):
    x = WL.with_spikes((1, 1, int(np.prod(shape))), seed, p_nonfinite=2e-3 if specials else 0.0).reshape(shape)
    if specials:
        x.reshape(-1)[:6] = [np.nan, np.inf, -np.inf, -0.0, 1e-40, 3e38]
    return np.ascontiguousarray(x)


def _run(torch, orc, x, block, **bound):
    mode, val = next(iter(bound.items()))
    want = orc.compress_lorenzo(x, block, **bound)
    st, plan = E.eblc_plan_create(list(x.shape), None, f"{mode}={val!r},block={block},lorenzo=nd")
    assert st == E.EBLC_OK, E.STATUS_NAMES[st]
    try:
        _, lim = E.eblc_plan_get_limits(plan)
        cap = lim["max_compressed_bytes"]
        xd = torch.from_numpy(x).cuda()
        out = torch.full((cap,), 0xCD, dtype=torch.uint8, device="cuda")
        sc = E.eblc_sidecar_t()
        st, nb = E.eblc_compress(plan, _ex(torch), xd.data_ptr(), out.data_ptr(), cap, sc)
        assert st == E.EBLC_OK, E.STATUS_NAMES[st]
        got = out[:nb].cpu().numpy()
        assert got.size == want.size, (got.size, want.size)
        diff = np.flatnonzero(got != want)
        assert diff.size == 0, ("first differing byte", int(diff[0]) if diff.size else None)
        assert sc.flags & 2
        y = torch.empty_like(xd)
        assert E.eblc_decompress(plan, _ex(torch), out.data_ptr(), nb, sc, y.data_ptr()) == E.EBLC_OK
        assert E.eblc_check(plan, _ex(torch)) == E.EBLC_OK
        y_ref = orc.decompress(want, x.size)
        assert np.array_equal(y.cpu().numpy().reshape(-1).view(np.uint32), y_ref.view(np.uint32))
        # without the sidecar: the header is read back from the device
        y.zero_()
        assert E.eblc_decompress(plan, _ex(torch), out.data_ptr(), nb, None, y.data_ptr()) == E.EBLC_OK
        assert E.eblc_check(plan, _ex(torch)) == E.EBLC_OK
        assert np.array_equal(y.cpu().numpy().reshape(-1).view(np.uint32), y_ref.view(np.uint32))
    finally:
        E.eblc_plan_destroy(plan)
    return want


@pytest.mark.parametrize("block", [64, 256])
@pytest.mark.parametrize("bound", [{"rel": 1e-3}, {"rel": 1e-5}, {"abs": 1e-7}, {"abs": 0.0}])
def test_nd3_parity(torch_cuda, orc, block, bound):
    _run(torch_cuda, orc, _field((32, 48, 64), 11), block, **bound)


@pytest.mark.parametrize("block", [64, 256])
@pytest.mark.parametrize("bound", [{"rel": 1e-3}, {"rel": 1e-5}, {"abs": 1e-7}, {"abs": 0.0}])
def test_nd2_parity(torch_cuda, orc, block, bound):
    _run(torch_cuda, orc, _field((128, 192), 12), block, **bound)


@pytest.mark.parametrize("block", [64, 256])
def test_nd_fields(torch_cuda, orc, block):
    _run(torch_cuda, orc, WL.kfield((48, 32, 64), 3).reshape(48, 32, 64), block, rel=1e-4)
    _run(torch_cuda, orc, WL.kfield((1, 192, 256), 4).reshape(192, 256), block, rel=1e-4)
    _run(torch_cuda, orc, np.full((16, 32, 16), -3.25, np.float32), block, abs=1e-3)


def test_nd_unsupported_and_mismatch(torch_cuda, orc):
    torch = torch_cuda
    for dims, opts in (([16, 16, 17], "rel=1e-3,block=64,lorenzo=nd"), ([16, 16, 16], "rel=1e-3,block=128,lorenzo=nd"),
                       ([64, 60], "rel=1e-3,block=64,lorenzo=nd"), ([4096], "rel=1e-3,block=64,lorenzo=nd"),
                       ([2, 16, 16, 16], "rel=1e-3,block=64,lorenzo=nd")):
        st, plan = E.eblc_plan_create(dims, None, opts)
        assert st == E.EBLC_UNSUPPORTED and not plan, (dims, opts)
    st, plan = E.eblc_plan_create([16, 16, 16], None, "rel=1e-3,block=64,lorenzo=xyz")
    assert st == E.EBLC_INVALID_ARG
    # a stream of the 3-D predictor given to a plan of the 1-D path is refused
    x = _field((16, 16, 16), 5)
    want = orc.compress_lorenzo(x, 64, rel=1e-3)
    st, plan = E.eblc_plan_create([x.size], None, "rel=1e-3,block=64")
    try:
        d = torch.from_numpy(want).cuda()
        y = torch.empty(x.size, dtype=torch.float32, device="cuda")
        assert E.eblc_decompress(plan, _ex(torch), d.data_ptr(), want.size, None, y.data_ptr()) == E.EBLC_INVALID_ARG
    finally:
        E.eblc_plan_destroy(plan)


@pytest.mark.slow
@pytest.mark.parametrize("name,shape,block,bound", [("field512cube_spikes", (512, 512, 512), 64, 1e-3),
                                                    ("field256x384x384", (256, 384, 384), 256, 1e-4)])
def test_nd_full_size(torch_cuda, orc, name, shape, block, bound):
    _run(torch_cuda, orc, WL.standard(name).reshape(shape), block, rel=bound)
