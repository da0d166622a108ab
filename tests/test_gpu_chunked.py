"""The chunk-cooperative codec (plan option codec=chunked) on the GPU,
through the C ABI: streams byte-identical to the oracle's
orc_compress_chunked_coder and reconstructions bit-identical to its decode,
for both coders (RZE, RRE), 4096/8192/16384-byte chunks, both bound modes,
ragged and empty inputs, verbatim chunks, the HOST execution kind; corrupt
streams and streams of the other coder are reported."""
import numpy as np
import pytest

import error_bounded_lossy_encode_b200 as E
from error_bounded_lossy_encode_b200 import workloads as WL

pytestmark = pytest.mark.gpu

CHUNK_BYTES = (4096, 8192, 16384)


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _ex(torch):
    return E.cuda_exec(torch.cuda.current_stream().cuda_stream)


def _run(torch, orc, x, cb, coder="rze", **bound):
    mode, val = next(iter(bound.items()))
    want = orc.compress_chunked(x, cb, coder=coder, **bound)
    st, plan = E.eblc_plan_create([x.size], None, f"{mode}={val!r},codec=chunked,chunk={cb},coder={coder}")
    assert st == E.EBLC_OK, E.STATUS_NAMES[st]
    try:
        _, lim = E.eblc_plan_get_limits(plan)
        cap = lim["max_compressed_bytes"]
        assert lim["chunk"] == cb // 4 and lim["block"] == 0
        xd = torch.from_numpy(np.ascontiguousarray(x)).cuda() if x.size else torch.zeros(4, device="cuda")[:0]
        out = torch.full((max(cap, 16),), 0xCD, dtype=torch.uint8, device="cuda")
        sc = E.eblc_sidecar_t()
        st, nb = E.eblc_compress(plan, _ex(torch), xd.data_ptr(), out.data_ptr(), cap, sc)
        assert st == E.EBLC_OK, E.STATUS_NAMES[st]
        got = out[:nb].cpu().numpy()
        diff = np.flatnonzero(got[:min(got.size, want.size)] != want[:min(got.size, want.size)])
        assert got.size == want.size and diff.size == 0, (got.size, want.size, diff[:1])
        assert sc.flags & 4 and bool(sc.flags & 8) == (coder == "rre")
        assert sc.chunk == cb // 4 and sc.total_bytes == want.size
        y = torch.empty(max(x.size, 4), dtype=torch.float32, device="cuda")
        for side in (sc, None):
            y.fill_(7.0)
            assert E.eblc_decompress(plan, _ex(torch), out.data_ptr(), nb, side, y.data_ptr()) == E.EBLC_OK
            assert E.eblc_check(plan, _ex(torch)) == E.EBLC_OK
            y_ref = orc.decompress(want, x.size)
            assert np.array_equal(y[:x.size].cpu().numpy().view(np.uint32), y_ref.view(np.uint32))
    finally:
        E.eblc_plan_destroy(plan)
    return want


@pytest.mark.parametrize("coder", ["rze", "rre"])
@pytest.mark.parametrize("cb", CHUNK_BYTES)
@pytest.mark.parametrize("bound", [{"rel": 1e-3}, {"rel": 1e-6}, {"abs": 1e-7}, {"abs": 0.0}])
def test_chunked_parity(torch_cuda, orc, cb, bound, coder):
    x = np.concatenate([WL.with_spikes((8, 32, 64), 3, p_nonfinite=2e-3), WL.edge_mix(cb // 4 * 2 + 77, 5),
                        WL.sine_noise(5000, 2)])
    _run(torch_cuda, orc, x, cb, coder, **bound)


@pytest.mark.parametrize("coder", ["rze", "rre"])
@pytest.mark.parametrize("cb", CHUNK_BYTES)
@pytest.mark.parametrize("n", [0, 1, 31, 33, 1023, 1024, 1025, 4097, 3 * 4096 + 5])
def test_chunked_sizes(torch_cuda, orc, cb, n, coder):
    _run(torch_cuda, orc, WL.edge_mix(n, n + cb), cb, coder, rel=1e-3)


@pytest.mark.parametrize("coder", ["rze", "rre"])
@pytest.mark.parametrize("cb", CHUNK_BYTES)
def test_chunked_verbatim_and_fields(torch_cuda, orc, cb, coder):
    rng = np.random.default_rng(cb)
    _run(torch_cuda, orc, rng.uniform(-1e9, 1e9, 3 * cb // 4 + 100).astype(np.float32), cb, coder, abs=1.0)
    _run(torch_cuda, orc, WL.kfield((16, 32, 64), 1), cb, coder, rel=1e-4)
    _run(torch_cuda, orc, WL.noise_zero_ramp(65536, 4), cb, coder, abs=1e-7)
    # a constant step per element: every group repeats the one before (RRE's case)
    _run(torch_cuda, orc, (np.arange(3 * cb // 4 + 50, dtype=np.float64) * 0.004).astype(np.float32), cb, coder,
         abs=1e-3)


def test_chunked_host_kind_and_unsupported(torch_cuda, orc):
    torch = torch_cuda
    x = WL.with_spikes((8, 16, 64), 6, p_nonfinite=1e-3)
    want = orc.compress_chunked(x, 8192, rel=1e-3)
    st, plan = E.eblc_plan_create([x.size], None, "rel=1e-3,codec=chunked,chunk=8192")
    try:
        _, lim = E.eblc_plan_get_limits(plan)
        cap = lim["max_compressed_bytes"]
        xh = torch.from_numpy(x).pin_memory()
        oh = torch.zeros(cap, dtype=torch.uint8).pin_memory()
        sc = E.eblc_sidecar_t()
        st, nb = E.eblc_compress(plan, E.host_exec(), xh.data_ptr(), oh.data_ptr(), cap, sc)
        assert st == E.EBLC_OK and np.array_equal(oh[:nb].numpy(), want)
        yh = torch.zeros(x.size, dtype=torch.float32).pin_memory()
        assert E.eblc_decompress(plan, E.host_exec(), oh.data_ptr(), nb, sc, yh.data_ptr()) == E.EBLC_OK
        assert np.array_equal(yh.numpy().view(np.uint32), orc.decompress(want, x.size).view(np.uint32))
        xd, out = xh.cuda(), oh.cuda()
        d_res = torch.zeros(32, dtype=torch.uint8, device="cuda")
        assert E.eblc_compress_async(plan, _ex(torch), xd.data_ptr(), out.data_ptr(), cap, d_res.data_ptr()) == \
            E.EBLC_UNSUPPORTED
        rng_d = torch.zeros(2, device="cuda")
        assert E.eblc_compress_range(plan, _ex(torch), xd.data_ptr(), rng_d.data_ptr(), out.data_ptr(), cap)[0] == \
            E.EBLC_UNSUPPORTED
        # corrupt: a record head that claims more words than its chunk holds
        bad = want.copy()
        rec0 = 128 + -(-8 * (-(-x.size // 2048)) // 16) * 16
        bad[rec0 + 3] ^= 0x40
        d = torch.from_numpy(bad).cuda()
        y = torch.empty(x.size, device="cuda")
        st = E.eblc_decompress(plan, _ex(torch), d.data_ptr(), bad.size, sc, y.data_ptr())
        assert st == E.EBLC_OK and E.eblc_check(plan, _ex(torch)) == E.EBLC_CORRUPT
    finally:
        E.eblc_plan_destroy(plan)
    # a stream of the other coder is not this plan's
    rre = orc.compress_chunked(x, 8192, rel=1e-3, coder="rre")
    st, plan = E.eblc_plan_create([x.size], None, "rel=1e-3,codec=chunked,chunk=8192")
    try:
        d = torch.from_numpy(rre).cuda()
        y = torch.empty(x.size, device="cuda")
        assert E.eblc_decompress(plan, _ex(torch), d.data_ptr(), rre.size, None, y.data_ptr()) == E.EBLC_INVALID_ARG
    finally:
        E.eblc_plan_destroy(plan)
    for opts in ("rel=1e-3,chunk=8192", "rel=1e-3,codec=bogus", "rel=1e-3,coder=rre",
                 "rel=1e-3,codec=chunked,coder=bogus"):
        st, p2 = E.eblc_plan_create([4096], None, opts)
        assert st == E.EBLC_INVALID_ARG and not p2
    st, p2 = E.eblc_plan_create([4096], None, "rel=1e-3,codec=chunked,chunk=2048")
    assert st == E.EBLC_UNSUPPORTED


@pytest.mark.slow
def test_chunked_full_size(torch_cuda, orc):
    _run(torch_cuda, orc, WL.standard("field512cube_spikes"), 16384, rel=1e-3)
