"""The sharded compress on the GPU, through the C ABI: eblc_value_range
against the oracle's value range, and eblc_compress_range for chunk-aligned
parts of one array under the whole array's range (the ranks of a multi-GPU
run, taken one after another on this GPU; the range all-reduce is done on
the host here) -- each part's stream byte-identical to the oracle's
compress_range of that part, its reconstruction bit-identical to the
oracle's decode.  Argument errors are reported."""
import numpy as np
import pytest

import error_bounded_lossy_encode_b200 as E
from error_bounded_lossy_encode_b200 import sharded as SH
from error_bounded_lossy_encode_b200 import workloads as WL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _ex(torch):
    return E.cuda_exec(torch.cuda.current_stream().cuda_stream)


def _plan(n, block, rel):
    st, plan = E.eblc_plan_create([n], None, f"rel={rel!r},block={block}")
    assert st == E.EBLC_OK, E.STATUS_NAMES[st]
    _, lim = E.eblc_plan_get_limits(plan)
    return plan, lim["max_compressed_bytes"]


def _gpu_range(torch, plan, xd):
    rng = torch.full((2,), 7.0, dtype=torch.float32, device="cuda")
    assert E.eblc_value_range(plan, _ex(torch), xd.data_ptr(), rng.data_ptr()) == E.EBLC_OK
    return rng.cpu().numpy()


@pytest.mark.parametrize("case", ["field", "all_nan", "neg_zero", "empty", "inf_mix"])
def test_value_range_matches_oracle(torch_cuda, orc, case):
    torch = torch_cuda
    x = {"field": WL.with_spikes((16, 32, 64), 2, p_nonfinite=1e-3),
         "all_nan": np.full(5000, np.nan, np.float32),
         "neg_zero": np.array([-0.0, -0.0, 0.0, -0.0] * 1000, np.float32),
         "empty": np.zeros(0, np.float32),
         "inf_mix": np.array([np.inf, -2.5, np.nan, 7.0, -np.inf] * 999, np.float32)}[case]
    plan, _ = _plan(x.size, 64, 1e-3)
    try:
        xd = torch.from_numpy(x).cuda() if x.size else torch.zeros(4, device="cuda")[:0]
        got = _gpu_range(torch, plan, xd)
        lo, hi, _ = orc.value_range(x)
        assert got.view(np.uint32).tolist() == np.array([lo, hi], np.float32).view(np.uint32).tolist()
    finally:
        E.eblc_plan_destroy(plan)


@pytest.mark.parametrize("block", [32, 64, 128, 256])
@pytest.mark.parametrize("parts", [2, 3])
def test_parts_under_the_whole_range_match_oracle(torch_cuda, orc, block, parts):
    torch = torch_cuda
    rel = 1e-3
    x = np.concatenate([WL.kfield((8, 32, 64), 3), WL.with_spikes((8, 16, 64), 4, p_nonfinite=2e-3),
                        WL.edge_mix(3 * 4096 + 77, 5)])
    bounds = [SH.part_bounds(x.size, parts, r) for r in range(parts)]
    plans, ranges = [], []
    try:
        for a, b in bounds:  # every "rank" computes its part's range
            plan, cap = _plan(b - a, block, rel)
            plans.append((plan, cap))
            ranges.append(_gpu_range(torch, plan, torch.from_numpy(x[a:b]).cuda()))
        lo = min(float(r[0]) for r in ranges)  # the all-reduce, on the host here
        hi = max(float(r[1]) for r in ranges)
        g = torch.tensor([lo, hi], dtype=torch.float32, device="cuda")
        for (a, b), (plan, cap) in zip(bounds, plans):
            xd = torch.from_numpy(x[a:b]).cuda()
            out = torch.empty(cap, dtype=torch.uint8, device="cuda")
            sc = E.eblc_sidecar_t()
            st, nbytes = E.eblc_compress_range(plan, _ex(torch), xd.data_ptr(), g.data_ptr(), out.data_ptr(), cap, sc)
            assert st == E.EBLC_OK, E.STATUS_NAMES[st]
            want = orc.compress_range(x[a:b], block, rel, lo, hi)
            got = out[:nbytes].cpu().numpy()
            assert got.size == want.size and np.array_equal(got, want), (a, b)
            y = torch.empty(b - a, dtype=torch.float32, device="cuda")
            assert E.eblc_decompress(plan, _ex(torch), out.data_ptr(), nbytes, sc, y.data_ptr()) == E.EBLC_OK
            assert E.eblc_check(plan, _ex(torch)) == E.EBLC_OK
            assert np.array_equal(y.cpu().numpy().view(np.uint32), orc.decompress(want, b - a).view(np.uint32))
    finally:
        for plan, _ in plans:
            E.eblc_plan_destroy(plan)


def test_own_range_equals_compress_and_errors(torch_cuda, orc):
    torch = torch_cuda
    x = WL.with_spikes((16, 32, 64), 7, p_nonfinite=1e-3)
    plan, cap = _plan(x.size, 128, 1e-4)
    try:
        xd = torch.from_numpy(x).cuda()
        rng = torch.from_numpy(_gpu_range(torch, plan, xd)).cuda()
        out = torch.empty(cap, dtype=torch.uint8, device="cuda")
        st, nb = E.eblc_compress_range(plan, _ex(torch), xd.data_ptr(), rng.data_ptr(), out.data_ptr(), cap)
        assert st == E.EBLC_OK and np.array_equal(out[:nb].cpu().numpy(), orc.compress(x, 128, rel=1e-4))
        for bad in ([1.0, 0.0], [float("nan"), 1.0], [0.0, float("inf")]):
            b = torch.tensor(bad, dtype=torch.float32, device="cuda")
            st, _ = E.eblc_compress_range(plan, _ex(torch), xd.data_ptr(), b.data_ptr(), out.data_ptr(), cap)
            assert st == E.EBLC_INVALID_ARG, bad
        # the plan's next call is unaffected
        st, nb = E.eblc_compress_range(plan, _ex(torch), xd.data_ptr(), rng.data_ptr(), out.data_ptr(), cap)
        assert st == E.EBLC_OK and np.array_equal(out[:nb].cpu().numpy(), orc.compress(x, 128, rel=1e-4))
        st, _ = E.eblc_compress_range(plan, E.host_exec(), xd.data_ptr(), rng.data_ptr(), out.data_ptr(), cap)
        assert st == E.EBLC_UNSUPPORTED
    finally:
        E.eblc_plan_destroy(plan)
    st, aplan = E.eblc_plan_create([x.size], None, "abs=1e-3,block=64")
    try:
        st, _ = E.eblc_compress_range(aplan, _ex(torch), xd.data_ptr(), rng.data_ptr(), out.data_ptr(), cap)
        assert st == E.EBLC_INVALID_ARG
    finally:
        E.eblc_plan_destroy(aplan)
