"""eblc_compress_noalloc: the plan-free compress entry point for callers that
cannot allocate device memory (for example code under an allocator that owns
all device memory, or inside a region where cudaMalloc is forbidden).  Its
scratch is a fixed file-scope device array, so it needs no plan and makes no
allocation.

Checked through the C ABI against the CPU oracle's stream and against the
plan-based eblc_compress.  The array keeps the previous call's contents, so
the calls are chained on purpose: the same input twice in a row, a smaller
input after a larger one with other data and another bound mode, and an empty
relative-bound call after a non-empty one.  A call that read anything left
over from the call before would produce a different stream.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import numpy as np
import pytest

import error_bounded_lossy_encode_b200 as E
from error_bounded_lossy_encode_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _plan_compress(torch, x, block, mode, bound):
    st, plan = E.eblc_plan_create([x.numel()], None, f"{mode}={bound!r},block={block}")
    assert st == E.EBLC_OK
    try:
        _, lim = E.eblc_plan_get_limits(plan)
        out = torch.empty(lim["max_compressed_bytes"], dtype=torch.uint8, device="cuda")
        sc = E.eblc_sidecar_t()
        ex = E.cuda_exec(torch.cuda.current_stream().cuda_stream)
        st, nbytes = E.eblc_compress(plan, ex, x.data_ptr(), out.data_ptr(), lim["max_compressed_bytes"], sc)
        assert st == E.EBLC_OK
        return out[:nbytes].cpu().numpy(), E.sidecar_dict(sc), lim["max_compressed_bytes"]
    finally:
        E.eblc_plan_destroy(plan)


def _noalloc(torch, x, block, mode, bound, cap):
    out = torch.full((max(cap, 16),), 0xAB, dtype=torch.uint8, device="cuda")
    sc = E.eblc_sidecar_t()
    stream = torch.cuda.current_stream().cuda_stream
    st, nbytes = E.eblc_compress_noalloc(x.data_ptr(), x.numel(), block, mode == "abs", bound, out.data_ptr(),
                                         cap, stream, sc)
    assert st == E.EBLC_OK, E.STATUS_NAMES[st]
    return out[:nbytes].cpu().numpy(), E.sidecar_dict(sc)


def _inputs():
    big = np.concatenate([WL.with_spikes((24, 64, 64), 2, p_nonfinite=1e-3), WL.edge_mix(5000, 1)])
    small = np.concatenate([WL.noise_zero_ramp(20000, 4), WL.edge_mix(777, 9)])
    return big, small


@pytest.mark.parametrize("block,mode,bound", [(64, "rel", 1e-3), (256, "abs", 1e-4)])
def test_noalloc_matches_oracle_and_plan_compress(orc, block, mode, bound):
    import torch

    assert torch.cuda.is_available()
    big, _ = _inputs()
    want = orc.compress(big, block, **{mode: bound})
    x = torch.from_numpy(big).cuda()
    plan_stream, plan_sc, cap = _plan_compress(torch, x, block, mode, bound)
    assert np.array_equal(plan_stream, want)
    for call in range(2):  # two calls in a row on the same input
        got, sc = _noalloc(torch, x, block, mode, bound, cap)
        assert got.size == want.size and np.array_equal(got, want), call
        assert sc == plan_sc, call


def test_noalloc_chained_calls_leave_nothing_behind(orc):
    """Larger input, then a smaller one with other data, block and bound mode,
    then an empty relative-bound call: each equals the oracle's stream."""
    import torch

    big, small = _inputs()
    cases = [(big, 64, "rel", 1e-3), (small, 128, "abs", 1e-6), (big[:9000], 32, "rel", 1e-2),
             (np.zeros(0, np.float32), 64, "rel", 1e-3), (small, 128, "rel", 1e-4)]
    for k, (x_np, block, mode, bound) in enumerate(cases):
        want = orc.compress(x_np, block, **{mode: bound})
        x = torch.from_numpy(np.ascontiguousarray(x_np)).cuda() if x_np.size else torch.zeros(4, device="cuda")
        xin = x if x_np.size else x[:0]
        got, sc = _noalloc(torch, xin, block, mode, bound, want.size)
        assert got.size == want.size and np.array_equal(got, want), (k, block, mode, bound)
        assert sc["total_bytes"] == want.size, k


def test_noalloc_rejects_sizes_beyond_its_limit():
    import torch

    x = torch.zeros(16, device="cuda")
    out = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    st, _ = E.eblc_compress_noalloc(x.data_ptr(), E.EBLC_NOALLOC_MAX_N + 1, 64, False, 1e-3, out.data_ptr(),
                                    out.numel())
    assert st == E.EBLC_UNSUPPORTED
