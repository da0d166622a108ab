"""eblc_compress_noalloc: the plan-free compress entry point for callers that
cannot allocate device memory (for example code under an allocator that owns
all device memory, or inside a region where cudaMalloc is forbidden).  Its
scratch is a fixed file-scope device array, so it needs no plan and makes no
allocation.  Checked through the C ABI against the plan-based eblc_compress on
two calls in a row (the array keeps the previous call's contents, so the
second call shows that everything that must start at zero is cleared).

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


@pytest.mark.parametrize("block,mode,bound", [(64, "rel", 1e-3), (256, "abs", 1e-4)])
def test_noalloc_matches_plan_compress(block, mode, bound):
    import torch

    assert torch.cuda.is_available()
    x_np = np.concatenate([WL.with_spikes((24, 64, 64), 2, p_nonfinite=1e-3), WL.edge_mix(5000, 1)])
    x = torch.from_numpy(x_np).cuda()
    want, want_sc, cap = _plan_compress(torch, x, block, mode, bound)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full((cap,), 0xAB, dtype=torch.uint8, device="cuda")
        sc = E.eblc_sidecar_t()
        st, nbytes = E.eblc_compress_noalloc(x.data_ptr(), x.numel(), block, mode == "abs", bound, out.data_ptr(),
                                             cap, stream, sc)
        assert st == E.EBLC_OK, (call, E.STATUS_NAMES[st])
        assert nbytes == want.size
        assert np.array_equal(out[:nbytes].cpu().numpy(), want), call
        assert E.sidecar_dict(sc) == want_sc


def test_noalloc_rejects_sizes_beyond_its_limit():
    import torch

    x = torch.zeros(16, device="cuda")
    out = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    st, _ = E.eblc_compress_noalloc(x.data_ptr(), E.EBLC_NOALLOC_MAX_N + 1, 64, False, 1e-3, out.data_ptr(),
                                    out.numel())
    assert st == E.EBLC_UNSUPPORTED
