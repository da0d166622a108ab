"""Full-size parity on the five standard workloads, in the same launch
configuration the benchmark times (one plan per workload, device-resident
input, CUDA stream): every stream byte-identical to the oracle's, every
reconstruction bit-identical to the oracle's decode, and |x - x'| <= eb (fp64)
on every non-outlier element with outliers bit-exact."""
import numpy as np
import pytest

from error_bounded_lossy_encode_b200 import workloads as WL
from tests import streamcheck as SC

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _full_check(orc, x, block, **mode):
    import torch
    from tests.gpu_util import GpuCodec

    want = orc.compress(x, block, **mode)
    h = SC.header(want)
    with GpuCodec(x.size, block, **mode) as g:
        xd = torch.from_numpy(x).cuda()
        st, out, nbytes, sc = g.compress(xd)
        assert st == 0
        got = out[:nbytes].cpu().numpy()
        assert nbytes == want.size
        if not np.array_equal(got, want):
            d = np.flatnonzero(got != want)
            raise AssertionError(f"{d.size} bytes differ, first at {d[0]} of {want.size}")
        del out
        sd = torch.from_numpy(want).cuda()
        st, y = g.decompress(sd, want.size, sc)
        assert st == 0 and g.check() == 0
        y = y.cpu().numpy()
    y_ref = orc.decompress(want, x.size)
    assert np.array_equal(y.view(np.uint32), y_ref.view(np.uint32))
    P = SC.parts(want)
    outl = np.zeros(x.size, bool)
    outl[P["idx"]] = True
    step = 1 << 24
    for s0 in range(0, x.size, step):  # chunked: fp64 temporaries stay small
        sl = slice(s0, s0 + step)
        keep = ~outl[sl]
        err = np.abs(x[sl][keep].astype(np.float64) - y[sl][keep].astype(np.float64))
        assert err.max(initial=0.0) <= h["eb"]
        assert np.array_equal(y[sl].view(np.uint32)[~keep], x[sl].view(np.uint32)[~keep])
    return h


@pytest.mark.parametrize("name", ["sine1m", "field256x384x384", "field512cube_spikes", "series2p28",
                                  "noise_zero_ramp2p30"])
def test_standard_workload(orc, name):
    x = WL.standard(name)
    o = WL.options_of(name)
    block = o.pop("block")
    h = _full_check(orc, x, block, **o)
    print(f"{name}: ratio {4 * x.size / h['total']:.3f} m={h['m']} eb={h['eb']:.3e}")


@pytest.mark.parametrize("block", WL.SWEEP_BLOCK)
def test_series_sweep(orc, block):
    """The 1-D 2^28 series over rel 1e-2..1e-6 x block 32..256 (20 points):
    stream parity at every point, full decode parity at rel 1e-4."""
    import torch
    from tests.gpu_util import GpuCodec

    x = WL.standard("series2p28")
    xd = torch.from_numpy(x).cuda()
    for rel in WL.SWEEP_REL:
        if rel == 1e-4:
            _full_check(orc, x, block, rel=rel)
            continue
        want = orc.compress(x, block, rel=rel)
        with GpuCodec(x.size, block, rel=rel) as g:
            st, out, nbytes, _ = g.compress(xd)
            assert st == 0 and nbytes == want.size
            assert np.array_equal(out[:nbytes].cpu().numpy(), want), (block, rel)
