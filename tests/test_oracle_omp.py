"""The all-core oracle build (oracle/eblc_oracle_omp.c, the benchmark's
all-core CPU baseline) runs the plain oracle's own steps over chunks in
parallel: its streams and reconstructions must be byte-identical to the
plain oracle's.  CPU only."""
import numpy as np
import pytest

from error_bounded_lossy_encode_b200 import workloads as WL

CASES = [
    ("spiky field rel", lambda: WL.with_spikes((32, 64, 64), 2, p_nonfinite=1e-3), 64, {"rel": 1e-3}),
    ("noise/zeros/ramp abs", lambda: WL.noise_zero_ramp(300008, 4), 128, {"abs": 1e-7}),
    ("edge mix ragged", lambda: WL.edge_mix(70001, 3), 32, {"rel": 1e-2}),
    ("field block 256", lambda: WL.kfield((24, 40, 48), 1), 256, {"rel": 1e-4}),
    ("empty", lambda: np.zeros(0, np.float32), 64, {"rel": 1e-3}),
    ("single element", lambda: np.array([np.nan], np.float32), 32, {"abs": 0.5}),
]


@pytest.mark.parametrize("name,make,block,bound", CASES, ids=[c[0] for c in CASES])
def test_omp_build_matches_oracle(orc, name, make, block, bound):
    x = make()
    want = orc.compress(x, block, **bound)
    got = orc.compress_omp(x, block, **bound)
    assert got.size == want.size and np.array_equal(got, want)
    y_ref = orc.decompress(want, x.size)
    y = orc.decompress_omp(want, x.size)
    assert np.array_equal(y.view(np.uint32), y_ref.view(np.uint32))


def test_omp_build_rejects_corrupt_stream(orc):
    x = WL.edge_mix(9000, 1)
    s = orc.compress(x, 64, rel=1e-3).copy()
    hdr = orc.parse_header(s)
    s[hdr["width_off"]] = 40  # a width above 32
    with pytest.raises(orc.OracleError):
        orc.decompress_omp(s, x.size)
