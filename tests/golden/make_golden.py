"""Write tests/golden/oracle_streams.json: small seeded inputs and the
sha256 of the stream the CPU oracle produces for each.

This script calls only the oracle (and the seeded workload generators).
It pins the oracle's output against accidental change: a change to the
oracle's arithmetic that alters these streams must be justified by a reading
of the method and the file regenerated with

    python -m tests.golden.make_golden
"""
import json
import os

import numpy as np

from error_bounded_lossy_encode_b200 import workloads as WL

HERE = os.path.dirname(os.path.abspath(__file__))

CASES = [
    dict(name="sine_4097_rel1e-3_b128", gen="sine", n=4097, seed=0, block=128, mode="rel", bound=1e-3),
    dict(name="edge_20011_rel1e-3_b32", gen="edge", n=20011, seed=1, block=32, mode="rel", bound=1e-3),
    dict(name="edge_9000_abs1e-2_b64", gen="edge", n=9000, seed=2, block=64, mode="abs", bound=1e-2),
    dict(name="field_12x16x20_rel1e-4_b256", gen="field", shape=[12, 16, 20], seed=1, block=256, mode="rel",
         bound=1e-4),
    dict(name="spikes_16x16x16_rel1e-3_b64", gen="spikes", shape=[16, 16, 16], seed=2, block=64, mode="rel",
         bound=1e-3),
    dict(name="nzr_65536_abs1e-7_b128", gen="nzr", n=65536, seed=4, block=128, mode="abs", bound=1e-7),
    dict(name="empty_b64", gen="edge", n=0, seed=0, block=64, mode="rel", bound=1e-3),
]


def case_input(c):
    if c["gen"] == "sine":
        return WL.sine_noise(c["n"], c["seed"])
    if c["gen"] == "edge":
        return WL.edge_mix(c["n"], c["seed"])
    if c["gen"] == "field":
        return WL.kfield(tuple(c["shape"]), c["seed"])
    if c["gen"] == "spikes":
        return WL.with_spikes(tuple(c["shape"]), c["seed"], p_nonfinite=1e-3)
    if c["gen"] == "nzr":
        return WL.noise_zero_ramp(c["n"], c["seed"])
    raise ValueError(c["gen"])


def main():
    import oracle

    out = []
    for c in CASES:
        x = case_input(c)
        s = oracle.compress(x, c["block"], **{c["mode"]: c["bound"]})
        out.append(dict(c, input_sha256=WL.sha256(x), stream_sha256=WL.sha256(s), total=int(s.size)))
    with open(os.path.join(HERE, "oracle_streams.json"), "w") as f:
        json.dump({"written_by": "tests/golden/make_golden.py (CPU oracle only)", "cases": out}, f, indent=1)


if __name__ == "__main__":
    main()
