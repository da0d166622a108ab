"""Host logic of the benchmark, on CPU: the cross-rank reductions that turn
per-rank timings into the job's numbers (world size 2 over gloo, the same
calls the multi-GPU run makes over NCCL), the JSON line contract, and the
reference arm's rank handling."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import pytest

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # ranks time different amounts; the job time is the slowest rank's
        t = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * rank], world)
        # every rank processed its own replica: bytes add up
        b = bench.sum_over_ranks([4.0 * (1 << 20) * (rank + 1)], world)
        q.put((rank, t, b))
    finally:
        dist.destroy_process_group()


def test_rank_reductions_gloo_world2():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, b in res:
        assert t == [2.0, 5.0, 0.25]
        assert b == [4.0 * (1 << 20) * 3]


def test_single_rank_reductions_are_identity():
    assert bench.max_over_ranks([3.0, 1.0], 1) == [3.0, 1.0]
    assert bench.sum_over_ranks([2.5], 1) == [2.5]


class _Args:
    steps = 4
    warmup = 3
    workload = "field512cube_spikes"
    elements = None
    no_cpu_baseline = True
    rel = None
    abs = None
    block = None
    codec = "block"
    chunk = 16384
    lorenzo = "1d"
    coder = "rze"


def test_report_line_contract(monkeypatch):
    """One JSON line with every key the benchmark contract names; value is the
    whole job's input bytes of one step over the slowest rank's median step
    (compress + decompress API calls), value_best over its best step."""
    n, nbytes, world = 1 << 20, 600_000, 2
    T = {"step": 0.006, "step_best": 0.005, "comp": 0.004, "dec": 0.002, "comp_dev": 0.0035, "dec_dev": 0.0018}
    kern = {"range": [0.1] * 4, "encode": [0.6] * 4, "decode": [0.5] * 4}
    e2e = {"value": 12.0, "unit": "GB/s", "h2d_bytes_per_step": 4 * n + nbytes, "d2h_bytes_per_step": nbytes + 4 * n}
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}
    step_bytes = 4.0 * n * world
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.report(_Args, world, n, nbytes, T, step_bytes, kern, e2e, 3, clk, np.zeros(n, np.float32), 64, "rel",
                     1e-3)
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["n_gpus"] == world and d["scaling"] == "weak" and d["higher_is_better"] is True
    assert d["value"] == pytest.approx(step_bytes / T["step"] / 1e9, abs=0.006)
    assert d["value_best"] == pytest.approx(step_bytes / T["step_best"] / 1e9, abs=0.006)
    assert d["ms_per_step"] == pytest.approx(1e3 * T["step"], rel=1e-3)
    assert "l2" in d["config"]
    assert d["config"]["workload"] == "field512cube_spikes"
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["kernel"] == "encode" and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], abs=1e-4)
    assert d["gpu_launches"] == 3 * _Args.steps
    assert d["ratio"] == pytest.approx(4.0 * n / nbytes, rel=1e-4)


def test_reference_arm_other_ranks_exit_quietly(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(_Args) == 0
    assert buf.getvalue() == ""


def test_both_arms_report_the_same_config():
    """The reference arm times the plain oracle on this arm's workload: its
    config is the one this arm prints (same workload, n, block, bound)."""
    a = bench.workload_config(_Args, 1 << 20, 64, "rel", 1e-3, 1)
    b = bench.workload_config(_Args, 1 << 20, 64, "rel", 1e-3, 1)
    assert a == b and a["workload"] == "field512cube_spikes" and a["n"] == 1 << 20


def test_host_info_names_cpu_and_cores():
    h = bench.host_info()
    assert h["cores_available"] >= 1
    assert "cpu_model" in h


def test_codec_variants_name_themselves():
    """--codec chunked and --lorenzo nd: the plan options and the config say
    which codec or predictor was timed (both arms build the config alike)."""
    class Ch(_Args):
        codec, chunk = "chunked", 4096

    class Nd(_Args):
        lorenzo = "nd"

    c = bench.workload_config(Ch, 1 << 20, 64, "rel", 1e-3, 1)
    assert c["codec"] == "chunked" and c["chunk_bytes"] == 4096 and c["coder"] == "rze" and "block" not in c
    assert bench.options_string(64, "rel", 1e-3, False, "chunked", 4096) == \
        "rel=0.001,codec=chunked,chunk=4096,coder=rze"
    d = bench.workload_config(Nd, 1 << 27, 64, "rel", 1e-3, 1)
    assert d["lorenzo"] == "nd" and d["dims"] == [512, 512, 512] and d["block"] == 64
    assert bench.options_string(64, "rel", 1e-3, False, "block", 16384, "nd") == "rel=0.001,block=64,lorenzo=nd"
    assert bench.variant_suffix(Ch) == "_chunked4096" and bench.variant_suffix(Nd) == "_nd"
    assert bench.variant_suffix(_Args) == ""
