"""Benchmark: compress + decompress throughput of float32 input on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline]

One step = one pass of the whole hot path over the workload: value range,
fused encode (one stream), fused decode.  Default workload: the 512^3 k^-3
field with 1 % spikes and 1e-6 NaN/+-Inf (relative bound 1e-3, block 64).
With torchrun (N > 1) every rank compresses its own replica of the workload
(independent arrays, no collective on the data path: weak scaling); the
timing is the max over ranks.

Printed JSON line (rank 0):
  value        GB/s of float32 input per compress + decompress round trip,
               device-resident input: CUDA events on the call's stream around
               each full API call (eblc_compress including its closing
               synchronisation, eblc_decompress), median step of --steps
               (best step in value_best); the L2 is flushed (256 MiB write)
               before every call and the flush is not timed
  e2e          the same through the HOST execution kind (host buffers,
               host<->device copies inside the timed region)
  roofline     the dominant kernel against the measured copy bandwidth
  cpu_baseline the plain single-threaded CPU oracle on a bounded sample of the
               workload; cpu_baseline_all_cores the same oracle steps run over
               chunks on all host cores (OpenMP build); host names the CPU
--impl reference times the plain CPU oracle itself (the only reference there
is) on the whole workload, with the same config as this arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "compress & decompress GB/s of fp32 input on 1 B200, % of HBM roofline; ratio"
DEFAULT_WORKLOAD = "field512cube_spikes"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
CPU_SAMPLE_ELEMS = 1 << 24  # 64 MiB of the workload for the CPU oracle legs


# ----------------------------------------------------------------------------------------------
# rank plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), ws, int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of a list of floats over all ranks (identity for one rank)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def sum_over_ranks(values, world: int, device=None):
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.cpu().tolist()


# ----------------------------------------------------------------------------------------------
# clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [p.strip() for p in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------------------------
# workload

def workload(name: str, elements: int | None = None, rel=None, abs_=None, block=None):
    """The named standard workload and its options; rel / abs_ / block override them."""
    from error_bounded_lossy_encode_b200 import workloads as WL

    x = WL.standard(name)
    if elements:
        x = np.ascontiguousarray(x[:elements])
    o = WL.options_of(name)
    blk = o.pop("block")
    mode, bound = next(iter(o.items()))
    if rel is not None:
        mode, bound = "rel", rel
    if abs_ is not None:
        mode, bound = "abs", abs_
    return x, (block or blk), mode, bound


def workload_config(args, n, block, mode, bound, world):
    """The `config` both arms report for the same workload."""
    c = {"workload": args.workload if not args.elements else f"{args.workload}[:{n}]", "n": int(n)}
    if args.codec == "chunked":
        c.update(codec="chunked", chunk_bytes=args.chunk, coder=args.coder)
    else:
        c["block"] = block
        if args.lorenzo == "nd":
            c.update(lorenzo="nd", dims=list(nd_dims(args)))
    c.update({mode: bound, "parallelism": f"replicas{world}",
              "l2": "flushed (256 MiB write, untimed) before every GPU compress and decompress call"})
    return c


def nd_dims(args):
    """The workload's own 2-D / 3-D shape for lorenzo=nd (whole arrays only)."""
    from error_bounded_lossy_encode_b200 import workloads as WL

    d = WL.dims_of(args.workload)
    if len(d) < 2 or args.elements:
        raise SystemExit("--lorenzo nd needs a whole 2-D or 3-D workload")
    return d


def variant_suffix(args) -> str:
    """'' for the default codec, else the codec's tag in profile file names."""
    if args.codec == "chunked":
        return f"_chunked{args.chunk}" + ("_rre" if args.coder == "rre" else "")
    return "_nd" if args.lorenzo == "nd" else ""


def host_info():
    """CPU model and the cores this process may run on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        cores = os.cpu_count()
    return {"cpu_model": model, "cores_available": cores}


def options_string(block, mode, bound, timing=False, codec="block", chunk=16384, lorenzo="1d", coder="rze"):
    if codec == "chunked":
        o = f"{mode}={bound!r},codec=chunked,chunk={chunk},coder={coder}"
    else:
        o = f"{mode}={bound!r},block={block}" + (",lorenzo=nd" if lorenzo == "nd" else "")
    return o + (",timing=1" if timing else "")


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha(kernel: str) -> str:
    csrc = os.path.join(ROOT, "error_bounded_lossy_encode_b200", "csrc")
    h = hashlib.sha256()
    for f in (f"{kernel}.cu", "common.cuh", "kernels.h"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload_name}.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_sha") != kernel_source_sha(kernel):
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------------------------
# CPU oracle legs

def cpu_oracle_sample(x, block, mode, bound, repeats=1, all_cores=False, elems=CPU_SAMPLE_ELEMS, codec="block",
                      chunk=16384, dims=None, coder="rze"):
    """Time the CPU oracle (compress + decompress) on the first `elems`
    elements: the plain single-threaded oracle, or (all_cores) the OpenMP
    build of the same steps (block codec, 1-D Lorenzo).  With dims (lorenzo
    nd) the sample is whole leading slabs of the array."""
    import oracle

    oracle.build()
    if all_cores and (codec != "block" or dims):
        return None
    s = x[:elems]
    if codec == "chunked":
        comp = lambda v, **b: oracle.compress_chunked(v, chunk, coder=coder, **b)
        decomp = oracle.decompress
    elif dims:
        slab = int(np.prod(dims[1:]))
        edge = 16 if len(dims) == 3 else 64  # whole bricks along the slowest axis
        k = max(edge, min(dims[0], elems // slab) // edge * edge)
        s = x[:k * slab]
        comp = lambda v, **b: oracle.compress_lorenzo(v.reshape((k,) + tuple(dims[1:])), block, **b)
        decomp = oracle.decompress
    else:
        comp0, decomp = (oracle.compress_omp, oracle.decompress_omp) if all_cores else \
            (oracle.compress, oracle.decompress)
        comp = lambda v, **b: comp0(v, block, **b)
    t_c = t_d = 0.0
    for _ in range(repeats):
        t0 = time.perf_counter()
        stream = comp(s, **{mode: bound})
        t1 = time.perf_counter()
        decomp(stream, s.size)
        t2 = time.perf_counter()
        t_c += t1 - t0
        t_d += t2 - t1
    gbs = repeats * 4 * s.size / (t_c + t_d) / 1e9
    cores = oracle.omp_threads() if all_cores else 1
    what = f"the oracle's steps run over chunks with OpenMP on {cores} threads" if all_cores else \
        "single-threaded plain C oracle" + (f", chunked codec ({chunk}-byte chunks, {coder})" if codec == "chunked" else
                                            ", multi-dimensional Lorenzo" if dims else "")
    part = "the whole workload" if s.size == x.size else f"first {s.size} elements ({4 * s.size >> 20} MiB) of the workload"
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle" if not all_cores else "oracle (all-core OpenMP build)",
            "sample": f"{part}, compress+decompress, {what}",
            "elements": int(s.size),
            "compress_gbs": round(repeats * 4 * s.size / t_c / 1e9, 4),
            "decompress_gbs": round(repeats * 4 * s.size / t_d / 1e9, 4)}


REFERENCE_BUDGET_S = 150.0  # wall-time budget of the reference arm's timed steps


def oracle_kwargs(args) -> dict:
    return {"codec": args.codec, "chunk": args.chunk, "coder": args.coder,
            "dims": nd_dims(args) if args.codec == "block" and args.lorenzo == "nd" else None}


def run_reference(args):
    """The plain CPU oracle, timed on this arm's workload and config.  Each
    step compresses and decompresses the whole workload when the steps fit
    the time budget (estimated from one warm-up on a 2^22-element sample),
    else a leading sample, which the config then names."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    x, block, mode, bound = workload(args.workload, args.elements, args.rel, args.abs, args.block)
    kw = oracle_kwargs(args)
    probe = cpu_oracle_sample(x, block, mode, bound, elems=1 << 22, **kw)
    est_step_s = 4.0 * x.size / (probe["value"] * 1e9)
    elems = x.size if est_step_s * args.steps <= REFERENCE_BUDGET_S else \
        max(1 << 22, int(REFERENCE_BUDGET_S / args.steps * probe["value"] * 1e9 / 4) // 4096 * 4096)
    warm = args.warmup if est_step_s * (args.steps + args.warmup) <= 1.5 * REFERENCE_BUDGET_S else 1
    for _ in range(warm):
        cpu_oracle_sample(x, block, mode, bound, elems=min(elems, 1 << 22), **kw)
    t0 = time.perf_counter()
    base = cpu_oracle_sample(x, block, mode, bound, repeats=args.steps, elems=elems, **kw)
    elapsed = time.perf_counter() - t0
    config = workload_config(args, x.size, block, mode, bound, world)
    if base["elements"] < x.size:
        config = dict(config, workload=f"{config['workload']}[:{base['elements']}]", n=int(base["elements"]))
        if kw["dims"]:  # whole leading slabs of the array
            d = list(kw["dims"])
            config["dims"] = [base["elements"] // int(np.prod(d[1:]))] + d[1:]
    line = {"metric": METRIC, "value": base["value"], "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * elapsed / max(1, args.steps), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "impl": "reference",
            "config": config,
            "cpu_baseline": base,
            "host": host_info(),
            "e2e": {"value": base["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------------------
# our arm

def run_ours(args):
    import torch

    import error_bounded_lossy_encode_b200 as E

    rank, world, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    x_np, block, mode, bound = workload(args.workload, args.elements, args.rel, args.abs, args.block)
    n = x_np.size
    kw = oracle_kwargs(args)
    dims = list(kw["dims"]) if kw["dims"] else [n]
    st, plan = E.eblc_plan_create(dims, None, options_string(block, mode, bound, True, args.codec, args.chunk,
                                                              args.lorenzo, args.coder))
    if st != E.EBLC_OK:
        raise RuntimeError("plan_create: " + E.STATUS_NAMES[st])
    _, lim = E.eblc_plan_get_limits(plan)
    cap = lim["max_compressed_bytes"]

    x = torch.from_numpy(x_np).to(dev)
    out = torch.empty(cap, dtype=torch.uint8, device=dev)
    y = torch.empty(n, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ex = E.cuda_exec(stream.cuda_stream)
    sc = E.eblc_sidecar_t()
    # [range,] encode (chunked: encode, scan, gather), finish; decode
    launches_per_step = (1 if mode == "rel" else 0) + (3 if args.codec == "chunked" else 1) + 1 + 1

    def step(timed):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        st, nbytes = E.eblc_compress(plan, ex, x.data_ptr(), out.data_ptr(), cap, sc)
        e1.record(stream)
        if st != E.EBLC_OK:
            raise RuntimeError("compress: " + E.STATUS_NAMES[st])
        _, kc = E.eblc_plan_kernel_times(plan)
        kc = [(("compress_call" if k == "call" else k), ms, l) for k, ms, l in kc]
        flush.fill_(2)
        e2.record(stream)
        st = E.eblc_decompress(plan, ex, out.data_ptr(), nbytes, sc, y.data_ptr())
        e3.record(stream)
        if st != E.EBLC_OK:
            raise RuntimeError("decompress: " + E.STATUS_NAMES[st])
        _, kd = E.eblc_plan_kernel_times(plan)
        kd = [(("decompress_call" if k == "call" else k), ms, l) for k, ms, l in kd]
        return e0, e1, e2, e3, nbytes, {k: ms for k, ms, _ in kc + kd}

    for _ in range(max(3, args.warmup)):
        step(False)
    torch.cuda.synchronize()
    if E.eblc_check(plan, ex) != E.EBLC_OK:
        raise RuntimeError("device reported an error during warm-up")

    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    recs = [step(True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None

    # CUDA events on the call's stream around each full API call (compress
    # includes its closing synchronisation and readback): per step, seconds
    comp_api = [r[0].elapsed_time(r[1]) / 1e3 for r in recs]
    dec_api = [r[2].elapsed_time(r[3]) / 1e3 for r in recs]
    steps_api = [c + d for c, d in zip(comp_api, dec_api)]
    # the library's own events, first launch to last device operation of the call
    comp_dev = [r[5]["compress_call"] / 1e3 for r in recs]
    dec_dev = [r[5]["decompress_call"] / 1e3 for r in recs]
    nbytes = recs[-1][4]
    kern = {}
    for r in recs:
        for k, ms in r[5].items():
            if not k.endswith("_call"):
                kern.setdefault(k, []).append(ms)
    med = lambda v: float(np.median(v))
    T = dict(zip(["step", "step_best", "comp", "dec", "comp_dev", "dec_dev"],
                 max_over_ranks([med(steps_api), min(steps_api), med(comp_api), med(dec_api), med(comp_dev),
                                 med(dec_dev)], world, dev)))
    step_bytes = sum_over_ranks([4.0 * n], world, dev)[0]

    graph = run_graph_compress(E, plan, x, out, cap, flush, nbytes, args, world, dev) if args.codec == "block" \
        else {"error": "the chunked codec has its synchronous calls only"}

    # e2e: HOST execution kind, pinned host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(E, plan, x_np, cap, args, world, dev)
    if rank == 0:
        report(args, world, n, nbytes, T, step_bytes, kern, e2e, launches_per_step, clk, x_np, block, mode, bound,
               graph)
    E.eblc_plan_destroy(plan)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def run_sharded(args):
    """One array split across the ranks (chunk-aligned contiguous parts, one
    per GPU), each step: every rank's value range, one NCCL all-reduce of the
    ranges, each rank's compress under the combined range, the stream-size
    exchange, then each rank's decompress.  Strong scaling: the whole job
    processes the workload once per step.  CUDA events around the calls,
    median step, max over ranks."""
    import torch

    import error_bounded_lossy_encode_b200 as E
    from error_bounded_lossy_encode_b200 import sharded as SH

    rank, world, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    x_np, block, mode, bound = workload(args.workload, args.elements, args.rel, args.abs, args.block)
    if mode != "rel":
        raise SystemExit("--sharded needs a relative bound (the range all-reduce is its only exchange)")
    a, b = SH.part_bounds(x_np.size, world, rank)
    part = np.ascontiguousarray(x_np[a:b])
    st, plan = E.eblc_plan_create([part.size], None, options_string(block, mode, bound))
    if st != E.EBLC_OK:
        raise RuntimeError("plan_create: " + E.STATUS_NAMES[st])
    _, lim = E.eblc_plan_get_limits(plan)
    cap = lim["max_compressed_bytes"]
    x = torch.from_numpy(part).to(dev)
    out = torch.empty(cap, dtype=torch.uint8, device=dev)
    y = torch.empty(max(part.size, 1), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ex = E.cuda_exec(stream.cuda_stream)

    def step():
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush.fill_(1)
        ev[0].record(stream)
        st, nb, off, total, rng = SH.compress_part(plan, x, out, cap)
        ev[1].record(stream)
        if st != E.EBLC_OK:
            raise RuntimeError("compress_part: " + E.STATUS_NAMES[st])
        flush.fill_(2)
        ev[2].record(stream)
        if E.eblc_decompress(plan, ex, out.data_ptr(), nb, None, y.data_ptr()) != E.EBLC_OK:
            raise RuntimeError("decompress")
        ev[3].record(stream)
        return ev, nb, total

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    recs = [step() for _ in range(args.steps)]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    steps = [r[0][0].elapsed_time(r[0][1]) / 1e3 + r[0][2].elapsed_time(r[0][3]) / 1e3 for r in recs]
    (t_step,) = max_over_ranks([float(np.median(steps))], world, dev)
    total = recs[-1][2]
    if rank == 0:
        line = {"metric": METRIC, "value": round(4.0 * x_np.size / t_step / 1e9, 2), "unit": "GB/s",
                "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
                "ms_per_step": round(1e3 * t_step, 4), "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": dict(workload_config(args, x_np.size, block, mode, bound, world),
                               parallelism=f"sharded{world}"),
                "timing": "CUDA events around value range + range all-reduce + compress under the combined range + "
                          "size exchange, and around decompress; median step, max over ranks",
                "ratio": round(4.0 * x_np.size / total, 4), "stream_bytes_all_ranks": int(total),
                "gpu_launches": 4 * args.steps}
        print(json.dumps(line), flush=True)
    E.eblc_plan_destroy(plan)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_graph_compress(E, plan, x, out, cap, flush, nbytes, args, world, dev):
    """Compress captured once into a CUDA graph (eblc_compress_async: no host
    synchronisation inside) and replayed; CUDA events around each replay, L2
    flushed before each.  Reported beside the main metric, not in it."""
    import torch

    try:
        d_res = torch.zeros(32, dtype=torch.uint8, device=dev)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            st = E.eblc_compress_async(plan, E.cuda_exec(side.cuda_stream), x.data_ptr(), out.data_ptr(), cap,
                                       d_res.data_ptr())
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        if st != E.EBLC_OK:
            return {"error": "compress_async: " + E.STATUS_NAMES[st]}
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            E.eblc_compress_async(plan, E.cuda_exec(torch.cuda.current_stream().cuda_stream), x.data_ptr(),
                                  out.data_ptr(), cap, d_res.data_ptr())
        ms = []
        for _ in range(args.steps):
            flush.fill_(4)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            ms.append((e0, e1))
        torch.cuda.synchronize()
        r = E.async_result(d_res.cpu().numpy().tobytes())
        del g
        if r["status"] != E.EBLC_OK or r["compressed_bytes"] != nbytes:
            return {"error": f"replay result {r}"}
        t = sum(a.elapsed_time(b) for a, b in ms) / 1e3
        (t,) = max_over_ranks([t], world, dev)
        return {"avg_ms": round(1e3 * t / args.steps, 4), "compress_gbs": round(4.0 * x.numel() * args.steps / t / 1e9, 2),
                "api": "eblc_compress_async captured in a CUDA graph, replayed; CUDA events per replay"}
    except Exception as ex:  # capture not available: report why, keep the run
        return {"error": str(ex)[:200]}


def run_e2e(E, plan, x_np, cap, args, world, dev):
    import torch

    n = x_np.size
    xh = torch.from_numpy(x_np).pin_memory()
    sh = torch.empty(cap, dtype=torch.uint8).pin_memory()
    yh = torch.empty(n, dtype=torch.float32).pin_memory()
    hx = E.host_exec()
    sc2 = E.eblc_sidecar_t()
    for _ in range(2):
        E.eblc_compress(plan, hx, xh.data_ptr(), sh.data_ptr(), cap, sc2)
    t_e2e = 0.0  # device time: each HOST-kind call's events span its copies in and out
    t_wall = 0.0
    e2e_steps = max(1, min(args.steps, 5))
    for _ in range(e2e_steps):
        t0 = time.perf_counter()
        st, nb2 = E.eblc_compress(plan, hx, xh.data_ptr(), sh.data_ptr(), cap, sc2)
        _, kc = E.eblc_plan_kernel_times(plan)
        st2 = E.eblc_decompress(plan, hx, sh.data_ptr(), nb2, sc2, yh.data_ptr())
        _, kd = E.eblc_plan_kernel_times(plan)
        t_wall += time.perf_counter() - t0
        if st != E.EBLC_OK or st2 != E.EBLC_OK:
            raise RuntimeError("host-kind call failed")
        t_e2e += (dict((k, ms) for k, ms, _ in kc)["call"] + dict((k, ms) for k, ms, _ in kd)["call"]) / 1e3
    t_e2e, t_wall = max_over_ranks([t_e2e, t_wall], world, dev)
    e2e_bytes = sum_over_ranks([4.0 * n * e2e_steps], world, dev)[0]
    return {"value": round(e2e_bytes / t_e2e / 1e9, 3), "unit": "GB/s",
            "h2d_bytes_per_step": int(4 * n + nb2), "d2h_bytes_per_step": int(nb2 + 4 * n),
            "host_wall_gbs": round(e2e_bytes / t_wall / 1e9, 3),
            "api": "eblc_compress + eblc_decompress, EBLC_EXECUTION_HOST, pinned host buffers; CUDA events "
                   "from each call's input copy to its output copy, max over ranks"}


def report(args, world, n, nbytes, T, step_bytes, kern, e2e, launches_per_step, clk, x_np, block, mode, bound,
           graph=None):
    peak, peak_kind = measured_peak()
    ratio = 4.0 * n / nbytes
    algo = {"range": 4.0 * n, "encode": 4.0 * n + nbytes, "decode": 4.0 * n + nbytes}
    kstats = {}
    for k, v in kern.items():
        avg_ms = float(np.mean(v))
        ach = algo[k] / (avg_ms / 1e3) / 1e9
        kstats[k] = {"avg_ms": round(avg_ms, 4), "median_ms": round(float(np.median(v)), 4), "launches": len(v),
                     "algorithmic_bytes": int(algo[k]), "achieved_gbs": round(ach, 1),
                     "frac_of_measured_peak": round(ach / peak, 4)}
    if args.codec == "chunked":
        kstats["encode"]["what"] = "chunk_encode + chunk_scan + chunk_gather (one timing mark around the three)"
    dom = max(kstats, key=lambda k: kstats[k]["avg_ms"])
    traffic = profiled_traffic(dom, args.workload + variant_suffix(args))
    line = {
        "metric": METRIC,
        "value": round(step_bytes / T["step"] / 1e9, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": round(1e3 * T["step"], 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(args, n, block, mode, bound, world),
        "timing": "CUDA events on the call's stream around each full API call (compress includes its closing "
                  "synchronisation); median step, max over ranks",
        "value_best": round(step_bytes / T["step_best"] / 1e9, 2),
        "compress_gbs": round(4.0 * n / T["comp"] / 1e9, 2),
        "decompress_gbs": round(4.0 * n / T["dec"] / 1e9, 2),
        "api_ms_per_step": {"compress": round(1e3 * T["comp"], 4), "decompress": round(1e3 * T["dec"], 4)},
        "device_ms_per_step": {"compress": round(1e3 * T["comp_dev"], 4), "decompress": round(1e3 * T["dec_dev"], 4),
                               "what": "library events: first launch to the last device operation of the call"},
        "ratio": round(ratio, 4),
        "stream_bytes": int(nbytes),
        "hbm_frac_8tbs": {"compress": round((4.0 * n + nbytes) / T["comp"] / 8e12, 4),
                          "decompress": round((4.0 * n + nbytes) / T["dec"] / 8e12, 4),
                          "compress_required_bytes": round((8.0 * n + nbytes) / T["comp"] / 8e12, 4)
                          if mode == "rel" else None},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": kstats[dom]["achieved_gbs"], "peak": peak,
                     "peak_kind": f"{peak_kind} copy bandwidth", "unit": "GB/s",
                     "frac": kstats[dom]["frac_of_measured_peak"], "traffic": traffic},
        "kernels": kstats,
        "e2e": e2e,
        "graph_compress": graph,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if n <= (1 << 22):
        line["note"] = ("input fits in L2 and each call is a few tens of microseconds: the synchronous compress is "
                        "bound by launch and host synchronisation latency, not HBM (graph_compress shows the "
                        "sync-free form)")
    if not args.no_cpu_baseline:
        kw = oracle_kwargs(args)
        line["cpu_baseline"] = cpu_oracle_sample(x_np, block, mode, bound, **kw)
        allc = cpu_oracle_sample(x_np, block, mode, bound, all_cores=True, **kw)
        line["cpu_baseline_all_cores"] = allc if allc is not None else \
            {"unavailable": "the OpenMP oracle build covers the block codec with the 1-D predictor only"}
        line["host"] = host_info()
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--elements", type=int, default=None, help="use only the first N elements of the workload")
    ap.add_argument("--rel", type=float, default=None, help="override the workload's bound: relative")
    ap.add_argument("--abs", type=float, default=None, help="override the workload's bound: absolute")
    ap.add_argument("--block", type=int, default=None, choices=(32, 64, 128, 256), help="override the block size")
    ap.add_argument("--codec", choices=("block", "chunked"), default="block",
                    help="block: the fused block codec (default); chunked: the chunk-cooperative codec")
    ap.add_argument("--chunk", type=int, choices=(4096, 8192, 16384), default=16384,
                    help="bytes of input per chunk of the chunked codec")
    ap.add_argument("--coder", choices=("rze", "rre"), default="rze",
                    help="zero elimination of the chunked codec: rze (default) or rre")
    ap.add_argument("--lorenzo", choices=("1d", "nd"), default="1d",
                    help="nd: the 2-D / 3-D Lorenzo predictor over the workload's own shape")
    ap.add_argument("--sharded", action="store_true",
                    help="split one array across the ranks (range all-reduce; strong scaling) instead of replicas")
    args = ap.parse_args(argv)
    if args.codec == "chunked" and args.lorenzo == "nd":
        ap.error("--lorenzo nd belongs to the block codec")
    if args.coder != "rze" and args.codec != "chunked":
        ap.error("--coder belongs to the chunked codec")
    if args.sharded and (args.codec != "block" or args.lorenzo != "1d"):
        ap.error("--sharded runs the block codec with the 1-D predictor")
    if args.impl == "reference":
        return run_reference(args)
    if args.sharded:
        return run_sharded(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
