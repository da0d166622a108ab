"""Host side of the sharded compress, on CPU over gloo (world size 2 and 3):
part boundaries, the range all-reduce and the stream offsets, with the CPU
oracle standing in for the GPU codec (the GPU kernels of the same flow are
checked in test_gpu_sharded.py).  Each rank's stream must equal the oracle's
stream of its part under the whole array's range, and the rank offsets must
lay the streams out back to back."""
import os
import socket

import numpy as np
import pytest

from error_bounded_lossy_encode_b200 import sharded as SH
from error_bounded_lossy_encode_b200 import workloads as WL


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _x():
    return np.concatenate([WL.with_spikes((8, 32, 64), 2, p_nonfinite=1e-3), WL.edge_mix(3 * 4096 + 77, 5)])


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _x()
        a, b = SH.part_bounds(x.size, world, rank)
        part = x[a:b]
        lo, hi, _ = oracle.value_range(part)
        rng = torch.tensor([lo, hi], dtype=torch.float32)
        SH.combine_ranges(rng)
        s = oracle.compress_range(part, 64, 1e-3, float(rng[0]), float(rng[1]))
        off, total = SH.stream_offsets(s.size)
        q.put((rank, a, b, float(rng[0]), float(rng[1]), s.tobytes(), off, total))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_exchange_gloo(orc, world):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = _x()
    lo, hi, _ = orc.value_range(x)
    expect_off = 0
    for rank, a, b, glo, ghi, s, off, total in res:
        assert (a, b) == SH.part_bounds(x.size, world, rank)
        assert glo == np.float32(lo) and ghi == np.float32(hi)
        want = orc.compress_range(x[a:b], 64, 1e-3, lo, hi)
        assert np.array_equal(np.frombuffer(s, np.uint8), want)
        assert off == expect_off
        expect_off += len(s)
    assert all(r[-1] == expect_off for r in res)


def test_part_bounds_cover_the_array_at_chunk_cuts():
    for n in (0, 1, 4095, 4096, 4097, 10 * 4096 + 3, 12345678):
        for world in (1, 2, 3, 8):
            parts = [SH.part_bounds(n, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            for (a0, b0), (a1, b1) in zip(parts, parts[1:]):
                assert b0 == a1
            for a, b in parts:
                assert a % 4096 == 0 and a <= b
            sizes = [-(-(b - a) // 4096) for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        SH.part_bounds(10, 2, 2)


def test_combined_range_canonical_zero():
    """-0 from the negation in the all-reduce never reaches the header."""
    import torch

    r = torch.tensor([0.0, 0.0])
    t = torch.stack([-r[0], r[1]])
    r[0] = -t[0]
    r.add_(0.0)
    assert not np.signbit(r[0].item())
