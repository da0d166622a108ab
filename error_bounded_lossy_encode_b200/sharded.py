"""One array split across processes (one GPU each), coded under one relative
bound: each rank compresses its own contiguous part into its own stream.

The only exchange step of the method is the value range the relative bound
is taken from ("Pipeline specialization internals", Priming: the value-range
scan that resolves the bound before the fused kernel): every rank computes
its part's range with ``eblc_value_range``, one all-reduce combines them
(the minimum of vmin, the maximum of vmax), and every rank compresses its
part with ``eblc_compress_range`` under the combined range.  A second small
exchange (the ranks' stream sizes) gives each rank's offset in a file or
buffer that holds the parts back to back.  Parts are cut at multiples of
the 4096-element chunk, so each part's stream holds exactly the whole
array's chunk records for its chunks ("DevitoComp provider interface",
Validating a private provider: the provider runs under an MPI-run consumer,
one part of the domain per process).

The collectives go through ``torch.distributed`` (NCCL between GPUs, gloo
on the host); every rank takes the same collective steps in the same order.
Nothing here computes any part of the method: the kernels do.
"""
from __future__ import annotations

CHUNK = 4096


def part_bounds(n: int, world: int, rank: int) -> tuple[int, int]:
    """Element range [a, b) of rank's part: contiguous, cut at multiples of
    the 4096-element chunk, chunk counts differing by at most one."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad part request")
    nc = -(-n // CHUNK)
    a = (nc * rank // world) * CHUNK
    b = min(n, (nc * (rank + 1) // world) * CHUNK)
    return min(a, n), b


def combine_ranges(local, group=None):
    """Combine each rank's [vmin, vmax] (a float32 tensor of 2, on the
    collective's device) into the range of the whole array, in place: one
    MAX all-reduce of [-vmin, vmax]."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return local.add_(0.0)
    t = torch.stack([-local[0], local[1]])
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    local[0] = -t[0]
    local[1] = t[1]
    local.add_(0.0)  # -0 reads as +0
    return local


def stream_offsets(nbytes: int, device=None, group=None) -> tuple[int, int]:
    """(offset of this rank's stream, total bytes of all ranks' streams) when
    the streams are laid out back to back in rank order."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return 0, int(nbytes)
    world = dist.get_world_size(group)
    sizes = torch.zeros(world, dtype=torch.int64, device=device)
    sizes[dist.get_rank(group)] = int(nbytes)
    dist.all_reduce(sizes, op=dist.ReduceOp.SUM, group=group)
    s = sizes.cpu().tolist()
    r = dist.get_rank(group)
    return int(sum(s[:r])), int(sum(s))


def compress_part(plan, x_part, out, capacity: int, group=None, stream=None):
    """Compress this rank's part (a CUDA float32 tensor; the plan made for its
    length with a relative bound) under the range of the whole array.
    Returns (status, compressed_bytes, offset, total, range) with the
    combined range as a host pair."""
    import torch

    import error_bounded_lossy_encode_b200 as E

    s = stream or torch.cuda.current_stream()
    ex = E.cuda_exec(s.cuda_stream)
    rng = torch.zeros(2, dtype=torch.float32, device=x_part.device)
    st = E.eblc_value_range(plan, ex, x_part.data_ptr(), rng.data_ptr())
    if st != E.EBLC_OK:
        return st, 0, 0, 0, None
    with torch.cuda.stream(s):
        combine_ranges(rng, group)
    st, nbytes = E.eblc_compress_range(plan, ex, x_part.data_ptr(), rng.data_ptr(), out.data_ptr(), capacity)
    off, total = stream_offsets(nbytes if st == E.EBLC_OK else 0, device=x_part.device, group=group)
    return st, nbytes, off, total, tuple(float(v) for v in rng.cpu())
