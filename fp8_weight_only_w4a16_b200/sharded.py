"""Column-parallel (output-sharded) weight-only GEMM over torch.distributed.

Output channels of y = x . W^T are independent, so W can be split by rows
across the ranks of a process group: rank r holds rows [start_r, stop_r) of W
(packed on its own GPU), computes y[:, start_r:stop_r] with the library's
kernel, and an all-gather assembles y on every rank.  x is replicated (it is
at most a few hundred KB at M <= 8).  The pages' model is served this way
across four GPUs (taozi.news article, section "v1.1 的关键改进"; the
aiwitness.kr post, section "내가 실제로 만든 것"); this module supplies the
shard boundaries and the gather, the GEMM itself is the library's.

torch.distributed is plumbing here: NCCL over NVLink on GPUs, gloo in the
CPU tests of the host logic.
"""
from __future__ import annotations

TILE_ROWS = 128   # shard boundaries fall on whole 128-row tiles of the packed layout


def shard_rows(N: int, world: int, rank: int, align: int = TILE_ROWS) -> tuple[int, int]:
    """Rows [start, stop) of W owned by `rank`: contiguous ranges in rank order,
    boundaries on multiples of `align` (except the end, N), sizes as equal as
    the alignment allows.  A rank may own no rows when N < world * align."""
    if N <= 0 or world <= 0 or not 0 <= rank < world or align <= 0:
        raise ValueError("bad shard arguments")
    units = (N + align - 1) // align
    lo = units * rank // world
    hi = units * (rank + 1) // world
    return min(N, lo * align), min(N, hi * align)


def gather_columns(y_local, N: int, group=None):
    """All-gather the ranks' column blocks y[:, start_r:stop_r] (each [M, width_r],
    same dtype and device) into the full y [M, N] on every rank.  Blocks may
    differ in width (the last shard is ragged); they travel padded to the widest
    one and are trimmed back in rank order.

    Device tensors are gathered in the order of torch's current stream (NCCL
    waits on it).  A gloo group moves host tensors only, so device blocks are
    staged through host memory there and the result is returned on y_local's
    device."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    M = y_local.shape[0]
    widths = [shard_rows(N, world, r)[1] - shard_rows(N, world, r)[0] for r in range(world)]
    rank = dist.get_rank(group)
    if y_local.shape[1] != widths[rank]:
        raise ValueError("y_local must hold this rank's %d columns" % widths[rank])
    staged = y_local.is_cuda and dist.get_backend(group) == "gloo"
    where = torch.device("cpu") if staged else y_local.device
    w_max = max(widths)
    send = torch.zeros((M, w_max), dtype=y_local.dtype, device=where)
    send[:, :widths[rank]] = y_local
    recv = [torch.empty((M, w_max), dtype=y_local.dtype, device=where) for _ in range(world)]
    dist.all_gather(recv, send, group=group)
    y = torch.cat([recv[r][:, :widths[r]] for r in range(world)], dim=1)
    return y.to(y_local.device) if staged else y


def column_parallel_gemm(x, w_shard, N: int, group=None, out_dtype=None, workspace=None, stream=None):
    """y [M, N] = x . W^T on every rank, each rank holding the packed rows
    shard_rows(N, world, rank) of W as `w_shard` (PackedNVFP4 or PackedFP8).

    With `stream` given, the local GEMM, the staging copies and the all-gather
    are all issued on that stream (torch's current stream is switched to it for
    the call), so the gather reads the GEMM's output only after the kernel has
    written it; x must be ready in that stream's order, and the returned y is
    ready in it too.  Without `stream`, everything runs on the current stream."""
    import contextlib

    import torch
    import torch.distributed as dist

    from . import gemm

    world, rank = dist.get_world_size(group), dist.get_rank(group)
    start, stop = shard_rows(N, world, rank)
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        if stop == start:   # N < world * 128: this rank owns no rows
            y_local = torch.empty((x.shape[0], 0), dtype=out_dtype or torch.float16, device=x.device)
        else:
            if w_shard is None or w_shard.N != stop - start:
                raise ValueError("w_shard must hold rows [%d, %d) of W" % (start, stop))
            y_local = gemm(x, w_shard, out_dtype=out_dtype, workspace=workspace)
        return gather_columns(y_local, N, group)
