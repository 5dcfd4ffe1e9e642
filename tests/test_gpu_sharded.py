"""Column-parallel GEMM through the CUDA kernel: gloo ranks on one GPU.

Each rank packs its own tile-aligned slice of W's rows (shard_rows), runs
sharded.column_parallel_gemm -- the library's kernel on the local shard, then
the all-gather of the column blocks -- and the gathered y must match the
float64 oracle's full y element by element at the parity tolerance.  The
ranks' kernels are independent launches (no rank waits on another inside a
kernel); the gather goes through host memory because the group is gloo.
Rank 0 passes a side stream, so the stream hand-off between the GEMM and the
gather is exercised.  The shapes cover a ragged last shard, a rank that owns
no rows (N < world * 128), both weight formats and both schedules."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, fmt, N, K, M, split, out):
    import fp8_weight_only_w4a16_b200 as sk
    import synthetic_inputs as si
    from fp8_weight_only_w4a16_b200.sharded import column_parallel_gemm, shard_rows
    from parity import REL_TOL, oracle_fp8, oracle_nvfp4

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        start, stop = shard_rows(N, world, rank)
        x_np = si.activations(M, K, seed=5, cfg_id=72)
        x = torch.from_numpy(x_np).cuda()
        if fmt == "nvfp4":
            codes, scales = si.nvfp4_weights(N, K, seed=5, cfg_id=72)
            w = sk.PackedNVFP4.from_logical(codes[start:stop], scales[start:stop], 0.5) if stop > start else None
            y_ref, bound = oracle_nvfp4(x_np, codes, scales, 0.5)
        else:
            q, s = si.fp8_weights(N, K, seed=5, cfg_id=72)
            w = sk.PackedFP8.from_logical(q[start:stop], s[start:stop]) if stop > start else None
            y_ref, bound = oracle_fp8(x_np, q, s)
        ws = None
        if split and w is not None:
            ws = sk.make_workspace(w.fmt, M, w.N, K)
        side = torch.cuda.Stream() if rank == 0 else None
        if side is not None:
            side.wait_stream(torch.cuda.current_stream())   # x and w were written on the current stream
        y = column_parallel_gemm(x, w, N, out_dtype=torch.float32, workspace=ws, stream=side)
        (side or torch.cuda.current_stream()).synchronize()
        y = y.double().cpu().numpy()
        ok = y.shape == (M, N) and bool(np.all(np.abs(y - y_ref) <= REL_TOL * bound))
        out[rank] = (ok, stop - start, sk.device_error(clear=True))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("fmt,N,K,M,world,split", [
    ("nvfp4", 5120, 1024, 8, 2, True),    # two 2560-row shards, split-K
    ("nvfp4", 300, 1040, 3, 2, False),    # ragged last shard: rows [0, 128) and [128, 300), no split-K
    ("nvfp4", 200, 512, 1, 3, True),      # rank 0 owns no rows
    ("fp8", 640, 1536, 4, 2, True),
])
def test_column_parallel_gemm_matches_oracle(fmt, N, K, M, world, split):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), fmt, N, K, M, split, out), nprocs=world, join=True,
                       start_method="spawn")
    res = dict(out)
    assert sorted(res) == list(range(world)), res
    assert all(res[r][0] for r in range(world)), res
    assert all(res[r][2] == 0 for r in range(world)), res
    assert sum(res[r][1] for r in range(world)) == N
    if N < world * 128:
        assert any(res[r][1] == 0 for r in range(world))
