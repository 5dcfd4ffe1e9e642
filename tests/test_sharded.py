"""Column-parallel sharding (fp8_weight_only_w4a16_b200.sharded): shard
boundaries, and the gather of the ranks' column blocks, as gloo ranks on CPU.

Each rank computes its block y[:, start:stop] with the float64 oracle on its
own rows of W (output channels are independent, and the oracle's rows do not
depend on which other rows it is given); the gathered y must equal the
oracle's full result bit for bit, on every rank."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp8_weight_only_w4a16_b200.sharded import gather_columns, shard_rows


@pytest.mark.parametrize("N,world", [(5120, 2), (5120, 3), (34816, 8), (300, 4), (151936, 8), (100, 3)])
def test_shard_rows_partition(N, world):
    spans = [shard_rows(N, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == N
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0 and a0 <= a1
    for a0, a1 in spans:
        assert a0 % 128 == 0 and (a1 % 128 == 0 or a1 == N)
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(s for s in sizes) <= 128 or N < world * 128


def test_shard_rows_rejects_bad_arguments():
    with pytest.raises(ValueError):
        shard_rows(0, 2, 0)
    with pytest.raises(ValueError):
        shard_rows(128, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, N, K, M, out):
    import oracle
    import synthetic_inputs as si

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        codes, scales = si.nvfp4_weights(N, K, seed=3, cfg_id=71)
        x = si.activations(M, K, seed=3, cfg_id=71)
        start, stop = shard_rows(N, world, rank)
        y_local, _ = oracle.nvfp4_gemm(x, codes[start:stop], scales[start:stop], 0.5)
        y = gather_columns(torch.from_numpy(y_local.astype(np.float32)), N)
        full, _ = oracle.nvfp4_gemm(x, codes, scales, 0.5)
        out[rank] = bool(np.array_equal(y.numpy(), full.astype(np.float32)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world,N", [(2, 640), (3, 300)])
def test_gather_columns_reassembles_the_full_output_gloo(world, N):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), N, 512, 3, out), nprocs=world, join=True,
                       start_method="spawn")
    assert all(out[r] for r in range(world)), dict(out)
