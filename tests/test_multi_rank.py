"""Host logic of the N-GPU bench (replicas): every rank times its own replica,
the job's time is the max over ranks, and the value is the aggregate over all
ranks.  Runs as world_size-2 gloo ranks on CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(my_ms, world)
        value = bench.whole_job_gbs(world, bench.step_bytes(), 100, ms)
        out[rank] = (ms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_aggregate_value_gloo():
    world = 2
    out = mp.get_context("spawn").Manager().dict()   # no fork of a threaded process
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == 5.0
    expected = world * bench.step_bytes() * 100 / 5e-3 / 1e9
    assert abs(out[0][1] - expected) < 1e-9 * expected and out[0][1] == out[1][1]


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.whole_job_gbs(1, 10 ** 9, 2, 1000.0) == pytest.approx(2.0)


def test_step_bytes_formula():
    """469 MB per step: five GEMMs at M=1 and at M=8, packed weights + scales + x + y."""
    b = bench.step_bytes()
    w = sum(bench.weight_bytes(s) for s in bench.si.MIXED_LAYER)
    assert w == 3 * (5120 * 5120 * 9 // 16 + 4) + (34816 * 5120 * 9 // 16 + 4) + (5120 * 17408 + 4 * 5120)
    act = sum(M * s.K * 2 + M * s.N * 2 for M in (1, 8) for s in bench.si.MIXED_LAYER)
    assert b == 2 * w + act


def test_kernel_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    """The DRAM traffic record is keyed by the kernel code: a comment or
    whitespace edit keeps the key, a code edit changes it."""
    import shutil

    src = os.path.join(bench.ROOT, "fp8_weight_only_w4a16_b200", "csrc")
    dst = tmp_path / "fp8_weight_only_w4a16_b200" / "csrc"
    dst.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(src, name), dst / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_source_hash()
    layout = dst / "layout.h"
    text = layout.read_text()
    layout.write_text("// a new comment\n" + text.replace("\n", "\n\n", 3) + "/* trailing */\n")
    assert bench.kernel_source_hash() == base
    layout.write_text(text.replace("constexpr int kTileRows = 128;", "constexpr int kTileRows = 64;"))
    assert bench.kernel_source_hash() != base
