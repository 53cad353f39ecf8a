"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2).

The hot path shards by image with no data-path collective; the only cross-rank
operations are the barrier around the timed region and the max over ranks of the
measured time.  These run here on CPU processes; no GPU is involved.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    first, n = bench.shard_images(rank, world, 8)
    dist.barrier()
    mx = bench.max_over_ranks(1.5 + rank, world)
    out[rank] = (first, n, mx)
    dist.destroy_process_group()


def test_two_ranks_shard_disjoint_and_take_max():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    firsts = sorted(out[r][0] for r in range(world))
    assert firsts == [0, 8] and all(out[r][1] == 8 for r in range(world))
    assert all(out[r][2] == 2.5 for r in range(world))


def test_shard_rejects_bad_rank():
    import bench
    with pytest.raises(ValueError):
        bench.shard_images(2, 2, 8)


def test_reference_arm_other_ranks_do_nothing(capsys):
    import bench
    bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1"]), 1, 2)
    assert capsys.readouterr().out == ""
