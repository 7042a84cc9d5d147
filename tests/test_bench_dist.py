"""bench.py's multi-rank host logic on CPU: two gloo ranks on 127.0.0.1 (the
GPU path launches one process per GPU the same way, over NCCL).

Checked: the timed value is the max over ranks on every rank, the barrier
releases both ranks, replicas draw distinct seeds, and the reference arm
runs on rank 0 only.
"""
import os
import socket
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        mx = bench.max_over_ranks(1.5 + 2.0 * rank, w)
        bench.barrier(w)
        out[rank] = (r, w, local, mx, bench.replica_seed(r))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        for p in procs:
            if p.is_alive():
                p.kill()
            assert p.exitcode == 0
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank in range(world):
        r, w, local, mx, seed = res[rank]
        assert (r, w, local) == (rank, world, rank)
        assert mx == 3.5  # the slower rank's time, on both ranks
    assert res[0][4] != res[1][4]


def test_reference_arm_rank0_only():
    args = types.SimpleNamespace(steps=1, warmup=1)
    assert bench.run_reference(args, rank=1, world=2) is None


def test_song_positions_cover_the_song():
    pos = bench.song_positions(4)
    assert pos == sorted(pos) and 0 <= pos[0] and pos[-1] < bench.SONG_FRAMES
    assert len(set(bench.song_positions(60))) == 60
