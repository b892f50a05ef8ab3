"""Replicas on two ranks (gloo, CPU): each rank draws its own batch, runs the
path's oracle on it with no collective in the data path, and the timing
reduction takes the maximum over ranks; the job's throughput counts both
ranks' units.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth
from kv_cache_compression_layer_b200.replicas import job_throughput, max_over_ranks, replica_seed


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist

    import oracle as orc
    from kv_cache_compression_layer_b200.replicas import init_group

    assert init_group("gloo", world, timeout_s=60.0)
    try:
        base = synth.small("tiny", L=(512,))
        cfg = base.with_(seed=replica_seed(base.seed, rank))
        bt = synth.make_batch(cfg, steps=2)
        # the rank's own path, no exchange with the other rank
        s = orc.score(bt.qwin, bt.K, bt.L_rows)
        s_hat, _ = orc.sss(s, bt.L_rows, cfg.alpha, cfg.rho)
        b = orc.allocate(bt.S, cfg.L, cfg.w, cfg.budget_pct, cfg.r).reshape(-1)
        idx = orc.select(s_hat, bt.L_rows, cfg.w, b.tolist())
        fingerprint = float(np.concatenate([x.astype(np.float64) for x in idx]).sum() + s.sum())
        # the timing reduction: a per-rank "step time" that differs by rank
        ms_rank = 2.0 + rank
        ms_max = max_over_ranks(ms_rank, world)
        fps = [None] * world
        dist.all_gather_object(fps, fingerprint)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([ms_max, job_throughput(sum(cfg.L), world, ms_max), fps[0], fps[1], fingerprint]))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    # both ranks agree on the job's step time: the slower rank's
    assert r0[0] == r1[0] == 3.0
    # throughput counts both ranks' tokens over the slowest rank's time
    assert r0[1] == pytest.approx(2 * 512 / 3e-3)
    # each rank worked on its own batch (different seeds give different results)
    assert r0[2] == r0[4] and r1[3] == r1[4] and r0[2] != r0[3]


def test_replica_seed_and_throughput():
    assert replica_seed(7, 0) == 7 and replica_seed(7, 3) == 10
    assert max_over_ranks(1.5, 1) == 1.5
    assert job_throughput(6000, 4, 2.0) == pytest.approx(4 * 6000 / 2e-3)
    with pytest.raises(ValueError):
        job_throughput(1, 1, 0.0)
