"""One batch split over ranks (kv_cache_compression_layer_b200.partition):
host checks of the split, and two gloo ranks on CPU that each run their part
of the batch (the library's host-side row and slot accounting, then the
oracle's budgets, scores, smoothing and selection on the part's own inputs,
sliced from the batch by the part's key ranges) and reassemble the per-row
results, which must equal the one-process results row for row.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth
from kv_cache_compression_layer_b200 import partition as pt


def test_splits_cover_every_row_once():
    for n_layers, H, L, world in [(28, 4, (2000, 3500, 5000, 7500, 9000, 12000, 14000, 16000), 8),
                                  (48, 4, (16000,), 4), (36, 2, (6000,), 8), (3, 4, (600, 1000, 1400), 2)]:
        rows = n_layers * H * len(L)
        for parts in ([pt.partition(n_layers, H, L, world)] +
                      ([pt.split_by_layers(n_layers, H, L, world)] if world <= n_layers else []) +
                      ([pt.split_by_sequences(n_layers, H, L, world)] if world <= len(L) else [])):
            allrows = np.sort(np.concatenate([p.rows for p in parts]))
            np.testing.assert_array_equal(allrows, np.arange(rows))
            assert pt.assemble_rows(parts, [p.rows.tolist() for p in parts]) == list(range(rows))


def test_split_choice_and_balance():
    L = (2000, 3500, 5000, 7500, 9000, 12000, 14000, 16000)  # the ragged batch
    parts = pt.partition(28, 4, L, 8)
    # by layers: 3 or 4 of 28 layers of every sequence; by sequences one rank would hold 16000 alone
    assert all(p.seqs == tuple(range(8)) for p in parts)
    assert pt.largest_share(parts) == 4 * sum(L)
    seq = pt.split_by_sequences(28, 4, L, 2)
    assert sorted(sum(p.L) for p in seq) == [34500, 34500]  # greedy longest first balances exactly here
    with pytest.raises(ValueError):
        pt.partition(2, 4, (100,), 3)


def test_key_ranges_slice_the_batch():
    cfg = synth.small("ragged", n_layers=3, L=(600, 1000, 1400))
    bt = synth.make_batch(cfg, steps=1)
    koff = bt.key_off
    for parts in (pt.split_by_layers(3, 4, cfg.L, 2), pt.split_by_sequences(3, 4, cfg.L, 2)):
        for p in parts:
            got = np.concatenate([bt.K[a:b] for a, b in p.key_ranges(3, 4, cfg.L)])
            want = np.concatenate([bt.K[koff[r]:koff[r + 1]] for r in p.rows])
            np.testing.assert_array_equal(got, want)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_part(cfg, bt, part, rows):
    """The path on one part: host accounting from the library, then the oracle's steps."""
    import kv_cache_compression_layer_b200 as kv
    import oracle as orc

    shape = kv.make_shape(part.n_layers, cfg.n_kv_heads, cfg.group, cfg.head_dim, cfg.w, kv.KV_BF16)
    params = kv.make_params(cfg.budget_pct, cfg.alpha, cfg.rho, cfg.r, cfg.gamma, cfg.sinks_T, cfg.recent_pct)
    assert kv.kv_rows(shape, len(part.L)) == len(rows)
    slots = kv.kv_total_slots(shape, part.L, params)
    S = bt.S[part.layers[0]:part.layers[1]]
    b = orc.allocate(S, part.L, cfg.w, cfg.budget_pct, cfg.r).reshape(-1)
    K = np.concatenate([bt.K[a:e] for a, e in part.key_ranges(cfg.n_layers, cfg.n_kv_heads, cfg.L)])
    L_rows = [cfg.row_L(int(r)) for r in rows]
    s = orc.score(bt.qwin[rows], K, L_rows, n_threads=2)
    s_hat, ks = orc.sss(s, L_rows, cfg.alpha, cfg.rho, n_threads=2)
    idx = orc.select(s_hat, L_rows, cfg.w, b.tolist(), n_threads=2)
    return slots, [(int(b[i]), int(ks[i]), idx[i].tolist()) for i in range(len(rows))]


def _rank_main(rank: int, world: int, port: int, out_dir: str, by: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import pickle

    import torch.distributed as dist

    from kv_cache_compression_layer_b200.replicas import init_group

    assert init_group("gloo", world, timeout_s=120.0)
    try:
        cfg = synth.small("ragged", n_layers=3, L=(600, 1000, 1400))
        bt = synth.make_batch(cfg, steps=1)
        split = pt.split_by_layers if by == "layers" else pt.split_by_sequences
        parts = split(cfg.n_layers, cfg.n_kv_heads, cfg.L, world)
        part = parts[rank]
        slots, res = _run_part(cfg, bt, part, part.rows)
        gathered = [None] * world
        dist.all_gather_object(gathered, (slots, res))
        if rank == 0:
            with open(os.path.join(out_dir, f"{by}.pkl"), "wb") as f:
                pickle.dump((parts, gathered), f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("by", ["layers", "sequences"])
def test_two_ranks_reassemble_the_one_rank_result(tmp_path, by):
    import pickle

    import kv_cache_compression_layer_b200 as kv

    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), by), nprocs=world, join=True,
                       start_method="spawn")
    with open(tmp_path / f"{by}.pkl", "rb") as f:
        parts, gathered = pickle.load(f)
    cfg = synth.small("ragged", n_layers=3, L=(600, 1000, 1400))
    bt = synth.make_batch(cfg, steps=1)
    whole = pt.Part(0, tuple(range(cfg.n_seq)), (0, cfg.n_layers), cfg.L, np.arange(cfg.rows))
    slots_one, res_one = _run_part(cfg, bt, whole, np.arange(cfg.rows))
    assert sum(g[0] for g in gathered) == slots_one  # the slot accounting adds up
    shape = kv.make_shape(cfg.n_layers, cfg.n_kv_heads, cfg.group, cfg.head_dim, cfg.w, kv.KV_BF16)
    assert slots_one == kv.kv_total_slots(shape, cfg.L, kv.make_params(cfg.budget_pct, cfg.alpha, cfg.rho, cfg.r,
                                                                       cfg.gamma, cfg.sinks_T, cfg.recent_pct))
    assert pt.assemble_rows(parts, [g[1] for g in gathered]) == res_one
