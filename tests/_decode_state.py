"""Decode state for GPU tests: the oracle's own budgets and kept positions of
a seeded batch, and a GPU compacted cache built from them (every input from
the generator and the oracle, none from a CUDA output)."""
import numpy as np
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
from tests._harness import dev, params_of, shape_of, tdtype, up


def initial_state(cfg, bt):
    """The oracle's budgets and kept positions for every row of the batch."""
    b = orc.allocate(bt.S, cfg.L, cfg.w, cfg.budget_pct, cfg.r).reshape(-1)
    s = orc.score(bt.qwin, bt.K, bt.L_rows)
    s_hat, _ = orc.sss(s, bt.L_rows, cfg.alpha, cfg.rho)
    idx = orc.select(s_hat, bt.L_rows, cfg.w, b)
    return b.astype(np.int64), idx


def gpu_cache(cfg, bt, b, idx, count0=None):
    dt = tdtype(cfg)
    d = cfg.head_dim
    rows = cfg.rows
    cap = b + 1
    off = np.concatenate([[0], np.cumsum(cap)]).astype(np.int64)
    total = int(off[-1])
    Kc = np.zeros((total, d), np.float32)
    Vc = np.zeros((total, d), np.float32)
    pos = np.zeros(total, np.int32)
    koff = bt.key_off
    for r in range(rows):
        n0 = len(idx[r])
        Kc[off[r]:off[r] + n0] = bt.K[koff[r] + idx[r]]
        Vc[off[r]:off[r] + n0] = bt.V[koff[r] + idx[r]]
        pos[off[r]:off[r] + n0] = idx[r]
    t = dict(Kc=up(Kc, dt), Vc=up(Vc, dt), A=torch.zeros(total, dtype=torch.float32, device=dev()),
             pos=up(pos, torch.int32), slot_off=up(off, torch.int64), b=up(b.astype(np.int32), torch.int32),
             meta=torch.zeros(rows * kv.META_INTS, dtype=torch.int32, device=dev()),
             status=torch.zeros(4, dtype=torch.int32, device=dev()))
    nbytes = kv.kv_decode_scratch_bytes(shape_of(cfg), cfg.L, params_of(cfg), total)
    t["scratch"] = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev())
    cache = kv.make_cache(t["Kc"], t["Vc"], t["A"], t["pos"], t["slot_off"], t["b"], t["meta"], t["status"],
                          t["scratch"])
    kv.kv_decode_init(shape_of(cfg), cfg.L, params_of(cfg), cache)
    if count0 is not None:  # a cache that is not full yet (no eviction until it is)
        count0 = np.broadcast_to(np.asarray(count0, np.int32), (rows,))
        m = np.zeros((rows, kv.META_INTS), np.int32)
        m[:, 0] = count0
        m[:, 1] = count0
        m[:, 3] = -1
        m[:, 4] = count0
        t["meta"].copy_(torch.from_numpy(m.reshape(-1)))
    torch.cuda.synchronize()
    return cache, t, off
