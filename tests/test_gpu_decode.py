"""Parity of kv_decode_attn_update with the oracle's literal VoxZip step.

Both sides start from the same kept set (the oracle's own selection on the
seeded rows) and run their own trajectories with the same decode inputs. Each
step compares the attention output, the evicted position and, at the end,
the decayed scores A. When the evictions differ, the oracle's A must show a
near tie between the two choices (1e-5 relative); the row is then exempt from
further comparison (its trajectories legitimately part), and such rows are
counted.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._harness import dev, params_of, shape_of, tdtype, up

pytestmark = pytest.mark.gpu

TIE_RTOL = 1e-5


def _initial_state(cfg, bt):
    """The oracle's budgets and kept positions for every row of the batch."""
    b = orc.allocate(bt.S, cfg.L, cfg.w, cfg.budget_pct, cfg.r).reshape(-1)
    s = orc.score(bt.qwin, bt.K, bt.L_rows)
    s_hat, _ = orc.sss(s, bt.L_rows, cfg.alpha, cfg.rho)
    idx = orc.select(s_hat, bt.L_rows, cfg.w, b)
    return b.astype(np.int64), idx


def _gpu_cache(cfg, bt, b, idx, count0=None):
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


def _run_lockstep(cfg, steps, bt=None, init=None, count0=None, V_ones=False, o_tol=None):
    bt = bt or synth.make_batch(cfg, steps=steps)
    if V_ones:
        bt.V[:] = 1.0
        bt.v_dec[:] = 1.0
    b, idx = init if init is not None else _initial_state(cfg, bt)
    cache, t, off = _gpu_cache(cfg, bt, b, idx, count0)
    sh, p = shape_of(cfg), params_of(cfg)
    dt = tdtype(cfg)
    rows, G, d = cfg.rows, cfg.group, cfg.head_dim
    koff = bt.key_off
    lists = []
    for r in range(rows):
        lists.append(orc.DecodeList(bt.K[koff[r] + idx[r]], bt.V[koff[r] + idx[r]], idx[r],
                                    extra=max(1, (count0 is not None) * steps + 1)))
    M = [orc.recent_count(int(b[r]), cfg.recent_pct) for r in range(rows)]
    out = torch.empty(rows, G, d, dtype=dt, device=dev())
    diverged = np.zeros(rows, bool)
    ties = 0
    tol = o_tol if o_tol is not None else (2e-2 if cfg.dtype == "bf16" else 1e-4)
    for step in range(steps):
        q = up(bt.q_dec[step], dt)
        k = up(bt.k_dec[step], dt)
        v = up(bt.v_dec[step], dt)
        kv.kv_decode_attn_update(sh, cfg.L, p, cache, q, k, v, out)
        torch.cuda.synchronize()
        o_gpu = out.float().cpu().numpy()
        meta = t["meta"].cpu().numpy().reshape(rows, kv.META_INTS)
        pos_gpu = t["pos"].cpu().numpy()
        for r in range(rows):
            if diverged[r]:
                continue
            L = bt.L_rows[r]
            args = (bt.q_dec[step, r], bt.k_dec[step, r], bt.v_dec[step, r], L + step)
            before = lists[r].clone()
            o_orc, ev_orc = lists[r].step(*args, cfg.gamma, cfg.sinks_T, M[r], int(b[r]))
            err = np.abs(o_gpu[r] - o_orc)
            if cfg.dtype == "bf16":
                assert err.max() <= tol, (step, r, err.max())
            else:  # fp32: 1e-4 relative to the output row's scale
                assert err.max() <= tol * np.abs(o_orc).max(), (step, r, err.max())
            e_slot = int(meta[r, 3])
            ev_gpu = -1 if e_slot < 0 else int(pos_gpu[off[r] + e_slot])
            if ev_gpu != ev_orc:
                # the oracle's own decayed scores of the two choices must be a near tie:
                # replay the oracle step without eviction to read A of every entry
                before.step(*args, cfg.gamma, cfg.sinks_T, M[r], 1 << 40)
                _, _, A_all, pos_all = before.entries()
                amap = dict(zip(pos_all.tolist(), A_all.tolist()))
                assert ev_gpu in amap and ev_orc in amap, (step, r, ev_gpu, ev_orc)
                a_g, a_o = amap[ev_gpu], amap[ev_orc]
                assert abs(a_g - a_o) <= TIE_RTOL * max(abs(a_o), 1e-30), (step, r, a_g, a_o)
                ties += 1
                diverged[r] = True
    return bt, b, t, off, lists, diverged, ties


def _compare_A(cfg, b, t, off, lists, diverged):
    A = t["A"].cpu().numpy()
    pos = t["pos"].cpu().numpy()
    meta = t["meta"].cpu().numpy().reshape(cfg.rows, kv.META_INTS)
    for r in range(cfg.rows):
        if diverged[r]:
            continue
        _, _, A_o, pos_o = lists[r].entries()
        present = [s for s in range(int(b[r]) + 1) if s != meta[r, 1]]
        gp = {int(pos[off[r] + s]): A[off[r] + s] for s in present}
        assert sorted(gp) == sorted(pos_o.tolist())
        ga = np.array([gp[int(x)] for x in pos_o])
        np.testing.assert_allclose(ga, A_o, rtol=1e-4, atol=1e-6)


DECODE_CASES = [
    (synth.CONFIGS["tiny"], 32),
    (synth.small("3b", n_layers=1, L=(2000,)), 24),
    (synth.small("ragged", n_layers=1, L=(1000, 2000), budget_pct=10), 40),  # g = 7, small budgets
    # enough rows to fill the GPU as clusters: one cluster of 4 (36 rows) or 2 (72 rows) CTAs per row
    (synth.small("3b", n_layers=18, L=(2000,)), 12),
    (synth.small("ragged", n_layers=9, L=(1000, 2000), budget_pct=10), 12),  # g = 7
]


@pytest.mark.parametrize("cfg,steps", DECODE_CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_decode_lockstep(cfg, steps):
    bt, b, t, off, lists, diverged, ties = _run_lockstep(cfg, steps)
    assert ties <= max(1, cfg.rows // 4), ties
    _compare_A(cfg, b, t, off, lists, diverged)
    assert kv.kv_read_device_status(t["status"]) == 0


def test_decode_no_eviction_is_full_attention():
    # a cache that is not full: no eviction, so each step is full attention
    # over the kept prefill entries plus every appended token
    cfg = synth.small("3b", n_layers=1, L=(1000,))
    steps = 12
    bt = synth.make_batch(cfg, steps=steps)
    b0, idx = _initial_state(cfg, bt)
    count0 = np.array([len(i) for i in idx])
    b = b0 + steps  # room for every appended token
    _, _, t, off, lists, diverged, ties = _run_lockstep(cfg, steps, bt=bt, init=(b, idx), count0=count0)
    assert ties == 0
    meta = t["meta"].cpu().numpy().reshape(cfg.rows, kv.META_INTS)
    assert (meta[:, 0] == count0 + steps).all() and (meta[:, 3] == -1).all()


def test_decode_values_one_give_one():
    cfg = synth.small("3b", n_layers=1, L=(1000,))
    _, _, t, _, _, _, _ = _run_lockstep(cfg, 6, V_ones=True, o_tol=1e-12)
