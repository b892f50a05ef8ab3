"""End-to-end checking of the whole path run through ``Compressor`` (the
calls the benchmark times) on chosen rows of a batch: budgets on every row,
then per chosen row the scores, k*, s_hat, the selection and the gathers,
then decode steps in lock step (tests/_lockstep.py). Only the chosen rows'
slices of the GPU buffers are read back, so full-size workloads fit.
"""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
from kv_cache_compression_layer_b200 import Compressor
from tests._harness import (dev, f32, kstar_band_end_to_end, kth_exempt_mask, params_of, score_close, shape_of,
                            tdtype, up, valid_kstars)
from tests._lockstep import LockStep, Snapshot, oracle_lists


def compress(cfg, bt):
    """Uploads the batch and runs the compression stage; returns (comp, K, V)."""
    dt = tdtype(cfg)
    comp = Compressor(shape_of(cfg), cfg.L, params_of(cfg))
    spikes = None
    if bt.spikes is not None:
        spikes = up(np.where(bt.spikes, 10.0, 1.0).astype(np.float32), torch.float32)
    K, V = up(bt.K, dt), up(bt.V, dt)
    comp.compress(up(bt.qwin, dt), K, V, up(bt.S, torch.float32), spikes=spikes)
    torch.cuda.synchronize()
    assert kv.kv_read_device_status(comp.ws[:4].view(torch.int32)) == 0
    return comp, K, V


def check_compress_rows(cfg, bt, comp, rows) -> tuple:
    """Checks budgets (every row) and the compression of `rows`; returns
    (kept positions per checked row, rows whose selection equals the oracle's)."""
    b_gpu = comp.b.cpu().numpy()
    b_orc = orc.allocate(bt.S, cfg.L, cfg.w, cfg.budget_pct, cfg.r).reshape(-1)
    np.testing.assert_array_equal(b_gpu, b_orc)
    off = comp.slot_off.cpu().numpy()
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(b_orc.astype(np.int64) + 1)]))
    ks_gpu = comp.kstar.cpu().numpy()
    koff = bt.key_off
    alpha, rho = f32(cfg.alpha), f32(cfg.rho)  # the values the kernels received
    kept, same = {}, []
    for r in rows:
        L = int(bt.L_rows[r])
        sl = slice(int(koff[r]), int(koff[r + 1]))
        s_gpu = comp.s[sl].cpu().numpy()
        h_gpu = comp.s_hat[sl].cpu().numpy()
        s_orc = orc.score(bt.qwin[r:r + 1], bt.K[sl], [L])
        if bt.spikes is not None:  # the harness multiplies spike positions by 10 before smoothing
            s_orc = s_orc * np.where(bt.spikes[sl], 10.0, 1.0)
        ok, worst = score_close(s_gpu, s_orc, [L])
        assert ok, ("score", r, worst)
        valid = valid_kstars(s_orc, rho, orc, kstar_band_end_to_end(rho))
        assert int(ks_gpu[r]) in valid, ("kstar", r, int(ks_gpu[r]), valid[:4])
        h_orc, _ = orc.sss(s_orc, [L], alpha, rho, kstar_force=[int(ks_gpu[r])])
        ok, worst = score_close(h_gpu, h_orc, [L], floor="rms")
        assert ok, ("s_hat", r, worst)
        b_r = int(b_orc[r])
        idx_orc = orc.select(h_orc, [L], cfg.w, [b_r])[0]
        lo = int(off[r])
        idx_gpu = comp.pos[lo:lo + b_r].cpu().numpy()
        Kc = comp.Kc[lo:lo + b_r].float().cpu().numpy()
        Vc = comp.Vc[lo:lo + b_r].float().cpu().numpy()
        assert len(idx_gpu) == len(idx_orc) == min(b_r, L)
        assert (np.diff(idx_gpu) > 0).all() and set(range(L - cfg.w, L)) <= set(idx_gpu.tolist())
        diff = np.setxor1d(idx_gpu, idx_orc)
        if len(diff):
            exempt = np.flatnonzero(kth_exempt_mask(h_orc, L, cfg.w, b_r))
            assert set(diff.tolist()) <= set(exempt.tolist()), ("select", r, diff[:8])
        else:
            same.append(r)
        np.testing.assert_array_equal(Kc, bt.K[koff[r] + idx_gpu])
        np.testing.assert_array_equal(Vc, bt.V[koff[r] + idx_gpu])
        # a selection that differs only at exempt near ties is one of the correct
        # selections: decode checking starts from it
        kept[r] = idx_gpu
    return kept, same


def decode_lockstep(cfg, bt, comp, kept: dict, steps: int) -> LockStep:
    """Runs `steps` decode steps of the whole batch; checks the rows of `kept` in lock step."""
    rows = sorted(kept)
    b = comp.b.cpu().numpy()
    off = comp.slot_off.cpu().numpy()
    ls = LockStep(oracle_lists(bt, rows, kept), {r: int(b[r]) for r in rows}, {r: int(bt.L_rows[r]) for r in rows},
                  {r: orc.recent_count(int(b[r]), cfg.recent_pct) for r in rows}, cfg.gamma, cfg.sinks_T, cfg.dtype)
    dt = tdtype(cfg)
    out = torch.empty(cfg.rows, cfg.group, cfg.head_dim, dtype=dt, device=dev())
    state = {"meta": comp.meta, "pos": comp.pos, "A": comp.A}
    for t in range(steps):
        comp.decode_step(up(bt.q_dec[t], dt), up(bt.k_dec[t], dt), up(bt.v_dec[t], dt), out)
        torch.cuda.synchronize()
        o = out[rows].float().cpu().numpy()
        ls.step(t, Snapshot(state, off), {r: o[i] for i, r in enumerate(rows)}, bt.q_dec[t], bt.k_dec[t],
                bt.v_dec[t])
    ls.compare_A(Snapshot(state, off))
    assert kv.kv_read_device_status(comp.status) == 0
    return ls
