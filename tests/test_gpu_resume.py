"""Checkpoint and resume of the decode state, and poison fills.

The decode state is plain device memory: the compacted cache (K_c, V_c), the
decayed scores A, the positions, the per-row meta data and the decode
scratch (work items, step counters and stamped partial lists, carried
between steps; it holds no addresses). Copied out mid-run into fresh buffers,
it must continue bit-identically: the same outputs, evictions and state.

Poison fills: the outputs of the compression stage are filled with NaN (or
-7 for integers) before the call; afterwards every element the path defines
must be written and the spare decode slot of every row left untouched.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import synth
from tests._decode_state import gpu_cache, initial_state
from tests._harness import dev, params_of, shape_of, tdtype, up
from tests._pipeline import compress

pytestmark = pytest.mark.gpu

STATE = ("Kc", "Vc", "A", "pos", "meta", "scratch")


def _steps(cfg, bt, cache, t, steps, first):
    sh, p, dt = shape_of(cfg), params_of(cfg), tdtype(cfg)
    outs, metas = [], []
    out = torch.empty(cfg.rows, cfg.group, cfg.head_dim, dtype=dt, device=dev())
    for s in range(first, first + steps):
        kv.kv_decode_attn_update(sh, cfg.L, p, cache, up(bt.q_dec[s], dt), up(bt.k_dec[s], dt), up(bt.v_dec[s], dt),
                                 out)
        outs.append(out.clone())
        metas.append(t["meta"].clone())
    torch.cuda.synchronize()
    assert kv.kv_read_device_status(t["status"]) == 0
    return outs, metas


# a batch of 36 rows (g = 8) and a ragged one of 16 rows (g = 7)
RESUME_CASES = [synth.small("3b", n_layers=18, L=(2000,)), synth.small("ragged", n_layers=2, L=(1000, 3500))]


@pytest.mark.parametrize("cfg", RESUME_CASES, ids=lambda c: f"{c.name}-{c.rows}rows")
def test_decode_state_resumes_bit_identically(cfg):
    n1, n2 = 5, 6
    bt = synth.make_batch(cfg, steps=n1 + n2)
    b, idx = initial_state(cfg, bt)
    cache, t, off = gpu_cache(cfg, bt, b, idx)
    _steps(cfg, bt, cache, t, n1, 0)
    ckpt = {k: t[k].cpu().clone() for k in STATE}  # the checkpoint, on the host
    outs_a, metas_a = _steps(cfg, bt, cache, t, n2, n1)
    # resume from the checkpoint in fresh device buffers
    t2 = {k: v.clone() for k, v in t.items()}
    for k in STATE:
        t2[k] = torch.empty_like(t[k])
        t2[k].copy_(ckpt[k])
    t2["status"] = torch.zeros_like(t["status"])
    cache2 = kv.make_cache(t2["Kc"], t2["Vc"], t2["A"], t2["pos"], t2["slot_off"], t2["b"], t2["meta"],
                           t2["status"], t2["scratch"])
    outs_b, metas_b = _steps(cfg, bt, cache2, t2, n2, n1)
    for i in range(n2):
        assert torch.equal(outs_a[i], outs_b[i]), ("output", i)
        assert torch.equal(metas_a[i], metas_b[i]), ("meta", i)
    for k in ("Kc", "Vc", "A", "pos", "meta"):
        assert torch.equal(t[k], t2[k]), k


POISON_CASES = [synth.small("3b", n_layers=2, L=(2000,)), synth.small("ragged", n_layers=2, L=(1000, 3500)),
                synth.CONFIGS["tiny"]]


@pytest.mark.parametrize("cfg", POISON_CASES, ids=lambda c: c.name)
def test_compression_writes_exactly_its_outputs(cfg):
    bt = synth.make_batch(cfg, steps=2)
    comp, K, V = compress(cfg, bt)  # once to learn the budgets
    nan = float("nan")
    for x in (comp.s, comp.s_hat, comp.Kc, comp.Vc):
        x.fill_(nan)
    for x in (comp.pos, comp.kstar, comp.b):
        x.fill_(-7)
    comp.slot_off.fill_(-7)
    dt = tdtype(cfg)
    spikes = None if bt.spikes is None else up(np.where(bt.spikes, 10.0, 1.0).astype(np.float32), torch.float32)
    comp.compress(up(bt.qwin, dt), K, V, up(bt.S, torch.float32), spikes=spikes)
    torch.cuda.synchronize()
    assert torch.isfinite(comp.s).all() and torch.isfinite(comp.s_hat).all()
    assert (comp.kstar >= 0).all() and (comp.b >= cfg.w).all()
    off = comp.slot_off.cpu().numpy()
    b = comp.b.cpu().numpy()
    assert off[0] == 0 and (np.diff(off) == b + 1).all()
    pos = comp.pos.cpu().numpy()
    Kc = comp.Kc.float().cpu().numpy()
    Vc = comp.Vc.float().cpu().numpy()
    for r in range(cfg.rows):
        lo, n = int(off[r]), int(b[r])
        assert (pos[lo:lo + n] >= 0).all() and pos[lo + n] == -7, r  # the spare slot is left alone
        assert np.isfinite(Kc[lo:lo + n]).all() and np.isnan(Kc[lo + n]).all(), r
        assert np.isfinite(Vc[lo:lo + n]).all() and np.isnan(Vc[lo + n]).all(), r
    # decode writes every output element
    out = torch.full((cfg.rows, cfg.group, cfg.head_dim), nan, dtype=dt, device=dev())
    comp.decode_step(up(bt.q_dec[0], dt), up(bt.k_dec[0], dt), up(bt.v_dec[0], dt), out)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert kv.kv_read_device_status(comp.status) == 0
