"""Parity of kv_decode_attn_update with the oracle's literal VoxZip step.

Both sides start from the same kept set (the oracle's own selection on the
seeded rows) and run with the same decode inputs, in lock step on every row:
each step compares the attention output and the evicted position, and at the
end the decayed scores A. Where the evictions differ, the oracle's own A must
show a near tie between the two choices (1e-5 relative); the oracle then
takes the GPU's choice and the row stays under comparison (tests/_lockstep.py).
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._decode_state import gpu_cache, initial_state
from tests._harness import dev, params_of, shape_of, tdtype, up
from tests._lockstep import LockStep, Snapshot, oracle_lists

pytestmark = pytest.mark.gpu


def _run_lockstep(cfg, steps, bt=None, init=None, count0=None, V_ones=False, o_tol=None):
    bt = bt or synth.make_batch(cfg, steps=steps)
    if V_ones:
        bt.V[:] = 1.0
        bt.v_dec[:] = 1.0
    b, idx = init if init is not None else initial_state(cfg, bt)
    cache, t, off = gpu_cache(cfg, bt, b, idx, count0)
    sh, p = shape_of(cfg), params_of(cfg)
    dt = tdtype(cfg)
    rows, G, d = cfg.rows, cfg.group, cfg.head_dim
    extra = max(1, (count0 is not None) * steps + 1)
    ls = LockStep(oracle_lists(bt, range(rows), {r: idx[r] for r in range(rows)}, extra=extra),
                  {r: int(b[r]) for r in range(rows)}, {r: int(bt.L_rows[r]) for r in range(rows)},
                  {r: orc.recent_count(int(b[r]), cfg.recent_pct) for r in range(rows)},
                  cfg.gamma, cfg.sinks_T, cfg.dtype)
    if o_tol is not None:
        ls.tol = o_tol
    out = torch.empty(rows, G, d, dtype=dt, device=dev())
    for step in range(steps):
        q = up(bt.q_dec[step], dt)
        k = up(bt.k_dec[step], dt)
        v = up(bt.v_dec[step], dt)
        kv.kv_decode_attn_update(sh, cfg.L, p, cache, q, k, v, out)
        torch.cuda.synchronize()
        ls.step(step, Snapshot(t, off), out.float().cpu().numpy(), bt.q_dec[step], bt.k_dec[step], bt.v_dec[step])
    return bt, b, t, off, ls


DECODE_CASES = [
    (synth.CONFIGS["tiny"], 32),
    (synth.small("3b", n_layers=1, L=(2000,)), 24),
    (synth.small("ragged", n_layers=1, L=(1000, 2000), budget_pct=10), 40),  # g = 7, small budgets
    # many rows: 36 (g = 8) and 72 (g = 7), several rows per CTA of the persistent kernel
    (synth.small("3b", n_layers=18, L=(2000,)), 12),
    (synth.small("ragged", n_layers=9, L=(1000, 2000), budget_pct=10), 12),  # g = 7
]


@pytest.mark.parametrize("cfg,steps", DECODE_CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_decode_lockstep(cfg, steps):
    bt, b, t, off, ls = _run_lockstep(cfg, steps)
    assert ls.ties <= max(1, cfg.rows // 4), ls.ties  # near ties are rare
    assert ls.checked == cfg.rows * steps
    ls.compare_A(Snapshot(t, off))
    assert kv.kv_read_device_status(t["status"]) == 0


def test_decode_no_eviction_is_full_attention():
    # a cache that is not full: no eviction, so each step is full attention
    # over the kept prefill entries plus every appended token
    cfg = synth.small("3b", n_layers=1, L=(1000,))
    steps = 12
    bt = synth.make_batch(cfg, steps=steps)
    b0, idx = initial_state(cfg, bt)
    count0 = np.array([len(i) for i in idx])
    b = b0 + steps  # room for every appended token
    _, _, t, off, ls = _run_lockstep(cfg, steps, bt=bt, init=(b, idx), count0=count0)
    assert ls.ties == 0
    meta = t["meta"].cpu().numpy().reshape(cfg.rows, kv.META_INTS)
    assert (meta[:, 0] == count0 + steps).all() and (meta[:, 3] == -1).all()
    ls.compare_A(Snapshot(t, off))


def test_decode_values_one_give_one():
    cfg = synth.small("3b", n_layers=1, L=(1000,))
    _run_lockstep(cfg, 6, V_ones=True, o_tol=1e-12)
