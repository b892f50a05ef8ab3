"""The timeout paths of the bounded device waits, driven on the GPU without a
fault: with kv_set_wait_limit_ns(0) every wait gives up unless what it waits
for has already happened. The kernel then records KV_DEV_TIMEOUT in the
call's status word, lets the copies and tensor-core operations it issued
land, releases its tensor memory and returns, so the context stays usable:
with the default limit back, the same calls match the oracle again (decode
after kv_decode_init, which the header requires after a timed-out step).
Covered: kv_score (its tensor-core passes) and one step of the persistent
decode kernel (the path of every bf16 batch with g <= 8).
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._decode_state import gpu_cache, initial_state
from tests._harness import dev, params_of, score_close, shape_of, tdtype, up
from tests._lockstep import LockStep, Snapshot, oracle_lists

pytestmark = pytest.mark.gpu


class zero_wait_limit:
    def __enter__(self):
        self.prev = kv.kv_set_wait_limit_ns(0)

    def __exit__(self, *exc):
        kv.kv_set_wait_limit_ns(self.prev)


def test_score_timeout_then_recovers():
    cfg = synth.small("3b", n_layers=2)
    bt = synth.make_batch(cfg, steps=1)
    sh, dt = shape_of(cfg), tdtype(cfg)
    q, K = up(bt.qwin, dt), up(bt.K, dt)
    ws = torch.empty(kv.kv_workspace_bytes(sh, cfg.L), dtype=torch.uint8, device=dev())
    s = torch.empty(len(bt.K), dtype=torch.float32, device=dev())
    with zero_wait_limit():
        kv.kv_score(sh, cfg.L, q, K, s, ws)
        st = kv.kv_read_device_status(ws[:4].view(torch.int32))
    assert st & kv.KV_DEV_TIMEOUT, st
    kv.kv_score(sh, cfg.L, q, K, s, ws)  # default limit: a normal call clears the word and completes
    assert kv.kv_read_device_status(ws[:4].view(torch.int32)) == 0
    ok, worst = score_close(s.cpu().numpy(), orc.score(bt.qwin, bt.K, bt.L_rows), bt.L_rows)
    assert ok, worst


def test_persistent_decode_timeout_then_init_recovers():
    # 8 rows of g = 7: far fewer than the SM count, so the persistent kernel runs
    cfg = synth.small("ragged", n_layers=1, L=(1000, 2000), budget_pct=10)
    steps = 6
    bt = synth.make_batch(cfg, steps=steps + 1)
    b, idx = initial_state(cfg, bt)
    cache, t, off = gpu_cache(cfg, bt, b, idx)
    sh, p, dt = shape_of(cfg), params_of(cfg), tdtype(cfg)
    out = torch.empty(cfg.rows, cfg.group, cfg.head_dim, dtype=dt, device=dev())
    with zero_wait_limit():
        kv.kv_decode_attn_update(sh, cfg.L, p, cache, up(bt.q_dec[0], dt), up(bt.k_dec[0], dt),
                                 up(bt.v_dec[0], dt), out)
        st = kv.kv_read_device_status(t["status"])
    assert st & kv.KV_DEV_TIMEOUT, st
    # the state is undefined after a timed-out step: kv_decode_init makes it the
    # prefill state again (the kept slots are never written by a step)
    t["status"].zero_()
    kv.kv_decode_init(sh, cfg.L, p, cache)
    rows = range(cfg.rows)
    ls = LockStep(oracle_lists(bt, rows, {r: idx[r] for r in rows}), {r: int(b[r]) for r in rows},
                  {r: int(bt.L_rows[r]) for r in rows},
                  {r: orc.recent_count(int(b[r]), cfg.recent_pct) for r in rows}, cfg.gamma, cfg.sinks_T, cfg.dtype)
    for step in range(steps):
        kv.kv_decode_attn_update(sh, cfg.L, p, cache, up(bt.q_dec[step], dt), up(bt.k_dec[step], dt),
                                 up(bt.v_dec[step], dt), out)
        torch.cuda.synchronize()
        ls.step(step, Snapshot(t, off), out.float().cpu().numpy(), bt.q_dec[step], bt.k_dec[step], bt.v_dec[step])
    ls.compare_A(Snapshot(t, off))
    assert kv.kv_read_device_status(t["status"]) == 0
    assert np.isfinite(out.float().cpu().numpy()).all()
