"""kv_score_noalloc, the scoring entry point that allocates nothing.

Callers such as a serving runtime that has reserved the whole device for its
own memory pool, or a plugin whose host only hands it input and output
buffers, cannot obtain a workspace. For them the library keeps its scoring
scratch in one fixed device array of its own. These checks call that entry
point through the C ABI twice in a row (on two different batches, so the
array's leftover contents from the first call are in place for the second)
and compare each result with the oracle's scores and with kv_score given a
caller-owned workspace, under the score tolerance the other tests use; the
array's status word must read clean after each call. A batch whose scratch
does not fit the array must be refused before anything is launched.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._harness import dev, score_close, shape_of, tdtype, up

pytestmark = pytest.mark.gpu


def _inputs(cfg):
    bt = synth.make_batch(cfg, steps=1)
    dt = tdtype(cfg)
    return bt, up(bt.qwin, dt), up(bt.K, dt)


def _with_workspace(cfg, q, K, n):
    sh = shape_of(cfg)
    ws = torch.empty(kv.kv_workspace_bytes(sh, cfg.L), dtype=torch.uint8, device=dev())
    s = torch.empty(n, dtype=torch.float32, device=dev())
    kv.kv_score(sh, cfg.L, q, K, s, ws)
    return s


def test_noalloc_matches_oracle_and_kv_score_on_two_calls_in_a_row():
    cases = [synth.small("3b", n_layers=2), synth.small("ragged", n_layers=1, L=(2000, 3500))]
    for cfg in cases:
        sh = shape_of(cfg)
        assert kv.kv_workspace_bytes(sh, cfg.L) <= kv.KV_NOALLOC_SCRATCH_BYTES
    got = []
    for cfg in cases:  # back to back, sharing the library's scratch array
        bt, q, K = _inputs(cfg)
        s = torch.full((len(bt.K),), float("nan"), dtype=torch.float32, device=dev())
        kv.kv_score_noalloc(shape_of(cfg), cfg.L, q, K, s)
        assert kv.kv_score_noalloc_status() == 0  # this call's status word (synchronises)
        got.append((cfg, bt, q, K, s))
    for cfg, bt, q, K, s in got:
        ref = _with_workspace(cfg, q, K, len(bt.K))
        torch.cuda.synchronize()
        s_h = s.cpu().numpy()
        assert np.isfinite(s_h).all()
        ok, worst = score_close(s_h, orc.score(bt.qwin, bt.K, bt.L_rows), bt.L_rows)
        assert ok, ("oracle", worst)
        ok, worst = score_close(s_h, ref.cpu().numpy().astype(np.float64), bt.L_rows)
        assert ok, ("kv_score", worst)


def test_noalloc_refuses_batch_beyond_its_scratch():
    cfg = synth.CONFIGS["30b"]  # 48 x 4 rows of L = 16000: ~50 MB of scratch
    sh = shape_of(cfg)
    assert kv.kv_workspace_bytes(sh, cfg.L) > kv.KV_NOALLOC_SCRATCH_BYTES
    with pytest.raises(kv.KvError) as e:
        kv.kv_score_noalloc(sh, cfg.L, 16, 16, 16)
    assert e.value.status == kv.KV_ERR_WORKSPACE
