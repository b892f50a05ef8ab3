"""kv_decode_attn_update on a batch with many short rows (d = 64): each CTA
of the persistent decode kernel owns more rows than it holds constants for at
once, so its finish runs in several batches of rows. The initial caches are
built directly (seeded random kept sets); sampled rows, spread over the whole
batch, run in lock step against the oracle's literal VoxZip step (a near tie
of the oracle's own decayed scores lets the oracle take the GPU's eviction,
tests/_lockstep.py).
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._harness import dev, up
from tests._lockstep import LockStep, Snapshot

pytestmark = pytest.mark.gpu


def test_decode_many_short_rows():
    n_seq, n_layers, H, G, d, L, w = 64, 19, 8, 8, 64, 128, 32
    gamma, T, recent_pct = 0.95, 4, 20
    steps = 4
    rows = n_seq * n_layers * H  # 9728 rows, one 128-slot work item each
    rng = np.random.default_rng(7)
    b = rng.integers(48, 61, size=rows).astype(np.int64)
    cap = b + 1
    off = np.concatenate([[0], np.cumsum(cap)]).astype(np.int64)
    total = int(off[-1])
    Kc = synth.round_bf16(rng.standard_normal((total, d)).astype(np.float32))
    Vc = synth.round_bf16(rng.standard_normal((total, d)).astype(np.float32))
    pos = np.zeros(total, np.int32)
    for r in range(rows):
        head = rng.choice(L - w, size=int(b[r]) - w, replace=False)
        pos[off[r]:off[r] + b[r]] = np.sort(np.concatenate([head, np.arange(L - w, L)]))
    q = synth.round_bf16(rng.standard_normal((steps, rows, G, d)).astype(np.float32))
    kd = synth.round_bf16(rng.standard_normal((steps, rows, d)).astype(np.float32))
    vd = synth.round_bf16(rng.standard_normal((steps, rows, d)).astype(np.float32))

    bf = torch.bfloat16
    shape = kv.make_shape(n_layers, H, G, d, w, kv.KV_BF16)
    params = kv.make_params(40, 0.5, 0.7, 0.5, gamma, T, recent_pct)
    Ls = [L] * n_seq
    t = dict(Kc=up(Kc, bf), Vc=up(Vc, bf), A=torch.zeros(total, dtype=torch.float32, device=dev()),
             pos=up(pos, torch.int32), slot_off=up(off, torch.int64), b=up(b.astype(np.int32), torch.int32),
             meta=torch.zeros(rows * kv.META_INTS, dtype=torch.int32, device=dev()),
             status=torch.zeros(4, dtype=torch.int32, device=dev()))
    nbytes = kv.kv_decode_scratch_bytes(shape, Ls, params, total)
    t["scratch"] = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev())
    cache = kv.make_cache(t["Kc"], t["Vc"], t["A"], t["pos"], t["slot_off"], t["b"], t["meta"], t["status"],
                          t["scratch"], total_slots=total)
    kv.kv_decode_init(shape, Ls, params, cache)

    sample = np.unique(np.linspace(0, rows - 1, 48).astype(int))
    lists = {int(r): orc.DecodeList(Kc[off[r]:off[r] + b[r]], Vc[off[r]:off[r] + b[r]], pos[off[r]:off[r] + b[r]])
             for r in sample}
    ls = LockStep(lists, {int(r): int(b[r]) for r in sample}, {int(r): L for r in sample},
                  {int(r): orc.recent_count(int(b[r]), recent_pct) for r in sample}, gamma, T, "bf16")
    out = torch.empty(rows, G, d, dtype=bf, device=dev())
    for step in range(steps):
        kv.kv_decode_attn_update(shape, Ls, params, cache, up(q[step], bf), up(kd[step], bf), up(vd[step], bf),
                                 out)
        torch.cuda.synchronize()
        ls.step(step, Snapshot(t, off), out.float().cpu().numpy(), q[step], kd[step], vd[step])
    assert ls.ties <= 2 and ls.checked == len(sample) * steps
    assert kv.kv_read_device_status(t["status"]) == 0
    snap = Snapshot(t, off)
    assert (snap.meta[:, 2] == steps).all()
    ls.compare_A(snap)
