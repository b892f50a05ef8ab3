"""kv_wnw_update and kv_wnw_recall against the oracle's WnW step, in lock
step over many decode steps: chunk scores (float64, the same summation
order), idle counts, block slots, fetch and release lists all bit-exact;
after every recall the GPU copy of each resident block equals the host rows."""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._harness import dev, up

pytestmark = pytest.mark.gpu


def _run(Ls, n_anchor, steps, p, n_tidal=3, d=128, ties_every=7, seed=0):
    n_seq = len(Ls)
    S, cap = p.chunk_stride, p.top_c * (p.chunk_len // p.chunk_stride)
    att = [synth.anchor_attention(seed + i, L, n_anchor, steps) for i, L in enumerate(Ls)]
    for i in range(n_seq):
        att[i][::ties_every] = 0.25  # whole steps of equal scores: ties to the lower chunk
    n_state = kv.kv_wnw_state_ints(Ls, p)
    M_tot = kv.kv_wnw_chunk_count(Ls, p)
    state = torch.zeros(n_state, dtype=torch.int32, device=dev())
    score = torch.zeros(M_tot, dtype=torch.float64, device=dev())
    fetch = torch.full((n_seq, cap, 2), -3, dtype=torch.int32, device=dev())
    release = torch.full((n_seq, cap, 2), -3, dtype=torch.int32, device=dev())
    counts = torch.zeros(n_seq, 2, dtype=torch.int32, device=dev())
    kv.kv_wnw_init(Ls, p, state)
    rng = np.random.default_rng(seed)
    host_rows = sum(n_tidal * L for L in Ls)
    K_h = torch.from_numpy(synth.round_bf16(rng.standard_normal((host_rows, d)).astype(np.float32))).to(
        torch.bfloat16).pin_memory()
    V_h = torch.from_numpy(synth.round_bf16(rng.standard_normal((host_rows, d)).astype(np.float32))).to(
        torch.bfloat16).pin_memory()
    K_g = torch.zeros(n_seq * n_tidal * p.n_slots * S, d, dtype=torch.bfloat16, device=dev())
    V_g = torch.zeros_like(K_g)
    orcs = [orc.WnwState(L, p.chunk_len, S, p.top_c, p.release_after, p.n_slots) for L in Ls]
    hoff = np.concatenate([[0], np.cumsum([n_tidal * L for L in Ls])])
    soff = np.concatenate([[0], np.cumsum([o.M for o in orcs])])
    Kh, Vh = K_h.float().numpy(), V_h.float().numpy()
    for t in range(steps):
        s_dev = up(np.concatenate([att[i][t].reshape(-1) for i in range(n_seq)]), torch.float32)
        kv.kv_wnw_update(Ls, p, n_anchor, s_dev, state, score, fetch, release, counts)
        kv.kv_wnw_recall(Ls, p, n_tidal, d, kv.KV_BF16, fetch, counts, K_h, V_h, K_g, V_g)
        torch.cuda.synchronize()
        st_h, sc_h = state.cpu().numpy(), score.cpu().numpy()
        f_h, r_h, c_h = fetch.cpu().numpy(), release.cpu().numpy(), counts.cpu().numpy()
        Kg, Vg = K_g.float().cpu().numpy(), V_g.float().cpu().numpy()
        so = 0
        for i, o in enumerate(orcs):
            sc_o, _, f_o, r_o = o.step(att[i][t])
            np.testing.assert_array_equal(sc_h[soff[i]:soff[i + 1]], sc_o, err_msg=f"step {t} seq {i}")
            words = o.M + o.nb + p.n_slots
            np.testing.assert_array_equal(st_h[so:so + words],
                                          np.concatenate([o.idle, o.block_slot, o.slot_block]),
                                          err_msg=f"step {t} seq {i}")
            so += words
            assert c_h[i].tolist() == [len(f_o), len(r_o)], (t, i)
            np.testing.assert_array_equal(f_h[i, :len(f_o)], f_o)
            np.testing.assert_array_equal(r_h[i, :len(r_o)], r_o)
            for b in np.nonzero(o.block_slot >= 0)[0]:
                k = o.block_slot[b]
                rows = min(S, Ls[i] - b * S)
                for r in range(n_tidal):
                    g0 = ((i * n_tidal + r) * p.n_slots + k) * S
                    h0 = hoff[i] + r * Ls[i] + b * S
                    np.testing.assert_array_equal(Kg[g0:g0 + rows], Kh[h0:h0 + rows])
                    np.testing.assert_array_equal(Vg[g0:g0 + rows], Vh[h0:h0 + rows])
    return orcs


def test_wnw_lockstep_default_rule():
    p = kv.make_wnw_params()  # 4 s / 2 s chunks at 12.5 rows/s, top 3, released after 3 steps
    orcs = _run([3000, 40, 1237, 51], n_anchor=5, steps=40, p=p)
    assert any((o.idle >= 0).sum() > p.top_c for o in orcs)  # the hysteresis held chunks over


def test_wnw_lockstep_other_rules():
    _run([997, 2048], n_anchor=2, steps=25, p=kv.make_wnw_params(60, 20, 2, 1), n_tidal=2, d=64)
    _run([5000], n_anchor=7, steps=25, p=kv.make_wnw_params(50, 25, 8, 4, n_slots=70), n_tidal=1, ties_every=3)
    # 20000 chunks of 2 rows: too many to stage in shared memory, the update works on global memory
    _run([20000, 300], n_anchor=2, steps=6, p=kv.make_wnw_params(2, 1, 3, 3), n_tidal=1, d=64)


def test_wnw_long_audio():
    """32768 audio rows (about 44 min at 12.5 rows/s), 5 anchor rows, 24 tidal rows."""
    p = kv.make_wnw_params()
    _run([32768, 32768], n_anchor=5, steps=12, p=p, n_tidal=24, d=128, ties_every=5)
