"""Parity of each CUDA kernel with the CPU oracle, on seeded inputs.

Every input comes from the generator or from the oracle (never from a CUDA
output); the oracle is run on exactly the values the kernel sees (bf16 inputs
are bf16-exact floats on both sides, fp32 scores are upcast exactly).
"""
import math

import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._harness import (KSTAR_BAND_SAME_INPUT, dev, f32, kth_exempt_mask, params_of, score_close, shape_of,
                            tdtype, up, valid_kstars)

pytestmark = pytest.mark.gpu


def _score_case(cfg):
    bt = synth.make_batch(cfg, steps=1)
    sh = shape_of(cfg)
    dt = tdtype(cfg)
    q = up(bt.qwin, dt)
    K = up(bt.K, dt)
    s = torch.empty(len(bt.K), dtype=torch.float32, device=dev())
    wsb = kv.kv_workspace_bytes(sh, cfg.L)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev())
    kv.kv_score(sh, cfg.L, q, K, s, ws)
    torch.cuda.synchronize()
    assert kv.kv_read_device_status(ws[:4].view(torch.int32)) == 0
    return bt, s.cpu().numpy()


SCORE_CASES = [
    synth.CONFIGS["tiny"],
    synth.small("3b", n_layers=2),
    synth.small("3b", n_layers=1, L=(1000,), head_dim=64),  # d = 64, ragged tail tile
    synth.small("ragged", n_layers=1, L=(2000, 3500)),  # R = 7 * 32 = 224
    synth.small("30b", n_layers=1),
    synth.small("3b", n_layers=1, L=(210,), w=8, group=4),  # tiny L, R = 32
]


@pytest.mark.parametrize("cfg", SCORE_CASES, ids=lambda c: f"{c.name}-L{c.L[0]}-d{c.head_dim}-R{c.R}")
def test_score_matches_oracle(cfg):
    bt, s_gpu = _score_case(cfg)
    s_orc = orc.score(bt.qwin, bt.K, bt.L_rows)
    ok, worst = score_close(s_gpu, s_orc, bt.L_rows)
    assert ok, f"worst error / tolerance = {worst:.3g}"
    off = bt.key_off
    for i in range(len(bt.L_rows)):
        assert abs(s_gpu[off[i]:off[i + 1]].astype(np.float64).sum() - cfg.R) < 1e-4 * cfg.R


def test_score_long_row_sample():
    # long-form stress length L = 32768, one layer of 4 KV heads; oracle on two rows
    cfg = synth.small("long", n_layers=1)
    bt, s_gpu = _score_case(cfg)
    off = bt.key_off
    for r in (0, 3):
        s_orc = orc.score(bt.qwin[r:r + 1], bt.K[off[r]:off[r + 1]], [bt.L_rows[r]])
        ok, worst = score_close(s_gpu[off[r]:off[r + 1]], s_orc, [bt.L_rows[r]])
        assert ok, worst


# ---------------------------------------------------------------------- SSS --
def _run_sss(L_list, s_rows, alpha, rho):
    cfg = synth.Config("sss", 1, 1, 1, 64, tuple(L_list), "f32", w=2)
    sh = shape_of(cfg)
    s = up(np.concatenate(s_rows).astype(np.float32), torch.float32)
    s_hat = torch.empty_like(s)
    ks = torch.empty(len(L_list), dtype=torch.int32, device=dev())
    kv.kv_sss(sh, L_list, s, s_hat, ks, alpha, rho)
    torch.cuda.synchronize()
    return s_hat.cpu().numpy(), ks.cpu().numpy()


def _check_sss(L_list, s_rows, alpha, rho):
    s32 = [np.asarray(x, np.float32) for x in s_rows]
    g_hat, g_ks = _run_sss(L_list, s32, alpha, rho)
    off = np.concatenate([[0], np.cumsum(L_list)])
    for i, L in enumerate(L_list):
        srow = s32[i].astype(np.float64)
        # the kernel received alpha and rho as float32: the oracle computes with those values
        valid = valid_kstars(srow, f32(rho), orc, KSTAR_BAND_SAME_INPUT)
        assert int(g_ks[i]) in valid, (L, int(g_ks[i]), valid[:5])
        o_hat, _ = orc.sss(srow, [L], f32(alpha), f32(rho), kstar_force=[int(g_ks[i])])
        ok, worst = score_close(g_hat[off[i]:off[i + 1]], o_hat, [L])
        assert ok, (L, worst)


ALL_L = [1024, 2000, 3500, 5000, 6000, 7500, 9000, 12000, 14000, 16000, 32768]


def test_sss_matches_oracle_on_every_config_length():
    rows = []
    for L in ALL_L:
        cfg = synth.small("30b", n_layers=1, L=(L,))
        row = synth.make_row(cfg, 0, 0, 0, steps=1)
        rows.append(orc.score(row.qwin[None], row.K, [L]))
    _check_sss(ALL_L, rows, 0.5, 0.7)


def test_sss_spiky_and_small_rows():
    rng = np.random.default_rng(5)
    Ls = [64, 210, 2000, 3500]
    rows = []
    for L in Ls:
        s = rng.gamma(0.3, 1.0, L)
        s[rng.choice(L, size=max(1, L // 20), replace=False)] *= 10  # spike positions
        rows.append(s)
    for alpha, rho in [(0.5, 0.7), (0.8, 0.3), (0.3, 0.95)]:
        _check_sss(Ls, rows, alpha, rho)


def test_sss_closed_forms_on_gpu():
    rng = np.random.default_rng(6)
    Ls = [300, 1000]
    rows = [rng.random(L).astype(np.float32) for L in Ls]
    s = np.concatenate(rows)
    h, _ = _run_sss(Ls, rows, 0.0, 0.7)
    np.testing.assert_array_equal(h, s)  # alpha = 0 leaves s unchanged
    h, ks = _run_sss(Ls, rows, 0.7, 1.0)
    np.testing.assert_allclose(h, s, rtol=1e-5, atol=1e-6)  # rho = 1 reconstructs s
    h, ks = _run_sss(Ls, rows, 0.4, 0.0)
    assert (ks == 0).all()
    off = [0, 300, 1300]
    for i in range(2):
        r = rows[i].astype(np.float64)
        np.testing.assert_allclose(h[off[i]:off[i + 1]], 0.6 * r + 0.4 * r.mean(), rtol=1e-5)
    L, f = 1000, 37
    cosrow = (0.01 + 0.03 * np.cos(2 * np.pi * f * np.arange(L) / L)).astype(np.float32)
    h, ks = _run_sss([L], [cosrow], 0.6, 0.7)
    assert ks[0] == f


# ----------------------------------------------------------------- allocate --
ALLOC_CASES = [synth.CONFIGS[k] for k in ("tiny", "3b", "30b", "ragged", "long")]


@pytest.mark.parametrize("cfg", ALLOC_CASES, ids=lambda c: c.name)
def test_allocate_bit_exact(cfg):
    sh = shape_of(cfg)
    p = params_of(cfg)
    S = synth.head_scores(cfg)
    rows = cfg.rows
    b = torch.empty(rows, dtype=torch.int32, device=dev())
    off = torch.empty(rows + 1, dtype=torch.int64, device=dev())
    kv.kv_allocate(sh, cfg.L, p, up(S, torch.float32), b, off)
    torch.cuda.synchronize()
    b_orc = orc.allocate(S, cfg.L, cfg.w, cfg.budget_pct, cfg.r).reshape(-1)
    np.testing.assert_array_equal(b.cpu().numpy(), b_orc)
    np.testing.assert_array_equal(off.cpu().numpy(), np.concatenate([[0], np.cumsum(b_orc.astype(np.int64) + 1)]))
    assert off[-1].item() == kv.kv_total_slots(sh, cfg.L, p)


def test_allocate_random_scores_and_caps():
    rng = np.random.default_rng(7)
    for trial in range(20):
        H = int(rng.integers(1, 9))
        nl = int(rng.integers(1, 5))
        L = [int(x) for x in rng.choice([64, 210, 1000, 2000], size=int(rng.integers(1, 4)))]
        w = int(rng.integers(1, 9))
        pct = int(rng.integers(20, 101))
        r = float(rng.choice([0.0, 0.5, 1.0, rng.random()]))
        S = (rng.random((nl, H)) ** 3).astype(np.float32)
        if trial % 5 == 0:
            S[0] = 0
        try:
            b_orc = orc.allocate(S, L, w, pct, r).reshape(-1)
        except orc.BudgetError:
            continue
        cfg = synth.Config("a", nl, H, 1, 64, tuple(L), "f32", w=w, budget_pct=pct, r=r)
        b = torch.empty(cfg.rows, dtype=torch.int32, device=dev())
        off = torch.empty(cfg.rows + 1, dtype=torch.int64, device=dev())
        kv.kv_allocate(shape_of(cfg), L, params_of(cfg), up(S, torch.float32), b, off)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(b.cpu().numpy(), b_orc)


# ------------------------------------------------------------ select/gather --
def _select_case(L_list, s_hat_rows, b_rows, w, d=128, dtype=torch.bfloat16, seed=0):
    """Runs kv_select_gather on oracle/generator inputs; returns GPU idx, Kc, Vc per row and K, V."""
    rng = np.random.default_rng(seed)
    n_keys = sum(L_list)
    K = synth.round_bf16(rng.standard_normal((n_keys, d)).astype(np.float32))
    V = synth.round_bf16(rng.standard_normal((n_keys, d)).astype(np.float32))
    cfg = synth.Config("sel", 1, 1, 1, d, tuple(L_list), "bf16" if dtype == torch.bfloat16 else "f32", w=w)
    b = torch.tensor(b_rows, dtype=torch.int32, device=dev())
    off_h = np.concatenate([[0], np.cumsum(np.asarray(b_rows, np.int64) + 1)])
    off = torch.tensor(off_h, dtype=torch.int64, device=dev())
    total = int(off_h[-1])
    idx = torch.full((total,), -7, dtype=torch.int32, device=dev())
    Kc = torch.zeros(total, d, dtype=dtype, device=dev())
    Vc = torch.zeros(total, d, dtype=dtype, device=dev())
    s_hat = up(np.concatenate(s_hat_rows).astype(np.float32), torch.float32)
    kv.kv_select_gather(shape_of(cfg), L_list, s_hat, up(K, dtype), up(V, dtype), b, off, idx, Kc, Vc)
    torch.cuda.synchronize()
    idx_h, Kc_h, Vc_h = idx.cpu().numpy(), Kc.float().cpu().numpy(), Vc.float().cpu().numpy()
    res = []
    for i in range(len(L_list)):
        o = off_h[i]
        res.append((idx_h[o:o + b_rows[i]], Kc_h[o:o + b_rows[i]], Vc_h[o:o + b_rows[i]], idx_h[o + b_rows[i]]))
    return res, K, V


def _check_select(L_list, s_hat_rows, b_rows, w, **kw):
    res, K, V = _select_case(L_list, s_hat_rows, b_rows, w, **kw)
    koff = np.concatenate([[0], np.cumsum(L_list)])
    expect = orc.select(np.concatenate([np.asarray(r, np.float32).astype(np.float64) for r in s_hat_rows]),
                        L_list, w, b_rows)
    for i, (idx, Kc, Vc, spare) in enumerate(res):
        np.testing.assert_array_equal(idx, expect[i])
        np.testing.assert_array_equal(Kc, K[koff[i] + expect[i]])
        np.testing.assert_array_equal(Vc, V[koff[i] + expect[i]])
        assert spare == -7  # the spare decode slot is left untouched


def test_select_gather_bit_exact_random():
    rng = np.random.default_rng(11)
    Ls = [1000, 2000, 6000, 16000]
    rows = [rng.random(L) for L in Ls]
    _check_select(Ls, rows, [409, 1500, 3600, 6400], 32)


def test_select_gather_ties_signed_zero_and_edges():
    rng = np.random.default_rng(12)
    Ls = [64, 64, 256, 300, 1024, 40]
    rows = [
        np.zeros(64),  # all equal: lowest indices
        np.where(rng.random(64) < 0.5, 0.0, -0.0),  # signed zeros tie
        rng.integers(0, 3, 256).astype(np.float64),  # heavy ties
        rng.random(300) - 0.5,  # negatives
        rng.random(1024),
        rng.random(40),
    ]
    b = [20, 33, 100, 300, 8, 38]  # includes b = L (keep all) and b = w (window only)
    _check_select(Ls, rows, b, 8)


def test_select_gather_fp32_d64():
    rng = np.random.default_rng(13)
    Ls = [1024, 512]
    _check_select(Ls, [rng.random(L) for L in Ls], [409, 300], 32, d=64, dtype=torch.float32)


def test_select_long_row():
    rng = np.random.default_rng(14)
    _check_select([32768], [rng.random(32768)], [1638], 32)
