"""Parity of the variants of steps 3 and 4 with the oracle, bit for bit:
kv_allocate_global (one allocation over all layers of a sequence) and
kv_select_gather_segmented (WnW's segment-wise static subset)."""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._harness import dev, params_of, shape_of, up

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "3b", "30b", "ragged", "long"])
def test_allocate_global_bit_exact(name):
    cfg = synth.CONFIGS[name]
    S = synth.head_scores(cfg)
    b = torch.empty(cfg.rows, dtype=torch.int32, device=dev())
    off = torch.empty(cfg.rows + 1, dtype=torch.int64, device=dev())
    kv.kv_allocate_global(shape_of(cfg), cfg.L, params_of(cfg), up(S, torch.float32), b, off)
    torch.cuda.synchronize()
    b_orc = orc.allocate_global(S, cfg.L, cfg.w, cfg.budget_pct, cfg.r).reshape(-1)
    np.testing.assert_array_equal(b.cpu().numpy(), b_orc)
    np.testing.assert_array_equal(off.cpu().numpy(), np.concatenate([[0], np.cumsum(b_orc.astype(np.int64) + 1)]))
    assert off[-1].item() == kv.kv_total_slots(shape_of(cfg), cfg.L, params_of(cfg))  # the same total


def test_allocate_global_random_scores_and_caps():
    rng = np.random.default_rng(17)
    for trial in range(20):
        H, nl = int(rng.integers(1, 9)), int(rng.integers(1, 7))
        L = [int(x) for x in rng.choice([64, 210, 1000, 2000], size=int(rng.integers(1, 4)))]
        w, pct = int(rng.integers(1, 9)), int(rng.integers(20, 101))
        r = float(rng.choice([0.0, 0.5, 1.0, rng.random()]))
        S = (rng.random((nl, H)) ** 4).astype(np.float32)  # skewed: some heads hit L and are capped
        if trial % 5 == 0:
            S[0] = 0
        try:
            b_orc = orc.allocate_global(S, L, w, pct, r).reshape(-1)
        except orc.BudgetError:
            continue
        cfg = synth.Config("a", nl, H, 1, 64, tuple(L), "f32", w=w, budget_pct=pct, r=r)
        b = torch.empty(cfg.rows, dtype=torch.int32, device=dev())
        off = torch.empty(cfg.rows + 1, dtype=torch.int64, device=dev())
        kv.kv_allocate_global(shape_of(cfg), L, params_of(cfg), up(S, torch.float32), b, off)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(b.cpu().numpy(), b_orc, err_msg=f"trial {trial}")


def _check_segmented(L_list, s_rows, b_rows, w, nseg, d=128, seed=0):
    rng = np.random.default_rng(seed)
    K = synth.round_bf16(rng.standard_normal((sum(L_list), d)).astype(np.float32))
    V = synth.round_bf16(rng.standard_normal((sum(L_list), d)).astype(np.float32))
    cfg = synth.Config("seg", 1, 1, 1, d, tuple(L_list), "bf16", w=w)
    b = torch.tensor(b_rows, dtype=torch.int32, device=dev())
    off_h = np.concatenate([[0], np.cumsum(np.asarray(b_rows, np.int64) + 1)])
    off = torch.tensor(off_h, dtype=torch.int64, device=dev())
    total = int(off_h[-1])
    idx = torch.full((total,), -7, dtype=torch.int32, device=dev())
    Kc = torch.zeros(total, d, dtype=torch.bfloat16, device=dev())
    Vc = torch.zeros(total, d, dtype=torch.bfloat16, device=dev())
    s32 = np.concatenate(s_rows).astype(np.float32)
    kv.kv_select_gather_segmented(shape_of(cfg), L_list, up(s32, torch.float32), up(K, torch.bfloat16),
                                  up(V, torch.bfloat16), b, off, nseg, idx, Kc, Vc)
    torch.cuda.synchronize()
    expect = orc.select_segmented(s32.astype(np.float64), L_list, w, b_rows, nseg)
    idx_h, Kc_h, Vc_h = idx.cpu().numpy(), Kc.float().cpu().numpy(), Vc.float().cpu().numpy()
    koff = np.concatenate([[0], np.cumsum(L_list)])
    for i in range(len(L_list)):
        o, n = off_h[i], min(b_rows[i], L_list[i])
        np.testing.assert_array_equal(idx_h[o:o + n], expect[i], err_msg=f"row {i} nseg {nseg}")
        np.testing.assert_array_equal(Kc_h[o:o + n], K[koff[i] + expect[i]])
        np.testing.assert_array_equal(Vc_h[o:o + n], V[koff[i] + expect[i]])


@pytest.mark.parametrize("nseg", [1, 3, 16, 257])
def test_select_segmented_bit_exact(nseg):
    rng = np.random.default_rng(nseg)
    Ls = [1000, 2000, 6000, 16000]
    rows = [rng.random(L).astype(np.float32) for L in Ls]
    rows[1] = np.round(rows[1] * 8).astype(np.float32)  # heavy ties
    _check_segmented(Ls, rows, [409, 1500, 3600, 6400], 32, nseg)


def test_select_segmented_edges():
    rng = np.random.default_rng(3)
    Ls = [64, 1000, 2000, 2000]
    rows = [rng.standard_normal(L).astype(np.float32) for L in Ls]
    rows[2][:] = 0.0
    rows[2][::3] = -0.0  # signed zeros are equal
    # b = L (bypass), b = w (window only), one candidate per segment, more segments than kept
    _check_segmented(Ls, rows, [64, 32, 1000, 500], 32, 1968)
    _check_segmented(Ls, rows, [50, 33, 999, 1999], 32, 7)
