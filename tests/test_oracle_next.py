"""Pins of the oracle's variants of steps 3 and 4: one allocation over every
(layer, head) of a sequence, and segment-wise selection (WnW fixed heads)."""
import numpy as np
import pytest

import oracle as orc


# ---------------------------------------------------------------- allocation
def test_allocate_global_hand_example():
    # 2 layers x 2 heads, L = 100, w = 4, 50 %: B = 2 * 100 = 200, B_rem = 200 - 4 * 4 = 184;
    # r = 1/2: x_h = 4 + 92 / 4 + 92 S_h / 4 = 27 + 23 S_h for S = (1, 1, 2, 0)
    S = np.array([[1, 1], [2, 0]], np.float32)
    b = orc.allocate_global(S, [100], 4, 50, 0.5)
    assert b.reshape(-1).tolist() == [50, 50, 73, 27]


def test_allocate_global_cap_and_reallocate():
    # head 0 asks 4 + 23 + 92 = 119 > L = 100: capped; the other three split 100 evenly
    # (ΣS = 0 among them): 4 + 88 / 3 = 33.33 each, the one extra slot to the lowest head
    S = np.array([[10, 0], [0, 0]], np.float32)
    b = orc.allocate_global(S, [100], 4, 50, 0.5)
    assert b.reshape(-1).tolist() == [100, 34, 33, 33]


@pytest.mark.parametrize("seed", range(5))
def test_allocate_global_invariants(seed):
    rng = np.random.default_rng(seed)
    n_layers, H, w = int(rng.integers(1, 6)), int(rng.integers(1, 9)), 32
    S = rng.random((n_layers, H)).astype(np.float32)
    L = [int(x) for x in rng.integers(400, 4000, size=3) // 2 * 2]
    pct = int(rng.integers(20, 90))
    b = orc.allocate_global(S, L, w, pct, float(rng.random()))
    for s, Ls in enumerate(L):
        assert b[s].sum() == n_layers * ((pct * Ls * H) // 100)  # the per-layer total, shared
        assert (b[s] >= w).all() and (b[s] <= Ls).all()


def test_allocate_global_one_layer_is_per_layer():
    S = np.random.default_rng(3).random((1, 8)).astype(np.float32)
    np.testing.assert_array_equal(orc.allocate_global(S, [3000, 5000], 32, 40, 0.5),
                                  orc.allocate(S, [3000, 5000], 32, 40, 0.5))


def test_allocate_global_r1_is_even():
    S = np.random.default_rng(4).random((4, 4)).astype(np.float32)
    b = orc.allocate_global(S, [6000], 32, 60, 1.0).reshape(-1)
    assert b.max() - b.min() <= 1 and b.sum() == 4 * (60 * 6000 * 4 // 100)


# ---------------------------------------------------------------- selection
def test_select_segmented_one_segment_is_select():
    rng = np.random.default_rng(5)
    s = rng.standard_normal(3000)
    s[::7] = s[3]  # ties
    for b in (32, 33, 500, 2999, 3000):
        np.testing.assert_array_equal(orc.select_segmented(s, [3000], 32, [b], 1)[0],
                                      orc.select(s, [3000], 32, [b])[0])


def test_select_segmented_hand_quotas():
    # L = 20, w = 4: candidates 0..15 in segments [0,5), [5,10), [10,16); b = 11 keeps k = 7:
    # floor(7*5/16) = 2, 2, floor(7*6/16) = 2 (remainders 3, 3, 10) -> the extra one to
    # segment 2: quotas (2, 2, 3). With s_hat = -j the lowest positions of each segment win.
    s = -np.arange(20, dtype=np.float64)
    idx = orc.select_segmented(s, [20], 4, [11], 3)[0]
    assert idx.tolist() == [0, 1, 5, 6, 10, 11, 12, 16, 17, 18, 19]


def test_select_segmented_unit_segments_take_the_first():
    # one candidate per segment: every quota is floor(k / n) = 0 with remainder k, so the
    # k extra slots go to the lowest segments whatever the scores
    s = np.random.default_rng(6).standard_normal(40)
    idx = orc.select_segmented(s, [40], 8, [13], 32)[0]
    assert idx.tolist() == list(range(5)) + list(range(32, 40))


@pytest.mark.parametrize("nseg", [2, 5, 16])
def test_select_segmented_best_within_each_segment(nseg):
    rng = np.random.default_rng(nseg)
    L, w, b = 2000, 32, 700
    s = np.round(rng.standard_normal(L), 1)  # many ties
    idx = orc.select_segmented(s, [L], w, [b], nseg)[0]
    n, k = L - w, b - w
    assert len(idx) == b and (np.diff(idx) > 0).all() and set(range(n, L)) <= set(idx.tolist())
    kept = set(idx.tolist())
    total = 0
    for i in range(nseg):
        lo, hi = i * n // nseg, (i + 1) * n // nseg
        seg_kept = [j for j in range(lo, hi) if j in kept]
        seg_drop = [j for j in range(lo, hi) if j not in kept]
        q = len(seg_kept)
        total += q
        assert abs(q - k * (hi - lo) / n) < 1.0  # the quota follows the segment's share
        if seg_kept and seg_drop:  # no dropped position beats a kept one (ties: lower index kept)
            worst_kept = min(seg_kept, key=lambda j: (s[j], -j))
            best_drop = max(seg_drop, key=lambda j: (s[j], -j))
            assert (s[worst_kept], -worst_kept) > (s[best_drop], -best_drop)
    assert total == k


def test_select_segmented_bypass_and_window_only():
    s = np.random.default_rng(7).standard_normal(100)
    assert orc.select_segmented(s, [100], 8, [100], 4)[0].tolist() == list(range(100))
    assert orc.select_segmented(s, [100], 8, [8], 4)[0].tolist() == list(range(92, 100))
