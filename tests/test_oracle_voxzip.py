"""Pins of the oracle's VoxZip first stage (semantic-anchored pooling of the
audio features): hand-worked layouts, the timestamp-to-index map on exact
timings, the mean checked through the mass each group carries, the background
left verbatim, and the edge cases of the readings (confidence cut, overlap,
more text tokens than audio tokens)."""
import numpy as np
import pytest

import oracle as orc
import synth


def _one(L, d=2, segs=(), E_T=None, tau_total=None, conf_min=0.3):
    E = np.arange(L, dtype=np.float64)[:, None] * np.ones((1, d)) + np.arange(d)[None, :] * 1000.0
    tau = np.array([s[0:2] for s in segs], np.float64).reshape(-1, 2)
    conf = np.array([s[2] for s in segs], np.float32)
    n_text = np.array([s[3] for s in segs], np.int32)
    text_row = np.concatenate([[0], np.cumsum(n_text)[:-1]]).astype(np.int32) if len(segs) else np.zeros(0, np.int32)
    return E, orc.voxzip_pool(E, float(L if tau_total is None else tau_total), tau, conf, n_text, text_row, E_T,
                              conf_min)


def test_hand_example():
    # L = 10 tokens over 10 s: [2.5 s, 7.9 s) -> tokens [2, 7); 2 text tokens -> groups [2, 4), [4, 7)
    E_T = np.array([[100.0, 200.0], [1000.0, 2000.0]])
    E, (out, src) = _one(10, segs=[(2.5, 7.9, 0.9, 2)], E_T=E_T)
    assert src.tolist() == [[0, 1, -1], [1, 1, -1], [2, 2, 0], [4, 3, 1], [7, 1, -1], [8, 1, -1], [9, 1, -1]]
    np.testing.assert_array_equal(out[2], [2.5 + 100, 1002.5 + 200])
    np.testing.assert_array_equal(out[3], [5.0 + 1000, 1005.0 + 2000])
    np.testing.assert_array_equal(out[[0, 1, 4, 5, 6]], E[[0, 1, 7, 8, 9]])


def test_no_segment_and_low_confidence_are_identity():
    E, (out, src) = _one(37)
    np.testing.assert_array_equal(out, E)
    assert (src[:, 0] == np.arange(37)).all() and (src[:, 1] == 1).all() and (src[:, 2] == -1).all()
    # confidence must exceed the cut: float32(0.3) itself is dropped, the next float32 is kept
    c = float(np.float32(0.3))
    _, (out2, _) = _one(37, segs=[(3, 20, c, 2)])
    np.testing.assert_array_equal(out2, E)
    _, (out3, _) = _one(37, segs=[(3, 20, float(np.nextafter(np.float32(0.3), np.float32(1))), 2)])
    assert len(out3) == 37 - 17 + 2


def test_timestamp_map_exact_timings():
    # tau_total = 2 L: token t spans [2t, 2t + 2) s; floor(L * tau / (2 L)) = floor(tau / 2)
    L = 50
    segs = [(4.0, 9.99, 0.5, 1), (10.0, 10.0, 0.5, 1), (11.0, 30.0, 0.5, 3), (-5.0, 1.0, 0.9, 1),
            (98.0, 1e9, 0.9, 2)]
    _, (out, src) = _one(L, segs=segs, tau_total=2 * L)
    pooled = src[src[:, 2] >= 0]
    # [2, 4) one group; [5, 5) empty (not kept); [5, 15) in 3 groups; [0, 0) empty; [49, 50) one group
    assert pooled[:, :2].tolist() == [[2, 2], [5, 3], [8, 3], [11, 4], [49, 1]]
    assert len(out) == L - 2 - 10 - 1 + 1 + 3 + 1


def test_overlap_starts_at_the_earlier_end():
    # [5, 20) then [10, 30): the second starts at 20; an earlier-starting one inside is emptied
    segs = [(5, 20, 0.9, 3), (10, 30, 0.9, 2), (12, 18, 0.9, 4)]
    _, (out, src) = _one(40, segs=segs)
    pooled = src[src[:, 2] >= 0]
    assert pooled[:, :2].tolist() == [[5, 5], [10, 5], [15, 5], [20, 5], [25, 5]]
    assert pooled[:, 2].tolist() == [0, 1, 2, 3, 4]
    covered = np.zeros(40, int)
    for lo, n, _ in src:
        covered[lo:lo + n] += 1
    assert (covered == 1).all()  # every token lands in exactly one output row


def test_more_text_than_tokens_is_one_token_per_group():
    E_T = np.arange(16, dtype=np.float64).reshape(8, 2) * 0.5
    E, (out, src) = _one(12, segs=[(3, 6, 0.9, 8)], E_T=E_T)
    pooled = src[src[:, 2] >= 0]
    assert pooled.tolist() == [[3, 1, 0], [4, 1, 1], [5, 1, 2]]
    np.testing.assert_array_equal(out[3:6], E[3:6] + E_T[:3])


@pytest.mark.parametrize("seed", range(4))
def test_random_layout_invariants(seed):
    L, d = 3000, 16
    a = synth.asr_segments(seed, L)
    rng = np.random.default_rng(seed)
    E = rng.standard_normal((L, d))
    E_T = rng.standard_normal((int(a.n_text.sum()), d))
    out, src = orc.voxzip_pool(E, a.tau_total, a.tau, a.conf, a.n_text, a.text_row, E_T)
    covered = np.zeros(L, int)
    for lo, n, _ in src:
        covered[lo:lo + n] += 1
    assert (covered == 1).all()
    assert (np.diff(src[:, 0]) > 0).all()  # time order
    # each row carries the mass of its tokens: (row - text) * count = sum of the group's features
    mass = np.zeros(d)
    for r, (lo, n, tr) in enumerate(src):
        row = out[r] - (E_T[tr] if tr >= 0 else 0.0)
        np.testing.assert_allclose(row * n, E[lo:lo + n].sum(0), rtol=1e-12, atol=1e-12)
        mass += row * n
    np.testing.assert_allclose(mass, E.sum(0), rtol=1e-10, atol=1e-10)
    # groups of one segment differ in size by at most one and follow each other
    pooled = src[src[:, 2] >= 0]
    seg_of = np.searchsorted(a.text_row, pooled[:, 2], side="right") - 1
    for i in np.unique(seg_of):
        rows = pooled[seg_of == i]
        assert rows[0, 2] == a.text_row[i]  # group j takes text row text_row + j
        assert (np.diff(rows[:, 2]) == 1).all()
        if len(rows):
            assert rows[:, 1].max() - rows[:, 1].min() <= 1
            assert (rows[1:, 0] == rows[:-1, 0] + rows[:-1, 1]).all()
    # about a quarter of the speech tokens remain (3 text tokens/s against 12.5 audio tokens/s)
    pooled = src[src[:, 2] >= 0]
    assert 0.15 < len(pooled) / pooled[:, 1].sum() < 0.3
