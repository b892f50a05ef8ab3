"""Pins of the oracle's WnW step (anchor-chunk importance, top-3 selection,
3-step release hysteresis, block slots of the tidal heads' GPU copy):
the chunk layout by brute force, hand-worked steps, a release timeline,
chunk scores against an independent sum, and the residency invariants."""
import numpy as np
import pytest

import oracle as orc

C, S = 50, 25  # 4 s chunks, 2 s apart, at 12.5 audio tokens/s


@pytest.mark.parametrize("L", [1, 24, 25, 49, 50, 51, 74, 75, 76, 110, 1000, 32768])
def test_chunk_layout(L):
    st = orc.WnwState(L, C, S, 3, 3, 18)
    # brute force: the fewest chunks [m S, m S + C) that reach the last position
    M = 1
    while (M - 1) * S + C < L:
        M += 1
    assert st.M == M and st.nb == -(-L // S)
    cover = np.zeros(L, int)
    for m in range(M):
        cover[m * S:min(m * S + C, L)] += 1
    assert (cover >= 1).all() and (cover <= C // S).all()


def test_hand_step():
    st = orc.WnwState(110, C, S, 3, 3, 18)
    s = np.zeros((2, 110), np.float32)
    s[0, 80:90] = 1.0
    s[1, 99] = 0.5
    score, sel, fetch, release = st.step(s)
    # chunks [0,50) [25,75) [50,100) [75,110): 0, 0, 10 + 0.5, 10 + 0.5 -> 2 and 3 tie (lower first), then 0
    assert score.tolist() == [0.0, 0.0, 10.5, 10.5]
    assert sel.tolist() == [2, 3, 0]
    # chunks 0, 2, 3 hold blocks 0, 1 and 2, 3 and 3, 4: all five blocks, slots in block order
    assert fetch.tolist() == [[0, 0], [1, 1], [2, 2], [3, 3], [4, 4]] and len(release) == 0


def test_release_after_three_idle_steps():
    L = 400  # 15 chunks, 16 blocks
    st = orc.WnwState(L, C, S, 1, 3, 6)
    def focus(a, b):
        s = np.zeros((1, L), np.float32)
        s[0, a:b] = 1.0
        return s

    timeline = []
    for t in range(6):
        s = focus(0, 10) if t == 0 else focus(300, 310)  # chunk 0 once, then chunk 11 (ties to the lower of 11, 12)
        _, sel, fetch, release = st.step(s)
        timeline.append((sel.tolist(), fetch.tolist(), release.tolist(), st.idle[0]))
    assert timeline[0] == ([0], [[0, 0], [1, 1]], [], 0)
    assert timeline[1] == ([11], [[11, 2], [12, 3]], [], 1)
    assert timeline[2] == ([11], [], [], 2)
    assert timeline[3] == ([11], [], [[0, 0], [1, 1]], -1)  # third idle step: released
    assert timeline[4] == ([11], [], [], -1)


def test_scores_against_an_independent_sum():
    rng = np.random.default_rng(0)
    L = 1234
    s = rng.random((5, L)).astype(np.float32) * np.float32(1e-3)
    st = orc.WnwState(L, C, S, 3, 3, 18)
    score, sel, _, _ = st.step(s)
    tot = s.astype(np.float64).sum(0)
    ref = np.array([tot[m * S:min(m * S + C, L)].sum() for m in range(st.M)])
    np.testing.assert_allclose(score, ref, rtol=1e-12)
    assert sel.tolist() == np.lexsort((np.arange(st.M), -score))[:3].tolist()


def test_ties_and_few_chunks():
    st = orc.WnwState(1000, C, S, 3, 3, 18)
    _, sel, _, _ = st.step(np.zeros((2, 1000), np.float32))
    assert sel.tolist() == [0, 1, 2]
    st2 = orc.WnwState(60, C, S, 3, 3, 18)  # two chunks
    _, sel2, fetch2, _ = st2.step(np.ones((1, 60), np.float32))
    assert sorted(sel2.tolist()) == [0, 1] and fetch2[:, 0].tolist() == [0, 1, 2]


@pytest.mark.parametrize("seed", range(3))
def test_residency_invariants(seed):
    rng = np.random.default_rng(seed)
    L, top_c, R = 5000, 3, 3
    n_slots = top_c * R * (C // S)
    st = orc.WnwState(L, C, S, top_c, R, n_slots)
    for t in range(60):
        s = (rng.random((5, L)) ** 8).astype(np.float32)
        before = st.block_slot.copy()
        _, sel, fetch, release = st.step(s)
        assert (st.idle[sel] == 0).all()
        assert ((st.idle >= 0).sum()) <= top_c * R
        assert (before[fetch[:, 0]] < 0).all() and (st.block_slot[fetch[:, 0]] == fetch[:, 1]).all()
        assert (before[release[:, 0]] == release[:, 1]).all() and (st.block_slot[release[:, 0]] < 0).all()
        used = st.block_slot[st.block_slot >= 0]
        assert len(set(used.tolist())) == len(used) <= n_slots
        for b in np.nonzero(st.block_slot >= 0)[0]:
            assert st.slot_block[st.block_slot[b]] == b
            # resident iff a resident chunk holds it
            assert any(st.idle[m] >= 0 for m in range(max(0, b - 1), min(b, st.M - 1) + 1))
        assert (st.slot_block >= 0).sum() == len(used)
        for m in np.nonzero(st.idle >= 0)[0]:  # and every block of a resident chunk is resident
            assert (st.block_slot[m:min(m + C // S, st.nb)] >= 0).all()
