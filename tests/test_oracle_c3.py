"""Pins of the oracle's C3 row (key-space index, shared-GQA competition,
adaptive resolution): the generator's published test vector, the index
structure and centroids, a two-blob split, the frontier partition, the scores,
selection and attention against independent numpy code, the bypass, the EMA
closed form, and the split/merge exchange restated step by step."""
import numpy as np
import pytest

import oracle as orc


def test_splitmix64_test_vector():
    # SplitMix64 seeded with 0 (Steele, Lea and Flood): the first two outputs
    assert orc.splitmix64(0, 0) == 0xE220A8397B1DCDAF
    assert orc.splitmix64(0, 1) == 0x6E789E6AA1B965F4


def _row(L=2000, d=32, seed=0, **kw):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    return orc.C3Row(K, V, **kw), rng


@pytest.mark.parametrize("L", [1, 5, 17, 300, 2000])
def test_index_structure(L):
    r, _ = _row(L)
    assert r.cnt[0] == L and sorted(r.members(0).tolist()) == list(range(L))
    for n in range(r.n_nodes):
        m = r.members(n)
        np.testing.assert_allclose(r.cent[n], r.K[m].astype(np.float64).mean(0), rtol=1e-12, atol=1e-12)
        if r.left[n] < 0:
            assert r.cnt[n] <= 4 or L < 2
            assert (np.diff(m) > 0).all()  # a leaf in ascending position
        else:
            a, b = r.left[n], r.left[n] + 1
            assert a > n and r.parent[a] == r.parent[b] == n and r.depth[a] == r.depth[n] + 1
            assert r.cnt[a] > 0 and r.cnt[b] > 0
            # index order: the left child's members, then the right child's
            assert np.concatenate([r.members(a), r.members(b)]).tolist() == m.tolist()


def test_two_blobs_split_at_the_root():
    rng = np.random.default_rng(1)
    L, d = 400, 16
    blob = rng.random(L) < 0.3
    K = rng.standard_normal((L, d)).astype(np.float32) * 0.1
    K[blob, 0] += 20.0
    r = orc.C3Row(K, K)
    a, b = r.left[0], r.left[0] + 1
    got = {tuple(sorted(r.members(a).tolist())), tuple(sorted(r.members(b).tolist()))}
    assert got == {tuple(np.nonzero(blob)[0].tolist()), tuple(np.nonzero(~blob)[0].tolist())}


@pytest.mark.parametrize("L", [300, 2000, 4096])
def test_frontier_partitions_at_granularity_16(L):
    r, _ = _row(L)
    cover = np.zeros(L, int)
    for n in r.front:
        cover[r.members(n)] += 1
    assert (cover == 1).all()
    assert 16 / np.sqrt(2) - 4 <= L / r.A <= 16 * np.sqrt(2) + 4  # mean node size near 16


def _reference_step(r, q, B):
    """Scores, selection and attention restated with numpy."""
    qn = q / np.linalg.norm(q, axis=1, keepdims=True)
    c = r.cent[r.front]
    cn = c / np.linalg.norm(c, axis=1, keepdims=True)
    sigma = (qn @ cn.T).max(0)
    order = sorted(range(r.A), key=lambda i: (-sigma[i], r.front[i]))
    chosen = []
    for i in order:
        m = r.members(r.front[i]).tolist()
        chosen += m[:B - len(chosen)]
        if len(chosen) >= B:
            break
    sel = np.array(sorted(chosen))
    lg = q.astype(np.float64) @ r.K[sel].T.astype(np.float64) / np.sqrt(r.d)
    p = np.exp(lg - lg.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    return sigma, sel, p @ r.V[sel].astype(np.float64)


def test_scores_selection_and_attention():
    r, rng = _row(3000, 64)
    for t in range(5):
        q = rng.standard_normal((4, 64)).astype(np.float32)
        sig_ref, sel_ref, o_ref = _reference_step(r, q.astype(np.float64), 300)
        o, sel, sig = r.step(q, 300)
        np.testing.assert_allclose(sig, sig_ref, rtol=1e-12, atol=1e-14)
        assert sel.tolist() == sel_ref.tolist() and len(sel) == 300
        np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)


def test_bypass_keeps_everything_and_state():
    r, rng = _row(200, 16)
    front, e = r.front.copy(), r.e.copy()
    q = rng.standard_normal((2, 16)).astype(np.float32)
    o, sel, _ = r.step(q, 200)
    assert sel.tolist() == list(range(200))
    lg = q.astype(np.float64) @ r.K.T.astype(np.float64) / 4.0
    p = np.exp(lg - lg.max(1, keepdims=True))
    np.testing.assert_allclose(o, (p / p.sum(1, keepdims=True)) @ r.V.astype(np.float64), rtol=1e-10)
    assert (r.front == front).all() and (r.e == e).all()


def test_ema_closed_form_without_exchanges():
    r, rng = _row(2000, 32)
    q = rng.standard_normal((3, 32)).astype(np.float32)
    front0 = r.front.copy()
    for t in range(1, 6):
        _, _, sig = r.step(q, 128, lam=0.5, R=0)
        assert (r.front == front0).all()
        np.testing.assert_allclose(r.e[front0], (1 - 0.5 ** t) * sig, rtol=1e-12)


def test_lambda_one_never_absorbs():
    r, rng = _row(2000, 32)
    for t in range(4):
        r.step(rng.standard_normal((2, 32)).astype(np.float32), 128, lam=1.0, R=2)
    assert (r.e == 0).all()


@pytest.mark.parametrize("R", [1, 2, 4])
def test_exchanges_restated(R):
    r, rng = _row(3000, 32, seed=R)
    lam = 0.5
    for t in range(12):
        front, e = r.front.copy(), r.e.copy()
        q = rng.standard_normal((4, 32)).astype(np.float32)
        _, _, sig = r.step(q, 256, lam=lam, R=R)
        # restate: EMA, then R rounds of (split argmax e, merge argmin max-e sibling pair)
        e[front] = lam * e[front] + (1 - lam) * sig
        on, fresh = set(front.tolist()), set()
        for _ in range(R):
            cand = [n for n in on if n not in fresh and r.left[n] >= 0]
            if not cand:
                break
            s = min(cand, key=lambda n: (-e[n], n))
            pairs = [p for p in range(r.n_nodes) if r.left[p] >= 0 and {r.left[p], r.left[p] + 1} <= on
                     and not ({r.left[p], r.left[p] + 1} & fresh) and s not in (r.left[p], r.left[p] + 1)]
            if not pairs:
                break
            p = min(pairs, key=lambda p: (max(e[r.left[p]], e[r.left[p] + 1]), p))
            pv = max(e[r.left[p]], e[r.left[p] + 1])
            c = r.left[s]
            on -= {s, r.left[p], r.left[p] + 1}
            on |= {c, c + 1, p}
            fresh |= {c, c + 1, p}
            e[c] = e[c + 1] = e[s]
            e[p] = pv
        assert sorted(on) == r.front.tolist(), t
        np.testing.assert_array_equal(r.e[r.front], e[r.front])
        assert len(r.front) == len(front)  # A is fixed
        cover = np.zeros(r.L, int)
        for n in r.front:
            cover[r.members(n)] += 1
        assert (cover == 1).all()


@pytest.mark.parametrize("seed", [0, 3])
def test_root_split_is_eight_lloyd_iterations(seed):
    """The root's children equal an independent numpy 2-means (8 iterations) from the
    two member keys SplitMix64 picks for node 0."""
    r, _ = _row(700, 24, seed=seed)
    n = r.L
    i0 = orc.splitmix64(0, 0) % n
    i1 = (i0 + 1 + orc.splitmix64(0, 1) % (n - 1)) % n
    X = r.K.astype(np.float64)
    c = np.stack([X[i0], X[i1]])
    for _ in range(8):
        dist = ((X[:, None, :] - c[None]) ** 2).sum(-1)
        side = (dist[:, 1] < dist[:, 0]).astype(int)
        for k in (0, 1):
            if (side == k).any():
                c[k] = X[side == k].mean(0)
    a = r.left[0]
    assert sorted(r.members(a).tolist()) == np.nonzero(side == 0)[0].tolist()
    assert sorted(r.members(a + 1).tolist()) == np.nonzero(side == 1)[0].tolist()


def test_resolution_levels_32_16_8_4():
    """The cuts one level above and one and two below the initial frontier have mean node
    sizes near 32, 8 and 4 (the resolutions the page lists around granularity 16)."""
    r, _ = _row(4096, 32)
    D0 = int(r.depth[r.front].max())
    for D, want in ((D0 - 1, 32), (D0, 16), (D0 + 1, 8), (D0 + 2, 4)):
        cut = [n for n in range(r.n_nodes) if r.depth[n] == D or (r.depth[n] < D and r.left[n] < 0)]
        assert sum(r.cnt[n] for n in cut) == r.L  # every cut partitions the keys
        assert want / 1.6 <= r.L / len(cut) <= want * 1.6, (D, r.L / len(cut))
