"""Pins for the oracle's budget allocation, top-k selection and decode step.

Allocation: hand-worked examples (tests/golden/allocate_examples.json) plus
invariants. Selection: brute force over all subsets on tiny rows. Decode:
full attention via torch float64 when nothing is evicted, closed forms for the
decayed score sum, V = 1, the C3 retained-mass identity, and brute-force
checks of which entry the eviction rule removes.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------- allocate ----
def test_allocate_golden(orc):
    for c in json.load(open(os.path.join(GOLDEN, "allocate_examples.json")))["cases"]:
        S = np.array([c["S"]], np.float32)
        b = orc.allocate(S, [c["L"]], c["w"], c["budget_pct"], c["r"])
        assert b[0, 0].tolist() == c["b"], c["note"]


@pytest.mark.parametrize("seed", range(6))
def test_allocate_invariants(orc, seed):
    rng = np.random.default_rng(seed)
    n_layers, H = 5, int(rng.integers(1, 9))
    S = rng.random((n_layers, H)).astype(np.float32) * (rng.random() * 10)
    if seed == 3:
        S[2] = 0.0  # an all-zero layer splits evenly
    L = [int(rng.integers(200, 5000)) for _ in range(2)]
    w = 32
    pct = int(rng.integers(5, 101))
    r = float(rng.random())
    try:
        b = orc.allocate(S, L, w, pct, r)
    except orc.BudgetError:
        for Ls in L:
            assert (pct * Ls * H) // 100 < H * w
        return
    for si, Ls in enumerate(L):
        B = (pct * Ls * H) // 100
        assert (b[si].sum(axis=1) == B).all()
        assert (b[si] >= w).all() and (b[si] <= Ls).all()


def test_allocate_r_one_is_even(orc):
    S = np.random.default_rng(3).random((4, 6)).astype(np.float32)
    b = orc.allocate(S, [3000], 32, 37, 1.0)
    assert (b.max(axis=2) - b.min(axis=2) <= 1).all()


def test_allocate_r_zero_is_proportional(orc):
    S = np.random.default_rng(4).random((3, 5)).astype(np.float32)
    L, w, pct, H = 4000, 32, 30, 5
    b = orc.allocate(S, [L], w, pct, 0.0)
    B = (pct * L * H) // 100
    B_rem = B - H * w
    for l in range(3):
        x = w + B_rem * S[l].astype(np.float64) / S[l].astype(np.float64).sum()
        assert (np.abs(b[0, l] - x) < 1.0).all()


def test_allocate_budget_error(orc):
    with pytest.raises(orc.BudgetError):
        orc.allocate(np.ones((1, 4), np.float32), [100], 32, 10, 0.5)


# ----------------------------------------------------------------- select ----
def _brute_topk(v, k):
    """The unique k-subset whose every member beats every non-member under
    (value descending, index ascending), found by enumerating all subsets."""
    n = len(v)
    found = []
    for sub in itertools.combinations(range(n), k):
        inside = set(sub)
        ok = all((v[i] > v[j]) or (v[i] == v[j] and i < j)
                 for i in inside for j in range(n) if j not in inside)
        if ok:
            found.append(sub)
    assert len(found) == 1
    return list(found[0])


@pytest.mark.parametrize("seed", range(12))
def test_select_brute_force(orc, seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(4, 13))
    w = int(rng.integers(0, min(4, L)))
    b = int(rng.integers(w, L + 1))
    v = rng.integers(0, 4, size=L).astype(np.float64)  # many ties
    idx = orc.select(v, [L], w, [b])[0]
    expect = sorted(_brute_topk(v[:L - w], b - w) + list(range(L - w, L))) if b < L else list(range(L))
    assert idx.tolist() == expect


def test_select_properties_large(orc):
    rng = np.random.default_rng(20)
    L, w, b = 6000, 32, 3600
    v = rng.random(L)
    idx = orc.select(v, [L], w, [b])[0]
    assert len(idx) == b and (np.diff(idx) > 0).all()
    assert set(range(L - w, L)) <= set(idx.tolist())
    chosen = np.setdiff1d(idx, np.arange(L - w, L))
    rest = np.setdiff1d(np.arange(L - w), chosen)
    assert v[chosen].min() >= v[rest].max()


def test_select_all_equal_takes_lowest(orc):
    L, w, b = 100, 8, 30
    idx = orc.select(np.full(L, 0.25), [L], w, [b])[0]
    assert idx.tolist() == list(range(22)) + list(range(92, 100))


def test_select_signed_zero_ties(orc):
    v = np.array([0.0, -0.0, -0.0, 0.0, -1.0, 0.0])
    idx = orc.select(v, [6], 0, [3])[0]
    assert idx.tolist() == [0, 1, 2]


def test_select_budget_at_least_L_keeps_all(orc):
    idx = orc.select(np.random.default_rng(0).random(50), [50], 4, [50])[0]
    assert idx.tolist() == list(range(50))


# ----------------------------------------------------------------- decode ----
def _rand_cache(rng, n, d):
    K = rng.standard_normal((n, d)).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32)
    pos = np.sort(rng.choice(10 * n, size=n, replace=False)).astype(np.int64)
    return K, V, pos


def test_decode_no_eviction_is_full_attention(orc):
    rng = np.random.default_rng(30)
    n, d, g, steps = 50, 64, 4, 6
    K, V, pos = _rand_cache(rng, n, d)
    lst = orc.DecodeList(K, V, pos, extra=steps)
    Kall, Vall = K.copy(), V.copy()
    for t in range(steps):
        q = rng.standard_normal((g, d)).astype(np.float32)
        k = rng.standard_normal(d).astype(np.float32)
        v = rng.standard_normal(d).astype(np.float32)
        o, ev = lst.step(q, k, v, 10 * n + t, gamma=0.95, T=4, M=5, b=n + steps)
        assert ev == -1
        Kall = np.vstack([Kall, k])
        Vall = np.vstack([Vall, v])
        x = torch.from_numpy(q).double() @ torch.from_numpy(Kall).double().T / math.sqrt(d)
        ref = torch.softmax(x, -1) @ torch.from_numpy(Vall).double()
        np.testing.assert_allclose(o, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_decode_value_one_gives_one(orc):
    rng = np.random.default_rng(31)
    n, d, g = 40, 32, 3
    K, _, pos = _rand_cache(rng, n, d)
    lst = orc.DecodeList(K, np.ones((n, d), np.float32), pos)
    for t in range(5):
        o, _ = lst.step(rng.standard_normal((g, d)), rng.standard_normal(d), np.ones(d), 1000 + t, 0.9, 4, 6, n)
        np.testing.assert_allclose(o, 1.0, rtol=1e-13)


@pytest.mark.parametrize("gamma", [0.95, 1.0, 0.5])
def test_decode_decayed_sum_closed_form(orc, gamma):
    # without eviction, sum_j A_j = g (1 - gamma^t) / (1 - gamma) (g t at gamma = 1)
    rng = np.random.default_rng(32)
    n, d, g, steps = 30, 16, 5, 9
    K, V, pos = _rand_cache(rng, n, d)
    lst = orc.DecodeList(K, V, pos, extra=steps)
    for t in range(1, steps + 1):
        lst.step(rng.standard_normal((g, d)), rng.standard_normal(d), rng.standard_normal(d), 10 ** 6 + t, gamma,
                 2, 2, n + steps)
        A = lst.entries()[2]
        expect = g * t if gamma == 1.0 else g * (1 - gamma ** t) / (1 - gamma)
        assert abs(A.sum() - expect) < 1e-12 * expect


def test_decode_c3_retained_mass_identity(orc):
    # C3: o_R - o = (1 - rho)(o_R - o_{R^c}) with rho the full-attention mass on R
    rng = np.random.default_rng(33)
    n, d, g = 60, 32, 1
    K, V, pos = _rand_cache(rng, n, d)
    q = rng.standard_normal((g, d)).astype(np.float32)
    kn, vn = rng.standard_normal(d).astype(np.float32), rng.standard_normal(d).astype(np.float32)
    R = np.sort(rng.choice(n, size=25, replace=False))
    o_full, _ = orc.DecodeList(K, V, pos).step(q, kn, vn, 10 ** 6, 0.9, 0, 0, n + 1)
    o_R, _ = orc.DecodeList(K[R], V[R], pos[R]).step(q, kn, vn, 10 ** 6, 0.9, 0, 0, n + 1)
    # mass of R (plus the appended entry, which both lists hold) in the full softmax
    x = (np.vstack([K, kn]).astype(np.float64) @ q[0].astype(np.float64)) / math.sqrt(d)
    p = np.exp(x - x.max())
    p /= p.sum()
    inR = np.zeros(n + 1, bool)
    inR[R] = True
    inR[n] = True
    rho = p[inR].sum()
    Vall = np.vstack([V, vn]).astype(np.float64)
    o_comp = (p[~inR, None] * Vall[~inR]).sum(0) / (1 - rho)
    np.testing.assert_allclose(o_R[0] - o_full[0], (1 - rho) * (o_R[0] - o_comp), rtol=1e-9, atol=1e-12)


def _middle(pos_sorted, T, M):
    n = len(pos_sorted)
    return list(range(T, n - M))


@pytest.mark.parametrize("seed", range(8))
def test_decode_eviction_removes_middle_argmin(orc, seed):
    rng = np.random.default_rng(40 + seed)
    n, d, g = 24, 8, 2
    T, M, b = 3, 5, n
    K, V, pos = _rand_cache(rng, n, d)
    lst = orc.DecodeList(K, V, pos)
    for t in range(12):
        _, _, A_before, pos_before = lst.entries()
        q = rng.standard_normal((g, d)).astype(np.float32)
        kn, vn = rng.standard_normal(d).astype(np.float32), rng.standard_normal(d).astype(np.float32)
        pnew = 10 ** 6 + t
        # brute-force expectation: softmax increments on the appended list
        Kall = np.vstack([lst.entries()[0], kn]).astype(np.float64)
        x = (q.astype(np.float64) @ Kall.T) / math.sqrt(d)
        p = np.exp(x - x.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        A_new = np.append(0.95 * A_before, 0.0) + p.sum(0)
        pos_all = np.append(pos_before, pnew)
        mid = _middle(pos_all, T, M)
        amin = min(A_new[i] for i in mid)
        cand = [i for i in mid if A_new[i] == amin]
        expect = pos_all[max(cand, key=lambda i: pos_all[i])]
        _, ev = lst.step(q, kn, vn, pnew, 0.95, T, M, b)
        assert ev == expect
        _, _, A_after, pos_after = lst.entries()
        assert len(pos_after) == b
        assert (np.diff(pos_after) > 0).all()
        assert pos_after[:T].tolist() == pos_all[:T].tolist()
        assert pos_after[-M:].tolist() == pos_all[-M:].tolist()


def test_decode_tie_evicts_higher_position(orc):
    # all keys identical -> all middle entries get the same A; the highest middle pos goes
    n, d, g, T, M = 12, 4, 1, 2, 3
    K = np.ones((n, d), np.float32)
    V = np.zeros((n, d), np.float32)
    pos = np.arange(n, dtype=np.int64) * 3
    lst = orc.DecodeList(K, V, pos)
    _, ev = lst.step(np.ones((g, d)), np.ones(d), np.zeros(d), 100, 0.95, T, M, n)
    # appended list: positions 0,3,...,33,100; middle = entries T .. n+1-M-1
    pos_all = list(pos) + [100]
    middle = pos_all[T:len(pos_all) - M]
    assert ev == max(middle)
