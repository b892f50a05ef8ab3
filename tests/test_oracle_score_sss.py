"""Pins for the oracle's window scores and Spectral Score Smoothing.

Each check ties the oracle to something other than itself: an exact
invariant, a closed form, or an independent library routine (torch softmax in
float64, numpy's FFT). A dropped term, a wrong sign or a transposed operand in
the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_row(rng, R, L, d, scale=1.0):
    q = (rng.standard_normal((1, R, d)) * scale).astype(np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    return q, K


# ------------------------------------------------------------------ score ----
def test_score_sums_to_window_rows(orc):
    # softmax over the L keys of each of the R window rows sums to 1, so the
    # column sums add up to R; a softmax taken over the rows would give L.
    rng = np.random.default_rng(1)
    for R, L, d in [(32, 1024, 64), (7 * 32, 300, 128), (5, 17, 8)]:
        q, K = _rand_row(rng, R, L, d)
        s = orc.score(q, K, [L])
        assert abs(s.sum() - R) < 1e-9 * R
        assert (s > 0).all()


def test_score_zero_queries_uniform(orc):
    R, L, d = 24, 500, 64
    q = np.zeros((1, R, d), np.float32)
    K = np.random.default_rng(2).standard_normal((L, d)).astype(np.float32)
    s = orc.score(q, K, [L])
    np.testing.assert_allclose(s, R / L, rtol=1e-13)


def test_score_dominant_key(orc):
    # one key aligned with every query at a huge logit takes all the mass
    rng = np.random.default_rng(3)
    R, L, d = 16, 200, 64
    u = rng.standard_normal(d).astype(np.float32)
    u /= np.linalg.norm(u)
    K = (0.01 * rng.standard_normal((L, d))).astype(np.float32)
    K[77] = 400.0 * u  # logit 50 above the rest: the others hold < L e^-49 of the mass
    q = np.tile(u, (1, R, 1)).astype(np.float32)
    s = orc.score(q, K, [L])
    assert abs(s[77] - R) < 1e-9
    assert s.argmax() == 77


def test_score_matches_torch_softmax(orc):
    # library reference: torch.softmax in float64 over the key axis
    rng = np.random.default_rng(4)
    rows = [(64, 333, 64), (256, 700, 128)]
    for R, L, d in rows:
        q, K = _rand_row(rng, R, L, d, scale=0.5)
        s = orc.score(q, K, [L])
        x = torch.from_numpy(q[0]).double() @ torch.from_numpy(K).double().T / math.sqrt(d)
        ref = torch.softmax(x, dim=-1).sum(0).numpy()
        np.testing.assert_allclose(s, ref, rtol=1e-11, atol=0)


def test_score_key_permutation_equivariant(orc):
    rng = np.random.default_rng(5)
    R, L, d = 32, 257, 64
    q, K = _rand_row(rng, R, L, d)
    perm = rng.permutation(L)
    s = orc.score(q, K, [L])
    sp = orc.score(q, K[perm], [L])
    np.testing.assert_allclose(sp, s[perm], rtol=1e-12)


def test_score_rows_are_independent(orc):
    # batched rows (ragged L) equal the rows scored one by one
    rng = np.random.default_rng(6)
    Ls = [40, 96, 18]
    R, d = 12, 64
    q = rng.standard_normal((3, R, d)).astype(np.float32)
    K = rng.standard_normal((sum(Ls), d)).astype(np.float32)
    s = orc.score(q, K, Ls)
    off = np.concatenate([[0], np.cumsum(Ls)])
    for i in range(3):
        si = orc.score(q[i:i + 1], K[off[i]:off[i + 1]], [Ls[i]])
        np.testing.assert_array_equal(s[off[i]:off[i + 1]], si)


def test_score_on_synthetic_row_sums(orc):
    cfg = synth.small("3b", n_layers=1, L=(600,))
    row = synth.make_row(cfg, 0, 0, 1, steps=1)
    s = orc.score(row.qwin[None], row.K, [row.L])
    assert abs(s.sum() - cfg.R) < 1e-9 * cfg.R


# -------------------------------------------------------------------- SSS ----
@pytest.mark.parametrize("L", [8, 30, 210, 1000, 2 * 3 * 5 * 7 * 4])
def test_rdft_matches_numpy_fft(orc, L):
    s = np.random.default_rng(L).random(L)
    F = orc.rdft(s)
    ref = np.fft.rfft(s)
    assert F.shape == ref.shape
    np.testing.assert_allclose(F, ref, rtol=0, atol=1e-10 * np.abs(ref).max())


def test_rdft_parseval(orc):
    L = 420
    s = np.random.default_rng(7).standard_normal(L)
    F = orc.rdft(s)
    two_sided = abs(F[0]) ** 2 + 2 * (np.abs(F[1:L // 2]) ** 2).sum() + abs(F[L // 2]) ** 2
    assert abs(two_sided - L * (s ** 2).sum()) < 1e-9 * two_sided


@pytest.mark.parametrize("L,k", [(16, 0), (16, 3), (16, 8), (210, 57), (210, 105), (1000, 1)])
def test_irdft_lowpass_matches_numpy_irfft(orc, L, k):
    s = np.random.default_rng(L + k).random(L)
    F = np.fft.rfft(s)
    y = orc.irdft_lowpass(F, L, k)
    G = F.copy()
    G[k + 1:] = 0
    ref = np.fft.irfft(G, n=L)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))


def test_kstar_definition(orc):
    L = 64
    s = np.random.default_rng(8).random(L)
    F = np.fft.rfft(s)
    for rho in [0.0, 0.1, 0.5, 0.7, 0.95, 1.0]:
        k, E = orc.kstar(F, L, rho)
        np.testing.assert_allclose(E, np.cumsum(np.abs(F) ** 2), rtol=1e-12)
        assert E[k] >= rho * E[-1]
        assert k == 0 or E[k - 1] < rho * E[-1]


def test_sss_alpha_zero_is_identity(orc):
    L = [300, 64]
    s = np.random.default_rng(9).random(sum(L))
    s_hat, _ = orc.sss(s, L, alpha=0.0, rho=0.7)
    np.testing.assert_array_equal(s_hat, s)


def test_sss_rho_one_reconstructs(orc):
    L = [300, 64, 1000]
    s = np.random.default_rng(10).random(sum(L))
    s_hat, ks = orc.sss(s, L, alpha=0.8, rho=1.0)
    np.testing.assert_allclose(s_hat, s, rtol=0, atol=1e-12)
    assert list(ks) == [l // 2 for l in L]


def test_sss_rho_zero_is_mean_blend(orc):
    L = 500
    s = np.random.default_rng(11).random(L)
    s_hat, ks = orc.sss(s, [L], alpha=0.3, rho=0.0)
    assert ks[0] == 0
    np.testing.assert_allclose(s_hat, 0.7 * s + 0.3 * s.mean(), rtol=1e-12)


def test_sss_cosine_golden(orc):
    cases = json.load(open(os.path.join(GOLDEN, "sss_cosine.json")))["cases"]
    for c in cases:
        L, f = c["L"], c["f"]
        n = np.arange(L)
        s = c["c"] + c["a"] * np.cos(2 * np.pi * f * n / L)
        s_hat, ks = orc.sss(s, [L], alpha=c["alpha"], rho=c["rho"])
        assert ks[0] == c["kstar"], c
        expect = s if c["kstar"] == f else (1 - c["alpha"]) * s + c["alpha"] * c["c"]
        np.testing.assert_allclose(s_hat, expect, rtol=0, atol=1e-12)


def test_sss_forced_kstar_matches_numpy(orc):
    L = 300
    s = np.random.default_rng(12).random(L)
    s_hat, ks = orc.sss(s, [L], alpha=0.5, rho=0.7, kstar_force=[17])
    assert ks[0] == 17
    F = np.fft.rfft(s)
    F[18:] = 0
    ref = 0.5 * s + 0.5 * np.fft.irfft(F, n=L)
    np.testing.assert_allclose(s_hat, ref, rtol=0, atol=1e-12)


def test_sss_kstar_monotone_in_rho(orc):
    L = 400
    s = np.random.default_rng(13).random(L)
    prev = -1
    for rho in np.linspace(0, 1, 21):
        _, ks = orc.sss(s, [L], alpha=0.5, rho=float(rho))
        assert ks[0] >= prev
        prev = ks[0]
