"""Shared pieces of the GPU parity tests: uploads of the seeded inputs,
shape/parameter structs, and the comparison rules.

Comparison rules (from the method's stated tolerances, made checkable):
* scores and smoothed scores on identical inputs: |gpu - orc| <= 1e-4 *
  max(|orc_j|, 1e-6 * max_j |orc|);
* smoothed scores end to end (each side smooths its own scores): the floor is
  the row's RMS, since the low-pass spreads every input's rounding over the
  whole row and s_hat rings through zero (a per-element bound cannot hold
  at its zero crossings);
* k*: a cutoff is valid when the oracle's own energy prefix reaches the
  threshold within a band (kstar_band_*): on identical float32 inputs both
  sides transform in float64, so the band only covers summation order; end to
  end it is the shift that scores within their tolerance can cause. The GPU's
  s_hat is compared with the oracle's s_hat at the GPU's cutoff;
* selected indices: bit-exact on identical inputs; end to end, positions whose
  oracle s_hat lies within 1e-5 (relative) of the k-th kept score are exempt;
* compacted K/V: bit-exact copies;
* decode outputs: 2e-2 absolute for bf16, 1e-4 relative for fp32; evictions
  equal, except where the oracle's own decayed scores of the two choices are
  within 1e-5 (relative): both choices are then correct, the oracle takes the
  GPU's and checking goes on.
"""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_compression_layer_b200 as kv
import synth

SCORE_RTOL = 1e-4
SCORE_FLOOR = 1e-6
# k* on identical float32 rows: the kernel (a float64 Stockham FFT) and the
# oracle (a float64 direct DFT) agree on every energy prefix to ~1e-15 of the
# row's energy; the band leaves room for summation order and nothing else.
# The kernel's rho is a float32 parameter, so the oracle is given that value.
KSTAR_BAND_SAME_INPUT = 1e-9
SELECT_EXEMPT = 1e-5


def dev():
    return torch.device("cuda")


def tdtype(cfg: synth.Config):
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def shape_of(cfg: synth.Config):
    return kv.make_shape(cfg.n_layers, cfg.n_kv_heads, cfg.group, cfg.head_dim, cfg.w,
                         kv.KV_BF16 if cfg.dtype == "bf16" else kv.KV_F32)


def params_of(cfg: synth.Config):
    return kv.make_params(cfg.budget_pct, cfg.alpha, cfg.rho, cfg.r, cfg.gamma, cfg.sinks_T, cfg.recent_pct)


def up(x: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=dev(), dtype=dtype)


def score_close(gpu: np.ndarray, orc: np.ndarray, L_rows, rtol=SCORE_RTOL, floor="max") -> tuple:
    """Returns (ok, worst ratio) of the per-element score rule, row by row.

    floor="max": 1e-6 of the row's largest magnitude; floor="rms": the row's RMS.
    """
    off = np.concatenate([[0], np.cumsum(L_rows)])
    worst = 0.0
    for i in range(len(L_rows)):
        g = gpu[off[i]:off[i + 1]].astype(np.float64)
        o = orc[off[i]:off[i + 1]]
        if floor == "rms":
            floor_v = np.sqrt(np.mean(o * o))
        else:
            floor_v = SCORE_FLOOR * np.abs(o).max()
        floor_ = floor_v
        ratio = np.abs(g - o) / (rtol * np.maximum(np.abs(o), floor_))
        worst = max(worst, float(ratio.max()))
    return worst <= 1.0, worst


def kstar_band_end_to_end(rho: float, score_rtol: float = SCORE_RTOL) -> float:
    """Band (relative to the threshold rho E(L/2)) within which scores that
    each lie within score_rtol of the oracle's can move an energy prefix.

    With s' = s (1 + e), |e| <= t, the spectrum moves by dF = DFT(s e), and
    sum_i |dF_i|^2 <= L sum_j (s_j e_j)^2 <= t^2 L sum s^2 <= 2 t^2 E(L/2)
    (Parseval over the one-sided bins). Then |dE(k)| <= 2 sqrt(E(k) |dF|^2) +
    |dF|^2 <= (2 sqrt 2 t + 2 t^2) E(L/2) for every k, and the threshold moves
    by rho times that: the prefix and the threshold can shift against each
    other by (1 + rho) (2 sqrt 2 t + 2 t^2) E(L/2).
    """
    return (1.0 + rho) * (2.0 * np.sqrt(2.0) * score_rtol + 2.0 * score_rtol ** 2) / rho


def valid_kstars(s_row: np.ndarray, rho: float, orc, band: float) -> list:
    """Cutoffs k whose oracle energies bracket the threshold within `band`:
    E(k) >= thr (1 - band) and (k = 0 or E(k - 1) < thr (1 + band))."""
    L = len(s_row)
    F = orc.rdft(s_row)
    _, E = orc.kstar(F, L, rho)
    thr = rho * E[-1]
    ks = []
    for k in range(L // 2 + 1):
        lo = E[k] >= thr * (1 - band) - 1e-300
        hi = k == 0 or E[k - 1] < thr * (1 + band)
        if lo and hi:
            ks.append(k)
    return ks


def f32(x: float) -> float:
    """The float32 value a float parameter takes at the C ABI."""
    return float(np.float32(x))


def kth_exempt_mask(s_hat_orc: np.ndarray, L: int, w: int, b: int) -> np.ndarray:
    """Positions in [0, L-w) whose oracle s_hat is within SELECT_EXEMPT of the k-th kept value."""
    k = b - w
    cand = s_hat_orc[:L - w]
    if k <= 0 or b >= L:
        return np.zeros(L - w, bool)
    kth = np.sort(cand)[::-1][k - 1]
    return np.abs(cand - kth) <= SELECT_EXEMPT * max(abs(kth), 1e-30)
