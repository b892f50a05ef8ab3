"""Seeded synthetic inputs for the KV-selection hot path.

This module only draws random inputs. It holds none of the method's
arithmetic (no scoring, smoothing, allocation, selection or attention), so
the CUDA path and the CPU oracle can both consume exactly the same arrays.

Every array comes from numpy's Philox counter-based generator, keyed by
(config seed, sequence, layer, KV head, tensor id), so any single row can be
regenerated on its own without drawing the others.

The workloads stand in for the shapes of the audio-LLM workloads on the
pages (AudioKV, VoxZip, WnW, C3); no dataset is read or reproduced:

* keys: an AR(1) latent ``z_t = phi z_{t-1} + sqrt(1-phi^2) e_t`` of width
  d/4 (phi = 0.95, stationary start), projected by ``P ~ N(0, 1/(d/4))``
  (d x d/4, one per layer and head) plus ``N(0, 0.5)`` noise (variance);
* values: i.i.d. ``N(0, 1)``;
* observation-window queries: ``q = 0.8 K[p] + N(0, 0.3)`` with ``p`` on a
  diagonal alignment band ``floor((i+0.5) L/w) + U{-floor(L/2w)..floor(L/2w)}``,
  clamped, jitter drawn independently per query head;
* decode step t: ``k_t`` continues the key AR(1) at position L+t, ``v_t`` is
  ``N(0,1)``, ``q_t = 0.8 K[p_t] + N(0, 0.3)`` with ``p_t`` on the band
  ``floor((t+0.5) L/steps)`` (or slowly drifting for the long-form stress
  case: ``floor(L/4) + floor(t L / (4 steps))``);
* per-head audio relevance S: ``U(0,1)``, or ``Beta(0.5, 2)`` with the top
  18% of (layer, head) pairs multiplied by 4 (ties to the lower index);
* spikes (ragged batch): 5% of positions per row, whose raw score is
  multiplied by 10 before smoothing (a harness step, not part of the path).
* ASR segments for the VoxZip pooling row (``asr_segments``): audio features
  at 12.5 tokens/s (tau_total = L / 12.5 s), speech runs of U(1, 10) s
  separated by U(0.2, 2) s pauses, confidence U(0, 1) (about 70% above the
  0.3 cut), 3 text tokens per second of speech (at least 1), text rows laid
  out segment after segment; features ``E_A ~ N(0, 1)``, text embeddings
  ``E_T ~ N(0, 0.02)`` (standard deviation).
* anchor attention for the WnW row (``anchor_attention``): per step and
  anchor row a mass of g (the query heads of the KV head) spread as 10% over
  the first tenth of the audio (the sink), 60% in a Gaussian bump of 25 rows
  (2 s) around a focus that walks through the audio with the decode step
  (jittered per anchor by U{-50..50} rows), 30% uniform, times U(0.5, 1.5)
  noise per row before normalising.

Values are drawn in float32 and rounded to nearest-even bfloat16 for the
bf16 workloads; the returned float32 arrays hold those bf16-exact values.
"""
from __future__ import annotations

import dataclasses
import os
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional, Sequence

import numpy as np
from scipy.signal import lfilter

# tensor ids of the counter-based streams
_T_KEYS, _T_PROJ, _T_KNOISE, _T_VALUES, _T_QWIN, _T_QDEC, _T_VDEC, _T_SPIKE = range(8)
_T_HEADSCORES = 100
_T_ASR, _T_FEAT, _T_TEXT, _T_ANCHOR = 200, 201, 202, 203


@dataclasses.dataclass(frozen=True)
class Config:
    """One synthetic workload: shapes, the method's parameters and the input recipe."""

    name: str
    n_layers: int
    n_kv_heads: int
    group: int  # query heads per KV head (GQA group)
    head_dim: int
    L: tuple  # audio keys per sequence
    dtype: str  # "f32" or "bf16"
    w: int = 32  # observation window and local window
    budget_pct: int = 40  # kept fraction of the audio keys, percent
    alpha: float = 0.5
    rho: float = 0.7
    r: float = 0.5
    gamma: float = 0.95
    sinks_T: int = 4
    recent_pct: int = 20
    decode_steps: int = 32
    head_scores: str = "uniform"  # "uniform" or "beta_top18x4"
    queries: str = "band"  # "band" or "drift"
    spike_frac: float = 0.0
    seed: int = 0

    @property
    def n_seq(self) -> int:
        return len(self.L)

    @property
    def rows(self) -> int:
        return self.n_seq * self.n_layers * self.n_kv_heads

    @property
    def R(self) -> int:
        return self.group * self.w

    def row_index(self, seq: int, layer: int, head: int) -> int:
        return (seq * self.n_layers + layer) * self.n_kv_heads + head

    def row_triplet(self, row: int):
        head = row % self.n_kv_heads
        layer = (row // self.n_kv_heads) % self.n_layers
        seq = row // (self.n_kv_heads * self.n_layers)
        return seq, layer, head

    def row_L(self, row: int) -> int:
        return self.L[self.row_triplet(row)[0]]

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, Config] = {
    "tiny": Config("tiny", 1, 4, 1, 64, (1024,), "f32", budget_pct=40, alpha=0.5, rho=0.7,
                   r=0.5, decode_steps=32),
    "3b": Config("3b", 36, 2, 8, 128, (6000,), "bf16", budget_pct=60, alpha=0.5, rho=0.7,
                 decode_steps=128),
    "30b": Config("30b", 48, 4, 8, 128, (16000,), "bf16", budget_pct=40, alpha=0.6, rho=0.7,
                  decode_steps=256, head_scores="beta_top18x4"),
    "ragged": Config("ragged", 28, 4, 7, 128,
                     (2000, 3500, 5000, 7500, 9000, 12000, 14000, 16000), "bf16",
                     budget_pct=25, decode_steps=128, spike_frac=0.05),
    "long": Config("long", 48, 4, 8, 128, (32768,), "bf16", budget_pct=5, alpha=0.5,
                   rho=0.7, decode_steps=512, queries="drift"),
}


def _rng(cfg: Config, seq: int, layer: int, head: int, tensor: int) -> np.random.Generator:
    ss = np.random.SeedSequence([cfg.seed, seq, layer, head, tensor])
    return np.random.Generator(np.random.Philox(ss))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16-exact float32 values -> their uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _finish(cfg: Config, x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return round_bf16(x) if cfg.dtype == "bf16" else x


def keys(cfg: Config, seq: int, layer: int, head: int, n: int) -> np.ndarray:
    """Key rows for positions 0..n-1 of one (sequence, layer, KV head): [n][d]."""
    d = cfg.head_dim
    dl = max(1, d // 4)
    phi = 0.95
    e = _rng(cfg, seq, layer, head, _T_KEYS).standard_normal((n, dl))
    e[1:] *= math.sqrt(1.0 - phi * phi)
    z = lfilter([1.0], [1.0, -phi], e, axis=0)
    P = _rng(cfg, 0, layer, head, _T_PROJ).standard_normal((d, dl)) / math.sqrt(dl)
    noise = _rng(cfg, seq, layer, head, _T_KNOISE).standard_normal((n, d)) * math.sqrt(0.5)
    return _finish(cfg, z @ P.T + noise)


def values(cfg: Config, seq: int, layer: int, head: int, n: int, tensor: int = _T_VALUES) -> np.ndarray:
    return _finish(cfg, _rng(cfg, seq, layer, head, tensor).standard_normal((n, cfg.head_dim)))


def _band(rng: np.random.Generator, centers: np.ndarray, half: int, L: int) -> np.ndarray:
    jitter = rng.integers(-half, half + 1, size=centers.shape) if half > 0 else 0
    return np.clip(centers + jitter, 0, L - 1)


def window_queries(cfg: Config, seq: int, layer: int, head: int, K: np.ndarray) -> np.ndarray:
    """Observation-window queries of one KV head's group: [g*w][d], query head major."""
    L = cfg.L[seq]
    w, g, d = cfg.w, cfg.group, cfg.head_dim
    rng = _rng(cfg, seq, layer, head, _T_QWIN)
    centers = np.floor((np.arange(w) + 0.5) * L / w).astype(np.int64)
    half = L // (2 * w)
    out = np.empty((g, w, d), np.float32)
    for gi in range(g):
        p = _band(rng, centers, half, L)
        out[gi] = 0.8 * K[p] + rng.standard_normal((w, d)) * math.sqrt(0.3)
    return _finish(cfg, out.reshape(g * w, d))


def decode_queries(cfg: Config, seq: int, layer: int, head: int, K: np.ndarray, steps: int) -> np.ndarray:
    """Decode-step queries of one KV head's group: [steps][g][d]."""
    L = cfg.L[seq]
    g, d = cfg.group, cfg.head_dim
    rng = _rng(cfg, seq, layer, head, _T_QDEC)
    t = np.arange(steps)
    if cfg.queries == "drift":
        centers = L // 4 + (t * L) // (4 * steps)
        half = max(1, L // (8 * steps))
    else:
        centers = np.floor((t + 0.5) * L / steps).astype(np.int64)
        half = L // (2 * steps)
    out = np.empty((steps, g, d), np.float32)
    for gi in range(g):
        p = _band(rng, centers, half, L)
        out[:, gi] = 0.8 * K[p] + rng.standard_normal((steps, d)) * math.sqrt(0.3)
    return _finish(cfg, out)


def head_scores(cfg: Config) -> np.ndarray:
    """Per-(layer, KV head) audio relevance S: [layers][H_kv] float32."""
    rng = _rng(cfg, 0, 0, 0, _T_HEADSCORES)
    n = cfg.n_layers * cfg.n_kv_heads
    if cfg.head_scores == "beta_top18x4":
        S = rng.beta(0.5, 2.0, size=n)
        top = int(math.ceil(0.18 * n))
        order = np.lexsort((np.arange(n), -S))  # descending S, ties to the lower index
        S[order[:top]] *= 4.0
    else:
        S = rng.random(n)
    return S.astype(np.float32).reshape(cfg.n_layers, cfg.n_kv_heads)


def spike_mask(cfg: Config, seq: int, layer: int, head: int) -> Optional[np.ndarray]:
    """Positions whose raw score is multiplied by 10 (ragged batch only)."""
    if cfg.spike_frac <= 0:
        return None
    L = cfg.L[seq]
    rng = _rng(cfg, seq, layer, head, _T_SPIKE)
    n = int(round(cfg.spike_frac * L))
    m = np.zeros(L, bool)
    m[rng.choice(L, size=n, replace=False)] = True
    return m


@dataclasses.dataclass
class Row:
    """All inputs of one (sequence, layer, KV head)."""

    seq: int
    layer: int
    head: int
    L: int
    qwin: np.ndarray  # [g*w][d]
    K: np.ndarray  # [L][d]
    V: np.ndarray  # [L][d]
    q_dec: np.ndarray  # [steps][g][d]
    k_dec: np.ndarray  # [steps][d]
    v_dec: np.ndarray  # [steps][d]
    spikes: Optional[np.ndarray]


def make_row(cfg: Config, seq: int, layer: int, head: int, steps: Optional[int] = None) -> Row:
    steps = cfg.decode_steps if steps is None else steps
    L = cfg.L[seq]
    Kall = keys(cfg, seq, layer, head, L + steps)
    K = np.ascontiguousarray(Kall[:L])
    V = values(cfg, seq, layer, head, L)
    return Row(seq, layer, head, L,
               qwin=window_queries(cfg, seq, layer, head, K),
               K=K, V=V,
               q_dec=decode_queries(cfg, seq, layer, head, K, steps),
               k_dec=np.ascontiguousarray(Kall[L:]),
               v_dec=values(cfg, seq, layer, head, steps, tensor=_T_VDEC),
               spikes=spike_mask(cfg, seq, layer, head))


@dataclasses.dataclass
class Batch:
    """Concatenated inputs of every row, in (sequence, layer, KV head) order.

    qwin [rows][g*w][d]; K, V concatenated [sum_rows L][d]; S [layers][H];
    decode tensors [steps][rows][g][d] (q) and [steps][rows][d] (k, v).
    """

    cfg: Config
    rows: List[int]
    L_rows: np.ndarray
    qwin: np.ndarray
    K: np.ndarray
    V: np.ndarray
    S: np.ndarray
    q_dec: np.ndarray
    k_dec: np.ndarray
    v_dec: np.ndarray
    spikes: Optional[np.ndarray]  # concatenated like the scores, or None

    @property
    def key_off(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.L_rows)]).astype(np.int64)


def make_batch(cfg: Config, steps: Optional[int] = None, threads: int = 0) -> Batch:
    """Every row of the workload, generated row by row (each row from its own
    seeded streams, so the result does not depend on `threads`) into
    preallocated concatenated arrays; rows are generated on a thread pool."""
    steps = cfg.decode_steps if steps is None else steps
    rows = list(range(cfg.rows))
    L_rows = np.array([cfg.row_L(r) for r in rows], np.int64)
    off = np.concatenate([[0], np.cumsum(L_rows)]).astype(np.int64)
    g, d, R = cfg.group, cfg.head_dim, cfg.R
    qwin = np.empty((cfg.rows, R, d), np.float32)
    K = np.empty((int(off[-1]), d), np.float32)
    V = np.empty((int(off[-1]), d), np.float32)
    q_dec = np.empty((steps, cfg.rows, g, d), np.float32)
    k_dec = np.empty((steps, cfg.rows, d), np.float32)
    v_dec = np.empty((steps, cfg.rows, d), np.float32)
    spikes = np.empty(int(off[-1]), bool) if cfg.spike_frac > 0 else None

    def fill(r: int) -> None:
        p = make_row(cfg, *cfg.row_triplet(r), steps=steps)
        qwin[r] = p.qwin
        K[off[r]:off[r + 1]] = p.K
        V[off[r]:off[r + 1]] = p.V
        q_dec[:, r] = p.q_dec
        k_dec[:, r] = p.k_dec
        v_dec[:, r] = p.v_dec
        if spikes is not None:
            spikes[off[r]:off[r + 1]] = p.spikes

    n_thr = threads or min(32, os.cpu_count() or 1)
    if n_thr <= 1 or cfg.rows <= 1:
        for r in rows:
            fill(r)
    else:
        with ThreadPoolExecutor(max_workers=n_thr) as ex:
            list(ex.map(fill, rows))
    return Batch(cfg=cfg, rows=rows, L_rows=L_rows, qwin=qwin, K=K, V=V, S=head_scores(cfg),
                 q_dec=q_dec, k_dec=k_dec, v_dec=v_dec, spikes=spikes)


@dataclasses.dataclass
class AsrSegments:
    """Timestamped ASR segments of one sequence (inputs of the VoxZip pooling)."""
    tau_total: float
    tau: np.ndarray       # [n][2] float64 start, end (seconds)
    conf: np.ndarray      # [n] float32
    n_text: np.ndarray    # [n] int32 text tokens
    text_row: np.ndarray  # [n] int32 first text-embedding row


def asr_segments(seed: int, L: int, rate: float = 12.5) -> AsrSegments:
    """Seeded speech/pause layout over L audio tokens at `rate` tokens/s."""
    rng = np.random.Generator(np.random.Philox(key=[seed, _T_ASR]))
    tau_total = L / rate
    starts, ends = [], []
    t = float(rng.uniform(0.0, 2.0))
    while t < tau_total:
        e = t + float(rng.uniform(1.0, 10.0))
        starts.append(t)
        ends.append(min(e, tau_total))
        t = e + float(rng.uniform(0.2, 2.0))
    n = len(starts)
    tau = np.stack([np.asarray(starts), np.asarray(ends)], axis=1).reshape(n, 2).astype(np.float64)
    conf = rng.uniform(0.0, 1.0, size=n).astype(np.float32)
    n_text = np.maximum(1, np.floor(3.0 * (tau[:, 1] - tau[:, 0]))).astype(np.int32)
    text_row = np.concatenate([[0], np.cumsum(n_text)[:-1]]).astype(np.int32) if n else np.zeros(0, np.int32)
    return AsrSegments(tau_total, tau, conf, n_text, text_row)


def audio_features(seed: int, L: int, d: int, bf16: bool = True) -> np.ndarray:
    """E_A ~ N(0, 1), [L][d] float32 (bf16-exact when bf16)."""
    rng = np.random.Generator(np.random.Philox(key=[seed, _T_FEAT]))
    x = rng.standard_normal((L, d), dtype=np.float32)
    return round_bf16(x) if bf16 else x


def text_embeddings(seed: int, n: int, d: int, bf16: bool = True) -> np.ndarray:
    """E_T ~ N(0, 0.02^2), [n][d] float32 (bf16-exact when bf16)."""
    rng = np.random.Generator(np.random.Philox(key=[seed, _T_TEXT]))
    x = (0.02 * rng.standard_normal((max(n, 0), d), dtype=np.float32)).astype(np.float32)
    return round_bf16(x) if bf16 else x


def anchor_attention(seed: int, L: int, n_anchor: int, steps: int, g: int = 4) -> np.ndarray:
    """[steps][n_anchor][L] float32 attention mass of the anchor rows, each summing to g."""
    rng = np.random.Generator(np.random.Philox(key=[seed, _T_ANCHOR]))
    out = np.empty((steps, n_anchor, L), np.float32)
    x = np.arange(L, dtype=np.float64)
    sink = np.where(x < max(1, L // 10), 1.0, 0.0)
    sink /= sink.sum()
    for t in range(steps):
        focus = (t + 0.5) * L / steps
        for a in range(n_anchor):
            c = focus + rng.integers(-50, 51)
            bump = np.exp(-0.5 * ((x - c) / 25.0) ** 2)
            bump /= max(bump.sum(), 1e-300)
            p = (0.1 * sink + 0.6 * bump + 0.3 / L) * rng.uniform(0.5, 1.5, L)
            out[t, a] = (g * p / p.sum()).astype(np.float32)
    return out


def small(cfg_name: str, **kw) -> Config:
    """A reduced copy of a named workload (fewer layers / shorter audio) for fast tests."""
    return CONFIGS[cfg_name].with_(**kw)


__all__ = ["Config", "CONFIGS", "Row", "Batch", "make_row", "make_batch", "keys", "values",
           "window_queries", "decode_queries", "head_scores", "spike_mask", "round_bf16",
           "to_bf16_bits", "small", "AsrSegments", "asr_segments", "audio_features", "text_embeddings",
           "anchor_attention"]
