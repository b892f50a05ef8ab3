"""CPU oracle for the KV selection / compaction path (double precision).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use this package; the product library
never does. It shares no code with the CUDA path and does not import it.

The arithmetic lives in ``kvcomp_oracle.c`` (plain C, double, no FMA
contraction); this module compiles it with gcc on first use and wraps it with
numpy. Each wrapper names the page passage it restates:

* ``score``     AudioKV blog §1.2 (raw importance scores), window-softmax sum.
* ``sss``       AudioKV blog §2.2 (Spectral Score Smoothing) via a direct DFT.
* ``allocate``  AudioKV blog §3.1 / §5.1 (head-aware budget allocation).
* ``select``    AudioKV blog §3.1 (local window kept) + top-k by smoothed score.
* ``decode_*``  VoxZip, second stage (temporally decayed cumulative attention,
                Concat(K[:T], K[I_hist], K[-M:]) eviction).

Parity status: pinned (see tests/test_oracle_*.py); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvcomp_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-pthread"]


def build(force: bool = False) -> str:
    """Compile the C oracle into liboracle.so (gcc); returns the path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _get():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P = C.c_void_p
            I64, I32, D = C.c_int64, C.c_int, C.c_double
            lib.orc_score_rows.argtypes = [I64, P, P, P, I32, I32, P, P, I32]
            lib.orc_rdft.argtypes = [P, I64, P, P]
            lib.orc_kstar.argtypes = [P, P, I64, D, P]
            lib.orc_kstar.restype = I64
            lib.orc_irdft_lowpass.argtypes = [P, P, I64, I64, P]
            lib.orc_sss_rows.argtypes = [I64, P, P, P, D, D, P, P, P, I32]
            lib.orc_allocate.argtypes = [I32, P, I32, I32, I32, I32, C.c_float, P, P]
            lib.orc_allocate.restype = I32
            lib.orc_select_rows.argtypes = [I64, P, P, P, I32, P, P, P, I32]
            lib.orc_select_rows_seg.argtypes = [I64, P, P, P, I32, P, I32, P, P, I32]
            lib.orc_allocate_global.argtypes = [I32, P, I32, I32, I32, I32, C.c_float, P, P]
            lib.orc_allocate_global.restype = I32
            lib.orc_decode_step.argtypes = [P, I32, I32, P, P, P, P, P, P, P, I64, D, I32, I32, I64, P]
            lib.orc_decode_step.restype = I64
            lib.orc_voxzip_pool.argtypes = [I64, I32, P, D, I64, P, P, P, P, P, C.c_float, P, P]
            lib.orc_voxzip_pool.restype = I64
            lib.orc_wnw_chunks.argtypes = [I64, I64, I64]
            lib.orc_wnw_chunks.restype = I64
            lib.orc_wnw_step.argtypes = [I64, I32, P, I32, I32, I32, I32, I32, P, P, P, P, P, P, P, P, P]
            lib.orc_wnw_step.restype = I32
            lib.orc_splitmix64.argtypes = [C.c_uint64, C.c_uint64]
            lib.orc_splitmix64.restype = C.c_uint64
            lib.orc_c3_build.argtypes = [I64, I32, P, I32, I32, C.c_uint64, P, P, P, P, P, P, P]
            lib.orc_c3_build.restype = I64
            lib.orc_c3_frontier.argtypes = [I64, I64, I32, P, P, P]
            lib.orc_c3_frontier.restype = I64
            lib.orc_c3_step.argtypes = [I64, I32, I32, P, P, P, I64, P, P, P, P, P, I64, P, P, I64, D, I32, P, P, P]
            lib.orc_c3_step.restype = I64
            lib.orc_decode_run_heads.argtypes = [I64, P, I32, I32, P, P, P, P, P, I64, P, P, P, P, D, I32, P, P,
                                                 P, P, I32]
            _lib = lib
        return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def default_threads() -> int:
    return os.cpu_count() or 1


# ---------------------------------------------------------------- step 1 ----
def score(qwin: np.ndarray, K: np.ndarray, L_rows: Sequence[int], n_threads: int = 0) -> np.ndarray:
    """Window scores of every row (AudioKV blog §1.2 raw importance scores).

    qwin [rows][R][d]; K concatenated [sum L][d] in row order. Returns the
    concatenated scores [sum L] (float64): s_j = sum_r softmax_j(q_r.K_j/sqrt d).
    """
    qwin = _c(qwin, np.float32)
    K = _c(K, np.float32)
    L = _c(L_rows, np.int64)
    off = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
    rows, R, d = qwin.shape
    assert K.shape == (off[-1], d)
    s = np.zeros(off[-1], np.float64)
    _get().orc_score_rows(rows, _p(L), _p(off), _p(qwin), R, d, _p(K), _p(s), n_threads or default_threads())
    return s


# ---------------------------------------------------------------- step 2 ----
def rdft(s: np.ndarray) -> np.ndarray:
    """One-sided DFT bins 0..L/2 of a real row, by direct summation (complex128)."""
    s = _c(s, np.float64)
    L = s.shape[0]
    re = np.zeros(L // 2 + 1)
    im = np.zeros(L // 2 + 1)
    _get().orc_rdft(_p(s), L, _p(re), _p(im))
    return re + 1j * im


def kstar(F: np.ndarray, L: int, rho: float) -> Tuple[int, np.ndarray]:
    """Smallest k with E(k) >= rho E(L/2); returns (k*, E prefix)."""
    re = _c(F.real, np.float64)
    im = _c(F.imag, np.float64)
    E = np.zeros(L // 2 + 1)
    k = _get().orc_kstar(_p(re), _p(im), L, rho, _p(E))
    return int(k), E


def irdft_lowpass(F: np.ndarray, L: int, k: int) -> np.ndarray:
    """IRFFT (length L, 1/L scaling) of the spectrum kept up to bin k, by direct sums."""
    re = _c(F.real, np.float64)
    im = _c(F.imag, np.float64)
    y = np.zeros(L)
    _get().orc_irdft_lowpass(_p(re), _p(im), L, k, _p(y))
    return y


def sss(s: np.ndarray, L_rows: Sequence[int], alpha: float, rho: float,
        kstar_force: Optional[Sequence[int]] = None, n_threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Spectral Score Smoothing of every row (AudioKV blog §2.2).

    s is the concatenated scores; returns (s_hat concatenated, k* per row).
    ``kstar_force[i] >= 0`` smooths row i at that cutoff instead of its own.
    """
    s = _c(s, np.float64)
    L = _c(L_rows, np.int64)
    off = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
    assert s.shape[0] == off[-1]
    s_hat = np.zeros_like(s)
    ks = np.zeros(len(L), np.int64)
    kf = None if kstar_force is None else _c(kstar_force, np.int64)
    _get().orc_sss_rows(len(L), _p(L), _p(off), _p(s), alpha, rho, None if kf is None else _p(kf), _p(s_hat),
                        _p(ks), n_threads or default_threads())
    return s_hat, ks


# ---------------------------------------------------------------- step 3 ----
class BudgetError(ValueError):
    pass


def allocate(S: np.ndarray, L_seq: Sequence[int], w: int, budget_pct: int, r: float) -> np.ndarray:
    """Per-head budgets b [n_seq][layers][H] (AudioKV blog §3.1, §5.1)."""
    S = _c(S, np.float32)
    n_layers, H = S.shape
    L = _c(L_seq, np.int64)
    b = np.zeros((len(L), n_layers, H), np.int32)
    st = _get().orc_allocate(len(L), _p(L), n_layers, H, w, budget_pct, C.c_float(r), _p(S), _p(b))
    if st == 3:
        raise BudgetError("budget below H*w")
    if st:
        raise ValueError(f"allocate failed ({st})")
    return b


def allocate_global(S: np.ndarray, L_seq: Sequence[int], w: int, budget_pct: int, r: float) -> np.ndarray:
    """Budgets b [n_seq][layers][H] from one allocation over all (layer, head) of a sequence
    (variant of step 3: the same total, formula and rounding over n_layers * H heads)."""
    S = _c(S, np.float32)
    n_layers, H = S.shape
    L = _c(L_seq, np.int64)
    b = np.zeros((len(L), n_layers, H), np.int32)
    st = _get().orc_allocate_global(len(L), _p(L), n_layers, H, w, budget_pct, C.c_float(r), _p(S), _p(b))
    if st == 3:
        raise BudgetError("budget below n_layers*H*w")
    if st:
        raise ValueError(f"allocate_global failed ({st})")
    return b


# ---------------------------------------------------------------- step 4 ----
def select(s_hat: np.ndarray, L_rows: Sequence[int], w: int, b_rows: Sequence[int],
           n_threads: int = 0) -> list:
    """Kept positions per row, ascending: last w + top-(b-w) of s_hat over [0, L-w)."""
    s_hat = _c(s_hat, np.float64)
    L = _c(L_rows, np.int64)
    off = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
    b = _c(b_rows, np.int32)
    keep = np.minimum(b.astype(np.int64), L)
    ioff = np.concatenate([[0], np.cumsum(keep)]).astype(np.int64)
    idx = np.zeros(max(1, ioff[-1]), np.int32)
    _get().orc_select_rows(len(L), _p(L), _p(off), _p(s_hat), w, _p(b), _p(ioff), _p(idx),
                           n_threads or default_threads())
    return [idx[ioff[i]:ioff[i + 1]].copy() for i in range(len(L))]


def select_segmented(s_hat: np.ndarray, L_rows: Sequence[int], w: int, b_rows: Sequence[int], nseg: int,
                     n_threads: int = 0) -> list:
    """Kept positions per row, ascending: last w + per-segment top-q_i of s_hat over [0, L-w)
    (variant of step 4: nseg equal segments, quotas by largest remainder)."""
    s_hat = _c(s_hat, np.float64)
    L = _c(L_rows, np.int64)
    off = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
    b = _c(b_rows, np.int32)
    keep = np.minimum(b.astype(np.int64), L)
    ioff = np.concatenate([[0], np.cumsum(keep)]).astype(np.int64)
    idx = np.zeros(max(1, ioff[-1]), np.int32)
    _get().orc_select_rows_seg(len(L), _p(L), _p(off), _p(s_hat), w, _p(b), int(nseg), _p(ioff), _p(idx),
                               n_threads or default_threads())
    return [idx[ioff[i]:ioff[i + 1]].copy() for i in range(len(L))]


def gather(X: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Compacted rows X[idx] (an index copy)."""
    return np.ascontiguousarray(X[np.asarray(idx, np.int64)])


# ---------------------------------------------------------------- step 5 ----
class DecodeList:
    """One KV head's kept cache as the ordered list of the VoxZip eviction rule.

    Entries are in position order; arrays have room for one appended entry.
    """

    def __init__(self, K: np.ndarray, V: np.ndarray, pos: np.ndarray, A: Optional[np.ndarray] = None,
                 extra: int = 1):
        n, d = K.shape
        cap = n + extra
        self.d = d
        self.n = C.c_int64(n)
        self.K = np.zeros((cap, d), np.float32)
        self.V = np.zeros((cap, d), np.float32)
        self.A = np.zeros(cap, np.float64)
        self.pos = np.zeros(cap, np.int64)
        order = np.argsort(np.asarray(pos, np.int64), kind="stable")
        self.K[:n] = np.asarray(K, np.float32)[order]
        self.V[:n] = np.asarray(V, np.float32)[order]
        self.pos[:n] = np.asarray(pos, np.int64)[order]
        if A is not None:
            self.A[:n] = np.asarray(A, np.float64)[order]

    @property
    def size(self) -> int:
        return self.n.value

    def step(self, q: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, pos_new: int, gamma: float, T: int,
             M: int, b: int) -> Tuple[np.ndarray, int]:
        """Append, attend, update A, evict (VoxZip second stage). Returns (o [g][d], evicted pos or -1)."""
        if self.n.value + 1 > self.K.shape[0]:
            raise ValueError("DecodeList capacity exceeded")
        q = _c(q, np.float32)
        g = q.shape[0]
        o = np.zeros((g, self.d), np.float64)
        ev = _get().orc_decode_step(C.byref(self.n), self.d, g, _p(self.K), _p(self.V), _p(self.A), _p(self.pos),
                                    _p(q), _p(_c(k_new, np.float32)), _p(_c(v_new, np.float32)), int(pos_new),
                                    gamma, T, M, b, _p(o))
        return o, int(ev)

    def remove(self, pos: int) -> None:
        """Evicts the entry at position `pos`: the list becomes the Concat of the
        entries before and after it (the eviction of the VoxZip second stage
        with the evicted index given, for a tie the caller has resolved)."""
        n = self.n.value
        hit = np.flatnonzero(self.pos[:n] == pos)
        if len(hit) != 1:
            raise ValueError(f"position {pos} is not in the list")
        i = int(hit[0])
        for arr in (self.K, self.V, self.A, self.pos):
            arr[i:n - 1] = arr[i + 1:n].copy()
        self.n.value = n - 1

    def clone(self) -> "DecodeList":
        c = DecodeList.__new__(DecodeList)
        c.d = self.d
        c.n = C.c_int64(self.n.value)
        c.K, c.V, c.A, c.pos = self.K.copy(), self.V.copy(), self.A.copy(), self.pos.copy()
        return c

    def entries(self):
        n = self.n.value
        return self.K[:n].copy(), self.V[:n].copy(), self.A[:n].copy(), self.pos[:n].copy()


def recent_count(b: int, recent_pct: int) -> int:
    """M = floor(recent_pct * b / 100) (VoxZip: recent window = 20% of the budget)."""
    return (recent_pct * b) // 100


def decode_run_heads(Kc_list, Vc_list, pos_list, q, k_new, v_new, pos0, gamma, T, M, b, n_threads: int = 0):
    """Run every head's decode steps independently (CPU baseline).

    q [steps][heads][g][d]; k_new, v_new [steps][heads][d]. Returns
    (o [steps][heads][g][d] float64, evicted [steps][heads]).
    """
    heads = len(Kc_list)
    steps, _, g, d = q.shape
    caps = [len(k) + 1 for k in Kc_list]
    off = np.concatenate([[0], np.cumsum(caps)]).astype(np.int64)
    Kc = np.zeros((off[-1], d), np.float32)
    Vc = np.zeros((off[-1], d), np.float32)
    A = np.zeros(off[-1], np.float64)
    pos = np.zeros(off[-1], np.int64)
    n = np.zeros(heads, np.int64)
    for h in range(heads):
        order = np.argsort(pos_list[h], kind="stable")
        k = len(Kc_list[h])
        Kc[off[h]:off[h] + k] = Kc_list[h][order]
        Vc[off[h]:off[h] + k] = Vc_list[h][order]
        pos[off[h]:off[h] + k] = np.asarray(pos_list[h])[order]
        n[h] = k
    o = np.zeros((steps, heads, g, d), np.float64)
    ev = np.zeros((steps, heads), np.int64)
    _get().orc_decode_run_heads(heads, _p(n), d, g, _p(Kc), _p(Vc), _p(A), _p(pos), _p(off), steps,
                                _p(_c(q, np.float32)), _p(_c(k_new, np.float32)), _p(_c(v_new, np.float32)),
                                _p(_c(pos0, np.int64)), gamma, T, _p(_c(M, np.int32)), _p(_c(b, np.int64)),
                                _p(o), _p(ev), n_threads or default_threads())
    return o, ev


# ------------------------------------------------------ next row: VoxZip ----
def voxzip_pool(E_A: np.ndarray, tau_total: float, tau: np.ndarray, conf: np.ndarray, n_text: np.ndarray,
                text_row: np.ndarray, E_T: Optional[np.ndarray] = None, conf_min: float = 0.3):
    """VoxZip first stage on one sequence (方法概述和架构, first stage): ASR
    segments with confidence > conf_min mapped to token ranges, each split into
    L_t groups that are mean-pooled and fused with their text embeddings; the
    uncovered tokens kept; all in time order. Returns (E_comp [rows][d] float64,
    src [rows][3] int32 = first token, token count, text row or -1)."""
    E_A = _c(E_A, np.float64)
    L, d = E_A.shape
    tau = _c(tau, np.float64).reshape(-1, 2)
    n = tau.shape[0]
    out = np.zeros((max(L, 1), d), np.float64)
    src = np.zeros((max(L, 1), 3), np.int32)
    et = None if E_T is None else _c(E_T, np.float64)
    r = _get().orc_voxzip_pool(L, d, _p(E_A), float(tau_total), n, _p(tau), _p(_c(conf, np.float32)),
                               _p(_c(n_text, np.int32)), _p(_c(text_row, np.int32)),
                               None if et is None else _p(et), C.c_float(conf_min), _p(out), _p(src))
    return out[:r].copy(), src[:r].copy()


# --------------------------------------------------------- next row: WnW ----
class WnwState:
    """One sequence's WnW chunk/block residency (方法概述和架构, 细节详述):
    idle count per chunk (-1 = not resident), slot per block, block per slot."""

    def __init__(self, L: int, chunk_len: int, stride: int, top_c: int, release_after: int, n_slots: int):
        self.L, self.chunk_len, self.stride = L, chunk_len, stride
        self.top_c, self.release_after, self.n_slots = top_c, release_after, n_slots
        self.M = int(_get().orc_wnw_chunks(L, chunk_len, stride))
        self.nb = (L + stride - 1) // stride
        self.idle = np.full(self.M, -1, np.int32)
        self.block_slot = np.full(self.nb, -1, np.int32)
        self.slot_block = np.full(n_slots, -1, np.int32)

    def step(self, s: np.ndarray):
        """s [n_anchor][L] anchor attention mass. Returns (score [M] float64, selected,
        fetch [n][2] (block, slot), release [n][2])."""
        s = _c(s, np.float32)
        n_anchor = s.shape[0]
        score = np.zeros(self.M, np.float64)
        sel = np.zeros(max(1, min(self.top_c, self.M)), np.int32)
        cap = max(1, self.nb)
        fetch = np.zeros((cap, 2), np.int32)
        release = np.zeros((cap, 2), np.int32)
        nf, nr = C.c_int32(0), C.c_int32(0)
        st = _get().orc_wnw_step(self.L, n_anchor, _p(s), self.chunk_len, self.stride, self.top_c,
                                 self.release_after, self.n_slots, _p(self.idle), _p(self.block_slot),
                                 _p(self.slot_block), _p(score), _p(sel), _p(fetch), C.byref(nf), _p(release),
                                 C.byref(nr))
        if st:
            raise RuntimeError("WnW slots exhausted")
        return score, sel[:min(self.top_c, self.M)].copy(), fetch[:nf.value].copy(), release[:nr.value].copy()


# ---------------------------------------------------------- next row: C3 ----
def splitmix64(seed: int, k: int) -> int:
    """Output k (from 0) of SplitMix64 seeded with `seed` (Steele, Lea and Flood, 2014)."""
    return int(_get().orc_splitmix64(seed, k))


class C3Row:
    """One (layer, KV head) row of C3 ("C3: Speech-Guided KV Retrieval for
    Long-Context SpeechLLM Inference"): the bisecting 2-means index of its keys,
    the active frontier and its relevance EMA; `step` scores the frontier by the
    group's best cosine, retrieves up to B keys cluster by cluster, attends
    exactly, updates the EMA and runs R split/merge exchanges."""

    def __init__(self, K: np.ndarray, V: np.ndarray, leaf_max: int = 4, iters: int = 8, seed: int = 0,
                 granularity: int = 16):
        if iters < 1:
            raise ValueError("iters >= 1")
        self.K = _c(K, np.float32)
        self.V = _c(V, np.float32)
        L, d = self.K.shape
        self.L, self.d = L, d
        n = max(2 * L, 2)
        self.perm = np.zeros(max(L, 1), np.int32)
        self.lo, self.cnt, self.left, self.parent, self.depth = (np.zeros(n, np.int32) for _ in range(5))
        self.cent = np.zeros((n, d), np.float64)
        self.n_nodes = int(_get().orc_c3_build(L, d, _p(self.K), leaf_max, iters, seed, _p(self.perm), _p(self.lo),
                                               _p(self.cnt), _p(self.left), _p(self.parent), _p(self.depth),
                                               _p(self.cent)))
        front = np.zeros(max(self.n_nodes, 1), np.int32)
        self.A = int(_get().orc_c3_frontier(self.n_nodes, L, granularity, _p(self.left), _p(self.depth), _p(front)))
        self.front = front[:self.A].copy()
        self.e = np.zeros(self.n_nodes, np.float64)

    def members(self, node: int) -> np.ndarray:
        return self.perm[self.lo[node]:self.lo[node] + self.cnt[node]]

    def step(self, q: np.ndarray, B: int, lam: float = 0.5, R: int = 2):
        """q [G][d]. Returns (o [G][d] float64, selected positions, sigma of the frontier at entry)."""
        q = _c(q, np.float32)
        G = q.shape[0]
        sigma = np.zeros(max(self.A, 1), np.float64)
        sel = np.zeros(max(self.L, 1), np.int32)
        o = np.zeros((G, self.d), np.float64)
        front = self.front.copy()
        n = _get().orc_c3_step(self.L, self.d, G, _p(self.K), _p(self.V), _p(q), self.n_nodes, _p(self.perm),
                               _p(self.lo), _p(self.cnt), _p(self.left), _p(self.cent), self.A, _p(front),
                               _p(self.e), int(B), float(lam), int(R), _p(sigma), _p(sel), _p(o))
        sig = sigma[:self.A].copy()
        self.front = front
        return o, sel[:n].copy(), sig


__all__ = ["splitmix64", "C3Row", "WnwState", "voxzip_pool", "build", "score", "rdft", "kstar", "irdft_lowpass", "sss", "allocate", "BudgetError", "select",
           "gather", "DecodeList", "recent_count", "decode_run_heads", "default_threads"]
