"""Lock-step checking of decode steps against the oracle's literal VoxZip
step (append, attend, decayed-score update, sink/recent/top-N eviction).

Each checked row has an oracle list that runs every step from its own state.
Per step the attention output must match and the evicted position must be
the oracle's. Where they differ, the two choices must be a near tie in the
oracle's own decayed scores (1e-5 relative): both are then correct, the
oracle takes the GPU's choice (it evicts that position from its own list),
and the row stays under comparison. The oracle never reads a GPU value
other than that validated choice.
"""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc

TIE_RTOL = 1e-5


class Snapshot:
    """Host copy of a GPU decode state's meta data, positions and decayed
    scores (one read per tensor), sliced per row."""

    def __init__(self, t: dict, off: np.ndarray):
        self.meta = t["meta"].cpu().numpy().reshape(-1, kv.META_INTS)
        self.pos = t["pos"].cpu().numpy()
        self.A = t["A"].cpu().numpy()
        self.off = off

    def row(self, r: int):
        lo, hi = int(self.off[r]), int(self.off[r + 1])
        return self.meta[r], self.pos[lo:hi], self.A[lo:hi]

    @staticmethod
    def present_slots(meta: np.ndarray, cap: int) -> list:
        """Occupied slots: {0 .. count} without the next free slot."""
        count, nxt = int(meta[0]), int(meta[1])
        return [s for s in range(min(count + 1, cap)) if s != nxt]


class LockStep:
    """Oracle lists for `rows` of a GPU decode state, checked step by step."""

    def __init__(self, lists: dict, b: dict, L: dict, M: dict, gamma: float, T: int, dtype: str):
        self.lists, self.b, self.L, self.M = lists, b, L, M
        self.gamma, self.T = gamma, T
        self.tol = 2e-2 if dtype == "bf16" else 1e-4
        self.bf16 = dtype == "bf16"
        self.ties = 0
        self.checked = 0

    def step(self, t: int, snap: Snapshot, out: np.ndarray, q, k, v) -> None:
        """Checks step t on every row: out [rows][g][d] is the GPU output,
        q [rows][g][d], k, v [rows][d] the step's inputs (host)."""
        for r in list(self.lists):
            lst = self.lists[r]
            args = (q[r], k[r], v[r], self.L[r] + t)
            before = lst.clone()
            o_orc, ev_orc = lst.step(*args, self.gamma, self.T, self.M[r], self.b[r])
            err = np.abs(out[r] - o_orc).max()
            lim = self.tol if self.bf16 else self.tol * np.abs(o_orc).max()
            assert err <= lim, ("output", t, r, float(err))
            meta, pos, _ = snap.row(r)
            e_slot = int(meta[3])
            ev_gpu = -1 if e_slot < 0 else int(pos[e_slot])
            if ev_gpu != ev_orc:
                # replay the oracle step without eviction to read every entry's A
                before.step(*args, self.gamma, self.T, self.M[r], 1 << 40)
                _, _, A_all, pos_all = before.entries()
                amap = dict(zip(pos_all.tolist(), A_all.tolist()))
                assert ev_gpu in amap and ev_orc in amap, ("eviction", t, r, ev_gpu, ev_orc)
                a_g, a_o = amap[ev_gpu], amap[ev_orc]
                assert abs(a_g - a_o) <= TIE_RTOL * max(abs(a_o), 1e-30), ("eviction", t, r, a_g, a_o)
                before.remove(ev_gpu)  # the oracle follows the GPU's equally correct choice
                self.lists[r] = before
                self.ties += 1
            self.checked += 1

    def compare_A(self, snap: Snapshot) -> None:
        """Positions and decayed scores of every occupied slot against the oracle's list."""
        for r, lst in self.lists.items():
            meta, pos, A = snap.row(r)
            slots = Snapshot.present_slots(meta, len(pos))
            _, _, A_o, pos_o = lst.entries()
            gp = {int(pos[s]): float(A[s]) for s in slots}
            assert sorted(gp) == sorted(pos_o.tolist()), ("positions", r)
            ga = np.array([gp[int(x)] for x in pos_o])
            np.testing.assert_allclose(ga, A_o, rtol=1e-4, atol=1e-6, err_msg=f"A of row {r}")


def oracle_lists(bt, rows, kept: dict, extra: int = 1) -> dict:
    """Oracle lists of `rows` starting from the kept positions kept[r]."""
    koff = bt.key_off
    out = {}
    for r in rows:
        idx = np.asarray(kept[r], np.int64)
        out[r] = orc.DecodeList(bt.K[koff[r] + idx], bt.V[koff[r] + idx], idx, extra=extra)
    return out
