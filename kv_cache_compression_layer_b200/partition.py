"""Host logic of splitting one batch over several GPUs, one process each.

Every (sequence, layer, KV head) row of the path is an independent problem:
scoring, smoothing, selection, gathering and decoding read and write only
the row's own data, and the budget allocation couples only the KV heads of
one (sequence, layer) (AudioKV blog §3.1: the budget of a layer is shared by
its heads). So a batch splits without any data exchange along whole
sequences or along whole layers, and every rank runs the path on its part:

* by sequences: each rank takes some sequences with all their layers (the
  greedy longest-first assignment by audio length, which the work of a
  sequence is proportional to);
* by layers: each rank takes a contiguous range of layers of every sequence.

``partition`` picks whichever split has the smaller largest share. A part
carries the global index of each of its rows, so per-row results of all
ranks reassemble into the one-process result (``assemble_rows``). The pooled
allocation over all layers of a sequence (kv_allocate_global) couples the
layers of a sequence, so with it only the split by sequences applies.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence

import numpy as np


@dataclass(frozen=True)
class Part:
    """One rank's share of a batch."""

    rank: int
    seqs: tuple        # the batch's sequence indices this rank takes, ascending
    layers: tuple      # (first, end) layer range taken of each of those sequences
    L: tuple           # the audio lengths of those sequences
    rows: np.ndarray   # global row index of each of the rank's rows, in the rank's row order

    @property
    def n_layers(self) -> int:
        return self.layers[1] - self.layers[0]

    def key_ranges(self, n_layers: int, n_kv_heads: int, L_all: Sequence[int]) -> List[tuple]:
        """[(first key, end key)) blocks of the batch's concatenated per-key tensors
        (K, V, s) that make up this rank's rows, in the rank's row order."""
        H = n_kv_heads
        seq_key = np.concatenate([[0], np.cumsum([n_layers * H * int(x) for x in L_all])]).astype(np.int64)
        out = []
        for s in self.seqs:
            l0, l1 = self.layers
            base = int(seq_key[s])
            out.append((base + l0 * H * int(L_all[s]), base + l1 * H * int(L_all[s])))
        return out


def _rows_of(seqs, layers, n_layers: int, H: int) -> np.ndarray:
    l0, l1 = layers
    return np.array([(s * n_layers + l) * H + h for s in seqs for l in range(l0, l1) for h in range(H)], np.int64)


def split_by_sequences(n_layers: int, n_kv_heads: int, L: Sequence[int], world: int) -> List[Part]:
    """Sequences to ranks, longest first, each to the least-loaded rank (ties: lower rank)."""
    if world < 1 or world > len(L):
        raise ValueError("split by sequences needs 1 <= world <= n_seq")
    load = [0] * world
    owner = [0] * len(L)
    for s in sorted(range(len(L)), key=lambda i: (-int(L[i]), i)):
        r = min(range(world), key=lambda k: (load[k], k))
        owner[s] = r
        load[r] += int(L[s])
    parts = []
    for r in range(world):
        seqs = tuple(s for s in range(len(L)) if owner[s] == r)
        parts.append(Part(r, seqs, (0, n_layers), tuple(int(L[s]) for s in seqs),
                          _rows_of(seqs, (0, n_layers), n_layers, n_kv_heads)))
    return parts


def split_by_layers(n_layers: int, n_kv_heads: int, L: Sequence[int], world: int) -> List[Part]:
    """Contiguous layer ranges [floor(r n / world), floor((r + 1) n / world)) of every sequence."""
    if world < 1 or world > n_layers:
        raise ValueError("split by layers needs 1 <= world <= n_layers")
    seqs = tuple(range(len(L)))
    parts = []
    for r in range(world):
        rng = (r * n_layers // world, (r + 1) * n_layers // world)
        parts.append(Part(r, seqs, rng, tuple(int(x) for x in L), _rows_of(seqs, rng, n_layers, n_kv_heads)))
    return parts


def largest_share(parts: Sequence[Part]) -> int:
    """The largest rank's work in key rows (rows x audio length)."""
    return max(p.n_layers * sum(p.L) for p in parts)


def partition(n_layers: int, n_kv_heads: int, L: Sequence[int], world: int) -> List[Part]:
    """The split (by sequences or by layers) whose largest share is smaller; by layers on a tie."""
    cands = []
    if world <= n_layers:
        cands.append(split_by_layers(n_layers, n_kv_heads, L, world))
    if world <= len(L):
        cands.append(split_by_sequences(n_layers, n_kv_heads, L, world))
    if not cands:
        raise ValueError("more ranks than layers and sequences")
    return min(cands, key=largest_share)


def assemble_rows(parts: Sequence[Part], per_rank: Sequence[Sequence]) -> list:
    """Per-row values of every rank (in each rank's row order) in the batch's global row order;
    checks that every row comes from exactly one rank."""
    n = sum(len(p.rows) for p in parts)
    out = [None] * n
    seen = np.zeros(n, bool)
    for p, vals in zip(parts, per_rank):
        if len(vals) != len(p.rows):
            raise ValueError(f"rank {p.rank}: {len(vals)} values for {len(p.rows)} rows")
        for g, v in zip(p.rows.tolist(), vals):
            if seen[g]:
                raise ValueError(f"row {g} comes from two ranks")
            seen[g] = True
            out[g] = v
    if not seen.all():
        raise ValueError("rows missing from every rank")
    return out
