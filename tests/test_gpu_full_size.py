"""The full-size workloads in the benchmark's launch configuration: every row
of the batch runs through ``Compressor`` (the calls the benchmark times) and
32 decode steps of the whole batch; sampled rows are checked against the
oracle end to end (scores, k*, s_hat, selection, gathers, then every decode
step in lock step), budgets on every row.

The sampled rows include the row with the largest budget, so the largest
decode rows (30B-class: b near 6400, split over several work items and CTAs
of the persistent decode kernel), the L = 32768 chain end to end, and g = 7
on the persistent path (the ragged batch) are all covered.
"""
import numpy as np
import pytest

import synth
from tests._pipeline import check_compress_rows, compress, decode_lockstep

pytestmark = pytest.mark.gpu

STEPS = 32


def _sample(cfg, b):
    """The first and last rows, the largest budget, and one row of each sequence's middle layer."""
    rows = {0, cfg.rows - 1, int(np.argmax(b))}
    per_seq = cfg.n_layers * cfg.n_kv_heads
    for s in range(cfg.n_seq):
        rows.add(s * per_seq + per_seq // 2 + s % cfg.n_kv_heads)
    return sorted(rows)


@pytest.mark.parametrize("name", ["30b", "ragged", "long"])
def test_full_size_sampled_rows(name):
    cfg = synth.CONFIGS[name]
    bt = synth.make_batch(cfg, steps=STEPS)
    comp, K, V = compress(cfg, bt)
    del K, V
    rows = _sample(cfg, comp.b.cpu().numpy())
    kept, _ = check_compress_rows(cfg, bt, comp, rows)
    if bt.spikes is None:  # every row: its window rows' softmaxes sum to R (spikes rescale s in place)
        s = comp.s.cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(np.add.reduceat(s, bt.key_off[:-1]), cfg.R, rtol=1e-4)
    ls = decode_lockstep(cfg, bt, comp, kept, STEPS)
    assert ls.checked == len(rows) * STEPS
    assert ls.ties <= max(1, len(rows) // 4)
