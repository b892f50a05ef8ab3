"""End-to-end parity: the whole path through the C ABI (``Compressor``, the
same calls the benchmark times) against the oracle's chain on the same seeded
inputs. Small workloads are checked on every row (compression, then decode in
lock step); the full 3B-class workload (36 layers x 2 KV heads, L = 6000) on
sampled rows. The other full-size workloads are in test_gpu_full_size.py.
"""
import numpy as np
import pytest

import synth
from tests._pipeline import check_compress_rows, compress, decode_lockstep

pytestmark = pytest.mark.gpu

SMALL = [
    (synth.CONFIGS["tiny"], 8),
    (synth.small("3b", n_layers=2, L=(2000,)), 6),
    (synth.small("ragged", n_layers=2, L=(1000, 3500)), 6),  # spikes, g = 7
    (synth.small("30b", n_layers=2, L=(4000,)), 6),
    (synth.small("long", n_layers=1, L=(8000,)), 6),  # 5% budget
]


@pytest.mark.parametrize("cfg,steps", SMALL, ids=lambda c: getattr(c, "name", str(c)))
def test_pipeline_small_all_rows(cfg, steps):
    bt = synth.make_batch(cfg, steps=steps)
    comp, _, _ = compress(cfg, bt)
    kept, same = check_compress_rows(cfg, bt, comp, range(cfg.rows))
    assert len(same) >= cfg.rows // 2
    ls = decode_lockstep(cfg, bt, comp, kept, steps)
    assert ls.ties <= max(1, cfg.rows // 4)


def test_pipeline_3b_full_size_sampled_rows():
    cfg = synth.CONFIGS["3b"]
    steps = 32
    bt = synth.make_batch(cfg, steps=steps)
    comp, _, _ = compress(cfg, bt)
    kept, _ = check_compress_rows(cfg, bt, comp, [0, 37, 71])
    # invariant on every row: each window row's softmax sums to 1
    s = comp.s.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(np.add.reduceat(s, bt.key_off[:-1]), cfg.R, rtol=1e-4)
    ls = decode_lockstep(cfg, bt, comp, kept, steps)
    assert ls.checked == 3 * steps
