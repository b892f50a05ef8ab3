"""The debug build (libkvcomp_debug.so: the kernels with their data-dependent
index checks compiled in). The GPU parity suites run again against it in a
child process, and every test must leave the check word at 0 (the autouse
fixture in conftest reads and clears it after each test). One case trips a
check on purpose: kv_select_gather given a row whose slot range is smaller
than the entries it writes. The input keeps every access inside the buffers
in either build (the row's writes overlap the next row's slots, not the end
of the array), so the release build would mix the rows without faulting; the
debug build skips the row, sets KV_DEV_BOUNDS and leaves the other row as a
consistent input makes it.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import synth
from tests._harness import dev, params_of, shape_of

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_parity.py", "tests/test_gpu_decode.py", "tests/test_gpu_next.py", "tests/test_gpu_c3.py",
          "tests/test_gpu_voxzip.py", "tests/test_gpu_wnw.py", "tests/test_gpu_pipeline.py",
          "tests/test_gpu_debug_checks.py"]


@pytest.mark.gpu
@pytest.mark.skipif(kv.DEBUG_CHECKS, reason="runs the suites from the release process")
def test_gpu_suites_clean_under_debug_build():
    from kv_cache_compression_layer_b200 import build as kvbuild

    kvbuild.build(debug=True)
    env = dict(os.environ, KV_DEBUG_CHECKS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", *SUITES, "-m", "gpu", "-x", "-q", "-rs", "-p",
                        "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "needs the debug build" not in r.stdout, r.stdout[-2000:]


@pytest.mark.gpu
@pytest.mark.debug_trips
@pytest.mark.skipif(not kv.DEBUG_CHECKS, reason="needs the debug build (KV_DEBUG_CHECKS=1)")
def test_select_flags_a_row_its_slots_cannot_hold():
    cfg = synth.small("3b", n_layers=1, L=(600,))
    bt = synth.make_batch(cfg, steps=1)
    dt = torch.bfloat16
    up = lambda x, t: torch.from_numpy(np.ascontiguousarray(x)).to(dev(), t)  # noqa: E731
    K, V = up(bt.K, dt), up(bt.V, dt)
    comp = kv.Compressor(shape_of(cfg), cfg.L, params_of(cfg), device=dev())
    comp.allocate(up(bt.S, torch.float32))
    comp.score(up(bt.qwin, dt), K)
    comp.sss()
    comp.select_gather(K, V)
    torch.cuda.synchronize()
    assert kv.kv_debug_check_word(clear=True) == 0
    assert cfg.rows == 2
    b = comp.b.cpu().tolist()
    assert min(b) > 16

    # row 0 gets 10 slots for its b0 entries; row 1 sits right after them
    slot_off = torch.tensor([0, 10, 10 + b[1] + 1], dtype=torch.int64, device=dev())
    total = int(comp.slot_off[-1])  # the consistent layout's slot count: room for both rows' writes
    idx = torch.full((total,), -1, dtype=torch.int32, device=dev())
    Kc = torch.zeros(total, cfg.head_dim, dtype=dt, device=dev())
    Vc = torch.zeros_like(Kc)
    kv.kv_select_gather(comp.shape, cfg.L, comp.s_hat, K, V, comp.b, slot_off, idx, Kc, Vc)
    torch.cuda.synchronize()
    assert kv.kv_debug_check_word(clear=True) == kv.KV_DEV_BOUNDS
    assert kv.kv_debug_check_word() == 0  # cleared

    o1 = int(comp.slot_off[1])
    assert torch.equal(idx[10:10 + b[1]], comp.pos[o1:o1 + b[1]])  # row 1 as the consistent run made it
    assert torch.equal(Kc[10:10 + b[1]].view(torch.int16), comp.Kc[o1:o1 + b[1]].view(torch.int16))
    assert bool((idx[:10] == -1).all())  # row 0 was skipped
