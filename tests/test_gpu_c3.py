"""kv_c3_build and kv_c3_step against the oracle's C3 row, row by row: the
index (member order, node table, float64 centroids), the frontier, the
scores, the retrieved positions, the EMA and the frontier after the
exchanges bit-exact over several decode steps; the attention outputs within
2e-2 absolute (bf16) or 1e-4 relative (float32) of the oracle's float64."""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._harness import dev, up

pytestmark = pytest.mark.gpu


def _view(index, off, n, dtype):
    item = torch.tensor([], dtype=dtype).element_size()
    return index[off:off + n * item].view(dtype)


def _run(Ls, n_layers, H, G, d, bf16, B, steps, lam=0.5, R=2, seed=0):
    tdt = torch.bfloat16 if bf16 else torch.float32
    shape = kv.make_shape(n_layers, H, G, d, 1, kv.KV_BF16 if bf16 else kv.KV_F32)
    p = kv.make_c3_params(B, lam=lam, exchanges=R)
    rng = np.random.default_rng(seed)
    rows = len(Ls) * n_layers * H
    Lr = [Ls[r // (n_layers * H)] for r in range(rows)]
    koff = np.concatenate([[0], np.cumsum(Lr)]).astype(np.int64)
    T = int(koff[-1])
    # keys with cluster structure (an AR(1) latent, as in the audio workloads), values N(0, 1)
    K = np.concatenate([synth.round_bf16(np.cumsum(rng.standard_normal((L, d)), 0).astype(np.float32) * 0.1
                                         + rng.standard_normal((L, d)).astype(np.float32)) for L in Lr])
    V = synth.round_bf16(rng.standard_normal((T, d)).astype(np.float32))
    if not bf16:
        K = K.astype(np.float32)
    lay = kv.kv_c3_index_layout(shape, Ls, p)
    index = torch.zeros(lay.bytes, dtype=torch.uint8, device=dev())
    Kd, Vd = up(K, tdt), up(V, tdt)
    kv.kv_c3_build(shape, Ls, p, Kd, index)
    torch.cuda.synchronize()
    ref = [orc.C3Row(K[koff[r]:koff[r + 1]], V[koff[r]:koff[r + 1]]) for r in range(rows)]
    hdr = _view(index, lay.hdr, rows * 4, torch.int32).view(rows, 4).cpu().numpy()
    perm = _view(index, lay.perm, T, torch.int32).cpu().numpy()
    node = {k: _view(index, getattr(lay, k), 2 * T, torch.int32).cpu().numpy() for k in ("lo", "cnt", "left", "depth")}
    cent = _view(index, lay.cent, 2 * T * d, torch.float64).view(2 * T, d).cpu().numpy()
    for r, o in enumerate(ref):
        no = 2 * koff[r]
        assert hdr[r, 0] == o.n_nodes and hdr[r, 1] == o.A, r
        np.testing.assert_array_equal(perm[koff[r]:koff[r + 1]], o.perm[:Lr[r]])
        for k in ("lo", "cnt", "left", "depth"):
            np.testing.assert_array_equal(node[k][no:no + o.n_nodes], getattr(o, k)[:o.n_nodes], err_msg=k)
        np.testing.assert_array_equal(cent[no:no + o.n_nodes], o.cent[:o.n_nodes])
    out = torch.zeros(rows, G, d, dtype=tdt, device=dev())
    for t in range(steps):
        q = synth.round_bf16(rng.standard_normal((rows, G, d)).astype(np.float32))
        kv.kv_c3_step(shape, Ls, p, Kd, Vd, up(q, tdt), index, out)
        torch.cuda.synchronize()
        hdr = _view(index, lay.hdr, rows * 4, torch.int32).view(rows, 4).cpu().numpy()
        sel = _view(index, lay.sel, T, torch.int32).cpu().numpy()
        sig = _view(index, lay.sigma, 2 * T, torch.float64).cpu().numpy()
        e = _view(index, lay.e, 2 * T, torch.float64).cpu().numpy()
        front = _view(index, lay.front, 2 * T, torch.int32).cpu().numpy()
        o_gpu = out.float().cpu().numpy()
        for r, o in enumerate(ref):
            no = 2 * koff[r]
            A0 = o.A
            o_ref, sel_ref, sig_ref = o.step(q[r], B, lam=lam, R=R)
            assert hdr[r, 2] == len(sel_ref), (t, r)
            np.testing.assert_array_equal(sel[koff[r]:koff[r] + len(sel_ref)], sel_ref, err_msg=f"step {t} row {r}")
            if Lr[r] > B:
                np.testing.assert_array_equal(sig[no:no + A0], sig_ref, err_msg=f"step {t} row {r}")
            np.testing.assert_array_equal(front[no:no + o.A], o.front)
            np.testing.assert_array_equal(e[no:no + o.n_nodes], o.e)
            if bf16:
                assert np.abs(o_gpu[r] - o_ref).max() <= 2e-2, (t, r)
            else:
                np.testing.assert_allclose(o_gpu[r], o_ref, rtol=1e-4, atol=1e-5)


def test_c3_bf16_two_sequences():
    # 2 sequences x 2 layers x 2 KV heads, g = 4, d = 64; budget 128 (the tight setting on the page)
    _run([700, 1500], n_layers=2, H=2, G=4, d=64, bf16=True, B=128, steps=6)


def test_c3_f32_wide_heads_and_bypass():
    # d = 128, g = 8; the 200-key sequence is below the budget and bypasses retrieval
    _run([3000, 200], n_layers=1, H=2, G=8, d=128, bf16=False, B=256, steps=5, R=4)


def test_c3_long_row():
    _run([8192], n_layers=1, H=1, G=4, d=128, bf16=True, B=512, steps=4, lam=0.2, R=3)
