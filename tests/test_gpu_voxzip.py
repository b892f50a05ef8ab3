"""kv_voxzip_pool against the oracle's VoxZip first stage: output row
descriptors and lengths bit-exact, copied rows bit-exact, pooled rows within
the rounding of a float32 sum and one rounding to the output type.

Tolerance per element of a pooled row (oracle in float64): rel * |o| +
count * 2^-23 * (max |E_A| + max |E_T|), rel = 2^-8 for bf16 output (one
rounding to 8 significant bits), 2^-22 for float32 output."""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import oracle as orc
import synth
from tests._harness import dev, up


def _segments_dev(tau, conf, n_text, text_row):
    raw = kv.pack_segments(tau, conf, n_text, text_row)
    if not raw:
        return None
    return torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(dev())


def _run(seqs, d, bf16, with_text=True, n_text_rows=None, conf_min=0.3):
    """seqs: list of (E_A, tau_total, tau, conf, n_text, text_row_local); text rows are laid out
    sequence after sequence. Returns GPU (E_comp, src, out_len, status) and the packed inputs."""
    tdt = torch.bfloat16 if bf16 else torch.float32
    L_a = [len(s[0]) for s in seqs]
    seg_off = np.concatenate([[0], np.cumsum([len(s[3]) for s in seqs])]).astype(np.int64)
    text_base = np.concatenate([[0], np.cumsum([int(np.maximum(s[4], 0).sum()) for s in seqs])]).astype(np.int64)
    tau = np.concatenate([s[2].reshape(-1, 2) for s in seqs]) if seg_off[-1] else np.zeros((0, 2))
    conf = np.concatenate([s[3] for s in seqs]).astype(np.float32)
    n_text = np.concatenate([s[4] for s in seqs]).astype(np.int32)
    text_row = np.concatenate([s[5] + text_base[i] for i, s in enumerate(seqs)]).astype(np.int32)
    E_A = np.concatenate([s[0] for s in seqs]).astype(np.float32)
    n_tr = int(text_base[-1])
    E_T = synth.text_embeddings(7, max(n_tr, 1), d, bf16) if with_text else None
    rows = sum(L_a)
    E_comp = torch.full((rows, d), 7.0, dtype=tdt, device=dev())
    src = torch.full((rows, 3), -5, dtype=torch.int32, device=dev())
    out_len = torch.zeros(len(seqs), dtype=torch.int32, device=dev())
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    E_T_dev = up(E_T, tdt) if with_text else None
    kv.kv_voxzip_pool(L_a, [s[1] for s in seqs], seg_off, d, kv.KV_BF16 if bf16 else kv.KV_F32,
                      _segments_dev(tau, conf, n_text, text_row), up(E_A, tdt), E_T_dev,
                      n_tr if n_text_rows is None else n_text_rows, E_comp, src, out_len,
                      status if with_text else None, conf_min=conf_min)
    torch.cuda.synchronize()
    return (E_comp.float().cpu().numpy(), src.cpu().numpy(), out_len.cpu().numpy(), int(status.item()),
            dict(L_a=L_a, E_A=E_A, E_T=E_T, tau=tau, conf=conf, n_text=n_text, text_row=text_row, seg_off=seg_off))


def _check(seqs, d, bf16, with_text=True, cols=None):
    E_comp, src, out_len, status, inp = _run(seqs, d, bf16, with_text)
    assert status == 0
    rel = 2.0 ** -8 if bf16 else 2.0 ** -22
    scale = float(np.abs(inp["E_A"]).max()) + (float(np.abs(inp["E_T"]).max()) if with_text else 0.0)
    row0 = 0
    for i, s in enumerate(seqs):
        a, b = inp["seg_off"][i], inp["seg_off"][i + 1]
        E = inp["E_A"][row0:row0 + len(s[0])]
        c = slice(None) if cols is None else cols
        o_out, o_src = orc.voxzip_pool(E[:, c], s[1], inp["tau"][a:b], inp["conf"][a:b], inp["n_text"][a:b],
                                       inp["text_row"][a:b], inp["E_T"][:, c] if with_text else None)
        n = len(o_src)
        assert out_len[i] == n
        np.testing.assert_array_equal(src[row0:row0 + n], o_src)
        g = E_comp[row0:row0 + n][:, c]
        copied = o_src[:, 2] < 0
        np.testing.assert_array_equal(g[copied], o_out[copied])  # copied rows are exact
        tol = rel * np.abs(o_out) + o_src[:, 1:2] * 2.0 ** -23 * scale
        assert (np.abs(g - o_out) <= tol).all(), float((np.abs(g - o_out) / tol).max())
        assert (E_comp[row0 + n:row0 + len(s[0])] == 7.0).all()  # rows past out_len untouched
        row0 += len(s[0])


def _seq(seed, L, d, bf16=True):
    a = synth.asr_segments(seed, L)
    return (synth.audio_features(seed, L, d, bf16), a.tau_total, a.tau, a.conf, a.n_text, a.text_row)


@pytest.mark.gpu
@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("d", [64, 1000, 2048])
def test_pool_random_layouts(bf16, d):
    if not bf16 and d == 1000:
        d = 1004  # 16-byte float32 rows
    _check([_seq(1, 3000, d, bf16), _seq(2, 64, d, bf16), _seq(3, 1777, d, bf16)], d, bf16)


@pytest.mark.gpu
def test_pool_without_text_and_edge_layouts():
    d = 256
    rng = np.random.default_rng(5)
    L = 500
    E = synth.audio_features(9, L, d)
    # overlap, out of order, empty, negative and past-the-end times, a cut exactly at 0.3, text > rows
    tau = np.array([[5, 20], [10, 30], [2, 8], [31, 31], [-4, 3], [38, 1e6], [33, 36], [32.5, 33.5]], np.float64)
    conf = np.array([0.9, 0.8, 0.95, 0.9, 0.5, 0.7, np.float32(0.3), 0.99], np.float32)
    n_text = np.array([4, 3, 2, 1, 9, 17, 2, 40], np.int32)
    tr = np.concatenate([[0], np.cumsum(n_text)[:-1]]).astype(np.int32)
    seqs = [(E, 40.0, tau, conf, n_text, tr), (synth.audio_features(10, 333, d), 1.0, np.zeros((0, 2)),
                                               np.zeros(0, np.float32), np.zeros(0, np.int32),
                                               np.zeros(0, np.int32))]
    _check(seqs, d, True, with_text=True)
    _check(seqs, d, True, with_text=False)
    del rng


@pytest.mark.gpu
def test_pool_text_rows_out_of_range_are_reported():
    d = 128
    s = _seq(4, 2000, d)
    _, src, out_len, status, inp = _run([s], d, True, n_text_rows=10)
    assert status & kv.KV_DEV_RANGE
    n = out_len[0]
    kept = src[:n][src[:n, 1] > 1]
    assert len(kept) > 0 and (src[:n, 2] < 10).all()  # no text row at or past the limit is used


@pytest.mark.gpu
def test_pool_full_size_sampled_columns():
    """The bench's workload (8 sequences of 32768 feature rows, d = 2048, bf16),
    compared on 64 columns spread over the row (the pooling is column-wise)."""
    d = 2048
    seqs = [_seq(100 + i, 32768, d) for i in range(8)]
    cols = np.unique(np.linspace(0, d - 1, 64).astype(int))
    _check(seqs, d, True, cols=cols)
