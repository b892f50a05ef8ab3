"""bench.py's host-side bookkeeping, without a GPU: the kernel the roofline
names, the ncu traffic record and its source check, the peak's fallback, the
oracle sample's rows and the audio tokens they stand for, and the config dict
both arms print."""
import dataclasses
import json

import pytest

import bench
import synth


def test_decode_kernel_follows_the_library_rule():
    assert bench.decode_kernel(synth.CONFIGS["ragged"]) == "decode_tc_kernel"  # bf16, g = 7
    assert bench.decode_kernel(synth.CONFIGS["3b"]) == "decode_tc_kernel"  # bf16, g = 8
    assert bench.decode_kernel(synth.CONFIGS["tiny"]) == "decode_simple_kernel"  # fp32
    assert bench.decode_kernel(synth.small("3b", n_layers=1, group=16)) == "decode_simple_kernel"


def test_traffic_record_holds_only_for_the_captured_source(monkeypatch):
    for name in ("ragged", "3b"):
        rec = bench.NCU_TRAFFIC[name]
        assert bench.measured_traffic(name) == rec["bytes"] > 0
    assert bench.measured_traffic("long") is None  # no capture recorded
    stale = dict(bench.NCU_TRAFFIC, ragged=dict(bench.NCU_TRAFFIC["ragged"], sha256="0" * 16))
    monkeypatch.setattr(bench, "NCU_TRAFFIC", stale)
    assert bench.measured_traffic("ragged") is None


def test_peak_falls_back_without_the_measured_file(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    assert bench.hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    p = tmp_path / "peaks.json"
    p.write_text(json.dumps({"hbm_gbs": 6400.5, "bf16_tflops": 1600}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(p))
    assert bench.hbm_peak() == (6400.5, "measured")


@pytest.mark.parametrize("name,n", [("ragged", 64), ("ragged", 8), ("3b", 64), ("long", 5)])
def test_sample_rows_spread_over_the_batch(name, n):
    cfg = synth.CONFIGS[name]
    rows = bench.sample_rows(cfg, n)
    assert rows == sorted(set(rows)) and len(rows) == min(n, cfg.rows)
    assert rows[0] == 0 and rows[-1] == cfg.rows - 1
    per_seq = cfg.n_layers * cfg.n_kv_heads
    if n % cfg.n_seq == 0:  # the batch's length mix: the same count from every sequence
        counts = [sum(1 for r in rows if r // per_seq == s) for s in range(cfg.n_seq)]
        assert counts == [n // cfg.n_seq] * cfg.n_seq


def test_sample_tokens_add_up_to_the_batch():
    cfg = synth.CONFIGS["ragged"]
    assert bench.sample_tokens(cfg, range(cfg.rows)) == pytest.approx(sum(cfg.L))
    one_seq = range(cfg.n_layers * cfg.n_kv_heads)  # all rows of the first sequence
    assert bench.sample_tokens(cfg, one_seq) == pytest.approx(cfg.L[0])


def test_both_arms_describe_the_workload_alike():
    cfg = synth.CONFIGS["ragged"]
    d = bench.config_dict(cfg, 1)
    assert set(d) == {"workload", "n_seq", "rows", "l2", "parallelism"}
    assert d["rows"] == 896 and d["n_seq"] == 8 and "ragged" in d["workload"]
    assert bench.config_dict(cfg, 4)["parallelism"].startswith("replicas x4")
    layered = dataclasses.replace(cfg, n_layers=7) if dataclasses.is_dataclass(cfg) else cfg.with_(n_layers=7)
    assert bench.config_dict(layered, 1)["rows"] == 224
