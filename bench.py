#!/usr/bin/env python
"""Benchmark of the KV selection/compaction path on B200.

One step = one pass of the whole path over one batch of the workload:
kv_allocate -> kv_score -> kv_sss -> kv_select_gather -> kv_decode_init ->
the workload's decode steps (kv_decode_attn_update, all layers per launch).
`value` = audio tokens of the batch processed per second of step time (for N
ranks: N x that, each rank running its own replica; no data-path collective).

Default workload: the ragged batch (8 sequences, L 2000-16000, 28 layers,
28 q / 4 kv heads, budget 25%, 128 decode steps), the largest that fits one
GPU; --config names another.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--config ragged]
       python bench.py --impl reference ...   (the CPU oracle as the arm)
Multi-GPU: python -m torch.distributed.run --nproc-per-node N bench.py --gpus N
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "compressed audio tokens/s (score→SSS→top-k→gather), decode µs/step; % HBM peak"
UNIT = "audio tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (read + write) of one decode kernel launch from an ncu capture of
# this benchmark's workload (its summary is kept under profiles/), valid while
# the kernel source is the one captured (its SHA-256 below); otherwise null.
# (Source b74cfb7b… differs from the captured 683f49d2… only by index checks
# that release builds compile away: the two compile to the same device code.)
NCU_TRAFFIC = {"3b": {"bytes": 140328704,  # profiles/decode_tc_kernel_3b.md (the full workload)
                      "source": "kv_cache_compression_layer_b200/csrc/decode_tc.cu",
                      "sha256": "b74cfb7b71ccce01"},
               # profiles/decode_tc_kernel_ragged7.md: the 7-layer capture (257,023,232 B for
               # 483,224 slots) scaled by the slots of the full batch (x 4)
               "ragged": {"bytes": 1028092928,
                          "source": "kv_cache_compression_layer_b200/csrc/decode_tc.cu",
                          "sha256": "b74cfb7b71ccce01"}}


def decode_kernel(cfg: synth.Config) -> str:
    """The decode kernel kv_decode_attn_update launches for this workload (the library's rule)."""
    if cfg.dtype != "bf16" or cfg.group > 8:
        return "decode_simple_kernel"
    return "decode_tc_kernel"


def measured_traffic(cfg_name: str):
    import hashlib
    rec = NCU_TRAFFIC.get(cfg_name)
    if not rec:
        return None
    try:
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return rec["bytes"] if rec["bytes"] and digest.startswith(rec["sha256"]) else None


def workload(args) -> synth.Config:
    """The named workload, or (--layers N) the same with N layers per sequence,
    a reduced case for profiler captures."""
    cfg = synth.CONFIGS[args.config]
    if args.layers:
        cfg = cfg.with_(n_layers=args.layers)
    return cfg


def describe(cfg: synth.Config) -> str:
    return (f"{cfg.name}: {cfg.n_seq} seq, L={list(cfg.L)}, {cfg.n_layers} layers, "
            f"{cfg.n_kv_heads * cfg.group} q / {cfg.n_kv_heads} kv heads, d={cfg.head_dim}, {cfg.dtype}, w={cfg.w}, "
            f"budget {cfg.budget_pct}%, alpha={cfg.alpha}, rho={cfg.rho}, r={cfg.r}, {cfg.decode_steps} decode steps "
            f"(gamma={cfg.gamma}, T={cfg.sinks_T}, M={cfg.recent_pct}%)")


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------- clocks --
class ClockSampler:
    """Samples the SM clock and throttle reasons through NVML (read-only)."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, torch_dev: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
            self._h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------ CPU baseline --
def oracle_sample(cfg: synth.Config, bt: synth.Batch, rows, n_threads: int):
    """Runs the oracle's whole path on `rows` of the batch; returns seconds."""
    import oracle as orc

    t0 = time.perf_counter()
    L_rows = [int(bt.L_rows[r]) for r in rows]
    koff = bt.key_off
    Ks = np.concatenate([bt.K[koff[r]:koff[r + 1]] for r in rows])
    b_all = orc.allocate(bt.S, cfg.L, cfg.w, cfg.budget_pct, cfg.r).reshape(-1)
    s = orc.score(bt.qwin[rows], Ks, L_rows, n_threads=n_threads)
    if bt.spikes is not None:
        s = s * np.concatenate([np.where(bt.spikes[koff[r]:koff[r + 1]], 10.0, 1.0) for r in rows])
    s_hat, _ = orc.sss(s, L_rows, cfg.alpha, cfg.rho, n_threads=n_threads)
    b = [int(b_all[r]) for r in rows]
    idx = orc.select(s_hat, L_rows, cfg.w, b, n_threads=n_threads)
    Kc = [bt.K[koff[r] + idx[i]] for i, r in enumerate(rows)]
    Vc = [bt.V[koff[r] + idx[i]] for i, r in enumerate(rows)]
    M = [orc.recent_count(x, cfg.recent_pct) for x in b]
    orc.decode_run_heads(Kc, Vc, idx, bt.q_dec[:, rows], bt.k_dec[:, rows], bt.v_dec[:, rows],
                         np.array(L_rows, np.int64), cfg.gamma, cfg.sinks_T, M, np.array(b, np.int64),
                         n_threads=n_threads)
    return time.perf_counter() - t0


def sample_rows(cfg: synth.Config, n: int):
    """n rows spread evenly over the batch (the same number from every
    sequence when n is a multiple of n_seq), so the sample has the batch's
    length mix."""
    n = max(1, min(n, cfg.rows))
    return sorted({int(x) for x in np.linspace(0, cfg.rows - 1, n).round()})


def sample_tokens(cfg: synth.Config, rows) -> float:
    """Audio tokens a sample of rows stands for: each of a sequence's
    n_layers x n_kv_heads rows carries 1/(n_layers x n_kv_heads) of its L."""
    per_seq = cfg.n_layers * cfg.n_kv_heads
    return float(sum(cfg.row_L(r) for r in rows)) / per_seq


def config_dict(cfg: synth.Config, world: int) -> dict:
    """The workload description both arms print (identical keys and values)."""
    return {"workload": describe(cfg), "n_seq": cfg.n_seq, "rows": cfg.rows,
            "l2": "256 MB write between timed steps (outside the events)",
            "parallelism": f"replicas x{world} (rows independent, no collective)"}


def cpu_baseline(cfg, bt, n_rows_sample: int):
    """The oracle timed on a bounded sample of the batch's rows (all host threads)."""
    import oracle as orc

    threads = orc.default_threads()
    rows = sample_rows(cfg, n_rows_sample)
    orc.build()
    secs = oracle_sample(cfg, bt, rows, threads)
    return {"value": sample_tokens(cfg, rows) / secs, "unit": UNIT, "cores": min(threads, len(rows)),
            "kind": "oracle", "seconds": secs,
            "sample": f"{len(rows)} of {cfg.rows} rows ({len(rows) // cfg.n_seq if len(rows) % cfg.n_seq == 0 else '~'}"
                      f" per sequence) through the whole path incl. {cfg.decode_steps} decode steps, timed "
                      f"{secs:.2f} s; value = the sample's share of the batch's audio tokens / that time"}


# ------------------------------------------------------------------ our arm --
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import kv_cache_compression_layer_b200 as kv
    from kv_cache_compression_layer_b200 import Compressor
    from kv_cache_compression_layer_b200.replicas import init_group, job_throughput, max_over_ranks, replica_seed

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    init_group("nccl", world, dev)
    cfg = workload(args)
    cfg = cfg.with_(seed=replica_seed(cfg.seed, rank))
    bt = synth.make_batch(cfg)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = kv.make_shape(cfg.n_layers, cfg.n_kv_heads, cfg.group, cfg.head_dim, cfg.w,
                          kv.KV_BF16 if cfg.dtype == "bf16" else kv.KV_F32)
    params = kv.make_params(cfg.budget_pct, cfg.alpha, cfg.rho, cfg.r, cfg.gamma, cfg.sinks_T, cfg.recent_pct)

    def h(x, dtype):
        return torch.from_numpy(np.ascontiguousarray(x)).to(dtype)

    host = {"qwin": h(bt.qwin, dt), "K": h(bt.K, dt), "V": h(bt.V, dt), "S": h(bt.S, torch.float32),
            "q": h(bt.q_dec, dt), "k": h(bt.k_dec, dt), "v": h(bt.v_dec, dt)}
    if bt.spikes is not None:
        host["spikes"] = h(np.where(bt.spikes, 10.0, 1.0), torch.float32)
    d_in = {k: v.to(dev) for k, v in host.items()}
    comp = Compressor(shape, cfg.L, params, device=dev)
    D = cfg.decode_steps
    out = torch.empty(D, cfg.rows, cfg.group, cfg.head_dim, dtype=dt, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2

    def step(x, dec_events=None):
        comp.compress(x["qwin"], x["K"], x["V"], x["S"], spikes=x.get("spikes"), stream=stream)
        for t in range(D):
            if dec_events is not None:
                dec_events[t][0].record(stream)
            comp.decode_step(x["q"][t], x["k"][t], x["v"][t], out[t], stream=stream)
            if dec_events is not None:
                dec_events[t][1].record(stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for _ in range(args.warmup):
        step(d_in)
    torch.cuda.synchronize()
    st = kv.kv_read_device_status(comp.status, stream) | kv.kv_read_device_status(comp.ws[:4].view(torch.int32),
                                                                                  stream)
    if st:
        raise RuntimeError(f"device status {st:#x} after warm-up")

    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    step_ev = [(E(), E(), E()) for _ in range(args.steps)]
    dec_ev = [[(E(), E()) for _ in range(D)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            torch.cuda._sleep(SPACER_CYCLES)  # the host enqueues the step meanwhile (outside the events)
            step_ev[i][0].record(stream)
            comp.compress(d_in["qwin"], d_in["K"], d_in["V"], d_in["S"], spikes=d_in.get("spikes"), stream=stream)
            step_ev[i][1].record(stream)
            for t in range(D):
                dec_ev[i][t][0].record(stream)
                comp.decode_step(d_in["q"][t], d_in["k"][t], d_in["v"][t], out[t], stream=stream)
                dec_ev[i][t][1].record(stream)
            step_ev[i][2].record(stream)
        torch.cuda.synchronize()
    barrier()
    step_ms = [a.elapsed_time(c) for a, _, c in step_ev]
    comp_ms = [a.elapsed_time(b) for a, b, _ in step_ev]
    dec_us = [1e3 * s.elapsed_time(e) for row in dec_ev for s, e in row]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), world, dev)
    tokens = sum(cfg.L)
    value = job_throughput(tokens, world, ms)

    # end to end through the library from pinned host buffers: every step copies its inputs
    # over the host link and reads all decode outputs back inside the timed region. K goes
    # over one sequence at a time while the sequences already on the device are scored and
    # smoothed; V stays on the host and select + gather reads the kept rows; the decode
    # inputs and outputs cross during the decode steps (Compressor.compress_from_host,
    # Compressor.decode_from_host)
    pinned = {k: v.pin_memory() for k, v in host.items()}
    out_host = torch.empty(out.shape, dtype=dt).pin_memory()
    copy_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    e2e_ms = []
    h2d = 0
    for i in range(args.warmup + args.steps):
        flush.fill_(i & 0xFF)
        torch.cuda._sleep(SPACER_CYCLES)  # the host enqueues the step meanwhile (outside the events)
        a, c = E(), E()
        a.record(stream)
        copied = comp.compress_from_host(pinned, d_in, stream=stream, copy_stream=copy_stream)
        comp.decode_from_host(pinned["q"], pinned["k"], pinned["v"], out_host, d_in["q"], d_in["k"], d_in["v"], out,
                              stream=stream, copy_stream=copy_stream, d2h_stream=d2h_stream)
        c.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(c))
        h2d = copied + sum(pinned[k].numel() * pinned[k].element_size() for k in ("q", "k", "v"))
    e2e = max_over_ranks(sum(e2e_ms) / len(e2e_ms), world, dev)
    kept_v = int(comp.b.to(torch.int64).sum().item()) * cfg.head_dim * (2 if cfg.dtype == "bf16" else 4)
    h2d += kept_v  # the kept V rows select + gather reads over the link
    d2h = out_host.numel() * out_host.element_size()

    # roofline of the dominant kernel (the decode step) and of the compress stage
    b = comp.b.cpu().numpy().astype(np.int64)
    d = cfg.head_dim
    eb = 2 if cfg.dtype == "bf16" else 4
    dec_bytes = int(((b + 1) * (2 * eb * d + 8) + 2 * eb * d).sum())
    dec_avg_us = sum(dec_us) / len(dec_us)
    L_rows = np.array([cfg.L[cfg.row_triplet(r)[0]] for r in range(cfg.rows)], np.int64)
    # K read once, kept V read once, compacted K and V written once
    comp_bytes = int((eb * d * (L_rows + 3 * b)).sum())
    comp_avg_ms = sum(comp_ms) / len(comp_ms)
    peak, peak_kind = hbm_peak()
    dec_gbs = dec_bytes / (dec_avg_us * 1e-6) / 1e9
    comp_gbs = comp_bytes / (comp_avg_ms * 1e-3) / 1e9
    # our kernels per step: allocate 2, score 3, SSS 1, select 1, gather 1,
    # decode init 1 (+ the work-item builder on the tensor-core decode path),
    # then one kernel per decode call
    tc = cfg.dtype == "bf16" and cfg.group <= 8
    launches_per_step = 2 + 3 + 1 + 1 + 1 + 1 + (1 if tc else 0) + D

    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic (seeded AR(1) keys, diagonal-band queries; stands in for long-audio workloads)",
        "config": config_dict(cfg, world),
        "stages": {"compress_ms": comp_avg_ms, "compress_tokens_per_s": world * tokens / (comp_avg_ms * 1e-3),
                   "compress_bytes_alg": comp_bytes, "compress_gbs": comp_gbs,
                   "compress_hbm_frac": comp_gbs / peak, "decode_us_per_step": dec_avg_us,
                   "decode_bytes_alg": dec_bytes, "decode_steps": D},
        "roofline": {"kernel": decode_kernel(cfg)
                     + " (kv_decode_attn_update)", "bound": "hbm", "achieved": dec_gbs,
                     "peak": peak, "unit": "GB/s", "frac": dec_gbs / peak, "traffic": measured_traffic(args.config) if tc and not args.layers else None,
                     "peak_kind": peak_kind + " (hbm_gbs copy)"},
        "e2e": {"value": job_throughput(tokens, world, e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e,
                "path": "pinned host inputs; K copied a sequence at a time under the scoring of the sequences "
                        "already on the device, the kept V rows read over the host link by select + gather, "
                        "decode inputs and outputs crossing during the decode steps"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_next_rows and world == 1:  # per-GPU kernel timings; the scaling runs skip them
        res["next_rows"] = {"voxzip_pool": measure_voxzip(args, rank, world, dev, stream, flush),
                            "wnw_chunks_recall": measure_wnw(args, rank, world, dev, stream, flush)}
        try:  # the newest row: a failure here is reported and leaves the line intact
            c3 = measure_c3(args, rank, world, dev, stream, flush, cfg, d_in)
        except Exception as exc:  # noqa: BLE001
            c3 = {"error": f"{type(exc).__name__}: {exc}"[:300], "build_ms": -1.0, "us_per_step": -1.0}
        # every rank takes the same collectives, failed or not
        c3["build_ms"] = max_over_ranks(c3["build_ms"], world, dev)
        c3["us_per_step"] = max_over_ranks(c3["us_per_step"], world, dev)
        if "error" not in c3:
            c3["gbs"] = c3["bytes_alg_per_step"] / (c3["us_per_step"] * 1e-6) / 1e9
            c3["frac"] = c3["gbs"] / c3["peak"]
        res["next_rows"]["c3_retrieval"] = c3
        try:
            res["next_rows"]["pooled_alloc_segmented_select"] = measure_variants(args, dev, stream, flush, cfg, comp,
                                                                                 d_in, shape, params)
        except Exception as exc:  # noqa: BLE001
            res["next_rows"]["pooled_alloc_segmented_select"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, bt, args.cpu_rows)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


# A GPU-side wait of about 1 ms before each timed region, outside its events:
# the host enqueues the region's launches meanwhile, so the events time the
# kernels and not the host's launch gaps.
SPACER_CYCLES = 2_000_000


# ------------------------------------------------------- next rows (VoxZip) --
VZ_SEQS, VZ_L, VZ_D = 8, 32768, 2048


def measure_voxzip(args, rank, world, dev, stream, flush):
    """kv_voxzip_pool on 8 sequences of 32768 audio feature rows (12.5 rows/s,
    about 44 min each), d = 2048, bf16, seeded ASR segments; the features are
    drawn on the device by a seeded generator. Timed with CUDA events per call,
    L2 flushed between calls."""
    import torch

    import kv_cache_compression_layer_b200 as kv
    from kv_cache_compression_layer_b200.replicas import max_over_ranks, replica_seed

    base = replica_seed(11, rank)
    segs = [synth.asr_segments(base + i, VZ_L) for i in range(VZ_SEQS)]
    seg_off = np.concatenate([[0], np.cumsum([len(a.conf) for a in segs])]).astype(np.int64)
    tbase = np.concatenate([[0], np.cumsum([int(a.n_text.sum()) for a in segs])]).astype(np.int64)
    raw = kv.pack_segments(np.concatenate([a.tau for a in segs]), np.concatenate([a.conf for a in segs]),
                           np.concatenate([a.n_text for a in segs]),
                           np.concatenate([a.text_row + tbase[i] for i, a in enumerate(segs)]))
    seg_dev = torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(base)
    rows = VZ_SEQS * VZ_L
    E_A = torch.randn(rows, VZ_D, generator=g, device=dev).to(torch.bfloat16)
    E_T = (0.02 * torch.randn(int(tbase[-1]), VZ_D, generator=g, device=dev)).to(torch.bfloat16)
    E_comp = torch.empty(rows, VZ_D, dtype=torch.bfloat16, device=dev)
    src = torch.empty(rows, 3, dtype=torch.int32, device=dev)
    out_len = torch.empty(VZ_SEQS, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    tt = [a.tau_total for a in segs]

    def call():
        kv.kv_voxzip_pool([VZ_L] * VZ_SEQS, tt, seg_off, VZ_D, kv.KV_BF16, seg_dev, E_A, E_T, E_T.shape[0], E_comp,
                          src, out_len, status, stream=stream)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    if status.item():
        raise RuntimeError(f"kv_voxzip_pool status {status.item():#x}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        torch.cuda._sleep(SPACER_CYCLES)
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    us = max_over_ranks(1e3 * sum(a.elapsed_time(b) for a, b in ev) / args.steps, world, dev)
    n_out = int(out_len.sum().item())
    s_h = src.cpu().numpy()
    lens = out_len.cpu().numpy()
    pooled = sum(int((s_h[i * VZ_L:i * VZ_L + lens[i], 2] >= 0).sum()) for i in range(VZ_SEQS))
    eb = 2
    # E_A read once, the text rows of the pooled groups read, E_comp written,
    # one 12-byte descriptor written by the plan and read by the pool kernel
    bytes_alg = rows * VZ_D * eb + pooled * VZ_D * eb + n_out * VZ_D * eb + 24 * n_out + len(raw)
    peak, kind = hbm_peak()
    gbs = bytes_alg / (us * 1e-6) / 1e9
    return {"workload": f"{VZ_SEQS} seq x {VZ_L} feature rows, d={VZ_D}, bf16, seeded ASR segments "
                        f"({int(seg_off[-1])} segments, {n_out} output rows)",
            "kernels": "vz_plan_kernel + vz_pool_kernel (kv_voxzip_pool)", "us_per_call": us,
            "rows_per_s": world * rows / (us * 1e-6), "bytes_alg": bytes_alg, "gbs": gbs, "peak": peak,
            "frac": gbs / peak, "peak_kind": kind + " (hbm_gbs copy)", "launches_per_call": 2}


# ---------------------------------------------------------- next rows (WnW) --
WNW_L, WNW_ANCHOR, WNW_TIDAL, WNW_D, WNW_STEPS = 32768, 5, 235, 128, 32


def measure_wnw(args, rank, world, dev, stream, flush):
    """kv_wnw_update + kv_wnw_recall over 32 decode steps of one 32768-row
    audio (about 44 min at 12.5 rows/s) with 5 anchor and 235 tidal KV rows
    (d = 128, bf16), 4 s / 2 s chunks, top 3, released after 3 steps. The
    tidal rows' full copy is pinned host memory; the recall reads it over the
    host link. Its peak is a plain pinned host-to-device copy measured here."""
    import torch

    import kv_cache_compression_layer_b200 as kv
    from kv_cache_compression_layer_b200.replicas import max_over_ranks, replica_seed

    p = kv.make_wnw_params()
    Ls = [WNW_L]
    seed = replica_seed(23, rank)
    att = synth.anchor_attention(seed, WNW_L, WNW_ANCHOR, args.warmup + WNW_STEPS)
    att_dev = torch.from_numpy(att).to(dev)
    # host copies (2 x 2 GB, pinned): a seeded 64 MB random block, tiled
    g = torch.Generator()
    g.manual_seed(seed)
    tile = 1 << 18
    base = torch.randn(2 * tile, WNW_D, generator=g).to(torch.bfloat16)
    K_h = torch.empty(WNW_TIDAL * WNW_L, WNW_D, dtype=torch.bfloat16, pin_memory=True)
    V_h = torch.empty(K_h.shape, dtype=torch.bfloat16, pin_memory=True)
    for i, r0 in enumerate(range(0, K_h.shape[0], tile)):
        n = min(tile, K_h.shape[0] - r0)
        K_h[r0:r0 + n] = base[(i % 2) * tile:(i % 2) * tile + n]
        V_h[r0:r0 + n] = base[((i + 1) % 2) * tile:((i + 1) % 2) * tile + n]
    S, cap = p.chunk_stride, p.top_c * (p.chunk_len // p.chunk_stride)
    K_g = torch.zeros(WNW_TIDAL * p.n_slots * S, WNW_D, dtype=torch.bfloat16, device=dev)
    V_g = torch.zeros_like(K_g)
    state = torch.empty(kv.kv_wnw_state_ints(Ls, p), dtype=torch.int32, device=dev)
    score = torch.empty(kv.kv_wnw_chunk_count(Ls, p), dtype=torch.float64, device=dev)
    fetch = torch.empty(1, cap, 2, dtype=torch.int32, device=dev)
    release = torch.empty_like(fetch)
    counts = torch.empty(1, 2, dtype=torch.int32, device=dev)
    kv.kv_wnw_init(Ls, p, state, stream=stream)
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for t in range(args.warmup):
        kv.kv_wnw_update(Ls, p, WNW_ANCHOR, att_dev[t], state, score, fetch, release, counts, stream=stream)
        kv.kv_wnw_recall(Ls, p, WNW_TIDAL, WNW_D, kv.KV_BF16, fetch, counts, K_h, V_h, K_g, V_g, stream=stream)
    torch.cuda.synchronize()
    ev = [(E(), E(), E()) for _ in range(WNW_STEPS)]
    fetched = 0
    for i in range(WNW_STEPS):
        t = args.warmup + i
        flush.fill_(i & 0xFF)
        torch.cuda._sleep(SPACER_CYCLES)
        ev[i][0].record(stream)
        kv.kv_wnw_update(Ls, p, WNW_ANCHOR, att_dev[t], state, score, fetch, release, counts, stream=stream)
        ev[i][1].record(stream)
        kv.kv_wnw_recall(Ls, p, WNW_TIDAL, WNW_D, kv.KV_BF16, fetch, counts, K_h, V_h, K_g, V_g, stream=stream)
        ev[i][2].record(stream)
        torch.cuda.synchronize()
        fetched += int(counts[0, 0].item())  # blocks recalled this step (read outside the events)
    upd_us = max_over_ranks(1e3 * sum(a.elapsed_time(b) for a, b, _ in ev) / WNW_STEPS, world, dev)
    rec_us = max_over_ranks(1e3 * sum(b.elapsed_time(c) for _, b, c in ev) / WNW_STEPS, world, dev)
    rec_bytes = fetched * WNW_TIDAL * 2 * S * WNW_D * 2 / WNW_STEPS  # per step, host read = HBM write
    # the host link's measured copy bandwidth: one 256 MB pinned host-to-device copy
    blob = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    dst = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    dst.copy_(blob, non_blocking=True)
    a, b = E(), E()
    a.record(stream)
    dst.copy_(blob, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize()
    h2d_gbs = (256 << 20) / (a.elapsed_time(b) * 1e-3) / 1e9
    rec_gbs = rec_bytes / (rec_us * 1e-6) / 1e9
    return {"workload": f"1 seq x {WNW_L} audio rows, {WNW_ANCHOR} anchor + {WNW_TIDAL} tidal KV rows, d={WNW_D}, "
                        f"bf16, chunks 4 s / 2 s at 12.5 rows/s, top 3, release after 3, {WNW_STEPS} steps",
            "kernels": "wnw_score_kernel + wnw_update_kernel (kv_wnw_update), wnw_recall_kernel (kv_wnw_recall)",
            "update_us_per_step": upd_us, "recall_us_per_step": rec_us, "recalled_blocks_per_step":
            fetched / WNW_STEPS, "recall_bytes_per_step": rec_bytes, "recall_gbs": rec_gbs,
            "h2d_copy_gbs_measured": h2d_gbs, "recall_frac_of_h2d_copy": rec_gbs / h2d_gbs,
            "launches_per_step": 3}


# ------------------------------------------- next rows (step 3 and 4 variants) --
VARIANT_SEGMENTS = 32


def measure_variants(args, dev, stream, flush, cfg, comp, d_in, shape, params):
    """kv_allocate_global over the main workload's head scores, then
    kv_select_gather_segmented (32 segments a row) on the smoothed scores the
    timed steps left in the Compressor, into buffers of their own. N = 1."""
    import torch

    import kv_cache_compression_layer_b200 as kv

    rows, d = cfg.rows, cfg.head_dim
    total = kv.kv_total_slots(shape, cfg.L, params)
    b = torch.empty(rows, dtype=torch.int32, device=dev)
    off = torch.empty(rows + 1, dtype=torch.int64, device=dev)
    idx = torch.empty(total, dtype=torch.int32, device=dev)
    Kc = torch.empty(total, d, dtype=d_in["K"].dtype, device=dev)
    Vc = torch.empty_like(Kc)
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def once():
        kv.kv_allocate_global(shape, cfg.L, params, d_in["S"], b, off, stream=stream)
        kv.kv_select_gather_segmented(shape, cfg.L, comp.s_hat, d_in["K"], d_in["V"], b, off, VARIANT_SEGMENTS, idx,
                                      Kc, Vc, stream=stream)

    for _ in range(args.warmup):
        once()
    torch.cuda.synchronize()
    ev = [(E(), E(), E()) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        torch.cuda._sleep(SPACER_CYCLES)
        ev[i][0].record(stream)
        kv.kv_allocate_global(shape, cfg.L, params, d_in["S"], b, off, stream=stream)
        ev[i][1].record(stream)
        kv.kv_select_gather_segmented(shape, cfg.L, comp.s_hat, d_in["K"], d_in["V"], b, off, VARIANT_SEGMENTS, idx,
                                      Kc, Vc, stream=stream)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    alloc_us = 1e3 * sum(a.elapsed_time(x) for a, x, _ in ev) / args.steps
    sel_us = 1e3 * sum(x.elapsed_time(c) for _, x, c in ev) / args.steps
    bb = b.cpu().numpy().astype(np.int64)
    eb = Kc.element_size()
    L_rows = np.array([cfg.L[cfg.row_triplet(r)[0]] for r in range(rows)], np.int64)
    # smoothed scores read, indices written, kept K and V read and written compacted
    sel_bytes = int((4 * L_rows + 4 * bb + 4 * d * eb * bb).sum())
    peak, kind = hbm_peak()
    gbs = sel_bytes / (sel_us * 1e-6) / 1e9
    return {"workload": f"{cfg.name}: {rows} rows, L={list(cfg.L)}, d={d}, {cfg.dtype}, one budget over the "
                        f"{cfg.n_layers * cfg.n_kv_heads} heads of a sequence, {VARIANT_SEGMENTS} segments a row",
            "kernels": "allocate_kernel + slot_offsets_kernel (kv_allocate_global); select_kernel + gather_kernel "
                       "(kv_select_gather_segmented)",
            "allocate_us": alloc_us, "select_gather_us": sel_us, "select_gather_bytes_alg": sel_bytes,
            "select_gather_gbs": gbs, "peak": peak, "select_gather_frac": gbs / peak,
            "peak_kind": kind + " (hbm_gbs copy)", "launches_per_call": 4}


# ----------------------------------------------------------- next rows (C3) --
C3_BUDGET, C3_STEPS = 256, 32


def measure_c3(args, rank, world, dev, stream, flush, cfg, d_in):
    """kv_c3_build over the K of the main workload's longest sequence (every
    layer and KV head of it), then kv_c3_step for 32 decode steps with its
    decode queries: budget 256 keys, granularity 16, lambda 0.5, R = 2. The
    build synchronises once per tree level, so its time includes those host
    round trips."""
    import torch

    import kv_cache_compression_layer_b200 as kv

    bf = cfg.dtype == "bf16"
    shape = kv.make_shape(cfg.n_layers, cfg.n_kv_heads, cfg.group, cfg.head_dim, 1, kv.KV_BF16 if bf else kv.KV_F32)
    seq = int(np.argmax(cfg.L))
    rps = cfg.n_layers * cfg.n_kv_heads
    r0, r1 = seq * rps, (seq + 1) * rps
    k0 = sum(rps * cfg.L[s] for s in range(seq))
    Ls = [cfg.L[seq]]
    K = d_in["K"][k0:k0 + rps * Ls[0]]
    V = d_in["V"][k0:k0 + rps * Ls[0]]
    Q = d_in["q"][:, r0:r1]
    p = kv.make_c3_params(C3_BUDGET)
    lay = kv.kv_c3_index_layout(shape, Ls, p)
    index = torch.empty(lay.bytes, dtype=torch.uint8, device=dev)
    out = torch.empty(rps, cfg.group, cfg.head_dim, dtype=d_in["q"].dtype, device=dev)
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    torch.cuda.synchronize()
    b0, b1 = E(), E()
    b0.record(stream)
    kv.kv_c3_build(shape, Ls, p, K, index, stream=stream)
    b1.record(stream)
    torch.cuda.synchronize()
    build_ms = b0.elapsed_time(b1)
    D = Q.shape[0]
    for t in range(args.warmup):
        kv.kv_c3_step(shape, Ls, p, K, V, Q[t % D].contiguous(), index, out, stream=stream)
    torch.cuda.synchronize()
    ev = [(E(), E()) for _ in range(C3_STEPS)]
    qs = [Q[(args.warmup + i) % D].contiguous() for i in range(C3_STEPS)]
    for i in range(C3_STEPS):
        flush.fill_(i & 0xFF)
        torch.cuda._sleep(SPACER_CYCLES)
        ev[i][0].record(stream)
        kv.kv_c3_step(shape, Ls, p, K, V, qs[i], index, out, stream=stream)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    us = 1e3 * sum(a.elapsed_time(b) for a, b in ev) / C3_STEPS  # this rank's; the caller takes the max
    hdr = index[lay.hdr:lay.hdr + 16 * rps].view(torch.int32).view(rps, 4).cpu().numpy()
    eb = 2 if bf else 4
    # per step: the frontier's float64 centroids read, the retrieved K and V rows read, the queries and outputs
    A = int(hdr[:, 1].sum())
    kept = int(hdr[:, 2].sum())
    bytes_alg = A * cfg.head_dim * 8 + kept * 2 * cfg.head_dim * eb + 2 * rps * cfg.group * cfg.head_dim * eb
    peak, kind = hbm_peak()
    gbs = bytes_alg / (us * 1e-6) / 1e9
    return {"workload": f"{cfg.name}, sequence {seq}: {rps} rows, L={Ls[0]}, d={cfg.head_dim}, g={cfg.group}, {cfg.dtype}, "
                        f"budget {C3_BUDGET} keys, granularity 16, lambda 0.5, R 2, {C3_STEPS} steps "
                        f"(frontier {A} clusters)",
            "kernels": "c3_plan/split/centroid/frontier (kv_c3_build); c3_score, c3_select, c3_attn, c3_update "
                       "(kv_c3_step)",
            "build_ms": build_ms, "us_per_step": us, "bytes_alg_per_step": bytes_alg, "gbs": gbs, "peak": peak,
            "frac": gbs / peak, "peak_kind": kind + " (hbm_gbs copy)", "launches_per_step": 4}


# ------------------------------------------------------------ reference arm --
def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: every step runs the whole path on
    the same bounded sample of the workload's rows (all host threads); the
    line reports the time it measured for that sample."""
    if rank != 0:
        return
    import oracle as orc

    orc.build()
    cfg = workload(args)
    rows = sample_rows(cfg, args.ref_rows)
    bt = synth.make_batch(cfg)
    threads = orc.default_threads()
    for _ in range(args.warmup):
        oracle_sample(cfg, bt, rows, threads)
    secs = [oracle_sample(cfg, bt, rows, threads) for _ in range(args.steps)]
    step_s = sum(secs) / len(secs)
    value = sample_tokens(cfg, rows) / step_s
    sample = (f"{len(rows)} of {cfg.rows} rows per step through the whole path incl. {cfg.decode_steps} decode "
              f"steps; value = the sample's share of the batch's audio tokens / the measured step time")
    res = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded AR(1) keys, diagonal-band queries; stands in for long-audio workloads)",
           "config": config_dict(cfg, world),
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(threads, len(rows)), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="ragged", choices=sorted(synth.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=0,
                    help="layers per sequence (default: the workload's); a reduced case for profiler captures")
    ap.add_argument("--cpu-rows", type=int, default=64,
                    help="rows of the oracle sample for cpu_baseline, spread over the batch")
    ap.add_argument("--ref-rows", type=int, default=64,
                    help="rows per step of the reference (oracle) arm, spread over the batch")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true", help="skip the timing of the rows beyond the path")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
