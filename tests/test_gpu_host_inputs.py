"""The path with its inputs in pinned host memory (Compressor.compress_from_host,
Compressor.decode_from_host: copies overlapped with the work, V's kept rows read
over the host link by select + gather) gives bit for bit what the path gives with
device inputs: every row is an independent problem, so scoring and smoothing a
batch one sequence at a time changes no value. Also: kv_select_gather refuses V
in pageable host memory before any launch.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_layer_b200 as kv
import synth
from kv_cache_compression_layer_b200 import Compressor
from tests._harness import dev, params_of, shape_of

pytestmark = pytest.mark.gpu


def _inputs(cfg, bt):
    dt = torch.bfloat16
    host = {"qwin": torch.from_numpy(np.ascontiguousarray(bt.qwin)).to(dt),
            "K": torch.from_numpy(np.ascontiguousarray(bt.K)).to(dt),
            "V": torch.from_numpy(np.ascontiguousarray(bt.V)).to(dt),
            "S": torch.from_numpy(np.ascontiguousarray(bt.S)).to(torch.float32),
            "q": torch.from_numpy(np.ascontiguousarray(bt.q_dec)).to(dt),
            "k": torch.from_numpy(np.ascontiguousarray(bt.k_dec)).to(dt),
            "v": torch.from_numpy(np.ascontiguousarray(bt.v_dec)).to(dt)}
    if bt.spikes is not None:
        host["spikes"] = torch.from_numpy(np.where(bt.spikes, 10.0, 1.0)).to(torch.float32)
    return host


@pytest.mark.parametrize("cfg", [synth.small("ragged", n_layers=2, L=(1000, 3500, 2000)),
                                 synth.small("3b", n_layers=2, L=(2000,))], ids=["ragged3", "3b1"])
def test_host_inputs_match_device_inputs(cfg):
    steps = 6
    bt = synth.make_batch(cfg, steps=steps)
    host = _inputs(cfg, bt)
    d_in = {k: v.to(dev()) for k, v in host.items()}
    shape, params = shape_of(cfg), params_of(cfg)

    ref = Compressor(shape, cfg.L, params, device=dev())
    ref.compress(d_in["qwin"], d_in["K"], d_in["V"], d_in["S"], spikes=d_in.get("spikes"))
    out_ref = torch.empty(steps, cfg.rows, cfg.group, cfg.head_dim, dtype=torch.bfloat16, device=dev())
    for t in range(steps):
        ref.decode_step(d_in["q"][t], d_in["k"][t], d_in["v"][t], out_ref[t])
    torch.cuda.synchronize()

    pinned = {k: v.pin_memory() for k, v in host.items()}
    bufs = {k: torch.full_like(v, float("nan")) for k, v in d_in.items() if k != "V"}
    got = Compressor(shape, cfg.L, params, device=dev())
    out = torch.full_like(out_ref, float("nan"))
    out_host = torch.empty(out_ref.shape, dtype=torch.bfloat16).pin_memory()
    copied = got.compress_from_host(pinned, bufs)
    assert copied == sum(pinned[k].numel() * pinned[k].element_size() for k in ("qwin", "K", "S", "spikes")
                         if k in pinned)
    got.decode_from_host(pinned["q"], pinned["k"], pinned["v"], out_host, bufs["q"], bufs["k"], bufs["v"], out)
    torch.cuda.synchronize()

    for name in ("s", "s_hat", "kstar", "b", "slot_off", "pos", "Kc", "Vc", "A", "meta"):
        a, b = getattr(ref, name), getattr(got, name)
        assert torch.equal(a.view(torch.uint8) if a.is_floating_point() else a,
                           b.view(torch.uint8) if b.is_floating_point() else b), name
    assert torch.equal(out_ref.view(torch.int16).cpu(), out_host.view(torch.int16))
    assert kv.kv_read_device_status(got.status) == 0


def test_select_gather_refuses_pageable_host_v():
    cfg = synth.small("3b", n_layers=1, L=(600,))
    bt = synth.make_batch(cfg, steps=1)
    host = _inputs(cfg, bt)
    d_in = {k: v.to(dev()) for k, v in host.items()}
    comp = Compressor(shape_of(cfg), cfg.L, params_of(cfg), device=dev())
    comp.allocate(d_in["S"])
    comp.score(d_in["qwin"], d_in["K"])
    comp.sss()
    pageable_v = host["V"].clone()  # not page-locked
    assert not pageable_v.is_pinned()
    with pytest.raises(kv.KvError):
        comp.select_gather(d_in["K"], pageable_v)
    comp.select_gather(d_in["K"], host["V"].pin_memory())  # pinned: accepted
    torch.cuda.synchronize()
