"""Device buffers and call order of the whole path for one batch.

``Compressor`` owns the device memory (allocated through torch, the only use
of torch here besides streams) and calls the C-ABI entry points in the
path's order: allocate -> score -> SSS -> select + gather -> decode init,
then one ``kv_decode_attn_update`` per decode step.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import (KV_BF16, META_INTS, kv_allocate, kv_decode_attn_update, kv_decode_init, kv_decode_scratch_bytes,
               kv_params, kv_score, kv_select_gather, kv_shape, kv_sss, kv_total_slots, kv_workspace_bytes,
               make_cache)


def torch_dtype(dtype_code: int):
    return torch.bfloat16 if dtype_code == KV_BF16 else torch.float32


class Compressor:
    """All buffers of one batch (shape, audio lengths L per sequence, parameters)."""

    def __init__(self, shape: kv_shape, L: Sequence[int], params: kv_params, device="cuda"):
        self.shape, self.L, self.params = shape, [int(x) for x in L], params
        self.device = torch.device(device)
        H, nl, d = shape.n_kv_heads, shape.n_layers, shape.head_dim
        self.rows = len(self.L) * nl * H
        self.R = shape.group * shape.w
        self.L_rows = [l for l in self.L for _ in range(nl * H)]
        self.n_keys = sum(self.L_rows)
        self.n_slots = kv_total_slots(shape, self.L, params)
        if self.n_slots < 0:
            raise ValueError("invalid shape or parameters")
        dt = torch_dtype(shape.dtype)
        dev = self.device
        f32, i32 = torch.float32, torch.int32
        self.ws_bytes = kv_workspace_bytes(shape, self.L)
        self.ws = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)
        self.s = torch.empty(self.n_keys, dtype=f32, device=dev)
        self.s_hat = torch.empty(self.n_keys, dtype=f32, device=dev)
        self.kstar = torch.empty(self.rows, dtype=i32, device=dev)
        self.b = torch.empty(self.rows, dtype=i32, device=dev)
        self.slot_off = torch.empty(self.rows + 1, dtype=torch.int64, device=dev)
        self.pos = torch.zeros(self.n_slots, dtype=i32, device=dev)
        self.Kc = torch.zeros(self.n_slots, d, dtype=dt, device=dev)
        self.Vc = torch.zeros(self.n_slots, d, dtype=dt, device=dev)
        self.A = torch.zeros(self.n_slots, dtype=f32, device=dev)
        self.meta = torch.zeros(self.rows * META_INTS, dtype=i32, device=dev)
        self.status = torch.zeros(4, dtype=i32, device=dev)
        self.scratch = torch.empty(max(256, kv_decode_scratch_bytes(shape, self.L, params, self.n_slots)),
                                   dtype=torch.uint8, device=dev)
        self.cache = make_cache(self.Kc, self.Vc, self.A, self.pos, self.slot_off, self.b, self.meta, self.status,
                                self.scratch)

    # -- prefill compression -------------------------------------------------
    def allocate(self, S: torch.Tensor, stream=None):
        kv_allocate(self.shape, self.L, self.params, S, self.b, self.slot_off, stream)

    def score(self, qwin: torch.Tensor, K: torch.Tensor, stream=None):
        kv_score(self.shape, self.L, qwin, K, self.s, self.ws, self.ws_bytes, stream)

    def sss(self, stream=None):
        kv_sss(self.shape, self.L, self.s, self.s_hat, self.kstar, self.params.alpha, self.params.rho, stream)

    def select_gather(self, K: torch.Tensor, V: torch.Tensor, stream=None):
        kv_select_gather(self.shape, self.L, self.s_hat, K, V, self.b, self.slot_off, self.pos, self.Kc, self.Vc,
                         stream)

    def decode_init(self, stream=None):
        kv_decode_init(self.shape, self.L, self.params, self.cache, stream)

    def compress(self, qwin, K, V, S, spikes: Optional[torch.Tensor] = None, stream=None):
        """allocate -> score -> (harness spikes) -> SSS -> select + gather -> decode init."""
        self.allocate(S, stream)
        self.score(qwin, K, stream)
        if spikes is not None:
            self.s.mul_(spikes)
        self.sss(stream)
        self.select_gather(K, V, stream)
        self.decode_init(stream)

    def compress_from_host(self, host: dict, dev: dict, stream=None, copy_stream=None) -> int:
        """The same path with its inputs in pinned host memory, the copies overlapped with the work.

        ``host`` holds pinned CPU tensors qwin, K, V, S (and the harness's spikes); ``dev`` device
        buffers of the same shapes for qwin, K, S (and spikes). On ``copy_stream`` S and the window
        queries are copied first, then K one sequence at a time; on ``stream`` each sequence is
        scored and smoothed as soon as its keys have arrived (every row is an independent problem,
        so a sequence is a batch of its own for kv_score and kv_sss). V is not copied: select +
        gather reads the kept rows straight from the pinned host tensor over the host link (the
        path needs only those b rows of each row's L). Errors of the scoring calls are OR-ed into
        the batch's device status word (``self.status``). Returns the host bytes the device reads.
        """
        dev_ = self.device
        stream = stream if stream is not None else torch.cuda.current_stream(dev_)
        copy_stream = copy_stream if copy_stream is not None else torch.cuda.Stream(dev_)
        copy_stream.wait_stream(stream)  # the device buffers are no longer in use
        rps = self.shape.n_layers * self.shape.n_kv_heads
        spikes = "spikes" in host
        nbytes = 0

        def copy(name, lo=None, hi=None):
            nonlocal nbytes
            src = host[name] if lo is None else host[name][lo:hi]
            dst = dev[name] if lo is None else dev[name][lo:hi]
            dst.copy_(src, non_blocking=True)
            nbytes += src.numel() * src.element_size()

        with torch.cuda.stream(copy_stream):
            copy("S")
            copy("qwin")
        ev = torch.cuda.Event()
        ev.record(copy_stream)
        stream.wait_event(ev)
        self.allocate(dev["S"], stream)
        key0 = 0
        for sq, L in enumerate(self.L):
            key1 = key0 + rps * L
            with torch.cuda.stream(copy_stream):
                copy("K", key0, key1)
                if spikes:
                    copy("spikes", key0, key1)
            ev = torch.cuda.Event()
            ev.record(copy_stream)
            stream.wait_event(ev)
            r0, r1 = sq * rps, (sq + 1) * rps
            kv_score(self.shape, [L], dev["qwin"][r0:r1], dev["K"][key0:key1], self.s[key0:key1], self.ws,
                     self.ws_bytes, stream)
            with torch.cuda.stream(stream):
                # each kv_score call restarts its workspace status word: keep every call's in the batch's
                self.status[:1].bitwise_or_(self.ws[:4].view(torch.int32))
                if spikes:
                    self.s[key0:key1].mul_(dev["spikes"][key0:key1])
            kv_sss(self.shape, [L], self.s[key0:key1], self.s_hat[key0:key1], self.kstar[r0:r1], self.params.alpha,
                   self.params.rho, stream)
            key0 = key1
        self.select_gather(dev["K"], host["V"], stream)
        self.decode_init(stream)
        return nbytes

    # -- decode ----------------------------------------------------------------
    def decode_step(self, q_t, k_t, v_t, out, stream=None):
        kv_decode_attn_update(self.shape, self.L, self.params, self.cache, q_t, k_t, v_t, out, stream)

    def decode_from_host(self, q, k, v, out_host, dq, dk, dv, out, stream=None, copy_stream=None, d2h_stream=None):
        """Decode steps t = 0.. with their inputs q[t], k[t], v[t] in pinned host memory and each
        step's output read back into out_host[t]: the inputs go over the host link on ``copy_stream``
        (after the work already queued on ``stream``) and the outputs on ``d2h_stream``, both
        overlapped with the steps. dq, dk, dv, out: device buffers shaped like q, k, v, out_host."""
        dev_ = self.device
        stream = stream if stream is not None else torch.cuda.current_stream(dev_)
        copy_stream = copy_stream if copy_stream is not None else torch.cuda.Stream(dev_)
        d2h_stream = d2h_stream if d2h_stream is not None else torch.cuda.Stream(dev_)
        copy_stream.wait_stream(stream)
        d2h_stream.wait_stream(stream)
        ev_in = []
        with torch.cuda.stream(copy_stream):
            for t in range(q.shape[0]):
                dq[t].copy_(q[t], non_blocking=True)
                dk[t].copy_(k[t], non_blocking=True)
                dv[t].copy_(v[t], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_stream)
                ev_in.append(ev)
        for t in range(q.shape[0]):
            stream.wait_event(ev_in[t])
            self.decode_step(dq[t], dk[t], dv[t], out[t], stream)
            ev = torch.cuda.Event()
            ev.record(stream)
            d2h_stream.wait_event(ev)
            with torch.cuda.stream(d2h_stream):
                out_host[t].copy_(out[t], non_blocking=True)
        stream.wait_stream(d2h_stream)  # the caller's later work on stream sees every output on the host

    # -- host views for checks -------------------------------------------------
    def kept(self):
        """Per row (b, kept positions, compacted K, compacted V) on the host."""
        b = self.b.cpu().tolist()
        off = self.slot_off.cpu().tolist()
        pos = self.pos.cpu()
        Kc = self.Kc.float().cpu()
        Vc = self.Vc.float().cpu()
        out = []
        for i in range(self.rows):
            o = off[i]
            out.append((b[i], pos[o:o + b[i]].numpy(), Kc[o:o + b[i]].numpy(), Vc[o:o + b[i]].numpy()))
        return out
