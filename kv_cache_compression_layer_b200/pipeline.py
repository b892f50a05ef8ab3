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

    # -- decode ----------------------------------------------------------------
    def decode_step(self, q_t, k_t, v_t, out, stream=None):
        kv_decode_attn_update(self.shape, self.L, self.params, self.cache, q_t, k_t, v_t, out, stream)

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
