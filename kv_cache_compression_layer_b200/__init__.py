"""Python binding of libkvcomp.so (the C ABI declared in include/kvcomp.h and
include/kvcomp_next.h).

Argument marshalling only: every step of the path runs in the library's
sm_100a kernels. Functions take torch tensors (or raw device addresses as
ints) and the current CUDA stream, and raise ``KvError`` on a non-zero
status. The library must be built (``python -m
kv_cache_compression_layer_b200.build``); importing the binding without it
fails loudly, there is no fallback. With KV_DEBUG_CHECKS=1 in the
environment the binding loads the debug build, libkvcomp_debug.so (built by
``python -m kv_cache_compression_layer_b200.build --debug``), whose kernels
check their data-dependent indices (see kv_debug_check_word).
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG_CHECKS = os.environ.get("KV_DEBUG_CHECKS", "0") not in ("", "0")
LIB_PATH = os.path.join(HERE, "libkvcomp_debug.so" if DEBUG_CHECKS else "libkvcomp.so")

KV_OK, KV_ERR_ARG, KV_ERR_UNSUPPORTED_L, KV_ERR_BUDGET, KV_ERR_WORKSPACE, KV_ERR_CUDA, KV_ERR_TIMEOUT = range(7)
KV_DEV_TIMEOUT, KV_DEV_BUDGET, KV_DEV_CAPACITY, KV_DEV_RANGE, KV_DEV_BOUNDS = 0x1, 0x2, 0x4, 0x8, 0x10
KV_F32, KV_BF16 = 0, 1
KV_MAX_SEQ = 64
META_INTS = 8

# Every symbol the headers under include/ declare.
EXPORTS = ("kv_rows", "kv_check_lengths", "kv_workspace_bytes", "kv_total_slots", "kv_score", "kv_sss",
           "kv_allocate", "kv_select_gather", "kv_decode_init", "kv_decode_attn_update", "kv_read_device_status",
           "kv_status_string", "kv_score_noalloc", "kv_decode_scratch_bytes", "kv_allocate_global",
           "kv_select_gather_segmented", "kv_voxzip_pool", "kv_wnw_chunk_count", "kv_wnw_state_ints",
           "kv_wnw_init", "kv_wnw_update", "kv_wnw_recall", "kv_c3_index_layout", "kv_c3_build", "kv_c3_step",
           "kv_set_wait_limit_ns", "kv_score_noalloc_status", "kv_debug_checks", "kv_debug_check_word")
KV_NOALLOC_SCRATCH_BYTES = 8 << 20


class kv_shape(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("n_kv_heads", C.c_int32), ("group", C.c_int32), ("head_dim", C.c_int32),
                ("w", C.c_int32), ("dtype", C.c_int32)]


class kv_wnw_params(C.Structure):
    _fields_ = [("chunk_len", C.c_int32), ("chunk_stride", C.c_int32), ("top_c", C.c_int32),
                ("release_after", C.c_int32), ("n_slots", C.c_int32)]


class kv_c3_params(C.Structure):
    _fields_ = [("leaf_max", C.c_int32), ("iters", C.c_int32), ("granularity", C.c_int32), ("budget", C.c_int32),
                ("lam", C.c_double), ("exchanges", C.c_int32), ("reserved", C.c_int32), ("seed", C.c_uint64)]


class kv_c3_layout(C.Structure):
    _fields_ = [(n, C.c_uint64) for n in ("perm", "lo", "cnt", "left", "depth", "e", "cent", "front", "sigma", "sel",
                                          "hdr", "bytes")]


class kv_params(C.Structure):
    _fields_ = [("budget_pct", C.c_int32), ("alpha", C.c_float), ("rho", C.c_float), ("r", C.c_float),
                ("gamma", C.c_float), ("sinks_T", C.c_int32), ("recent_pct", C.c_int32)]


class kv_cache(C.Structure):
    _fields_ = [("Kc", C.c_void_p), ("Vc", C.c_void_p), ("A", C.c_void_p), ("pos", C.c_void_p),
                ("slot_off", C.c_void_p), ("b", C.c_void_p), ("meta", C.c_void_p), ("status", C.c_void_p),
                ("total_slots", C.c_int64), ("scratch", C.c_void_p), ("scratch_bytes", C.c_size_t)]


class KvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


_lib = None


def lib():
    """The loaded libkvcomp.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            flag = " --debug" if DEBUG_CHECKS else ""
            raise ImportError(f"{LIB_PATH} is missing: build it with python -m kv_cache_compression_layer_b200.build{flag}")
        L = C.CDLL(LIB_PATH)
        P, I32, SZ, I64 = C.c_void_p, C.c_int32, C.c_size_t, C.c_int64
        Ps, Pp, Pc = C.POINTER(kv_shape), C.POINTER(kv_params), C.POINTER(kv_cache)
        Pw = C.POINTER(kv_wnw_params)
        Pc3, Pl3 = C.POINTER(kv_c3_params), C.POINTER(kv_c3_layout)
        sig = {
            "kv_rows": (I64, [Ps, I32]),
            "kv_check_lengths": (C.c_int, [Ps, P, I32]),
            "kv_workspace_bytes": (SZ, [Ps, P, I32]),
            "kv_total_slots": (I64, [Ps, P, I32, Pp]),
            "kv_score": (C.c_int, [Ps, P, I32, P, P, P, P, SZ, P]),
            "kv_sss": (C.c_int, [Ps, P, I32, P, P, P, C.c_float, C.c_float, P]),
            "kv_allocate": (C.c_int, [Ps, P, I32, Pp, P, P, P, P]),
            "kv_select_gather": (C.c_int, [Ps, P, I32, P, P, P, P, P, P, P, P, P]),
            "kv_allocate_global": (C.c_int, [Ps, P, I32, Pp, P, P, P, P]),
            "kv_select_gather_segmented": (C.c_int, [Ps, P, I32, P, P, P, P, P, I32, P, P, P, P]),
            "kv_decode_init": (C.c_int, [Ps, P, I32, Pp, Pc, P]),
            "kv_decode_attn_update": (C.c_int, [Ps, P, I32, Pp, Pc, P, P, P, P, P]),
            "kv_read_device_status": (C.c_int, [P, P, P]),
            "kv_status_string": (C.c_char_p, [C.c_int]),
            "kv_score_noalloc": (C.c_int, [Ps, P, I32, P, P, P, P]),
            "kv_score_noalloc_status": (C.c_int, [P, P]),
            "kv_set_wait_limit_ns": (C.c_uint64, [C.c_uint64]),
            "kv_debug_checks": (C.c_int, []),
            "kv_debug_check_word": (C.c_int, [P, I32]),
            "kv_decode_scratch_bytes": (SZ, [Ps, P, I32, Pp, I64]),
            "kv_voxzip_pool": (C.c_int, [P, I32, P, P, I32, I32, C.c_float, P, P, P, I64, P, P, P, P, P]),
            "kv_wnw_chunk_count": (I64, [P, I32, Pw]),
            "kv_wnw_state_ints": (I64, [P, I32, Pw]),
            "kv_wnw_init": (C.c_int, [P, I32, Pw, P, P]),
            "kv_wnw_update": (C.c_int, [P, I32, Pw, I32, P, P, P, P, P, P, P]),
            "kv_wnw_recall": (C.c_int, [P, I32, Pw, I32, I32, I32, P, P, P, P, P, P, P]),
            "kv_c3_index_layout": (C.c_int, [Ps, P, I32, Pc3, Pl3]),
            "kv_c3_build": (C.c_int, [Ps, P, I32, Pc3, P, P, P]),
            "kv_c3_step": (C.c_int, [Ps, P, I32, Pc3, P, P, P, P, P, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(st: int) -> str:
    return lib().kv_status_string(st).decode()


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _L(L: Sequence[int]):
    arr = (C.c_int32 * len(L))(*[int(x) for x in L])
    return arr, len(L)


def _check(fn: str, st: int):
    if st != KV_OK:
        raise KvError(fn, st)


def make_shape(n_layers: int, n_kv_heads: int, group: int, head_dim: int, w: int, dtype: int) -> kv_shape:
    return kv_shape(n_layers, n_kv_heads, group, head_dim, w, dtype)


def make_params(budget_pct: int, alpha: float, rho: float, r: float, gamma: float, sinks_T: int,
                recent_pct: int) -> kv_params:
    return kv_params(budget_pct, alpha, rho, r, gamma, sinks_T, recent_pct)


def kv_rows(shape: kv_shape, n_seq: int) -> int:
    return lib().kv_rows(C.byref(shape), n_seq)


def kv_check_lengths(shape: kv_shape, L: Sequence[int]) -> int:
    arr, n = _L(L)
    return lib().kv_check_lengths(C.byref(shape), arr, n)


def kv_workspace_bytes(shape: kv_shape, L: Sequence[int]) -> int:
    arr, n = _L(L)
    return lib().kv_workspace_bytes(C.byref(shape), arr, n)


def kv_total_slots(shape: kv_shape, L: Sequence[int], params: kv_params) -> int:
    arr, n = _L(L)
    return lib().kv_total_slots(C.byref(shape), arr, n, C.byref(params))


def kv_score(shape, L, qwin, K, s, ws, ws_bytes: Optional[int] = None, stream=None):
    arr, n = _L(L)
    nbytes = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    _check("kv_score", lib().kv_score(C.byref(shape), arr, n, _ptr(qwin), _ptr(K), _ptr(s), _ptr(ws), nbytes,
                                      _stream(stream)))


def kv_score_noalloc(shape, L, qwin, K, s, stream=None):
    """kv_score without a workspace: the library's own fixed scratch array is used
    (for callers that cannot allocate device memory; see include/kvcomp.h)."""
    arr, n = _L(L)
    _check("kv_score_noalloc", lib().kv_score_noalloc(C.byref(shape), arr, n, _ptr(qwin), _ptr(K), _ptr(s),
                                                      _stream(stream)))


def kv_score_noalloc_status(stream=None) -> int:
    """The device status word of the last kv_score_noalloc call on the current device."""
    host = C.c_int32(0)
    _check("kv_score_noalloc_status", lib().kv_score_noalloc_status(C.byref(host), _stream(stream)))
    return host.value


def kv_set_wait_limit_ns(limit_ns: int) -> int:
    """Sets the limit of the library's bounded device waits for later launches; returns the previous one."""
    return int(lib().kv_set_wait_limit_ns(int(limit_ns)))


DEFAULT_WAIT_LIMIT_NS = 2_000_000_000


def kv_sss(shape, L, s, s_hat, kstar, alpha: float, rho: float, stream=None):
    arr, n = _L(L)
    _check("kv_sss", lib().kv_sss(C.byref(shape), arr, n, _ptr(s), _ptr(s_hat), _ptr(kstar), alpha, rho,
                                  _stream(stream)))


def kv_allocate(shape, L, params, S, b, slot_off, stream=None):
    arr, n = _L(L)
    _check("kv_allocate", lib().kv_allocate(C.byref(shape), arr, n, C.byref(params), _ptr(S), _ptr(b),
                                            _ptr(slot_off), _stream(stream)))


def kv_select_gather(shape, L, s_hat, K, V, b, slot_off, idx, Kc, Vc, stream=None):
    arr, n = _L(L)
    _check("kv_select_gather", lib().kv_select_gather(C.byref(shape), arr, n, _ptr(s_hat), _ptr(K), _ptr(V),
                                                      _ptr(b), _ptr(slot_off), _ptr(idx), _ptr(Kc), _ptr(Vc),
                                                      _stream(stream)))


def kv_allocate_global(shape, L, params, S, b, slot_off, stream=None):
    arr, n = _L(L)
    _check("kv_allocate_global", lib().kv_allocate_global(C.byref(shape), arr, n, C.byref(params), _ptr(S), _ptr(b),
                                                          _ptr(slot_off), _stream(stream)))


def kv_select_gather_segmented(shape, L, s_hat, K, V, b, slot_off, n_segments, idx, Kc, Vc, stream=None):
    arr, n = _L(L)
    _check("kv_select_gather_segmented",
           lib().kv_select_gather_segmented(C.byref(shape), arr, n, _ptr(s_hat), _ptr(K), _ptr(V), _ptr(b),
                                            _ptr(slot_off), int(n_segments), _ptr(idx), _ptr(Kc), _ptr(Vc),
                                            _stream(stream)))


def make_cache(Kc, Vc, A, pos, slot_off, b, meta, status, scratch=None, total_slots: Optional[int] = None,
               scratch_bytes: Optional[int] = None) -> kv_cache:
    if total_slots is None:
        total_slots = Kc.shape[0] if hasattr(Kc, "shape") else 0
    if scratch_bytes is None:
        scratch_bytes = scratch.numel() * scratch.element_size() if scratch is not None else 0
    return kv_cache(_ptr(Kc), _ptr(Vc), _ptr(A), _ptr(pos), _ptr(slot_off), _ptr(b), _ptr(meta), _ptr(status),
                    int(total_slots), _ptr(scratch), int(scratch_bytes))


def kv_decode_scratch_bytes(shape: kv_shape, L: Sequence[int], params: kv_params, total_slots: int) -> int:
    arr, n = _L(L)
    return lib().kv_decode_scratch_bytes(C.byref(shape), arr, n, C.byref(params), int(total_slots))


def kv_decode_init(shape, L, params, cache: kv_cache, stream=None):
    arr, n = _L(L)
    _check("kv_decode_init", lib().kv_decode_init(C.byref(shape), arr, n, C.byref(params), C.byref(cache),
                                                  _stream(stream)))


def kv_decode_attn_update(shape, L, params, cache: kv_cache, q_t, k_t, v_t, out, stream=None):
    arr, n = _L(L)
    _check("kv_decode_attn_update",
           lib().kv_decode_attn_update(C.byref(shape), arr, n, C.byref(params), C.byref(cache), _ptr(q_t),
                                       _ptr(k_t), _ptr(v_t), _ptr(out), _stream(stream)))


# kv_asr_segment (include/kvcomp_next.h), 32 bytes
ASR_SEGMENT_BYTES = 32


def pack_segments(tau, conf, n_text, text_row) -> bytes:
    """Packs per-segment arrays into kv_asr_segment records (little-endian)."""
    import struct

    out = bytearray()
    for (t0, t1), c, n, r in zip(tau, conf, n_text, text_row):
        out += struct.pack("<ddfiii", float(t0), float(t1), float(c), int(n), int(r), 0)
    return bytes(out)


def kv_voxzip_pool(L_a, tau_total, seg_off, d, dtype, segs, E_A, E_T, n_text_rows, E_comp, src, out_len, status=None,
                   conf_min: float = 0.3, stream=None):
    n = len(L_a)
    La = (C.c_int32 * n)(*[int(x) for x in L_a])
    tt = (C.c_double * n)(*[float(x) for x in tau_total])
    so = (C.c_int32 * (n + 1))(*[int(x) for x in seg_off])
    _check("kv_voxzip_pool",
           lib().kv_voxzip_pool(La, n, tt, so, int(d), int(dtype), C.c_float(conf_min), _ptr(segs), _ptr(E_A),
                                _ptr(E_T), int(n_text_rows), _ptr(E_comp), _ptr(src), _ptr(out_len), _ptr(status),
                                _stream(stream)))


def make_wnw_params(chunk_len: int = 50, chunk_stride: int = 25, top_c: int = 3, release_after: int = 3,
                    n_slots: Optional[int] = None) -> kv_wnw_params:
    """WnW's chunk rule in audio rows (defaults: 4 s / 2 s at 12.5 rows/s, top 3, 3 steps);
    n_slots defaults to the bound top_c * release_after * chunk_len / chunk_stride."""
    if n_slots is None:
        n_slots = top_c * release_after * (chunk_len // max(1, chunk_stride))
    return kv_wnw_params(chunk_len, chunk_stride, top_c, release_after, n_slots)


def kv_wnw_chunk_count(L, p: kv_wnw_params) -> int:
    arr, n = _L(L)
    return lib().kv_wnw_chunk_count(arr, n, C.byref(p))


def kv_wnw_state_ints(L, p: kv_wnw_params) -> int:
    arr, n = _L(L)
    return lib().kv_wnw_state_ints(arr, n, C.byref(p))


def kv_wnw_init(L, p, state, stream=None):
    arr, n = _L(L)
    _check("kv_wnw_init", lib().kv_wnw_init(arr, n, C.byref(p), _ptr(state), _stream(stream)))


def kv_wnw_update(L, p, n_anchor, s, state, score, fetch, release, counts, stream=None):
    arr, n = _L(L)
    _check("kv_wnw_update", lib().kv_wnw_update(arr, n, C.byref(p), int(n_anchor), _ptr(s), _ptr(state), _ptr(score),
                                                _ptr(fetch), _ptr(release), _ptr(counts), _stream(stream)))


def kv_wnw_recall(L, p, n_tidal, d, dtype, fetch, counts, K_host, V_host, K_gpu, V_gpu, stream=None):
    arr, n = _L(L)
    _check("kv_wnw_recall", lib().kv_wnw_recall(arr, n, C.byref(p), int(n_tidal), int(d), int(dtype), _ptr(fetch),
                                                _ptr(counts), _ptr(K_host), _ptr(V_host), _ptr(K_gpu), _ptr(V_gpu),
                                                _stream(stream)))


def make_c3_params(budget: int, leaf_max: int = 4, iters: int = 8, granularity: int = 16, lam: float = 0.5,
                   exchanges: int = 2, seed: int = 0) -> kv_c3_params:
    """C3's settings (defaults as on the C3 page: 8 iterations, seed 0, granularity 16, lambda 0.5, R 2)."""
    return kv_c3_params(leaf_max, iters, granularity, budget, lam, exchanges, 0, seed)


def kv_c3_index_layout(shape, L, p) -> kv_c3_layout:
    arr, n = _L(L)
    out = kv_c3_layout()
    _check("kv_c3_index_layout", lib().kv_c3_index_layout(C.byref(shape), arr, n, C.byref(p), C.byref(out)))
    return out


def kv_c3_build(shape, L, p, K, index, stream=None):
    arr, n = _L(L)
    _check("kv_c3_build", lib().kv_c3_build(C.byref(shape), arr, n, C.byref(p), _ptr(K), _ptr(index),
                                            _stream(stream)))


def kv_c3_step(shape, L, p, K, V, q, index, out, stream=None):
    arr, n = _L(L)
    _check("kv_c3_step", lib().kv_c3_step(C.byref(shape), arr, n, C.byref(p), _ptr(K), _ptr(V), _ptr(q),
                                          _ptr(index), _ptr(out), _stream(stream)))


def kv_read_device_status(status_dev, stream=None) -> int:
    host = C.c_int32(0)
    _check("kv_read_device_status", lib().kv_read_device_status(_ptr(status_dev), C.byref(host), _stream(stream)))
    return host.value


def kv_debug_checks() -> bool:
    """True when the loaded library is the debug build (index checks compiled in)."""
    return bool(lib().kv_debug_checks())


def kv_debug_check_word(clear: bool = False) -> int:
    """The debug build's check word (KV_DEV_BOUNDS or 0; 0 in a release build),
    read after all earlier work on the current device; clear resets it."""
    host = C.c_int32(0)
    _check("kv_debug_check_word", lib().kv_debug_check_word(C.byref(host), 1 if clear else 0))
    return host.value


from .pipeline import Compressor  # noqa: E402  (the torch-side convenience wrapper)

__all__ = ["kv_shape", "kv_params", "kv_cache", "KvError", "lib", "make_shape", "make_params", "make_cache",
           "kv_rows", "kv_check_lengths", "kv_workspace_bytes", "kv_total_slots", "kv_score", "kv_score_noalloc",
           "kv_score_noalloc_status", "kv_set_wait_limit_ns", "DEFAULT_WAIT_LIMIT_NS", "kv_sss",
           "kv_debug_checks", "kv_debug_check_word",
           "kv_allocate", "kv_select_gather", "kv_decode_init", "kv_decode_attn_update", "kv_read_device_status",
           "kv_decode_scratch_bytes", "kv_allocate_global", "kv_select_gather_segmented", "kv_voxzip_pool",
           "pack_segments", "ASR_SEGMENT_BYTES", "kv_wnw_params", "make_wnw_params", "kv_wnw_chunk_count",
           "kv_wnw_state_ints", "kv_wnw_init", "kv_wnw_update", "kv_wnw_recall", "kv_c3_params", "kv_c3_layout",
           "make_c3_params", "kv_c3_index_layout", "kv_c3_build", "kv_c3_step", "status_string",
           "Compressor", "EXPORTS", "KV_F32", "KV_BF16", "META_INTS"]
