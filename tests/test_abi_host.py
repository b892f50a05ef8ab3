"""The C ABI without a GPU: the library loads, exports every symbol the
header declares, and its host-side checks (sizes, argument errors, fault
injection) behave as documented. No call here reaches a kernel."""
import ctypes as C
import os
import re

import pytest

import kv_cache_compression_layer_b200 as kv
from kv_cache_compression_layer_b200 import build as kvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kvbuild.build()
    return kv.lib()


def _declared():
    import glob

    hdr = "".join(open(f).read() for f in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))))
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(kv_\w+)\s*\(", hdr, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert "kv_score" in names and "kv_decode_attn_update" in names
    for n in names:
        assert hasattr(L, n), n
    assert sorted(kv.EXPORTS) == names


def _shape(dtype=kv.KV_BF16):
    return kv.make_shape(36, 2, 8, 128, 32, dtype)


def _params():
    return kv.make_params(60, 0.5, 0.7, 0.5, 0.95, 4, 20)


def test_rows_and_lengths(L):
    sh = _shape()
    assert kv.kv_rows(sh, 1) == 72
    assert kv.kv_rows(sh, 0) == -1
    assert kv.kv_check_lengths(sh, [6000]) == kv.KV_OK
    assert kv.kv_check_lengths(sh, [6001]) == kv.KV_ERR_UNSUPPORTED_L  # odd
    assert kv.kv_check_lengths(sh, [2 * 11 * 16]) == kv.KV_ERR_UNSUPPORTED_L  # factor 11
    assert kv.kv_check_lengths(sh, [32768 * 2]) == kv.KV_ERR_UNSUPPORTED_L  # too long
    assert kv.kv_check_lengths(sh, [30]) == kv.KV_ERR_UNSUPPORTED_L  # shorter than w
    assert kv.kv_check_lengths(sh, [2000, 3500, 16000]) == kv.KV_OK
    bad = kv.make_shape(1, 1, 1, 96, 32, kv.KV_BF16)
    assert kv.kv_check_lengths(bad, [1024]) == kv.KV_ERR_ARG


def test_total_slots_matches_budget_formula(L):
    sh = _shape()
    p = _params()
    # per layer: sum_h b_h = floor(60 * 6000 * 2 / 100) = 7200, plus one spare slot per head
    assert kv.kv_total_slots(sh, [6000], p) == 36 * (7200 + 2)
    p2 = kv.make_params(25, 0.5, 0.7, 0.5, 0.95, 4, 20)
    sh2 = kv.make_shape(28, 4, 7, 128, 32, kv.KV_BF16)
    Ls = [2000, 3500]
    assert kv.kv_total_slots(sh2, Ls, p2) == sum(28 * ((25 * l * 4) // 100 + 4) for l in Ls)
    assert kv.kv_total_slots(sh, [6000], kv.make_params(0, .5, .7, .5, .95, 4, 20)) == -1


def test_workspace_grows_with_tiles(L):
    sh = _shape()
    a = kv.kv_workspace_bytes(sh, [6000])
    b = kv.kv_workspace_bytes(sh, [12000])
    assert 0 < a < b
    tiles = 72 * ((6000 + 127) // 128)
    assert a >= tiles * 256 * 8  # (max, sum) per tile and window row


def test_argument_errors_launch_nothing(L):
    sh = _shape()
    Larr = (C.c_int32 * 1)(6000)
    st = L.kv_score(C.byref(sh), Larr, 1, None, None, None, None, 0, None)
    assert st == kv.KV_ERR_ARG
    st = L.kv_score(C.byref(sh), Larr, 1, 16, 16, 16, None, 0, None)
    assert st == kv.KV_ERR_WORKSPACE
    st = L.kv_score(C.byref(sh), Larr, 1, 17, 16, 16, 16, 1 << 30, None)  # misaligned
    assert st == kv.KV_ERR_ARG
    st = L.kv_sss(C.byref(sh), Larr, 1, 16, 16, 16, C.c_float(0.5), C.c_float(0.7), None)  # s aliases s_hat
    assert st == kv.KV_ERR_ARG
    st = L.kv_sss(C.byref(sh), Larr, 1, 16, 32, 48, C.c_float(1.5), C.c_float(0.7), None)  # alpha > 1
    assert st == kv.KV_ERR_ARG
    p = kv.make_params(5, 0.5, 0.7, 0.5, 0.95, 4, 20)
    L2 = (C.c_int32 * 1)(256)  # B = 5% of 256*2 = 25 < 2*32
    st = L.kv_allocate(C.byref(sh), L2, 1, C.byref(p), 16, 16, 16, None)
    assert st == kv.KV_ERR_BUDGET
    cache = kv.kv_cache()
    st = L.kv_decode_attn_update(C.byref(sh), Larr, 1, C.byref(_params()), C.byref(cache), 16, 16, 16, 16, None)
    assert st == kv.KV_ERR_ARG


def test_voxzip_argument_errors_launch_nothing(L):
    def call(L_a=(1000,), tau=(80.0,), seg_off=(0, 0), d=2048, dtype=kv.KV_BF16, segs=None, E_A=16, E_T=None,
             n_text_rows=0, E_comp=4096, src=256, out_len=512, status=None):
        n = len(L_a)
        return L.kv_voxzip_pool((C.c_int32 * n)(*L_a), n, (C.c_double * n)(*tau), (C.c_int32 * (n + 1))(*seg_off),
                                d, dtype, C.c_float(0.3), segs, E_A, E_T, n_text_rows, E_comp, src, out_len,
                                status, None)

    assert call(d=3) == kv.KV_ERR_ARG  # 6-byte rows
    assert call(d=4, dtype=kv.KV_BF16) == kv.KV_ERR_ARG  # 8-byte rows
    assert call(tau=(0.0,)) == kv.KV_ERR_ARG
    assert call(tau=(float("inf"),)) == kv.KV_ERR_ARG
    assert call(L_a=(0,)) == kv.KV_ERR_ARG
    assert call(seg_off=(0, 4097), segs=64) == kv.KV_ERR_ARG  # too many segments
    assert call(seg_off=(0, 3), segs=None) == kv.KV_ERR_ARG
    assert call(seg_off=(1, 3), segs=64) == kv.KV_ERR_ARG
    assert call(E_A=24) == kv.KV_ERR_ARG  # misaligned
    assert call(E_T=32, n_text_rows=10) == kv.KV_ERR_ARG  # text rows but no status word
    assert len(kv.pack_segments([(0.0, 1.0)], [0.5], [1], [0])) == kv.ASR_SEGMENT_BYTES


def test_wnw_argument_errors_launch_nothing(L):
    p = kv.make_wnw_params()
    assert kv.kv_wnw_chunk_count([110], p) == 4 and kv.kv_wnw_state_ints([110], p) == 4 + 5 + 18
    assert kv.kv_wnw_chunk_count([50], p) == 1 and kv.kv_wnw_chunk_count([51], p) == 2
    for bad in (kv.kv_wnw_params(50, 30, 3, 3, 18), kv.kv_wnw_params(50, 25, 3, 3, 17),
                kv.kv_wnw_params(50, 25, 9, 3, 54), kv.kv_wnw_params(50, 25, 3, 0, 18),
                kv.kv_wnw_params(50, 0, 3, 3, 18), kv.kv_wnw_params(50, 25, 3, 3, 1025)):
        assert kv.kv_wnw_chunk_count([110], bad) == -1
    Larr = (C.c_int32 * 1)(1000)
    st = L.kv_wnw_update(Larr, 1, C.byref(p), 0, 16, 16, 16, 16, 16, 16, None)  # no anchors
    assert st == kv.KV_ERR_ARG
    st = L.kv_wnw_update(Larr, 1, C.byref(p), 5, 16, 16, 20, 16, 16, 16, None)  # misaligned float64 scores
    assert st == kv.KV_ERR_ARG
    host = (C.c_uint8 * 4096)()  # pageable memory is refused before any launch
    addr = (C.addressof(host) + 15) // 16 * 16
    st = L.kv_wnw_recall(Larr, 1, C.byref(p), 2, 128, kv.KV_BF16, 16, 16, addr, addr, 4096, 8192, None)
    assert st == kv.KV_ERR_ARG
    st = L.kv_wnw_recall(Larr, 1, C.byref(p), 2, 4, kv.KV_BF16, 16, 16, addr, addr, 4096, 8192, None)  # 8 B rows
    assert st == kv.KV_ERR_ARG


def test_c3_argument_errors_launch_nothing(L):
    sh = kv.make_shape(2, 2, 4, 64, 1, kv.KV_BF16)
    p = kv.make_c3_params(128)
    lay = kv.kv_c3_index_layout(sh, [700, 1500], p)
    # the per-node float64 centroids dominate: 2 nodes per key x d x 8 bytes
    assert lay.bytes >= 2 * (4 * 700 + 4 * 1500) * 64 * 8 and lay.hdr % 256 == 0 and lay.cent % 256 == 0
    bad_params = [kv.make_c3_params(0), kv.make_c3_params(8193), kv.make_c3_params(128, iters=0),
                  kv.make_c3_params(128, granularity=3), kv.make_c3_params(128, lam=1.5),
                  kv.make_c3_params(128, exchanges=65), kv.make_c3_params(128, leaf_max=0)]
    Larr = (C.c_int32 * 2)(700, 1500)
    out = kv.kv_c3_layout()
    for bp in bad_params:
        assert L.kv_c3_index_layout(C.byref(sh), Larr, 2, C.byref(bp), C.byref(out)) == kv.KV_ERR_ARG
    wide = kv.make_shape(2, 2, 4, 96, 1, kv.KV_BF16)  # head_dim 96
    assert L.kv_c3_index_layout(C.byref(wide), Larr, 2, C.byref(p), C.byref(out)) == kv.KV_ERR_ARG
    big_g = kv.make_shape(2, 2, 17, 64, 1, kv.KV_BF16)
    assert L.kv_c3_index_layout(C.byref(big_g), Larr, 2, C.byref(p), C.byref(out)) == kv.KV_ERR_ARG
    Llong = (C.c_int32 * 1)(40000)
    assert L.kv_c3_index_layout(C.byref(sh), Llong, 1, C.byref(p), C.byref(out)) == kv.KV_ERR_UNSUPPORTED_L
    assert L.kv_c3_build(C.byref(sh), Larr, 2, C.byref(p), 256, 4096 + 8, None) == kv.KV_ERR_ARG  # misaligned index
    assert L.kv_c3_step(C.byref(sh), Larr, 2, C.byref(p), 256, 256, None, 4096, 4096, None) == kv.KV_ERR_ARG


def test_fault_injection_env(L, monkeypatch):
    sh = _shape()
    Larr = (C.c_int32 * 1)(6000)
    monkeypatch.setenv("KV_FAULT_INJECT", "kv_select_gather")
    st = L.kv_select_gather(C.byref(sh), Larr, 1, 16, 16, 16, 16, 16, 16, 16, 16, None)
    assert st == kv.KV_ERR_CUDA
    monkeypatch.delenv("KV_FAULT_INJECT")
    st = L.kv_select_gather(C.byref(sh), Larr, 1, None, 16, 16, 16, 16, 16, 16, 16, None)
    assert st == kv.KV_ERR_ARG


def test_status_strings(L):
    assert kv.status_string(kv.KV_OK) == "ok"
    assert "budget" in kv.status_string(kv.KV_ERR_BUDGET)
    assert kv.status_string(99) == "unknown status"


def test_wait_limit_round_trips(L):
    # host-side setting only: launches made after the call take the new limit
    prev = kv.kv_set_wait_limit_ns(12345)
    try:
        assert prev == kv.DEFAULT_WAIT_LIMIT_NS
        assert kv.kv_set_wait_limit_ns(0) == 12345
    finally:
        kv.kv_set_wait_limit_ns(prev)
    assert kv.kv_set_wait_limit_ns(prev) == prev


def test_debug_build_exports_and_reports_itself(L):
    # the debug build (index checks compiled in) exports the same symbols and
    # says it is one; the release build loaded by the binding says it is not
    D = C.CDLL(kvbuild.build(debug=True))
    for n in _declared():
        assert hasattr(D, n), n
    D.kv_debug_checks.restype = C.c_int
    assert D.kv_debug_checks() == 1
    assert kv.kv_debug_checks() == kv.DEBUG_CHECKS
