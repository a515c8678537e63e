"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, reports layouts, rejects bad arguments before any CUDA
work, and its record decoder is a bijection on the packed bits."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from bit_kv_cache_jfa_b200 import build
    build.build()
    from bit_kv_cache_jfa_b200 import _lib
    return _lib


def header_symbols():
    text = open(os.path.join(ROOT, "include", "jfa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(jfa_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    syms = header_symbols()
    assert len(syms) >= 12
    so = ctypes.CDLL(lib.LIB_PATH)
    for s in syms:
        assert hasattr(so, s), s
        assert s in lib.SIGNATURES, s
    assert sorted(lib.SIGNATURES) == syms


def G(**kw):
    from bit_kv_cache_jfa_b200 import Geom
    d = dict(batch=2, num_heads=8, num_kv_heads=2, head_dim=128, capacity=4096, key_bits=3,
             val_bits=2, n_ctx=100)
    d.update(kw)
    return Geom(**d)


@pytest.mark.parametrize("kb,vb,rec", [(3, 2, 6656), (4, 4, 9728), (3, 4, 8704), (4, 2, 7680)])
def test_cache_layout(lib, kb, vb, rec):
    L = lib.jfa_cache_layout_get(G(key_bits=kb, val_bits=vb))
    assert L.record_bytes == rec
    # bytes per token per KV head: codes + scales (104 for K3V2, 152 for K4V4)
    assert L.record_bytes == 64 * (128 * kb // 8 + 8 + 128 * vb // 8 + 16)
    assert L.groups_bytes == 2 * 2 * (4096 // 64) * rec
    assert L.tail_bytes == 2 * 2 * 64 * 128 * 2
    assert (L.off_key_scales, L.off_key_codes) == (0, 512)
    assert L.off_val_scales == 512 + 1024 * kb and L.off_val_codes == L.off_val_scales + 1024
    for off in (L.off_key_codes, L.off_val_scales, L.off_val_codes):
        assert off % 16 == 0


def test_workspace_layout(lib):
    a = lib.jfa_workspace_layout_get(G(), 64)
    b = lib.jfa_workspace_layout_get(G(), 4096)
    assert b.total_bytes >= a.total_bytes and b.max_topk == 4096
    for L in (a, b):
        offs = [L.off_flag, L.off_scores, L.off_partials, L.off_mused, L.off_wts,
                L.off_scan_hist, L.off_hist, L.off_cand, L.off_sel, L.off_fp4q, L.off_sparse,
                L.off_ticket, L.off_bkeys, L.off_chan, L.off_qstage, L.total_bytes]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert L.off_counters == L.off_hist + 4 * 4 * 2048
        assert L.off_scores + 4 * 4 * 4096 <= L.off_partials


@pytest.mark.parametrize("batch,kv", [(1, 1), (1, 2), (1, 8), (2, 8), (3, 4), (4, 8), (8, 8),
                                      (16, 4)])
def test_workspace_histogram_copies_and_query_region(lib, batch, kv):
    # the scan's histogram: 32768 bins + 32 words per copy, R copies per
    # (sequence, KV head): 16 up to 2 segments, 32 / segments below 32, else 1
    n_seg = batch * kv
    reps = 1 if n_seg >= 32 else (16 if n_seg <= 2 else 32 // n_seg)
    L = lib.jfa_workspace_layout_get(G(batch=batch, num_heads=4 * kv, num_kv_heads=kv), 64)
    assert L.off_hist - L.off_scan_hist >= n_seg * reps * (32768 + 32) * 4
    assert L.off_hist - L.off_scan_hist < n_seg * reps * (32768 + 32) * 4 + 256
    # the staged query of a step given q in pinned host memory: bf16 [B][H][128]
    assert L.total_bytes - L.off_qstage >= batch * 4 * kv * 128 * 2
    assert L.off_qstage % 256 == 0


@pytest.mark.parametrize("bad", [dict(head_dim=64), dict(num_heads=12, num_kv_heads=1),
                                 dict(num_heads=9), dict(capacity=100), dict(key_bits=2),
                                 dict(val_bits=3), dict(n_ctx=5000), dict(batch=0)])
def test_bad_geometry_rejected(lib, bad):
    g = G(**bad)
    assert lib.load().jfa_cache_layout_get(ctypes.byref(g), ctypes.byref(lib.CacheLayout())) == 1
    c = lib.Cache(256, 512, 1024)
    assert lib.jfa_pack_kv(g, c, 256, 256, 1, 256) == lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_decode_scores(g, c, 256, 0.1, 256) == lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_topk(g, 8, 256, 256) == lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_decode_step_launches(g, 8) == 0


def test_bad_arguments_rejected_before_launch(lib):
    g, c = G(), lib.Cache(256, 512, 1024)
    inv = lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_pack_kv(g, lib.Cache(0, 512, 1024), 256, 256, 1, 256) == inv
    assert lib.jfa_pack_kv(g, lib.Cache(257, 512, 1024), 256, 256, 1, 256) == inv  # misaligned
    assert lib.jfa_pack_kv(g, c, 256, 256, 4000, 256) == inv                       # > capacity
    assert lib.jfa_pack_kv(g, c, None, 256, 1, 256) == inv
    assert lib.jfa_pack_kv(g, c, 256, 256, -1, 256) == inv
    assert lib.jfa_decode_scores(g, c, 256, -1.0, 256) == inv
    assert lib.jfa_decode_scores(G(n_ctx=0), c, 256, 0.1, 256) == inv
    assert lib.jfa_topk(g, 0, 256, 256) == inv
    assert lib.jfa_topk(g, 4097, 256, 256) == inv
    assert lib.jfa_correct_merge(g, c, 256, 0.1, 256, 8, 256, 256, 0, 256, None) == inv
    assert lib.jfa_correct_merge(g, c, 256, 0.1, None, 8, 256, 256, 0, 256, 256) == inv
    assert lib.jfa_correct_merge(g, c, 256, 0.1, 256, 8, 258, 256, 0, 256, 256) == inv
    assert lib.jfa_decode_step(g, c, 256, 0.1, 0, 256, 256, 256, 0, 256, 256) == inv
    with pytest.raises(ctypes.ArgumentError):
        lib.jfa_topk(g, 1.5, 256, 256)


def test_launch_accounting(lib):
    # scan + the fused finishing kernel
    assert lib.jfa_decode_step_launches(G(n_ctx=4096), 64) == 2
    assert lib.jfa_decode_step_launches(G(n_ctx=100), 64) == 2
    # N_q = 0: no scan
    assert lib.jfa_decode_step_launches(G(n_ctx=64), 8) == 1


def test_status_strings(lib):
    assert lib.status_string(0) == "ok"
    assert lib.status_string(4) == "device error flag set"


@pytest.mark.parametrize("kb,vb", [(3, 2), (4, 4)])
def test_record_decoder_is_a_bijection_on_bits(lib, kb, vb):
    L = lib.jfa_cache_layout_get(G(key_bits=kb, val_bits=vb))
    n = L.record_bytes
    zero = bytes(n)
    base = [a.copy() for a in lib.jfa_unpack_record(kb, vb, zero)]
    assert all(int(a.max()) == 0 for a in base)
    rng = np.random.default_rng(0)
    seen = {}
    # every bit of every section decodes into exactly one output element
    bits = list(range(n * 8))
    rng.shuffle(bits)
    for bit in bits[:3000]:
        rec = bytearray(n)
        rec[bit // 8] = 1 << (bit % 8)
        outs = lib.jfa_unpack_record(kb, vb, bytes(rec))
        hits = [(i, tuple(np.argwhere(a != 0)[0])) for i, a in enumerate(outs) if a.any()]
        assert len(hits) == 1 and sum(int(np.count_nonzero(a)) for a in outs) == 1, bit
        i, pos = hits[0]
        val = int(outs[i][pos])
        assert val & (val - 1) == 0  # a single bit of one code / half
        key = (i, pos, val)
        assert key not in seen, (bit, seen.get(key))
        seen[key] = bit


def test_topk_blocks_rejects_bad_block_counts(lib):
    g = G()
    buf = ctypes.create_string_buffer(1024 + 256)
    ws = (ctypes.addressof(buf) + 255) // 256 * 256
    idx = ws
    for n in (0, -1, lib.MAX_BLOCKS + 1):
        assert lib.jfa_topk_blocks(g, n, ws, idx) == lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_topk_blocks(g, 4, 0, idx) == lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_topk_blocks(g, 4, ws, 0) == lib.JFA_ERR_INVALID_ARG


def test_fp4_pool_size_and_argument_checks(lib):
    rc, n = lib.jfa_fp4_pool_bytes(G(capacity=4096))
    assert rc == 0 and n == 2 * 2 * 32 * 9232
    rc, _ = lib.jfa_fp4_pool_bytes(G(capacity=4096 + 64))   # not a multiple of 128
    assert rc == lib.JFA_ERR_INVALID_ARG
    g = G(capacity=4096, n_ctx=1000)
    bad = lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_fp4_pack_keys(g, 0, 100, 256, 256, 256) == bad            # not a group edge
    assert lib.jfa_fp4_pack_keys(g, 128, 64, 256, 256, 256) == bad           # n_to < n_from
    assert lib.jfa_fp4_pack_keys(g, 0, 4160, 256, 256, 256) == bad           # past capacity
    assert lib.jfa_fp4_pack_keys(g, 64, 64, 256, 256, 256) == 0              # nothing to do
    assert lib.jfa_fp4_scores(g, 256, 256, 0.0, 256) == bad                  # scale
    assert lib.jfa_fp4_scores(g, 8, 256, 0.1, 256) == bad                    # pool alignment
    assert lib.jfa_sparse_attend(g, 256, 0.1, 256, 0, 256, 256, 0, 256, 256) == bad   # k = 0
    assert lib.jfa_sparse_attend(g, 256, 0.1, 256, 8193, 256, 256, 0, 256, 256) == bad
    assert lib.jfa_fp4_decode_step(g, 256, 256, 0.1, 0, 256, 256, 256, 0, 256, 256) == bad
    assert lib.jfa_fp4_decode_step(g, 256, 256, 0.1, 65, 256, 256, 256, 0, 256, 256) == bad


def test_channel_argument_checks(lib):
    g = G(capacity=4096, n_ctx=1000)
    bad = lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_channel_pack(g, 0, 100, 256, 256, 256) == bad        # not a group edge
    assert lib.jfa_channel_pack(g, 0, 4160, 256, 256, 256) == bad       # past capacity
    assert lib.jfa_channel_pack(g, 64, 64, 256, 256, 256) == 0          # nothing to do
    assert lib.jfa_channel_scores(g, 256, 256, 256, 0.1, 0, 256) == bad     # r = 0
    assert lib.jfa_channel_scores(g, 256, 256, 256, 0.1, 129, 256) == bad   # r > 128
    assert lib.jfa_channel_scores(g, 8, 256, 256, 0.1, 16, 256) == bad      # k_t alignment
    assert lib.jfa_channel_decode_step(g, 256, 256, 256, 0.1, 16, 0, 256, 256, 256, 0, 256,
                                       256) == bad                          # k = 0
    assert lib.jfa_channel_decode_step(g, 256, 256, 256, 0.1, 16, 4097, 256, 256, 256, 0, 256,
                                       256) == bad                          # k > JFA_MAX_TOPK


def test_onebit_argument_checks(lib):
    rc, n = lib.jfa_onebit_pool_bytes(G(capacity=4096))
    assert rc == 0 and n == 2 * 2 * 64 * 3584
    g = G(capacity=4096, n_ctx=1000)
    bad = lib.JFA_ERR_INVALID_ARG
    assert lib.jfa_onebit_pack(g, 0, 100, 256, 256, 256, 256) == bad       # not a group edge
    assert lib.jfa_onebit_pack(g, 0, 4160, 256, 256, 256, 256) == bad      # past capacity
    assert lib.jfa_onebit_pack(g, 64, 64, 256, 256, 256, 256) == 0         # nothing to do
    assert lib.jfa_onebit_attend(g, 256, 256, 0.0, 256, 256, 0, 256, 256) == bad   # scale
    assert lib.jfa_onebit_attend(g, 8, 256, 0.1, 256, 256, 0, 256, 256) == bad     # pool alignment
    assert lib.jfa_onebit_attend(G(capacity=4096, n_ctx=0), 256, 256, 0.1, 256, 256, 0, 256,
                                 256) == bad                                     # empty context
