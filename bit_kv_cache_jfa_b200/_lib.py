"""ctypes binding of libjfa.so (the C ABI in include/jfa.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels behind these calls.  If the shared library is missing the import
fails loudly; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int32, c_size_t, c_uint8, c_uint16, c_uint32, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libjfa.so")

JFA_OK = 0
JFA_ERR_INVALID_ARG = 1
JFA_ERR_UNSUPPORTED = 2
JFA_ERR_CUDA = 3
JFA_ERR_DEVICE = 4
DEVERR_NONFINITE_QUANT = 0x1
DEVERR_BAD_INDEX = 0x2
DEVERR_TIMEOUT = 0x4

HEAD_DIM = 128
KEY_GROUP = 64
VAL_GROUP = 32
TAIL_MAX = 64
MAX_GQA = 8
MAX_TOPK = 4096
MAX_EXACT = 8192
BLOCK_TOKENS = 128
MAX_BLOCKS = MAX_EXACT // BLOCK_TOKENS


class JfaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_string(status)})")


class Geom(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("num_heads", c_int32), ("num_kv_heads", c_int32),
                ("head_dim", c_int32), ("capacity", c_int32), ("key_bits", c_int32),
                ("val_bits", c_int32), ("n_ctx", c_int32)]


class Cache(ctypes.Structure):
    _fields_ = [("groups", c_void_p), ("tail_k", c_void_p), ("tail_v", c_void_p)]


class CacheLayout(ctypes.Structure):
    _fields_ = [("record_bytes", c_size_t), ("groups_bytes", c_size_t), ("tail_bytes", c_size_t),
                ("off_key_scales", c_size_t), ("off_key_codes", c_size_t),
                ("off_val_scales", c_size_t), ("off_val_codes", c_size_t)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [("total_bytes", c_size_t), ("off_flag", c_size_t), ("off_scores", c_size_t),
                ("off_partials", c_size_t), ("off_mused", c_size_t), ("off_wts", c_size_t),
                ("off_scan_hist", c_size_t),
                ("off_hist", c_size_t), ("off_counters", c_size_t),
                ("off_cand", c_size_t), ("off_sel", c_size_t),
                ("off_fp4q", c_size_t), ("off_sparse", c_size_t), ("off_ticket", c_size_t),
                ("off_bkeys", c_size_t), ("off_chan", c_size_t), ("off_qstage", c_size_t),
                ("max_topk", c_int32), ("partial_slots", c_int32), ("cand_cap", c_int32),
                ("reserved", c_int32)]


# name -> (restype, argtypes) for every symbol include/jfa.h declares
SIGNATURES = {
    "jfa_status_string": (ctypes.c_char_p, [c_int32]),
    "jfa_cache_layout_get": (c_int32, [POINTER(Geom), POINTER(CacheLayout)]),
    "jfa_workspace_layout_get": (c_int32, [POINTER(Geom), c_int32, POINTER(WorkspaceLayout)]),
    "jfa_pack_kv": (c_int32, [POINTER(Geom), POINTER(Cache), c_void_p, c_void_p, c_int32,
                              c_void_p, c_void_p]),
    "jfa_decode_scores": (c_int32, [POINTER(Geom), POINTER(Cache), c_void_p, c_float, c_void_p,
                                    c_void_p]),
    "jfa_topk": (c_int32, [POINTER(Geom), c_int32, c_void_p, c_void_p, c_void_p]),
    "jfa_topk_blocks": (c_int32, [POINTER(Geom), c_int32, c_void_p, c_void_p, c_void_p]),
    "jfa_topk_noalloc": (c_int32, [c_void_p, c_int32, c_int32, c_int32, c_int32, c_void_p,
                                   c_void_p]),
    "jfa_correct_merge": (c_int32, [POINTER(Geom), POINTER(Cache), c_void_p, c_float, c_void_p,
                                    c_int32, c_void_p, c_void_p, c_int32, c_void_p, c_void_p,
                                    c_void_p]),
    "jfa_decode_step": (c_int32, [POINTER(Geom), POINTER(Cache), c_void_p, c_float, c_int32,
                                  c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p,
                                  c_void_p]),
    "jfa_decode_step_ragged": (c_int32, [POINTER(Geom), c_void_p, POINTER(Cache), c_void_p, c_float,
                                         c_int32, c_void_p, c_void_p, c_void_p, c_int32, c_void_p,
                                         c_void_p, c_void_p]),
    "jfa_append_decode_step": (c_int32, [POINTER(Geom), c_void_p, POINTER(Cache), c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_int32,
                                         c_void_p, c_int32, c_void_p, c_void_p, c_void_p]),
    "jfa_decode_finish": (c_int32, [POINTER(Geom), POINTER(Cache), c_void_p, c_float, c_int32,
                                    c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p,
                                    c_void_p]),
    "jfa_clear_error": (c_int32, [POINTER(Geom), c_void_p, c_void_p]),
    "jfa_check_error": (c_int32, [POINTER(Geom), c_void_p, c_void_p, POINTER(c_uint32)]),
    "jfa_unpack_record": (c_int32, [c_int32, c_int32, c_void_p, POINTER(c_uint8),
                                    POINTER(c_uint16), POINTER(c_uint16), POINTER(c_uint8),
                                    POINTER(c_uint16), POINTER(c_uint16)]),
    "jfa_decode_step_launches": (c_int32, [POINTER(Geom), c_int32]),
    "jfa_selftest_bounded_wait": (c_int32, [POINTER(Geom), c_void_p, c_void_p]),
    "jfa_scan_warps": (c_int32, [POINTER(Geom)]),
    "jfa_fp4_pool_bytes": (c_int32, [POINTER(Geom), POINTER(c_size_t)]),
    "jfa_fp4_pack_keys": (c_int32, [POINTER(Geom), c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                    c_void_p]),
    "jfa_fp4_scores": (c_int32, [POINTER(Geom), c_void_p, c_void_p, c_float, c_void_p, c_void_p]),
    "jfa_sparse_attend": (c_int32, [POINTER(Geom), c_void_p, c_float, c_void_p, c_int32, c_void_p,
                                    c_void_p, c_int32, c_void_p, c_void_p, c_void_p]),
    "jfa_fp4_decode_step": (c_int32, [POINTER(Geom), c_void_p, c_void_p, c_float, c_int32,
                                      c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p,
                                      c_void_p]),
    "jfa_onebit_pool_bytes": (c_int32, [POINTER(Geom), POINTER(c_size_t)]),
    "jfa_onebit_pack": (c_int32, [POINTER(Geom), c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p]),
    "jfa_onebit_attend": (c_int32, [POINTER(Geom), c_void_p, c_void_p, c_float, c_void_p, c_void_p,
                                    c_int32, c_void_p, c_void_p, c_void_p]),
    "jfa_channel_pack": (c_int32, [POINTER(Geom), c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                   c_void_p]),
    "jfa_channel_scores": (c_int32, [POINTER(Geom), c_void_p, c_void_p, c_void_p, c_float,
                                     c_int32, c_void_p, c_void_p]),
    "jfa_channel_decode_step": (c_int32, [POINTER(Geom), c_void_p, c_void_p, c_void_p, c_float,
                                          c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32,
                                          c_void_p, c_void_p, c_void_p]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libjfa.so (built in-tree by bit_kv_cache_jfa_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libjfa.so not found at {LIB_PATH}; build it with "
                "`python -m bit_kv_cache_jfa_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    try:
        return load().jfa_status_string(status).decode()
    except ImportError:
        return "?"


def check(status: int, where: str) -> None:
    if status != JFA_OK:
        raise JfaError(status, where)


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------------------
# one-to-one wrappers (same names as the C ABI)
# ----------------------------------------------------------------------------
def jfa_cache_layout_get(geom: Geom) -> CacheLayout:
    out = CacheLayout()
    check(load().jfa_cache_layout_get(ctypes.byref(geom), ctypes.byref(out)), "jfa_cache_layout_get")
    return out


def jfa_workspace_layout_get(geom: Geom, max_topk: int) -> WorkspaceLayout:
    out = WorkspaceLayout()
    check(load().jfa_workspace_layout_get(ctypes.byref(geom), max_topk, ctypes.byref(out)),
          "jfa_workspace_layout_get")
    return out


def jfa_pack_kv(geom, cache, k_new, v_new, n_new, ws, stream=None) -> int:
    return load().jfa_pack_kv(ctypes.byref(geom), ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                              n_new, _ptr(ws), _stream(stream))


def jfa_decode_scores(geom, cache, q, scale, ws, stream=None) -> int:
    return load().jfa_decode_scores(ctypes.byref(geom), ctypes.byref(cache), _ptr(q), scale,
                                    _ptr(ws), _stream(stream))


def jfa_topk(geom, k, ws, idx, stream=None) -> int:
    return load().jfa_topk(ctypes.byref(geom), k, _ptr(ws), _ptr(idx), _stream(stream))


def jfa_topk_blocks(geom, n_blocks, ws, idx, stream=None) -> int:
    return load().jfa_topk_blocks(ctypes.byref(geom), n_blocks, _ptr(ws), _ptr(idx),
                                  _stream(stream))


def jfa_topk_noalloc(scores, n_seg, stride, n_scores, k, idx, stream=None) -> int:
    """Top-k without any device allocation (scratch is a fixed array in the
    library); scores is an int device address or a tensor."""
    return load().jfa_topk_noalloc(_ptr(scores), n_seg, stride, n_scores, k, _ptr(idx),
                                   _stream(stream))


def jfa_correct_merge(geom, cache, q, scale, idx, k, k_exact, v_exact, exact_on_host, ws, out,
                      stream=None) -> int:
    return load().jfa_correct_merge(ctypes.byref(geom), ctypes.byref(cache), _ptr(q), scale,
                                    _ptr(idx), k, _ptr(k_exact), _ptr(v_exact),
                                    int(exact_on_host), _ptr(ws), _ptr(out), _stream(stream))


def jfa_decode_step(geom, cache, q, scale, k, idx, k_exact, v_exact, exact_on_host, ws, out,
                    stream=None) -> int:
    return load().jfa_decode_step(ctypes.byref(geom), ctypes.byref(cache), _ptr(q), scale, k,
                                  _ptr(idx), _ptr(k_exact), _ptr(v_exact), int(exact_on_host),
                                  _ptr(ws), _ptr(out), _stream(stream))


def jfa_fp4_pool_bytes(geom) -> tuple[int, int]:
    n = c_size_t(0)
    rc = load().jfa_fp4_pool_bytes(ctypes.byref(geom), ctypes.byref(n))
    return rc, n.value


def jfa_fp4_pack_keys(geom, n_from, n_to, k_src, pool, ws, stream=None) -> int:
    return load().jfa_fp4_pack_keys(ctypes.byref(geom), n_from, n_to, _ptr(k_src), _ptr(pool),
                                    _ptr(ws), _stream(stream))


def jfa_fp4_scores(geom, pool, q, scale, ws, stream=None) -> int:
    return load().jfa_fp4_scores(ctypes.byref(geom), _ptr(pool), _ptr(q), scale, _ptr(ws),
                                 _stream(stream))


def jfa_sparse_attend(geom, q, scale, idx, k, k_exact, v_exact, exact_on_host, ws, out,
                      stream=None) -> int:
    return load().jfa_sparse_attend(ctypes.byref(geom), _ptr(q), scale, _ptr(idx), k,
                                    _ptr(k_exact), _ptr(v_exact), int(exact_on_host), _ptr(ws),
                                    _ptr(out), _stream(stream))


def jfa_fp4_decode_step(geom, pool, q, scale, n_blocks, idx, k_exact, v_exact, exact_on_host, ws,
                        out, stream=None) -> int:
    return load().jfa_fp4_decode_step(ctypes.byref(geom), _ptr(pool), _ptr(q), scale, n_blocks,
                                      _ptr(idx), _ptr(k_exact), _ptr(v_exact), int(exact_on_host),
                                      _ptr(ws), _ptr(out), _stream(stream))


def jfa_onebit_pool_bytes(geom) -> tuple[int, int]:
    n = c_size_t(0)
    rc = load().jfa_onebit_pool_bytes(ctypes.byref(geom), ctypes.byref(n))
    return rc, n.value


def jfa_onebit_pack(geom, n_from, n_to, k_src, v_src, pool, ws, stream=None) -> int:
    return load().jfa_onebit_pack(ctypes.byref(geom), n_from, n_to, _ptr(k_src), _ptr(v_src),
                                  _ptr(pool), _ptr(ws), _stream(stream))


def jfa_onebit_attend(geom, pool, q, scale, k_exact, v_exact, exact_on_host, ws, out,
                      stream=None) -> int:
    return load().jfa_onebit_attend(ctypes.byref(geom), _ptr(pool), _ptr(q), scale, _ptr(k_exact),
                                    _ptr(v_exact), int(exact_on_host), _ptr(ws), _ptr(out),
                                    _stream(stream))


def jfa_channel_pack(geom, n_from, n_to, k_src, k_t, k_max, stream=None) -> int:
    return load().jfa_channel_pack(ctypes.byref(geom), n_from, n_to, _ptr(k_src), _ptr(k_t),
                                   _ptr(k_max), _stream(stream))


def jfa_channel_scores(geom, k_t, k_max, q, scale, r, ws, stream=None) -> int:
    return load().jfa_channel_scores(ctypes.byref(geom), _ptr(k_t), _ptr(k_max), _ptr(q), scale,
                                     r, _ptr(ws), _stream(stream))


def jfa_channel_decode_step(geom, k_t, k_max, q, scale, r, k, idx, k_exact, v_exact,
                            exact_on_host, ws, out, stream=None) -> int:
    return load().jfa_channel_decode_step(ctypes.byref(geom), _ptr(k_t), _ptr(k_max), _ptr(q),
                                          scale, r, k, _ptr(idx), _ptr(k_exact), _ptr(v_exact),
                                          int(exact_on_host), _ptr(ws), _ptr(out),
                                          _stream(stream))


def _lens(seq_lens):
    """Host int32 array of per-sequence lengths (kept alive by the caller's
    reference for the duration of the call)."""
    import numpy as np
    a = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    return a, a.ctypes.data


def jfa_decode_step_ragged(geom, seq_lens, cache, q, scale, k, idx, k_exact, v_exact,
                           exact_on_host, ws, out, stream=None) -> int:
    a, p = _lens(seq_lens)
    return load().jfa_decode_step_ragged(ctypes.byref(geom), p, ctypes.byref(cache), _ptr(q),
                                         scale, k, _ptr(idx), _ptr(k_exact), _ptr(v_exact),
                                         int(exact_on_host), _ptr(ws), _ptr(out), _stream(stream))


def jfa_append_decode_step(geom, seq_lens, cache, k_new, v_new, k_exact, v_exact, q, scale, k,
                           idx, exact_on_host, ws, out, stream=None) -> int:
    a, p = _lens(seq_lens)
    return load().jfa_append_decode_step(ctypes.byref(geom), p, ctypes.byref(cache), _ptr(k_new),
                                         _ptr(v_new), _ptr(k_exact), _ptr(v_exact), _ptr(q),
                                         scale, k, _ptr(idx), int(exact_on_host), _ptr(ws),
                                         _ptr(out), _stream(stream))


def jfa_decode_finish(geom, cache, q, scale, k, idx, k_exact, v_exact, exact_on_host, ws, out,
                      stream=None) -> int:
    return load().jfa_decode_finish(ctypes.byref(geom), ctypes.byref(cache), _ptr(q), scale, k,
                                    _ptr(idx), _ptr(k_exact), _ptr(v_exact), int(exact_on_host),
                                    _ptr(ws), _ptr(out), _stream(stream))


def jfa_selftest_bounded_wait(geom, ws, stream=None) -> int:
    return load().jfa_selftest_bounded_wait(ctypes.byref(geom), _ptr(ws), _stream(stream))


def jfa_clear_error(geom, ws, stream=None) -> int:
    return load().jfa_clear_error(ctypes.byref(geom), _ptr(ws), _stream(stream))


def jfa_check_error(geom, ws, stream=None) -> tuple[int, int]:
    flag = c_uint32(0)
    st = load().jfa_check_error(ctypes.byref(geom), _ptr(ws), _stream(stream), ctypes.byref(flag))
    return st, flag.value


def jfa_unpack_record(key_bits: int, val_bits: int, record: bytes):
    """Decode one record (host bytes) -> numpy arrays of codes/scales/zeros."""
    import numpy as np
    kc = np.zeros((64, 128), np.uint8)
    ks = np.zeros(128, np.uint16)
    kz = np.zeros(128, np.uint16)
    vc = np.zeros((64, 128), np.uint8)
    vs = np.zeros((64, 4), np.uint16)
    vz = np.zeros((64, 4), np.uint16)
    buf = ctypes.create_string_buffer(bytes(record), len(record))

    def p(a, t):
        return a.ctypes.data_as(POINTER(t))
    check(load().jfa_unpack_record(key_bits, val_bits, buf, p(kc, c_uint8), p(ks, c_uint16),
                                   p(kz, c_uint16), p(vc, c_uint8), p(vs, c_uint16),
                                   p(vz, c_uint16)), "jfa_unpack_record")
    return kc, ks, kz, vc, vs, vz


def jfa_decode_step_launches(geom: Geom, k: int) -> int:
    return load().jfa_decode_step_launches(ctypes.byref(geom), k)


def jfa_scan_warps(geom: Geom) -> int:
    return load().jfa_scan_warps(ctypes.byref(geom))
