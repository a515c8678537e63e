"""B200-native approximate-then-correct low-bit KV decode attention.

A thin Python layer over ``libjfa.so`` (C ABI in ``include/jfa.h``).  Torch
provides device memory and streams; every step of the decode path runs in
the library's sm_100a kernels:

    cache = KVCache(batch, heads, kv_heads, capacity, key_bits=3, val_bits=2)
    ws = Workspace(cache, max_topk=256)
    cache.append(k_new, v_new, ws)              # jfa_pack_kv
    out, idx = decode_step(cache, q, 256, k_exact, v_exact, ws)
"""
from __future__ import annotations

import math

from . import _lib
from ._lib import (  # noqa: F401  (re-exported C ABI names)
    Cache, CacheLayout, Geom, JfaError, WorkspaceLayout, check, jfa_cache_layout_get,
    jfa_check_error, jfa_clear_error, jfa_correct_merge, jfa_decode_finish, jfa_decode_scores,
    jfa_append_decode_step, jfa_decode_step, jfa_decode_step_ragged,
    jfa_channel_decode_step, jfa_channel_pack, jfa_channel_scores,
    jfa_decode_step_launches, jfa_fp4_decode_step, jfa_fp4_pack_keys, jfa_fp4_pool_bytes,
    jfa_onebit_attend, jfa_onebit_pack, jfa_onebit_pool_bytes,
    jfa_fp4_scores, jfa_pack_kv, jfa_sparse_attend, jfa_topk, jfa_topk_blocks,
    jfa_unpack_record, jfa_workspace_layout_get, load)

__all__ = ["KVCache", "Workspace", "decode_step", "decode_step_blocks", "decode_step_ragged",
           "append_decode_step", "FP4KeyPool", "fp4_decode_step", "sparse_attend",
           "ChannelKeys", "channel_decode_step", "OneBitCache", "onebit_attend", "DecodeGraph",
           "JfaError", "load"]


def _torch():
    import torch
    return torch


class KVCache:
    """One layer's quantized KV cache (device buffers owned by torch)."""

    def __init__(self, batch: int, num_heads: int, num_kv_heads: int, capacity: int,
                 key_bits: int = 3, val_bits: int = 2, device="cuda", head_dim: int = 128):
        torch = _torch()
        self.batch, self.num_heads, self.num_kv_heads = batch, num_heads, num_kv_heads
        self.capacity, self.key_bits, self.val_bits = capacity, key_bits, val_bits
        self.head_dim = head_dim
        self.n_ctx = 0
        self.layout = jfa_cache_layout_get(self.geom())
        self.groups = torch.empty(self.layout.groups_bytes, dtype=torch.uint8, device=device)
        shape = (batch, num_kv_heads, _lib.TAIL_MAX, head_dim)
        self.tail_k = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.tail_v = torch.zeros(shape, dtype=torch.bfloat16, device=device)

    def geom(self, n_ctx: int | None = None) -> Geom:
        return Geom(self.batch, self.num_heads, self.num_kv_heads, self.head_dim, self.capacity,
                    self.key_bits, self.val_bits, self.n_ctx if n_ctx is None else n_ctx)

    def struct(self) -> Cache:
        return Cache(self.groups.data_ptr(), self.tail_k.data_ptr(), self.tail_v.data_ptr())

    @property
    def n_quant(self) -> int:
        return 0 if self.n_ctx <= 0 else 64 * ((self.n_ctx - 1) // 64)

    def append(self, k_new, v_new, ws: "Workspace", stream=None) -> None:
        """Append bf16 [B, H_kv, n, 128] keys/values (contiguous, on device)."""
        n = k_new.shape[2]
        check(jfa_pack_kv(self.geom(), self.struct(), k_new, v_new, n, ws.buf, stream),
              "jfa_pack_kv")
        self.n_ctx += n

    def record(self, b: int, h: int, g: int):
        """Host bytes of the packed record of (sequence b, KV head h, group g)."""
        rb = self.layout.record_bytes
        seg = b * self.num_kv_heads + h
        off = (seg * (self.capacity // 64) + g) * rb
        return self.groups[off:off + rb].cpu().numpy().tobytes()


class Workspace:
    """Scratch of the decode step for a cache geometry and a maximum k."""

    def __init__(self, cache: KVCache, max_topk: int, device="cuda"):
        torch = _torch()
        self.layout = jfa_workspace_layout_get(cache.geom(), max_topk)
        self.buf = torch.zeros(self.layout.total_bytes, dtype=torch.uint8, device=device)
        self.max_topk = max_topk

    def scores(self, cache: KVCache):
        """View of the selection scores S: fp32 [B, H_kv, capacity]."""
        torch = _torch()
        n = cache.batch * cache.num_kv_heads * cache.capacity
        v = self.buf[self.layout.off_scores:self.layout.off_scores + 4 * n].view(torch.float32)
        return v.view(cache.batch, cache.num_kv_heads, cache.capacity)

    def error_flag(self, cache: KVCache, stream=None) -> int:
        return jfa_check_error(cache.geom(), self.buf, stream)[1]


def default_scale(head_dim: int = 128) -> float:
    return 1.0 / math.sqrt(head_dim)


def decode_step(cache: KVCache, q, k: int, k_exact, v_exact, ws: Workspace, scale=None,
                out=None, idx=None, exact_on_host: bool = False, stream=None):
    """One decode step for every sequence and query head.

    q: bf16 [B, H, 128], device or pinned host memory (a host query is
    copied into the workspace by the step's first kernel); k_exact/v_exact:
    bf16 [B, H_kv, capacity, 128] (device, or pinned host with
    exact_on_host=True).  Returns (out fp32 [B, H, 128], idx int32
    [B, H_kv, k]), on the cache's device unless given."""
    torch = _torch()
    if scale is None:
        scale = default_scale(cache.head_dim)
    dev = cache.groups.device  # q may be in pinned host memory
    if out is None:
        out = torch.empty(cache.batch, cache.num_heads, cache.head_dim, dtype=torch.float32,
                          device=dev)
    if idx is None:
        idx = torch.empty(cache.batch, cache.num_kv_heads, k, dtype=torch.int32, device=dev)
    check(jfa_decode_step(cache.geom(), cache.struct(), q, float(scale), k, idx, k_exact,
                          v_exact, exact_on_host, ws.buf, out, stream), "jfa_decode_step")
    return out, idx


def decode_step_blocks(cache: KVCache, q, n_blocks: int, k_exact, v_exact, ws: Workspace,
                       scale=None, out=None, idx=None, exact_on_host: bool = False, stream=None):
    """One decode step with 128-token block selection: jfa_decode_scores,
    jfa_topk_blocks (the n_blocks best blocks per sequence and KV head), then
    jfa_correct_merge on their tokens.  Returns (out fp32 [B, H, 128], idx
    int32 [B, H_kv, n_blocks * 128])."""
    torch = _torch()
    if scale is None:
        scale = default_scale(cache.head_dim)
    dev = cache.groups.device  # q may be in pinned host memory
    k = n_blocks * _lib.BLOCK_TOKENS
    if out is None:
        out = torch.empty(cache.batch, cache.num_heads, cache.head_dim, dtype=torch.float32,
                          device=dev)
    if idx is None:
        idx = torch.empty(cache.batch, cache.num_kv_heads, k, dtype=torch.int32, device=dev)
    g, cs = cache.geom(), cache.struct()
    check(jfa_decode_scores(g, cs, q, float(scale), ws.buf, stream), "jfa_decode_scores")
    check(jfa_topk_blocks(g, n_blocks, ws.buf, idx, stream), "jfa_topk_blocks")
    check(jfa_correct_merge(g, cs, q, float(scale), idx, k, k_exact, v_exact, exact_on_host,
                            ws.buf, out, stream), "jfa_correct_merge")
    return out, idx


def decode_step_ragged(cache: KVCache, seq_lens, q, k: int, k_exact, v_exact, ws: Workspace,
                       scale=None, out=None, idx=None, exact_on_host: bool = False, stream=None):
    """decode_step for sequences of different lengths: seq_lens (host ints,
    one per sequence) gives each sequence's cached tokens."""
    torch = _torch()
    if scale is None:
        scale = default_scale(cache.head_dim)
    dev = cache.groups.device  # q may be in pinned host memory
    if out is None:
        out = torch.empty(cache.batch, cache.num_heads, cache.head_dim, dtype=torch.float32,
                          device=dev)
    if idx is None:
        idx = torch.empty(cache.batch, cache.num_kv_heads, k, dtype=torch.int32, device=dev)
    check(jfa_decode_step_ragged(cache.geom(), seq_lens, cache.struct(), q, float(scale), k, idx,
                                 k_exact, v_exact, exact_on_host, ws.buf, out, stream),
          "jfa_decode_step_ragged")
    return out, idx


def append_decode_step(cache: KVCache, seq_lens, k_new, v_new, q, k: int, k_exact, v_exact,
                       ws: Workspace, scale=None, out=None, idx=None, exact_on_host: bool = False,
                       stream=None):
    """Append one token per sequence (bf16 [B, H_kv, 128] k_new / v_new, at
    position seq_lens[b]; also written into the exact copy) and run the
    decode step over the grown cache.  The caller adds one to every length
    afterwards."""
    torch = _torch()
    if scale is None:
        scale = default_scale(cache.head_dim)
    dev = cache.groups.device  # q may be in pinned host memory
    if out is None:
        out = torch.empty(cache.batch, cache.num_heads, cache.head_dim, dtype=torch.float32,
                          device=dev)
    if idx is None:
        idx = torch.empty(cache.batch, cache.num_kv_heads, k, dtype=torch.int32, device=dev)
    check(jfa_append_decode_step(cache.geom(), seq_lens, cache.struct(), k_new, v_new, k_exact,
                                 v_exact, q, float(scale), k, idx, exact_on_host, ws.buf, out,
                                 stream), "jfa_append_decode_step")
    return out, idx


class FP4KeyPool:
    """NVFP4 keys of one layer, one record per (sequence, KV head, 128-token
    block), packed from the exact bf16 keys (device buffer owned by torch).
    The geometry's key_bits / val_bits are not used by the FP4 calls."""

    def __init__(self, batch: int, num_heads: int, num_kv_heads: int, capacity: int,
                 device="cuda", head_dim: int = 128):
        torch = _torch()
        self.batch, self.num_heads, self.num_kv_heads = batch, num_heads, num_kv_heads
        self.capacity, self.head_dim = capacity, head_dim
        self.n_packed = 0
        rc, nbytes = _lib.jfa_fp4_pool_bytes(self.geom(0))
        check(rc, "jfa_fp4_pool_bytes")
        self.pool = torch.zeros(nbytes, dtype=torch.uint8, device=device)

    def geom(self, n_ctx: int = 0) -> Geom:
        return Geom(self.batch, self.num_heads, self.num_kv_heads, self.head_dim, self.capacity,
                    4, 4, n_ctx)

    def pack(self, k_exact, n_to: int, ws: "Workspace", stream=None) -> None:
        """Quantize the key groups from the packed length up to n_to (a
        multiple of 64) from k_exact bf16 [B, H_kv, capacity, 128]."""
        check(_lib.jfa_fp4_pack_keys(self.geom(n_to), self.n_packed, n_to, k_exact, self.pool,
                                     ws.buf, stream), "jfa_fp4_pack_keys")
        self.n_packed = max(self.n_packed, n_to)

    def sync(self, k_exact, n_ctx: int, ws: "Workspace", stream=None) -> None:
        """Pack every group below N_q of a context of n_ctx tokens."""
        nq = 0 if n_ctx <= 0 else 64 * ((n_ctx - 1) // 64)
        if nq > self.n_packed:
            self.pack(k_exact, nq, ws, stream)


def fp4_decode_step(pool: FP4KeyPool, n_ctx: int, q, n_blocks: int, k_exact, v_exact,
                    ws: Workspace, scale=None, out=None, idx=None, exact_on_host: bool = False,
                    stream=None):
    """One NVFP4 decode step over n_ctx cached tokens (groups below N_q must
    be packed): FP4 scan, the n_blocks best 128-token blocks, exact
    attention over them and the tail.  Returns (out fp32 [B, H, 128], idx
    int32 [B, H_kv, n_blocks * 128])."""
    torch = _torch()
    if scale is None:
        scale = default_scale(pool.head_dim)
    dev = q.device
    if out is None:
        out = torch.empty(pool.batch, pool.num_heads, pool.head_dim, dtype=torch.float32,
                          device=dev)
    if idx is None:
        idx = torch.empty(pool.batch, pool.num_kv_heads, n_blocks * _lib.BLOCK_TOKENS,
                          dtype=torch.int32, device=dev)
    check(_lib.jfa_fp4_decode_step(pool.geom(n_ctx), pool.pool, q, float(scale), n_blocks, idx,
                                   k_exact, v_exact, exact_on_host, ws.buf, out, stream),
          "jfa_fp4_decode_step")
    return out, idx


def sparse_attend(geom: Geom, q, idx, k_exact, v_exact, ws: Workspace, scale=None, out=None,
                  exact_on_host: bool = False, stream=None):
    """Exact attention over the tokens idx [B, H_kv, k] (-1 = none) and the
    tail [N_q, n_ctx) of every sequence; returns out fp32 [B, H, 128]."""
    torch = _torch()
    if scale is None:
        scale = default_scale(geom.head_dim)
    if out is None:
        out = torch.empty(geom.batch, geom.num_heads, geom.head_dim, dtype=torch.float32,
                          device=q.device)
    check(_lib.jfa_sparse_attend(geom, q, float(scale), idx, idx.shape[-1], k_exact, v_exact,
                                 exact_on_host, ws.buf, out, stream), "jfa_sparse_attend")
    return out


class ChannelKeys:
    """Channel-major bf16 copy of one layer's keys and the per-channel max|K|
    (device buffers owned by torch), for the critical-channel selection."""

    def __init__(self, batch: int, num_heads: int, num_kv_heads: int, capacity: int,
                 device="cuda", head_dim: int = 128):
        torch = _torch()
        self.batch, self.num_heads, self.num_kv_heads = batch, num_heads, num_kv_heads
        self.capacity, self.head_dim = capacity, head_dim
        self.n_packed = 0
        self.k_t = torch.zeros(batch, num_kv_heads, head_dim, capacity, dtype=torch.bfloat16,
                               device=device)
        self.k_max = torch.zeros(batch, num_kv_heads, head_dim, dtype=torch.float32,
                                 device=device)

    def geom(self, n_ctx: int = 0) -> Geom:
        return Geom(self.batch, self.num_heads, self.num_kv_heads, self.head_dim, self.capacity,
                    4, 4, n_ctx)

    def sync(self, k_exact, n_ctx: int, stream=None) -> None:
        """Copy every group below N_q of a context of n_ctx tokens."""
        nq = 0 if n_ctx <= 0 else 64 * ((n_ctx - 1) // 64)
        if nq > self.n_packed:
            check(_lib.jfa_channel_pack(self.geom(nq), self.n_packed, nq, k_exact, self.k_t,
                                        self.k_max, stream), "jfa_channel_pack")
            self.n_packed = nq


def channel_decode_step(keys: ChannelKeys, n_ctx: int, q, r: int, k: int, k_exact, v_exact,
                        ws: Workspace, scale=None, out=None, idx=None, exact_on_host: bool = False,
                        stream=None):
    """One decode step with critical-channel selection: scores over the r
    most important channels, the top-k tokens, exact attention over them and
    the tail.  Returns (out fp32 [B, H, 128], idx int32 [B, H_kv, k])."""
    torch = _torch()
    if scale is None:
        scale = default_scale(keys.head_dim)
    dev = q.device
    if out is None:
        out = torch.empty(keys.batch, keys.num_heads, keys.head_dim, dtype=torch.float32,
                          device=dev)
    if idx is None:
        idx = torch.empty(keys.batch, keys.num_kv_heads, k, dtype=torch.int32, device=dev)
    check(_lib.jfa_channel_decode_step(keys.geom(n_ctx), keys.k_t, keys.k_max, q, float(scale), r,
                                       k, idx, k_exact, v_exact, exact_on_host, ws.buf, out,
                                       stream), "jfa_channel_decode_step")
    return out, idx


class OneBitCache:
    """One layer's 1-bit KV cache (records of 64-token groups packed from the
    exact bf16 rows; device buffer owned by torch)."""

    def __init__(self, batch: int, num_heads: int, num_kv_heads: int, capacity: int,
                 device="cuda", head_dim: int = 128):
        torch = _torch()
        self.batch, self.num_heads, self.num_kv_heads = batch, num_heads, num_kv_heads
        self.capacity, self.head_dim = capacity, head_dim
        self.n_packed = 0
        rc, nbytes = _lib.jfa_onebit_pool_bytes(self.geom(0))
        check(rc, "jfa_onebit_pool_bytes")
        self.pool = torch.zeros(nbytes, dtype=torch.uint8, device=device)

    def geom(self, n_ctx: int = 0) -> Geom:
        return Geom(self.batch, self.num_heads, self.num_kv_heads, self.head_dim, self.capacity,
                    4, 4, n_ctx)

    def sync(self, k_exact, v_exact, n_ctx: int, ws: "Workspace", stream=None) -> None:
        """Pack every group below N_q of a context of n_ctx tokens."""
        nq = 0 if n_ctx <= 0 else 64 * ((n_ctx - 1) // 64)
        if nq > self.n_packed:
            check(_lib.jfa_onebit_pack(self.geom(nq), self.n_packed, nq, k_exact, v_exact,
                                       self.pool, ws.buf, stream), "jfa_onebit_pack")
            self.n_packed = nq


def onebit_attend(cache: OneBitCache, n_ctx: int, q, k_exact, v_exact, ws: Workspace, scale=None,
                  out=None, exact_on_host: bool = False, stream=None):
    """Dense attention over the 1-bit tokens and the exact tail; returns out
    fp32 [B, H, 128]."""
    torch = _torch()
    if scale is None:
        scale = default_scale(cache.head_dim)
    if out is None:
        out = torch.empty(cache.batch, cache.num_heads, cache.head_dim, dtype=torch.float32,
                          device=q.device)
    check(_lib.jfa_onebit_attend(cache.geom(n_ctx), cache.pool, q, float(scale), k_exact, v_exact,
                                 exact_on_host, ws.buf, out, stream), "jfa_onebit_attend")
    return out


class DecodeGraph:
    """decode_step captured once in a CUDA graph and replayed.

    The graph holds the step's two kernel launches with their arguments as
    they were at capture: the cache length, every buffer address (q, the
    exact rows, the workspace, out, idx) and k.  Write the next query into
    the same q tensor and call replay(); after appending to the cache,
    capture a new graph (the length is part of the launch arguments)."""

    def __init__(self, cache: KVCache, q, k: int, k_exact, v_exact, ws: Workspace, scale=None,
                 out=None, idx=None, exact_on_host: bool = False):
        torch = _torch()
        dev = cache.groups.device
        if out is None:
            out = torch.empty(cache.batch, cache.num_heads, cache.head_dim, dtype=torch.float32,
                              device=dev)
        if idx is None:
            idx = torch.empty(cache.batch, cache.num_kv_heads, k, dtype=torch.int32, device=dev)
        self.out, self.idx = out, idx
        args = (cache, q, k, k_exact, v_exact, ws)
        kw = dict(scale=scale, out=out, idx=idx, exact_on_host=exact_on_host)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):  # one eager step: one-time kernel set-up stays out of the graph
            decode_step(*args, stream=side, **kw)
        torch.cuda.current_stream(dev).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            decode_step(*args, stream=torch.cuda.current_stream(dev), **kw)

    def replay(self):
        """Run the captured step on the current stream; returns (out, idx)."""
        self.graph.replay()
        return self.out, self.idx
