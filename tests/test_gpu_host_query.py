"""A decode step whose query is in pinned host memory: the step's first kernel
copies it into the workspace, then the same kernels run.  Outputs and index
sets must equal the device-query path's bit for bit (same kernels, same
inputs), over a loop of steps with a new query each (the staging of one step
must not overwrite the query the previous step's kernels still read), for
the plain, ragged and append steps and a replayed graph; pageable host
memory is refused before any launch."""
import numpy as np
import pytest
import torch

import oracle.jfa_oracle as O
import workloads as W
import bit_kv_cache_jfa_b200 as jfa
from bit_kv_cache_jfa_b200 import _lib

from jfa_testutil import assert_out_close

pytestmark = pytest.mark.gpu


def _setup(kb=3, vb=2, batch=2, heads=32, kv=8, ctx=4992, k=128, seed=11):
    # ctx a multiple of 64: the cache's capacity (the exact copy is [B][H_kv][ctx][128])
    w = W.Workload("hostq", batch=batch, heads=heads, kv_heads=kv, ctx=ctx, key_bits=kb,
                   val_bits=vb, topk=k, planted=16, seed=seed, value_lognormal=True)
    q = W.gen_q(w)
    k_all, v_all = W.gen_kv(w, q, ctx)
    cache = jfa.KVCache(batch, heads, kv, ctx, kb, vb)
    ws = jfa.Workspace(cache, k)
    ke, ve = k_all.cuda(), v_all.cuda()
    cache.append(ke, ve, ws)
    torch.cuda.synchronize()
    return w, q, k_all, v_all, cache, ws, ke, ve


def _queries(w, n):
    return [W.gen_q(w.with_(seed=w.seed + 100 + s)) for s in range(n)]


def test_host_query_loop_equals_device_query():
    w, q, k_all, v_all, cache, ws, ke, ve = _setup()
    qs = _queries(w, 12)
    scale = W.default_scale(w)
    # device-query reference, one step at a time
    ref = []
    for qq in qs:
        o, i = jfa.decode_step(cache, qq.cuda(), w.topk, ke, ve, ws, scale=scale)
        torch.cuda.synchronize()
        ref.append((o.clone(), i.clone()))
    # host queries: every step enqueued back to back, one pinned buffer each
    hq = [qq.pin_memory() for qq in qs]
    got = [jfa.decode_step(cache, h, w.topk, ke, ve, ws, scale=scale) for h in hq]
    torch.cuda.synchronize()
    assert ws.error_flag(cache) == 0
    for (o, i), (ro, ri) in zip(got, ref):
        assert o.device.type == "cuda"
        assert torch.equal(i, ri)
        assert torch.equal(o, ro)
    # and one step against the oracle
    oc = O.pack_cache(k_all.double().numpy(), v_all.double().numpy(), w.ctx, 3, 2)
    r = O.decode_step(qs[-1].double().numpy(), k_all.double().numpy(), v_all.double().numpy(),
                      oc, w.topk, scale, idx=got[-1][1].cpu().numpy())
    assert_out_close(got[-1][0].cpu().double().numpy(), r.out)


def test_host_query_into_host_output():
    w, q, k_all, v_all, cache, ws, ke, ve = _setup(kb=4, vb=4, batch=1, heads=16, kv=2, ctx=2944,
                                                   k=64)
    out_h = torch.empty(1, 16, 128, dtype=torch.float32).pin_memory()
    o_d, i_d = jfa.decode_step(cache, q.cuda(), 64, ke, ve, ws)
    o_h, i_h = jfa.decode_step(cache, q.pin_memory(), 64, ke, ve, ws, out=out_h)
    torch.cuda.synchronize()
    assert torch.equal(i_h, i_d)
    assert torch.equal(o_h, o_d.cpu())


def test_host_query_ragged_and_append_equal_device_query():
    w, q, k_all, v_all, cache, ws, ke, ve = _setup(ctx=3008, batch=3)
    lens = [3000, 1777, 130]
    for b, L in enumerate(lens):  # each sequence's own tail
        nq = O.split_point(L)
        cache.tail_k[b, :, :L - nq] = ke[b, :, nq:L]
        cache.tail_v[b, :, :L - nq] = ve[b, :, nq:L]
    o1, i1 = jfa.decode_step_ragged(cache, lens, q.cuda(), w.topk, ke, ve, ws)
    torch.cuda.synchronize()
    o1, i1 = o1.clone(), i1.clone()
    o2, i2 = jfa.decode_step_ragged(cache, lens, q.pin_memory(), w.topk, ke, ve, ws)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(o1, o2)

    # append: two caches grown the same way, one with device and one with host queries
    lens = [2000, 1000, 63]
    caches = []
    for _ in range(2):
        c = jfa.KVCache(w.batch, w.heads, w.kv_heads, 3008, 3, 2)
        wsx = jfa.Workspace(c, w.topk)
        c.append(ke[:, :, :2000].contiguous(), ve[:, :, :2000].contiguous(), wsx)
        for b, L in enumerate(lens):
            nq = O.split_point(L)
            c.tail_k[b, :, :L - nq] = ke[b, :, nq:L]
            c.tail_v[b, :, :L - nq] = ve[b, :, nq:L]
        kx = torch.zeros(w.batch, w.kv_heads, 3008, 128, dtype=torch.bfloat16, device="cuda")
        vx = torch.zeros_like(kx)
        for b, L in enumerate(lens):
            kx[b, :, :L], vx[b, :, :L] = ke[b, :, :L], ve[b, :, :L]
        caches.append((c, wsx, kx, vx))
    qs = _queries(w, 6)
    cur = list(lens)
    outs = [[], []]
    for s, qq in enumerate(qs):
        kn = torch.stack([ke[b, :, cur[b]] for b in range(w.batch)]).contiguous()
        vn = torch.stack([ve[b, :, cur[b]] for b in range(w.batch)]).contiguous()
        for j, (c, wsx, kx, vx) in enumerate(caches):
            qa = qq.cuda() if j == 0 else qq.pin_memory()
            outs[j].append(jfa.append_decode_step(c, cur, kn, vn, qa, w.topk, kx, vx, wsx))
        cur = [x + 1 for x in cur]
    torch.cuda.synchronize()
    for (oa, ia), (ob, ib) in zip(*outs):
        assert torch.equal(ia, ib) and torch.equal(oa, ob)


def test_host_query_graph_replay():
    w, q, k_all, v_all, cache, ws, ke, ve = _setup(batch=1, ctx=4096)
    qh = q.clone().pin_memory()
    g = jfa.DecodeGraph(cache, qh, w.topk, ke, ve, ws)
    for qq in _queries(w, 3):
        o_ref, i_ref = jfa.decode_step(cache, qq.cuda(), w.topk, ke, ve, ws)
        torch.cuda.synchronize()
        o_ref, i_ref = o_ref.clone(), i_ref.clone()
        qh.copy_(qq)
        o, i = g.replay()
        torch.cuda.synchronize()
        assert torch.equal(i, i_ref) and torch.equal(o, o_ref)


def test_pageable_host_query_is_refused():
    w, q, k_all, v_all, cache, ws, ke, ve = _setup(batch=1, ctx=1024)
    out = torch.empty(1, 32, 128, dtype=torch.float32, device="cuda")
    idx = torch.empty(1, 8, w.topk, dtype=torch.int32, device="cuda")
    rc = _lib.jfa_decode_step(cache.geom(), cache.struct(), q, 0.088, w.topk, idx, ke, ve, 0,
                              ws.buf, out)
    assert rc == _lib.JFA_ERR_INVALID_ARG
