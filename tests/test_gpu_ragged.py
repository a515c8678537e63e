"""GPU parity of the per-sequence-length paths against the fp64 oracle:
jfa_decode_step_ragged (every sequence its own N_q and tail) and
jfa_append_decode_step (one token per sequence appended at its own position,
full tails flushed into groups, then the step), over a loop of appends."""
import numpy as np
import pytest
import torch

import oracle.jfa_oracle as O
import workloads as W
import bit_kv_cache_jfa_b200 as jfa
from bit_kv_cache_jfa_b200 import _lib

from jfa_testutil import assert_out_close, assert_topk_valid

pytestmark = pytest.mark.gpu


def _wl(kb, vb, heads, kv, batch, ctx, k, seed=7):
    return W.Workload("ragged", batch=batch, heads=heads, kv_heads=kv, ctx=ctx, key_bits=kb,
                      val_bits=vb, topk=k, planted=16, seed=seed, value_lognormal=True)


def _ragged_cache(w, lens, cap, q, k_all, v_all):
    """A cache whose sequence b holds lens[b] tokens: groups packed to the
    longest length (a group depends on its own 64 tokens only), then each
    sequence's tail written for its own length."""
    cache = jfa.KVCache(w.batch, w.heads, w.kv_heads, cap, w.key_bits, w.val_bits)
    ws = jfa.Workspace(cache, max(w.topk, 1))
    n = max(lens)
    cache.append(k_all[:, :, :n].cuda().contiguous(), v_all[:, :, :n].cuda().contiguous(), ws)
    for b, L in enumerate(lens):
        nq = O.split_point(L)
        cache.tail_k[b, :, :L - nq] = k_all[b, :, nq:L].cuda()
        cache.tail_v[b, :, :L - nq] = v_all[b, :, nq:L].cuda()
    return cache, ws


def _oracle(w, lens, q, k_all, v_all, k, scale, idx=None):
    outs, sels = [], []
    for b, L in enumerate(lens):
        kk = k_all[b:b + 1].double().numpy()
        vv = v_all[b:b + 1].double().numpy()
        oc = O.pack_cache(kk, vv, L, w.key_bits, w.val_bits)
        r = O.decode_step(q[b:b + 1].double().numpy(), kk, vv, oc, k, scale,
                          idx=None if idx is None else idx[b:b + 1])
        outs.append(r.out[0])
        sels.append(r.select[0])
    return np.stack(outs), sels


@pytest.mark.parametrize("kb,vb,heads,kv", [(3, 2, 32, 8), (4, 4, 16, 2), (3, 4, 64, 8)])
def test_ragged_step_against_oracle(kb, vb, heads, kv):
    lens = [1, 63, 64, 65, 4097, 3000, 129, 2048]
    w = _wl(kb, vb, heads, kv, len(lens), max(lens), 64)
    cap = 64 * -(-max(lens) // 64)
    q = W.gen_q(w)
    k_all, v_all = W.gen_kv(w, q, max(lens))
    cache, ws = _ragged_cache(w, lens, cap, q, k_all, v_all)
    ke = torch.zeros(w.batch, w.kv_heads, cap, 128, dtype=torch.bfloat16, device="cuda")
    ve = torch.zeros_like(ke)
    ke[:, :, :max(lens)] = k_all.cuda()
    ve[:, :, :max(lens)] = v_all.cuda()
    scale = W.default_scale(w)
    out, idx = jfa.decode_step_ragged(cache, lens, q.cuda(), w.topk, ke, ve, ws, scale=scale)
    torch.cuda.synchronize()
    assert ws.error_flag(cache) == 0
    out, idx = out.cpu().double().numpy(), idx.cpu().numpy()
    ref_same, sels = _oracle(w, lens, q, k_all, v_all, w.topk, scale, idx=idx)
    assert_out_close(out, ref_same)
    for b, L in enumerate(lens):
        nq = O.split_point(L)
        assert_topk_valid(idx[b:b + 1], sels[b][None], w.topk)
        keff = min(w.topk, nq)
        assert np.all(idx[b, :, keff:] == -1)


def test_append_decode_loop_against_oracle():
    # ragged lengths, 70 steps of one appended token each: every sequence
    # crosses at least one 64-token boundary (its tail is flushed into a group)
    lens = [63, 64, 65, 127, 128, 200, 1, 500]
    steps = 70
    w = _wl(3, 2, 32, 8, len(lens), max(lens) + steps, 64, seed=9)
    cap = 64 * -(-(max(lens) + steps) // 64)
    q = W.gen_q(w)
    k_all, v_all = W.gen_kv(w, q, max(lens) + steps)
    cache, ws = _ragged_cache(w, lens, cap, q, k_all, v_all)
    # the exact copy holds only the tokens cached so far; appends add the rest
    ke = torch.zeros(w.batch, w.kv_heads, cap, 128, dtype=torch.bfloat16, device="cuda")
    ve = torch.zeros_like(ke)
    for b, L in enumerate(lens):
        ke[b, :, :L] = k_all[b, :, :L].cuda()
        ve[b, :, :L] = v_all[b, :, :L].cuda()
    scale = W.default_scale(w)
    cur = list(lens)
    rng = np.random.default_rng(3)
    for s in range(steps):
        kn = torch.stack([k_all[b, :, cur[b]] for b in range(w.batch)]).cuda().contiguous()
        vn = torch.stack([v_all[b, :, cur[b]] for b in range(w.batch)]).cuda().contiguous()
        qs = W.gen_q(w.with_(seed=w.seed + 1 + s))   # a new query token every step
        out, idx = jfa.append_decode_step(cache, cur, kn, vn, qs.cuda(), w.topk, ke, ve, ws,
                                          scale=scale)
        cur = [c + 1 for c in cur]
        if s in (0, 1, 37, steps - 1) or rng.random() < 0.05:
            torch.cuda.synchronize()
            assert ws.error_flag(cache) == 0
            o, ix = out.cpu().double().numpy(), idx.cpu().numpy()
            ref, sels = _oracle(w, cur, qs, k_all, v_all, w.topk, scale, idx=ix)
            print(f"step {s}: lengths {cur}")
            assert_out_close(o, ref)
            for b in range(w.batch):
                assert_topk_valid(ix[b:b + 1], sels[b][None], w.topk)
    # the packed state equals the oracle's pack at the final lengths
    torch.cuda.synchronize()
    for b, L in enumerate(cur):
        oc = O.pack_cache(k_all[b:b + 1].double().numpy(), v_all[b:b + 1].double().numpy(), L,
                          3, 2)
        nq = oc.n_quant
        for h in (0, w.kv_heads - 1):
            for gi in sorted({0, nq // 64 - 1}) if nq else []:
                kc, ks, kz, vc, vs, vz = _lib.jfa_unpack_record(3, 2, cache.record(b, h, gi))
                sl = slice(64 * gi, 64 * gi + 64)
                assert np.array_equal(kc, oc.k_codes[0, h, sl]), (b, h, gi)
                assert np.array_equal(vc, oc.v_codes[0, h, sl]), (b, h, gi)
                assert np.array_equal(ks, oc.k_scale[0, h, gi].view(np.uint16))
                assert np.array_equal(vz, oc.v_zero[0, h, sl].view(np.uint16))
            t = L - nq
            assert torch.equal(cache.tail_k[b, h, :t].cpu(), k_all[b, h, nq:L])
            assert torch.equal(cache.tail_v[b, h, :t].cpu(), v_all[b, h, nq:L])
        assert torch.equal(ke[b, :, :L].cpu(), k_all[b, :, :L])


def test_uniform_lengths_through_the_ragged_call_equal_the_step():
    w = _wl(4, 4, 32, 8, 2, 5000, 128)
    lens = [5000, 5000]
    q = W.gen_q(w)
    k_all, v_all = W.gen_kv(w, q, 5000)
    cap = 5056
    cache, ws = _ragged_cache(w, lens, cap, q, k_all, v_all)
    ke = torch.zeros(2, 8, cap, 128, dtype=torch.bfloat16, device="cuda")
    ve = torch.zeros_like(ke)
    ke[:, :, :5000], ve[:, :, :5000] = k_all.cuda(), v_all.cuda()
    o1, i1 = jfa.decode_step_ragged(cache, lens, q.cuda(), 128, ke, ve, ws)
    o2, i2 = jfa.decode_step(cache, q.cuda(), 128, ke, ve, ws)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2)
    assert torch.equal(o1, o2)
