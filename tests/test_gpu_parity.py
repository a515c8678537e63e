"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded
inputs (bit-exact for codes, scales, zeros, tails and top-k sets; fp
outputs within max-abs 2e-3 and rel-L2 1e-3)."""
import numpy as np
import pytest
import torch

import oracle.jfa_oracle as O
import workloads as W
import bit_kv_cache_jfa_b200 as jfa
from bit_kv_cache_jfa_b200 import _lib

from jfa_testutil import (DeviceRun, SCORE_ABS, assert_out_close, assert_topk_valid)

pytestmark = pytest.mark.gpu

TINY = W.WORKLOADS["tiny_k4v4_4k"]


def small(kb=4, vb=4, heads=8, kv=2, ctx=4096, batch=1, topk=64, planted=16, seed=0,
          lognormal=False):
    return W.Workload(f"small_k{kb}v{vb}_g{heads // kv}", batch=batch, heads=heads, kv_heads=kv,
                      ctx=ctx, key_bits=kb, val_bits=vb, topk=topk, planted=planted, seed=seed,
                      value_lognormal=lognormal)


def check_pack(run: DeviceRun):
    oc = run.oracle_cache()
    torch.cuda.synchronize()
    w = run.w
    for b in range(w.batch):
        for h in range(w.kv_heads):
            for g in range(oc.n_quant // 64):
                kc, ks, kz, vc, vs, vz = _lib.jfa_unpack_record(w.key_bits, w.val_bits,
                                                               run.cache.record(b, h, g))
                sl = slice(64 * g, 64 * g + 64)
                assert np.array_equal(kc, oc.k_codes[b, h, sl]), (b, h, g, "key codes")
                assert np.array_equal(ks, oc.k_scale[b, h, g].view(np.uint16)), (b, h, g)
                assert np.array_equal(kz, oc.k_zero[b, h, g].view(np.uint16)), (b, h, g)
                assert np.array_equal(vc, oc.v_codes[b, h, sl]), (b, h, g, "value codes")
                assert np.array_equal(vs, oc.v_scale[b, h, sl].view(np.uint16)), (b, h, g)
                assert np.array_equal(vz, oc.v_zero[b, h, sl].view(np.uint16)), (b, h, g)
    t = run.ctx - oc.n_quant
    tk = run.cache.tail_k[:, :, :t].cpu()
    tv = run.cache.tail_v[:, :, :t].cpu()
    assert torch.equal(tk, run.k_cpu[:, :, oc.n_quant:run.ctx])
    assert torch.equal(tv, run.v_cpu[:, :, oc.n_quant:run.ctx])


# ---------------------------------------------------------------- pack
@pytest.mark.parametrize("kb,vb", [(4, 4), (3, 2), (3, 4), (4, 2)])
def test_pack_bulk_bit_exact(kb, vb):
    w = small(kb, vb, ctx=1000, batch=2, lognormal=True)
    check_pack(DeviceRun(w))


def test_pack_appends_equal_bulk():
    # ragged appends crossing group and tail boundaries, including 1-token steps
    w = small(3, 2, ctx=777, batch=2)
    chunks = [1, 63, 1, 64, 65, 2, 1, 200, 127, 129, 64, 60]
    assert sum(chunks) == 777
    check_pack(DeviceRun(w, chunks=chunks))


def test_pack_single_token_appends():
    w = small(4, 4, ctx=200)
    check_pack(DeviceRun(w, chunks=[1] * 200))


# ---------------------------------------------------------------- scores
def scan_partials(run: DeviceRun):
    """Merge the scan's split partials on the host (log2 units)."""
    g = run.cache.geom()
    w = run.w
    nq = run.cache.n_quant
    ng = nq // 64
    n_seg = w.batch * w.kv_heads
    T = n_seg * ng
    Wn = _lib.jfa_scan_warps(g)  # warp w covers flattened groups [w T / Wn, (w + 1) T / Wn)
    assert 1 <= Wn <= min(T, 4096)
    L = run.ws.layout
    G = w.group
    part = run.ws.buf[L.off_partials:L.off_partials + 4 * L.partial_slots * G * 132]
    part = part.view(torch.float32).view(L.partial_slots, G, 132).cpu().double().numpy()
    res = {}
    for seg in range(n_seg):
        x0, x1 = seg * ng, seg * ng + ng - 1
        w0, w1 = ((x0 + 1) * Wn - 1) // T, ((x1 + 1) * Wn - 1) // T
        for j in range(G):
            m, l, acc = -np.inf, 0.0, np.zeros(128)
            for wi in range(w0, w1 + 1):
                row = part[wi + seg, j]
                mn = max(m, row[0])
                l = l * 2.0 ** (m - mn) + row[1] * 2.0 ** (row[0] - mn)
                acc = acc * 2.0 ** (m - mn) + row[4:] * 2.0 ** (row[0] - mn)
                m = mn
            res[(seg // w.kv_heads, (seg % w.kv_heads) * G + j)] = (m, l, acc)
    return res


@pytest.mark.parametrize("kb,vb,heads,kv", [(4, 4, 8, 2), (3, 2, 8, 2), (3, 2, 32, 8),
                                            (4, 4, 32, 4), (3, 4, 8, 8), (4, 2, 4, 2)])
def test_scores_and_scan_partials(kb, vb, heads, kv):
    w = small(kb, vb, heads=heads, kv=kv, ctx=2100, batch=2, lognormal=True)
    run = DeviceRun(w)
    run.scores()
    s_gpu = run.selection_scores()
    ref = run.oracle_step()
    err = np.abs(s_gpu - ref.select).max()
    assert err <= SCORE_ABS, err
    parts = scan_partials(run)
    for (b, hq), (m, l, acc) in parts.items():
        pa = ref.approx_all[b][hq]
        # The scan feeds each weight to the value MMAs as fp16(p) and fp16(p * s_v):
        # two round-to-nearest steps of relative error <= 2^-11 each, so the
        # aggregate and the mass are within 2^-10 relative of the fp64 values.
        want = O.finish(pa)
        tol = 2.0 ** -10 * 2 * max(1.0, np.abs(want).max())
        assert np.abs(acc / l - want).max() <= tol
        assert abs(m / np.log2(np.e) - pa.m) < 1e-4
        assert abs(l * 2.0 ** (m - pa.m * np.log2(np.e)) / pa.l - 1) < 2.0 ** -10


# ---------------------------------------------------------------- top-k
def write_scores(run: DeviceRun, s: np.ndarray):
    v = run.ws.scores(run.cache)
    v[:, :, :s.shape[2]] = torch.from_numpy(s.astype(np.float32)).cuda()


@pytest.mark.parametrize("nq_ctx,k,mode", [(4096, 64, "normal"), (4096, 1, "normal"),
                                           (32768, 256, "normal"), (32768, 4096, "normal"),
                                           (131072, 512, "normal"), (8192, 300, "ties"),
                                           (40000, 100, "constant"), (70000, 2000, "few_values"),
                                           (4096, 4031, "normal")])
def test_topk_bit_exact_on_synthetic_scores(nq_ctx, k, mode):
    w = small(4, 4, ctx=nq_ctx, batch=2, heads=8, kv=4)
    run = DeviceRun(w, k=k, chunks=[nq_ctx], kv=(torch.zeros(2, 4, nq_ctx, 128, dtype=torch.bfloat16),
                                              torch.zeros(2, 4, nq_ctx, 128, dtype=torch.bfloat16)))
    nq = run.cache.n_quant
    rng = np.random.default_rng(nq_ctx + k)
    if mode == "normal":
        s = rng.standard_normal((2, 4, nq)) * 2
    elif mode == "ties":
        s = np.round(rng.standard_normal((2, 4, nq)) * 4) / 4
    elif mode == "constant":     # every score equal: the lowest indices win; candidates overflow
        s = np.full((2, 4, nq), 1.5)
    else:                        # few distinct values, heavy ties at the threshold
        s = rng.integers(0, 5, (2, 4, nq)).astype(np.float64) - 2.0
    s = s.astype(np.float32)
    write_scores(run, s)
    run.topk()
    got = run.idx.cpu().numpy()
    ref = O.topk_indices(s.astype(np.float64), k)
    assert np.array_equal(got, ref)


def test_topk_k_at_least_nq_fills():
    w = small(4, 4, ctx=300)
    run = DeviceRun(w, k=300)
    run.topk()
    got = run.idx.cpu().numpy()
    nq = run.cache.n_quant
    assert np.array_equal(got[0, 0], np.r_[np.arange(nq), -np.ones(300 - nq)])


# ---------------------------------------------------------------- correct + merge
@pytest.mark.parametrize("kb,vb,heads,kv,ctx,k", [(4, 4, 8, 2, 4096, 64), (3, 2, 32, 8, 3000, 128),
                                                  (3, 2, 32, 4, 2048, 256), (4, 4, 8, 8, 1000, 7),
                                                  (4, 2, 4, 1, 777, 33)])
def test_correct_merge_with_oracle_index_set(kb, vb, heads, kv, ctx, k):
    w = small(kb, vb, heads=heads, kv=kv, ctx=ctx, batch=2, topk=k, lognormal=True)
    run = DeviceRun(w)
    ref = run.oracle_step()
    run.scores()
    oidx = torch.from_numpy(ref.idx.astype(np.int32)).cuda()
    run.correct_merge(oidx)
    torch.cuda.synchronize()
    assert_out_close(run.out.cpu().numpy(), ref.out)


@pytest.mark.parametrize("wl", ["tiny_k4v4_4k"])
def test_end_to_end_tiny_workload(wl):
    w = W.WORKLOADS[wl]
    run = DeviceRun(w)
    out, idx = run.step()
    ref = run.oracle_step()
    assert_topk_valid(idx, ref.select, w.topk)
    assert_out_close(out, run.oracle_step(idx=idx).out)
    assert_out_close(out, ref.out)
    # planted tokens are found
    pos = set(W.planted_positions(w, 0).tolist())
    for h in range(w.kv_heads):
        assert pos <= set(idx[0, h].tolist())


@pytest.mark.parametrize("kb,vb,heads,kv,ctx,k,batch", [(3, 2, 32, 8, 5000, 256, 2),
                                                        (4, 4, 32, 4, 4500, 96, 3),
                                                        (3, 2, 64, 8, 3333, 256, 1)])
def test_end_to_end_no_planted(kb, vb, heads, kv, ctx, k, batch):
    # without planted tokens the bulk of the distribution carries the output
    w = small(kb, vb, heads=heads, kv=kv, ctx=ctx, batch=batch, topk=k, planted=0, seed=5)
    run = DeviceRun(w)
    out, idx = run.step()
    ref = run.oracle_step()
    assert_topk_valid(idx, ref.select, k)
    assert_out_close(out, run.oracle_step(idx=idx).out)
    assert_out_close(out, ref.out)


def test_host_resident_rows_match_device_rows():
    w = small(4, 4, heads=32, kv=8, ctx=3000, batch=2, topk=128)
    a = DeviceRun(w)
    b = DeviceRun(w, exact_on_host=True)
    oa, ia = a.step()
    ob, ib = b.step()
    assert np.array_equal(ia, ib)
    assert np.array_equal(oa, ob)


def test_output_in_pinned_host_memory():
    # the finishing kernel writes out straight into pinned host memory
    w = small(3, 2, heads=32, kv=8, ctx=3000, batch=2, topk=128)
    run = DeviceRun(w)
    od, idd = run.fused_step()
    out_h = torch.full(tuple(run.out.shape), float("nan"), dtype=torch.float32).pin_memory()
    idx = torch.empty_like(run.idx)
    _lib.check(_lib.jfa_decode_step(run.cache.geom(), run.cache.struct(), run.q, run.scale, run.k,
                                    idx, run.k_exact, run.v_exact, run.exact_on_host, run.ws.buf,
                                    out_h), "decode_step")
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idd)
    assert np.array_equal(out_h.double().numpy(), od)


def test_decode_graph_replay_equals_eager_step():
    w = small(3, 2, heads=32, kv=8, ctx=5000, batch=2, topk=128)
    run = DeviceRun(w)
    od, idd = run.fused_step()
    q = run.q.clone()
    graph = jfa.DecodeGraph(run.cache, q, run.k, run.k_exact, run.v_exact, run.ws,
                            scale=run.scale, exact_on_host=bool(run.exact_on_host))
    for _ in range(3):
        out, idx = graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idd)
    assert np.array_equal(out.cpu().double().numpy(), od)
    # a new query written into the captured q buffer is picked up by the next replay
    q.copy_(torch.flip(run.q, dims=[1]))
    out, idx = graph.replay()
    torch.cuda.synchronize()
    ref = jfa.decode_step(run.cache, q, run.k, run.k_exact, run.v_exact, run.ws, scale=run.scale,
                          exact_on_host=bool(run.exact_on_host))
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), ref[1].cpu().numpy())
    assert np.array_equal(out.cpu().numpy(), ref[0].cpu().numpy())


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    # a wait that nothing completes ends after ~1 s with the timeout flag set
    w = small(3, 2, heads=8, kv=2, ctx=3000, batch=1, topk=64)
    run = DeviceRun(w)
    g = run.cache.geom()
    _lib.check(_lib.jfa_clear_error(g, run.ws.buf), "clear")
    _lib.check(_lib.jfa_selftest_bounded_wait(g, run.ws.buf), "selftest")
    st, flag = _lib.jfa_check_error(g, run.ws.buf)
    assert flag == _lib.DEVERR_TIMEOUT and st == _lib.JFA_ERR_DEVICE
    _lib.check(_lib.jfa_clear_error(g, run.ws.buf), "clear")
    out, idx = run.fused_step()  # asserts a clear flag itself
    assert_out_close(out, run.oracle_step(idx=idx).out)


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("ctx", [1, 37, 64, 65, 127, 128, 129, 191])
def test_short_contexts(ctx):
    w = small(3, 2, heads=8, kv=2, ctx=ctx, batch=2, topk=16, planted=0)
    run = DeviceRun(w)
    out, idx = run.step()
    ref = run.oracle_step()
    assert np.array_equal(idx, ref.idx)
    assert_out_close(out, ref.out)


def test_k_at_least_nq_is_exact_attention():
    w = small(4, 4, heads=8, kv=2, ctx=700, batch=1, topk=700)
    run = DeviceRun(w)
    out, idx = run.step()
    ref = O.exact_attention(run.q_cpu.double().numpy(), run.k_cpu.double().numpy(),
                            run.v_cpu.double().numpy(), 700, run.scale)
    assert_out_close(out, ref)


def test_bad_index_sets_device_flag_without_fault():
    w = small(4, 4, ctx=600, topk=8)
    run = DeviceRun(w)
    run.scores()
    bad = torch.full((1, 2, 8), -1, dtype=torch.int32, device="cuda")
    bad[0, 0, 0] = 10_000_000
    bad[0, 1, 0] = 5
    run.correct_merge(bad)
    st, flag = _lib.jfa_check_error(run.cache.geom(), run.ws.buf)
    assert st == _lib.JFA_ERR_DEVICE and flag & _lib.DEVERR_BAD_INDEX
    _lib.check(_lib.jfa_clear_error(run.cache.geom(), run.ws.buf), "clear")
    st, flag = _lib.jfa_check_error(run.cache.geom(), run.ws.buf)
    assert st == 0 and flag == 0


def test_capacity_larger_than_context():
    w = small(3, 2, heads=32, kv=8, ctx=1500, batch=2, topk=100)
    run = DeviceRun(w, capacity=4096)
    out, idx = run.step()
    ref = run.oracle_step()
    assert_topk_valid(idx, ref.select, 100)
    assert_out_close(out, run.oracle_step(idx=idx).out)


# ---------------------------------------------------------------- fused step
@pytest.mark.parametrize("kb,vb,heads,kv,ctx,k,batch", [
    (4, 4, 8, 2, 4096, 64, 1), (3, 2, 32, 8, 5000, 256, 2), (4, 4, 32, 4, 9000, 512, 1),
    (3, 2, 8, 8, 2100, 33, 3), (4, 2, 64, 8, 3333, 256, 2), (3, 4, 4, 1, 700, 700, 2),
    (3, 2, 32, 8, 100, 16, 2), (4, 4, 8, 2, 64, 8, 1), (3, 2, 32, 8, 40000, 4096, 1)])
def test_fused_step_matches_separate_calls(kb, vb, heads, kv, ctx, k, batch):
    w = small(kb, vb, heads=heads, kv=kv, ctx=ctx, batch=batch, topk=k, lognormal=True)
    run = DeviceRun(w)
    out3, idx3 = run.step()
    out1, idx1 = run.fused_step()
    assert np.array_equal(idx1, idx3)
    assert np.allclose(out1, out3, rtol=1e-5, atol=1e-6)
    ref = run.oracle_step()
    assert_topk_valid(idx1, ref.select, k)
    assert_out_close(out1, run.oracle_step(idx=idx1).out)


@pytest.mark.parametrize("kb,vb,heads,kv", [(3, 2, 8, 2), (4, 4, 32, 4)])
def test_long_segments_sixteen_cta_clusters(kb, vb, heads, kv):
    # few segments of >= 16K quantized tokens: the finishing kernel runs
    # clusters of 16 CTAs; it must agree with the separate calls and the oracle
    w = small(kb, vb, heads=heads, kv=kv, ctx=20000, batch=1, topk=384, planted=32)
    run = DeviceRun(w)
    out3, idx3 = run.step()
    out1, idx1 = run.fused_step()
    assert np.array_equal(idx1, idx3)
    assert np.allclose(out1, out3, rtol=1e-5, atol=1e-6)
    assert_topk_valid(idx1, run.oracle_step().select, w.topk)
    assert_out_close(out1, run.oracle_step(idx=idx1).out)


def test_fused_step_tiny_workload_against_oracle():
    w = W.WORKLOADS["tiny_k4v4_4k"]
    run = DeviceRun(w)
    out, idx = run.fused_step()
    ref = run.oracle_step()
    assert_topk_valid(idx, ref.select, w.topk)
    assert_out_close(out, ref.out)


def test_whole_segment_fallback_selection():
    # scan once, then run the finishing kernel twice: the first consumes and
    # clears the scan's score histogram, so the second must select over the
    # whole segment from the stored scores (the fallback path); both choices
    # equal the bit-exact top-k of those scores
    w = small(3, 2, heads=32, kv=8, ctx=9000, batch=2, topk=256, lognormal=True)
    run = DeviceRun(w)
    run.scores()
    g, cs = run.cache.geom(), run.cache.struct()
    outs = []
    for _ in range(2):
        out = torch.empty_like(run.out)
        idx = torch.empty_like(run.idx)
        _lib.check(_lib.jfa_decode_finish(g, cs, run.q, run.scale, run.k, idx, run.k_exact,
                                          run.v_exact, 0, run.ws.buf, out), "finish")
        torch.cuda.synchronize()
        outs.append((out.cpu().double().numpy(), idx.cpu().numpy()))
    assert run.ws.error_flag(run.cache) == 0
    s_gpu = run.selection_scores()
    want = O.topk_indices(s_gpu, run.k)
    for out, idx in outs:
        assert np.array_equal(idx, want)
        assert_out_close(out, run.oracle_step(idx=idx).out)
    # the two paths spread the correction differently over the cluster: fp32
    # sums in another order
    assert np.allclose(outs[0][0], outs[1][0], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("ctx,k", [(20000, 4096), (6000, 1000)])
def test_all_scores_tied_picks_lowest_indices(ctx, k):
    # constant keys: every selection score is equal, so the chosen set is the
    # k lowest indices; the tie bin overflows every shared-memory list
    w = small(4, 4, heads=32, kv=8, ctx=ctx, batch=1, topk=k, planted=0)
    q = W.gen_q(w)
    kc = torch.full((1, 8, ctx, 128), 0.375, dtype=torch.bfloat16)
    vc = W.gen_kv(w, q, ctx)[1]
    run = DeviceRun(w, q=q, kv=(kc, vc))
    out, idx = run.fused_step()
    nq = run.cache.n_quant
    s_gpu = run.selection_scores()
    assert np.all(s_gpu == s_gpu[:, :, :1])   # equal within every (sequence, KV head) row
    want = np.broadcast_to(np.arange(k, dtype=np.int32), idx.shape)
    assert np.array_equal(idx, want)
    ref = run.oracle_step()
    assert np.array_equal(ref.idx, want)
    assert_out_close(out, ref.out)
