"""GPU parity of the critical-channel selection (TailorKV review) against the
fp64 oracle: the channel-major key copy and per-channel max|K| bit for bit;
selection scores within the fp32-accumulation bound; top-k sets bit for bit
on the GPU's own scores and within the tie window on the oracle's; outputs
of the exact attention over the chosen tokens and the tail within the output
tolerances."""
import math

import numpy as np
import pytest
import torch

import oracle.jfa_oracle as O
import workloads as W
from bit_kv_cache_jfa_b200 import _lib
import bit_kv_cache_jfa_b200 as jfa

from jfa_testutil import assert_out_close, assert_topk_valid

pytestmark = pytest.mark.gpu


class ChanRun:
    def __init__(self, batch, heads, kv, ctx, seed=0, lognormal=False, device_gen=False):
        self.w = W.Workload(f"ch_{heads}_{kv}_{ctx}", batch=batch, heads=heads, kv_heads=kv,
                            ctx=ctx, key_bits=4, val_bits=4, topk=64, planted=16, seed=seed,
                            value_lognormal=lognormal)
        self.ctx = ctx
        self.cap = max(64, 64 * math.ceil(ctx / 64))
        self.q_cpu = W.gen_q(self.w)
        self.q = self.q_cpu.cuda()
        shape = (batch, kv, self.cap, 128)
        self.k_dev = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        self.v_dev = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        if device_gen:
            kd, vd = W.gen_kv_device(self.w, "cuda", self.q_cpu, ctx)
            self.k_cpu = self.v_cpu = None
        else:
            kd, vd = W.gen_kv(self.w, self.q_cpu, ctx)
            self.k_cpu, self.v_cpu = kd, vd
        self.k_dev[:, :, :ctx], self.v_dev[:, :, :ctx] = kd.cuda(), vd.cuda()
        del kd, vd
        self.scale = 1.0 / math.sqrt(128)
        self.keys = jfa.ChannelKeys(batch, heads, kv, self.cap)
        self.ws = jfa.Workspace(self.keys, 4096)
        self.keys.sync(self.k_dev, ctx)
        self.nq = O.split_point(ctx)
        self.G = heads // kv

    def seg(self, b, h):
        if self.k_cpu is not None:
            return self.k_cpu[b, h].double().numpy(), self.v_cpu[b, h].double().numpy()
        return (self.k_dev[b, h, :self.ctx].cpu().double().numpy(),
                self.v_dev[b, h, :self.ctx].cpu().double().numpy())

    def q_seg(self, b, h):
        return self.q_cpu[b, h * self.G:(h + 1) * self.G].double().numpy()


def oracle_scores(run, b, h, r):
    """Oracle selection scores of one segment and a per-token bound of the
    fp32 accumulation (1e-5 of scale * sum over kept channels |q k|)."""
    k, _ = run.seg(b, h)
    q = run.q_seg(b, h)
    s = O.channel_scores(q[None], k[None, None], run.ctx, r, run.scale)[0, 0]
    c = O.critical_channels(O.channel_importance(q[None], k[None, None], run.nq), r)[0, 0]
    mag = run.scale * (np.abs(k[:run.nq][:, c]) @ np.abs(q[:, c]).T)
    return s, 1e-5 * mag.max(1) + 1e-7


@pytest.mark.parametrize("ctx", [1000, 4097])
def test_channel_copy_bit_exact(ctx):
    run = ChanRun(2, 8, 2, ctx, seed=1)
    kt = run.keys.k_t.cpu()
    km = run.keys.k_max.cpu().numpy()
    for b in range(2):
        for h in range(2):
            k = run.k_dev[b, h, :run.nq].cpu()
            assert torch.equal(kt[b, h, :, :run.nq], k.T)
            assert np.array_equal(km[b, h], k.float().abs().max(0).values.numpy())


@pytest.mark.parametrize("batch,heads,kv,ctx,r", [(2, 8, 2, 1000, 16), (1, 32, 8, 9000, 32),
                                                  (2, 64, 8, 3000, 8), (1, 24, 6, 777, 128),
                                                  (1, 32, 4, 129, 1)])
def test_channel_scores_against_oracle(batch, heads, kv, ctx, r):
    run = ChanRun(batch, heads, kv, ctx, seed=3)
    _lib.check(_lib.jfa_channel_scores(run.keys.geom(ctx), run.keys.k_t, run.keys.k_max, run.q,
                                       run.scale, r, run.ws.buf), "channel_scores")
    torch.cuda.synchronize()
    s = run.ws.scores(run.keys)[:, :, :run.nq].cpu().double().numpy()
    for b in range(batch):
        for h in range(kv):
            ref, tol = oracle_scores(run, b, h, r)
            assert np.all(np.abs(s[b, h] - ref) <= tol), (b, h)


@pytest.mark.parametrize("batch,heads,kv,ctx,r,k", [
    (2, 8, 2, 1000, 16, 64), (1, 32, 8, 9000, 32, 256), (2, 64, 8, 3000, 8, 128),
    (1, 32, 4, 20000, 16, 1024), (2, 8, 2, 65, 16, 64), (1, 8, 2, 1, 16, 8),
    (1, 24, 6, 777, 128, 100)])
def test_channel_step_against_oracle(batch, heads, kv, ctx, r, k):
    run = ChanRun(batch, heads, kv, ctx, seed=5, lognormal=True)
    out, idx = jfa.channel_decode_step(run.keys, ctx, run.q, r, k, run.k_dev, run.v_dev, run.ws,
                                       scale=run.scale)
    torch.cuda.synchronize()
    assert run.ws.error_flag(run.keys) == 0
    idx = idx.cpu().numpy()
    s_gpu = run.ws.scores(run.keys)[:, :, :run.nq].cpu().double().numpy()
    if run.nq:
        assert np.array_equal(idx, O.topk_indices(s_gpu, k))
    got = out.cpu().double().numpy()
    for b in range(batch):
        for h in range(kv):
            kk, vv = run.seg(b, h)
            q = run.q_seg(b, h)
            if run.nq:
                ref_s, _ = oracle_scores(run, b, h, r)
                assert_topk_valid(idx[b:b + 1, h:h + 1], ref_s[None, None], k)
            ref = O.attend_set(q[None], kk[None, None], vv[None, None], ctx,
                               idx[b:b + 1, h:h + 1], run.scale)
            assert_out_close(got[b, h * run.G:(h + 1) * run.G], ref[0])


def test_channel_full_size_llama8b_sampled():
    # Llama-3.1-8B-shaped layer: batch 4, 32 query / 8 KV heads, 32K
    # context, 16 critical channels, top-k 256
    run = ChanRun(4, 32, 8, 32768, seed=7, device_gen=True)
    out, idx = jfa.channel_decode_step(run.keys, run.ctx, run.q, 16, 256, run.k_dev, run.v_dev,
                                       run.ws, scale=run.scale)
    torch.cuda.synchronize()
    assert run.ws.error_flag(run.keys) == 0
    s_gpu = run.ws.scores(run.keys)[:, :, :run.nq].cpu().double().numpy()
    idx = idx.cpu().numpy()
    got = out.cpu().double().numpy()
    for b, h in W.sample_segments(run.w, 4, seed=2):
        ref_s, tol = oracle_scores(run, b, h, 16)
        assert np.all(np.abs(s_gpu[b, h] - ref_s) <= tol)
        assert np.array_equal(idx[b, h], O.topk_indices(s_gpu[b:b + 1, h:h + 1], 256)[0, 0])
        assert_topk_valid(idx[b:b + 1, h:h + 1], ref_s[None, None], 256)
        kk, vv = run.seg(b, h)
        ref = O.attend_set(run.q_seg(b, h)[None], kk[None, None], vv[None, None], run.ctx,
                           idx[b:b + 1, h:h + 1], run.scale)
        assert_out_close(got[b, 4 * h:4 * h + 4], ref[0])
