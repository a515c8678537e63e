"""GPU parity of the 1-bit KV cache with dense attention (TailorKV review)
against the fp64 oracle: codes and fp16 scale / zero bits of every record bit
for bit (decoded in the test), outputs of the dense attention over the
dequantized tokens and the exact tail within the output tolerances."""
import math

import numpy as np
import pytest
import torch

import oracle.jfa_oracle as O
import workloads as W
from bit_kv_cache_jfa_b200 import _lib
import bit_kv_cache_jfa_b200 as jfa

from jfa_testutil import assert_out_close

pytestmark = pytest.mark.gpu

REC = 3584


def decode_record(rec):
    """(key codes [64 tok][128], key scale/zero fp16 bits [128], value codes
    [64][128], value scale/zero fp16 bits [64][4]) of one record."""
    rec = np.asarray(rec, dtype=np.uint8)
    kw = rec[:1024].view(np.uint64)                               # per channel, bit t
    kc = ((kw[None, :] >> np.arange(64, dtype=np.uint64)[:, None]) & np.uint64(1)).astype(np.uint8)
    ks = rec[1024:1280].view(np.uint16)
    kz = rec[1280:1536].view(np.uint16)
    vw = rec[1536:2560].view(np.uint32).reshape(64, 4)           # word j bit i = channel 32 j + i
    vc = ((vw[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(64, 128).astype(np.uint8)
    vs = rec[2560:3072].view(np.uint16).reshape(64, 4)
    vz = rec[3072:3584].view(np.uint16).reshape(64, 4)
    return kc, ks, kz, vc, vs, vz


class OneBitRun:
    def __init__(self, batch, heads, kv, ctx, seed=0, lognormal=False, exact_on_host=False,
                 device_gen=False):
        self.w = W.Workload(f"b1_{heads}_{kv}_{ctx}", batch=batch, heads=heads, kv_heads=kv,
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
        if exact_on_host:
            self.k_exact = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
            self.v_exact = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
            self.k_exact.copy_(self.k_dev)
            self.v_exact.copy_(self.v_dev)
        else:
            self.k_exact, self.v_exact = self.k_dev, self.v_dev
        self.on_host = exact_on_host
        self.scale = 1.0 / math.sqrt(128)
        self.cache = jfa.OneBitCache(batch, heads, kv, self.cap)
        self.ws = jfa.Workspace(self.cache, 64)
        self.cache.sync(self.k_dev, self.v_dev, ctx, self.ws)
        self.nq = O.split_point(ctx)
        self.G = heads // kv

    def seg(self, b, h):
        if self.k_cpu is not None:
            return self.k_cpu[b, h].double().numpy(), self.v_cpu[b, h].double().numpy()
        return (self.k_dev[b, h, :self.ctx].cpu().double().numpy(),
                self.v_dev[b, h, :self.ctx].cpu().double().numpy())

    def attend(self):
        out = jfa.onebit_attend(self.cache, self.ctx, self.q, self.k_exact, self.v_exact, self.ws,
                                scale=self.scale, exact_on_host=self.on_host)
        torch.cuda.synchronize()
        assert self.ws.error_flag(self.cache) == 0
        return out.cpu().double().numpy()

    def oracle_seg(self, b, h):
        k, v = self.seg(b, h)
        q = self.q_cpu[b, h * self.G:(h + 1) * self.G].double().numpy()
        c = O.pack_cache(k[None, None], v[None, None], self.ctx, 1, 1)
        return O.decode_step(q[None], k[None, None], v[None, None], c, 0, self.scale).out[0], c


@pytest.mark.parametrize("ctx", [1000, 200])
def test_onebit_pack_bit_exact(ctx):
    run = OneBitRun(2, 8, 2, ctx, seed=3)
    pool = run.cache.pool.cpu().numpy().reshape(2, 2, run.cap // 64, REC)
    for b in range(2):
        for h in range(2):
            k, v = run.seg(b, h)
            c = O.pack_cache(k[None, None], v[None, None], ctx, 1, 1)
            for g in range(run.nq // 64):
                kc, ks, kz, vc, vs, vz = decode_record(pool[b, h, g])
                t = slice(64 * g, 64 * g + 64)
                assert np.array_equal(kc, c.k_codes[0, 0, t]), (b, h, g)
                assert np.array_equal(ks, c.k_scale[0, 0, g].view(np.uint16)), (b, h, g)
                assert np.array_equal(kz, c.k_zero[0, 0, g].view(np.uint16)), (b, h, g)
                assert np.array_equal(vc, c.v_codes[0, 0, t]), (b, h, g)
                assert np.array_equal(vs, c.v_scale[0, 0, t].view(np.uint16)), (b, h, g)
                assert np.array_equal(vz, c.v_zero[0, 0, t].view(np.uint16)), (b, h, g)


@pytest.mark.parametrize("batch,heads,kv,ctx,host", [
    (2, 8, 2, 1000, False), (1, 32, 8, 9000, False), (2, 64, 8, 3000, False),
    (1, 32, 4, 20000, False), (2, 8, 2, 65, False), (1, 8, 2, 1, False), (2, 8, 4, 129, False),
    (1, 24, 6, 777, False), (2, 32, 8, 5000, True)])
def test_onebit_attend_against_oracle(batch, heads, kv, ctx, host):
    run = OneBitRun(batch, heads, kv, ctx, seed=5, lognormal=True, exact_on_host=host)
    got = run.attend()
    for b in range(batch):
        for h in range(kv):
            ref, _ = run.oracle_seg(b, h)
            assert_out_close(got[b, h * run.G:(h + 1) * run.G], ref)


def test_onebit_full_size_llama8b_sampled():
    # Llama-3.1-8B-shaped layer: batch 4, 32 query / 8 KV heads, 32K context
    run = OneBitRun(4, 32, 8, 32768, seed=7, device_gen=True)
    got = run.attend()
    for b, h in W.sample_segments(run.w, 3, seed=3):
        ref, _ = run.oracle_seg(b, h)
        assert_out_close(got[b, h * run.G:(h + 1) * run.G], ref)
