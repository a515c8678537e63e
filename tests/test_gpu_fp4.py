"""GPU parity of the NVFP4 path (Jet-QSparse abstract) against the fp64
oracle: packed codes, block scales and group scales bit for bit; FP4 scores
within the fp32-accumulation bound; block sets bit for bit on the GPU's own
scores and within the tie window on the oracle's; outputs of the sparse
exact attention within the output tolerances."""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle.jfa_oracle as O
import workloads as W
from bit_kv_cache_jfa_b200 import _lib
import bit_kv_cache_jfa_b200 as jfa

from jfa_testutil import TIE_WINDOW, assert_out_close

pytestmark = pytest.mark.gpu

REC = 9232


# --------------------------------------------------------------------------
# the record layout, restated for the test (rows = tokens of a 128-block)
# --------------------------------------------------------------------------
_r, _c = np.meshgrid(np.arange(128), np.arange(0, 128, 2), indexing="ij")
_CODE_OFF = (((_r >> 3) << 2) + (_c >> 5)) * 128 + (_r & 7) * 16 + (_c & 31) // 2
_r8, _j8 = np.meshgrid(np.arange(128), np.arange(8), indexing="ij")
_SF_OFF = 8192 + (_j8 >> 2) * 512 + (_r8 & 31) * 16 + (_r8 >> 5) * 4 + (_j8 & 3)


def decode_record(rec):
    """(codes uint8 [128, 128], block scales fp64 [128, 8], group scales [2])."""
    rec = np.asarray(rec, dtype=np.uint8)
    byte = rec[_CODE_OFF]
    codes = np.empty((128, 128), np.uint8)
    codes[:, 0::2] = byte & 15
    codes[:, 1::2] = byte >> 4
    bs = rec[_SF_OFF].view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    gs = rec[9216:9224].view(np.float32).astype(np.float64)
    return codes, bs, gs


def cap128(n):
    return max(128, 128 * math.ceil(n / 128))


class Fp4Run:
    def __init__(self, batch, heads, kv, ctx, seed=0, planted=16, lognormal=False,
                 exact_on_host=False, device_gen=False):
        self.w = W.Workload(f"fp4_{heads}_{kv}_{ctx}", batch=batch, heads=heads, kv_heads=kv,
                            ctx=ctx, key_bits=4, val_bits=4, topk=64, planted=planted, seed=seed,
                            value_lognormal=lognormal)
        self.ctx, self.cap = ctx, cap128(ctx)
        self.q_cpu = W.gen_q(self.w)
        self.q = self.q_cpu.cuda()
        shape = (batch, kv, self.cap, 128)
        if device_gen:
            kd, vd = W.gen_kv_device(self.w, "cuda", self.q_cpu, ctx)
            self.k_dev = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
            self.v_dev = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
            self.k_dev[:, :, :ctx], self.v_dev[:, :, :ctx] = kd, vd
            del kd, vd
            self.k_cpu = self.v_cpu = None
        else:
            k, v = W.gen_kv(self.w, self.q_cpu, ctx)
            self.k_cpu, self.v_cpu = k, v
            self.k_dev = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
            self.v_dev = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
            self.k_dev[:, :, :ctx], self.v_dev[:, :, :ctx] = k.cuda(), v.cuda()
        if exact_on_host:
            self.k_exact = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
            self.v_exact = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
            self.k_exact.copy_(self.k_dev)
            self.v_exact.copy_(self.v_dev)
        else:
            self.k_exact, self.v_exact = self.k_dev, self.v_dev
        self.on_host = exact_on_host
        self.scale = 1.0 / math.sqrt(128)
        self.pool = jfa.FP4KeyPool(batch, heads, kv, self.cap)
        self.ws = jfa.Workspace(self.pool, 64)
        self.pool.sync(self.k_dev, ctx, self.ws)
        self.nq = O.split_point(ctx)

    def geom(self):
        return self.pool.geom(self.ctx)

    def scores(self):
        _lib.check(_lib.jfa_fp4_scores(self.geom(), self.pool.pool, self.q, self.scale,
                                       self.ws.buf), "fp4_scores")
        torch.cuda.synchronize()
        return self.ws.scores(self.pool)[:, :, :self.nq].cpu().double().numpy()

    def seg_kv(self, b, h):
        if self.k_cpu is not None:
            return self.k_cpu[b, h].double().numpy(), self.v_cpu[b, h].double().numpy()
        return (self.k_dev[b, h, :self.ctx].cpu().double().numpy(),
                self.v_dev[b, h, :self.ctx].cpu().double().numpy())


def oracle_seg_scores(run, b, h):
    """Oracle selection scores of one segment and the per-token bound of the
    fp32 accumulation (2e-5 of scale * sum |q_hat k_hat|, largest head)."""
    k, _ = run.seg_kv(b, h)
    G = run.w.heads // run.w.kv_heads
    q = run.q_cpu[b, h * G:(h + 1) * G].double().numpy()
    s = O.nvfp4_scores(q[None], k[None, None], run.ctx, run.scale)[0]      # [G, nq]
    kh = O.nvfp4_keys(k, run.nq)
    qh = np.stack([O.nvfp4_dequantize(*O.nvfp4_quantize(q[j][None]))[0] for j in range(G)])
    mag = run.scale * (np.abs(kh) @ np.abs(qh).T)                             # [nq, G]
    return s.max(0), 2e-5 * mag.max(1) + 1e-6 * np.abs(s).max(0)


def assert_blocks_valid(idx, sel, n_blocks, window=TIE_WINDOW):
    bs = O.block_scores(sel[None])[0]
    ref = O.topk_blocks(sel[None], n_blocks)[0]
    got = set((idx[idx >= 0] // 128).tolist())
    want = set((ref[ref >= 0] // 128).tolist())
    if bs.size == 0:
        assert not got
        return
    kth = np.sort(bs)[-min(n_blocks, bs.size)]
    for blk in got ^ want:
        assert abs(bs[blk] - kth) <= window, (blk, bs[blk], kth)


# --------------------------------------------------------------------------
@pytest.mark.parametrize("ctx", [1000, 4097, 200])
def test_fp4_pack_bit_exact(ctx):
    run = Fp4Run(2, 8, 2, ctx, seed=3)
    pool = run.pool.pool.cpu().numpy().reshape(2, 2, run.cap // 128, REC)
    for b in range(2):
        for h in range(2):
            k, _ = run.seg_kv(b, h)
            for g in range(run.nq // 64):
                codes, bs, s = O.nvfp4_quantize(k[64 * g:64 * g + 64])
                gc, gb, gs = decode_record(pool[b, h, g // 2])
                rows = slice(64 * (g % 2), 64 * (g % 2) + 64)
                assert np.array_equal(gc[rows], codes), (b, h, g)
                assert np.array_equal(gb[rows], bs), (b, h, g)
                assert gs[g % 2] == s, (b, h, g)
            if run.nq % 128 == 64:      # the half of the last record not yet packed
                assert not pool[b, h, run.nq // 128, :8192].reshape(16, 4, 8, 16)[8:].any()


@pytest.mark.parametrize("batch,heads,kv,ctx", [(2, 8, 2, 1000), (1, 32, 4, 9000),
                                                (2, 64, 8, 3000), (1, 32, 8, 129)])
def test_fp4_scores_against_oracle(batch, heads, kv, ctx):
    run = Fp4Run(batch, heads, kv, ctx, seed=5)
    s = run.scores()
    for b in range(batch):
        for h in range(kv):
            ref, tol = oracle_seg_scores(run, b, h)
            err = np.abs(s[b, h] - ref)
            assert np.all(err <= tol), (b, h, float((err - tol).max()))


@pytest.mark.parametrize("batch,heads,kv,ctx,n_blocks", [
    (2, 8, 2, 1000, 3), (1, 32, 4, 9000, 16), (2, 64, 8, 3000, 30), (1, 32, 8, 20000, 64),
    (2, 8, 2, 65, 1), (1, 8, 2, 1, 1), (2, 8, 4, 129, 2), (1, 8, 2, 4096, 40),
    (1, 24, 6, 777, 2)])
def test_fp4_step_against_oracle(batch, heads, kv, ctx, n_blocks):
    run = Fp4Run(batch, heads, kv, ctx, seed=7, lognormal=True)
    out, idx = jfa.fp4_decode_step(run.pool, ctx, run.q, n_blocks, run.k_exact, run.v_exact,
                                   run.ws, scale=run.scale)
    torch.cuda.synchronize()
    assert run.ws.error_flag(run.pool) == 0
    idx = idx.cpu().numpy()
    s_gpu = run.ws.scores(run.pool)[:, :, :run.nq].cpu().double().numpy()
    assert np.array_equal(idx, O.topk_blocks(s_gpu, n_blocks))
    got = out.cpu().double().numpy()
    G = heads // kv
    for b in range(batch):
        for h in range(kv):
            k, v = run.seg_kv(b, h)
            if run.nq:
                ref_sel, _ = oracle_seg_scores(run, b, h)
                assert_blocks_valid(idx[b, h], ref_sel, n_blocks)
            q = run.q_cpu[b, h * G:(h + 1) * G].double().numpy()
            ref, _, _ = O.sparse_block_step(q[None], k[None, None], v[None, None], ctx, n_blocks,
                                            run.scale, idx=idx[b:b + 1, h:h + 1])
            assert_out_close(got[b, h * G:(h + 1) * G], ref[0])
    if run.nq and n_blocks * 128 >= run.nq:
        ref = O.exact_attention(run.q_cpu.double().numpy(), run.k_cpu.double().numpy(),
                                run.v_cpu.double().numpy(), ctx, run.scale)
        assert_out_close(got, ref)


@pytest.mark.parametrize("on_host", [False, True])
def test_sparse_attend_token_sets(on_host):
    # token-level index sets in any order, with unused (-1) entries
    run = Fp4Run(2, 32, 4, 5000, seed=9, exact_on_host=on_host)
    rng = np.random.default_rng(11)
    k = 300
    idx = np.full((2, 4, k), -1, np.int32)
    for b in range(2):
        for h in range(4):
            n = int(rng.integers(200, k + 1))
            idx[b, h, :n] = rng.choice(run.nq, n, replace=False)
    out = jfa.sparse_attend(run.geom(), run.q, torch.from_numpy(idx).cuda(), run.k_exact,
                            run.v_exact, run.ws, scale=run.scale, exact_on_host=on_host)
    torch.cuda.synchronize()
    assert run.ws.error_flag(run.pool) == 0
    got = out.cpu().double().numpy()
    for b in range(2):
        for h in range(4):
            k_, v_ = run.seg_kv(b, h)
            q = run.q_cpu[b, 8 * h:8 * h + 8].double().numpy()
            ref, _, _ = O.sparse_block_step(q[None], k_[None, None], v_[None, None], run.ctx, 0,
                                            run.scale, idx=idx[b:b + 1, h:h + 1])
            assert_out_close(got[b, 8 * h:8 * h + 8], ref[0])


def test_sparse_attend_flags_bad_index():
    run = Fp4Run(1, 8, 2, 1000, seed=2)
    idx = np.tile(np.arange(10, dtype=np.int32), (1, 2, 1))
    idx[0, 1, 3] = run.nq          # outside [0, N_q): flagged and skipped
    out = jfa.sparse_attend(run.geom(), run.q, torch.from_numpy(idx).cuda(), run.k_exact,
                            run.v_exact, run.ws, scale=run.scale)
    torch.cuda.synchronize()
    assert run.ws.error_flag(run.pool) == _lib.DEVERR_BAD_INDEX
    idx[0, 1, 3] = -1
    k_, v_ = run.seg_kv(0, 1)
    q = run.q_cpu[0, 4:8].double().numpy()
    ref, _, _ = O.sparse_block_step(q[None], k_[None, None], v_[None, None], run.ctx, 0, run.scale,
                                    idx=idx[:, 1:2])
    assert_out_close(out[0, 4:8].cpu().double().numpy(), ref[0])


def test_fp4_full_size_qwen_sampled():
    # Qwen3-30B-A3B-shaped layer: batch 16, 32 query / 4 KV heads, 32K
    # context, 64 blocks per KV head; sampled segments against the oracle
    run = Fp4Run(16, 32, 4, 32768, seed=13, planted=64, lognormal=True, device_gen=True)
    out, idx = jfa.fp4_decode_step(run.pool, run.ctx, run.q, 64, run.k_exact, run.v_exact, run.ws,
                                   scale=run.scale)
    torch.cuda.synchronize()
    assert run.ws.error_flag(run.pool) == 0
    s_gpu = run.ws.scores(run.pool)[:, :, :run.nq].cpu().double().numpy()
    idx = idx.cpu().numpy()
    got = out.cpu().double().numpy()
    for b, h in W.sample_segments(run.w, 3, seed=1):
        ref_sel, tol = oracle_seg_scores(run, b, h)
        assert np.all(np.abs(s_gpu[b, h] - ref_sel) <= tol)
        assert np.array_equal(idx[b, h], O.topk_blocks(s_gpu[b:b + 1, h:h + 1], 64)[0, 0])
        assert_blocks_valid(idx[b, h], ref_sel, 64)
        k, v = run.seg_kv(b, h)
        q = run.q_cpu[b, 8 * h:8 * h + 8].double().numpy()
        ref, _, _ = O.sparse_block_step(q[None], k[None, None], v[None, None], run.ctx, 64,
                                        run.scale, idx=idx[b:b + 1, h:h + 1])
        assert_out_close(got[b, 8 * h:8 * h + 8], ref[0])
