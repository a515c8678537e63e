"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle.jfa_oracle as O
import workloads as W
from bit_kv_cache_jfa_b200 import _lib
import bit_kv_cache_jfa_b200 as jfa

# Output tolerances against the fp64 oracle.
MAX_ABS = 2e-3
REL_L2 = 1e-3
TIE_WINDOW = 1e-3   # top-k indices whose oracle score is this close to the k-th may differ
# Selection scores (natural-log units).  A score error below half the tie
# window keeps every index whose oracle score lies outside the window on the
# same side of the k-th score, which is what the top-k criterion needs; the
# tensor-core fp32 accumulation over 128 channels (outlier channels included)
# stays well inside it.
SCORE_ABS = TIE_WINDOW / 2


def cap_for(ctx: int) -> int:
    return max(64, 64 * math.ceil(ctx / 64))


class DeviceRun:
    """One workload on the device: packed cache, exact copies, workspace."""

    def __init__(self, w: W.Workload, ctx: int | None = None, k: int | None = None,
                 chunks: list[int] | None = None, capacity: int | None = None,
                 exact_on_host: bool = False, q=None, kv=None):
        self.w = w
        self.ctx = w.ctx if ctx is None else ctx
        self.k = w.topk if k is None else k
        self.q_cpu = W.gen_q(w) if q is None else q
        if kv is None:
            kv = W.gen_kv(w, self.q_cpu, self.ctx)
        self.k_cpu, self.v_cpu = kv
        cap = cap_for(self.ctx) if capacity is None else capacity
        self.cache = jfa.KVCache(w.batch, w.heads, w.kv_heads, cap, w.key_bits, w.val_bits)
        self.ws = jfa.Workspace(self.cache, max(self.k, 1))
        kd, vd = self.k_cpu.cuda(), self.v_cpu.cuda()
        pos = 0
        for n in (chunks or [self.ctx]):
            if n == 0:
                continue
            self.cache.append(kd[:, :, pos:pos + n].contiguous(), vd[:, :, pos:pos + n].contiguous(),
                              self.ws)
            pos += n
        assert pos == self.ctx
        shape = (w.batch, w.kv_heads, cap, w.head_dim)
        self.exact_on_host = exact_on_host
        if exact_on_host:
            self.k_exact = torch.zeros(shape, dtype=torch.bfloat16, pin_memory=True)
            self.v_exact = torch.zeros(shape, dtype=torch.bfloat16, pin_memory=True)
        else:
            self.k_exact = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
            self.v_exact = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        self.k_exact[:, :, :self.ctx] = self.k_cpu
        self.v_exact[:, :, :self.ctx] = self.v_cpu
        self.q = self.q_cpu.cuda()
        self.scale = W.default_scale(w)
        self.out = torch.empty(w.batch, w.heads, w.head_dim, dtype=torch.float32, device="cuda")
        self.idx = torch.empty(w.batch, w.kv_heads, self.k, dtype=torch.int32, device="cuda")

    def scores(self):
        _lib.check(_lib.jfa_decode_scores(self.cache.geom(), self.cache.struct(), self.q,
                                          self.scale, self.ws.buf), "scores")

    def topk(self):
        _lib.check(_lib.jfa_topk(self.cache.geom(), self.k, self.ws.buf, self.idx), "topk")

    def correct_merge(self, idx=None):
        idx = self.idx if idx is None else idx
        _lib.check(_lib.jfa_correct_merge(self.cache.geom(), self.cache.struct(), self.q,
                                          self.scale, idx, self.k, self.k_exact, self.v_exact,
                                          self.exact_on_host, self.ws.buf, self.out),
                   "correct_merge")

    def step(self):
        self.scores()
        self.topk()
        self.correct_merge()
        torch.cuda.synchronize()
        st, flag = _lib.jfa_check_error(self.cache.geom(), self.ws.buf)
        assert flag == 0, f"device error flag {flag:#x}"
        return self.out.cpu().double().numpy(), self.idx.cpu().numpy()

    def fused_step(self):
        """jfa_decode_step (scan + fused finishing kernel) into fresh outputs."""
        out = torch.empty_like(self.out)
        idx = torch.empty_like(self.idx)
        _lib.check(_lib.jfa_decode_step(self.cache.geom(), self.cache.struct(), self.q, self.scale,
                                        self.k, idx, self.k_exact, self.v_exact,
                                        self.exact_on_host, self.ws.buf, out), "decode_step")
        torch.cuda.synchronize()
        st, flag = _lib.jfa_check_error(self.cache.geom(), self.ws.buf)
        assert flag == 0, f"device error flag {flag:#x}"
        return out.cpu().double().numpy(), idx.cpu().numpy()

    def selection_scores(self):
        torch.cuda.synchronize()
        nq = self.cache.n_quant
        return self.ws.scores(self.cache)[:, :, :nq].cpu().double().numpy()

    # ---- oracle side on the same inputs ----
    def oracle_cache(self) -> O.PackedCache:
        return O.pack_cache(self.k_cpu.double().numpy(), self.v_cpu.double().numpy(), self.ctx,
                            self.w.key_bits, self.w.val_bits)

    def oracle_step(self, idx=None) -> O.StepResult:
        return O.decode_step(self.q_cpu.double().numpy(), self.k_cpu.double().numpy(),
                             self.v_cpu.double().numpy(), self.oracle_cache(), self.k, self.scale,
                             idx=idx)


def assert_out_close(got, ref, max_abs=MAX_ABS, rel_l2=REL_L2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.isfinite(got).all(), "non-finite output"
    assert err.max() <= max_abs, f"max-abs {err.max():.3e} > {max_abs}"
    assert rel <= rel_l2, f"rel-L2 {rel:.3e} > {rel_l2}"
    return err.max(), rel


def assert_topk_valid(idx_gpu, sel_oracle, k, window=TIE_WINDOW):
    """GPU index sets equal the oracle's except for indices whose oracle score
    lies within `window` of the k-th score; format checks on every row."""
    idx_gpu = np.asarray(idx_gpu)
    ref = O.topk_indices(sel_oracle, k)
    b, h, nq = sel_oracle.shape
    keff = min(k, nq)
    n_diff = 0
    for bi in range(b):
        for hi in range(h):
            g = idx_gpu[bi, hi]
            assert np.all(g[keff:] == -1)
            gs = g[:keff]
            assert np.all(np.diff(gs) > 0), "indices not strictly ascending"
            assert keff == 0 or (gs[0] >= 0 and gs[-1] < nq)
            if keff == 0:
                continue
            s = sel_oracle[bi, hi]
            kth = np.sort(s)[-keff]
            diff = set(gs.tolist()) ^ set(ref[bi, hi, :keff].tolist())
            for i in diff:
                assert abs(s[i] - kth) <= window, (bi, hi, i, s[i], kth)
            n_diff += len(diff)
    return n_diff
