"""GPU parity of the 128-token block selection (jfa_topk_blocks, Jet-QSparse
abstract) against the fp64 oracle: the chosen token sets bit for bit on the
same scores, and the whole step (scores, block selection, correction and
merge through jfa_correct_merge) within the output tolerances."""
import numpy as np
import pytest
import torch

import oracle.jfa_oracle as O
import workloads as W
from bit_kv_cache_jfa_b200 import _lib
import bit_kv_cache_jfa_b200 as jfa

from jfa_testutil import DeviceRun, TIE_WINDOW, assert_out_close

pytestmark = pytest.mark.gpu


def small(kb, vb, heads, kv, ctx, batch, k, planted=16, seed=0, lognormal=False):
    return W.Workload(f"blk_k{kb}v{vb}", batch=batch, heads=heads, kv_heads=kv, ctx=ctx,
                      key_bits=kb, val_bits=vb, topk=k, planted=planted, seed=seed,
                      value_lognormal=lognormal)


@pytest.mark.parametrize("ctx,n_blocks,mode", [
    (4097, 5, "normal"), (4097, 40, "normal"), (32768, 1, "normal"), (32768, 64, "normal"),
    (32768, 32, "ties"), (8193, 64, "constant"), (131072, 64, "normal"), (200, 3, "normal"),
    (20000, 64, "few_values")])
def test_topk_blocks_bit_exact_on_written_scores(ctx, n_blocks, mode):
    w = small(4, 4, 8, 4, ctx, 2, 64)
    zeros = torch.zeros(2, 4, ctx, 128, dtype=torch.bfloat16)
    run = DeviceRun(w, kv=(zeros, zeros))
    nq = run.cache.n_quant
    rng = np.random.default_rng(ctx + n_blocks)
    if mode == "normal":
        s = rng.standard_normal((2, 4, nq)) * 2
    elif mode == "ties":
        s = np.round(rng.standard_normal((2, 4, nq)) * 2) / 2
    elif mode == "constant":
        s = np.full((2, 4, nq), -0.75)
    else:
        s = rng.integers(0, 3, (2, 4, nq)).astype(np.float64)
    s = s.astype(np.float32)
    run.ws.scores(run.cache)[:, :, :nq] = torch.from_numpy(s).cuda()
    idx = torch.full((2, 4, n_blocks * 128), -7, dtype=torch.int32, device="cuda")
    _lib.check(_lib.jfa_topk_blocks(run.cache.geom(), n_blocks, run.ws.buf, idx), "topk_blocks")
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), O.topk_blocks(s.astype(np.float64), n_blocks))


def _block_sets_valid(idx, sel, n_blocks, window=TIE_WINDOW):
    """Chosen blocks equal the oracle's except blocks whose oracle block score
    lies within the tie window of the n-th block score."""
    bs = O.block_scores(sel)
    ref = O.topk_blocks(sel, n_blocks)
    for b in range(idx.shape[0]):
        for h in range(idx.shape[1]):
            got = set((idx[b, h][idx[b, h] >= 0] // 128).tolist())
            want = set((ref[b, h][ref[b, h] >= 0] // 128).tolist())
            nb = bs.shape[-1]
            kth = np.sort(bs[b, h])[-min(n_blocks, nb)]
            for blk in got ^ want:
                assert abs(bs[b, h, blk] - kth) <= window, (b, h, blk)


@pytest.mark.parametrize("kb,vb,heads,kv,ctx,n_blocks,batch", [
    (3, 2, 32, 8, 5000, 4, 2), (4, 4, 32, 4, 9000, 16, 1), (3, 2, 8, 2, 20000, 64, 1),
    (4, 2, 64, 8, 3000, 30, 2)])
def test_block_step_against_oracle(kb, vb, heads, kv, ctx, n_blocks, batch):
    w = small(kb, vb, heads, kv, ctx, batch, 64, lognormal=True)
    run = DeviceRun(w)   # the block path takes its own idx; the workspace is sized for jfa_topk
    out, idx = jfa.decode_step_blocks(run.cache, run.q, n_blocks, run.k_exact, run.v_exact,
                                      run.ws, scale=run.scale)
    torch.cuda.synchronize()
    assert run.ws.error_flag(run.cache) == 0
    idx = idx.cpu().numpy()
    s_gpu = run.selection_scores()
    assert np.array_equal(idx, O.topk_blocks(s_gpu, n_blocks))
    ref = run.oracle_step()
    _block_sets_valid(idx, ref.select, n_blocks)
    got = out.cpu().double().numpy()
    assert_out_close(got, run.oracle_step(idx=idx).out)
    # the planted tokens' blocks are chosen
    for b in range(batch):
        pos = W.planted_positions(w, b).numpy()
        for h in range(kv):
            chosen = set(idx[b, h][idx[b, h] >= 0].tolist())
            if n_blocks * 128 >= 16 * 128:
                assert set(pos.tolist()) <= chosen
