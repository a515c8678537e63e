"""Parity at the benchmark sizes, through the call sequence bench.py times
(jfa_decode_scores + jfa_decode_finish on the device-generated workloads).

The fp64 oracle cannot afford whole caches of this size, so a deterministic
sample of (sequence, KV head) segments is checked one segment at a time: the
segment's bf16 keys/values are copied back, packed by the oracle, and
compared with the device's packed records (bit-exact codes and fp16
scales/zeros for the first, a middle and the last group), its top-k set
(equal outside the tie window) and its output rows (max-abs / rel-L2).
"""
import numpy as np
import pytest
import torch

import bit_kv_cache_jfa_b200 as jfa
from bit_kv_cache_jfa_b200 import _lib
import oracle.jfa_oracle as O
import workloads as W
from jfa_testutil import SCORE_ABS, assert_out_close, assert_topk_valid

pytestmark = pytest.mark.gpu

CASES = [
    ("llama8b_k3v2_32k", False, 3),
    ("llama8b_k4v4_128k", False, 2),
    ("llama8b_k4v4_128k", True, 2),
    ("qwen30b_k3v2_32k", False, 3),
    ("llama70b_k3v2_32k_b8", False, 2),
    ("llama70b_k4v4_32k_b8", False, 2),
    ("llama70b_k3v2_8k_b1", False, 2),
    ("llama70b_k3v2_128k_b32", False, 2),
    ("llama70b_k3v2_256k_b1", False, 2),
    ("llama70b_k4v4_256k_b1", False, 2),
]


@pytest.mark.parametrize("name,host_rows,n_seg", CASES)
def test_fullsize_sampled_segments(name, host_rows, n_seg):
    w = W.WORKLOADS[name]
    dev = torch.device("cuda")
    q = W.gen_q(w)
    k_all, v_all = W.gen_kv_device(w, dev, W.gen_q(w))
    cache = jfa.KVCache(w.batch, w.heads, w.kv_heads, w.ctx, w.key_bits, w.val_bits, device=dev)
    ws = jfa.Workspace(cache, w.topk, device=dev)
    cache.append(k_all, v_all, ws)
    if host_rows:
        k_exact = k_all.cpu().pin_memory()
        v_exact = v_all.cpu().pin_memory()
    else:
        k_exact, v_exact = k_all, v_all
    qd = q.to(dev)
    out = torch.empty(w.batch, w.heads, 128, dtype=torch.float32, device=dev)
    idx = torch.empty(w.batch, w.kv_heads, w.topk, dtype=torch.int32, device=dev)
    geom, cst = cache.geom(), cache.struct()
    scale = W.default_scale(w)
    for _ in range(2):  # the second step runs on the workspace state the first left
        _lib.check(_lib.jfa_decode_scores(geom, cst, qd, scale, ws.buf), "scores")
        _lib.check(_lib.jfa_decode_finish(geom, cst, qd, scale, w.topk, idx, k_exact, v_exact,
                                          1 if host_rows else 0, ws.buf, out), "finish")
    torch.cuda.synchronize()
    assert ws.error_flag(cache) == 0
    out_h, idx_h = out.cpu().double().numpy(), idx.cpu().numpy()
    g = w.group
    nq = cache.n_quant
    scores = ws.scores(cache)
    worst = 0.0
    for (b, h) in W.sample_segments(w, n_seg, seed=7):
        kk = k_all[b, h].cpu().double().numpy()[None, None]
        vv = v_all[b, h].cpu().double().numpy()[None, None]
        qq = q[b:b + 1, h * g:(h + 1) * g].double().numpy()
        oc = O.pack_cache(kk, vv, w.ctx, w.key_bits, w.val_bits)
        for gi in sorted({0, (nq // 64) // 2, nq // 64 - 1}):
            kc, ks, kz, vc, vs, vz = _lib.jfa_unpack_record(w.key_bits, w.val_bits,
                                                           cache.record(b, h, gi))
            sl = slice(64 * gi, 64 * gi + 64)
            assert np.array_equal(kc, oc.k_codes[0, 0, sl]), (b, h, gi, "key codes")
            assert np.array_equal(ks, oc.k_scale[0, 0, gi].view(np.uint16)), (b, h, gi)
            assert np.array_equal(kz, oc.k_zero[0, 0, gi].view(np.uint16)), (b, h, gi)
            assert np.array_equal(vc, oc.v_codes[0, 0, sl]), (b, h, gi, "value codes")
            assert np.array_equal(vs, oc.v_scale[0, 0, sl].view(np.uint16)), (b, h, gi)
            assert np.array_equal(vz, oc.v_zero[0, 0, sl].view(np.uint16)), (b, h, gi)
        ref = O.decode_step(qq, kk, vv, oc, w.topk, scale)
        s_gpu = scores[b, h, :nq].cpu().double().numpy()
        err = float(np.abs(s_gpu - ref.select[0, 0]).max())
        worst = max(worst, err)
        assert err <= SCORE_ABS, (b, h, err)
        assert_topk_valid(idx_h[b:b + 1, h:h + 1], ref.select, w.topk)
        # the output with the device's own index set (a tie-window swap changes
        # which tokens are exact, so the oracle follows the same choice)
        ref_same = O.decode_step(qq, kk, vv, oc, w.topk, scale, idx=idx_h[b:b + 1, h:h + 1])
        assert_out_close(out_h[b:b + 1, h * g:(h + 1) * g], ref_same.out)
    print(f"{name}: max selection-score error {worst:.2e} (bound {SCORE_ABS:.0e})")
