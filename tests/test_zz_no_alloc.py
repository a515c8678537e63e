"""jfa_topk_noalloc (top-k with its scratch in a fixed device array of the
library, for callers that cannot allocate) against jfa_topk on the same
scores, on two calls in a row.  Collected last on purpose."""
import numpy as np
import pytest
import torch

import bit_kv_cache_jfa_b200 as jfa
import oracle.jfa_oracle as O
from bit_kv_cache_jfa_b200 import _lib


def _reference_and_noalloc(n_seg, nq, k, scores):
    # existing path: scores in a workspace, jfa_topk
    cache = jfa.KVCache(n_seg, 1, 1, nq + 64, 4, 4)
    cache.n_ctx = nq + 1                 # N_q = nq quantized tokens
    ws = jfa.Workspace(cache, k)
    ws.scores(cache)[:, 0, :nq] = torch.from_numpy(scores).cuda()
    idx_ref = torch.empty(n_seg, 1, k, dtype=torch.int32, device="cuda")
    _lib.check(_lib.jfa_topk(cache.geom(), k, ws.buf, idx_ref), "jfa_topk")
    # allocation-free path on a separate copy of the same scores
    stride = nq + 8
    src = torch.zeros(n_seg, stride, dtype=torch.float32, device="cuda")
    src[:, :nq] = torch.from_numpy(scores).cuda()
    idx_new = torch.full((n_seg, k), -7, dtype=torch.int32, device="cuda")
    _lib.check(_lib.jfa_topk_noalloc(src, n_seg, stride, nq, k, idx_new), "jfa_topk_noalloc")
    torch.cuda.synchronize()
    return idx_ref.view(n_seg, k).cpu().numpy(), idx_new.cpu().numpy()


@pytest.mark.gpu
def test_noalloc_topk_matches_topk_twice():
    rng = np.random.default_rng(11)
    # first call: 8 rows of 32704 normal scores
    s1 = (rng.standard_normal((8, 32704)) * 2).astype(np.float32)
    ref1, new1 = _reference_and_noalloc(8, 32704, 256, s1)
    assert np.array_equal(ref1, new1)
    assert np.array_equal(new1, O.topk_indices(s1.astype(np.float64), 256))
    # second call on the shared scratch: other shape, many ties
    s2 = (np.round(rng.standard_normal((4, 8192)) * 4) / 4).astype(np.float32)
    ref2, new2 = _reference_and_noalloc(4, 8192, 300, s2)
    assert np.array_equal(ref2, new2)
    assert np.array_equal(new2, O.topk_indices(s2.astype(np.float64), 300))


@pytest.mark.gpu
def test_noalloc_topk_rejects_sizes_beyond_its_scratch():
    src = torch.zeros(65, 64, dtype=torch.float32, device="cuda")
    idx = torch.empty(65, 8, dtype=torch.int32, device="cuda")
    assert _lib.jfa_topk_noalloc(src, 65, 64, 64, 8, idx) == _lib.JFA_ERR_UNSUPPORTED
    big = torch.zeros(2, 262144, dtype=torch.float32, device="cuda")
    idx2 = torch.empty(2, 8, dtype=torch.int32, device="cuda")
    assert _lib.jfa_topk_noalloc(big, 2, 262144, 262144, 8, idx2) == _lib.JFA_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_noalloc_topk_k_at_least_n_scores_pads():
    # k >= n_scores: every index in order, then -1
    n_seg, nq, k = 3, 100, 128
    src = torch.randn(n_seg, nq, dtype=torch.float32, device="cuda")
    idx = torch.full((n_seg, k), -7, dtype=torch.int32, device="cuda")
    _lib.check(_lib.jfa_topk_noalloc(src, n_seg, nq, nq, k, idx), "jfa_topk_noalloc")
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    assert np.array_equal(got, O.topk_indices(src.double().cpu().numpy(), k))
    assert np.all(got[:, :nq] == np.arange(nq)) and np.all(got[:, nq:] == -1)
