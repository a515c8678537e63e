"""Pins for the fp64 CPU oracle against facts fixed by the pages and by
mathematics (not against the oracle itself): hand-derived fixtures, closed
forms, invariants, library routines for special cases, and brute force."""
import math
import os

import numpy as np
import pytest
import torch

import oracle.jfa_oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases(fname):
    cases, cur = [], None
    with open(os.path.join(GOLDEN, fname)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(" ")
            if key == "case":
                cur = {"name": val}
                cases.append(cur)
            else:
                cur[key] = val.split()
    return cases


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()


# --------------------------------------------------------------------------
# quantization
# --------------------------------------------------------------------------
@pytest.mark.parametrize("case", _cases("quantization_cases.txt"), ids=lambda c: c["name"])
def test_quantization_golden(case):
    bits = int(case["bits"][0])
    x = np.array([float(v) for v in case["x"]])
    codes, scale, zero = O.quantize_last_axis(x[None, :], bits)
    assert codes[0].tolist() == [int(c) for c in case["codes"]]
    assert int(zero.view(np.uint16)[0]) == int(case["zero_bits"][0], 16)
    assert int(scale.view(np.uint16)[0]) == int(case["scale_bits"][0], 16)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_quantization_error_bound(bits):
    rng = np.random.default_rng(bits)
    x = _bf16(rng.standard_normal((500, 64)) * rng.choice([0.01, 1, 10, 300], (500, 1)))
    codes, scale, zero = O.quantize_last_axis(x, bits)
    xh = O.dequantize(codes, scale, zero)
    s = scale.astype(np.float64)[:, None]
    assert codes.max() <= (1 << bits) - 1
    # exact invariant of round-down zero / round-up scale / nearest code
    assert np.all(np.abs(x - xh) <= s / 2 * (1 + 1e-12))
    # the group minimum maps to code 0, the maximum to the top code
    assert np.all(codes[np.arange(500), x.argmin(1)] == 0)
    assert np.all(codes[np.arange(500), x.argmax(1)] == (1 << bits) - 1)
    # zero <= min and zero + levels * scale >= max
    assert np.all(zero.astype(np.float64) <= x.min(1))
    assert np.all(zero.astype(np.float64) + ((1 << bits) - 1) * scale.astype(np.float64)
                  >= x.max(1))


def test_round_to_nearest_even_brute_force():
    # build x = zero + (n + 1/2) * scale exactly: ties must go to even n
    bits = 4
    scale, zero = 0.5, -1.0
    n = np.arange(15)
    x = zero + (n + 0.5) * scale
    x = np.concatenate([[zero, zero + 15 * scale], x])
    codes, s, z = O.quantize_last_axis(x[None], bits)
    assert float(s[0]) == scale and float(z[0]) == zero
    expect = [0, 15] + [int(k) if k % 2 == 0 else int(k) + 1 for k in n]
    assert codes[0].tolist() == expect


def test_key_groups_run_along_tokens_per_channel():
    # channel c is constant c + g/2 inside key group g: every key group has
    # scale 0 and zero = that constant only if groups are (64 tokens, 1 channel)
    ng, d = 3, 128
    t = np.arange(64 * ng)[:, None]
    c = np.arange(d)[None, :]
    k = (c + 0.5 * (t // 64)).astype(np.float64)[None, None]
    codes, scale, zero = O.quantize_keys(k, 3)
    assert scale.shape == (1, 1, ng, d)
    assert np.all(scale == 0) and np.all(codes == 0)
    assert np.array_equal(zero[0, 0].astype(np.float64),
                          np.arange(d)[None, :] + 0.5 * np.arange(ng)[:, None])


def test_value_groups_run_along_channels_per_token():
    n, d = 64, 128
    t = np.arange(n)[:, None]
    c = np.arange(d)[None, :]
    v = (t + 0.25 * (c // 32)).astype(np.float64)[None, None]
    codes, scale, zero = O.quantize_values(v, 2)
    assert scale.shape == (1, 1, n, 4)
    assert np.all(scale == 0) and np.all(codes == 0)
    assert np.array_equal(zero[0, 0].astype(np.float64),
                          np.arange(n)[:, None] + 0.25 * np.arange(4)[None, :])


def test_grid_data_reconstructs_exactly():
    rng = np.random.default_rng(7)
    for bits in (2, 3, 4):
        lv = (1 << bits) - 1
        codes = rng.integers(0, lv + 1, (64, 128))
        codes[0], codes[1] = 0, lv           # min and max present in every channel
        k = -0.75 + 0.125 * codes.astype(np.float64)
        kc, ks, kz = O.quantize_keys(k[None, None], bits)
        assert np.array_equal(kc[0, 0], codes)
        assert np.all(ks == np.float16(0.125)) and np.all(kz == np.float16(-0.75))
        assert np.array_equal(O.dequantize_keys(kc, ks, kz)[0, 0], k)


def test_value_round_trip_through_pack_cache():
    # values are quantized per (token, 32-channel group): the dequantized
    # cache the step aggregates stays within half a step of the bf16 input
    for kb, vb, lognormal in ((3, 2, False), (4, 4, True)):
        w = W.Workload("vrt", batch=2, heads=4, kv_heads=2, ctx=321, key_bits=kb,
                       val_bits=vb, topk=8, planted=4, seed=23, value_lognormal=lognormal)
        q = W.gen_q(w)
        k, v = W.gen_kv(w, q)
        v = v.double().numpy()
        cache = O.pack_cache(k.double().numpy(), v, w.ctx, kb, vb)
        nq = cache.n_quant
        vh = cache.v_hat()
        assert vh.shape == (2, 2, nq, 128)
        step = np.repeat(cache.v_scale.astype(np.float64), 32, axis=-1)   # [B,H,N_q,128]
        assert np.all(np.abs(v[:, :, :nq] - vh) <= step / 2 * (1 + 1e-12))
        # the bound is tight somewhere (not a vacuous huge scale)
        assert np.max(np.abs(v[:, :, :nq] - vh) / step) > 0.4
        grp = v[:, :, :nq].reshape(2, 2, nq, 4, 32)
        assert np.all(cache.v_zero.astype(np.float64) <= grp.min(-1))


def test_value_grid_data_reconstructs_exactly():
    # value rows on a grid zero + scale * code (per token and channel group)
    # come back bit for bit, with the codes, scales and zeros that built them
    rng = np.random.default_rng(9)
    for bits in (2, 4):
        lv = (1 << bits) - 1
        n = 128
        codes = rng.integers(0, lv + 1, (n, 4, 32))
        codes[:, :, 0], codes[:, :, 1] = 0, lv
        zero = rng.choice([-2.0, -0.5, 0.25, 1.0], (n, 4))
        scale = rng.choice([0.0625, 0.25, 1.0], (n, 4))
        v = (zero[..., None] + scale[..., None] * codes).reshape(n, 128)
        vc, vs, vz = O.quantize_values(v[None, None], bits)
        assert np.array_equal(vc[0, 0].reshape(n, 4, 32), codes)
        assert np.array_equal(vs[0, 0].astype(np.float64), scale)
        assert np.array_equal(vz[0, 0].astype(np.float64), zero)
        assert np.array_equal(O.dequantize_values(vc, vs, vz)[0, 0], v)


@pytest.mark.parametrize("kb,vb", [(3, 2), (4, 4)])
def test_affine_identity_on_the_value_side(kb, vb):
    # HACK review, Eq. (4) applied to P V: sum_t p_t (s_v v' + m_v) is the
    # integer-code product weighted by p_t s_v plus the zero-point term
    # sum_t p_t m_v, computed here from the raw codes, scales and zeros
    w, q, k, v, cache = _small(kb=kb, vb=vb, lognormal=True)
    rng = np.random.default_rng(4)
    nq = cache.n_quant
    p = rng.random(nq)
    codes = cache.v_codes[1, 0].astype(np.float64).reshape(nq, 4, 32)
    s = cache.v_scale[1, 0].astype(np.float64)          # [N_q, 4]
    z = cache.v_zero[1, 0].astype(np.float64)
    integer_part = np.einsum("tj,tjc->jc", p[:, None] * s, codes)
    zero_part = (p[:, None] * z).sum(0)[:, None]
    direct = (integer_part + zero_part).reshape(128)
    assert np.allclose(p @ cache.v_hat()[1, 0], direct, rtol=1e-12, atol=1e-12)


def test_exact_attention_is_torch_softmax_attention():
    w, q, k, v, cache = _small(heads=8, kv=2)
    scale = 0.083
    got = O.exact_attention(q, k, v, w.ctx, scale)
    for b in range(2):
        for hq in range(8):
            h = hq // 4
            ref = _torch_attention(q[b, hq], k[b, h, :w.ctx], v[b, h, :w.ctx], scale)
            assert np.allclose(got[b, hq], ref, rtol=1e-12, atol=1e-13)
    # a shorter context ignores the later tokens
    got2 = O.exact_attention(q, k, v, 100, scale)
    ref2 = _torch_attention(q[1, 3], k[1, 0, :100], v[1, 0, :100], scale)
    assert np.allclose(got2[1, 3], ref2, rtol=1e-12, atol=1e-13)


def test_split_point_closed_form():
    assert [O.split_point(n) for n in (0, 1, 63, 64, 65, 128, 129, 4096)] == \
        [0, 0, 0, 0, 64, 64, 128, 4032]
    for n in range(1, 400):
        t = n - O.split_point(n)
        assert 1 <= t <= 64 and O.split_point(n) % 64 == 0


# --------------------------------------------------------------------------
# scoring: affine identity (HACK review, Eq. (4)) and selection
# --------------------------------------------------------------------------
def _small(ctx=300, heads=4, kv=2, kb=4, vb=4, planted=4, seed=11, lognormal=False):
    w = W.Workload("t", batch=2, heads=heads, kv_heads=kv, ctx=ctx, key_bits=kb,
                   val_bits=vb, topk=16, planted=planted, seed=seed,
                   value_lognormal=lognormal)
    q = W.gen_q(w)
    k, v = W.gen_kv(w, q)
    cache = O.pack_cache(k.double().numpy(), v.double().numpy(), ctx, kb, vb)
    return w, q.double().numpy(), k.double().numpy(), v.double().numpy(), cache


@pytest.mark.parametrize("kb,vb", [(3, 2), (4, 4)])
def test_affine_identity_equals_dequantize_then_multiply(kb, vb):
    w, q, k, v, cache = _small(kb=kb, vb=vb)
    a = O.approx_logits(q, cache, 0.1)
    b = O.affine_logits(q, cache, 0.1)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_selection_is_max_over_group_heads():
    w, q, k, v, cache = _small(heads=8, kv=2)
    s = O.approx_logits(q, cache, 0.09)
    sel = O.selection_scores(s, 2)
    for b in range(2):
        for h in range(2):
            for t in (0, 5, 100, 255):
                assert sel[b, h, t] == max(s[b, h * 4 + j, t] for j in range(4))


# --------------------------------------------------------------------------
# top-k
# --------------------------------------------------------------------------
@pytest.mark.parametrize("case", _cases("topk_cases.txt"), ids=lambda c: c["name"])
def test_topk_golden(case):
    s = np.array([float(x) for x in case["scores"]])
    k = int(case["k"][0])
    got = O.topk_indices(s[None], k)[0].tolist()
    assert got == [int(x) for x in case.get("idx", [])]


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(3)
    for trial in range(50):
        n = int(rng.integers(1, 200))
        k = int(rng.integers(0, 220))
        s = rng.integers(-5, 5, n).astype(np.float64) * 0.5   # many ties
        ref = sorted(range(n), key=lambda i: (-s[i], i))[:k]
        ref = sorted(ref) + [-1] * max(0, k - n)
        assert O.topk_indices(s[None], k)[0].tolist() == ref


# --------------------------------------------------------------------------
# softmax partials and merge
# --------------------------------------------------------------------------
def test_split_and_merge_equals_unsplit():
    rng = np.random.default_rng(5)
    s = rng.standard_normal(300) * 4
    v = rng.standard_normal((300, 16))
    full = O.softmax_partial(s, v)
    perm = rng.permutation(300)
    a = O.softmax_partial(s[perm[:77]], v[perm[:77]])
    b = O.softmax_partial(s[perm[77:]], v[perm[77:]])
    m = O.merge(a, b)
    assert math.isclose(m.m, full.m)
    assert np.allclose(O.finish(m), O.finish(full), rtol=1e-13, atol=1e-13)
    # softmax(s) @ v by the library
    ref = torch.softmax(torch.tensor(s), 0) @ torch.tensor(v)
    assert np.allclose(O.finish(full), ref.numpy(), rtol=1e-12, atol=1e-12)
    e = O.merge(O.Partial.empty(16), a)
    assert np.allclose(O.finish(e), O.finish(a))


# --------------------------------------------------------------------------
# whole step: special cases that reduce to plain attention
# --------------------------------------------------------------------------
def _torch_attention(q, keys, vals, scale):
    q, keys, vals = map(torch.tensor, (q, keys, vals))
    return (torch.softmax(scale * keys @ q, dim=0) @ vals).numpy()


@pytest.mark.parametrize("kb,vb", [(3, 2), (4, 4)])
def test_k_at_least_nq_is_exact_attention(kb, vb):
    w, q, k, v, cache = _small(kb=kb, vb=vb)
    scale = 1 / math.sqrt(128)
    res = O.decode_step(q, k, v, cache, cache.n_quant + 5, scale)
    for b in range(2):
        for h in range(4):
            ref = _torch_attention(q[b, h], k[b, h // 2], v[b, h // 2], scale)
            assert np.allclose(res.out[b, h], ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("kb,vb", [(3, 2), (4, 4), (1, 1)])
def test_k_zero_is_attention_over_dequantized_plus_exact_tail(kb, vb):
    w, q, k, v, cache = _small(kb=kb, vb=vb, lognormal=True)
    scale = 0.07
    res = O.decode_step(q, k, v, cache, 0, scale)
    kh, vh = cache.k_hat(), cache.v_hat()
    nq = cache.n_quant
    for b in range(2):
        for h in range(4):
            keys = np.concatenate([kh[b, h // 2], k[b, h // 2, nq:]])
            vals = np.concatenate([vh[b, h // 2], v[b, h // 2, nq:]])
            ref = _torch_attention(q[b, h], keys, vals, scale)
            assert np.allclose(res.out[b, h], ref, rtol=1e-11, atol=1e-12)


def test_given_index_set_matches_hand_mixture():
    # with idx given, token t in idx uses bf16 K/V, others use x_hat; check
    # against a torch softmax over the mixed key/value matrix
    w, q, k, v, cache = _small()
    scale = 0.1
    nq = cache.n_quant
    rng = np.random.default_rng(1)
    idx = np.full((2, 2, 16), -1, dtype=np.int32)
    for b in range(2):
        for h in range(2):
            idx[b, h, :10] = np.sort(rng.choice(nq, 10, replace=False))
    res = O.decode_step(q, k, v, cache, 16, scale, idx=idx)
    kh, vh = cache.k_hat(), cache.v_hat()
    for b in range(2):
        for hq in range(4):
            h = hq // 2
            keys, vals = kh[b, h].copy(), vh[b, h].copy()
            sel = idx[b, h][idx[b, h] >= 0]
            keys[sel], vals[sel] = k[b, h, sel], v[b, h, sel]
            keys = np.concatenate([keys, k[b, h, nq:]])
            vals = np.concatenate([vals, v[b, h, nq:]])
            ref = _torch_attention(q[b, hq], keys, vals, scale)
            assert np.allclose(res.out[b, hq], ref, rtol=1e-11, atol=1e-12)


def test_output_is_convex_combination_of_value_rows():
    w, q, k, v, cache = _small(kb=3, vb=2)
    res = O.decode_step(q, k, v, cache, 16, 1 / math.sqrt(128))
    vh = cache.v_hat()
    nq = cache.n_quant
    for b in range(2):
        for hq in range(4):
            h = hq // 2
            sel = res.idx[b, h][res.idx[b, h] >= 0]
            rest = np.setdiff1d(np.arange(nq), sel)
            rows = np.concatenate([v[b, h, sel], v[b, h, nq:], vh[b, h, rest]])
            o = res.out[b, hq]
            assert np.all(o <= rows.max(0) + 1e-12) and np.all(o >= rows.min(0) - 1e-12)


def test_appending_never_changes_written_codes():
    w, q, k, v, _ = _small(ctx=400, kb=3, vb=2)
    prev = None
    for n in (1, 64, 65, 130, 200, 256, 257, 400):
        c = O.pack_cache(k, v, n, 3, 2)
        assert c.tail_k.shape[2] == n - c.n_quant
        assert np.array_equal(c.tail_k, k[:, :, c.n_quant:n])
        if prev is not None:
            nq = prev.n_quant
            assert np.array_equal(c.k_codes[:, :, :nq], prev.k_codes)
            assert np.array_equal(c.k_scale[:, :, :nq // 64], prev.k_scale)
            assert np.array_equal(c.v_codes[:, :, :nq], prev.v_codes)
            assert np.array_equal(c.v_zero[:, :, :nq], prev.v_zero)
        prev = c


def test_planted_tokens_are_selected_in_tiny_workload():
    w = W.WORKLOADS["tiny_k4v4_4k"]
    q = W.gen_q(w)
    k, v = W.gen_kv(w, q)
    cache = O.pack_cache(k.double().numpy(), v.double().numpy(), w.ctx, 4, 4)
    res = O.decode_step(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                        cache, w.topk, W.default_scale(w))
    pos = set(W.planted_positions(w, 0).tolist())
    for h in range(w.kv_heads):
        assert pos <= set(res.idx[0, h].tolist())


# --------------------------------------------------------------------------
# the pins above catch plausible oracle mistakes (planted on the CPU)
# --------------------------------------------------------------------------
def test_pins_reject_round_to_nearest_scale(monkeypatch):
    monkeypatch.setattr(O, "fp16_round_up", lambda x: np.asarray(x).astype(np.float16))
    case = [c for c in _cases("quantization_cases.txt") if c["name"] == "round_up_scale"][0]
    with pytest.raises(AssertionError):
        test_quantization_golden(case)


def test_pins_reject_wrong_merge_sign(monkeypatch):
    def bad_merge(a, b):
        m = max(a.m, b.m)
        wa, wb = np.exp(m - a.m), np.exp(m - b.m)
        return O.Partial(m, a.l * wa + b.l * wb, a.acc * wa + b.acc * wb)
    monkeypatch.setattr(O, "merge", bad_merge)
    with pytest.raises(AssertionError):
        test_k_zero_is_attention_over_dequantized_plus_exact_tail(4, 4)


def test_topk_empty_rows_pad_with_minus_one():
    # N_q = 0 (context within the tail): no quantized token can be chosen
    out = O.topk_indices(np.zeros((2, 3, 0)), 4)
    assert out.shape == (2, 3, 4) and np.all(out == -1)


def test_pins_reject_swapped_value_scale_and_zero(monkeypatch):
    monkeypatch.setattr(O.PackedCache, "v_hat",
                        lambda self: O.dequantize_values(self.v_codes, self.v_zero, self.v_scale))
    with pytest.raises(AssertionError):
        test_value_round_trip_through_pack_cache()


def test_pins_reject_value_groups_along_tokens(monkeypatch):
    # a value dequantizer that broadcasts the per-token scales along the wrong
    # axis (group index taken from the token instead of the channel)
    def bad(codes, scale, zero):
        *lead, nq, d = codes.shape
        s = np.repeat(scale.astype(np.float64), 32, axis=-1)
        z = np.repeat(zero.astype(np.float64), 32, axis=-1)
        return np.swapaxes(s, -1, -2).reshape(s.shape) * codes + z
    monkeypatch.setattr(O, "dequantize_values", bad)
    with pytest.raises(AssertionError):
        test_value_grid_data_reconstructs_exactly()


def test_pins_reject_unscaled_exact_attention(monkeypatch):
    real = O.softmax_partial
    monkeypatch.setattr(O, "exact_attention",
                        lambda q, k, v, n, scale: O.__dict__["_exact_attention_unscaled"](q, k, v, n))
    def unscaled(q, k, v, n):
        q = np.asarray(q, dtype=np.float64)
        b, h, d = q.shape
        g = h // np.asarray(k).shape[1]
        out = np.zeros((b, h, d))
        for bi in range(b):
            for hq in range(h):
                out[bi, hq] = O.finish(real(np.asarray(k)[bi, hq // g, :n] @ q[bi, hq],
                                            np.asarray(v)[bi, hq // g, :n]))
        return out
    monkeypatch.setitem(O.__dict__, "_exact_attention_unscaled", unscaled)
    with pytest.raises(AssertionError):
        test_exact_attention_is_torch_softmax_attention()


# --------------------------------------------------------------------------
# block selection (Jet-QSparse abstract: 128-token blocks)
# --------------------------------------------------------------------------
def test_block_scores_are_block_maxima_by_brute_force():
    rng = np.random.default_rng(21)
    for n in (1, 64, 127, 128, 129, 320, 1000):
        s = rng.standard_normal(n)
        got = O.block_scores(s[None], 128)[0]
        want = [max(s[i:i + 128]) for i in range(0, n, 128)]
        assert got.tolist() == want


def test_block_selection_with_unit_blocks_is_token_topk():
    rng = np.random.default_rng(22)
    s = np.round(rng.standard_normal((3, 300)) * 3) / 3       # ties included
    for k in (1, 7, 64, 300, 310):
        assert np.array_equal(O.topk_blocks(s, k, block=1), O.topk_indices(s, k))


def test_block_selection_brute_force():
    rng = np.random.default_rng(23)
    for trial in range(30):
        n = int(rng.integers(64, 1500))
        nb = -(-n // 128)
        k = int(rng.integers(1, nb + 3))
        s = rng.integers(-3, 3, n).astype(np.float64)          # many equal block maxima
        bmax = [max(s[i:i + 128]) for i in range(0, n, 128)]
        order = sorted(range(nb), key=lambda b: (-bmax[b], b))[:k]
        toks = [t for b in sorted(order) for t in range(128 * b, min(n, 128 * b + 128))]
        want = toks + [-1] * (128 * k - len(toks))
        assert O.topk_blocks(s[None], k)[0].tolist() == want


def test_block_selection_hand_case():
    # 300 tokens: blocks [0,128), [128,256), [256,300); the best token sits in
    # block 2 (partial), the second best in block 0
    s = np.zeros(300)
    s[290], s[5], s[200] = 9.0, 7.0, 1.0
    got = O.topk_blocks(s[None], 2)[0]
    assert got[:128].tolist() == list(range(128))
    assert got[128:172].tolist() == list(range(256, 300))
    assert np.all(got[172:] == -1)


def test_block_selection_step_matches_hand_mixture():
    # the decode step with the chosen blocks' tokens as the exact set equals
    # softmax attention over the mixed key/value matrix (exact rows for the
    # chosen blocks, dequantized for the rest, exact tail)
    w, q, k, v, cache = _small(ctx=700, kb=3, vb=2)
    scale = 0.09
    s_hat = O.approx_logits(q, cache, scale)
    sel = O.selection_scores(s_hat, 2)
    idx = O.topk_blocks(sel, 2)
    res = O.decode_step(q, k, v, cache, 256, scale, idx=idx)
    kh, vh = cache.k_hat(), cache.v_hat()
    nq = cache.n_quant
    for b in range(2):
        for hq in range(4):
            h = hq // 2
            keys, vals = kh[b, h].copy(), vh[b, h].copy()
            chosen = idx[b, h][idx[b, h] >= 0]
            assert len(chosen) == 256 and np.all(np.diff(chosen) > 0)
            keys[chosen], vals[chosen] = k[b, h, chosen], v[b, h, chosen]
            keys = np.concatenate([keys, k[b, h, nq:]])
            vals = np.concatenate([vals, v[b, h, nq:]])
            ref = _torch_attention(q[b, hq], keys, vals, scale)
            assert np.allclose(res.out[b, hq], ref, rtol=1e-11, atol=1e-12)


def test_pins_reject_block_mean_instead_of_max(monkeypatch):
    def mean_blocks(scores, block=128):
        scores = np.asarray(scores, dtype=np.float64)
        *lead, n = scores.shape
        nb = -(-n // block)
        return np.stack([scores[..., i * block:(i + 1) * block].mean(-1) for i in range(nb)], -1)
    monkeypatch.setattr(O, "block_scores", mean_blocks)
    with pytest.raises(AssertionError):
        test_block_scores_are_block_maxima_by_brute_force()


# --------------------------------------------------------------------------
# NVFP4 keys and FP4 scores (Jet-QSparse abstract)
# --------------------------------------------------------------------------
import ml_dtypes  # noqa: E402  (independent library casts for the two minifloat formats)


def _e2m1_library(x):
    return np.asarray(x, dtype=np.float32).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)


def test_e2m1_rounding_matches_library_cast():
    grid = O.E2M1_GRID
    mids = (grid[1:] + grid[:-1]) / 2
    x = np.concatenate([grid, mids, mids + 1e-6, mids - 1e-6, [6.5, 7.0, 100.0],
                        np.linspace(0, 8, 4001)])
    x = np.concatenate([x, -x])
    assert np.array_equal(O.e2m1_value(O.e2m1_round(x)), _e2m1_library(x))


def test_e4m3_values_and_rounding_match_library():
    lib = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(O.e4m3_values(), lib)           # 0x00..0x7E, 0x7F is NaN
    mids = (lib[1:] + lib[:-1]) / 2
    x = np.concatenate([lib, mids, mids * (1 + 1e-6), mids * (1 - 1e-6),
                        np.geomspace(1e-4, 448, 3000)])
    want = x.astype(np.float32).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(O.e4m3_round_positive(x), want)
    assert O.e4m3_round_positive(1e4) == 448.0             # saturates


def test_nvfp4_hand_case():
    # one 16-element block with tensor amax 12: s = 12 / 2688 (as fp32), the
    # block scale is the E4M3 nearest to 12 / (6 s) = 448, and x / (448 s) is
    # x / 2 up to fp32 rounding of s: [6, -1.5, 0.35, 2.4, 0.6] -> E2M1
    # [6, -1.5, 0.5, 2, 0.5], so x_hat = [12, -3, 1, 4, 1] up to that rounding
    x = np.zeros(16)
    x[:5] = [12.0, -3.0, 0.7, 4.8, 1.2]
    codes, bs, s = O.nvfp4_quantize(x[None])
    assert s == float(np.float32(12.0 / 2688.0))
    assert bs.tolist() == [[448.0]]
    assert O.e2m1_value(codes[0]).tolist()[:5] == [6.0, -1.5, 0.5, 2.0, 0.5]
    xh = O.nvfp4_dequantize(codes, bs, s)[0]
    assert np.allclose(xh[:5], [12.0, -3.0, 1.0, 4.0, 1.0], rtol=1e-6)
    assert np.all(xh[5:] == 0)


def _grid_block(rng, shape, unit):
    """Values on the E2M1 grid times unit, every 16-block holding a +-6."""
    v = rng.choice(np.concatenate([O.E2M1_GRID, -O.E2M1_GRID]), size=shape)
    v[..., ::16] = 6.0 * rng.choice([-1.0, 1.0], size=v[..., ::16].shape)
    return v * unit


def test_nvfp4_grid_data_round_trips_exactly():
    rng = np.random.default_rng(31)
    # tensor amax 6 * 448 * 2^-10 gives s = 2^-10 and block scale 448 for
    # blocks reaching the amax; a block reaching 6 * 28 * 2^-10 gets 28
    x = _grid_block(rng, (64, 128), 448 * 2.0 ** -10)
    x[3, 16:32] = _grid_block(rng, (16,), 28 * 2.0 ** -10)
    codes, bs, s = O.nvfp4_quantize(x)
    assert s == 2.0 ** -10
    assert bs[3, 1] == 28.0 and bs[0, 0] == 448.0
    assert np.array_equal(O.nvfp4_dequantize(codes, bs, s), x)


def test_nvfp4_dequant_error_is_below_one_block_unit():
    # |q - e2m1(q)| <= 1 for |q| <= 6 (the widest grid gap is 2), and the
    # block scale is rounded so that |q| <= 6 (1 + 2^-4) / (1 - 2^-4) < 7:
    # the error of every element is at most one unit bs * s of its block
    rng = np.random.default_rng(32)
    x = rng.standard_normal((64, 128))
    x[:, [3, 77]] *= 30.0
    x[5] *= 1e-3
    codes, bs, s = O.nvfp4_quantize(x)
    err = np.abs(x - O.nvfp4_dequantize(codes, bs, s))
    unit = np.repeat(bs * s, 16, axis=-1)
    assert np.all(err <= unit * (1 + 1e-12))
    assert np.all(bs > 0) and np.all(bs <= 448)
    # and the representable range is used: every block's largest |x_hat| is
    # within an eighth of its largest |x|
    xb = np.abs(x).reshape(64, 8, 16).max(-1)
    xhb = np.abs(O.nvfp4_dequantize(codes, bs, s)).reshape(64, 8, 16).max(-1)
    assert np.all(np.abs(xhb - xb) <= xb / 8)


def test_nvfp4_scores_are_exact_on_grid_data():
    # keys (per 64-token group) and queries (per head) exactly representable:
    # the FP4 scores equal scale * q . k for every query head of the KV group
    rng = np.random.default_rng(33)
    b, h, hkv, n = 2, 6, 2, 200
    unit = 448 * 2.0 ** -10
    k = _grid_block(rng, (b, hkv, n, 128), unit)
    q = _grid_block(rng, (b, h, 128), unit)
    scale = 0.125
    got = O.nvfp4_scores(q, k, n, scale)
    nq = O.split_point(n)
    for bi in range(b):
        for hq in range(h):
            want = scale * (k[bi, hq // 3, :nq] @ q[bi, hq])
            assert np.array_equal(got[bi, hq], want)


def _attend(q, keys, vals, scale):
    t = torch.softmax(torch.as_tensor(keys) @ torch.as_tensor(q) * scale, 0)
    return (t[:, None] * torch.as_tensor(vals)).sum(0).numpy()


def _sparse_inputs(n=700, seed=34):
    rng = np.random.default_rng(seed)
    q = _bf16(rng.standard_normal((2, 4, 128)))
    k = _bf16(rng.standard_normal((2, 2, n, 128)))
    v = _bf16(rng.standard_normal((2, 2, n, 128)))
    return q, k, v


def test_sparse_step_with_every_block_is_exact_attention():
    q, k, v = _sparse_inputs()
    out, idx, _ = O.sparse_block_step(q, k, v, 700, 8, 0.09)
    assert np.allclose(out, O.exact_attention(q, k, v, 700, 0.09), rtol=1e-12, atol=1e-13)
    assert np.all(idx[..., :O.split_point(700)] >= 0)


def test_sparse_step_with_no_block_is_attention_over_the_tail():
    q, k, v = _sparse_inputs()
    nq = O.split_point(700)
    out, idx, _ = O.sparse_block_step(q, k, v, 700, 0, 0.09)
    for bi in range(2):
        for hq in range(4):
            ref = _attend(q[bi, hq], k[bi, hq // 2, nq:700], v[bi, hq // 2, nq:700], 0.09)
            assert np.allclose(out[bi, hq], ref, rtol=1e-12, atol=1e-13)


def test_sparse_step_is_attention_over_chosen_blocks_and_tail():
    q, k, v = _sparse_inputs()
    nq = O.split_point(700)
    out, idx, sel = O.sparse_block_step(q, k, v, 700, 2, 0.09)
    assert np.array_equal(idx, O.topk_blocks(sel, 2))
    for bi in range(2):
        for hq in range(4):
            h = hq // 2
            toks = [t for t in idx[bi, h] if t >= 0] + list(range(nq, 700))
            assert len(toks) == len(set(toks))
            ref = _attend(q[bi, hq], k[bi, h, toks], v[bi, h, toks], 0.09)
            assert np.allclose(out[bi, hq], ref, rtol=1e-12, atol=1e-13)


def test_pins_reject_e2m1_ties_away_from_zero(monkeypatch):
    def away(v):
        v = np.asarray(v, dtype=np.float64)
        a = np.minimum(np.abs(v), 6.0)
        d = np.abs(a[..., None] - O.E2M1_GRID)
        code = np.argmax(np.isclose(d, d.min(-1, keepdims=True)) * np.arange(8), axis=-1)
        return (code + 8 * ((v < 0) & (code > 0))).astype(np.uint8)
    monkeypatch.setattr(O, "e2m1_round", away)
    with pytest.raises(AssertionError):
        test_e2m1_rounding_matches_library_cast()


def test_pins_reject_unscaled_fp4_scores(monkeypatch):
    real = O.nvfp4_dequantize
    monkeypatch.setattr(O, "nvfp4_dequantize", lambda c, bs, s: real(c, bs, 1.0))
    with pytest.raises(AssertionError):
        test_nvfp4_scores_are_exact_on_grid_data()


# --------------------------------------------------------------------------
# critical-channel scores (TailorKV review)
# --------------------------------------------------------------------------
def test_all_channels_give_the_exact_logits():
    # r = d: the channel scores are the exact logits, max over the group's heads
    q, k, v = _sparse_inputs(n=300, seed=41)
    nq = O.split_point(300)
    got = O.channel_scores(q, k, 300, 128, 0.07)
    for bi in range(2):
        for h in range(2):
            t = torch.as_tensor(k[bi, h, :nq]) @ torch.as_tensor(q[bi, 2 * h:2 * h + 2]).T
            assert np.allclose(got[bi, h], 0.07 * t.max(1).values.numpy(), rtol=1e-13, atol=1e-13)


def test_critical_channels_brute_force_with_ties():
    rng = np.random.default_rng(42)
    for _ in range(20):
        imp = rng.integers(0, 4, 128).astype(np.float64)
        r = int(rng.integers(1, 129))
        want = sorted(sorted(range(128), key=lambda c: (-imp[c], c))[:r])
        assert O.critical_channels(imp[None], r)[0].tolist() == want


def test_channel_scores_hand_case():
    # one sequence, one KV head, two query heads; channel 3: |q| max 2,
    # max|K| 1 -> 2; channel 7: |q| max 5 (a negative query), max|K| 0.5 ->
    # 2.5; channel 9: |q| 1, max|K| 4 -> 4.  r = 2 keeps channels 7 and 9.
    q = np.zeros((1, 2, 128))
    q[0, 0, 3], q[0, 1, 3] = 2.0, 1.0
    q[0, 0, 7], q[0, 1, 7] = -5.0, 1.0
    q[0, 0, 9], q[0, 1, 9] = 1.0, 0.5
    k = np.zeros((1, 1, 129, 128))
    k[0, 0, 0, 3], k[0, 0, 1, 7], k[0, 0, 2, 9], k[0, 0, 5, 9] = 1.0, -0.5, 4.0, -2.0
    imp = O.channel_importance(q, k, 128)[0, 0]
    assert (imp[3], imp[7], imp[9]) == (2.0, 2.5, 4.0)
    assert O.critical_channels(imp[None], 2)[0].tolist() == [7, 9]
    s = O.channel_scores(q, k, 129, 2, 1.0)[0, 0]
    # token 1: head 0 gives -5 * -0.5 = 2.5, head 1 gives -0.5; token 2:
    # 1 * 4 = 4 and 0.5 * 4 = 2; token 5: -2 and -1; token 0 (channel 3 is
    # not critical): 0
    assert (s[0], s[1], s[2], s[5]) == (0.0, 2.5, 4.0, -1.0)


def test_channel_step_with_every_token_is_exact_attention():
    q, k, v = _sparse_inputs(n=300, seed=43)
    out, idx, _ = O.channel_step(q, k, v, 300, 16, 256, 0.09)
    assert np.all(idx >= 0)
    assert np.allclose(out, O.exact_attention(q, k, v, 300, 0.09), rtol=1e-12, atol=1e-13)


def test_attend_set_matches_torch_attention():
    q, k, v = _sparse_inputs(n=300, seed=44)
    nq = O.split_point(300)
    rng = np.random.default_rng(45)
    idx = np.full((2, 2, 40), -1, np.int32)
    idx[..., :30] = rng.choice(nq, 30, replace=False)
    out = O.attend_set(q, k, v, 300, idx, 0.09)
    for bi in range(2):
        for hq in range(4):
            toks = list(idx[bi, hq // 2, :30]) + list(range(nq, 300))
            ref = _attend(q[bi, hq], k[bi, hq // 2, toks], v[bi, hq // 2, toks], 0.09)
            assert np.allclose(out[bi, hq], ref, rtol=1e-12, atol=1e-13)


def test_pins_reject_signed_channel_importance(monkeypatch):
    def signed(q, k, n_quant):
        q = np.asarray(q, dtype=np.float64)
        k = np.asarray(k, dtype=np.float64)
        b, h, d = q.shape
        hkv = k.shape[1]
        return q.reshape(b, hkv, h // hkv, d).max(axis=2) * np.abs(k[:, :, :n_quant]).max(axis=2)
    monkeypatch.setattr(O, "channel_importance", signed)
    with pytest.raises(AssertionError):
        test_channel_scores_hand_case()


# --------------------------------------------------------------------------
# 1-bit cache (TailorKV review: the whole cache at 1 bit, attended densely)
# --------------------------------------------------------------------------
def test_one_bit_two_level_data_reconstructs_exactly():
    # every key channel group and value channel group takes two fp16-exact
    # levels a < b with b - a fp16-exact: zero = a, scale = b - a, codes exact
    rng = np.random.default_rng(51)
    a = np.round(rng.standard_normal((1, 2, 1, 128)) * 4) / 4
    d = rng.integers(1, 8, (1, 2, 1, 128)) / 4.0
    bits = rng.integers(0, 2, (1, 2, 256, 128))
    bits[:, :, 0], bits[:, :, 1] = 0, 1          # both levels in every group
    bits[:, :, 64], bits[:, :, 65] = 0, 1
    bits[:, :, 128], bits[:, :, 129] = 0, 1
    bits[:, :, 192], bits[:, :, 193] = 0, 1
    k = a + d * bits
    lv = np.round(rng.standard_normal((1, 2, 256, 4, 1)) * 4) / 4
    dv = rng.integers(1, 8, (1, 2, 256, 4, 1)) / 4.0
    vb = rng.integers(0, 2, (1, 2, 256, 4, 32))
    vb[..., 0], vb[..., 1] = 0, 1
    v = (lv + dv * vb).reshape(1, 2, 256, 128)
    k = np.concatenate([k, np.zeros((1, 2, 10, 128))], axis=2)
    v = np.concatenate([v, np.zeros((1, 2, 10, 128))], axis=2)
    c = O.pack_cache(k, v, 266, 1, 1)
    assert np.array_equal(c.k_hat(), k[:, :, :256]) and np.array_equal(c.v_hat(), v[:, :, :256])
    assert np.array_equal(c.k_codes, bits) and np.array_equal(c.v_codes, vb.reshape(1, 2, 256, 128))


# ---------------------------------------------------------------- directed fp16 rounding
def _all_finite_fp16():
    v = np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float64)
    return np.unique(v[np.isfinite(v)])  # sorted, -0 and +0 merged


@pytest.mark.filterwarnings("ignore:overflow encountered in nextafter")
def test_fp16_directed_rounding_brackets_by_enumeration():
    # the neighbours of x among all finite fp16 values, found by search in the
    # enumerated table: round-down is the largest <= x, round-up the smallest >= x
    table = _all_finite_fp16()
    rng = np.random.default_rng(41)
    x = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 5, 4000),  # subnormal .. 1e4
        table[rng.integers(0, table.size, 500)],                          # exact fp16 values
        (table[:-1] + np.diff(table) / 2)[rng.integers(0, table.size - 1, 500)],  # midpoints
        [0.0, -0.0, 65504.0, -65504.0, 6.0e-8, -6.0e-8]])
    down = O.fp16_round_down(x).astype(np.float64)
    up = O.fp16_round_up(x).astype(np.float64)
    i = np.searchsorted(table, x, side="right") - 1
    j = np.searchsorted(table, x, side="left")
    assert np.array_equal(down, table[i])
    assert np.array_equal(up, table[j])
    exact = np.isin(x, table)
    assert np.array_equal(down[exact], x[exact]) and np.array_equal(up[exact], x[exact])


def test_fp16_directed_rounding_rejects_nearest():
    # nearest rounding is not a directed rounding: just above and just below
    # an fp16 value the two differ from it
    x = np.array([1.0 + 2.0 ** -12, 1.0 - 2.0 ** -13])
    assert O.fp16_round_down(x)[0] == np.float16(1.0)
    assert O.fp16_round_up(x)[0] == np.float16(1.0 + 2.0 ** -10)
    assert O.fp16_round_down(x)[1] == np.float16(1.0 - 2.0 ** -11)
    assert O.fp16_round_up(x)[1] == np.float16(1.0)


# ---------------------------------------------------------------- NVFP4 keys per 64-token group
def test_nvfp4_keys_quantize_each_64_token_group_on_its_own():
    rng = np.random.default_rng(43)
    # group g exactly representable with its own tensor scale 2^(-10 - g):
    # the keys come back exactly only if each group gets its own fp32 scale
    k = np.concatenate([_grid_block(rng, (64, 128), 448 * 2.0 ** (-10 - g)) for g in range(3)])
    k = np.concatenate([k, rng.standard_normal((10, 128))])  # tokens past n_quant ignored
    got = O.nvfp4_keys(k[None], 192)[0]
    assert got.shape == (192, 128)
    assert np.array_equal(got, k[:192])
    # locality: a change inside group 1 leaves groups 0 and 2 unchanged
    k2 = k.copy()
    k2[70, 5] = 1e3
    got2 = O.nvfp4_keys(k2[None], 192)[0]
    assert np.array_equal(got2[:64], got[:64]) and np.array_equal(got2[128:], got[128:])
    assert not np.array_equal(got2[64:128], got[64:128])
