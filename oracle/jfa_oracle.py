"""fp64 CPU oracle for approximate-then-correct low-bit KV decode attention.

TEST INFRASTRUCTURE ONLY.  This module is a plain, slow, obviously correct
statement of what the decode step computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs
may import it.  The CUDA library (``bit_kv_cache_jfa_b200``) never imports it
and shares no code with it; the only shared module is ``workloads`` (seeded
random inputs, no method arithmetic).

What is computed, and where the pages say so:

* The method (JetFire README, introduction): keep a low-bit KV cache on the
  GPU, score every cached token approximately from it, pick the top-k tokens
  and correct them with a high-precision copy ("approximate-then-correct").
* Low-bit formats K3V2 and K4V4 (JetFire README, benchmark section).
* Partition-wise asymmetric quantization x ~ s * x' + m, with m the
  partition minimum and s the scale (HACK review, Eq. (4) and its context);
  group size 64 with an FP16 zero point and scale (TailorKV review, "free
  parameters": quantization bit size and group size).
* The most recent tokens stay high-precision so that appending never
  requantizes (HACK review: last partial block of V kept in FP16, Figure 8;
  Jet-QSparse abstract: at most two BF16 pages per sequence and layer).
* A dense scan scores the full key history; selected tokens get
  high-precision value aggregation with FP32 accumulation (Jet-QSparse
  abstract).
* Affine identity (HACK review, Eq. (4)): a product against affinely
  quantized data is an integer product plus row/column correction terms.

Readings taken where the pages are silent (each is also listed in the
design notes): softmax scale is a parameter (default 1/sqrt(d)); the tail
holds the last 1..64 tokens and is always exact; key groups are 64 tokens
per channel, value groups 32 channels per token; the zero point is the fp16
rounding *down* of the group minimum and the scale the fp16 rounding *up* of
(max - zero) / (2^b - 1); codes round half to even on an fp64 quotient; the
per-(sequence, KV head) selection score is the max over the group's query
heads; top-k order is (score descending, index ascending); exact and
approximate parts are merged in log-sum-exp form.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(hand-derived fixtures in ``tests/golden/``, closed forms, invariants and
brute force); none is "parity unpinned".
"""
from __future__ import annotations

import dataclasses

import numpy as np

KEY_GROUP = 64    # tokens per key group (one scale/zero per channel)
VAL_GROUP = 32    # channels per value group (one scale/zero per token)
TAIL_MAX = 64     # most recent tokens kept exact (bf16)


# ---------------------------------------------------------------------------
# Tail split
# ---------------------------------------------------------------------------
def split_point(n_ctx: int) -> int:
    """Number of quantized tokens N_q for a sequence of n_ctx tokens.

    Reading of the HACK review (Figure 8: the last partial block stays
    unquantized): tokens are appended to a bf16 tail; when a token arrives at
    a full tail of 64, the 64 tail tokens are first quantized as one key
    group.  Hence the tail always holds T = N - N_q in [1, 64] tokens.
    """
    if n_ctx <= 0:
        return 0
    return KEY_GROUP * ((n_ctx - 1) // KEY_GROUP)


# ---------------------------------------------------------------------------
# fp16 directed rounding (zero point rounds down, scale rounds up)
# ---------------------------------------------------------------------------
def fp16_round_down(x) -> np.ndarray:
    """Largest fp16 value <= x (elementwise; x in fp64)."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        h = x.astype(np.float16)
    above = h.astype(np.float64) > x
    return np.where(above, np.nextafter(h, np.float16(-np.inf)), h).astype(np.float16)


def fp16_round_up(x) -> np.ndarray:
    """Smallest fp16 value >= x (elementwise; x in fp64)."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        h = x.astype(np.float16)
    below = h.astype(np.float64) < x
    return np.where(below, np.nextafter(h, np.float16(np.inf)), h).astype(np.float16)


# ---------------------------------------------------------------------------
# Group-wise asymmetric quantization (HACK review Eq. (4) context; TailorKV
# review: group size 64, FP16 zero point and scale)
# ---------------------------------------------------------------------------
def quantize_last_axis(x, bits: int):
    """Quantize every row of ``x`` (fp64 view of bf16 data) as one group.

    zero  = fp16 round-down of min(row)
    scale = fp16 round-up of (max(row) - zero) / (2^bits - 1)   [fp64 quotient]
    code  = clip(rint((x - zero) / scale), 0, 2^bits - 1)       [fp64 quotient,
                                                                 half to even]
    A group with scale 0 (max == zero) gets code 0 everywhere.
    Returns (codes uint8 like x, scale fp16 [rows], zero fp16 [rows]).
    """
    x = np.asarray(x, dtype=np.float64)
    levels = (1 << bits) - 1
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    zero = fp16_round_down(mn)
    scale = fp16_round_up((mx - zero.astype(np.float64)) / levels)
    s = scale.astype(np.float64)[..., None]
    z = zero.astype(np.float64)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint((x - z) / s)
    q = np.where(s == 0.0, 0.0, q)
    codes = np.clip(q, 0, levels).astype(np.uint8)
    return codes, scale, zero


def dequantize(codes, scale, zero) -> np.ndarray:
    """x_hat = scale * code + zero (fp64); scale/zero broadcast over the group."""
    return scale.astype(np.float64)[..., None] * codes.astype(np.float64) \
        + zero.astype(np.float64)[..., None]


def quantize_keys(k, bits: int):
    """Keys [..., N_q, d]: one group per (64-token block, channel).

    Returns codes uint8 [..., N_q, d], scale/zero fp16 [..., N_q/64, d].
    """
    k = np.asarray(k, dtype=np.float64)
    *lead, nq, d = k.shape
    assert nq % KEY_GROUP == 0
    ng = nq // KEY_GROUP
    blocks = k.reshape(*lead, ng, KEY_GROUP, d)
    per_channel = np.swapaxes(blocks, -1, -2)          # [..., ng, d, 64]
    codes, scale, zero = quantize_last_axis(per_channel, bits)
    codes = np.swapaxes(codes, -1, -2).reshape(*lead, nq, d)
    return codes, scale, zero


def dequantize_keys(codes, scale, zero) -> np.ndarray:
    *lead, nq, d = codes.shape
    ng = nq // KEY_GROUP
    c = np.swapaxes(codes.reshape(*lead, ng, KEY_GROUP, d), -1, -2)   # [..., ng, d, 64]
    x = dequantize(c, scale, zero)
    return np.swapaxes(x, -1, -2).reshape(*lead, nq, d)


def quantize_values(v, bits: int):
    """Values [..., N_q, d]: one group per (token, 32-channel block).

    Returns codes uint8 [..., N_q, d], scale/zero fp16 [..., N_q, d/32].
    """
    v = np.asarray(v, dtype=np.float64)
    *lead, nq, d = v.shape
    groups = v.reshape(*lead, nq, d // VAL_GROUP, VAL_GROUP)
    codes, scale, zero = quantize_last_axis(groups, bits)
    return codes.reshape(*lead, nq, d), scale, zero


def dequantize_values(codes, scale, zero) -> np.ndarray:
    *lead, nq, d = codes.shape
    c = codes.reshape(*lead, nq, d // VAL_GROUP, VAL_GROUP)
    return dequantize(c, scale, zero).reshape(*lead, nq, d)


@dataclasses.dataclass
class PackedCache:
    """Quantized state of a cache after n_ctx tokens (per sequence, uniform)."""
    n_ctx: int
    n_quant: int
    key_bits: int
    val_bits: int
    k_codes: np.ndarray   # uint8 [B, H_kv, N_q, d]
    k_scale: np.ndarray   # fp16  [B, H_kv, N_q/64, d]
    k_zero: np.ndarray    # fp16  [B, H_kv, N_q/64, d]
    v_codes: np.ndarray   # uint8 [B, H_kv, N_q, d]
    v_scale: np.ndarray   # fp16  [B, H_kv, N_q, d/32]
    v_zero: np.ndarray    # fp16  [B, H_kv, N_q, d/32]
    tail_k: np.ndarray    # fp64 view of bf16 [B, H_kv, T, d]
    tail_v: np.ndarray

    def k_hat(self) -> np.ndarray:
        return dequantize_keys(self.k_codes, self.k_scale, self.k_zero)

    def v_hat(self) -> np.ndarray:
        return dequantize_values(self.v_codes, self.v_scale, self.v_zero)


def pack_cache(k, v, n_ctx: int, key_bits: int, val_bits: int) -> PackedCache:
    """Quantize the first N_q tokens of K/V [B, H_kv, >=n_ctx, d]; keep the
    rest as the exact tail.  Codes of a group depend only on that group's 64
    tokens, so the state is a function of n_ctx alone: appending tokens never
    changes codes already written (HACK review: no requantization)."""
    k = np.asarray(k, dtype=np.float64)[:, :, :n_ctx]
    v = np.asarray(v, dtype=np.float64)[:, :, :n_ctx]
    nq = split_point(n_ctx)
    kc, ks, kz = quantize_keys(k[:, :, :nq], key_bits)
    vc, vs, vz = quantize_values(v[:, :, :nq], val_bits)
    return PackedCache(n_ctx, nq, key_bits, val_bits, kc, ks, kz, vc, vs, vz,
                       k[:, :, nq:].copy(), v[:, :, nq:].copy())


# ---------------------------------------------------------------------------
# Approximate scoring
# ---------------------------------------------------------------------------
def approx_logits(q, cache: PackedCache, scale: float) -> np.ndarray:
    """s_hat[b, h, t] = scale * q[b, h] . x_hat_K[b, h // G, t] for t < N_q,
    computed by dequantize-then-multiply in fp64.  Returns [B, H, N_q]."""
    q = np.asarray(q, dtype=np.float64)
    b, h, d = q.shape
    hkv = cache.k_codes.shape[1]
    g = h // hkv
    kh = cache.k_hat()                                  # [B, H_kv, N_q, d]
    qg = q.reshape(b, hkv, g, d)
    s = np.einsum("bkgd,bktd->bkgt", qg, kh)
    return scale * s.reshape(b, h, -1)


def affine_logits(q, cache: PackedCache, scale: float) -> np.ndarray:
    """The same logits through the affine identity (HACK review, Eq. (4)),
    specialised to an unquantized query:  q . (s * k' + m)
    = sum_c (q_c s_c) k'_c + sum_c q_c m_c, per key group."""
    q = np.asarray(q, dtype=np.float64)
    b, h, d = q.shape
    hkv = cache.k_codes.shape[1]
    g = h // hkv
    ng = cache.n_quant // KEY_GROUP
    qg = q.reshape(b, hkv, g, d)
    s = cache.k_scale.astype(np.float64)                # [B, H_kv, ng, d]
    m = cache.k_zero.astype(np.float64)
    codes = cache.k_codes.astype(np.float64).reshape(b, hkv, ng, KEY_GROUP, d)
    q_tilde = qg[:, :, None, :, :] * s[:, :, :, None, :]      # [B,H_kv,ng,G,d]
    integer_part = np.einsum("bkngd,bkntd->bkngt", q_tilde, codes)
    correction = np.einsum("bkgd,bknd->bkng", qg, m)[..., None]
    out = (integer_part + correction)                         # [B,H_kv,ng,G,64]
    out = np.moveaxis(out, 3, 2).reshape(b, hkv, g, ng * KEY_GROUP)
    return scale * out.reshape(b, h, -1)


def selection_scores(s_hat, kv_heads: int) -> np.ndarray:
    """Per-(sequence, KV head) selection score: max over the G query heads
    that share the KV head.  [B, H, N_q] -> [B, H_kv, N_q]."""
    s_hat = np.asarray(s_hat)
    b, h, n = s_hat.shape
    return s_hat.reshape(b, kv_heads, h // kv_heads, n).max(axis=2)


# ---------------------------------------------------------------------------
# Top-k selection
# ---------------------------------------------------------------------------
def topk_indices(scores, k: int) -> np.ndarray:
    """k largest scores per row, order (score descending, index ascending);
    the chosen indices are returned sorted ascending, padded with -1 when
    k > row length.  scores [..., N] -> int32 [..., k]."""
    scores = np.asarray(scores)
    *lead, n = scores.shape
    rows = int(np.prod(lead)) if lead else 1
    flat = scores.reshape(rows, n)
    out = np.full((rows, k), -1, dtype=np.int32)
    keff = min(k, n)
    idx = np.arange(n)
    for r in range(flat.shape[0]):
        order = np.lexsort((idx, -flat[r]))       # primary: -score, then index
        out[r, :keff] = np.sort(order[:keff])
    return out.reshape(*lead, k)


# ---------------------------------------------------------------------------
# Block selection (Jet-QSparse abstract: 128-token blocks are selected for the
# sparse high-precision value aggregation, so the exact rows are contiguous)
# ---------------------------------------------------------------------------
BLOCK = 128


def block_scores(scores, block: int = BLOCK) -> np.ndarray:
    """Score of every block of ``block`` consecutive quantized tokens: the
    largest selection score inside it (the last block may be partial).
    scores [..., N] -> [..., ceil(N / block)]."""
    scores = np.asarray(scores, dtype=np.float64)
    *lead, n = scores.shape
    nb = -(-n // block)
    pad = np.full((*lead, nb * block - n), -np.inf)
    return np.concatenate([scores, pad], axis=-1).reshape(*lead, nb, block).max(axis=-1)


def topk_blocks(scores, n_blocks: int, block: int = BLOCK) -> np.ndarray:
    """The n_blocks blocks with the largest block score, order (score
    descending, block index ascending), expanded to their token indices:
    every token of a chosen block, ascending, then -1 padding up to
    n_blocks * block entries (tokens past N in a partial last block are
    -1).  scores [..., N] -> int32 [..., n_blocks * block]."""
    scores = np.asarray(scores, dtype=np.float64)
    *lead, n = scores.shape
    bs = block_scores(scores, block)
    rows = int(np.prod(lead)) if lead else 1
    flat = bs.reshape(rows, -1)
    out = np.full((rows, n_blocks * block), -1, dtype=np.int32)
    for r in range(rows):
        chosen = topk_indices(flat[r][None], n_blocks)[0]
        toks = [t for b in chosen if b >= 0 for t in range(b * block, (b + 1) * block) if t < n]
        out[r, :len(toks)] = toks
    return out.reshape(*lead, n_blocks * block)


# ---------------------------------------------------------------------------
# NVFP4 keys and FP4 scores (Jet-QSparse abstract: compact NVFP4 cache storage,
# native FP4 query-key computation, then block selection and sparse FP16
# value aggregation with FP32 accumulation)
# ---------------------------------------------------------------------------
FP4_BLOCK = 16                    # elements per UE4M3 block scale
E2M1_MAX = 6.0
E4M3_MAX = 448.0
# the non-negative E2M1 values, by code 0..7 (sign bit 8)
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_round(v) -> np.ndarray:
    """Codes (0..15, bit 3 = sign) of the E2M1 values nearest to v, ties to
    the even code (the one whose mantissa bit is 0); |v| > 6 saturates."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E2M1_MAX)
    d = np.abs(a[..., None] - E2M1_GRID)                  # distance to every grid value
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    # among equally near values prefer an even code (mantissa bit 0)
    even = cand & (np.arange(8) % 2 == 0)
    code = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    sign = (v < 0) & (code > 0)
    return (code + 8 * sign).astype(np.uint8)


def e2m1_value(codes) -> np.ndarray:
    codes = np.asarray(codes).astype(np.int64)
    mag = E2M1_GRID[codes & 7]
    return np.where(codes & 8, -mag, mag)


def e4m3_values() -> np.ndarray:
    """Every finite non-negative E4M3 value, ascending (bias 7, 3 mantissa
    bits, subnormals below 2^-6; the largest finite value is 448)."""
    vals = [m / 8 * 2.0 ** -6 for m in range(8)]
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:       # the NaN encoding
                continue
            vals.append((1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


_E4M3 = e4m3_values()


def e4m3_round_positive(v) -> np.ndarray:
    """Nearest non-negative E4M3 value to v >= 0, ties to the even mantissa,
    saturating at 448."""
    v = np.minimum(np.asarray(v, dtype=np.float64), E4M3_MAX)
    d = np.abs(v[..., None] - _E4M3)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    even = cand & (np.arange(_E4M3.size) % 2 == 0)      # code parity = mantissa parity
    i = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    return _E4M3[i]


def nvfp4_quantize(x, tensor_amax=None):
    """NVFP4 of the rows of x [..., n] (n a multiple of 16): one fp32 scale
    over the whole array, amax / (6 * 448) (stored as fp32; 1 when amax is
    0), one UE4M3 scale per 16 consecutive elements of a row, the nearest
    E4M3 to amax_block / (6 * s), and E2M1 codes of x / (block scale * s),
    all quotients in fp64.  Returns (codes uint8 [..., n], block scales
    fp64 [..., n/16], s float).  x_hat = e2m1 * block scale * s."""
    x = np.asarray(x, dtype=np.float64)
    amax = float(np.abs(x).max()) if tensor_amax is None else float(tensor_amax)
    s = float(np.float32(amax / (E2M1_MAX * E4M3_MAX))) if amax > 0 else 1.0
    *lead, n = x.shape
    blocks = x.reshape(*lead, n // FP4_BLOCK, FP4_BLOCK)
    bs = e4m3_round_positive(np.abs(blocks).max(axis=-1) / (E2M1_MAX * s))
    with np.errstate(divide="ignore", invalid="ignore"):
        q = blocks / (bs[..., None] * s)
    q = np.where(bs[..., None] == 0, 0.0, q)
    codes = e2m1_round(q).reshape(*lead, n)
    return codes, bs, s


def nvfp4_dequantize(codes, bs, s) -> np.ndarray:
    codes = np.asarray(codes)
    *lead, n = codes.shape
    v = e2m1_value(codes).reshape(*lead, n // FP4_BLOCK, FP4_BLOCK)
    return (v * np.asarray(bs, dtype=np.float64)[..., None] * s).reshape(*lead, n)


def nvfp4_keys(k, n_quant: int):
    """Keys [..., N, d] of one (sequence, KV head) list: every 64-token group
    of the first n_quant tokens quantized with its own fp32 scale.  Returns
    the dequantized keys [..., n_quant, d]."""
    k = np.asarray(k, dtype=np.float64)[..., :n_quant, :]
    out = np.zeros_like(k)
    for g in range(n_quant // KEY_GROUP):
        sl = slice(KEY_GROUP * g, KEY_GROUP * (g + 1))
        blk = k[..., sl, :]
        c, bs, s = nvfp4_quantize(blk)
        out[..., sl, :] = nvfp4_dequantize(c, bs, s)
    return out


def nvfp4_scores(q, k, n_ctx: int, scale: float) -> np.ndarray:
    """FP4 scores of every quantized token: scale * q_hat . k_hat with the
    keys in NVFP4 per 64-token group and every query head in NVFP4 with its
    own fp32 scale.  q [B, H, d], k [B, H_kv, >=N, d] -> [B, H, N_q]."""
    q = np.asarray(q, dtype=np.float64)
    b, h, d = q.shape
    hkv = np.asarray(k).shape[1]
    g = h // hkv
    nq = split_point(n_ctx)
    out = np.zeros((b, h, nq))
    for bi in range(b):
        for kv in range(hkv):
            kh = nvfp4_keys(np.asarray(k)[bi, kv], nq)
            for j in range(g):
                hq = kv * g + j
                cq, bq, sq = nvfp4_quantize(q[bi, hq][None])
                qh = nvfp4_dequantize(cq, bq, sq)[0]
                out[bi, hq] = scale * (kh @ qh)
    return out


def sparse_block_step(q, k_exact, v_exact, n_ctx: int, n_blocks: int, scale: float,
                      idx=None):
    """The Jet-QSparse step: FP4 scores, the n_blocks best 128-token blocks
    per (sequence, KV head) by the largest score over the KV head's query
    heads, and exact softmax attention over the chosen blocks' tokens plus
    the bf16 tail (the other tokens are left out).  Returns (out [B, H, d],
    idx [B, H_kv, n_blocks * 128], selection scores [B, H_kv, N_q])."""
    q = np.asarray(q, dtype=np.float64)
    ke = np.asarray(k_exact, dtype=np.float64)
    ve = np.asarray(v_exact, dtype=np.float64)
    b, h, d = q.shape
    hkv = ke.shape[1]
    g = h // hkv
    nq = split_point(n_ctx)
    sel = selection_scores(nvfp4_scores(q, ke, n_ctx, scale), hkv)
    if idx is None:
        idx = topk_blocks(sel, n_blocks)
    out = np.zeros((b, h, d))
    for bi in range(b):
        for kv in range(hkv):
            chosen = idx[bi, kv][idx[bi, kv] >= 0]
            ex = np.concatenate([chosen, np.arange(nq, n_ctx)]).astype(np.int64)
            for j in range(g):
                hq = kv * g + j
                out[bi, hq] = finish(softmax_partial(scale * (ke[bi, kv, ex] @ q[bi, hq]),
                                                     ve[bi, kv, ex]))
    return out, idx, sel


# ---------------------------------------------------------------------------
# Critical-channel scores (TailorKV review: a channel's importance is the
# product of the query's magnitude in it and the largest key magnitude in it,
# s_i = |q_i| * max|K_i|; approximate attention scores from the critical
# channels pick the top-k tokens, which are then fetched and attended exactly)
# ---------------------------------------------------------------------------
def channel_importance(q, k, n_quant: int) -> np.ndarray:
    """Per (sequence, KV head) and channel: the largest |q_i| over the KV
    head's query heads times the largest |K_{t,i}| over the quantized tokens
    t < n_quant.  q [B, H, d], k [B, H_kv, >=n_quant, d] -> [B, H_kv, d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    b, h, d = q.shape
    hkv = k.shape[1]
    qmax = np.abs(q).reshape(b, hkv, h // hkv, d).max(axis=2)
    kmax = np.abs(k[:, :, :n_quant]).max(axis=2) if n_quant > 0 else np.zeros((b, hkv, d))
    return qmax * kmax


def critical_channels(importance, r: int) -> np.ndarray:
    """The r most important channels per row (importance descending, channel
    index ascending on ties), sorted ascending.  [..., d] -> int [..., r]."""
    return topk_indices(importance, r)


def channel_scores(q, k, n_ctx: int, r: int, scale: float) -> np.ndarray:
    """Selection scores from the r critical channels of each KV head: for
    every quantized token t < N_q the largest over the KV head's query heads
    of scale * sum over the critical channels i of q_{h,i} K_{t,i}.
    -> [B, H_kv, N_q]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    b, h, d = q.shape
    hkv = k.shape[1]
    g = h // hkv
    nq = split_point(n_ctx)
    chans = critical_channels(channel_importance(q, k, nq), r)
    out = np.zeros((b, hkv, nq))
    for bi in range(b):
        for kv in range(hkv):
            c = chans[bi, kv]
            keys = k[bi, kv, :nq][:, c]                       # [N_q, r]
            per_head = [scale * (keys @ q[bi, kv * g + j, c]) for j in range(g)]
            out[bi, kv] = np.max(per_head, axis=0) if nq else out[bi, kv]
    return out


def attend_set(q, k_exact, v_exact, n_ctx: int, idx, scale: float) -> np.ndarray:
    """Exact softmax attention of every query head over the tokens idx[b,
    h_kv] (entries >= 0) and the tail N_q .. n_ctx - 1, nothing else."""
    q = np.asarray(q, dtype=np.float64)
    ke = np.asarray(k_exact, dtype=np.float64)
    ve = np.asarray(v_exact, dtype=np.float64)
    b, h, d = q.shape
    hkv = ke.shape[1]
    g = h // hkv
    nq = split_point(n_ctx)
    out = np.zeros((b, h, d))
    for bi in range(b):
        for kv in range(hkv):
            chosen = idx[bi, kv][idx[bi, kv] >= 0]
            ex = np.concatenate([chosen, np.arange(nq, n_ctx)]).astype(np.int64)
            for j in range(g):
                hq = kv * g + j
                out[bi, hq] = finish(softmax_partial(scale * (ke[bi, kv, ex] @ q[bi, hq]),
                                                     ve[bi, kv, ex]))
    return out


def channel_step(q, k_exact, v_exact, n_ctx: int, r: int, k: int, scale: float):
    """Critical-channel scores, the top-k tokens per (sequence, KV head), and
    exact attention over them and the tail.  Returns (out, idx, scores)."""
    sel = channel_scores(q, k_exact, n_ctx, r, scale)
    idx = topk_indices(sel, k)
    return attend_set(q, k_exact, v_exact, n_ctx, idx, scale), idx, sel


# ---------------------------------------------------------------------------
# Softmax partials and log-sum-exp merge
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class Partial:
    """Unnormalised softmax state over a token set: m = max logit,
    l = sum exp(s - m), acc = sum exp(s - m) * v."""
    m: float
    l: float
    acc: np.ndarray

    @staticmethod
    def empty(d: int) -> "Partial":
        return Partial(-np.inf, 0.0, np.zeros(d))


def softmax_partial(logits, values) -> Partial:
    logits = np.asarray(logits, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    if logits.size == 0:
        return Partial.empty(values.shape[-1])
    m = logits.max()
    w = np.exp(logits - m)
    return Partial(float(m), float(w.sum()), w @ values)


def merge(a: Partial, b: Partial) -> Partial:
    """Log-sum-exp merge of two disjoint partials."""
    m = max(a.m, b.m)
    if m == -np.inf:
        return Partial(m, 0.0, a.acc + b.acc)
    wa = np.exp(a.m - m) if a.m > -np.inf else 0.0
    wb = np.exp(b.m - m) if b.m > -np.inf else 0.0
    return Partial(m, a.l * wa + b.l * wb, a.acc * wa + b.acc * wb)


def finish(p: Partial) -> np.ndarray:
    return p.acc / p.l


# ---------------------------------------------------------------------------
# The whole decode step
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class StepResult:
    out: np.ndarray          # [B, H, d] fp64
    s_hat: np.ndarray        # [B, H, N_q]
    select: np.ndarray       # [B, H_kv, N_q]
    idx: np.ndarray          # [B, H_kv, k] int32
    approx_all: list         # [B][H] Partial over all N_q quantized tokens


def decode_step(q, k_exact, v_exact, cache: PackedCache, k: int, scale: float,
                idx=None) -> StepResult:
    """One decode step for every sequence and query head.

    1. approximate logits s_hat over the N_q quantized tokens;
    2. selection score per (sequence, KV head) and its top-k (unless ``idx``
       is given, in which case that index set is used as the exact set);
    3. exact part: logits from the bf16 keys of the top-k tokens and the
       tail, aggregated with bf16 values;
    4. approximate remainder: the other quantized tokens with dequantized
       keys and values;
    5. log-sum-exp merge of the two, normalised.
    ``k_exact``/``v_exact`` [B, H_kv, >=N, d] are the high-precision copies.
    """
    q = np.asarray(q, dtype=np.float64)
    b, h, d = q.shape
    hkv = cache.k_codes.shape[1]
    g = h // hkv
    n, nq = cache.n_ctx, cache.n_quant
    ke = np.asarray(k_exact, dtype=np.float64)
    ve = np.asarray(v_exact, dtype=np.float64)
    s_hat = approx_logits(q, cache, scale)
    sel = selection_scores(s_hat, hkv)
    if idx is None:
        idx = topk_indices(sel, k)
    idx = np.asarray(idx)
    vh = cache.v_hat()
    out = np.zeros((b, h, d))
    approx_all = [[None] * h for _ in range(b)]
    for bi in range(b):
        for kv in range(hkv):
            chosen = idx[bi, kv]
            chosen = np.unique(chosen[chosen >= 0])
            exact_set = np.concatenate([chosen, np.arange(nq, n)]).astype(np.int64)
            rest = np.setdiff1d(np.arange(nq), chosen)
            for j in range(g):
                hq = kv * g + j
                exact_logits = scale * (ke[bi, kv, exact_set] @ q[bi, hq])
                pe = softmax_partial(exact_logits, ve[bi, kv, exact_set])
                pa = softmax_partial(s_hat[bi, hq, rest], vh[bi, kv, rest])
                out[bi, hq] = finish(merge(pe, pa))
                approx_all[bi][hq] = softmax_partial(s_hat[bi, hq], vh[bi, kv])
    return StepResult(out, s_hat, sel, idx, approx_all)


def exact_attention(q, k_exact, v_exact, n_ctx: int, scale: float) -> np.ndarray:
    """Plain softmax attention over all n_ctx bf16 tokens (GQA), fp64."""
    q = np.asarray(q, dtype=np.float64)
    b, h, d = q.shape
    ke = np.asarray(k_exact, dtype=np.float64)[:, :, :n_ctx]
    ve = np.asarray(v_exact, dtype=np.float64)[:, :, :n_ctx]
    hkv = ke.shape[1]
    g = h // hkv
    out = np.zeros((b, h, d))
    for bi in range(b):
        for hq in range(h):
            p = softmax_partial(scale * (ke[bi, hq // g] @ q[bi, hq]), ve[bi, hq // g])
            out[bi, hq] = finish(p)
    return out
