// scores.cu — jfa_decode_scores: the approximate scan over packed keys and
// values (Jet-QSparse abstract: a dense scan scores the full key history).
//
// Per 64-token group g of a (sequence, KV head) and query head h the logit
//   s_hat[h][t] = scale * ( sum_c (q[h][c]*s[g][c]) * k'[t][c] + sum_c q[h][c]*m[g][c] )
// is HACK's affine identity (HACK review, Eq. (4)) with an unquantized query;
// jfa_approx.cuh holds that arithmetic: mma.sync with the 16 tokens of an
// m-tile as A rows (codes extracted by one AND as fp16 subnormals), q*s as an
// exact (hi, lo) fp16 column pair per head as B, the bias as an MMA chain.
//
// The same pass accumulates, per query head, the online-softmax partial over
// the dequantized values v_hat = s_v * v' + m_v (v' codes exact in fp16):
//   sum_t p_t v_hat[t][c] = sum_t (p_t s_v[t][j]) v'[t][c] + sum_t p_t m_v[t][j]
// as an MMA with A = value codes (rows = channels, columns = tokens) and
// B = fp16(p) * s_v (columns = heads; the weights move from the QK output
// layout to this operand layout by two shuffles per 16 tokens), plus a small
// MMA whose A rows are the value zeros of the four channel groups and a row
// of ones (giving sum p).  The fp16 weights p themselves (one coalesced
// 32-bit store per lane and m-tile) and the running maximum each group's
// weights were taken against (m_used) are stored, so the correction step
// removes exactly these terms for the top-k tokens, without a rounding
// residue.
//
// Also written per token: the selection score S_t = max over the G heads
// (natural-log units), and a per-segment histogram of its top 13 key bits
// (the first radix level of the top-k selection).
//
// Work split: W warps (NW per CTA, one CTA per SM) take balanced contiguous
// ranges of the flattened (segment, group) list.  Each warp streams its
// records through a private two-stage shared-memory ring filled by
// cp.async.bulk (one bulk copy per 6.5-9.5 KB record, completion on an
// mbarrier) and writes one softmax partial per segment it touched.
#include "jfa_approx.cuh"
#include "jfa_internal.cuh"

namespace jfa {

struct ScanParams {
  const uint8_t* groups;
  const uint16_t* q;
  float* scores;
  float* partials;
  float* m_used;    // [n_seg][ng_cap][8]: running maxima per head
  uint32_t* wts;    // [n_seg][ng_cap][4][NT][32]: the fp16 weights, lane order
  uint32_t* hist;   // [n_seg][hist_reps][kScanHistStride]: bins, then the largest key
  uint32_t* flag;
  long long total;  // entries of the flattened (segment, group) list
  int ng_cap, capacity;
  int hkv, G, H, n_seg;
  int n_warps;
  int hist_reps;    // histogram copies per segment
  int defer_last;   // request no record of a sequence's last group before the dependency wait
  float kappa;      // scale * log2(e): logits are kept in log2 units
  SeqTable seq;     // per-sequence lengths and group offsets
};

// (segment, group) of flattened entry x: the sequence by binary search over
// the group offsets (a sequence without groups has an empty range), then the
// KV head and group inside it.
__device__ __forceinline__ void locate_group(const ScanParams& p, long long x, int& seg, int& g) {
  int lo = 0, hi = p.n_seg / p.hkv;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.seq.gpre[mid] <= x) lo = mid;
    else hi = mid;
  }
  const int ngb = seq_groups(p.seq, lo);
  const int r = (int)(x - p.seq.gpre[lo]);
  seg = lo * p.hkv + r / ngb;
  g = r % ngb;
}
// The entry after the last group of segment seg: the next segment with groups.
__device__ __forceinline__ int next_segment(const ScanParams& p, int seg) {
  ++seg;
  while (seg < p.n_seg && seq_groups(p.seq, seg / p.hkv) == 0) seg += p.hkv;
  return seg;
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ uint2 lds64(const uint8_t* p) {
  return *reinterpret_cast<const uint2*>(p);
}

constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned kFull = 0xFFFFFFFFu;

template <int KB, int VB, int NT>
struct ScanCfg {
  static constexpr int REC = 512 + 1024 * KB + 1024 + 1024 * VB;
  static constexpr int NW = scan_cta_warps(KB, VB, NT);
  static constexpr int STAGES = 2;
  static constexpr int SMEM = NW * STAGES * REC + NW * STAGES * 8;
  static_assert(SMEM <= 227 * 1024, "scan ring exceeds shared memory");
};

template <int KB, int VB, int NT>
__global__ void __launch_bounds__(ScanCfg<KB, VB, NT>::NW * 32, 1)
    scan_kernel(const __grid_constant__ ScanParams p) {
  using Cfg = ScanCfg<KB, VB, NT>;
  constexpr int REC = Cfg::REC;
  constexpr int S = Cfg::STAGES;
  constexpr int NW = Cfg::NW;
  constexpr int OFF_KC = 512;
  constexpr int OFF_VS = 512 + 1024 * KB;
  constexpr int OFF_VC = OFF_VS + 1024;
  constexpr int KW = KeyPos<KB>::WORDS;
  extern __shared__ __align__(128) uint8_t smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const long long wg = (long long)blockIdx.x * NW + warp;
  const long long W = p.n_warps, T = p.total;
  const long long g0 = wg < W ? scan_range_begin(wg, W, T) : 0;
  const long long g1 = wg < W ? scan_range_begin(wg + 1, W, T) : 0;
  const bool has_work = g0 < g1;  // warp-uniform
  const int hrep = (int)(wg % p.hist_reps);  // this warp's histogram copy

  uint8_t* ring = smem + (size_t)warp * S * REC;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (size_t)NW * S * REC) + warp * S;
  const uint64_t pol = policy_evict_first();
  if (lane == 0 && has_work) {
#pragma unroll
    for (int i = 0; i < S; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  // prefetch cursor (segment, group) of the next record to request
  int pf_seg = 0, pf_g = 0;
  if (has_work) locate_group(p, g0, pf_seg, pf_g);
  int pf_ng = has_work ? seq_groups(p.seq, pf_seg / p.hkv) : 0;
  auto issue_next = [&](int stage) {
    mbar_expect_tx(&bar[stage], REC);
    bulk_g2s(ring + stage * REC, p.groups + ((size_t)pf_seg * p.ng_cap + (size_t)pf_g) * REC,
             REC, &bar[stage], pol);
    if (++pf_g == pf_ng) {
      pf_g = 0;
      pf_seg = next_segment(p, pf_seg);
      pf_ng = pf_seg < p.n_seg ? seq_groups(p.seq, pf_seg / p.hkv) : 0;
    }
  };
  // only the first stage now: every warp's first record is requested before
  // any second one, so the first records arrive sooner; the other stages
  // follow once the first has landed
  // Only now wait for the previous kernel in the stream: the first record
  // copy reads the packed cache, which no kernel that releases this one
  // early writes (the append kernel writes a sequence's last group: with
  // defer_last that record is requested after the wait); the scores,
  // histogram, partials and running maxima this kernel writes are read or
  // cleared by the previous step's finishing kernel.
  const bool early = has_work && !(p.defer_last && pf_g == pf_ng - 1);
  if (lane == 0 && early) issue_next(0);
  pdl_wait();
  if (lane == 0 && has_work && !early) issue_next(0);

  // lane roles: B column gid of n-tile n = (head (gid >> 1) + 4n, limb gid & 1);
  // logits of head tig + 4n; value columns (heads) 2 tig, 2 tig + 1
  const bool lo_lane = (gid & 1) != 0;
  bool hv[NT];  // head tig + 4n exists
#pragma unroll
  for (int n = 0; n < NT; ++n) hv[n] = tig + 4 * n < p.G;
  const float kappa_u = p.kappa * KeyPos<KB>::unscale;
  float acc[8][4];
  float dz[4];
  float m_run[NT];
  uint32_t q2[NT][16];
  long long cur = -1;

  auto reset = [&](long long seg) {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    dz[0] = dz[1] = dz[2] = dz[3] = 0.f;
    const int b = (int)(seg / p.hkv), h = (int)(seg % p.hkv);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      m_run[n] = hv[n] ? -INFINITY : 0.f;
      const int hq = (gid >> 1) + 4 * n;
      const bool ok = hq < p.G;
      q_frag(p.q + ((size_t)b * p.H + (size_t)h * p.G + (ok ? hq : 0)) * kD, ok, tig, q2[n]);
    }
  };

  // running maximum of head hh (held by lanes with tig = hh & 3)
  auto head_m = [&](int hh) {
    float v[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) v[n] = __shfl_sync(kFull, m_run[n], hh & 3);
    return NT == 2 && (hh >> 2) ? v[NT - 1] : v[0];
  };

  auto flush = [&](long long seg) {
    float* base = p.partials + (size_t)(wg + seg) * p.G * kPartStride;
    float zj[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      zj[j][0] = __shfl_sync(kFull, dz[0], j * 4 + tig);
      zj[j][1] = __shfl_sync(kFull, dz[1], j * 4 + tig);
    }
    const float l0 = __shfl_sync(kFull, dz[0], 16 + tig);
    const float l1 = __shfl_sync(kFull, dz[1], 16 + tig);
    const float mh0 = head_m(2 * tig), mh1 = head_m(2 * tig + 1);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * tig + e;
      if (h < p.G) {
        float* row = base + h * kPartStride;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          // undo the code position 2^(p - 24) of the tile's value codes
          const float us = VB == 4 ? ((mt >> 2) ? 1048576.0f : 16777216.0f)
                                   : (float)(1 << (24 - 2 * (mt >> 1)));
          row[4 + 16 * mt + gid] = fmaf(acc[mt][e], us, zj[mt >> 1][e]);
          row[4 + 16 * mt + gid + 8] = fmaf(acc[mt][2 + e], us, zj[mt >> 1][e]);
        }
        if (gid == 0) {
          row[0] = e ? mh1 : mh0;
          row[1] = e ? l1 : l0;
        }
      }
    }
  };

  int seg = 0, g = 0;
  if (has_work) locate_group(p, g0, seg, g);
  int ng_cur = has_work ? seq_groups(p.seq, seg / p.hkv) : 0;
  int st = 0;
  uint32_t par = 0;
  bool failed = false;
  for (long long gi = g0; gi < g1; ++gi) {
    if (seg != cur) {
      if (cur >= 0) flush(cur);
      reset(seg);
      cur = seg;
    }
    const bool ok = __all_sync(kFull, mbar_wait_bounded(&bar[st], par));
    if (!ok) {
      if (lane == 0) {
        set_flag(p.flag, JFA_DEVERR_TIMEOUT);
        // drain the copies still in flight before leaving (bounded)
        for (int i = 0; i < S; ++i) {
          const long long gj = gi + i;
          if (gj >= g1 || (gi == g0 && i > 0)) break;  // later stages not yet requested
          const int sj = (st + i) % S;
          const uint32_t pj = par ^ (uint32_t)((st + i) / S);
          mbar_wait_bounded(&bar[sj], pj & 1u);
        }
      }
      __syncwarp();
      failed = true;
      break;
    }
    if (gi == g0 && lane == 0) {
#pragma unroll
      for (int i = 1; i < S; ++i)
        if (g0 + i < g1) issue_next(i);
    }
    const uint8_t* r = ring + st * REC;

    // ---- B operands: q~ = q * s * F (hi or lo per lane) and the group bias
    uint32_t qb[NT][16];
    float bk[NT];
    {
      uint32_t sk[16], zk[16], sf[16];
      key_sz(r, tig, sk, zk);
#pragma unroll
      for (int n = 0; n < NT; ++n) bk[n] = bias_mma(q2[n], zk, p.kappa);
      scale_pos<KB>(sk, sf);
#pragma unroll
      for (int n = 0; n < NT; ++n) q_tilde_col(q2[n], sf, lo_lane, qb[n]);
    }
    // the bias of an absent head is -inf, so its logits are -inf without a
    // select per logit (kept per logit for K4V4 with two n-tiles, where the
    // register allocation measured slower the other way)
    constexpr bool kInfBias = !(KB == 4 && VB == 4 && NT == 2);
    float bku[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) bku[n] = (!kInfBias || hv[n]) ? bk[n] : -INFINITY;

    // ---- approximate logits (log2 units): u[mt][n][r] of head tig + 4n,
    // token 16 mt + gid + 8 r
    float u[4][NT][2];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      uint32_t w[KW];
      const uint8_t* kp = r + OFF_KC + mt * (32 * 4 * KW) + lane * 4 * KW;
      if constexpr (KB == 4) {
        const uint4 c0 = lds128(kp), c1 = lds128(kp + 16);
        w[0] = c0.x; w[1] = c0.y; w[2] = c0.z; w[3] = c0.w;
        w[4] = c1.x; w[5] = c1.y; w[6] = c1.z; w[7] = c1.w;
      } else {
        const uint2 c0 = lds64(kp), c1 = lds64(kp + 8), c2 = lds64(kp + 16);
        w[0] = c0.x; w[1] = c0.y; w[2] = c1.x; w[3] = c1.y; w[4] = c2.x; w[5] = c2.y;
      }
      uint32_t a[16][2];
      key_afrag<KB>(w, a);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        float d[4];
        qk_chain(a, qb[n], d);
        u[mt][n][0] = (kInfBias || hv[n]) ? approx_logit(d, 0, kappa_u, bku[n]) : -INFINITY;
        u[mt][n][1] = (kInfBias || hv[n]) ? approx_logit(d, 1, kappa_u, bku[n]) : -INFINITY;
      }
    }

    // ---- online softmax bookkeeping, head tig + 4n (reduce over gid)
    bool grow = false;
    float m_new[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float mx = u[0][n][0];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) mx = fmaxf(mx, fmaxf(u[mt][n][0], u[mt][n][1]));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      m_new[n] = fmaxf(m_run[n], mx);
      grow |= m_new[n] > m_run[n];
    }
    if (__any_sync(kFull, grow)) {
      float al[NT];
#pragma unroll
      for (int n = 0; n < NT; ++n) al[n] = exp2f(m_run[n] - m_new[n]);
      // value columns are heads 2 tig, 2 tig + 1: their factors from lanes tig' = h & 3
      float a0v[NT], a1v[NT];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        a0v[n] = __shfl_sync(kFull, al[n], (2 * tig) & 3);
        a1v[n] = __shfl_sync(kFull, al[n], (2 * tig + 1) & 3);
      }
      const float a0 = (NT == 2 && tig >= 2) ? a0v[NT - 1] : a0v[0];
      const float a1 = (NT == 2 && tig >= 2) ? a1v[NT - 1] : a1v[0];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        acc[mt][0] *= a0;
        acc[mt][1] *= a1;
        acc[mt][2] *= a0;
        acc[mt][3] *= a1;
      }
      dz[0] *= a0;
      dz[1] *= a1;
      dz[2] *= a0;
      dz[3] *= a1;
#pragma unroll
      for (int n = 0; n < NT; ++n) m_run[n] = m_new[n];
    }
    // the maximum this group's weights are taken against, for the correction
    if (gid == 0) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
        if (hv[n]) p.m_used[((size_t)seg * p.ng_cap + g) * kMaxG + tig + 4 * n] = m_run[n];
    }

    // ---- selection score S = max over heads; lane ends with m-tile tig,
    // tokens 16 tig + gid and + 8
    {
      float v[4][2];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          float x = u[mt][0][rr];
#pragma unroll
          for (int n = 1; n < NT; ++n) x = fmaxf(x, u[mt][n][rr]);
          v[mt][rr] = x;
        }
      const bool b1 = (tig & 2) != 0, b0 = (tig & 1) != 0;
      float w2[2][2];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const float keep = b1 ? v[2 + i][rr] : v[i][rr];
          const float send = b1 ? v[i][rr] : v[2 + i][rr];
          w2[i][rr] = fmaxf(keep, __shfl_xor_sync(kFull, send, 2));
        }
      float sc[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const float keep = b0 ? w2[1][rr] : w2[0][rr];
        const float send = b0 ? w2[0][rr] : w2[1][rr];
        sc[rr] = fmaxf(keep, __shfl_xor_sync(kFull, send, 1)) * kLn2;
      }
      float* srow = p.scores + (size_t)seg * p.capacity + (size_t)g * kKG + 16 * tig + gid;
      srow[0] = sc[0];
      srow[8] = sc[1];
      uint32_t* hs = p.hist + ((size_t)seg * p.hist_reps + hrep) * kScanHistStride;
      const uint32_t k0 = float_key(sc[0]), k1 = float_key(sc[1]);
      atomicAdd(hs + (k0 >> (32 - kScanHistBits)), 1u);
      atomicAdd(hs + (k1 >> (32 - kScanHistBits)), 1u);
      // the segment's largest key: where the finishing kernel starts its
      // search for the k-th largest
      const uint32_t kmax = __reduce_max_sync(kFull, max(k0, k1));
      if (lane == 0) atomicMax(hs + kScanHistBins, kmax);
    }

    // ---- weights fp16(2^(u - m)) packed per m-tile: (token gid, token gid + 8),
    // stored as they are (word (mt, n) of the lane) for the correction
    uint32_t X[4][NT];
    uint32_t* wrec = p.wts + ((size_t)seg * p.ng_cap + g) * (4 * NT * 32) + lane;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        X[mt][n] = pack_h2(approx_weight(u[mt][n][0], m_run[n]), approx_weight(u[mt][n][1], m_run[n]));
        wrec[(mt * NT + n) * 32] = X[mt][n];
      }

    // ---- value aggregate: acc^T[c][h] += sum_t v'[t][c] * fp16(p[t][h] s_v[t][j]) ----
    const int src0 = (2 * tig) * 4 + (gid & 3), src1 = (2 * tig + 1) * 4 + (gid & 3);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      // weights of head gid, tokens 16kk + 2tig, +1 (pa) and + 8, + 9 (pb)
      uint32_t y0 = __shfl_sync(kFull, X[kk][0], src0), y1 = __shfl_sync(kFull, X[kk][0], src1);
      if constexpr (NT == 2) {
        const uint32_t z0 = __shfl_sync(kFull, X[kk][NT - 1], src0);
        const uint32_t z1 = __shfl_sync(kFull, X[kk][NT - 1], src1);
        if (gid >= 4) {
          y0 = z0;
          y1 = z1;
        }
      }
      const uint32_t pa = __byte_perm(y0, y1, 0x5410), pb = __byte_perm(y0, y1, 0x7632);
      const uint4 s0 = lds128(r + OFF_VS + kk * 128 + tig * 32);
      const uint4 s1 = lds128(r + OFF_VS + kk * 128 + tig * 32 + 16);
      const uint32_t sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      uint32_t bh[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bh[j][0] = h2_mul(pa, sv[2 * j]);
        bh[j][1] = h2_mul(pb, sv[2 * j + 1]);
      }
      uint32_t za0 = 0u, za2 = 0u;
      if (gid < 4) {
        const uint2 zz = lds64(r + OFF_VS + 512 + kk * 128 + tig * 32 + gid * 8);
        za0 = zz.x;
        za2 = zz.y;
      } else if (gid == 4) {
        za0 = za2 = kOneH2;
      }
      mma16816(dz, za0, 0u, za2, 0u, pa, pb);
      // value codes: one AND per register (fp16 subnormals, position p(mt))
      if constexpr (VB == 4) {
        const uint4 v0 = lds128(r + OFF_VC + (2 * kk) * 512 + lane * 16);
        const uint4 v1 = lds128(r + OFF_VC + (2 * kk + 1) * 512 + lane * 16);
        const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t vs[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) vs[i] = vw[i] >> 8;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int q = mt & 3;
          const uint32_t mask = 0x000F000Fu << (4 * (mt >> 2));
          mma16816(acc[mt], vw[2 * q] & mask, vs[2 * q] & mask, vw[2 * q + 1] & mask,
                   vs[2 * q + 1] & mask, bh[mt >> 1][0], bh[mt >> 1][1]);
        }
      } else {
        const uint4 v = lds128(r + OFF_VC + kk * 512 + lane * 16);
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
        uint32_t vs[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) vs[i] = vw[i] >> 8;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int q = mt & 1;
          const uint32_t mask = 0x00030003u << (2 * (mt >> 1));
          mma16816(acc[mt], vw[2 * q] & mask, vs[2 * q] & mask, vw[2 * q + 1] & mask,
                   vs[2 * q + 1] & mask, bh[mt >> 1][0], bh[mt >> 1][1]);
        }
      }
    }

    __syncwarp();
    if (lane == 0 && gi + S < g1) issue_next(st);
    if (++st == S) {
      st = 0;
      par ^= 1u;
    }
    if (++g == ng_cur) {
      g = 0;
      seg = next_segment(p, seg);
      ng_cur = seg < p.n_seg ? seq_groups(p.seq, seg / p.hkv) : 0;
    }
  }
  if (has_work && !failed) flush(cur);

  // No explicit launch_dependents: the dependent kernel is released as the
  // scan's CTAs exit, so its thread-block clusters find whole SMs free (an
  // early release measured slower: clusters placed beside the last scan CTAs
  // left some of them a second wave).

}

template <int KB, int VB, int NT>
static int launch_scan_t(const ScanParams& sp, int n_ctas, bool pdl, cudaStream_t st) {
  using Cfg = ScanCfg<KB, VB, NT>;
  static bool configured[64] = {false};  // per device: the attribute is set on each
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    if (cudaFuncSetAttribute(scan_kernel<KB, VB, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM) != cudaSuccess)
      return JFA_ERR_CUDA;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  if (!pdl) {
    scan_kernel<KB, VB, NT><<<dim3(n_ctas), dim3(Cfg::NW * 32), (size_t)Cfg::SMEM, st>>>(sp);
    return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
  }
  return launch_pdl(scan_kernel<KB, VB, NT>, dim3(n_ctas), dim3(Cfg::NW * 32), (size_t)Cfg::SMEM,
                    st, sp) == cudaSuccess
             ? JFA_OK
             : JFA_ERR_CUDA;
}

template <int KB, int VB>
static int launch_scan_g(const ScanParams& sp, int n_ctas, bool pdl, cudaStream_t st) {
  return sp.G > 4 ? launch_scan_t<KB, VB, 2>(sp, n_ctas, pdl, st)
                  : launch_scan_t<KB, VB, 1>(sp, n_ctas, pdl, st);
}

int launch_scores(const jfa_geom& g, const SeqTable& t, const jfa_cache& c, const uint16_t* q,
                  float scale, uint8_t* ws, const jfa_workspace_layout& L, cudaStream_t st,
                  bool pdl, bool defer_last) {
  ScanPlan plan = scan_plan(g, t, num_sms_current());
  if (plan.total_groups == 0) return JFA_OK;
  ScanParams sp;
  sp.groups = static_cast<const uint8_t*>(c.groups);
  sp.q = q;
  sp.scores = reinterpret_cast<float*>(ws + L.off_scores);
  sp.partials = reinterpret_cast<float*>(ws + L.off_partials);
  sp.m_used = reinterpret_cast<float*>(ws + L.off_mused);
  sp.wts = reinterpret_cast<uint32_t*>(ws + L.off_wts);
  sp.hist = reinterpret_cast<uint32_t*>(ws + L.off_scan_hist);
  sp.flag = reinterpret_cast<uint32_t*>(ws + L.off_flag);
  sp.total = plan.total_groups;
  sp.ng_cap = g.capacity / kKG;
  sp.n_seg = g.batch * g.num_kv_heads;
  sp.seq = t;
  sp.capacity = g.capacity;
  sp.hkv = g.num_kv_heads;
  sp.G = g.num_heads / g.num_kv_heads;
  sp.H = g.num_heads;
  sp.n_warps = plan.n_warps;
  sp.hist_reps = scan_hist_reps(sp.n_seg);
  sp.defer_last = defer_last ? 1 : 0;
  sp.kappa = scale * 1.4426950408889634f;
  if (g.key_bits == 3 && g.val_bits == 2) return launch_scan_g<3, 2>(sp, plan.n_ctas, pdl, st);
  if (g.key_bits == 4 && g.val_bits == 4) return launch_scan_g<4, 4>(sp, plan.n_ctas, pdl, st);
  if (g.key_bits == 3 && g.val_bits == 4) return launch_scan_g<3, 4>(sp, plan.n_ctas, pdl, st);
  if (g.key_bits == 4 && g.val_bits == 2) return launch_scan_g<4, 2>(sp, plan.n_ctas, pdl, st);
  return JFA_ERR_UNSUPPORTED;
}

}  // namespace jfa
