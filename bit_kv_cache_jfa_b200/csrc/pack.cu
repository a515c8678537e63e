// pack.cu — jfa_pack_kv kernels: group-wise asymmetric quantization and
// bit-packing of complete 64-token groups, and bf16 tail maintenance.
//
// Quantization rule (HACK review, Eq. (4) context: x ~ s * x' + m with m the
// partition minimum; TailorKV review: FP16 zero point and scale per group):
//   zero  = largest fp16 <= min,  scale = smallest fp16 >= (max - zero)/(2^b - 1)
//   code  = round-half-even((x - zero) / scale), clipped; both quotients fp64.
// Keys: one (scale, zero) per (64-token group, channel); values: one per
// (token, 32-channel group).
#include "jfa_quant.cuh"

namespace jfa {

struct PackParams {
  uint8_t* groups;
  uint16_t* tail_k;
  uint16_t* tail_v;
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint32_t* flag;
  int hkv, ng_cap, n_new;
  int n0, nq0;      // tokens and quantized tokens before the append
  int g_first;      // first group to flush (= nq0 / 64)
  int key_bits, val_bits, rec_bytes;
};

// Source of token tau (absolute position) of segment seg: the old tail for
// tau < n0, else the new tokens.
__device__ __forceinline__ const uint16_t* token_row(const uint16_t* tail, const uint16_t* fresh,
                                                     int seg, int tau, const PackParams& p) {
  if (tau < p.n0) return tail + ((size_t)seg * kTail + (tau - p.nq0)) * kD;
  return fresh + ((size_t)seg * p.n_new + (tau - p.n0)) * kD;
}

// Quantize one 64-token group staged in shared memory (bf16 bits, token
// rows) into a zeroed record image rb; all 256 threads take part.
__device__ __forceinline__ void quantize_tile(const uint16_t (*xk)[kD + 2], const uint16_t (*xv)[kD + 2],
                                              uint8_t* rb, int key_bits, int val_bits, uint32_t* flag) {
  const int tid = threadIdx.x;
  bool bad = false;
  // keys: thread c < 128 owns channel c
  if (tid < kD) {
    const int c = tid;
    float mn = bf(xk[0][c]), mx = mn;
    for (int t = 1; t < kKG; ++t) {
      mn = fminf(mn, bf(xk[t][c]));
      mx = fmaxf(mx, bf(xk[t][c]));
    }
    uint16_t zb, sb;
    double z, s;
    quant_params((double)mn, (double)mx, key_bits, zb, sb, z, s);
    bad |= !finite_h(zb) || !finite_h(sb);
    *reinterpret_cast<uint16_t*>(rb + off_ks() + ks_scale_off(c)) = sb;
    *reinterpret_cast<uint16_t*>(rb + off_ks() + ks_zero_off(c)) = zb;
    for (int t = 0; t < kKG; ++t) {
      uint32_t code = quant_code((double)bf(xk[t][c]), z, s, key_bits);
      BitLoc L[3];
      const int n = kc_bits(key_bits, t, c, L);
      if (n == 1) {
        if (code) atomicOr(reinterpret_cast<uint32_t*>(rb + off_kc() + L[0].byte), code << L[0].bit);
      } else {
        for (int b = 0; b < 3; ++b)
          if ((code >> b) & 1u)
            atomicOr(reinterpret_cast<uint32_t*>(rb + off_kc() + L[b].byte), 1u << L[b].bit);
      }
    }
  } else {
    // values: threads 128..255 own (token, group) pairs 2 each
    for (int u = tid - kD; u < kKG * (kD / kVG); u += 128) {
      const int t = u >> 2, j = u & 3;
      float mn = bf(xv[t][j * kVG]), mx = mn;
      for (int c = 1; c < kVG; ++c) {
        mn = fminf(mn, bf(xv[t][j * kVG + c]));
        mx = fmaxf(mx, bf(xv[t][j * kVG + c]));
      }
      uint16_t zb, sb;
      double z, s;
      quant_params((double)mn, (double)mx, val_bits, zb, sb, z, s);
      bad |= !finite_h(zb) || !finite_h(sb);
      *reinterpret_cast<uint16_t*>(rb + off_vs(key_bits) + vs_scale_off(t, j)) = sb;
      *reinterpret_cast<uint16_t*>(rb + off_vs(key_bits) + vs_zero_off(t, j)) = zb;
      for (int cc = 0; cc < kVG; ++cc) {
        const int c = j * kVG + cc;
        uint32_t code = quant_code((double)bf(xv[t][c]), z, s, val_bits);
        BitLoc L = vc_loc(val_bits, t, c);
        if (code) atomicOr(reinterpret_cast<uint32_t*>(rb + off_vc(key_bits) + L.byte), code << L.bit);
      }
    }
  }
  if (bad) set_flag(flag, JFA_DEVERR_NONFINITE_QUANT);
}

// One CTA (256 threads) quantizes one 64-token group of one segment.
__global__ void __launch_bounds__(256) pack_groups_kernel(PackParams p) {
  __shared__ uint16_t xk[kKG][kD + 2];  // bf16 bits
  __shared__ uint16_t xv[kKG][kD + 2];
  __shared__ __align__(16) uint32_t rec[9728 / 4];
  const int seg = blockIdx.y;
  const int g = p.g_first + blockIdx.x;
  const int tid = threadIdx.x;

  for (int i = tid; i < p.rec_bytes / 4; i += 256) rec[i] = 0u;
  for (int i = tid; i < kKG * kD / 2; i += 256) {
    int t = i / (kD / 2), c2 = (i % (kD / 2)) * 2;
    int tau = g * kKG + t;
    const uint32_t* rk = reinterpret_cast<const uint32_t*>(token_row(p.tail_k, p.k_new, seg, tau, p));
    const uint32_t* rv = reinterpret_cast<const uint32_t*>(token_row(p.tail_v, p.v_new, seg, tau, p));
    uint32_t wk = rk[c2 / 2], wv = rv[c2 / 2];
    xk[t][c2] = (uint16_t)(wk & 0xFFFFu);
    xk[t][c2 + 1] = (uint16_t)(wk >> 16);
    xv[t][c2] = (uint16_t)(wv & 0xFFFFu);
    xv[t][c2 + 1] = (uint16_t)(wv >> 16);
  }
  __syncthreads();
  quantize_tile(xk, xv, reinterpret_cast<uint8_t*>(rec), p.key_bits, p.val_bits, p.flag);
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(p.groups + ((size_t)seg * p.ng_cap + g) * p.rec_bytes);
  const uint4* src = reinterpret_cast<const uint4*>(rec);
  for (int i = tid; i < p.rec_bytes / 16; i += 256) dst[i] = src[i];
}

// One new token per sequence, each at its own position n0 = n_ctx[b] (one
// CTA per (sequence, KV head)).  A full tail (n0 a positive multiple of 64)
// is first quantized as group n0/64 - 1 and the token starts a new tail;
// else it joins the tail.  The token's rows also go to the exact copy at
// position n0 when one is given.
struct AppendParams {
  uint8_t* groups;
  uint16_t* tail_k;
  uint16_t* tail_v;
  const uint16_t* k_new;  // [n_seg][128]
  const uint16_t* v_new;
  uint16_t* k_exact;      // [n_seg][capacity][128] or null
  uint16_t* v_exact;
  uint32_t* flag;
  int hkv, ng_cap, capacity, key_bits, val_bits, rec_bytes;
  SeqTable seq;           // lengths after the append
};

__global__ void __launch_bounds__(256) append1_kernel(const __grid_constant__ AppendParams p) {
  __shared__ uint16_t xk[kKG][kD + 2];
  __shared__ uint16_t xv[kKG][kD + 2];
  __shared__ __align__(16) uint32_t rec[9728 / 4];
  const int seg = blockIdx.x, tid = threadIdx.x;
  const int n0 = p.seq.n_ctx[seg / p.hkv] - 1;  // the table holds the lengths after
  const int tl = n0 - split_point(n0);  // tail tokens before the append
  const bool flush = tl == kTail;        // n0 a positive multiple of 64
  // Launched as a programmatic dependent: its CTAs are resident when the
  // previous kernel ends, and everything below comes after the wait (the
  // previous step's kernels read the tail slots and the exact copy; the new
  // rows may come from the kernel just before).  The scan that follows may
  // start at once: before its own wait it copies no record of a sequence's
  // last group, the only record written here.
  pdl_launch_dependents();
  pdl_wait();
  if (flush) {
    const int g = n0 / kKG - 1;
    for (int i = tid; i < p.rec_bytes / 4; i += 256) rec[i] = 0u;
    for (int i = tid; i < kKG * kD / 2; i += 256) {
      const int t = i / (kD / 2), c2 = (i % (kD / 2)) * 2;
      const uint32_t wk = reinterpret_cast<const uint32_t*>(p.tail_k + ((size_t)seg * kTail + t) * kD)[c2 / 2];
      const uint32_t wv = reinterpret_cast<const uint32_t*>(p.tail_v + ((size_t)seg * kTail + t) * kD)[c2 / 2];
      xk[t][c2] = (uint16_t)(wk & 0xFFFFu);
      xk[t][c2 + 1] = (uint16_t)(wk >> 16);
      xv[t][c2] = (uint16_t)(wv & 0xFFFFu);
      xv[t][c2 + 1] = (uint16_t)(wv >> 16);
    }
    __syncthreads();
    quantize_tile(xk, xv, reinterpret_cast<uint8_t*>(rec), p.key_bits, p.val_bits, p.flag);
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(p.groups + ((size_t)seg * p.ng_cap + g) * p.rec_bytes);
    const uint4* src = reinterpret_cast<const uint4*>(rec);
    for (int i = tid; i < p.rec_bytes / 16; i += 256) dst[i] = src[i];
  }
  // the token: tail slot (0 after a flush), then the exact copy
  const int slot = flush ? 0 : tl;
  if (tid < 16) {
    const uint4 kv = reinterpret_cast<const uint4*>(p.k_new + (size_t)seg * kD)[tid];
    reinterpret_cast<uint4*>(p.tail_k + ((size_t)seg * kTail + slot) * kD)[tid] = kv;
    if (p.k_exact) reinterpret_cast<uint4*>(p.k_exact + ((size_t)seg * p.capacity + n0) * kD)[tid] = kv;
  } else if (tid < 32) {
    const uint4 vv = reinterpret_cast<const uint4*>(p.v_new + (size_t)seg * kD)[tid - 16];
    reinterpret_cast<uint4*>(p.tail_v + ((size_t)seg * kTail + slot) * kD)[tid - 16] = vv;
    if (p.v_exact) reinterpret_cast<uint4*>(p.v_exact + ((size_t)seg * p.capacity + n0) * kD)[tid - 16] = vv;
  }
}

int launch_append1(const jfa_geom& g, const SeqTable& t, const jfa_cache& c, const uint16_t* k_new,
                   const uint16_t* v_new, uint16_t* k_exact, uint16_t* v_exact, uint32_t* flag,
                   cudaStream_t st) {
  AppendParams p;
  p.groups = static_cast<uint8_t*>(c.groups);
  p.tail_k = c.tail_k;
  p.tail_v = c.tail_v;
  p.k_new = k_new;
  p.v_new = v_new;
  p.k_exact = k_exact;
  p.v_exact = v_exact;
  p.flag = flag;
  p.hkv = g.num_kv_heads;
  p.ng_cap = g.capacity / kKG;
  p.capacity = g.capacity;
  p.key_bits = g.key_bits;
  p.val_bits = g.val_bits;
  p.rec_bytes = record_bytes(g.key_bits, g.val_bits);
  p.seq = t;
  return launch_pdl(append1_kernel, dim3(g.batch * g.num_kv_heads), dim3(256), 0, st, p) == cudaSuccess
             ? JFA_OK
             : JFA_ERR_CUDA;
}

// Tail update: copy new tokens [src0, n_new) to tail slots [dst0, ...).
__global__ void pack_tail_kernel(uint16_t* tail_k, uint16_t* tail_v, const uint16_t* k_new,
                                 const uint16_t* v_new, int n_new, int src0, int dst0, int count) {
  const int seg = blockIdx.y;
  const int nvec = count * (kD / 8);  // uint4 per row = 16
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += gridDim.x * blockDim.x) {
    int t = i / (kD / 8), v = i % (kD / 8);
    size_t s = ((size_t)seg * n_new + src0 + t) * (kD / 8) + v;
    size_t d = ((size_t)seg * kTail + dst0 + t) * (kD / 8) + v;
    reinterpret_cast<uint4*>(tail_k)[d] = reinterpret_cast<const uint4*>(k_new)[s];
    reinterpret_cast<uint4*>(tail_v)[d] = reinterpret_cast<const uint4*>(v_new)[s];
  }
}

int launch_pack(const jfa_geom& g, const jfa_cache& c, const uint16_t* k_new,
                const uint16_t* v_new, int n_new, uint32_t* flag, cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  const int n0 = g.n_ctx, n1 = g.n_ctx + n_new;
  const int nq0 = split_point(n0), nq1 = split_point(n1);
  const int flush = (nq1 - nq0) / kKG;
  if (flush > 0) {
    PackParams p;
    p.groups = static_cast<uint8_t*>(c.groups);
    p.tail_k = c.tail_k;
    p.tail_v = c.tail_v;
    p.k_new = k_new;
    p.v_new = v_new;
    p.flag = flag;
    p.hkv = g.num_kv_heads;
    p.ng_cap = g.capacity / kKG;
    p.n_new = n_new;
    p.n0 = n0;
    p.nq0 = nq0;
    p.g_first = nq0 / kKG;
    p.key_bits = g.key_bits;
    p.val_bits = g.val_bits;
    p.rec_bytes = record_bytes(g.key_bits, g.val_bits);
    pack_groups_kernel<<<dim3(flush, n_seg), 256, 0, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return JFA_ERR_CUDA;
  }
  // new tail = tokens [nq1, n1); the ones that are new come from k_new
  int src0, dst0, count;
  if (nq1 == nq0) {          // no flush: append after the current tail
    src0 = 0;
    dst0 = n0 - nq0;
    count = n_new;
  } else {                   // flushed: the tail restarts at nq1 (all new tokens)
    src0 = nq1 - n0;
    dst0 = 0;
    count = n1 - nq1;
  }
  if (count > 0) {
    int blocks = (count * (kD / 8) + 255) / 256;
    pack_tail_kernel<<<dim3(blocks, n_seg), 256, 0, st>>>(c.tail_k, c.tail_v, k_new, v_new,
                                                          n_new, src0, dst0, count);
    if (cudaGetLastError() != cudaSuccess) return JFA_ERR_CUDA;
  }
  return JFA_OK;
}

}  // namespace jfa
