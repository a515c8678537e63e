// fp4.cu — NVFP4 keys (Jet-QSparse abstract: compact NVFP4 cache storage,
// query-key products in FP4 on Blackwell tensor cores, a dense scan over the
// whole key history that feeds 128-token block selection).
//
//   fp4_pack_kernel   one CTA per (64-token group, segment): the group's
//                     tensor scale s = amax / (6 * 448), per 16 channels of a
//                     token a UE4M3 scale nearest to amax_16 / (6 s), and
//                     E2M1 codes of x / (scale_16 * s) (fp64 quotients);
//   fp4_query_kernel  the same quantization of each query head (one tensor
//                     scale per head) into a query record per segment;
//   fp4_scan_kernel   tcgen05 block-scaled MMA (kind::mxf4nvf4, M = 128
//                     tokens, N = 8 query heads, K = 2 x 64 channels) per
//                     record, fp32 accumulators in tensor memory; the
//                     epilogue scales a token's 8 head logits by its group's
//                     and each head's tensor scale and stores the largest over
//                     the KV head's query heads as the selection score.
// Scan roles per CTA (6 warps, 6 CTAs per SM: a CTA's throughput is set by
// its one-thread issue chains, so more small CTAs beat deeper rings — with 2
// CTAs per SM the scan reached 0.52 of HBM bandwidth at any ring depth, with
// 6 CTAs of 3 stages 0.88): warp 0 streams records (bulk copies into a
// 3-stage ring), warp 1 owns the tensor memory, copies each record's scales
// aside and issues scale copies and MMAs (a stage is free again once its
// MMAs have read it), warps 2-5 read the accumulators (one 32-lane quarter
// each).  Every wait is bounded: on a timeout the kernel records
// JFA_DEVERR_TIMEOUT, lets its copies and MMAs drain, frees its tensor memory
// and returns.
#include "jfa_fp4.cuh"

namespace jfa {

// ---------------------------------------------------------------------------
// pack
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bf16x8(const uint4 v, float* x) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Codes of 16 values x[0..16) against one block unit (bs * s); 8 bytes.
__device__ __forceinline__ uint2 e2m1_block(const float* x, double unit) {
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t c = unit > 0.0 ? e2m1_code((double)x[e] / unit) : 0u;
    w[e >> 3] |= c << (4 * (e & 7));
  }
  return make_uint2(w[0], w[1]);
}

// Thread t: token row r = t / 2 of the group, channels 64 (t mod 2) .. +63.
// The kernel never lets its dependents start early: the scan requests its
// first records before its own dependency wait, which is safe only because
// every kernel after this one starts after it has finished.
__global__ void __launch_bounds__(128) fp4_pack_kernel(const uint16_t* __restrict__ k_src,
                                                       uint8_t* __restrict__ pool, int capacity,
                                                       int g_from, uint32_t* flag) {
  __shared__ float red[4];
  const int seg = blockIdx.y, gi = g_from + blockIdx.x, t = threadIdx.x;
  const int r = t >> 1, half = t & 1;
  const uint16_t* src = k_src + ((size_t)seg * capacity + (size_t)gi * kKG + r) * kD + 64 * half;
  float x[64];
#pragma unroll
  for (int i = 0; i < 8; ++i) bf16x8(*reinterpret_cast<const uint4*>(src + 8 * i), x + 8 * i);
  float am = 0.f;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    am = fmaxf(am, fabsf(x[i]));
    finite &= isfinite(x[i]);
  }
  if (!__all_sync(0xFFFFFFFFu, finite) && (t & 31) == 0) set_flag(flag, JFA_DEVERR_NONFINITE_QUANT);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
  if ((t & 31) == 0) red[t >> 5] = am;
  __syncthreads();
  am = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float s = nvfp4_tensor_scale(am);
  const double sd = s, s6 = kE2M1Max * sd;

  uint8_t* rec = pool + ((size_t)seg * (capacity / kF4Tok) + gi / 2) * kF4RecBytes;
  const int row = kKG * (gi & 1) + r;
  uint32_t sfw = 0u;
  uint2 cw[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float ab = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) ab = fmaxf(ab, fabsf(x[16 * j + e]));
    const double bs = e4m3_rn_pos((double)ab / s6);
    sfw |= e4m3_bits(bs) << (8 * j);
    cw[j] = e2m1_block(x + 16 * j, bs * sd);
  }
  // channels 64 half + [0, 32) and + [32, 64): two 16-byte column chunks
  *reinterpret_cast<uint4*>(rec + f4_code_off(row, 64 * half)) =
      make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
  *reinterpret_cast<uint4*>(rec + f4_code_off(row, 64 * half + 32)) =
      make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
  *reinterpret_cast<uint32_t*>(rec + kF4SfOff + f4_sf_off(row, 4 * half)) = sfw;
  if (t == 0) reinterpret_cast<float*>(rec + kF4GsOff)[gi & 1] = s;
}

int launch_fp4_pack(const jfa_geom& g, int g_from, int g_to, const uint16_t* k_src, uint8_t* pool,
                    uint32_t* flag, cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  if (g_to <= g_from) return JFA_OK;
  fp4_pack_kernel<<<dim3(g_to - g_from, n_seg), 128, 0, st>>>(k_src, pool, g.capacity, g_from, flag);
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// query records: thread t quantizes channels 8 (t mod 16) .. +7 of head t / 16
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) fp4_query_kernel(const uint16_t* __restrict__ q, int H,
                                                        int Hkv, int G, uint8_t* __restrict__ qrec,
                                                        uint32_t* __restrict__ bkeys, int nb_cap) {
  __shared__ __align__(16) uint8_t rec[kF4QBytes];
  const int seg = blockIdx.x, b = seg / Hkv, kvh = seg % Hkv, t = threadIdx.x;
  const int h = t >> 4, c0 = (t & 15) * 8;
  for (int i = t; i < kF4QBytes / 16; i += 128) reinterpret_cast<uint4*>(rec)[i] = make_uint4(0, 0, 0, 0);
  pdl_launch_dependents();  // the scan's set-up may overlap; it waits for this grid before reading
  pdl_wait();
  float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (h < G) bf16x8(*reinterpret_cast<const uint4*>(q + ((size_t)b * H + kvh * G + h) * kD + c0), x);
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(x[i]));
  float ab = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));  // the 16-channel block
#pragma unroll
  for (int o = 2; o < 16; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
  am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));        // the head's 128 channels
  __syncthreads();
  if (h < G) {
    const float s = nvfp4_tensor_scale(am);
    const double sd = s;
    const double bs = e4m3_rn_pos((double)ab / (kE2M1Max * sd));
    uint32_t w = 0u;
    const double unit = bs * sd;
#pragma unroll
    for (int e = 0; e < 8; ++e) w |= (unit > 0.0 ? e2m1_code((double)x[e] / unit) : 0u) << (4 * e);
    *reinterpret_cast<uint32_t*>(rec + f4_code_off(h, c0)) = w;
    if ((t & 1) == 0) rec[kF4QSfOff + f4_sf_off(h, c0 >> 4)] = (uint8_t)e4m3_bits(bs);
    if ((t & 15) == 0) reinterpret_cast<float*>(rec + kF4QScaleOff)[h] = s;
  }
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(qrec + (size_t)seg * kF4QBytes);
  for (int i = t; i < kF4QBytes / 16; i += 128) dst[i] = reinterpret_cast<const uint4*>(rec)[i];
  // the scan raises every block key of this segment from zero
  for (int i = t; i < nb_cap; i += 128) bkeys[(size_t)seg * nb_cap + i] = 0u;
}

// ---------------------------------------------------------------------------
// tcgen05 scan
// ---------------------------------------------------------------------------
#ifndef JFA_F4_STAGES
#define JFA_F4_STAGES 3
#endif
#ifndef JFA_F4_CTAS_PER_SM
#define JFA_F4_CTAS_PER_SM 6
#endif
constexpr int kF4Stages = JFA_F4_STAGES;
constexpr int kF4StageStride = 11264;  // record, then the query record at +kF4QStageOff
constexpr int kF4QStageOff = 9344;
constexpr int kF4Acc = 4;              // accumulator buffers (8 columns each)
constexpr int kF4Threads = 192;
constexpr uint32_t kF4TmemCols = 64;   // [0,32) accumulators, [32,48) A scales, [48,64) B scales
constexpr int kF4Smem = kF4Stages * kF4StageStride + 1024;
static_assert(kF4QStageOff >= kF4RecBytes && kF4QStageOff % 128 == 0, "query record after the record");
static_assert(kF4QStageOff + kF4QBytes <= kF4StageStride, "stage holds both records");
static_assert(JFA_F4_CTAS_PER_SM * 64 <= 512, "tensor memory of the CTAs of one SM");

struct Fp4ScanParams {
  const uint8_t* pool;
  const uint8_t* qrec;
  float* scores;
  uint32_t* bkeys;  // [seg][nb_cap]: largest selection key of each record
  uint32_t* flag;
  long long total_tiles;
  int tiles_per_cta;
  int capacity;
  int nb_cap;  // records per segment in the pool
  int nts;     // tiles (records) scanned per segment
  int nq;
  int G;
  float scale;
};

// Shared-memory matrix descriptor, K-major, no swizzle: start address,
// leading-dimension byte offset (between the two 16-byte column chunks of
// one MMA's K), stride byte offset (between 8-row groups), version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Instruction descriptor of kind::mxf4nvf4: A and B E2M1 (1), K-major,
// UE4M3 scales (0), N = 8, M = 128, K = 64 per instruction.
constexpr uint32_t kF4Idesc = (1u << 7) | (1u << 10) | ((8u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 128 rows x 4 scale bytes (one 512-byte atom) into 4 columns of every
// tensor-memory lane quarter.
__device__ __forceinline__ void tc_copy_scales(uint32_t taddr, uint32_t saddr) {
  const uint64_t d = umma_desc(saddr, 0u, 128u);
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}
__device__ __forceinline__ void tc_mma_fp4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t sfa,
                                           uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %6, [%3], [%4], p;\n\t"
      "}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(sfa), "r"(sfb), "r"(accumulate), "r"(kF4Idesc)
      : "memory");
}

__global__ void __launch_bounds__(kF4Threads, 1) fp4_scan_kernel(const __grid_constant__ Fp4ScanParams p) {
  extern __shared__ uint8_t f4raw[];
  __shared__ __align__(8) uint64_t full[kF4Stages], empty[kF4Stages], tfull[kF4Acc], tempty[kF4Acc];
  // per accumulator buffer: the record's two group scales (times the softmax
  // scale) and the query heads' scales, copied out of the stage by the MMA
  // thread so that the stage is free as soon as the MMAs have read it
  __shared__ float s_scales[kF4Acc][2 + kMaxG];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(f4raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long t0 = (long long)blockIdx.x * p.tiles_per_cta;
  const long long left = p.total_tiles - t0;
  const int n_my = left <= 0 ? 0 : (int)(left < p.tiles_per_cta ? left : p.tiles_per_cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kF4Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kF4Acc; ++b) {
      mbar_init(&tfull[b], 2);  // the MMA thread's scales, then the MMAs
      mbar_init(&tempty[b], 4);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kF4TmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ---- producer: record + query record per tile into the ring.  The
    // records of the first stages are requested before the wait on the
    // previous kernel (the query kernel, which writes no record; the pool's
    // writer finished before that kernel began), their query records after.
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int n_first = n_my < kF4Stages ? n_my : kF4Stages;
      for (int i = 0; i < n_first; ++i) {
        const long long tile = t0 + i;
        const int seg = (int)(tile / p.nts), tb = (int)(tile % p.nts);
        mbar_expect_tx(&full[i], kF4RecBytes + kF4QBytes);
        bulk_g2s(base + i * kF4StageStride, p.pool + ((size_t)seg * p.nb_cap + tb) * kF4RecBytes,
                 kF4RecBytes, &full[i], pol);
      }
      pdl_wait();
      for (int i = 0; i < n_first; ++i) {
        const int seg = (int)((t0 + i) / p.nts);
        bulk_g2s_nohint(base + i * kF4StageStride + kF4QStageOff, p.qrec + (size_t)seg * kF4QBytes,
                        kF4QBytes, &full[i]);
      }
      int issued = n_first;
      for (int i = n_first; i < n_my; ++i) {
        const int s = i % kF4Stages;
        const uint32_t ph = (uint32_t)(i / kF4Stages) & 1u;
        if (i >= kF4Stages && !mbar_wait_bounded(&empty[s], ph ^ 1u)) {
          set_flag(p.flag, JFA_DEVERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        if (*(volatile int*)&s_abort) break;
        const long long tile = t0 + i;
        const int seg = (int)(tile / p.nts), tb = (int)(tile % p.nts);
        uint8_t* st = base + s * kF4StageStride;
        mbar_expect_tx(&full[s], kF4RecBytes + kF4QBytes);
        bulk_g2s(st, p.pool + ((size_t)seg * p.nb_cap + tb) * kF4RecBytes, kF4RecBytes, &full[s], pol);
        bulk_g2s_nohint(st + kF4QStageOff, p.qrec + (size_t)seg * kF4QBytes, kF4QBytes, &full[s]);
        issued = i + 1;
      }
      // let every copy land before the CTA can leave
      for (int i = issued > kF4Stages ? issued - kF4Stages : 0; i < issued; ++i)
        if (!mbar_wait_bounded(&full[i % kF4Stages], (uint32_t)(i / kF4Stages) & 1u)) {
          set_flag(p.flag, JFA_DEVERR_TIMEOUT);
          break;
        }
    }
  } else if (warp == 1) {
    // ---- MMA issuer
    pdl_wait();
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_my; ++i) {
        const int s = i % kF4Stages, b = i % kF4Acc;
        const uint32_t ph = (uint32_t)(i / kF4Stages) & 1u, bph = (uint32_t)(i / kF4Acc) & 1u;
        bool ok = mbar_wait_bounded(&full[s], ph);
        if (ok && i >= kF4Acc) ok = mbar_wait_bounded(&tempty[b], bph ^ 1u);
        if (!ok) {
          set_flag(p.flag, JFA_DEVERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        if (*(volatile int*)&s_abort) break;
        tc_fence_after();
        {
          const uint8_t* sp = base + s * kF4StageStride;
          const float* gs = reinterpret_cast<const float*>(sp + kF4GsOff);
          const float* qs = reinterpret_cast<const float*>(sp + kF4QStageOff + kF4QScaleOff);
          s_scales[b][0] = gs[0] * p.scale;
          s_scales[b][1] = gs[1] * p.scale;
#pragma unroll
          for (int h = 0; h < kMaxG; ++h) s_scales[b][2 + h] = qs[h];
          mbar_arrive1(&tfull[b]);
        }
        const uint32_t st = smem_u32(base + s * kF4StageStride);
        const uint32_t sfa = tmem + 32u + 8u * (uint32_t)(i & 1), sfb = tmem + 48u + 8u * (uint32_t)(i & 1);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          tc_copy_scales(sfa + 4u * kk, st + kF4SfOff + 512u * kk);
          tc_copy_scales(sfb + 4u * kk, st + kF4QStageOff + kF4QSfOff + 512u * kk);
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          tc_mma_fp4(tmem + 8u * b, umma_desc(st + 256u * kk, 128u, 512u),
                     umma_desc(st + kF4QStageOff + 256u * kk, 128u, 512u), sfa + 4u * kk, sfb + 4u * kk,
                     (uint32_t)kk);
        tc_commit(&empty[s]);
        tc_commit(&tfull[b]);
        issued = i + 1;
      }
      // the last commit covers every MMA issued: wait for it before the
      // tensor memory can be freed
      if (issued > 0 &&
          !mbar_wait_bounded(&tfull[(issued - 1) % kF4Acc], (uint32_t)((issued - 1) / kF4Acc) & 1u))
        set_flag(p.flag, JFA_DEVERR_TIMEOUT);
    }
  } else {
    // ---- epilogue: warp w reads lanes 32 (w mod 4) .. + 31 (its tokens)
    pdl_wait();
    const int sub = warp & 3, row = 32 * sub + lane;
    for (int i = 0; i < n_my; ++i) {
      const int b = i % kF4Acc;
      const uint32_t bph = (uint32_t)(i / kF4Acc) & 1u;
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&tfull[b], bph));
      if (!ok) {
        if (lane == 0) {
          set_flag(p.flag, JFA_DEVERR_TIMEOUT);
          s_abort = 1;
        }
        break;
      }
      tc_fence_after();
      uint32_t d[8];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
          : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]),
            "=r"(d[7])
          : "r"(tmem + ((uint32_t)(32 * sub) << 16) + 8u * b));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      const float sk = s_scales[b][row >> 6];
      float sq[kMaxG];
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) sq[h] = s_scales[b][2 + h];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&tempty[b]);  // accumulator and scales free
      float sel = -INFINITY;
#pragma unroll
      for (int h = 0; h < kMaxG; ++h)
        if (h < p.G) sel = fmaxf(sel, __uint_as_float(d[h]) * (sk * sq[h]));
      const long long tile = t0 + i;
      const int seg = (int)(tile / p.nts), tb = (int)(tile % p.nts), tok = tb * kF4Tok + row;
      if (tok < p.nq) p.scores[(size_t)seg * p.capacity + tok] = sel;
      // the block key: the largest selection score of the record's tokens
      const uint32_t bk = __reduce_max_sync(0xFFFFFFFFu, tok < p.nq ? float_key(sel) : 0u);
      if (lane == 0) atomicMax(p.bkeys + (size_t)seg * p.nb_cap + tb, bk);
    }
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kF4TmemCols)
                 : "memory");
  }
}

int launch_fp4_scores(const jfa_geom& g, const uint8_t* pool, const uint16_t* q, float scale,
                      uint8_t* ws, const jfa_workspace_layout& L, cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads, G = g.num_heads / g.num_kv_heads;
  const int nq = split_point(g.n_ctx);
  uint8_t* qrec = ws + L.off_fp4q;
  uint32_t* flag = reinterpret_cast<uint32_t*>(ws + L.off_flag);
  uint32_t* bkeys = reinterpret_cast<uint32_t*>(ws + L.off_bkeys);
  if (launch_pdl(fp4_query_kernel, dim3(n_seg), dim3(128), 0, st, q, g.num_heads, g.num_kv_heads, G,
                 qrec, bkeys, g.capacity / kF4Tok) != cudaSuccess)
    return JFA_ERR_CUDA;
  if (nq == 0) return JFA_OK;
  // Dynamic shared memory: the ring, padded so that at most
  // JFA_F4_CTAS_PER_SM CTAs share an SM (their tensor-memory allocations,
  // 64 columns each, then always fit the SM's 512 columns).
  static int smem_dev = -1;
  static size_t smem = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return JFA_ERR_CUDA;
  if (dev != smem_dev) {
    int per_sm = 0;
    if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
      return JFA_ERR_CUDA;
    const size_t floor_bytes = (size_t)per_sm / (JFA_F4_CTAS_PER_SM + 1) + 1;  // N + 1 do not fit
    const size_t need = (size_t)kF4Smem + 1024;  // + the per-CTA reservation
    smem = (need > floor_bytes ? need : floor_bytes) - 1024;
    if (cudaFuncSetAttribute(fp4_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return JFA_ERR_CUDA;
    smem_dev = dev;
  }
  Fp4ScanParams p;
  p.pool = pool;
  p.qrec = qrec;
  p.scores = reinterpret_cast<float*>(ws + L.off_scores);
  p.bkeys = bkeys;
  p.flag = flag;
  p.capacity = g.capacity;
  p.nb_cap = g.capacity / kF4Tok;
  p.nts = (nq + kF4Tok - 1) / kF4Tok;
  p.nq = nq;
  p.G = G;
  p.scale = scale;
  p.total_tiles = (long long)n_seg * p.nts;
  const long long slots = (long long)JFA_F4_CTAS_PER_SM * num_sms_current();
  const long long n_ctas0 = p.total_tiles < slots ? p.total_tiles : slots;
  p.tiles_per_cta = (int)((p.total_tiles + n_ctas0 - 1) / n_ctas0);
  const int n_ctas = (int)((p.total_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta);
  return launch_pdl(fp4_scan_kernel, dim3(n_ctas), dim3(kF4Threads), smem, st, p) ==
                 cudaSuccess
             ? JFA_OK
             : JFA_ERR_CUDA;
}

}  // namespace jfa
