// api.cu — the C ABI declared in include/jfa.h: argument validation, buffer
// layouts, launch plans and the host-side record decoder.
#include <string.h>

#include "jfa_fp4.cuh"

namespace jfa {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static bool geom_ok(const jfa_geom* g) {
  if (!g) return false;
  if (g->batch < 1 || g->num_heads < 1 || g->num_kv_heads < 1) return false;
  if (g->num_heads % g->num_kv_heads != 0) return false;
  const int G = g->num_heads / g->num_kv_heads;
  if (G > kMaxG) return false;
  if (g->head_dim != kD) return false;
  if (g->capacity < kKG || g->capacity % kKG != 0) return false;
  if (g->key_bits != 3 && g->key_bits != 4) return false;
  if (g->val_bits != 2 && g->val_bits != 4) return false;
  if (g->n_ctx < 0 || g->n_ctx > g->capacity) return false;
  return true;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int workspace_layout(const jfa_geom& g, int max_topk, jfa_workspace_layout* out) {
  const size_t n_seg = (size_t)g.batch * g.num_kv_heads;
  const size_t G = (size_t)(g.num_heads / g.num_kv_heads);
  jfa_workspace_layout L;
  memset(&L, 0, sizeof(L));
  size_t off = 0;
  L.off_flag = off;
  off += 256;
  L.off_scores = off;
  off = align_up(off + n_seg * g.capacity * sizeof(float), 256);
  L.partial_slots = (int32_t)(kMaxScanWarps + n_seg);
  L.off_partials = off;
  off = align_up(off + (size_t)L.partial_slots * G * kPartStride * sizeof(float), 256);
  L.off_mused = off;
  off = align_up(off + n_seg * (size_t)(g.capacity / kKG) * kMaxG * sizeof(float), 256);
  L.off_wts = off;
  off = align_up(off + n_seg * (size_t)(g.capacity / kKG) * 4 * (G > 4 ? 2 : 1) * 32 * sizeof(uint32_t), 256);
  L.off_scan_hist = off;
  off = align_up(off + n_seg * (size_t)scan_hist_reps((long long)n_seg) * kScanHistStride * sizeof(uint32_t), 256);
  L.off_hist = off;
  off += n_seg * kHistBins * sizeof(uint32_t);
  L.off_counters = off;
  off = align_up(off + n_seg * 8 * sizeof(uint32_t), 256);
  // top-k lists: per 4096-score chunk, up to 4096 (key, index) pairs; then counts
  // (also holds the per-CTA lists of the fused finishing kernel: slices of
  // the quantized tokens rounded up to 64, <= capacity + 64 per CTA)
  const size_t n_chunks_cap = ((size_t)g.capacity + 4095) / 4096;
  const size_t cap_fused = (size_t)g.capacity + 64 * kFinMaxCluster;
  L.cand_cap = (int32_t)(n_chunks_cap * 4096 > cap_fused ? n_chunks_cap * 4096 : cap_fused);
  L.off_cand = off;
  off = align_up(off + n_seg * (size_t)L.cand_cap * 2 * sizeof(uint32_t), 256);
  L.max_topk = max_topk;
  L.off_sel = off;
  off = align_up(off + n_seg * n_chunks_cap * sizeof(uint32_t), 256);
  L.off_fp4q = off;
  off = align_up(off + n_seg * kF4QBytes, 256);
  L.off_sparse = off;
  off = align_up(off + (n_seg > (size_t)kSpSlots ? n_seg : (size_t)kSpSlots) * kMaxG * 132 * sizeof(float), 256);
  L.off_ticket = off;
  off = align_up(off + n_seg * sizeof(uint32_t), 256);
  L.off_bkeys = off;
  off = align_up(off + n_seg * (size_t)((g.capacity + kF4Tok - 1) / kF4Tok) * sizeof(uint32_t), 256);
  L.off_chan = off;
  off = align_up(off + n_seg * (size_t)kChanRecBytes, 256);
  L.off_qstage = off;
  off = align_up(off + (size_t)g.batch * g.num_heads * kD * sizeof(uint16_t), 256);
  L.total_bytes = off;
  *out = L;
  return JFA_OK;
}

int num_sms_current() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

bool fill_seq_table(const jfa_geom& g, const int32_t* lens, SeqTable* t) {
  if (g.batch < 1 || g.batch > kMaxBatch) return false;
  memset(t, 0, sizeof(*t));
  int32_t acc = 0;
  for (int b = 0; b < g.batch; ++b) {
    const int32_t n = lens ? lens[b] : g.n_ctx;
    if (n < 1 || n > g.capacity) return false;
    t->n_ctx[b] = n;
    t->gpre[b] = acc;
    acc += g.num_kv_heads * seq_groups(*t, b);
  }
  t->gpre[g.batch] = acc;
  return true;
}

int max_nq(const jfa_geom& g, const SeqTable& t) {
  int m = 0;
  for (int b = 0; b < g.batch; ++b) m = t.n_ctx[b] > m ? t.n_ctx[b] : m;
  return split_point(m);
}

ScanPlan scan_plan(const jfa_geom& g, const SeqTable& t, int num_sms) {
  ScanPlan p;
  p.total_groups = t.gpre[g.batch];
  const int nw = scan_cta_warps(g.key_bits, g.val_bits, g.num_heads / g.num_kv_heads > 4 ? 2 : 1);
  long long w = (long long)num_sms * nw;
  if (w > kMaxScanWarps) w = kMaxScanWarps;
  const long long w_min_rec = (p.total_groups + kScanMinRecords - 1) / kScanMinRecords;
  if (w > w_min_rec) w = w_min_rec;
  if (w < 1) w = 1;
  if (w > p.total_groups) w = p.total_groups;
  p.n_warps = (int)w;
  p.n_ctas = (int)((w + nw - 1) / nw);
  return p;
}

}  // namespace jfa

using namespace jfa;

// selftest.cu: one warp waits on an mbarrier that never completes; the
// bounded wait sets JFA_DEVERR_TIMEOUT in *flag.
namespace jfa {
int launch_bounded_wait_selftest(uint32_t* flag, cudaStream_t st);
}

extern "C" {

const char* jfa_status_string(int status) {
  switch (status) {
    case JFA_OK: return "ok";
    case JFA_ERR_INVALID_ARG: return "invalid argument";
    case JFA_ERR_UNSUPPORTED: return "unsupported";
    case JFA_ERR_CUDA: return "CUDA error";
    case JFA_ERR_DEVICE: return "device error flag set";
    default: return "unknown status";
  }
}

int jfa_cache_layout_get(const jfa_geom* geom, jfa_cache_layout* out) {
  if (!geom_ok(geom) || !out) return JFA_ERR_INVALID_ARG;
  const size_t n_seg = (size_t)geom->batch * geom->num_kv_heads;
  out->record_bytes = (size_t)record_bytes(geom->key_bits, geom->val_bits);
  out->groups_bytes = n_seg * (geom->capacity / kKG) * out->record_bytes;
  out->tail_bytes = n_seg * kTail * kD * sizeof(uint16_t);
  out->off_key_scales = (size_t)off_ks();
  out->off_key_codes = (size_t)off_kc();
  out->off_val_scales = (size_t)off_vs(geom->key_bits);
  out->off_val_codes = (size_t)off_vc(geom->key_bits);
  return JFA_OK;
}

int jfa_workspace_layout_get(const jfa_geom* geom, int32_t max_topk, jfa_workspace_layout* out) {
  if (!geom_ok(geom) || !out || max_topk < 1 || max_topk > JFA_MAX_TOPK)
    return JFA_ERR_INVALID_ARG;
  return workspace_layout(*geom, max_topk, out);
}

static bool cache_ok(const jfa_cache* c) {
  return c && c->groups && c->tail_k && c->tail_v && aligned(c->groups, 16) &&
         aligned(c->tail_k, 16) && aligned(c->tail_v, 16);
}

int jfa_pack_kv(const jfa_geom* geom, const jfa_cache* cache, const uint16_t* k_new,
                const uint16_t* v_new, int32_t n_new, void* ws, void* stream) {
  if (!geom_ok(geom) || !cache_ok(cache) || !ws || !aligned(ws, 256)) return JFA_ERR_INVALID_ARG;
  if (n_new < 0 || (long long)geom->n_ctx + n_new > geom->capacity) return JFA_ERR_INVALID_ARG;
  if (n_new == 0) return JFA_OK;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_pack(*geom, *cache, k_new, v_new, n_new,
                     reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + L.off_flag),
                     static_cast<cudaStream_t>(stream));
}

int jfa_decode_scores(const jfa_geom* geom, const jfa_cache* cache, const uint16_t* q,
                      float scale, void* ws, void* stream) {
  if (!geom_ok(geom) || !cache_ok(cache) || !ws || !aligned(ws, 256)) return JFA_ERR_INVALID_ARG;
  if (geom->n_ctx < 1 || !q || !aligned(q, 16) || !(scale > 0.f) || scale != scale)
    return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  SeqTable t;
  if (!fill_seq_table(*geom, nullptr, &t)) return JFA_ERR_INVALID_ARG;
  return launch_scores(*geom, t, *cache, q, scale, static_cast<uint8_t*>(ws), L,
                       static_cast<cudaStream_t>(stream));
}

int jfa_topk(const jfa_geom* geom, int32_t k, void* ws, int32_t* idx, void* stream) {
  if (!geom_ok(geom) || !ws || !aligned(ws, 256) || !idx || !aligned(idx, 4))
    return JFA_ERR_INVALID_ARG;
  if (geom->n_ctx < 1 || k < 1 || k > JFA_MAX_TOPK) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, k, &L);
  return launch_topk(*geom, k, static_cast<uint8_t*>(ws), L, idx,
                     static_cast<cudaStream_t>(stream));
}

int jfa_topk_blocks(const jfa_geom* geom, int32_t n_blocks, void* ws, int32_t* idx, void* stream) {
  if (!geom_ok(geom) || !ws || !aligned(ws, 256) || !idx || !aligned(idx, 4))
    return JFA_ERR_INVALID_ARG;
  if (geom->n_ctx < 1 || n_blocks < 1 || n_blocks > JFA_MAX_BLOCKS) return JFA_ERR_INVALID_ARG;
  if ((split_point(geom->n_ctx) + JFA_BLOCK_TOKENS - 1) / JFA_BLOCK_TOKENS > kMaxSelBlocks)
    return JFA_ERR_UNSUPPORTED;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_topk_blocks(*geom, n_blocks, static_cast<uint8_t*>(ws), L, idx,
                            static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// NVFP4 keys and block-sparse exact attention
// ---------------------------------------------------------------------------
static bool fp4_geom_ok(const jfa_geom* g) { return geom_ok(g) && g->capacity % kF4Tok == 0; }

int jfa_fp4_pool_bytes(const jfa_geom* geom, size_t* pool_bytes) {
  if (!fp4_geom_ok(geom) || !pool_bytes) return JFA_ERR_INVALID_ARG;
  *pool_bytes = (size_t)geom->batch * geom->num_kv_heads * (geom->capacity / kF4Tok) * kF4RecBytes;
  return JFA_OK;
}

int jfa_fp4_pack_keys(const jfa_geom* geom, int32_t n_from, int32_t n_to, const uint16_t* k_src,
                      void* pool, void* ws, void* stream) {
  if (!fp4_geom_ok(geom) || !pool || !aligned(pool, 16) || !ws || !aligned(ws, 256))
    return JFA_ERR_INVALID_ARG;
  if (n_from < 0 || n_to < n_from || n_to > geom->capacity || n_from % kKG || n_to % kKG)
    return JFA_ERR_INVALID_ARG;
  if (n_to == n_from) return JFA_OK;
  if (!k_src || !aligned(k_src, 16)) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_fp4_pack(*geom, n_from / kKG, n_to / kKG, k_src, static_cast<uint8_t*>(pool),
                         reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + L.off_flag),
                         static_cast<cudaStream_t>(stream));
}

static bool fp4_scan_args_ok(const jfa_geom* geom, const void* pool, const uint16_t* q, float scale,
                             const void* ws) {
  return fp4_geom_ok(geom) && geom->n_ctx >= 1 && pool && aligned(pool, 16) && q && aligned(q, 16) &&
         scale > 0.f && ws && aligned(ws, 256);
}

int jfa_fp4_scores(const jfa_geom* geom, const void* pool, const uint16_t* q, float scale, void* ws,
                   void* stream) {
  if (!fp4_scan_args_ok(geom, pool, q, scale, ws)) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_fp4_scores(*geom, static_cast<const uint8_t*>(pool), q, scale, static_cast<uint8_t*>(ws),
                           L, static_cast<cudaStream_t>(stream));
}

static bool sparse_args_ok(const jfa_geom* geom, const uint16_t* q, float scale, const int32_t* idx,
                           int32_t k, const uint16_t* k_exact, const uint16_t* v_exact, const void* ws,
                           const float* out) {
  return geom_ok(geom) && geom->n_ctx >= 1 && q && aligned(q, 16) && scale > 0.f && idx &&
         aligned(idx, 4) && k >= 1 && k <= JFA_MAX_EXACT && k_exact && v_exact && aligned(k_exact, 16) &&
         aligned(v_exact, 16) && ws && aligned(ws, 256) && out && aligned(out, 16);
}

int jfa_sparse_attend(const jfa_geom* geom, const uint16_t* q, float scale, const int32_t* idx,
                      int32_t k, const uint16_t* k_exact, const uint16_t* v_exact,
                      int32_t exact_on_host, void* ws, float* out, void* stream) {
  if (!sparse_args_ok(geom, q, scale, idx, k, k_exact, v_exact, ws, out)) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_sparse_attend(*geom, q, scale, idx, k, k_exact, v_exact, exact_on_host != 0,
                              static_cast<uint8_t*>(ws), L, out, static_cast<cudaStream_t>(stream));
}

int jfa_fp4_decode_step(const jfa_geom* geom, const void* pool, const uint16_t* q, float scale,
                        int32_t n_blocks, int32_t* idx, const uint16_t* k_exact,
                        const uint16_t* v_exact, int32_t exact_on_host, void* ws, float* out,
                        void* stream) {
  if (!fp4_scan_args_ok(geom, pool, q, scale, ws)) return JFA_ERR_INVALID_ARG;
  if (n_blocks < 1 || n_blocks > JFA_MAX_BLOCKS) return JFA_ERR_INVALID_ARG;
  const int k = n_blocks * JFA_BLOCK_TOKENS;
  if (!sparse_args_ok(geom, q, scale, idx, k, k_exact, v_exact, ws, out)) return JFA_ERR_INVALID_ARG;
  if ((split_point(geom->n_ctx) + JFA_BLOCK_TOKENS - 1) / JFA_BLOCK_TOKENS > kMaxSelBlocks)
    return JFA_ERR_UNSUPPORTED;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  uint8_t* w = static_cast<uint8_t*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = launch_fp4_scores(*geom, static_cast<const uint8_t*>(pool), q, scale, w, L, st);
  // the scan leaves every block's largest score in the block keys
  if (rc == JFA_OK)
    rc = launch_topk_blocks(*geom, n_blocks, w, L, idx, st,
                            reinterpret_cast<const uint32_t*>(w + L.off_bkeys));
  if (rc == JFA_OK)
    rc = launch_sparse_attend(*geom, q, scale, idx, k, k_exact, v_exact, exact_on_host != 0, w, L, out, st);
  return rc;
}

// ---------------------------------------------------------------------------
// critical-channel selection
// ---------------------------------------------------------------------------
int jfa_channel_pack(const jfa_geom* geom, int32_t n_from, int32_t n_to, const uint16_t* k_src,
                     uint16_t* k_t, float* k_max, void* stream) {
  if (!geom_ok(geom) || !k_t || !aligned(k_t, 16) || !k_max || !aligned(k_max, 4))
    return JFA_ERR_INVALID_ARG;
  if (n_from < 0 || n_to < n_from || n_to > geom->capacity || n_from % kKG || n_to % kKG)
    return JFA_ERR_INVALID_ARG;
  if (n_to == n_from) return JFA_OK;
  if (!k_src || !aligned(k_src, 16)) return JFA_ERR_INVALID_ARG;
  return launch_channel_pack(*geom, n_from / kKG, n_to / kKG, k_src, k_t, k_max,
                             static_cast<cudaStream_t>(stream));
}

static bool channel_args_ok(const jfa_geom* geom, const uint16_t* k_t, const float* k_max,
                            const uint16_t* q, float scale, int32_t r, const void* ws) {
  return geom_ok(geom) && geom->n_ctx >= 1 && k_t && aligned(k_t, 16) && k_max && aligned(k_max, 4) &&
         q && aligned(q, 16) && scale > 0.f && r >= 1 && r <= kD && ws && aligned(ws, 256);
}

int jfa_channel_scores(const jfa_geom* geom, const uint16_t* k_t, const float* k_max,
                       const uint16_t* q, float scale, int32_t r, void* ws, void* stream) {
  if (!channel_args_ok(geom, k_t, k_max, q, scale, r, ws)) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_channel_scores(*geom, k_t, k_max, q, scale, r, static_cast<uint8_t*>(ws), L,
                               static_cast<cudaStream_t>(stream));
}

int jfa_channel_decode_step(const jfa_geom* geom, const uint16_t* k_t, const float* k_max,
                            const uint16_t* q, float scale, int32_t r, int32_t k, int32_t* idx,
                            const uint16_t* k_exact, const uint16_t* v_exact,
                            int32_t exact_on_host, void* ws, float* out, void* stream) {
  if (!channel_args_ok(geom, k_t, k_max, q, scale, r, ws)) return JFA_ERR_INVALID_ARG;
  if (k < 1 || k > JFA_MAX_TOPK) return JFA_ERR_INVALID_ARG;
  if (!sparse_args_ok(geom, q, scale, idx, k, k_exact, v_exact, ws, out)) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, k, &L);
  uint8_t* w = static_cast<uint8_t*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = launch_channel_scores(*geom, k_t, k_max, q, scale, r, w, L, st);
  if (rc == JFA_OK) rc = launch_topk(*geom, k, w, L, idx, st);
  if (rc == JFA_OK)
    rc = launch_sparse_attend(*geom, q, scale, idx, k, k_exact, v_exact, exact_on_host != 0, w, L, out, st);
  return rc;
}

// ---------------------------------------------------------------------------
// 1-bit KV cache, dense attention
// ---------------------------------------------------------------------------
int jfa_onebit_pool_bytes(const jfa_geom* geom, size_t* pool_bytes) {
  if (!geom_ok(geom) || !pool_bytes) return JFA_ERR_INVALID_ARG;
  *pool_bytes = (size_t)geom->batch * geom->num_kv_heads * (geom->capacity / kKG) * kOneBitRecBytes;
  return JFA_OK;
}

int jfa_onebit_pack(const jfa_geom* geom, int32_t n_from, int32_t n_to, const uint16_t* k_src,
                    const uint16_t* v_src, void* pool, void* ws, void* stream) {
  if (!geom_ok(geom) || !pool || !aligned(pool, 16) || !ws || !aligned(ws, 256))
    return JFA_ERR_INVALID_ARG;
  if (n_from < 0 || n_to < n_from || n_to > geom->capacity || n_from % kKG || n_to % kKG)
    return JFA_ERR_INVALID_ARG;
  if (n_to == n_from) return JFA_OK;
  if (!k_src || !v_src || !aligned(k_src, 16) || !aligned(v_src, 16)) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_onebit_pack(*geom, n_from / kKG, n_to / kKG, k_src, v_src, static_cast<uint8_t*>(pool),
                            reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + L.off_flag),
                            static_cast<cudaStream_t>(stream));
}

int jfa_onebit_attend(const jfa_geom* geom, const void* pool, const uint16_t* q, float scale,
                      const uint16_t* k_exact, const uint16_t* v_exact, int32_t exact_on_host,
                      void* ws, float* out, void* stream) {
  if (!geom_ok(geom) || geom->n_ctx < 1 || !pool || !aligned(pool, 16) || !q || !aligned(q, 16) ||
      !(scale > 0.f) || !k_exact || !v_exact || !aligned(k_exact, 16) || !aligned(v_exact, 16) || !ws ||
      !aligned(ws, 256) || !out || !aligned(out, 16))
    return JFA_ERR_INVALID_ARG;
  (void)exact_on_host;  // the tail rows are read with plain loads either way
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_onebit_attend(*geom, static_cast<const uint8_t*>(pool), q, scale, k_exact, v_exact,
                              static_cast<uint8_t*>(ws), L, out, static_cast<cudaStream_t>(stream));
}

int jfa_correct_merge(const jfa_geom* geom, const jfa_cache* cache, const uint16_t* q,
                      float scale, const int32_t* idx, int32_t k, const uint16_t* k_exact,
                      const uint16_t* v_exact, int32_t exact_on_host, void* ws, float* out,
                      void* stream) {
  if (!geom_ok(geom) || !cache_ok(cache) || !ws || !aligned(ws, 256)) return JFA_ERR_INVALID_ARG;
  if (geom->n_ctx < 1 || !q || !aligned(q, 16) || !(scale > 0.f)) return JFA_ERR_INVALID_ARG;
  if (k < 1 || k > JFA_MAX_EXACT || !idx || !out || !aligned(out, 16)) return JFA_ERR_INVALID_ARG;
  if (!k_exact || !v_exact || !aligned(k_exact, 16) || !aligned(v_exact, 16))
    return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  (void)exact_on_host;  // same loads either way; the rows are device-addressable
  SeqTable t;
  if (!fill_seq_table(*geom, nullptr, &t)) return JFA_ERR_INVALID_ARG;
  return launch_finish(*geom, t, *cache, q, scale, k, nullptr, idx, k_exact, v_exact,
                       static_cast<uint8_t*>(ws), L, out, static_cast<cudaStream_t>(stream));
}

int jfa_decode_step(const jfa_geom* geom, const jfa_cache* cache, const uint16_t* q, float scale,
                    int32_t k, int32_t* idx, const uint16_t* k_exact, const uint16_t* v_exact,
                    int32_t exact_on_host, void* ws, float* out, void* stream) {
  // validate everything before the first launch
  if (!geom_ok(geom) || !cache_ok(cache) || !ws || !aligned(ws, 256)) return JFA_ERR_INVALID_ARG;
  if (geom->n_ctx < 1 || !q || !aligned(q, 16) || !(scale > 0.f)) return JFA_ERR_INVALID_ARG;
  if (k < 1 || k > JFA_MAX_TOPK || !idx || !aligned(idx, 4) || !out || !aligned(out, 16))
    return JFA_ERR_INVALID_ARG;
  if (!k_exact || !v_exact || !aligned(k_exact, 16) || !aligned(v_exact, 16))
    return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, k, &L);
  const int sq = stage_query(*geom, &q, static_cast<uint8_t*>(ws), L, static_cast<cudaStream_t>(stream));
  if (sq != JFA_OK) return sq;
  const int s = jfa_decode_scores(geom, cache, q, scale, ws, stream);
  if (s != JFA_OK) return s;
  return jfa_decode_finish(geom, cache, q, scale, k, idx, k_exact, v_exact, exact_on_host, ws,
                           out, stream);
}

int jfa_decode_finish(const jfa_geom* geom, const jfa_cache* cache, const uint16_t* q, float scale,
                      int32_t k, int32_t* idx, const uint16_t* k_exact, const uint16_t* v_exact,
                      int32_t exact_on_host, void* ws, float* out, void* stream) {
  if (!geom_ok(geom) || !cache_ok(cache) || !ws || !aligned(ws, 256)) return JFA_ERR_INVALID_ARG;
  if (geom->n_ctx < 1 || !q || !aligned(q, 16) || !(scale > 0.f)) return JFA_ERR_INVALID_ARG;
  if (k < 1 || k > JFA_MAX_TOPK || !idx || !aligned(idx, 4) || !out || !aligned(out, 16))
    return JFA_ERR_INVALID_ARG;
  if (!k_exact || !v_exact || !aligned(k_exact, 16) || !aligned(v_exact, 16))
    return JFA_ERR_INVALID_ARG;
  (void)exact_on_host;  // same loads either way; the rows are device-addressable
  jfa_workspace_layout L;
  workspace_layout(*geom, k, &L);
  SeqTable t;
  if (!fill_seq_table(*geom, nullptr, &t)) return JFA_ERR_INVALID_ARG;
  return launch_finish(*geom, t, *cache, q, scale, k, idx, nullptr, k_exact, v_exact,
                       static_cast<uint8_t*>(ws), L, out, static_cast<cudaStream_t>(stream));
}

// The step for per-sequence lengths: scan over every sequence's own groups,
// then the finishing kernel with each cluster's own N_q and tail.
static int ragged_step(const jfa_geom* geom, const SeqTable& t, const jfa_cache* cache,
                       const uint16_t* q, float scale, int32_t k, int32_t* idx,
                       const uint16_t* k_exact, const uint16_t* v_exact, void* ws, float* out,
                       cudaStream_t st, bool defer_last) {
  jfa_workspace_layout L;
  workspace_layout(*geom, k, &L);
  uint8_t* w = static_cast<uint8_t*>(ws);
  const int sq = stage_query(*geom, &q, w, L, st);
  if (sq != JFA_OK) return sq;
  const int s = launch_scores(*geom, t, *cache, q, scale, w, L, st, true, defer_last);
  if (s != JFA_OK) return s;
  return launch_finish(*geom, t, *cache, q, scale, k, idx, nullptr, k_exact, v_exact, w, L, out, st);
}

static bool step_args_ok(const jfa_geom* geom, const jfa_cache* cache, const uint16_t* q,
                         float scale, int32_t k, const int32_t* idx, const uint16_t* k_exact,
                         const uint16_t* v_exact, const void* ws, const float* out) {
  if (!geom_ok(geom) || !cache_ok(cache) || !ws || !aligned(ws, 256)) return false;
  if (!q || !aligned(q, 16) || !(scale > 0.f)) return false;
  if (k < 1 || k > JFA_MAX_TOPK || !idx || !aligned(idx, 4) || !out || !aligned(out, 16))
    return false;
  if (!k_exact || !v_exact || !aligned(k_exact, 16) || !aligned(v_exact, 16)) return false;
  return true;
}

int jfa_decode_step_ragged(const jfa_geom* geom, const int32_t* seq_lens, const jfa_cache* cache,
                           const uint16_t* q, float scale, int32_t k, int32_t* idx,
                           const uint16_t* k_exact, const uint16_t* v_exact, int32_t exact_on_host,
                           void* ws, float* out, void* stream) {
  if (!seq_lens || !step_args_ok(geom, cache, q, scale, k, idx, k_exact, v_exact, ws, out))
    return JFA_ERR_INVALID_ARG;
  (void)exact_on_host;  // same loads either way; the rows are device-addressable
  SeqTable t;
  if (!fill_seq_table(*geom, seq_lens, &t)) return JFA_ERR_INVALID_ARG;
  return ragged_step(geom, t, cache, q, scale, k, idx, k_exact, v_exact, ws, out,
                     static_cast<cudaStream_t>(stream), false);
}

int jfa_append_decode_step(const jfa_geom* geom, const int32_t* seq_lens, const jfa_cache* cache,
                           const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_exact,
                           uint16_t* v_exact, const uint16_t* q, float scale, int32_t k,
                           int32_t* idx, int32_t exact_on_host, void* ws, float* out,
                           void* stream) {
  if (!seq_lens || !step_args_ok(geom, cache, q, scale, k, idx, k_exact, v_exact, ws, out))
    return JFA_ERR_INVALID_ARG;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return JFA_ERR_INVALID_ARG;
  (void)exact_on_host;  // the new rows are stored the same way either way
  if (!geom_ok(geom) || geom->batch > kMaxBatch) return JFA_ERR_INVALID_ARG;
  int32_t after[kMaxBatch];
  for (int b = 0; b < geom->batch; ++b) {
    if (seq_lens[b] < 0 || seq_lens[b] >= geom->capacity) return JFA_ERR_INVALID_ARG;
    after[b] = seq_lens[b] + 1;
  }
  SeqTable t;
  if (!fill_seq_table(*geom, after, &t)) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, k, &L);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int s = launch_append1(*geom, t, *cache, k_new, v_new, k_exact, v_exact,
                               reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + L.off_flag), st);
  if (s != JFA_OK) return s;
  // the scan follows the kernel that may write each sequence's last group:
  // that record is requested only after the scan's dependency wait
  return ragged_step(geom, t, cache, q, scale, k, idx, k_exact, v_exact, ws, out, st, true);
}

int jfa_decode_step_launches(const jfa_geom* geom, int32_t k) {
  if (!geom_ok(geom) || geom->n_ctx < 1 || k < 1 || k > JFA_MAX_TOPK) return 0;
  const int scan = split_point(geom->n_ctx) > 0 ? 1 : 0;
  return scan + 1;  // scan + fused finishing kernel
}

int jfa_scan_warps(const jfa_geom* geom) {
  if (!geom_ok(geom) || geom->n_ctx < 1) return 0;
  SeqTable t;
  if (!fill_seq_table(*geom, nullptr, &t)) return 0;
  const ScanPlan plan = scan_plan(*geom, t, num_sms_current());
  return plan.total_groups > 0 ? plan.n_warps : 0;
}

int jfa_selftest_bounded_wait(const jfa_geom* geom, void* ws, void* stream) {
  if (!geom_ok(geom) || !ws) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  return launch_bounded_wait_selftest(reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + L.off_flag),
                                      static_cast<cudaStream_t>(stream));
}

int jfa_clear_error(const jfa_geom* geom, void* ws, void* stream) {
  if (!geom_ok(geom) || !ws) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  if (cudaMemsetAsync(static_cast<uint8_t*>(ws) + L.off_flag, 0, sizeof(uint32_t),
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JFA_ERR_CUDA;
  return JFA_OK;
}

int jfa_check_error(const jfa_geom* geom, void* ws, void* stream, uint32_t* flag_out) {
  if (!geom_ok(geom) || !ws) return JFA_ERR_INVALID_ARG;
  jfa_workspace_layout L;
  workspace_layout(*geom, 1, &L);
  uint32_t f = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&f, static_cast<uint8_t*>(ws) + L.off_flag, sizeof(f),
                      cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return JFA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return JFA_ERR_CUDA;
  if (flag_out) *flag_out = f;
  return f ? JFA_ERR_DEVICE : JFA_OK;
}

int jfa_unpack_record(int32_t key_bits, int32_t val_bits, const void* record, uint8_t* k_codes,
                      uint16_t* k_scale, uint16_t* k_zero, uint8_t* v_codes, uint16_t* v_scale,
                      uint16_t* v_zero) {
  if ((key_bits != 3 && key_bits != 4) || (val_bits != 2 && val_bits != 4) || !record)
    return JFA_ERR_INVALID_ARG;
  const uint8_t* r = static_cast<const uint8_t*>(record);
  auto word = [&](int off) {
    uint32_t w;
    memcpy(&w, r + off, 4);
    return w;
  };
  auto half = [&](int off) {
    uint16_t h;
    memcpy(&h, r + off, 2);
    return h;
  };
  for (int c = 0; c < kD; ++c) {
    if (k_scale) k_scale[c] = half(off_ks() + ks_scale_off(c));
    if (k_zero) k_zero[c] = half(off_ks() + ks_zero_off(c));
  }
  const uint32_t km = (1u << key_bits) - 1u, vm = (1u << val_bits) - 1u;
  if (k_codes) {
    for (int t = 0; t < kKG; ++t)
      for (int c = 0; c < kD; ++c) {
        BitLoc L[3];
        uint32_t code = 0;
        if (kc_bits(key_bits, t, c, L) == 1) {
          code = (word(off_kc() + L[0].byte) >> L[0].bit) & km;
        } else {
          for (int b = 0; b < 3; ++b) code |= ((word(off_kc() + L[b].byte) >> L[b].bit) & 1u) << b;
        }
        k_codes[t * kD + c] = (uint8_t)code;
      }
  }
  for (int t = 0; t < kKG; ++t)
    for (int j = 0; j < kD / kVG; ++j) {
      if (v_scale) v_scale[t * 4 + j] = half(off_vs(key_bits) + vs_scale_off(t, j));
      if (v_zero) v_zero[t * 4 + j] = half(off_vs(key_bits) + vs_zero_off(t, j));
    }
  if (v_codes) {
    for (int t = 0; t < kKG; ++t)
      for (int c = 0; c < kD; ++c) {
        BitLoc L = vc_loc(val_bits, t, c);
        v_codes[t * kD + c] = (uint8_t)((word(off_vc(key_bits) + L.byte) >> L.bit) & vm);
      }
  }
  return JFA_OK;
}

}  // extern "C"
