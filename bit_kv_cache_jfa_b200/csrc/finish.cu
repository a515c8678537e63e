// finish.cu — host entry of the finishing kernel: fills its arguments and
// dispatches to the launcher of the cache's key/value widths
// (finish_k{3,4}v{2,4}.cu instantiate finish_impl.cuh once each).
#include "finish_params.cuh"

namespace jfa {

int launch_finish(const jfa_geom& g, const SeqTable& t, const jfa_cache& c, const uint16_t* q,
                  float scale, int k, int32_t* idx_out, const int32_t* idx_in,
                  const uint16_t* k_exact, const uint16_t* v_exact, uint8_t* ws,
                  const jfa_workspace_layout& L, float* out, cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  FinishParams fp;
  fp.groups = static_cast<const uint8_t*>(c.groups);
  fp.tail_k = c.tail_k;
  fp.tail_v = c.tail_v;
  fp.k_exact = k_exact;
  fp.v_exact = v_exact;
  fp.q = q;
  fp.scores = reinterpret_cast<const float*>(ws + L.off_scores);
  fp.scan_part = reinterpret_cast<const float*>(ws + L.off_partials);
  fp.m_used = reinterpret_cast<const float*>(ws + L.off_mused);
  fp.wts = reinterpret_cast<const uint32_t*>(ws + L.off_wts);
  fp.hist = reinterpret_cast<uint32_t*>(ws + L.off_scan_hist);
  fp.hist_reps = scan_hist_reps((long long)g.batch * g.num_kv_heads);
  fp.glists = reinterpret_cast<uint32_t*>(ws + L.off_cand);
  fp.idx_in = idx_in;
  fp.idx_out = idx_out;
  fp.out = out;
  fp.flag = reinterpret_cast<uint32_t*>(ws + L.off_flag);
  fp.k = k;
  fp.capacity = g.capacity;
  fp.ng_cap = g.capacity / kKG;
  fp.hkv = g.num_kv_heads;
  fp.H = g.num_heads;
  fp.key_bits = g.key_bits;
  fp.val_bits = g.val_bits;
  fp.rec_bytes = record_bytes(g.key_bits, g.val_bits);
  const ScanPlan plan = scan_plan(g, t, num_sms_current());
  fp.scan_total = plan.total_groups;
  fp.scan_warps = plan.n_warps;
  fp.kappa = scale * 1.4426950408889634f;
  fp.gl_stride = 2 * L.cand_cap;
  fp.seq = t;
  const int G = g.num_heads / g.num_kv_heads;
  const bool select = idx_in == nullptr;
  const int nq_max = max_nq(g, t);
  if (g.key_bits == 3)
    return g.val_bits == 2 ? launch_finish_k3v2(fp, G, n_seg, nq_max, select, st)
                           : launch_finish_k3v4(fp, G, n_seg, nq_max, select, st);
  return g.val_bits == 2 ? launch_finish_k4v2(fp, G, n_seg, nq_max, select, st)
                         : launch_finish_k4v4(fp, G, n_seg, nq_max, select, st);
}

}  // namespace jfa
