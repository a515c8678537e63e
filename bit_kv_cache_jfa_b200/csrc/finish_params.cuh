// finish_params.cuh — arguments of the finishing kernel (selection,
// correction and merge after the scan) and its per-format launchers.
#pragma once

#include "jfa_internal.cuh"

namespace jfa {

struct FinishParams {
  const uint8_t* groups;
  const uint16_t* tail_k;
  const uint16_t* tail_v;
  const uint16_t* k_exact;
  const uint16_t* v_exact;
  const uint16_t* q;
  const float* scores;     // [n_seg][capacity]
  const float* scan_part;  // per scan warp and segment: [slot][G][kPartStride]
  const float* m_used;     // [n_seg][ng_cap][8]: the scan's running maxima
  const uint32_t* wts;     // the scan's fp16 weights, [n_seg][ng_cap][4][NT][32] words
  uint32_t* hist;          // [n_seg][hist_reps][kScanHistStride] (bins, largest key), zeroed here after use
  uint32_t* glists;        // [n_seg][C][slice] chosen lists of the fallback
  const int32_t* idx_in;   // given index sets (no selection), [n_seg][k]
  int32_t* idx_out;        // [n_seg][k] (selection)
  float* out;
  uint32_t* flag;
  int k, capacity, ng_cap, hkv, H, key_bits, val_bits, rec_bytes;
  int gl_stride;           // uint32 entries of glists per segment
  long long scan_total;
  int scan_warps;
  int hist_reps;           // copies of each segment's histogram (scan_hist_reps)
  float kappa;
  SeqTable seq;            // per-sequence lengths and the scan's group offsets
};

// Launch the finishing kernel for G = num_heads / num_kv_heads query heads per
// KV head over n_seg (sequence, KV head) segments; select = run the top-k
// selection (else fp.idx_in holds the index sets).  One per key/value width.
// nq_max: the largest N_q of the batch (picks the cluster size).
int launch_finish_k3v2(const FinishParams& fp, int G, int n_seg, int nq_max, bool select, cudaStream_t st);
int launch_finish_k3v4(const FinishParams& fp, int G, int n_seg, int nq_max, bool select, cudaStream_t st);
int launch_finish_k4v2(const FinishParams& fp, int G, int n_seg, int nq_max, bool select, cudaStream_t st);
int launch_finish_k4v4(const FinishParams& fp, int G, int n_seg, int nq_max, bool select, cudaStream_t st);

}  // namespace jfa
