/*
 * jfa.h — C ABI of the approximate-then-correct low-bit KV decode-attention
 * library (sm_100a).
 *
 * The method (JetFire README, introduction): the KV cache lives on the GPU at
 * low bit width (K3V2: 3-bit keys / 2-bit values, or K4V4; README, benchmark
 * section), every cached token is scored approximately from it, the top-k
 * tokens are re-scored and re-aggregated from a high-precision BF16 copy
 * (held in GPU memory or in pinned host memory), and the exact and
 * approximate parts are merged.
 *
 * One decode step for all sequences of a batch and all heads of one layer is
 *     jfa_decode_scores -> jfa_topk -> jfa_correct_merge
 * and new tokens enter the cache through jfa_pack_kv.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor pointers are DEVICE pointers (or, where stated, pointers to
 *    pinned host memory that the device can address), caller-owned; the
 *    library never allocates, frees or synchronises (except
 *    jfa_check_error).  Work is ordered on the given stream.
 *  - bf16 tensors are raw 16-bit patterns (`uint16_t`), row-major.
 *  - Every call returns a jfa_status; on an argument error nothing is
 *    launched.  No exception or abort crosses the ABI.
 *  - Device-side problems (non-finite scale/zero while packing, an
 *    out-of-range index handed to jfa_correct_merge, an exhausted bounded
 *    wait) set a flag word in the workspace; jfa_check_error reads it.
 *  - head_dim is 128; query heads per KV head G = H / H_kv must be 1..8.
 *  - The sequences of a batch hold geom->n_ctx tokens each, except in
 *    jfa_decode_step_ragged and jfa_append_decode_step, which take a length
 *    per sequence (at most JFA_MAX_BATCH sequences per call).
 */
#ifndef JFA_H_
#define JFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Fixed quantization geometry.
 * Keys: one fp16 (scale, zero) per (64-token group, channel); values: one
 * per (token, 32-channel group).  Group size 64 with an FP16 zero point and
 * scale follows the TailorKV review ("free parameters": quantization bit
 * size and group size) and HACK's default partition size 64 (HACK review,
 * "free parameters").  The newest 1..64 tokens stay exact in a bf16 tail so
 * appends never requantize (HACK review, Figure 8: last block of V kept in
 * FP16; Jet-QSparse abstract: at most two BF16 pages per sequence). */
#define JFA_HEAD_DIM 128
#define JFA_KEY_GROUP 64
#define JFA_VAL_GROUP 32
#define JFA_TAIL_MAX 64
#define JFA_MAX_GQA 8
#define JFA_MAX_BATCH 256     /* sequences per call                              */
#define JFA_MAX_TOPK 4096
#define JFA_MAX_EXACT 8192    /* exact tokens per segment jfa_correct_merge takes */
#define JFA_BLOCK_TOKENS 128  /* tokens per block of jfa_topk_blocks             */
#define JFA_MAX_BLOCKS (JFA_MAX_EXACT / JFA_BLOCK_TOKENS)

typedef enum jfa_status {
  JFA_OK = 0,
  JFA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or geometry */
  JFA_ERR_UNSUPPORTED = 2, /* valid request this build does not implement   */
  JFA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed          */
  JFA_ERR_DEVICE = 4       /* the device error flag is set (jfa_check_error)*/
} jfa_status;

/* Device error flag bits (OR-ed into the workspace flag word). */
#define JFA_DEVERR_NONFINITE_QUANT 0x1u /* a packed scale/zero is inf/nan   */
#define JFA_DEVERR_BAD_INDEX 0x2u       /* top-k index outside [0, N_q)     */
#define JFA_DEVERR_TIMEOUT 0x4u         /* a bounded wait gave up           */

typedef struct jfa_geom {
  int32_t batch;        /* B: sequences                                   */
  int32_t num_heads;    /* H: query heads                                 */
  int32_t num_kv_heads; /* H_kv: KV heads; H % H_kv == 0, H/H_kv <= 8      */
  int32_t head_dim;     /* must be 128                                    */
  int32_t capacity;     /* max tokens per sequence; multiple of 64, >= 64 */
  int32_t key_bits;     /* 3 or 4                                         */
  int32_t val_bits;     /* 2 or 4                                         */
  int32_t n_ctx;        /* tokens currently cached per sequence           */
} jfa_geom;

/* Device buffers of one layer's quantized cache (caller-allocated with the
 * sizes jfa_cache_layout_get reports; every pointer 16-byte aligned).
 *   groups : packed group records, [B][H_kv][capacity/64][record_bytes].
 *            A record holds the codes and fp16 scales/zeros of the keys and
 *            values of 64 consecutive tokens, in a layout private to this
 *            library (decode it with jfa_unpack_record).
 *   tail_k, tail_v : bf16 [B][H_kv][64][128], the newest 1..64 tokens. */
typedef struct jfa_cache {
  void* groups;
  uint16_t* tail_k;
  uint16_t* tail_v;
} jfa_cache;

typedef struct jfa_cache_layout {
  size_t record_bytes; /* bytes per (sequence, KV head, 64-token group)   */
  size_t groups_bytes; /* size of jfa_cache.groups                        */
  size_t tail_bytes;   /* size of each of tail_k and tail_v               */
  /* byte offsets of the record sections */
  size_t off_key_scales, off_key_codes, off_val_scales, off_val_codes;
} jfa_cache_layout;

/* Workspace layout: scratch of the decode step (selection scores, split
 * softmax partials, the running maxima and score histogram of the scan,
 * top-k histograms/candidates, the error flag).  Sized by
 * jfa_workspace_layout_get for a geometry and a maximum k. */
typedef struct jfa_workspace_layout {
  size_t total_bytes;
  size_t off_flag;       /* uint32 device error flag                          */
  size_t off_scores;     /* fp32 [B][H_kv][capacity]: selection score S_t     */
  size_t off_partials;   /* fp32 split partials of the approximate scan       */
  size_t off_mused;      /* fp32 [B][H_kv][capacity/64][8]: per key group, for
                            each query head the running maximum the scan's
                            weights were taken against                       */
  size_t off_wts;        /* the scan's fp16 softmax weights of every quantized
                            token and query head, in a layout private to
                            this library (read by the correction)            */
  size_t off_scan_hist;  /* uint32 [B][H_kv][R][32768 + 32]: histogram of the
                            top 15 bits of the selection keys, then the
                            largest key, in R copies (R = 1 from 32 segments
                            B*H_kv up, else 32/(B*H_kv), at most 16), built
                            by the scan and cleared by the finishing kernel */
  size_t off_hist;       /* top-k histograms (jfa_topk)                       */
  size_t off_counters;   /* top-k counters (jfa_topk)                         */
  size_t off_cand;       /* top-k candidate lists                             */
  size_t off_sel;        /* top-k per-chunk list lengths (jfa_topk)           */
  size_t off_fp4q;       /* NVFP4 query records of jfa_fp4_scores, one per
                            (sequence, KV head)                               */
  size_t off_sparse;     /* split partials of jfa_sparse_attend              */
  size_t off_ticket;     /* uint32 [B][H_kv] split counters of
                            jfa_sparse_attend (zero between calls)           */
  size_t off_bkeys;      /* uint32 [B][H_kv][capacity/128]: per 128-token
                            block the largest selection score of the FP4
                            scan, as an order-preserving key                 */
  size_t off_chan;       /* per (sequence, KV head) the critical channels of
                            jfa_channel_scores and the query at them         */
  size_t off_qstage;     /* bf16 [B][H][128]: the query of a decode step
                            given in pinned host memory, copied here first   */
  int32_t max_topk;
  int32_t partial_slots; /* slots of off_partials                             */
  int32_t cand_cap;      /* list entries per segment                          */
  int32_t reserved;
} jfa_workspace_layout;

/* Human-readable name of a status code (static string). */
const char* jfa_status_string(int status);

/* Sizes and section offsets of the cache buffers for a geometry.
 * Pure host function; JFA_ERR_INVALID_ARG on a bad geometry. */
int jfa_cache_layout_get(const jfa_geom* geom, jfa_cache_layout* out);

/* Sizes and offsets of the decode workspace for a geometry and a maximum k
 * (1..JFA_MAX_TOPK).  Pure host function.  Zero-fill the workspace once
 * after allocating it: the top-k counters and histograms it holds start at
 * zero and every completed jfa_topk call leaves them at zero again. */
int jfa_workspace_layout_get(const jfa_geom* geom, int32_t max_topk,
                             jfa_workspace_layout* out);

/* jfa_pack_kv — append n_new tokens to every sequence.
 * Definition: partition-wise asymmetric quantization x ~ s*x' + m with m the
 * partition minimum (HACK review, Eq. (4) and context), FP16 zero point and
 * scale per group of 64 (TailorKV review).  This library takes
 *   zero  = largest fp16 <= min, scale = smallest fp16 >= (max-zero)/(2^b-1),
 *   code  = round-half-even((x-zero)/scale) clipped to [0, 2^b-1],
 * both quotients in fp64; keys per (64-token group, channel), values per
 * (token, 32-channel group).  Tokens enter the bf16 tail; a token arriving
 * at a full tail (64) first flushes the tail as one group, so the tail holds
 * N - N_q in [1, 64] tokens with N_q = 64*floor((N-1)/64), and codes once
 * written never change.
 *   geom->n_ctx : tokens already cached (before this call); the caller adds
 *                 n_new to its own counter after the call.
 *   k_new, v_new: bf16 [B][H_kv][n_new][128] device pointers, 16-B aligned.
 *   ws          : workspace (only the error flag is used).
 * Requires n_ctx + n_new <= capacity.  The high-precision copy of K/V used
 * by jfa_correct_merge is the caller's (written by the caller). */
int jfa_pack_kv(const jfa_geom* geom, const jfa_cache* cache,
                const uint16_t* k_new, const uint16_t* v_new, int32_t n_new,
                void* ws, void* stream);

/* jfa_decode_scores — approximate scan over the N_q quantized tokens.
 * Definition (Jet-QSparse abstract: a dense scan scores the full key
 * history; HACK review, Eq. (4): the product with affinely quantized keys is
 * an integer product plus correction terms):
 *   s_hat[h][t] = scale * sum_c q[h][c] * (s[g][c]*k'[t][c] + m[g][c])
 * for every query head h and quantized token t (g = t/64), and the selection
 * score S[t] = max over the G query heads sharing the KV head.  In the same
 * pass it accumulates, per split of the token range, the softmax partial
 * (max, sum exp, sum exp * v_hat) of every query head over the dequantized
 * values, which jfa_correct_merge turns into the approximate remainder.
 *   q     : bf16 [B][H][128] device pointer, 16-B aligned.
 *   scale : softmax scale (e.g. 1/sqrt(128)).
 *   ws    : workspace for at least this geometry.
 * Writes S (workspace off_scores) and the split partials.  Launched as a
 * programmatic dependent of the previous kernel in the stream: each warp's
 * first packed-record copy may start before that kernel has finished when it
 * releases its dependents early, so the packed records must not be written
 * by such a kernel (this library's own packing kernel releases none). */
int jfa_decode_scores(const jfa_geom* geom, const jfa_cache* cache,
                      const uint16_t* q, float scale, void* ws, void* stream);

/* jfa_topk — per (sequence, KV head) the k tokens with the largest S
 * (JetFire README: correct the top-k tokens; Jet-QSparse abstract: selection
 * per KV head).  Order is (S descending, index ascending); the k_eff =
 * min(k, N_q) chosen indices are written sorted ascending to
 * idx[B][H_kv][k] (int32 device pointer), the remaining k - k_eff entries
 * set to -1.  1 <= k <= max_topk of the workspace.
 * Reads the selection scores jfa_decode_scores leaves in the workspace
 * (off_scores); a caller may also write its own scores there first. */
int jfa_topk(const jfa_geom* geom, int32_t k, void* ws, int32_t* idx,
             void* stream);

/* jfa_topk_blocks — selection of whole 128-token blocks instead of single
 * tokens (Jet-QSparse abstract: 128-token blocks are selected for the sparse
 * high-precision value aggregation, so the exact rows are read as contiguous
 * tiles).  Per (sequence, KV head) the score of block j is the largest
 * selection score S_t of its quantized tokens t in [128 j, 128 j + 128)
 * (the last block holds 64 when N_q is an odd multiple of 64); the n_blocks
 * blocks with the largest scores, order (score descending, block index
 * ascending), are chosen and their token indices written ascending to
 * idx[B][H_kv][n_blocks * 128] (int32 device pointer); tokens at or past N_q
 * of a partial block and the entries of unchosen blocks are -1.  The result
 * is a given index set for jfa_correct_merge with k = n_blocks * 128.
 *   1 <= n_blocks <= JFA_MAX_BLOCKS; N_q <= 1048576 (else
 *   JFA_ERR_UNSUPPORTED).  Reads the scores jfa_decode_scores leaves in the
 *   workspace; allocates nothing. */
int jfa_topk_blocks(const jfa_geom* geom, int32_t n_blocks, void* ws, int32_t* idx,
                    void* stream);

/* jfa_topk_noalloc — the selection of jfa_topk for callers that cannot
 * allocate device memory, such as an inference-engine plugin whose execute
 * callback must not allocate, or a latency-bound loop where an allocation
 * would stall the device.  The pages have no counterpart; it is a
 * deployment convenience.
 *   scores   : fp32 [n_seg][stride] device pointer, 16-B aligned; the first
 *              n_scores entries of each row are scored (n_scores % 4 == 0,
 *              stride % 4 == 0, stride >= n_scores).
 *   idx      : int32 [n_seg][k] output, as jfa_topk writes it.
 * Scratch lives in one fixed ~2.5 MB device array inside the library (held by
 * every device that loads it until exit): n_seg <= 64 and
 * n_seg * ceil(n_scores / 4096) <= 64 (e.g. 8 rows of 32768 scores, 2 of
 * 131072); larger requests return JFA_ERR_UNSUPPORTED before any work.
 * The call allocates nothing.  Its first call on a device looks up the
 * array's device address (cudaGetSymbolAddress).  Every call clears the
 * parts of the array that
 * must start at zero and otherwise reuses the previous call's contents, so
 * calls that overlap on the GPU (other streams, other threads) race: keep
 * them on one stream, and the stream must belong to the current device (the
 * array looked up is the current device's). */
int jfa_topk_noalloc(const float* scores, int32_t n_seg, int32_t stride,
                     int32_t n_scores, int32_t k, int32_t* idx, void* stream);

/* jfa_correct_merge — exact correction and log-sum-exp merge.
 * For every query head: exact logits scale*q.K_t from the bf16 copy for the
 * top-k tokens and the tail, aggregated with bf16 values in fp32 (Jet-QSparse
 * abstract: sparse high-precision value aggregation with FP32 accumulation;
 * JetFire README: high-precision correction of the top-k tokens); the
 * approximate remainder over the other quantized tokens (the scan partials
 * minus the top-k tokens' approximate terms); merged as
 *   m = max(m_e, m_a), out = (acc_e e^(m_e-m) + acc_a e^(m_a-m)) /
 *                            (l_e e^(m_e-m) + l_a e^(m_a-m)).
 *   idx          : int32 [B][H_kv][k] from jfa_topk or jfa_topk_blocks
 *                  (1 <= k <= JFA_MAX_EXACT; entries -1 ignored; the others
 *                  distinct, in [0, N_q), else the device flag
 *                  JFA_DEVERR_BAD_INDEX is set and the entry skipped).
 * The approximate terms of the top-k tokens are taken out of the scan's
 * partials by recomputing, from the packed records and the running maxima
 * the scan stored, exactly the fp16 weights the scan used, so the removal
 * leaves only fp32 rounding.
 *   k_exact,
 *   v_exact      : bf16 [B][H_kv][capacity][128], every cached token; device
 *                  memory, or pinned host memory the device can address
 *                  (exact_on_host = 1: rows are read by zero-copy loads).
 *   out          : fp32 [B][H][128]; device memory, or pinned host memory
 *                  the device can address (the kernel's stores then cross
 *                  the host link directly; no separate copy is needed).
 * Must follow jfa_decode_scores with the same geometry, q and scale. */
int jfa_correct_merge(const jfa_geom* geom, const jfa_cache* cache,
                      const uint16_t* q, float scale, const int32_t* idx,
                      int32_t k, const uint16_t* k_exact,
                      const uint16_t* v_exact, int32_t exact_on_host,
                      void* ws, float* out, void* stream);

/* The whole decode step (scores, top-k, correct+merge) in one call, with the
 * same results as the three calls in order (idx identical, out to rounding):
 * the scan, then one kernel in which a thread-block cluster per (sequence,
 * KV head) selects, corrects and merges.  idx is written as by jfa_topk.
 *   q : bf16 [B][H][128], 16-B aligned: device memory, or pinned host
 *       memory (the step then first copies it into the workspace's
 *       off_qstage region with one kernel, which reads it across the host
 *       link while the previous kernel in the stream is still running;
 *       pageable host memory: JFA_ERR_INVALID_ARG).  The same holds for
 *       jfa_decode_step_ragged and jfa_append_decode_step. */
int jfa_decode_step(const jfa_geom* geom, const jfa_cache* cache,
                    const uint16_t* q, float scale, int32_t k, int32_t* idx,
                    const uint16_t* k_exact, const uint16_t* v_exact,
                    int32_t exact_on_host, void* ws, float* out, void* stream);

/* jfa_decode_step_ragged — jfa_decode_step for a batch whose sequences hold
 * different numbers of tokens (the decode steps on either side of the path:
 * each sequence keeps its own quantized groups and bf16 tail; Jet-QSparse
 * abstract: at most two BF16 pages per sequence and layer).
 *   seq_lens : host int32[B], tokens cached per sequence, each in
 *              [1, capacity]; geom->n_ctx is not used.  Sequence b splits into
 *              N_q(b) = 64*floor((seq_lens[b]-1)/64) quantized tokens and a
 *              tail of seq_lens[b] - N_q(b), and its top-k takes
 *              min(k, N_q(b)) tokens.
 * Other arguments as jfa_decode_step.  The lengths are read on the host when
 * the call is made (they become launch arguments). */
int jfa_decode_step_ragged(const jfa_geom* geom, const int32_t* seq_lens,
                           const jfa_cache* cache, const uint16_t* q, float scale,
                           int32_t k, int32_t* idx, const uint16_t* k_exact,
                           const uint16_t* v_exact, int32_t exact_on_host, void* ws,
                           float* out, void* stream);

/* jfa_append_decode_step — one new token per sequence, then the decode step
 * over the grown cache, in one call.  The new token of sequence b goes to
 * position seq_lens[b]: into the bf16 tail, after the tail is first
 * quantized as one 64-token group if it is full (HACK review, Figure 8: the
 * last partial block stays in FP16, so an append never requantizes written
 * codes), and into the exact copy.
 *   seq_lens        : host int32[B], tokens cached before the append, each in
 *                     [0, capacity - 1]; the caller adds one after the call.
 *   k_new, v_new    : bf16 [B][H_kv][128] device pointers, 16-B aligned.
 *   k_exact, v_exact: the exact copy (device or pinned host memory the device
 *                     can address); row seq_lens[b] of every (sequence, KV
 *                     head) is written here, then read like the others.
 * Other arguments as jfa_decode_step (idx, out for the grown cache). */
int jfa_append_decode_step(const jfa_geom* geom, const int32_t* seq_lens,
                           const jfa_cache* cache, const uint16_t* k_new,
                           const uint16_t* v_new, uint16_t* k_exact, uint16_t* v_exact,
                           const uint16_t* q, float scale, int32_t k, int32_t* idx,
                           int32_t exact_on_host, void* ws, float* out, void* stream);

/* jfa_decode_finish — the rest of the step after jfa_decode_scores: top-k
 * selection, exact correction and merge in one kernel (a thread-block
 * cluster per (sequence, KV head)); results as jfa_topk followed by
 * jfa_correct_merge.  Arguments as jfa_decode_step. */
int jfa_decode_finish(const jfa_geom* geom, const jfa_cache* cache,
                      const uint16_t* q, float scale, int32_t k, int32_t* idx,
                      const uint16_t* k_exact, const uint16_t* v_exact,
                      int32_t exact_on_host, void* ws, float* out, void* stream);

/* Failure-detection self test: launches one warp that waits, with the same
 * bounded wait the scan uses for its record copies, on an mbarrier whose
 * phase cannot complete.  After about one second the wait gives up and the
 * kernel sets JFA_DEVERR_TIMEOUT in the workspace flag; nothing faults and the
 * context stays usable (read the flag with jfa_check_error, then clear it).
 * Stream-ordered; JFA_ERR_INVALID_ARG on a bad geometry or null workspace. */
int jfa_selftest_bounded_wait(const jfa_geom* geom, void* ws, void* stream);

/* Clear the workspace error flag (stream-ordered). */
int jfa_clear_error(const jfa_geom* geom, void* ws, void* stream);

/* Synchronise the stream and read the device error flag into *flag_out
 * (0 = no error).  Returns JFA_ERR_DEVICE if the flag is non-zero. */
int jfa_check_error(const jfa_geom* geom, void* ws, void* stream,
                    uint32_t* flag_out);

/* Host-side decoder of one packed group record (record_bytes from
 * jfa_cache_layout_get), for inspection and tests.  Outputs:
 *   k_codes [64][128] (token-major), k_scale/k_zero [128] fp16 bits,
 *   v_codes [64][128], v_scale/v_zero [64][4] fp16 bits.  Any output may be
 *   NULL to skip it. */
int jfa_unpack_record(int32_t key_bits, int32_t val_bits, const void* record,
                      uint8_t* k_codes, uint16_t* k_scale, uint16_t* k_zero,
                      uint8_t* v_codes, uint16_t* v_scale, uint16_t* v_zero);

/* Number of kernel launches one jfa_decode_step issues for a geometry with
 * q in device memory (for launch accounting; one more with q in pinned host
 * memory); 0 on a bad geometry. */
int jfa_decode_step_launches(const jfa_geom* geom, int32_t k);

/* ---------------------------------------------------------------------------
 * NVFP4 keys and block-sparse exact attention (Jet-QSparse abstract: compact
 * NVFP4 cache storage, query-key products in FP4 on Blackwell tensor cores,
 * a dense scan over the whole key history that selects 128-token blocks, and
 * the value aggregation over those blocks in high precision with FP32
 * accumulation).
 *
 * NVFP4 here: E2M1 elements (0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives), a
 * UE4M3 scale per 16 consecutive channels of a row, and an fp32 tensor scale
 * s = amax / (6 * 448) (1 when amax is 0) per 64-token key group, or per
 * query head for the query.  Block scale = the UE4M3 value nearest to
 * amax_16 / (6 s) (ties to even, at most 448); code = the E2M1 value nearest
 * to x / (block scale * s) (ties to even, saturating at 6); both quotients in
 * fp64.  The score of a token for a query head is
 *   scale * s_k s_q * sum_c (e2m1_k bs_k)(e2m1_q bs_q),
 * accumulated in fp32 by the tensor cores, and its selection score the
 * largest over the KV head's query heads.
 *
 * Geometry: jfa_geom with capacity a multiple of 128; key_bits and val_bits
 * are not used by these calls (any valid pair).  The workspace is the one
 * jfa_workspace_layout_get sizes (zero-filled once).  Errors as above.
 * ------------------------------------------------------------------------- */
#define JFA_FP4_RECORD_BYTES 9232 /* bytes per (sequence, KV head, 128-token block) */

/* NVFP4 key pool: B * H_kv * capacity/128 records of JFA_FP4_RECORD_BYTES,
 * [B][H_kv][capacity/128][record], in a layout private to this library
 * (E2M1 codes in the tensor core's operand order, the block scales as
 * scale-factor atoms, the two group scales).  Caller-allocated, 16-byte
 * aligned.  Returns the pool size in *pool_bytes. */
int jfa_fp4_pool_bytes(const jfa_geom* geom, size_t* pool_bytes);

/* Quantize the 64-token key groups covering tokens [n_from, n_to) of every
 * (sequence, KV head) into the pool, from the exact bf16 keys
 *   k_src : [B][H_kv][capacity][128] (device, or pinned host memory)
 * (the persistent cache packed straight from the BF16 activations).
 * n_from, n_to multiples of 64, 0 <= n_from <= n_to <= capacity.  Groups
 * already written are never rewritten.  A non-finite key sets
 * JFA_DEVERR_NONFINITE_QUANT.  Stream-ordered. */
int jfa_fp4_pack_keys(const jfa_geom* geom, int32_t n_from, int32_t n_to, const uint16_t* k_src,
                      void* pool, void* ws, void* stream);

/* FP4 scan: quantize q (bf16 [B][H][128], device) to NVFP4 per head and
 * compute the selection score of each of the N_q = 64 floor((n_ctx-1)/64)
 * quantized tokens (every group below N_q must have been packed) into the
 * workspace's score array, where jfa_topk / jfa_topk_blocks read it.  Two
 * launches (query records, then the tcgen05 scan).  Stream-ordered. */
int jfa_fp4_scores(const jfa_geom* geom, const void* pool, const uint16_t* q, float scale,
                   void* ws, void* stream);

/* Exact attention over an index set and the tail, nothing else:
 *   out[b, h] = softmax over T of (scale q_h . k_t) applied to v_t,
 *   T = {idx[b, h/G, j] >= 0, j < k} + {N_q, ..., n_ctx - 1},
 * with k_t, v_t rows of the exact bf16 copy
 *   k_exact, v_exact : [B][H_kv][capacity][128] (device, or pinned host with
 *                      exact_on_host = 1; read by zero-copy loads)
 *   idx              : int32 [B][H_kv][k] (device), -1 = no token; an entry
 *                      outside [-1, N_q) sets JFA_DEVERR_BAD_INDEX and is
 *                      skipped; indices must be distinct
 *   out              : fp32 [B][H][128] (device)
 * 1 <= k <= JFA_MAX_EXACT.  Logits in fp32 from bf16 products, softmax
 * weights carried at about 16 bits into an fp32 accumulation.  One launch.
 * Stream-ordered. */
int jfa_sparse_attend(const jfa_geom* geom, const uint16_t* q, float scale, const int32_t* idx,
                      int32_t k, const uint16_t* k_exact, const uint16_t* v_exact,
                      int32_t exact_on_host, void* ws, float* out, void* stream);

/* The NVFP4 decode step: jfa_fp4_scores, jfa_topk_blocks (the n_blocks best
 * 128-token blocks per (sequence, KV head), written to idx int32
 * [B][H_kv][n_blocks * 128]) and jfa_sparse_attend over them and the tail.
 * Four launches.  Stream-ordered. */
int jfa_fp4_decode_step(const jfa_geom* geom, const void* pool, const uint16_t* q, float scale,
                        int32_t n_blocks, int32_t* idx, const uint16_t* k_exact,
                        const uint16_t* v_exact, int32_t exact_on_host, void* ws, float* out,
                        void* stream);

/* ---------------------------------------------------------------------------
 * Critical-channel selection (TailorKV review: the importance of channel i is
 * s_i = |q_i| * max_t |K_{t,i}|; approximate attention scores over the most
 * important channels pick the top-k tokens, which are attended exactly).
 * Here, per (sequence, KV head): |q_i| is the largest over the KV head's
 * query heads, max|K_i| runs over the tokens packed into the channel copy
 * (pack the groups below N_q), the r most important channels are kept (ties
 * to the lower channel), and the selection score of a quantized token t is
 * the largest over the query heads of scale * sum over kept channels of
 * q_{h,i} K_{t,i} (fp32).  Geometry as for the NVFP4 calls (key_bits and
 * val_bits unused; capacity a multiple of 64).
 * ------------------------------------------------------------------------- */

/* Channel-major copy of the keys of tokens [n_from, n_to) (multiples of 64):
 *   k_src : bf16 [B][H_kv][capacity][128] (device or pinned host)
 *   k_t   : bf16 [B][H_kv][128][capacity] (device, 16-byte aligned)
 *   k_max : fp32 [B][H_kv][128] (device), zero before the first call; raised
 *           to the largest |K| of each channel.  Stream-ordered. */
int jfa_channel_pack(const jfa_geom* geom, int32_t n_from, int32_t n_to, const uint16_t* k_src,
                     uint16_t* k_t, float* k_max, void* stream);

/* Selection scores of the N_q quantized tokens from the r critical channels
 * (1 <= r <= 128) into the workspace's score array (read by jfa_topk).  One
 * launch.  Stream-ordered. */
int jfa_channel_scores(const jfa_geom* geom, const uint16_t* k_t, const float* k_max,
                       const uint16_t* q, float scale, int32_t r, void* ws, void* stream);

/* jfa_channel_scores, jfa_topk (k tokens per (sequence, KV head), written to
 * idx int32 [B][H_kv][k]) and jfa_sparse_attend over them and the tail.
 * 1 <= k <= JFA_MAX_TOPK.  Stream-ordered. */
int jfa_channel_decode_step(const jfa_geom* geom, const uint16_t* k_t, const float* k_max,
                            const uint16_t* q, float scale, int32_t r, int32_t k, int32_t* idx,
                            const uint16_t* k_exact, const uint16_t* v_exact,
                            int32_t exact_on_host, void* ws, float* out, void* stream);

/* ---------------------------------------------------------------------------
 * 1-bit KV cache with dense attention (TailorKV review: layers whose attention
 * is spread over many tokens keep the whole cache at 1 bit per number and
 * attend over all of it, an FP16 x INT1 product, with no tokens fetched back).
 * The quantization is jfa_pack_kv's rule at b = 1 (keys per channel over
 * 64-token groups, values per token over 32-channel groups, fp16 zero point
 * = the minimum rounded down, fp16 scale = the range rounded up, code = the
 * nearer end, ties to 0).  Geometry as for the NVFP4 calls (key_bits and
 * val_bits unused; capacity a multiple of 64).
 * ------------------------------------------------------------------------- */
#define JFA_ONEBIT_RECORD_BYTES 3584 /* bytes per (sequence, KV head, 64-token group) */

/* Pool of B * H_kv * capacity/64 records, [B][H_kv][capacity/64][record], in a
 * layout private to this library (key bit-planes, value bit-rows and their
 * fp16 scales and zeros).  Caller-allocated, 16-byte aligned. */
int jfa_onebit_pool_bytes(const jfa_geom* geom, size_t* pool_bytes);

/* Quantize the 64-token groups covering tokens [n_from, n_to) (multiples of
 * 64) of every (sequence, KV head) from the exact bf16 rows
 *   k_src, v_src : [B][H_kv][capacity][128] (device or pinned host).
 * A non-finite scale or zero sets JFA_DEVERR_NONFINITE_QUANT.  Stream-ordered. */
int jfa_onebit_pack(const jfa_geom* geom, int32_t n_from, int32_t n_to, const uint16_t* k_src,
                    const uint16_t* v_src, void* pool, void* ws, void* stream);

/* Dense attention: out[b, h] = softmax over every token t < n_ctx of
 * (scale q_h . k_t) applied to v_t, where tokens t < N_q use the dequantized
 * 1-bit keys and values of the pool (every group below N_q packed) and the
 * tail N_q .. n_ctx - 1 the exact rows k_exact / v_exact [B][H_kv][capacity]
 * [128] (device, or pinned host with exact_on_host = 1).  fp32 arithmetic.
 * One launch.  Stream-ordered. */
int jfa_onebit_attend(const jfa_geom* geom, const void* pool, const uint16_t* q, float scale,
                      const uint16_t* k_exact, const uint16_t* v_exact, int32_t exact_on_host,
                      void* ws, float* out, void* stream);

/* Number of warps jfa_decode_scores splits the quantized groups over on the
 * current device (0 on a bad geometry or when no group is quantized).  Warp w
 * takes a contiguous range of the flattened (segment, group) list and writes
 * its softmax partial for segment s to slot w + s of the workspace's
 * partials; exposed for inspection and tests. */
int jfa_scan_warps(const jfa_geom* geom);

#ifdef __cplusplus
}
#endif
#endif /* JFA_H_ */
