/*
 * cfr_paged.h -- C ABI of the B200 paged decode-attention library.
 *
 * One decode step of softmax attention for one query per head over a paged
 * KV cache, computed on one GPU by hand-written sm_100a kernels:
 *
 *   out[b][h] = softmax(q[b][h] . K_b^T * sigma + bias_h) V_b
 *
 * over the n_b = seq_lens[b] cached tokens of sequence b (scaled dot-product
 * attention as defined on the RustAttention page, "Mathematical Framework
 * Covered"; the decode query attends to every cached token).  K and V live in
 * fixed-size token pages reached through a page table (CFR-Atlas page, "page
 * identity and token ranges": a page holds a token range of one layer/head,
 * stored row-major [token][head_dim]).  Pages may be stored as fp32, bf16, or
 * as FP8 (E4M3) / int8 / int4 codes with a per-page, per-head scale (the FP8,
 * INT8 and INT4 tiers of the ARGUS page, "Visual Architecture"); quantised pages are
 * expanded only in on-chip memory ("Transient FP16 Reconstruction ... in GPU
 * SRAM").  Each page range's partial (running max, normaliser, weighted-V
 * accumulator) is folded exactly (CFR-Atlas page, "exact folded
 * online-softmax attention pass") and split partials are merged by their
 * log-sum-exp (CMF page, "split-K flash-decoding").
 *
 * Conventions for every entry point:
 *  - Ownership: every buffer belongs to the caller.  No entry point allocates
 *    or frees memory.  "device" pointers must be CUDA device memory (or
 *    managed memory) of the current device; "host" pointers host memory.
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *    default stream).  All GPU work is enqueued on it; no entry point
 *    synchronises with the host.
 *  - Errors: arguments are checked on the host before anything is launched; a
 *    rejected call returns a status and enqueues nothing.  Problems only the
 *    device can see (a page id outside its pool, an unknown page format, a
 *    sequence length outside [1, max_pages * page_tokens]) never fault: the
 *    kernel skips the offending page or sequence and ORs a CFR_DEVERR_* bit
 *    into *err_word (when err_word is not NULL).  The caller reads the word
 *    after synchronising; a non-zero word means the outputs of the affected
 *    sequences are not the attention result.
 *  - No data-value checks: non-finite K/V/q values propagate.
 */
#ifndef CFR_PAGED_H
#define CFR_PAGED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CFR_OK = 0,
  CFR_ERR_INVALID_ARG = 1,  /* NULL where a buffer is required, negative size, misalignment */
  CFR_ERR_UNSUPPORTED = 2,  /* valid but not implemented: head_dim, page_tokens, group size */
  CFR_ERR_OVERFLOW = 3,     /* a byte size or index does not fit its type */
  CFR_ERR_PAGE_INDEX = 4,   /* reserved for callers mapping a non-zero *err_word */
  CFR_ERR_CUDA = 5,         /* a CUDA runtime call failed (launch, attribute query) */
  CFR_ERR_TIMEOUT = 6,      /* reserved for callers mapping CFR_DEVERR_TIMEOUT */
  CFR_ERR_WORKSPACE = 7     /* workspace NULL, misaligned or smaller than required */
} cfr_status;

typedef enum {
  CFR_FMT_F32 = 0,   /* IEEE binary32 rows: 4 * head_dim bytes */
  CFR_FMT_BF16 = 1,  /* bfloat16 rows: 2 * head_dim bytes */
  CFR_FMT_I8 = 2,    /* int8 two's-complement codes: head_dim bytes; value = code * scale */
  CFR_FMT_I4 = 3,    /* int4 codes, 2 per byte: head_dim / 2 bytes; element 2i in the low
                        nibble, 2i+1 in the high nibble of byte i; value = code * scale */
  CFR_FMT_FP8 = 4,   /* FP8 E4M3 codes (sign, 4 exponent bits with bias 7, 3 mantissa bits,
                        no infinities, 0x7F/0xFF NaN, largest 448): head_dim bytes;
                        value = e4m3(code) * scale */
  CFR_FMT_COUNT = 5
} cfr_page_fmt;

/* Bits of the device error word (OR-ed, never cleared by the library). */
#define CFR_DEVERR_PAGE_ID 0x1u   /* page id < 0 or >= pool_pages[fmt]; page skipped */
#define CFR_DEVERR_PAGE_FMT 0x2u  /* page format >= CFR_FMT_COUNT; page skipped */
#define CFR_DEVERR_SEQ_LEN 0x4u   /* seq_lens[b] < 1 or > max_pages * page_tokens */
#define CFR_DEVERR_POOL 0x8u      /* page refers to a format whose pool (or scales) is NULL */
#define CFR_DEVERR_TIMEOUT 0x10u  /* a bounded on-device wait gave up; outputs undefined */
#define CFR_DEVERR_SCHEDULE 0x20u /* a call without CFR_PHASE_SCHEDULE found a split schedule in
                                     the workspace that does not fit its own arguments (more
                                     splits than its arrays hold, or a split outside its batch or
                                     page table); the extra or bad splits were skipped and the
                                     outputs are not the attention result */

/*
 * The paged K/V pools of one layer.  One pool per storage format; a page's
 * format selects its pool and the page table holds its slot inside that pool.
 *
 *   k_pool[f], v_pool[f]: device, uint8 [pool_pages[f]][num_kv_heads][page_tokens][row_bytes(f)]
 *       row_bytes: F32 4*d, BF16 2*d, I8 d, I4 d/2, FP8 d.  Every (slot, kv head)
 *       sub-page is a contiguous row-major [page_tokens][head_dim] block.
 *       Base addresses must be 16-byte aligned.  NULL for unused formats.
 *   scales[f]: device, float [pool_pages[f]][num_kv_heads][2] = (K scale, V scale)
 *       for f = I8, I4, FP8; ignored (may be NULL) for F32, BF16.
 *   pool_pages[f]: number of slots of pool f (0 when unused).
 *   Tokens of a sequence's last page at or past its length are never read
 *   as values (their bytes may hold anything, NaN included).
 */
typedef struct {
  int32_t num_kv_heads;
  int32_t head_dim;     /* 64 or 128 */
  int32_t page_tokens;  /* >= 8 */
  const void *k_pool[CFR_FMT_COUNT];
  const void *v_pool[CFR_FMT_COUNT];
  const float *scales[CFR_FMT_COUNT];
  int64_t pool_pages[CFR_FMT_COUNT];
} cfr_kv_pool;

/*
 * Bytes of device workspace that cfr_paged_decode needs for these sizes on
 * the current device (partials of every split plus the split schedule).
 * Returns 0 when the sizes are invalid or the byte count overflows.
 */
size_t cfr_paged_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t max_pages, int32_t page_tokens);

/*
 * One decode-attention step for every (sequence, query head).
 *
 *  q           device, [batch][num_q_heads][head_dim], fp32 (q_fmt = CFR_FMT_F32) or
 *              bf16 (CFR_FMT_BF16).  K is taken as already position-encoded
 *              (RoPE applied by the caller); ALiBi is applied here.
 *  kv          host pointer to the pool description above.
 *  page_table  device, int32 [batch][max_pages]: slot of logical page p of sequence b
 *              inside the pool of that page's format.  Entries past a
 *              sequence's last page are never read.
 *  seq_lens    device, int32 [batch]: n_b, 1 <= n_b <= max_pages * page_tokens.
 *  page_fmt    device, uint8 [batch][max_pages] format of every page, or NULL:
 *              every page has format uniform_fmt.
 *  head_map    host, int32 [num_q_heads]: kv head of each query head, or NULL:
 *              h -> h / (num_q_heads / num_kv_heads) (MHA, MQA, GQA; CFR-Atlas
 *              page, "MHA/MQA/GQA head mapping").  The query heads of a kv head
 *              are decoded together, reading its pages once, in groups of at
 *              most 16: a kv head serving more (MQA, wide GQA) has its pages
 *              read once per group of 16 (the groups of one split are taken
 *              side by side, so the later reads usually come from L2).
 *  alibi_slopes device, float [num_q_heads] or NULL: bias -slope_h * (n_b - 1 - j) is
 *              added to the score of token j (CFR-Atlas page, "RoPE/ALiBi
 *              positional policy").
 *  softmax_scale sigma; 0 selects 1/sqrt(head_dim).
 *  out         device, float [batch][num_q_heads][head_dim], written.
 *  lse         device, float [batch][num_q_heads] natural-log log-sum-exp of the
 *              scores, written; or NULL.
 *  workspace   device, >= cfr_paged_decode_workspace_size(...) bytes, 256-byte
 *              aligned; contents on entry are ignored, on return undefined.
 *              Calls that share a workspace must not overlap on the GPU.
 *  err_word    device uint32 or NULL; CFR_DEVERR_* bits are OR-ed into it.
 *
 * A sequence with n_b <= 0 or n_b > max_pages * page_tokens gets out = 0 and
 * lse = -inf and sets CFR_DEVERR_SEQ_LEN.
 */
cfr_status cfr_paged_decode(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                            const int32_t *page_table, int32_t max_pages,
                            const int32_t *seq_lens, int32_t batch, const uint8_t *page_fmt,
                            int32_t uniform_fmt, int32_t num_q_heads, const int32_t *head_map,
                            const float *alibi_slopes, float softmax_scale, float *out,
                            float *lse, void *workspace, size_t workspace_bytes,
                            uint32_t *err_word, void *stream);

/* Phase bits of cfr_paged_decode_phases. */
#define CFR_PHASE_SCHEDULE 0x1u  /* split schedule from seq_lens into the workspace */
#define CFR_PHASE_DECODE 0x2u    /* split partials into the workspace */
#define CFR_PHASE_MERGE 0x4u     /* partials -> out, lse */
#define CFR_PHASE_ALL 0x7u

/*
 * cfr_paged_decode split into its phases, for timing one at a time (CUDA
 * events between calls): the split schedule, the decode (on the tensor-core
 * path with a small launch before it that builds the query operands; a call
 * with both the schedule and the decode phase runs the schedule inside that
 * launch) and the merge.  Same arguments and checks as cfr_paged_decode;
 * `phases` selects which phases are enqueued.  A call
 * without CFR_PHASE_SCHEDULE relies on the workspace still holding what an
 * earlier call with the same arguments (all but q, out and lse) left there: the
 * split schedule, and the work-item counter that the schedule launch zeroes and
 * every completed decode launch leaves at zero.  The split count depends on the
 * pools and formats, not only on the sizes.  A call without CFR_PHASE_DECODE
 * merges the partials already in the workspace.  A call that breaks this rule
 * gets wrong outputs but no write outside its own workspace: the decode and
 * merge launches cap the split count and the split offsets at the capacity that
 * this call's workspace size provides, skip splits that name a sequence or page
 * outside this call's batch and page table, and set CFR_DEVERR_SCHEDULE.
 * cfr_paged_decode(...) == cfr_paged_decode_phases(..., CFR_PHASE_ALL).
 */
cfr_status cfr_paged_decode_phases(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                                   const int32_t *page_table, int32_t max_pages,
                                   const int32_t *seq_lens, int32_t batch,
                                   const uint8_t *page_fmt, int32_t uniform_fmt,
                                   int32_t num_q_heads, const int32_t *head_map,
                                   const float *alibi_slopes, float softmax_scale, float *out,
                                   float *lse, void *workspace, size_t workspace_bytes,
                                   uint32_t *err_word, void *stream, uint32_t phases);

/*
 * cfr_paged_decode restricted to a sink + recent-window token subset: each
 * softmax runs over the first sink_tokens tokens (attention sinks; ARGUS page,
 * "sink_tokens: keep initial attention sinks") and the last window_tokens
 * tokens (the recent window of the CFR-Atlas page's KeepRecent policy) of its
 * sequence, and over nothing else:
 *
 *   S_b = { j : j < sink_tokens or j >= n_b - window_tokens },
 *   out[b][h] = sum_{j in S_b} softmax_j(...) V_j,  ALiBi distance n_b - 1 - j as usual.
 *
 * The result is exact on the chosen set (no approximation of the skipped
 * tokens); pages holding no token of S_b are never read.  Same arguments,
 * workspace and errors as cfr_paged_decode, plus sink_tokens >= 0 and
 * window_tokens >= 1 (CFR_ERR_INVALID_ARG otherwise).  With
 * sink_tokens + window_tokens >= n_b the sequence is attended in full.
 * `phases` selects launches as for cfr_paged_decode_phases (CFR_PHASE_ALL for
 * one whole step); a call without CFR_PHASE_SCHEDULE needs the workspace of an
 * earlier call with the same arguments (all but q, out and lse), including
 * sink_tokens and window_tokens.
 */
cfr_status cfr_paged_decode_sink_window(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                                        const int32_t *page_table, int32_t max_pages,
                                        const int32_t *seq_lens, int32_t batch,
                                        const uint8_t *page_fmt, int32_t uniform_fmt,
                                        int32_t num_q_heads, const int32_t *head_map,
                                        const float *alibi_slopes, float softmax_scale,
                                        float *out, float *lse, void *workspace,
                                        size_t workspace_bytes, uint32_t *err_word, void *stream,
                                        int32_t sink_tokens, int32_t window_tokens,
                                        uint32_t phases);

/*
 * Multi-query decode over the paged cache: every sequence carries Q =
 * num_queries query tokens, its last Q positions (a speculative-decoding
 * verification step or a chunk of prefill over the cached prefix).  Query qi
 * (0 <= qi < Q) of sequence b sits at position n_b - Q + qi and attends
 * causally to the tokens j <= n_b - Q + qi (the causal mask of the
 * scaled dot-product definition, RustAttention page, "Mathematical Framework
 * Covered"); its ALiBi distance is n_b - Q + qi - j.  K/V of every query token
 * are already in the cache (as for cfr_paged_decode, whose num_queries = 1
 * case this is).
 *
 *  q    device [batch][num_queries][num_q_heads][head_dim] (fp32 or bf16 by q_fmt).
 *  out  device float [batch][num_queries][num_q_heads][head_dim];
 *  lse  device float [batch][num_queries][num_q_heads] or NULL.
 *  workspace  >= cfr_paged_decode_workspace_size(batch, num_q_heads * num_queries, ...).
 * Every K/V page is read once for all Q queries of a kv head's group: the
 * query rows (qi, h) of one kv head are decoded together in groups of at most
 * 16 rows (num_queries * query heads per kv head above 16 makes several
 * groups, each reading the kv head's pages).  num_queries in [1, 16]
 * (CFR_ERR_INVALID_ARG below 1, CFR_ERR_UNSUPPORTED above 16); at most 256
 * query rows (num_queries * num_q_heads) per sequence.  A sequence with
 * n_b < num_queries gets out = 0 and lse = -inf for every row and sets
 * CFR_DEVERR_SEQ_LEN.  `phases` as for cfr_paged_decode_phases.
 */
cfr_status cfr_paged_decode_multi(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                                  const int32_t *page_table, int32_t max_pages,
                                  const int32_t *seq_lens, int32_t batch, const uint8_t *page_fmt,
                                  int32_t uniform_fmt, int32_t num_q_heads, int32_t num_queries,
                                  const int32_t *head_map, const float *alibi_slopes,
                                  float softmax_scale, float *out, float *lse, void *workspace,
                                  size_t workspace_bytes, uint32_t *err_word, void *stream,
                                  uint32_t phases);

/*
 * Bytes of the scratch array compiled into the library for
 * cfr_paged_decode_static_workspace (one array per GPU that loads the library).
 */
#define CFR_STATIC_WORKSPACE_BYTES (16u << 20)

/*
 * cfr_paged_decode for callers that cannot allocate device memory: plugin or
 * operator interfaces that hand over only inputs and outputs, and code that
 * runs where another component owns every device allocation.  The pages this
 * library follows describe no counterpart of this entry point; it exists only
 * for such callers.
 *
 * Same arguments, checks and results as cfr_paged_decode, without `workspace`:
 * the split schedule and partials live in a fixed array of
 * CFR_STATIC_WORKSPACE_BYTES inside the library.  Nothing is allocated or
 * freed.  A problem whose cfr_paged_decode_workspace_size exceeds
 * CFR_STATIC_WORKSPACE_BYTES returns CFR_ERR_WORKSPACE and launches nothing.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it, so make that first call before any
 * stream capture.  All calls share the array: calls whose GPU work overlaps
 * race on it and must be serialised by the caller.  No part of the array needs
 * to start at zero.
 */
cfr_status cfr_paged_decode_static_workspace(const void *q, int32_t q_fmt,
                                             const cfr_kv_pool *kv,
                                             const int32_t *page_table, int32_t max_pages,
                                             const int32_t *seq_lens, int32_t batch,
                                             const uint8_t *page_fmt, int32_t uniform_fmt,
                                             int32_t num_q_heads, const int32_t *head_map,
                                             const float *alibi_slopes, float softmax_scale,
                                             float *out, float *lse, uint32_t *err_word,
                                             void *stream);

/*
 * Log-sum-exp merge of split partials into the attention output (the merge
 * step of split-K decoding, CMF page, "split-K flash-decoding"; the combine
 * rule of online softmax).  For each (b, h) over s in [split_off[b], split_off[b+1]):
 *
 *   M = max m_s over splits with l_s > 0,  w_s = 2^(m_s - M),
 *   out[b][h] = sum_s w_s a_s / sum_s w_s l_s,  lse[b][h] = (M + log2 sum_s w_s l_s) ln 2.
 *
 * part_m are base-2 maxima (scores times log2 e).  Splits with l_s = 0 are
 * skipped; with none left out = 0 and lse = -inf.  Summation runs over the
 * splits in index order, so results are deterministic.
 *
 *  part_acc device float [S][num_q_heads][head_dim]; part_m, part_l device
 *  float [S][num_q_heads]; split_off device int32 [batch + 1], non-decreasing,
 *  split_off[0] = 0.  out device float [batch][num_q_heads][head_dim]; lse
 *  device float [batch][num_q_heads] or NULL.  head_dim is 64 or 128.
 */
cfr_status cfr_merge_partials(const float *part_acc, const float *part_m, const float *part_l,
                              const int32_t *split_off, int32_t batch, int32_t num_q_heads,
                              int32_t head_dim, float *out, float *lse, void *stream);

/*
 * The ragged-batch split schedule that cfr_paged_decode uses, exposed for
 * inspection.  From seq_lens alone (device), every sequence is cut into
 * contiguous page ranges of `chunk` pages, where chunk = ceil(sum_b NP_b /
 * target_splits) (at least 1) and NP_b = ceil(n_b / page_tokens); sequence b
 * gets ceil(NP_b / chunk) splits.
 *
 *  split_off  device int32 [batch + 1]: first split index of each sequence.
 *  splits     device int32 [max_splits][3]: (b, first page, end page) of each split.
 *  num_splits device int32 [2]: (total splits, chunk pages), written.
 *  max_splits capacity of `splits`; schedules needing more set CFR_DEVERR_SEQ_LEN
 *             (cannot happen when max_splits >= target_splits + batch).
 */
cfr_status cfr_schedule_splits(const int32_t *seq_lens, int32_t batch, int32_t page_tokens,
                               int32_t max_pages, int32_t target_splits, int32_t *split_off,
                               int32_t *splits, int32_t max_splits, int32_t *num_splits,
                               uint32_t *err_word, void *stream);

/*
 * Raw page gather (diagnostic): copies the stored bytes of tokens [0, n_tokens)
 * of sequence b, kv head kv_head, in token order, through the same page-table
 * resolution as the decode kernels.  Row j of K goes to
 * k_raw_out + j * out_row_pitch (row_bytes of its page's format), likewise V.
 * Bytes of a row past its row_bytes are left untouched; rows of skipped pages
 * (bad id, bad format, NULL pool) are left untouched and set err_word bits.
 *
 *  page_table, page_fmt (or NULL + uniform_fmt): as for cfr_paged_decode, with
 *  `batch` rows; 0 <= b < batch, 0 <= n_tokens <= max_pages * page_tokens.
 *  k_raw_out, v_raw_out device, >= n_tokens * out_row_pitch bytes each;
 *  out_row_pitch a multiple of 16, >= the largest row_bytes in use.
 */
cfr_status cfr_gather_pages(const cfr_kv_pool *kv, const int32_t *page_table,
                            const uint8_t *page_fmt, int32_t uniform_fmt, int32_t batch,
                            int32_t max_pages, int32_t b, int32_t kv_head, int32_t n_tokens,
                            void *k_raw_out,
                            void *v_raw_out, int64_t out_row_pitch, uint32_t *err_word,
                            void *stream);

/*
 * Page demotion: re-encodes whole pages from one storage format into another,
 * the compression cascade of the ARGUS page ("Visual Architecture": full
 * precision hot pages, then FP8, INT8 and INT4 tiers).  Page k is read from
 * slot src_slots[k] of the src_fmt pool described by `kv` and written, every
 * kv head, K and V, to slot dst_slots[k] of the destination pool.  Per
 * (page, kv head, K-or-V) block, over its first valid_tokens[k] rows (all
 * page_tokens rows when valid_tokens is NULL):
 *   x     = the stored value as fp32 (quantised sources: code * scale, fp32 product);
 *   scale = max|x| / Q in fp32 with Q = 127 (I8), 7 (I4), 448 (FP8);
 *   I8/I4 code = clamp(round_half_even(x / scale), -Q, Q) (IEEE fp32 division);
 *   FP8   code = the E4M3 value nearest to x / scale, ties to even, saturating at 448;
 *   BF16  nearest bfloat16 (ties to even);  F32  x.
 * A block of zeros gets scale 0 and zero codes.  Rows at or past the valid
 * count are written as zero bytes.  Codes and scales are bit-exact functions
 * of the stored source bytes.  NaN values are left out of max|x| and get
 * integer code 0 and E4M3 code 0x7F; NaN bf16 and fp32 destination values are
 * unspecified NaNs.
 *
 *  kv           host; geometry (num_kv_heads, head_dim 64 or 128, page_tokens >= 8)
 *               and the source pool k_pool/v_pool/scales/pool_pages[src_fmt].
 *  src_fmt, dst_fmt  any two different formats.
 *  dst_k_pool, dst_v_pool  device, uint8 [dst_pool_pages][num_kv_heads][page_tokens]
 *               [row_bytes(dst_fmt)], 16-byte aligned, written; must not overlap
 *               the source pages.
 *  dst_scales   device float [dst_pool_pages][num_kv_heads][2], written for
 *               quantised dst_fmt (may be NULL otherwise).
 *  src_slots, dst_slots  device int32 [num_pages]; destination slots must be
 *               distinct.  A slot outside its pool skips the page and sets
 *               CFR_DEVERR_PAGE_ID.
 *  valid_tokens device int32 [num_pages] or NULL; a count outside [1, page_tokens]
 *               skips the page and sets CFR_DEVERR_SEQ_LEN.
 * The page table is the caller's: point page_table/page_fmt at the new slot
 * and format once the demotion has completed on the stream.
 */
cfr_status cfr_demote_pages(const cfr_kv_pool *kv, int32_t src_fmt, int32_t dst_fmt,
                            void *dst_k_pool, void *dst_v_pool, float *dst_scales,
                            int64_t dst_pool_pages, const int32_t *src_slots,
                            const int32_t *dst_slots, const int32_t *valid_tokens,
                            int32_t num_pages, uint32_t *err_word, void *stream);

/*
 * KV append: writes one new token per sequence into the full-precision tier
 * (recent tokens stay in high fidelity; ARGUS page, "The One-Minute
 * Explanation").  For every b with positions[b] >= 0, the rows
 * k_new[b][g][:], v_new[b][g][:] (every kv head g) become token
 * j = positions[b] of sequence b: row j % page_tokens of logical page
 * j / page_tokens, resolved through page_table / page_fmt exactly as the
 * decode resolves it.  Values are stored as fp32 (F32 pages) or rounded to
 * the nearest bfloat16 (BF16 pages).  positions[b] < 0 appends nothing.
 *
 *  kv          host; the F32 and BF16 pools in it are WRITTEN (their pointers
 *              must be writable device memory); other pools are ignored.
 *  page_table, page_fmt (or NULL + uniform_fmt F32/BF16), max_pages: as for
 *              cfr_paged_decode, `batch` rows.
 *  positions   device int32 [batch].
 *  k_new, v_new device [batch][num_kv_heads][head_dim], fp32 (new_fmt = CFR_FMT_F32)
 *              or bf16 (CFR_FMT_BF16).
 * Device-side faults skip the sequence and set err_word bits: a position at or
 * past max_pages * page_tokens (CFR_DEVERR_SEQ_LEN), a page that is not F32 or
 * BF16 or whose pool is NULL (CFR_DEVERR_PAGE_FMT), a slot outside its pool
 * (CFR_DEVERR_PAGE_ID).  Sequences must not share the written page row.
 */
cfr_status cfr_append_kv(const cfr_kv_pool *kv, const int32_t *page_table, int32_t max_pages,
                         const uint8_t *page_fmt, int32_t uniform_fmt, const int32_t *positions,
                         int32_t batch, const void *k_new, const void *v_new, int32_t new_fmt,
                         uint32_t *err_word, void *stream);

/*
 * Which decode kernel a call with these arguments would run (for tests and
 * benchmarks): 1 = general CUDA-core kernel (any format mix), 2 = tensor-core
 * (tcgen05) kernel, 3 = fp32 CUDA-core kernel with TMA tensor-map tiles, 0 if
 * the arguments would be rejected.  Host only; launches nothing.
 *
 * The tensor-core kernel takes bf16, FP8, int8 and int4 pages (no fp32) of
 * head_dim 64 or 128 with a 16-byte-aligned q, page_tokens dividing 128 or a
 * multiple of 128; quantised pages shorter than 128 tokens only when the cache
 * has one format (page_fmt NULL) and at most 8 query rows per kv head.  The
 * fp32 kernel takes fp32 caches with at most 2 query rows per kv head and the
 * same page sizes.  Everything else runs on the general kernel.
 */
int32_t cfr_paged_decode_path(int32_t q_fmt, const cfr_kv_pool *kv, int32_t max_pages,
                              const uint8_t *page_fmt, int32_t uniform_fmt,
                              int32_t num_q_heads, const int32_t *head_map);

/*
 * Diagnostic of the device-side failure handling (the pages have no
 * counterpart; it exists so that the bounded waits can be tested).  Every
 * wait of the decode kernels on an on-chip barrier gives up after a cycle limit
 * (about 4e9 SM cycles, two seconds at the top clock), ORs CFR_DEVERR_TIMEOUT
 * into *err_word and lets the kernel return, so a stalled pipeline ends as an
 * error bit the host reads rather than a hung GPU.  This call launches one
 * thread that runs that same wait on a shared-memory barrier, with a limit of
 * limit_cycles SM cycles, after arriving on the barrier itself when `arrive` is
 * non-zero and not arriving at all otherwise.
 *
 *  limit_cycles  1 .. 4e9 (CFR_ERR_INVALID_ARG otherwise).
 *  err_word      device uint32 or NULL; gets CFR_DEVERR_TIMEOUT when the wait gives up.
 *  result        device uint32 or NULL; written 1 when the barrier phase completed,
 *                0 when the wait gave up.
 * The kernel holds no copy or tensor-core operation in flight, so a wait that
 * gives up leaves the context usable.
 */
cfr_status cfr_wait_probe(int64_t limit_cycles, int32_t arrive, uint32_t *err_word,
                          uint32_t *result, void *stream);

/* Static description of a status code. */
const char *cfr_status_str(cfr_status status);

#ifdef __cplusplus
}
#endif

#endif /* CFR_PAGED_H */
