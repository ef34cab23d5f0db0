/*
 * csa.h -- C ABI of libcsa, a B200 (sm_100a) library for the hybrid attention
 * of DeepSeek-V4: Compressed Sparse Attention (CSA) and Heavily Compressed
 * Attention (HCA).
 *
 * Method source: the DeepSeek-V4 paper summary on hyper.ai (papers/2606.19348),
 * section "方法" (Method) -- the CSA paragraph (compression of every m tokens
 * with learnable weights and a position bias, a "lightning indexer" selecting
 * the top-k compressed entries, MQA with shared key and value), the HCA
 * paragraph (m' >> m tokens per entry without overlap, dense attention, and a
 * sliding-window branch in both), and the storage paragraph (RoPE dims in BF16,
 * the rest in FP8).  The DeepSeek-V4-Pro model cards (Hugging Face,
 * "Introduction", item 1 "hybrid attention architecture") state the same
 * CSA + HCA combination.
 *
 * Conventions (all entry points):
 *   - Every array argument is DEVICE memory owned by the caller, dense
 *     row-major in the shape given, and 16-byte aligned.  Structs passed by
 *     pointer (csa_kv_cache, csa_window) live in HOST memory; the pointers
 *     inside them are device pointers.  The library never allocates; scratch
 *     memory is queried with the *_workspace_size call and passed in.
 *   - bf16 = IEEE bfloat16; e4m3 = OCP FP8 E4M3 (bias 7, max 448, no inf).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL means
 *     the legacy default stream).  Argument and shape errors are detected on
 *     the host before anything is enqueued and returned synchronously; a
 *     kernel launch failure returns CSA_ERR_CUDA.  Faults inside an enqueued
 *     kernel surface at the caller's next synchronisation, as for any CUDA
 *     work.  csa_last_error() gives a message for the last failing call of
 *     the calling thread.
 *   - Positions are 0-based.  Entry i of a compression with stride s has
 *     nominal end e_i = (i+1)*s - 1; a query at position t sees entry i iff
 *     e_i <= t.  The sliding window of a query at t is the raw tokens at
 *     positions [max(0, t-win_len+1), t].  Entries and window keys share one
 *     softmax per head.
 *   - Fixed head geometry: qk dim 192 (128 "nope" + 64 RoPE channels), v dim
 *     128, indexer 4 heads x 64.  Query heads H must be 16 or 64.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA_API __attribute__((visibility("default")))
#else
#define CSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define CSA_D_QK 192
#define CSA_D_NOPE 128
#define CSA_D_ROPE 64
#define CSA_D_V 128
#define CSA_H_I 4
#define CSA_D_I 64

typedef enum csa_status {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or shape   */
  CSA_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels support   */
  CSA_ERR_WORKSPACE = 3,     /* workspace pointer NULL or smaller than asked */
  CSA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed         */
  CSA_ERR_DEVICE_TIMEOUT = 5 /* a kernel gave up a bounded wait (see below)  */
} csa_status;

typedef enum csa_kv_layout {
  /* k: bf16 [B, N, 192]; v: bf16 [B, N, 128], or NULL to use k[..., :128] */
  CSA_KV_BF16 = 0,
  /* split storage: nope e4m3 [B, N, 128], rope bf16 [B, N, 64], scale fp32
   * [B, N]; key = (nope * scale) ++ rope, value = nope * scale (shared K/V) */
  CSA_KV_SPLIT_FP8 = 1
} csa_kv_layout;

/* A compressed KV cache (host struct; device pointers). */
typedef struct csa_kv_cache {
  int32_t layout;            /* csa_kv_layout */
  int32_t reserved;          /* must be 0 */
  int64_t n_entries;         /* N, entries per sequence */
  const void* k;             /* CSA_KV_BF16 */
  const void* v;             /* CSA_KV_BF16, nullable */
  const uint8_t* nope;       /* CSA_KV_SPLIT_FP8 */
  const void* rope;          /* CSA_KV_SPLIT_FP8 */
  const float* scale;        /* CSA_KV_SPLIT_FP8 */
} csa_kv_cache;

/* Raw (uncompressed) tokens for the sliding-window branch (host struct). */
typedef struct csa_window {
  const void* k;             /* bf16 [B, rows, 192] */
  const void* v;             /* bf16 [B, rows, 128], or NULL to use k[..., :128] */
  int64_t pos0;              /* position of row 0 */
  int64_t rows;              /* rows held per sequence */
  int32_t len;               /* window length w_s (0 disables the branch) */
  int32_t reserved;          /* must be 0 */
} csa_window;

/*
 * Packed sequences (host struct; device pointers): several independent
 * sequences stored back to back in one buffer, e.g. the documents of a packed
 * pre-training batch.  The pages (DeepSeek-V4 summary, section "Datasets")
 * train on packed documents with sample-level attention masks: no compression
 * window, indexer score, sliding window or attention crosses from one sequence
 * into another.  Sequence s owns packed tokens [cu_tokens[s], cu_tokens[s+1])
 * (positions 0 .. len_s - 1 within the sequence) and compressed entries
 * [cu_entries[s], cu_entries[s+1]), ceil(len_s / stride) of them -- so a CSA
 * cache and an HCA cache of the same sequences need descriptors with their own
 * cu_entries.  Offsets are ascending int32 with cu_*[0] = 0.
 */
typedef struct csa_packed {
  const int32_t* cu_tokens;   /* device int32 [n_seqs + 1] */
  const int32_t* cu_entries;  /* device int32 [n_seqs + 1] */
  int32_t n_seqs;
  int32_t max_tokens;         /* length of the longest sequence (sizes launches and scratch) */
  int64_t total_tokens;       /* cu_tokens[n_seqs], < 2^31 */
  int64_t total_entries;      /* cu_entries[n_seqs], < 2^31 */
} csa_packed;

/* Library version string, e.g. "csa-b200 0.1.0 sm_100a". */
CSA_API const char* csa_version(void);
/* Name of a status code. */
CSA_API const char* csa_status_string(int32_t status);
/* Message for the last failing call made by this thread ("" if none). */
CSA_API const char* csa_last_error(void);

/*
 * csa_check_device_error -- synchronises `stream`, then reports (and clears)
 * the device error words of the attention and indexer kernels: their waits on
 * tensor-core and bulk-copy completion barriers are bounded, and a wait that
 * runs out records an error instead of hanging; the affected outputs are then
 * not valid.  Returns
 * CSA_OK, CSA_ERR_DEVICE_TIMEOUT, or CSA_ERR_CUDA if the synchronisation
 * itself fails.
 */
CSA_API csa_status csa_check_device_error(void* stream);

/*
 * csa_debug_expire_wait -- failure-detection check (library infrastructure,
 * not part of the method).  Enqueues one small kernel on `stream` whose single
 * bounded wait -- the same wait the attention and indexer kernels use on their
 * barriers -- is on a barrier nothing ever arrives at, so it runs out (2^14
 * rounds) and records a timeout.  The next csa_check_device_error on that
 * stream then returns CSA_ERR_DEVICE_TIMEOUT and clears the record; the
 * context stays usable.  Nothing faults, traps or hangs.  Returns CSA_OK or
 * CSA_ERR_CUDA (launch failure).
 */
CSA_API csa_status csa_debug_expire_wait(void* stream);

/*
 * csa_launch_count -- number of kernels this library has enqueued in this
 * process so far (library infrastructure, not part of the method).  Every
 * successful kernel launch counts once, including one recorded into a CUDA
 * graph capture (a replay of the graph does not count again).  Callers use
 * the difference around a call to see how many kernels it launched.
 */
CSA_API uint64_t csa_launch_count(void);

/*
 * csa_profile_next_call -- timing hook (library infrastructure, not part of
 * the method).  `start_event` and `stop_event` are cudaEvent_t handles created
 * by the caller.  The next entry point that enqueues work on this thread
 * records `start_event` on its stream immediately before its main kernel and
 * `stop_event` immediately after it (compression: the compression kernel;
 * indexer: the scoring kernel; attention: the attention kernel, without the
 * split combine), then forgets both.  Passing NULLs clears a pending hook.
 * Returns CSA_ERR_INVALID_ARG if exactly one handle is NULL.
 */
CSA_API csa_status csa_profile_next_call(void* start_event, void* stop_event);

/*
 * csa_compress -- CSA KV compression (Method section, CSA paragraph: every m
 * tokens become one entry through learnable compression weights and a position
 * bias; the windows overlap, in contrast to HCA's non-overlapping ones).
 *
 * Entry i (i < N = ceil(T/m)) covers the 2m tokens [(i-1)m, (i+1)m) clipped to
 * [0, T); for each channel c:
 *     alpha_j = softmax_j( w[c] * x[j,c] + b_pos[j - (i-1)m, c] )   (in-range j)
 *     y[i,c]  = sum_j alpha_j * x[j,c]
 *   x       bf16 [B, T, d], d a multiple of 8 in [8, 256]
 *   w       fp32 [d];  b_pos fp32 [2m, d]
 *   out_layout CSA_KV_BF16:      out = bf16 [B, N, d]   (out_rope, out_scale unused)
 *   out_layout CSA_KV_SPLIT_FP8: requires d == 192; out = e4m3 [B, N, 128],
 *       out_rope = bf16 [B, N, 64], out_scale = fp32 [B, N] with scale =
 *       max|y[:128]| / 448 (1 if zero) and codes = RNE-satfinite(y / scale).
 *   1 <= m <= 64.  T == 0 is a no-op.
 */
CSA_API csa_status csa_compress(const void* x, int64_t B, int64_t T, int32_t d, int32_t m,
                        const float* w, const float* b_pos, int32_t out_layout,
                        void* out, void* out_rope, float* out_scale, void* stream);

/*
 * hca_compress -- HCA KV compression (Method section, HCA paragraph: m' >> m
 * tokens per entry, no overlap).  Entry i covers [i m', (i+1) m') clipped to
 * [0, T) (the trailing entry may be partial); same per-channel softmax as
 * csa_compress with b_pos fp32 [m', d].  N = ceil(T/m'), 1 <= m' <= 4096.
 * Arguments and layouts as csa_compress.
 */
CSA_API csa_status hca_compress(const void* x, int64_t B, int64_t T, int32_t d, int32_t m_prime,
                        const float* w, const float* b_pos, int32_t out_layout,
                        void* out, void* out_rope, float* out_scale, void* stream);

/*
 * csa_compress_append / hca_compress_append -- incremental cache append at
 * decode time (same entry rule as csa_compress / hca_compress).  Every
 * sequence of the call has just received the token at position t.  When t + 1
 * is a multiple of the stride (m, or m' for HCA), entry i = (t+1)/stride - 1
 * has just become complete; it is computed from the sequence's recent raw
 * tokens and written into slot i of a resident cache that holds n_cap entries
 * per sequence.  Otherwise nothing completes and the call returns CSA_OK
 * without enqueueing work.
 *   x       bf16 [B, rows, d]: row j of a sequence holds its token at
 *           position x_pos0 + j; the rows must hold the entry's window
 *           [max(0, i m - (window - stride)), t]
 *   out...  the cache planes, as csa_compress with N replaced by n_cap
 *           (bf16 [B, n_cap, d], or the split FP8 planes for d == 192)
 *   i < n_cap.  Other arguments and errors as csa_compress.
 */
CSA_API csa_status csa_compress_append(const void* x, int64_t B, int64_t rows, int64_t x_pos0, int64_t t,
                                       int32_t d, int32_t m, const float* w, const float* b_pos,
                                       int32_t out_layout, void* out, void* out_rope, float* out_scale,
                                       int64_t n_cap, void* stream);
CSA_API csa_status hca_compress_append(const void* x, int64_t B, int64_t rows, int64_t x_pos0, int64_t t,
                                       int32_t d, int32_t m_prime, const float* w, const float* b_pos,
                                       int32_t out_layout, void* out, void* out_rope, float* out_scale,
                                       int64_t n_cap, void* stream);

/*
 * csa_compress_packed / hca_compress_packed -- compression of packed
 * sequences: each sequence is compressed on its own (its windows never reach
 * into a neighbour), its entries landing in rows [cu_entries[s],
 * cu_entries[s+1]) of out.
 *   x    bf16 [total_tokens, d];  out: as csa_compress with B*N replaced by
 *        total_entries.  packed->cu_entries must use this call's stride.
 */
CSA_API csa_status csa_compress_packed(const void* x, const csa_packed* packed, int32_t d, int32_t m,
                                       const float* w, const float* b_pos, int32_t out_layout, void* out,
                                       void* out_rope, float* out_scale, void* stream);
CSA_API csa_status hca_compress_packed(const void* x, const csa_packed* packed, int32_t d, int32_t m_prime,
                                       const float* w, const float* b_pos, int32_t out_layout, void* out,
                                       void* out_rope, float* out_scale, void* stream);

/* Workspace bytes csa_indexer_topk needs for these sizes (0 for prefill rows,
 * whose scores stay on chip; nonzero for the long decode rows). */
CSA_API size_t csa_indexer_topk_workspace_size(int64_t B, int64_t Tq, int64_t N, int32_t k);
/* Workspace bytes csa_indexer_topk_e4m3, csa_indexer_topk_e2m1 and
 * csa_indexer_topk_with_scores need (their prefill rows keep a score row per
 * query in the workspace). */
CSA_API size_t csa_indexer_topk_coded_workspace_size(int64_t B, int64_t Tq, int64_t N, int32_t k);

/*
 * csa_indexer_topk -- the lightning indexer and its top-k selection (Method
 * section, CSA paragraph).  For query row r of sequence b at position
 * t = q_pos0 + r and every visible entry i (e_i = (i+1)m - 1 <= t):
 *     s[i] = sum_{h<4} relu(qI[b,r,h,:] . kIc[b,i,:]) * wI[b,r,h]
 * and idx[b,r,:] receives the k entries with the highest scores, ties broken
 * toward the lower index, as an ascending list padded with -1 when fewer than
 * k entries are visible.
 *   qI  bf16 [B, Tq, 4, 64];  wI fp32 [B, Tq, 4];  kIc bf16 [B, N, 64]
 *   idx int32 [B, Tq, k] (output)
 *   1 <= k <= 4096, 1 <= m, 0 <= q_pos0 < 2^50, N < 2^31, B * Tq < 2^31.
 */
CSA_API csa_status csa_indexer_topk(const void* qI, const float* wI, const void* kIc,
                            int64_t B, int64_t Tq, int64_t N, int64_t q_pos0, int32_t m,
                            int32_t k, int32_t* idx, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * csa_indexer_topk_with_scores -- csa_indexer_topk that also returns, in
 * scores fp32 [B, Tq, k], the score of each selected entry (-inf in padded
 * slots).  Workspace: csa_indexer_topk_coded_workspace_size.  Errors as
 * csa_indexer_topk.  The
 * context-parallel decode uses it: each rank selects a local top-k over its
 * range of entries and the ranks' (score, index) candidates are merged by
 * csa_cp_topk_merge.
 */
CSA_API csa_status csa_indexer_topk_with_scores(const void* qI, const float* wI, const void* kIc, int64_t B,
                                                int64_t Tq, int64_t N, int64_t q_pos0, int32_t m, int32_t k,
                                                int32_t* idx, float* scores, void* workspace,
                                                size_t workspace_bytes, void* stream);

/*
 * csa_indexer_topk_e4m3 -- csa_indexer_topk over indexer keys stored in FP8
 * (Method section, storage paragraph: the lightning indexer runs at low
 * precision -- the pages give FP4; this layout stores E4M3 codes).  Entry i's
 * key is kI_codes[b,i,:] (64 E4M3 bytes) times kI_scale[b,i] (fp32, > 0); the
 * score is computed from those exact values (the scale factors out of the relu
 * and head sums).  Workspace: csa_indexer_topk_coded_workspace_size.  Same
 * selection rule, output and errors as csa_indexer_topk.
 *   kI_codes uint8 [B, N, 64];  kI_scale fp32 [B, N]
 */
CSA_API csa_status csa_indexer_topk_e4m3(const void* qI, const float* wI, const uint8_t* kI_codes,
                                         const float* kI_scale, int64_t B, int64_t Tq, int64_t N,
                                         int64_t q_pos0, int32_t m, int32_t k, int32_t* idx,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * csa_indexer_topk_e2m1 -- csa_indexer_topk over FP4 indexer keys (Method
 * section, storage paragraph: FP4 precision for the lightning indexer).  Each
 * key is 64 OCP MX E2M1 codes (sign, 2 exponent bits with bias 1, 1 mantissa
 * bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per byte -- dimension 2j in
 * the low nibble of byte j, 2j+1 in the high nibble -- times one fp32 scale
 * per entry (> 0; max|k| / 6 is the natural choice).  Scores are computed from
 * those exact values.  Workspace: csa_indexer_topk_coded_workspace_size.
 * Same selection rule, output and errors as csa_indexer_topk.
 *   kI_codes uint8 [B, N, 32];  kI_scale fp32 [B, N]
 */
CSA_API csa_status csa_indexer_topk_e2m1(const void* qI, const float* wI, const uint8_t* kI_codes,
                                         const float* kI_scale, int64_t B, int64_t Tq, int64_t N,
                                         int64_t q_pos0, int32_t m, int32_t k, int32_t* idx,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * csa_indexer_topk_noalloc -- csa_indexer_topk without a caller workspace.
 * The paper has no counterpart: this is a library convenience.  Some callers
 * cannot allocate device memory themselves (for example a plugin whose host
 * application owns every device allocation, or code on a latency-critical
 * path that must not call cudaMalloc); this call needs none.  Its scratch is a
 * 32 MiB static device array inside the library, held on every GPU that loads
 * the library until the process exits.  Sizes whose workspace
 * (csa_indexer_topk_workspace_size) exceeds 32 MiB are rejected with
 * CSA_ERR_UNSUPPORTED and a message; e.g. 8 decode rows over 262,144 entries
 * fit.  Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress, which allocates nothing); the first call on a device
 * may also load the library's device code there, so make it before any
 * stream capture.  No call allocates.  Every call
 * shares the array and it keeps the last call's contents (the call clears what
 * must start at zero), so calls that overlap on the GPU race on it.  Other
 * arguments, outputs and errors as csa_indexer_topk.
 */
CSA_API csa_status csa_indexer_topk_noalloc(const void* qI, const float* wI, const void* kIc,
                                            int64_t B, int64_t Tq, int64_t N, int64_t q_pos0,
                                            int32_t m, int32_t k, int32_t* idx, void* stream);

/* Workspace bytes csa_indexer_topk_packed needs for these packed sequences. */
CSA_API size_t csa_indexer_topk_packed_workspace_size(const csa_packed* packed, int32_t m, int32_t k);

/*
 * csa_indexer_topk_packed -- csa_indexer_topk over packed sequences: every
 * token of every sequence is a query row (prefill), sequence s's row at
 * position t (t = 0 at the sequence's first token) sees that sequence's
 * entries i with (i+1)m - 1 <= t only.  Output indices are entry indices
 * within the sequence (0 = its first entry), ascending, -1 padded.
 *   qI  bf16 [total_tokens, 4, 64];  wI fp32 [total_tokens, 4]
 *   kIc bf16 [total_entries, 64] (e.g. csa_compress_packed's output)
 *   idx int32 [total_tokens, k] (output)
 *   packed->cu_entries must use stride m.  Sequences of up to 65535 entries
 *   (ceil(max_tokens / m)); longer ones return CSA_ERR_UNSUPPORTED.  The
 *   scores stay on chip; the workspace (a few bytes per sequence) holds a
 *   table of the sequences' 32-row groups.  Other limits and errors as
 *   csa_indexer_topk.
 */
CSA_API csa_status csa_indexer_topk_packed(const void* qI, const float* wI, const void* kIc,
                                           const csa_packed* packed, int32_t m, int32_t k, int32_t* idx,
                                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace bytes csa_sparse_mqa needs for these sizes on the current device
 * (it depends on the device's SM count).  Nonzero when H = 64 and there are
 * too few query rows (B * Tq) to fill the device: each row's keys are then
 * split over several CTAs whose partial softmax states (per head: 128
 * unnormalised output channels, running max, sum) are merged from this
 * buffer.  Pass at least this many bytes, 16-byte aligned; otherwise the call
 * returns CSA_ERR_WORKSPACE.  The buffer holds no state between calls.
 */
CSA_API size_t csa_sparse_mqa_workspace_size(int64_t B, int64_t Tq, int32_t H, int32_t k, int32_t win_len);

/*
 * csa_sparse_mqa -- CSA core attention (Method section, CSA paragraph: MQA with
 * one key/value head shared by all query heads, over the selected entries; HCA
 * paragraph: plus a sliding-window branch of raw recent tokens).  For query
 * row r of sequence b at t = q_pos0 + r and each head h, one softmax over
 *     { scale * q[b,r,h] . K_entry(i) : i in idx[b,r,:], 0 <= i < N, e_i <= t }
 *   u { scale * q[b,r,h] . K_raw(p)   : p in [max(0,t-win_len+1), t] }
 * and out = sum of probabilities times the matching values.
 *   q     bf16 [B, Tq, H, 192]
 *   cache compressed entries (either layout), N = cache->n_entries
 *   idx   int32 [B, Tq, k] (slots that are -1, out of range or not visible
 *         are skipped)
 *   win   raw tokens; must hold every window position of every query
 *   out   bf16 [B, Tq, H, 128];  lse fp32 [B, Tq, H] natural-log
 *         log-sum-exp of the scaled logits (nullable).  A query with no keys
 *         gets out = 0 and lse = -inf.
 */
CSA_API csa_status csa_sparse_mqa(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0,
                          const csa_kv_cache* cache, int32_t m, const int32_t* idx, int32_t k,
                          const csa_window* win, float scale, void* out, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes hca_dense_mqa needs for these sizes on the current device
 * (same rule as csa_sparse_mqa_workspace_size with k replaced by N). */
CSA_API size_t hca_dense_mqa_workspace_size(int64_t B, int64_t Tq, int32_t H, int64_t N, int32_t win_len);

/*
 * hca_dense_mqa -- HCA core attention (Method section, HCA paragraph: dense
 * attention over all heavily compressed entries, no selection, plus the same
 * sliding window).  As csa_sparse_mqa with the entry set replaced by every
 * visible entry i < N (e_i = (i+1)m' - 1 <= t).
 */
CSA_API csa_status hca_dense_mqa(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0,
                         const csa_kv_cache* cache, int32_t m_prime, const csa_window* win,
                         float scale, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * hca_dense_mqa_budget -- hca_dense_mqa whose 64-head decode launch keeps to
 * at most max_sms SMs (one CTA per SM on that path, at least one CTA per
 * query row), so that work the caller runs beside it on another stream (the
 * CSA branch's indexer, which does not depend on the HCA branch) keeps the
 * other SMs.  max_sms = 0: every SM (identical to hca_dense_mqa).  The result
 * is the same attention up to the summation order of the split merge; the
 * workspace hca_dense_mqa_workspace_size reports is always enough.  Calls
 * with at least as many query rows as SMs, 16 heads, or the query-blocked
 * prefill kernel are unaffected.  max_sms < 0 returns CSA_ERR_INVALID_ARG.
 */
CSA_API csa_status hca_dense_mqa_budget(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0,
                                const csa_kv_cache* cache, int32_t m_prime, const csa_window* win,
                                float scale, void* out, float* lse, int32_t max_sms, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * csa_sparse_mqa_packed / hca_dense_mqa_packed -- the core attention over
 * packed sequences (sample-level masks): query row r is packed token r, at
 * position t within its sequence s; its entry set is drawn from s's entries
 * only (cache rows cu_entries[s] + i, visibility (i+1)*stride - 1 <= t) and
 * its sliding window from s's own tokens [max(0, t - len + 1), t].
 *   q     bf16 [total_tokens, H, 192]
 *   cache n_entries == total_entries (e.g. csa_compress_packed's output)
 *   idx   int32 [total_tokens, k] of entry indices within the sequence
 *         (csa_indexer_topk_packed's output)
 *   win   the packed raw tokens: k bf16 [total_tokens, 192], v nullable,
 *         pos0 = 0, rows = total_tokens
 *   out   bf16 [total_tokens, H, 128];  lse fp32 [total_tokens, H] (nullable)
 *   workspace: csa_sparse_mqa_workspace_size(1, total_tokens, H, k, len), or
 *   for HCA hca_dense_mqa_workspace_size(1, total_tokens, H,
 *   ceil(max_tokens / m'), len).  Other rules as csa_sparse_mqa.
 */
CSA_API csa_status csa_sparse_mqa_packed(const void* q, int32_t H, const csa_packed* packed,
                                         const csa_kv_cache* cache, int32_t m, const int32_t* idx, int32_t k,
                                         const csa_window* win, float scale, void* out, float* lse,
                                         void* workspace, size_t workspace_bytes, void* stream);
CSA_API csa_status hca_dense_mqa_packed(const void* q, int32_t H, const csa_packed* packed,
                                        const csa_kv_cache* cache, int32_t m_prime, const csa_window* win,
                                        float scale, void* out, float* lse, void* workspace,
                                        size_t workspace_bytes, void* stream);

/*
 * Context-parallel decode of one long sequence over G ranks (one process per
 * GPU).  The pages name no parallel scheme for the attention; this split is
 * exact: rank r holds the contiguous entry range [lo_r, lo_{r+1}) (lo
 * ascending with r) of the compressed caches and scores it with
 * csa_indexer_topk_with_scores (q_pos0 shifted by -lo_r * m so that
 * visibility is unchanged); the G candidate lists, all-gathered in rank order
 * and made global (local index + lo_r), are merged here into the global top-k,
 * which is exactly the top-k of the whole sequence; each rank attends over the
 * selected entries it holds (indices minus lo_r; the others fall outside its
 * range and are skipped) and one rank also over the window; the partial
 * (out, lse) of all ranks are merged by csa_cp_attn_merge.
 *
 * csa_cp_topk_merge -- per row, the k best of n_cand candidates.
 *   cand_scores fp32 [R, n_cand], cand_idx int32 [R, n_cand] (-1 = no
 *   candidate): the concatenation, in rank order, of each rank's ascending
 *   list, so that positions ascend with the global index.
 *   idx int32 [R, k]: the selected global indices, ascending, ties to the
 *   lower index, -1 padded.  1 <= k <= 4096, 1 <= n_cand <= 32768.
 */
CSA_API csa_status csa_cp_topk_merge(const float* cand_scores, const int32_t* cand_idx, int64_t R,
                                     int32_t n_cand, int32_t k, int32_t* idx, void* stream);

/*
 * csa_cp_attn_merge -- combines G partial attentions of the same query rows
 * over disjoint key sets (each with its own softmax) into the attention over
 * their union:  out = sum_g w_g out_g / sum_g w_g,  w_g = exp(lse_g - max lse),
 * lse = max lse + ln sum_g w_g.  A part with lse = -inf (no keys) has weight 0;
 * rows where every part is empty get out = 0, lse = -inf.
 *   outs bf16 [G, R, H, 128], lses fp32 [G, R, H] -> out bf16 [R, H, 128],
 *   lse fp32 [R, H] (nullable).
 */
CSA_API csa_status csa_cp_attn_merge(const void* outs, const float* lses, int32_t G, int64_t R, int32_t H,
                                     void* out, float* lse, void* stream);

/*
 * csa_grouped_out_proj -- grouped output projection after the core attention
 * (Method section, CSA paragraph: the MQA is followed by a grouped output
 * projection that keeps its compute cost down).  The H heads form G groups of
 * H/G consecutive heads; group g's outputs, concatenated head after head
 * (K = (H/G) * 128 values per row), are multiplied by the group's own weight:
 *     y[r, g, j] = sum_{c<K} o[r, g*H/G + c/128, c%128] * w[g, j, c]
 *   o  bf16 [R, H, 128]   (the attention output, e.g. csa_sparse_mqa's out with
 *                          R = B * Tq)
 *   w  bf16 [G, d_g, K]   (row j of w[g]: the weights of output channel j, the
 *                          layout of a linear layer's [out, in] weight)
 *   y  bf16 [R, G, d_g]   (output; fp32 accumulation)
 *   1 <= G, G divides H (H <= 256), d_g a multiple of 64.  R == 0 is a no-op.
 * A layer that mixes the G groups afterwards is an ordinary dense linear layer
 * outside this call.  Needs no workspace.
 */
CSA_API csa_status csa_grouped_out_proj(const void* o, int64_t R, int32_t H, int32_t G, int32_t d_g,
                                        const void* w, void* y, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H_ */
