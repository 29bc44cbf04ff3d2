/*
 * kld.h - C ABI of libkld: teacher-forced KL(reference || candidate) scoring
 * of next-token distributions on NVIDIA B200 (sm_100a).
 *
 * What is computed (sources are web pages, cited by title and section):
 *
 *  - Per scored position, KL(p || q) = sum_i p_i (log p_i - log q_i) where p
 *    and q are the softmax of the reference and candidate logits over the
 *    whole vocabulary ("Qwen3.8-27B Quantization Challenge", sections "How
 *    the references were made" and "The score"), the exact argmax of each
 *    side for top-1 agreement and the log-probability of the true next token
 *    for perplexity ("Qwopus3.8-27B-Coder-Flash: quality-eval reference",
 *    section "Method").
 *  - The top-64 + one tail bucket approximation of that KL from stored top-k
 *    lists ("Qwopus3.8-27B-Coder-Flash: quality-eval reference", "Method"
 *    and "Files").
 *  - The same full-vocabulary scores from final hidden states pushed through
 *    one shared BF16 LM head ("Qwen3.8-27B fidelity suite v5", opening
 *    paragraph).
 *  - Mean / percentile / top-1 / perplexity / exceedance reductions
 *    ("Qwen3.8-27B Quantization Challenge", "The score"; "Qwen3.8-27B IQ8R
 *    ... radiance container", "Quality"; "Qwen3.8-27B fidelity suite v5",
 *    "What is in here").
 *
 * Conventions shared by every entry point:
 *
 *  - Memory.  Every pointer argument is a DEVICE pointer unless its comment
 *    says "host".  The caller owns all memory; the library allocates nothing
 *    and keeps no state between calls.
 *  - Streams.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *    default stream).  Every call only enqueues work on that stream and
 *    returns without synchronising.
 *  - Errors detectable on the host (bad sizes, null or misaligned pointers,
 *    unsupported dtype, workspace too small) are returned synchronously and
 *    nothing is launched.  KLD_ERR_CUDA means a CUDA launch failed; the
 *    stream may then hold partial results.
 *  - Errors found on the device are OR-ed into *dev_status as KLD_DEV_* bits
 *    (dev_status may be NULL to ignore them).  The caller zeroes the word
 *    before the call and reads it after synchronising.  The library never
 *    traps or asserts on the device.
 *  - Determinism.  For a given shape every output is bitwise identical from
 *    run to run: all reductions use fixed trees and fixed orders, never
 *    floating-point atomics.
 *  - Thread safety.  Calls are reentrant; concurrent calls on different
 *    streams must not share output, workspace or dev_status buffers.
 */
#ifndef KLD_H_
#define KLD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kld_status {
  KLD_OK = 0,
  KLD_ERR_INVALID_ARG = 1, /* null required pointer, bad size or bad combination */
  KLD_ERR_ALIGNMENT = 2,   /* a pointer or leading dimension breaks the alignment rules */
  KLD_ERR_UNSUPPORTED = 3, /* dtype or size outside what the kernels implement */
  KLD_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than the *_workspace_size query */
  KLD_ERR_CUDA = 5         /* a CUDA runtime call or kernel launch failed */
} kld_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define KLD_DEV_BAD_TARGET 0x1 /* a target id was outside [0, vocab): that row's target lps are NaN */
#define KLD_DEV_BAD_ID 0x2     /* an id was outside its range: a top-k id (that row's KL is NaN),
                                  a cluster id or a bootstrap draw (see kld_paired_compare) */
#define KLD_DEV_TIMEOUT 0x4    /* a bounded wait inside a kernel gave up; outputs are invalid */

typedef enum kld_dtype {
  KLD_F32 = 0,  /* IEEE binary32 logits */
  KLD_BF16 = 1  /* bfloat16 logits (upper half of a binary32) */
} kld_dtype;

/* Library version (major * 10000 + minor * 100 + patch). */
int kld_version(void);

/* Static, NUL-terminated description of a status code. */
const char* kld_status_string(kld_status s);

/*
 * kld_full_vocab - full-vocabulary scoring of n_rows positions.
 *
 * Defines ("Qwen3.8-27B Quantization Challenge", "How the references were
 * made" / "The score"; "Qwopus3.8-27B-Coder-Flash: quality-eval reference",
 * "Method"): for row r with reference logits x = ref_logits[r, 0:vocab] and
 * candidate logits y = cand_logits[r, 0:vocab], p = softmax(x),
 * q = softmax(y), computed in f32 arithmetic (f64 for the final per-row
 * combination):
 *    kl[r]             = sum_i p_i (log p_i - log q_i)        (nats)
 *    ref_argmax[r]     = lowest i with x_i = max x   (cand_argmax: same on y)
 *    ref_target_lp[r]  = log p_t,  cand_target_lp[r] = log q_t,  t = target_ids[r]
 *
 * Each logit is read from HBM exactly once (single streaming pass).  The
 * work is split over a fixed set of warps that write per-row partial states
 * to `workspace`; a second kernel merges them in index order, so results
 * are bitwise reproducible and do not depend on the device.
 *
 * Arguments:
 *   ref_logits, cand_logits  [n_rows, ld_*] row-major, element type `dtype`.
 *                            16-byte aligned; ld_* * sizeof(element) must be
 *                            a multiple of 16 bytes, ld_* >= vocab.
 *   n_rows                   >= 0 (0 launches nothing).
 *   vocab                    1 .. 2^31 - 1.
 *   target_ids               int32 [n_rows], or NULL.  When NULL both
 *                            *_target_lp outputs must be NULL.
 *   kl                       f32 [n_rows], required.
 *   ref_argmax, cand_argmax  int32 [n_rows], each may be NULL.
 *   ref_target_lp, cand_target_lp  f32 [n_rows], each may be NULL.
 *   workspace                device scratch of at least
 *                            kld_full_vocab_workspace_size(n_rows) bytes,
 *                            256-byte aligned; no initial contents needed.
 *   dev_status               int32 device word, may be NULL.
 *
 * Non-finite input: -inf logits are allowed (an id with p_i = 0 contributes
 * nothing; p_i > 0 against a candidate -inf gives kl = +inf).  A row holding
 * NaN or +inf, or no finite logit, gives kl = NaN, argmax = -1 and NaN
 * target lps.  A target id outside [0, vocab) gives NaN target lps and sets
 * KLD_DEV_BAD_TARGET.
 * Range: differences ref_i - cand_i and z_i - max(z) are formed in f32, so
 * finite logits of any magnitude are scored as long as those differences
 * stay within the f32 range (always so when every |logit| <= 1.7e38); a
 * row where one overflows may give kl = inf or NaN.
 */
kld_status kld_full_vocab(const void* ref_logits, const void* cand_logits, kld_dtype dtype,
                          int64_t n_rows, int64_t vocab, int64_t ld_ref, int64_t ld_cand,
                          const int32_t* target_ids, float* kl, int32_t* ref_argmax,
                          int32_t* cand_argmax, float* ref_target_lp, float* cand_target_lp,
                          void* workspace, size_t workspace_bytes, int32_t* dev_status,
                          void* stream);

/* Workspace bytes kld_full_vocab needs for n_rows rows (any vocab, dtype). */
size_t kld_full_vocab_workspace_size(int64_t n_rows);

/*
 * kld_full_vocab_noalloc - kld_full_vocab for callers that cannot allocate
 * device memory.
 *
 * No counterpart on the pages: this entry exists for the library's users,
 * not for the method.  Some callers cannot call cudaMalloc, or hand this
 * library a workspace, at the point where they score: code running inside
 * another framework that owns every byte of device memory through its own
 * pool and forbids side allocations, a process already at its memory limit,
 * or a latency-sensitive loop where an allocation (which may synchronise the
 * device) is not acceptable.  They pass inputs and outputs only; the scratch
 * lives in a fixed device array inside the library.
 *
 * Same arguments and results as kld_full_vocab without the workspace.
 * Limits and behaviour:
 *   - n_rows <= KLD_NOALLOC_MAX_ROWS; larger n_rows returns
 *     KLD_ERR_UNSUPPORTED and launches nothing (split the batch instead).
 *   - The array takes about 1.1 MB on every GPU that loads the library and
 *     stays allocated until the process exits.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current, and so does the first
 *     call in a new context of that device (e.g. after cudaDeviceReset);
 *     make that first call before any stream capture.
 *   - Every call on a device shares the one array.  Calls that may overlap
 *     on the GPU (different streams, or several host threads) race and can
 *     corrupt each other's results: serialise them.  The array keeps the last
 *     call's contents; nothing in it needs to start at zero.
 */
#define KLD_NOALLOC_MAX_ROWS 32768
kld_status kld_full_vocab_noalloc(const void* ref_logits, const void* cand_logits, kld_dtype dtype,
                                  int64_t n_rows, int64_t vocab, int64_t ld_ref, int64_t ld_cand,
                                  const int32_t* target_ids, float* kl, int32_t* ref_argmax,
                                  int32_t* cand_argmax, float* ref_target_lp, float* cand_target_lp,
                                  int32_t* dev_status, void* stream);

/*
 * kld_topk_tail - KL over the reference's top-k ids plus one tail bucket.
 *
 * Defines ("Qwopus3.8-27B-Coder-Flash: quality-eval reference", "Method";
 * list layout from "Files"): per position, with reference list (R ids,
 * log-probs a_j) and candidate list (C ids, log-probs b_s), k entries each,
 * both sorted by descending probability:
 *    c_s      = exp(b_s);  leftover = max(0, 1 - sum_s c_s)
 *    spread   = leftover / (vocab - k)          (mass of each id outside C)
 *    q_j      = c_s and log q_j = b_s   if R_j = C_s (first such s)
 *             = spread, log q_j = log max(spread, 1e-12)   otherwise
 *    p_j      = exp(a_j);  p_tail = 1 - sum_j p_j;  q_tail = 1 - sum_j q_j
 *    kl       = sum_j p_j (a_j - log q_j)
 *             + [p_tail > 0] p_tail (log p_tail - log max(q_tail, 1e-12))
 *    top1     = (R_0 == C_0)
 * The two mass sums are accumulated in f64.
 *
 * Arguments:
 *   ref_ids, cand_ids    int32 [n_rows, k] row-major (row stride k), ids in [0, vocab).
 *   ref_lp, cand_lp      IEEE binary16 bit patterns [n_rows, k] (row stride k).
 *   k                    1 .. 64;  vocab: k < vocab < 2^25.
 *   kl                   f32 [n_rows], required.
 *   top1                 uint8 [n_rows] (0/1), may be NULL.
 *   n_matched            int32 [n_rows] (ids of R found in C), may be NULL.
 * All arrays need only their natural alignment.  An id outside [0, vocab)
 * makes that row's kl NaN and sets KLD_DEV_BAD_ID.
 */
kld_status kld_topk_tail(const int32_t* ref_ids, const uint16_t* ref_lp,
                         const int32_t* cand_ids, const uint16_t* cand_lp,
                         int64_t n_rows, int32_t k, int64_t vocab,
                         float* kl, uint8_t* top1, int32_t* n_matched,
                         int32_t* dev_status, void* stream);

/*
 * kld_sparse_ref_score - the challenge score: a candidate's full logits
 * against a sparse reference, KL over K + 1 cells.
 *
 * Defines ("Qwen3.8-27B Quantization Challenge", "Golden distributions" for
 * the reference layout, "The score" for the KL): per position, with
 * reference entries (R_j, a_j), j < k, the k most likely ids and their f32
 * log-probs (most likely first), reference tail mass p_tail (the mass of
 * every unlisted id), and candidate logits y over the whole vocabulary,
 *    q        = softmax(y) over all vocab ids
 *    q_tail   = sum of q over the ids not in R      (the tail cell)
 *    p_j      = exp(a_j)
 *    kl       = sum_j p_j (a_j - log q_{R_j})
 *             + [p_tail > 0] p_tail (log p_tail - log max(q_tail, 1e-12))
 *    top1     = (R_0 == cand_argmax)
 * cand_argmax is the lowest index of the candidate's maximum.  q_tail is
 * summed over the unlisted ids directly (the listed ids are masked out of
 * the streaming pass), never formed as 1 - sum_R q, so it stays accurate
 * when the listed ids hold all but a millionth of the mass.
 *
 * Arguments:
 *   cand_logits      DEVICE [n_rows, ld_cand] f32 or bf16, 16-byte aligned;
 *                    ld_cand * element size a multiple of 16.
 *   ref_top          DEVICE kld_top_entry [n_rows, k] (row stride k), 8-byte aligned.
 *   k                1 .. KLD_SPARSE_MAX_K and k <= vocab; vocab <= 2^22.
 *   ref_rows         DEVICE f32 [n_rows, 3] per row (NLL of the true next
 *                    token, entropy, tail mass), or NULL: p_tail is then
 *                    1 - sum_j p_j (in f64).
 *   target_ids       DEVICE int32 [n_rows], required when cand_target_lp is given.
 *   kl               DEVICE f32 [n_rows], required.
 *   cand_argmax      DEVICE int32 [n_rows], or NULL.
 *   top1             DEVICE uint8 [n_rows] (0/1), or NULL.
 *   cand_target_lp   DEVICE f32 [n_rows]: log q of the target, or NULL.
 *   ref_target_lp    DEVICE f32 [n_rows]: -NLL copied from ref_rows (so the
 *                    reductions can form the perplexity ratio), or NULL;
 *                    requires ref_rows.
 *   workspace        DEVICE, >= kld_sparse_ref_workspace_size(n_rows, k)
 *                    bytes, 256-byte aligned; holds nothing between calls.
 * A candidate row holding NaN or +inf, or no finite logit, gives kl NaN,
 * cand_argmax -1, top1 0 and NaN target log-prob.  A listed id outside
 * [0, vocab), or repeated within a row, gives kl NaN and sets
 * KLD_DEV_BAD_ID; a target outside [0, vocab) gives a NaN target log-prob
 * and sets KLD_DEV_BAD_TARGET.
 * Range: differences z_i - max(z) of the candidate's logits are formed in
 * f32, so finite logits of any magnitude are scored as long as those stay
 * within the f32 range (always so when every |logit| <= 1.7e38).
 */
#define KLD_SPARSE_MAX_K 1024
typedef struct {
  int32_t id;
  float lp;
} kld_top_entry;

size_t kld_sparse_ref_workspace_size(int64_t n_rows, int32_t k);
kld_status kld_sparse_ref_score(const void* cand_logits, kld_dtype dtype, int64_t n_rows, int64_t vocab,
                                int64_t ld_cand, const kld_top_entry* ref_top, int32_t k,
                                const float* ref_rows, const int32_t* target_ids, float* kl,
                                int32_t* cand_argmax, uint8_t* top1, float* cand_target_lp,
                                float* ref_target_lp, void* workspace, size_t workspace_bytes,
                                int32_t* dev_status, void* stream);

/*
 * kld_sparse_capture - the sparse record of a reference distribution, from
 * its full logits: the producer of kld_sparse_ref_score's reference.
 *
 * Defines ("Qwen3.8-27B Quantization Challenge", "Golden distributions"): per
 * row, with lp = log-softmax of the logits over all vocab ids and p = exp(lp),
 *    top[j], j < k   the k ids of largest lp with their lp (f32), most
 *                    likely first; equal lp keep the lower id first
 *    rows[0]         -lp[target], the NLL of the true next token
 *    rows[1]         -sum_i p_i lp_i, the entropy in nats
 *    rows[2]         sum of p_i over the ids not in top, summed over those
 *                    ids (never formed as 1 - sum of the listed masses)
 *
 * Arguments:
 *   logits       DEVICE [n_rows, ld] f32 or bf16, 16-byte aligned; ld * element
 *                size a multiple of 16.
 *   k            1 .. KLD_SPARSE_MAX_K and k <= vocab; vocab <= 2^22.
 *   target_ids   DEVICE int32 [n_rows], or NULL (rows[0] is then NaN).
 *   top          DEVICE kld_top_entry [n_rows, k], 8-byte aligned (output).
 *   rows         DEVICE f32 [n_rows, 3], 4-byte aligned (output).
 *   workspace    DEVICE, >= kld_sparse_capture_workspace_size(n_rows, k)
 *                bytes, 256-byte aligned; holds nothing between calls.
 * A row holding NaN or +inf, or no finite logit, gives ids -1 and NaN lp and
 * rows.  A target outside [0, vocab) gives NaN NLL and sets
 * KLD_DEV_BAD_TARGET.  Up to KLD_CAPTURE_CANDIDATES ids per row are kept as
 * candidates in one streaming pass; a row that needs more (many equal
 * logits, or its largest logits missed by the threshold sample) is redone
 * exactly from its logits, which is slower but gives the same result.
 */
#define KLD_CAPTURE_CANDIDATES 8192
size_t kld_sparse_capture_workspace_size(int64_t n_rows, int32_t k);
kld_status kld_sparse_capture(const void* logits, kld_dtype dtype, int64_t n_rows, int64_t vocab, int64_t ld,
                              int32_t k, const int32_t* target_ids, kld_top_entry* top, float* rows,
                              void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * kld_from_hidden_shared_head - full-vocabulary scoring from final hidden
 * states pushed through one shared LM head.
 *
 * Defines ("Qwen3.8-27B fidelity suite v5", opening paragraph: KLD from final
 * hidden states through one shared BF16 LM head, so no candidate is credited
 * or penalised for its own head): with x = W h_ref[r] and y = W h_cand[r]
 * (logits accumulated in f32 on the tensor cores, never rounded to bf16 and
 * never written to memory), the outputs are those of kld_full_vocab on x, y.
 *
 * Arguments:
 *   h_ref, h_cand   bf16 [n_rows, hidden] row-major, 16-byte aligned.
 *   head_w          bf16 [vocab, hidden] row-major, 16-byte aligned.
 *   hidden          8 .. 2^20, a multiple of 8.   vocab: 1 .. 2^31 - 1.
 *   target_ids .. cand_target_lp, dev_status: as in kld_full_vocab.
 *   workspace       >= kld_shared_head_workspace_size(n_rows, hidden, vocab)
 *                   bytes, 256-byte aligned (per 256-id vocabulary tile and
 *                   row, 32 bytes of partial state).
 * A bounded wait inside the kernel that gives up (after about 2 s) sets
 * KLD_DEV_TIMEOUT; the outputs are then invalid.
 */
size_t kld_shared_head_workspace_size(int64_t n_rows, int64_t hidden, int64_t vocab);
kld_status kld_from_hidden_shared_head(const void* h_ref, const void* h_cand, const void* head_w,
                                       int64_t n_rows, int64_t hidden, int64_t vocab,
                                       const int32_t* target_ids, float* kl, int32_t* ref_argmax,
                                       int32_t* cand_argmax, float* ref_target_lp,
                                       float* cand_target_lp, void* workspace, size_t workspace_bytes,
                                       int32_t* dev_status, void* stream);

/*
 * Result of kld_reduce_stats, written to DEVICE memory.  Plain C layout:
 * 8-byte fields first, then 4-byte fields; sizeof = 280 on LP64.
 */
#define KLD_MAX_QUANTILES 8
#define KLD_MAX_THRESHOLDS 8
typedef struct kld_stats {
  int64_t n;                 /* positions scored: mask set and kl not NaN */
  int64_t n_nan;             /* masked-in positions whose kl is NaN (excluded) */
  int64_t top1_agree;        /* agreeing scored positions, -1 if no agreement input */
  int64_t exceed[KLD_MAX_THRESHOLDS]; /* count of scored kl > thresholds[i] (f32 compare) */
  double mean_kl;            /* sum of scored kl / n (NaN if n == 0) */
  double top1_rate;          /* top1_agree / n (NaN if unavailable) */
  double ref_mean_nll, cand_mean_nll; /* mean of -target lp over scored positions (NaN if absent) */
  double ref_ppl, cand_ppl;  /* exp(mean NLL) */
  double ppl_ratio;          /* cand_ppl / ref_ppl */
  double q_value[KLD_MAX_QUANTILES]; /* linear-interpolated percentile of scored kl */
  float q_lo[KLD_MAX_QUANTILES];     /* order statistic s[floor((n-1) q)] */
  float q_hi[KLD_MAX_QUANTILES];     /* order statistic s[min(floor((n-1) q) + 1, n - 1)] */
  int32_t nq, nt;            /* echo of the counts requested */
} kld_stats;

/* Workspace bytes kld_reduce_stats needs for n positions. */
size_t kld_reduce_workspace_size(int64_t n);

/*
 * kld_reduce_stats - leaderboard reductions over per-position results.
 *
 * Defines ("Qwen3.8-27B Quantization Challenge", "The score": mean KL
 * ranks, median / p99 / p99.9, top-1 agreement, perplexity ratio;
 * "Qwen3.8-27B fidelity suite v5", "What is in here": percentiles and exact
 * exceedance counts; "Qwopus3.8-27B-Coder-Flash: quality-eval reference",
 * "Method": perplexity = exp(mean NLL)).  Scored positions are those with
 * mask[i] != 0 (all when mask is NULL) and kl[i] not NaN.  Percentile q uses
 * linear interpolation, h = (n - 1) q:
 *    q_value = s[lo] + (s[hi] - s[lo]) (h - lo),  lo = floor h, hi = min(lo + 1, n - 1)
 * over the ascending scored kl values s; both order statistics are exact
 * (radix select on the f32 bit patterns).  Sums are f64 in a fixed order.
 *
 * Arguments:
 *   kl                         f32 [n], required.
 *   ref_argmax, cand_argmax    int32 [n]: agreement = (ref == cand && ref >= 0);
 *                              both or neither.
 *   top1                       uint8 [n] agreement flags; used when the argmax
 *                              pair is NULL.  All three NULL: top1_agree = -1.
 *   ref_target_lp, cand_target_lp  f32 [n] each, may be NULL.
 *   mask                       uint8 [n] or NULL.
 *   n                          0 .. 2^31 - 1.
 *   quantiles                  HOST double[nq], each in [0, 1]; nq 0 .. 8.
 *   thresholds                 HOST float[nt]; nt 0 .. 8.
 *   out                        DEVICE kld_stats*, 8-byte aligned.
 *   workspace                  DEVICE, >= kld_reduce_workspace_size(n) bytes, 256-byte aligned.
 */
kld_status kld_reduce_stats(const float* kl, const int32_t* ref_argmax, const int32_t* cand_argmax,
                            const uint8_t* top1, const float* ref_target_lp,
                            const float* cand_target_lp, const uint8_t* mask, int64_t n,
                            const double* quantiles, int32_t nq, const float* thresholds,
                            int32_t nt, kld_stats* out, void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, void* stream);

/*
 * kld_reduce_shard_step - the statistics of kld_reduce_stats over the
 * positions of several shards (ranks, or chunks scored apart), exchanging
 * only a fixed-size block per shard and step.
 *
 * Defines the same quantities as kld_reduce_stats over the union of every
 * shard's positions (the per-shard tail reports of "Qwen3.8-27B fidelity
 * suite v5", "What is in here", are percentiles and exact exceedance counts
 * over two shards' positions).  Order statistics and counts are exact; each
 * shard sums its own positions in a fixed order and the shards' sums are
 * added in shard order, so every shard gets identical statistics.
 *
 * Protocol: every shard calls steps 0 .. KLD_SHARD_STEPS - 1 in order, with
 * its own arrays and workspace and the same n_shards, quantiles and
 * thresholds.  Steps 0 .. KLD_SHARD_STEPS - 2 write this shard's block
 * (kld_reduce_shard_block_bytes() bytes) to block_out.  Before step s + 1
 * the caller gathers the step-s blocks of all shards, in shard order, into
 * `gathered` (n_shards blocks back to back), e.g. with an all-gather.  The
 * last step writes the statistics to `out`.
 *
 * Arguments: as kld_reduce_stats, plus
 *   step         0 .. KLD_SHARD_STEPS - 1.
 *   n_shards     1 .. 65536.
 *   gathered     DEVICE, the previous step's blocks; required for step > 0; 16-byte aligned.
 *   block_out    DEVICE, kld_reduce_shard_block_bytes(); required before the last step; 16-byte aligned.
 *   out          DEVICE kld_stats; required at the last step only.
 *   workspace    DEVICE, >= kld_reduce_shard_workspace_size(n) bytes, 256-byte
 *                aligned; carries the shard's state from step to step.
 * Which inputs are given (non-NULL) must be the same on every shard: a shard
 * with n = 0 passes any non-NULL pointer for an input the others give (it is
 * never read).
 */
#define KLD_SHARD_STEPS 5
size_t kld_reduce_shard_block_bytes(void);
size_t kld_reduce_shard_workspace_size(int64_t n);
kld_status kld_reduce_shard_step(int32_t step, int32_t n_shards, const void* gathered, void* block_out,
                                 const float* kl, const int32_t* ref_argmax, const int32_t* cand_argmax,
                                 const uint8_t* top1, const float* ref_target_lp, const float* cand_target_lp,
                                 const uint8_t* mask, int64_t n, const double* quantiles, int32_t nq,
                                 const float* thresholds, int32_t nt, kld_stats* out, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * Result of kld_paired_compare, written to DEVICE memory (plain C layout,
 * 8-byte fields first; sizeof = 144 on LP64).
 */
typedef struct kld_paired {
  int64_t n_ctx;    /* contexts with at least one counted position */
  int64_t n_pos;    /* counted positions over all contexts */
  int64_t a_lower;  /* counted contexts whose mean KL is lower for candidate A */
  int64_t b_lower;  /* ... lower for candidate B */
  int64_t ties;     /* ... equal */
  int64_t n_boot;   /* replicates whose draws hold a counted context */
  double mean_a;    /* mean over counted contexts of A's per-context mean KL */
  double mean_b;    /* the same for B */
  double diff;      /* mean over counted contexts of (A's - B's per-context mean) */
  double ci[KLD_MAX_QUANTILES]; /* bootstrap percentiles of diff, one per quantile */
  int32_t nq;
  int32_t pad;
} kld_paired;

/* Workspace bytes kld_paired_compare needs. */
size_t kld_paired_workspace_size(int64_t n_ctx, int32_t n_clusters, int32_t n_boot);

/*
 * kld_paired_compare - two candidates scored against one reference, paired
 * per context, with a source-cluster bootstrap interval.
 *
 * Defines ("Qwen3.8-27B fidelity suite v5": contexts grouped into source
 * clusters, "What is in here"; the paired comparison of two candidates with
 * a 95 % source-cluster bootstrap interval and per-context win / tie counts,
 * in the sibling-rebuild paragraph and the "compare against a published
 * candidate" step).  The page gives no formulas; this library reads them so:
 * a position counts when mask[i] != 0 (all when mask is NULL) and neither
 * KL is NaN; per counted context c, m_A(c) and m_B(c) are the means of its
 * counted positions and d_c = m_A(c) - m_B(c); diff is the mean of d_c over
 * counted contexts.  Bootstrap replicate r draws the clusters
 * resample[r * n_clusters + j], j < n_clusters, and its statistic is
 *     sum over draws of D[k]  /  sum over draws of N[k]
 * with D[k] the sum of d_c and N[k] the number of counted contexts of
 * cluster k (NaN, and left out, when the draws hold no counted context).
 * ci[i] is the linear-interpolation percentile (h = (n_boot - 1) q, as in
 * kld_reduce_stats) of the replicate statistics; both order statistics are
 * exact.  Sums are f64 in a fixed order, so results are reproducible.
 *
 * Arguments (pointers DEVICE unless noted):
 *   kl_a, kl_b     f32 [n_ctx, ctx_len], context-major, per-position KL of
 *                  candidates A and B against the same reference; 16-byte aligned.
 *   mask           u8 [n_ctx, ctx_len] or NULL.
 *   n_ctx          >= 0 contexts; ctx_len >= 1 positions each (n_ctx * ctx_len < 2^40).
 *   cluster        int32 [n_ctx], each context's cluster in [0, n_clusters);
 *                  out-of-range ids set KLD_DEV_BAD_ID and drop the context.
 *   n_clusters     >= 1.
 *   resample       int32 [n_boot, n_clusters], the draws (the caller's random
 *                  numbers); out-of-range draws set KLD_DEV_BAD_ID and are skipped.
 *                  May be NULL when n_boot == 0.
 *   n_boot         >= 0 replicates; n_boot * n_clusters < 2^31.
 *   quantiles      HOST double [nq] in [0, 1]; nq <= KLD_MAX_QUANTILES.
 *   out            DEVICE kld_paired, 8-byte aligned.
 *   boot_stats     DEVICE double [n_boot] for the replicate statistics, or NULL.
 *   workspace      DEVICE, >= kld_paired_workspace_size(...) bytes, 256-byte aligned.
 *   dev_status     DEVICE int32 or NULL: KLD_DEV_BAD_ID bits are OR-ed in.
 *   stream         cudaStream_t or NULL.
 * Ownership: the caller owns every buffer; nothing is kept after the call.
 * Errors: KLD_ERR_INVALID_ARG for sizes or quantiles out of range or a
 * missing pointer, KLD_ERR_ALIGNMENT, KLD_ERR_WORKSPACE, KLD_ERR_CUDA.
 */
kld_status kld_paired_compare(const float* kl_a, const float* kl_b, const uint8_t* mask, int64_t n_ctx,
                              int32_t ctx_len, const int32_t* cluster, int32_t n_clusters,
                              const int32_t* resample, int32_t n_boot, const double* quantiles, int32_t nq,
                              kld_paired* out, double* boot_stats, void* workspace, size_t workspace_bytes,
                              int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KLD_H_ */
