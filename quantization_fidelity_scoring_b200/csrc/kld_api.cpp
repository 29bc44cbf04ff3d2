// C ABI of libkld: argument validation and kernel launch (see include/kld.h).
//
// Every check that can be made on the host is made here, before any CUDA
// call, so that a rejected call launches nothing and needs no device.
#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "../../include/kld.h"
#include "launch.h"

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline kld_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KLD_OK : KLD_ERR_CUDA; }

}  // namespace

extern "C" {

int kld_version(void) { return 100; }

const char* kld_status_string(kld_status s) {
  switch (s) {
    case KLD_OK: return "ok";
    case KLD_ERR_INVALID_ARG: return "invalid argument";
    case KLD_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case KLD_ERR_UNSUPPORTED: return "unsupported dtype or size";
    case KLD_ERR_WORKSPACE: return "workspace missing or too small";
    case KLD_ERR_CUDA: return "CUDA launch or runtime error";
  }
  return "unknown status";
}

static kld_status full_vocab_impl(const void* ref_logits, const void* cand_logits, kld_dtype dtype,
                                  int64_t n_rows, int64_t vocab, int64_t ld_ref, int64_t ld_cand,
                                  const int32_t* target_ids, float* kl, int32_t* ref_argmax,
                                  int32_t* cand_argmax, float* ref_target_lp, float* cand_target_lp,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                  void* stream, int warps) {
  if (dtype != KLD_F32 && dtype != KLD_BF16) return KLD_ERR_UNSUPPORTED;
  if (n_rows < 0 || vocab < 1 || vocab > INT32_MAX) return KLD_ERR_INVALID_ARG;
  if (ld_ref < vocab || ld_cand < vocab) return KLD_ERR_INVALID_ARG;
  if (!target_ids && (ref_target_lp || cand_target_lp)) return KLD_ERR_INVALID_ARG;
  if (warps < 0) return KLD_ERR_INVALID_ARG;
  if (n_rows == 0) return KLD_OK;
  if (!ref_logits || !cand_logits || !kl) return KLD_ERR_INVALID_ARG;
  if (n_rows > (int64_t)INT32_MAX - kld::kFullVocabMaxWarps) return KLD_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < kld::full_vocab_workspace_bytes(n_rows)) return KLD_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return KLD_ERR_ALIGNMENT;
  const int64_t esize = dtype == KLD_BF16 ? 2 : 4;
  if (!aligned(ref_logits, 16) || !aligned(cand_logits, 16)) return KLD_ERR_ALIGNMENT;
  if ((ld_ref * esize) % 16 != 0 || (ld_cand * esize) % 16 != 0) return KLD_ERR_ALIGNMENT;
  if (!aligned(kl, 4) || !aligned(ref_argmax, 4) || !aligned(cand_argmax, 4) ||
      !aligned(ref_target_lp, 4) || !aligned(cand_target_lp, 4) || !aligned(target_ids, 4) ||
      !aligned(dev_status, 4))
    return KLD_ERR_ALIGNMENT;

  kld::FullVocabArgs a;
  a.x = ref_logits;
  a.y = cand_logits;
  a.bf16 = dtype == KLD_BF16;
  a.n_rows = n_rows;
  a.vocab = vocab;
  a.ld_x = ld_ref;
  a.ld_y = ld_cand;
  a.targets = target_ids;
  a.kl = kl;
  a.ax = ref_argmax;
  a.ay = cand_argmax;
  a.lpx = ref_target_lp;
  a.lpy = cand_target_lp;
  a.dev_status = dev_status;
  a.workspace = workspace;
  a.warps_override = warps;
  return cuda_status(kld::launch_full_vocab(a, static_cast<cudaStream_t>(stream)));
}

size_t kld_full_vocab_workspace_size(int64_t n_rows) {
  return n_rows < 0 ? 0 : kld::full_vocab_workspace_bytes(n_rows);
}

kld_status kld_full_vocab(const void* ref_logits, const void* cand_logits, kld_dtype dtype,
                          int64_t n_rows, int64_t vocab, int64_t ld_ref, int64_t ld_cand,
                          const int32_t* target_ids, float* kl, int32_t* ref_argmax,
                          int32_t* cand_argmax, float* ref_target_lp, float* cand_target_lp,
                          void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  return full_vocab_impl(ref_logits, cand_logits, dtype, n_rows, vocab, ld_ref, ld_cand, target_ids, kl,
                         ref_argmax, cand_argmax, ref_target_lp, cand_target_lp, workspace, workspace_bytes,
                         dev_status, stream, 0);
}

// kld_full_vocab for callers that cannot allocate: the scratch is the
// library's own device array (see kld.h).  Too many rows is refused before
// any CUDA call; every other argument is checked by kld_full_vocab.
kld_status kld_full_vocab_noalloc(const void* ref_logits, const void* cand_logits, kld_dtype dtype,
                                  int64_t n_rows, int64_t vocab, int64_t ld_ref, int64_t ld_cand,
                                  const int32_t* target_ids, float* kl, int32_t* ref_argmax,
                                  int32_t* cand_argmax, float* ref_target_lp, float* cand_target_lp,
                                  int32_t* dev_status, void* stream) {
  if (n_rows > kld::kNoAllocMaxRows) return KLD_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (n_rows > 0 && kld::noalloc_scratch(&scratch, &scratch_bytes) != cudaSuccess) return KLD_ERR_CUDA;
  return kld_full_vocab(ref_logits, cand_logits, dtype, n_rows, vocab, ld_ref, ld_cand, target_ids, kl,
                        ref_argmax, cand_argmax, ref_target_lp, cand_target_lp, scratch, scratch_bytes,
                        dev_status, stream);
}

// kld_full_vocab with the number of streaming warps forced (0 = automatic),
// to test how pieces of rows merge.  Exported for tests; not in kld.h.
kld_status kld_full_vocab_split(const void* ref_logits, const void* cand_logits, kld_dtype dtype,
                                int64_t n_rows, int64_t vocab, int64_t ld_ref, int64_t ld_cand,
                                const int32_t* target_ids, float* kl, int32_t* ref_argmax,
                                int32_t* cand_argmax, float* ref_target_lp, float* cand_target_lp,
                                void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream,
                                int32_t warps) {
  return full_vocab_impl(ref_logits, cand_logits, dtype, n_rows, vocab, ld_ref, ld_cand, target_ids, kl,
                         ref_argmax, cand_argmax, ref_target_lp, cand_target_lp, workspace, workspace_bytes,
                         dev_status, stream, warps);
}

kld_status kld_topk_tail(const int32_t* ref_ids, const uint16_t* ref_lp, const int32_t* cand_ids,
                         const uint16_t* cand_lp, int64_t n_rows, int32_t k, int64_t vocab, float* kl,
                         uint8_t* top1, int32_t* n_matched, int32_t* dev_status, void* stream) {
  if (n_rows < 0 || k < 1 || k > 64 || vocab <= k || vocab >= (int64_t(1) << 25))
    return KLD_ERR_INVALID_ARG;
  if (n_rows == 0) return KLD_OK;
  if (!ref_ids || !ref_lp || !cand_ids || !cand_lp || !kl) return KLD_ERR_INVALID_ARG;
  if (n_rows > (int64_t(1) << 40)) return KLD_ERR_UNSUPPORTED;
  if (!aligned(ref_ids, 4) || !aligned(cand_ids, 4) || !aligned(ref_lp, 2) || !aligned(cand_lp, 2) ||
      !aligned(kl, 4) || !aligned(n_matched, 4) || !aligned(dev_status, 4))
    return KLD_ERR_ALIGNMENT;
  kld::TopkTailArgs a;
  a.ref_ids = ref_ids;
  a.ref_lp = ref_lp;
  a.cand_ids = cand_ids;
  a.cand_lp = cand_lp;
  a.n_rows = n_rows;
  a.k = k;
  a.vocab = vocab;
  a.kl = kl;
  a.top1 = top1;
  a.n_matched = n_matched;
  a.dev_status = dev_status;
  return cuda_status(kld::launch_topk_tail(a, static_cast<cudaStream_t>(stream)));
}

size_t kld_sparse_ref_workspace_size(int64_t n_rows, int32_t k) {
  if (n_rows < 0 || k < 1 || k > KLD_SPARSE_MAX_K) return 0;
  return kld::sparse_ref_workspace_bytes(n_rows, k);
}

static kld_status sparse_ref_impl(const void* cand_logits, kld_dtype dtype, int64_t n_rows, int64_t vocab,
                                  int64_t ld_cand, const kld_top_entry* ref_top, int32_t k,
                                  const float* ref_rows, const int32_t* target_ids, float* kl,
                                  int32_t* cand_argmax, uint8_t* top1, float* cand_target_lp,
                                  float* ref_target_lp, void* workspace, size_t workspace_bytes,
                                  int32_t* dev_status, void* stream, int warps) {
  if (warps < 0) return KLD_ERR_INVALID_ARG;
  if (dtype != KLD_F32 && dtype != KLD_BF16) return KLD_ERR_UNSUPPORTED;
  if (n_rows < 0 || vocab < 1 || ld_cand < vocab || k < 1 || k > KLD_SPARSE_MAX_K || k > vocab)
    return KLD_ERR_INVALID_ARG;
  if (vocab > (int64_t(1) << 22)) return KLD_ERR_UNSUPPORTED;
  if (!target_ids && cand_target_lp) return KLD_ERR_INVALID_ARG;
  if (!ref_rows && ref_target_lp) return KLD_ERR_INVALID_ARG;
  if (n_rows == 0) return KLD_OK;
  if (!cand_logits || !ref_top || !kl) return KLD_ERR_INVALID_ARG;
  if (n_rows > (int64_t)INT32_MAX - kld::kSparseMaxWarps) return KLD_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < kld::sparse_ref_workspace_bytes(n_rows, k)) return KLD_ERR_WORKSPACE;
  const int64_t esize = dtype == KLD_BF16 ? 2 : 4;
  if (!aligned(workspace, 256) || !aligned(cand_logits, 16) || (ld_cand * esize) % 16 != 0)
    return KLD_ERR_ALIGNMENT;
  if (!aligned(ref_top, 8) || !aligned(ref_rows, 4) || !aligned(target_ids, 4) || !aligned(kl, 4) ||
      !aligned(cand_argmax, 4) || !aligned(cand_target_lp, 4) || !aligned(ref_target_lp, 4) ||
      !aligned(dev_status, 4))
    return KLD_ERR_ALIGNMENT;
  kld::SparseRefArgs a;
  a.y = cand_logits;
  a.bf16 = dtype == KLD_BF16;
  a.n_rows = n_rows;
  a.vocab = vocab;
  a.ld = ld_cand;
  a.ref_top = ref_top;
  a.k = k;
  a.ref_rows = ref_rows;
  a.targets = target_ids;
  a.kl = kl;
  a.argmax = cand_argmax;
  a.top1 = top1;
  a.lp_cand = cand_target_lp;
  a.lp_ref = ref_target_lp;
  a.workspace = workspace;
  a.dev_status = dev_status;
  a.warps_override = warps;
  return cuda_status(kld::launch_sparse_ref(a, static_cast<cudaStream_t>(stream)));
}

kld_status kld_sparse_ref_score(const void* cand_logits, kld_dtype dtype, int64_t n_rows, int64_t vocab,
                                int64_t ld_cand, const kld_top_entry* ref_top, int32_t k,
                                const float* ref_rows, const int32_t* target_ids, float* kl,
                                int32_t* cand_argmax, uint8_t* top1, float* cand_target_lp,
                                float* ref_target_lp, void* workspace, size_t workspace_bytes,
                                int32_t* dev_status, void* stream) {
  return sparse_ref_impl(cand_logits, dtype, n_rows, vocab, ld_cand, ref_top, k, ref_rows, target_ids, kl,
                         cand_argmax, top1, cand_target_lp, ref_target_lp, workspace, workspace_bytes,
                         dev_status, stream, 0);
}

// kld_sparse_ref_score with the number of streaming warps forced (0 =
// automatic), to test long pieces and many-piece merges.  Exported for
// tests; not in kld.h.
kld_status kld_sparse_ref_score_split(const void* cand_logits, kld_dtype dtype, int64_t n_rows, int64_t vocab,
                                      int64_t ld_cand, const kld_top_entry* ref_top, int32_t k,
                                      const float* ref_rows, const int32_t* target_ids, float* kl,
                                      int32_t* cand_argmax, uint8_t* top1, float* cand_target_lp,
                                      float* ref_target_lp, void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, void* stream, int32_t warps) {
  return sparse_ref_impl(cand_logits, dtype, n_rows, vocab, ld_cand, ref_top, k, ref_rows, target_ids, kl,
                         cand_argmax, top1, cand_target_lp, ref_target_lp, workspace, workspace_bytes,
                         dev_status, stream, warps);
}

size_t kld_sparse_capture_workspace_size(int64_t n_rows, int32_t k) {
  if (n_rows < 0 || k < 1 || k > KLD_SPARSE_MAX_K) return 0;
  return kld::sparse_capture_workspace_bytes(n_rows);
}

static kld_status sparse_capture_impl(const void* logits, kld_dtype dtype, int64_t n_rows, int64_t vocab,
                                      int64_t ld, int32_t k, const int32_t* target_ids, kld_top_entry* top,
                                      float* rows, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                      void* stream, int force_exact) {
  if (dtype != KLD_F32 && dtype != KLD_BF16) return KLD_ERR_UNSUPPORTED;
  if (n_rows < 0 || vocab < 1 || ld < vocab || k < 1 || k > KLD_SPARSE_MAX_K || k > vocab)
    return KLD_ERR_INVALID_ARG;
  if (vocab > (int64_t(1) << 22)) return KLD_ERR_UNSUPPORTED;
  if (n_rows == 0) return KLD_OK;
  if (!logits || !top || !rows) return KLD_ERR_INVALID_ARG;
  if (n_rows > (int64_t)INT32_MAX - kld::kSparseMaxWarps) return KLD_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < kld::sparse_capture_workspace_bytes(n_rows)) return KLD_ERR_WORKSPACE;
  const int64_t esize = dtype == KLD_BF16 ? 2 : 4;
  if (!aligned(workspace, 256) || !aligned(logits, 16) || (ld * esize) % 16 != 0) return KLD_ERR_ALIGNMENT;
  if (!aligned(top, 8) || !aligned(rows, 4) || !aligned(target_ids, 4) || !aligned(dev_status, 4))
    return KLD_ERR_ALIGNMENT;
  kld::SparseCaptureArgs a;
  a.x = logits;
  a.bf16 = dtype == KLD_BF16;
  a.n_rows = n_rows;
  a.vocab = vocab;
  a.ld = ld;
  a.k = k;
  a.targets = target_ids;
  a.top = top;
  a.rows = rows;
  a.workspace = workspace;
  a.dev_status = dev_status;
  a.force_exact = force_exact;
  return cuda_status(kld::launch_sparse_capture(a, static_cast<cudaStream_t>(stream)));
}

kld_status kld_sparse_capture(const void* logits, kld_dtype dtype, int64_t n_rows, int64_t vocab, int64_t ld,
                              int32_t k, const int32_t* target_ids, kld_top_entry* top, float* rows,
                              void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  return sparse_capture_impl(logits, dtype, n_rows, vocab, ld, k, target_ids, top, rows, workspace,
                             workspace_bytes, dev_status, stream, 0);
}

// kld_sparse_capture with every row on the exact path (the one a row takes
// when its candidates do not fit or fall short).  Exported for tests; not in
// kld.h.
kld_status kld_sparse_capture_exact(const void* logits, kld_dtype dtype, int64_t n_rows, int64_t vocab, int64_t ld,
                                    int32_t k, const int32_t* target_ids, kld_top_entry* top, float* rows,
                                    void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  return sparse_capture_impl(logits, dtype, n_rows, vocab, ld, k, target_ids, top, rows, workspace,
                             workspace_bytes, dev_status, stream, 1);
}

static kld_status shared_head_impl(const void* h_ref, const void* h_cand, const void* head_w, int64_t n_rows,
                                   int64_t hidden, int64_t vocab, const int32_t* target_ids, float* kl,
                                   int32_t* ref_argmax, int32_t* cand_argmax, float* ref_target_lp,
                                   float* cand_target_lp, void* workspace, size_t workspace_bytes,
                                   int32_t* dev_status, void* stream, int withhold) {
  if (n_rows < 0 || vocab < 1 || vocab > INT32_MAX || hidden < 8 || hidden > (1 << 20) || hidden % 8 != 0)
    return KLD_ERR_INVALID_ARG;
  if (!target_ids && (ref_target_lp || cand_target_lp)) return KLD_ERR_INVALID_ARG;
  if (n_rows == 0) return KLD_OK;
  if (n_rows > INT32_MAX / 2) return KLD_ERR_UNSUPPORTED;
  if (!h_ref || !h_cand || !head_w || !kl) return KLD_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < kld::shared_head_workspace_bytes(n_rows, vocab)) return KLD_ERR_WORKSPACE;
  if (!aligned(h_ref, 16) || !aligned(h_cand, 16) || !aligned(head_w, 16) || !aligned(workspace, 256))
    return KLD_ERR_ALIGNMENT;
  if (!aligned(kl, 4) || !aligned(ref_argmax, 4) || !aligned(cand_argmax, 4) || !aligned(ref_target_lp, 4) ||
      !aligned(cand_target_lp, 4) || !aligned(target_ids, 4) || !aligned(dev_status, 4))
    return KLD_ERR_ALIGNMENT;
  kld::SharedHeadArgs a;
  a.h_ref = h_ref;
  a.h_cand = h_cand;
  a.head_w = head_w;
  a.n_rows = n_rows;
  a.hidden = hidden;
  a.vocab = vocab;
  a.targets = target_ids;
  a.kl = kl;
  a.ax = ref_argmax;
  a.ay = cand_argmax;
  a.lpx = ref_target_lp;
  a.lpy = cand_target_lp;
  a.workspace = workspace;
  a.dev_status = dev_status;
  a.withhold = withhold;
  return cuda_status(kld::launch_shared_head(a, static_cast<cudaStream_t>(stream)));
}

size_t kld_shared_head_workspace_size(int64_t n_rows, int64_t hidden, int64_t vocab) {
  (void)hidden;
  if (n_rows < 0 || vocab < 1) return 0;
  return kld::shared_head_workspace_bytes(n_rows, vocab);
}

kld_status kld_from_hidden_shared_head(const void* h_ref, const void* h_cand, const void* head_w, int64_t n_rows,
                                       int64_t hidden, int64_t vocab, const int32_t* target_ids, float* kl,
                                       int32_t* ref_argmax, int32_t* cand_argmax, float* ref_target_lp,
                                       float* cand_target_lp, void* workspace, size_t workspace_bytes,
                                       int32_t* dev_status, void* stream) {
  return shared_head_impl(h_ref, h_cand, head_w, n_rows, hidden, vocab, target_ids, kl, ref_argmax, cand_argmax,
                          ref_target_lp, cand_target_lp, workspace, workspace_bytes, dev_status, stream, 0);
}

// Test hook, not in kld.h: withhold the first TMA fill so that the kernel's
// bounded waits run out and report KLD_DEV_TIMEOUT.
kld_status kld_from_hidden_shared_head_withhold(const void* h_ref, const void* h_cand, const void* head_w,
                                                int64_t n_rows, int64_t hidden, int64_t vocab, float* kl,
                                                void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                                void* stream) {
  return shared_head_impl(h_ref, h_cand, head_w, n_rows, hidden, vocab, nullptr, kl, nullptr, nullptr, nullptr,
                          nullptr, workspace, workspace_bytes, dev_status, stream, 1);
}

size_t kld_reduce_workspace_size(int64_t n) { return kld::reduce_workspace_bytes(n); }

static kld_status reduce_impl(const float* kl, const int32_t* ref_argmax, const int32_t* cand_argmax,
                              const uint8_t* top1, const float* ref_target_lp, const float* cand_target_lp,
                              const uint8_t* mask, int64_t n, const double* quantiles, int32_t nq,
                              const float* thresholds, int32_t nt, kld_stats* out, void* workspace,
                              size_t workspace_bytes, int32_t* dev_status, void* stream, int withhold) {
  if (n < 0 || n > INT32_MAX) return KLD_ERR_INVALID_ARG;
  if (nq < 0 || nq > KLD_MAX_QUANTILES || nt < 0 || nt > KLD_MAX_THRESHOLDS) return KLD_ERR_INVALID_ARG;
  if ((nq > 0 && !quantiles) || (nt > 0 && !thresholds)) return KLD_ERR_INVALID_ARG;
  if ((ref_argmax == nullptr) != (cand_argmax == nullptr)) return KLD_ERR_INVALID_ARG;
  if (!out || (n > 0 && !kl)) return KLD_ERR_INVALID_ARG;
  for (int i = 0; i < nq; ++i)
    if (!(quantiles[i] >= 0.0 && quantiles[i] <= 1.0)) return KLD_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < kld::reduce_workspace_bytes(n)) return KLD_ERR_WORKSPACE;
  if (!aligned(out, 8) || !aligned(workspace, 256) || !aligned(kl, 4) || !aligned(ref_argmax, 4) ||
      !aligned(cand_argmax, 4) || !aligned(ref_target_lp, 4) || !aligned(cand_target_lp, 4) ||
      !aligned(dev_status, 4))
    return KLD_ERR_ALIGNMENT;
  kld::ReduceArgs a;
  std::memset(&a, 0, sizeof(a));
  a.kl = kl;
  a.ref_argmax = ref_argmax;
  a.cand_argmax = cand_argmax;
  a.top1 = top1;
  a.ref_lp = ref_target_lp;
  a.cand_lp = cand_target_lp;
  a.mask = mask;
  a.n = n;
  a.nq = nq;
  a.nt = nt;
  for (int i = 0; i < nq; ++i) a.quantiles[i] = quantiles[i];
  for (int i = 0; i < nt; ++i) a.thresholds[i] = thresholds[i];
  a.out = out;
  a.workspace = workspace;
  a.dev_status = dev_status;
  a.withhold = withhold;
  return cuda_status(kld::launch_reduce(a, static_cast<cudaStream_t>(stream)));
}

kld_status kld_reduce_stats(const float* kl, const int32_t* ref_argmax, const int32_t* cand_argmax,
                            const uint8_t* top1, const float* ref_target_lp,
                            const float* cand_target_lp, const uint8_t* mask, int64_t n,
                            const double* quantiles, int32_t nq, const float* thresholds, int32_t nt,
                            kld_stats* out, void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, void* stream) {
  return reduce_impl(kl, ref_argmax, cand_argmax, top1, ref_target_lp, cand_target_lp, mask, n, quantiles, nq,
                     thresholds, nt, out, workspace, workspace_bytes, dev_status, stream, 0);
}

// Test hook, not in kld.h: for more than 8192 positions (the cooperative
// grid), CTA 0 leaves before the first grid barrier, so the other CTAs'
// bounded waits run out and set KLD_DEV_TIMEOUT; the statistics are not
// written.
kld_status kld_reduce_stats_withhold(const float* kl, const int32_t* ref_argmax, const int32_t* cand_argmax,
                                     const uint8_t* top1, const float* ref_target_lp,
                                     const float* cand_target_lp, const uint8_t* mask, int64_t n,
                                     const double* quantiles, int32_t nq, const float* thresholds, int32_t nt,
                                     kld_stats* out, void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream) {
  return reduce_impl(kl, ref_argmax, cand_argmax, top1, ref_target_lp, cand_target_lp, mask, n, quantiles, nq,
                     thresholds, nt, out, workspace, workspace_bytes, dev_status, stream, 1);
}

size_t kld_reduce_shard_block_bytes(void) { return kld::reduce_shard_block_bytes(); }

size_t kld_reduce_shard_workspace_size(int64_t n) { return n < 0 ? 0 : kld::reduce_shard_workspace_bytes(n); }

kld_status kld_reduce_shard_step(int32_t step, int32_t n_shards, const void* gathered, void* block_out,
                                 const float* kl, const int32_t* ref_argmax, const int32_t* cand_argmax,
                                 const uint8_t* top1, const float* ref_target_lp, const float* cand_target_lp,
                                 const uint8_t* mask, int64_t n, const double* quantiles, int32_t nq,
                                 const float* thresholds, int32_t nt, kld_stats* out, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (step < 0 || step >= KLD_SHARD_STEPS || n_shards < 1 || n_shards > 65536) return KLD_ERR_INVALID_ARG;
  if (n < 0 || n > INT32_MAX) return KLD_ERR_INVALID_ARG;
  if (nq < 0 || nq > KLD_MAX_QUANTILES || nt < 0 || nt > KLD_MAX_THRESHOLDS) return KLD_ERR_INVALID_ARG;
  if ((nq > 0 && !quantiles) || (nt > 0 && !thresholds)) return KLD_ERR_INVALID_ARG;
  if ((ref_argmax == nullptr) != (cand_argmax == nullptr)) return KLD_ERR_INVALID_ARG;
  if (n > 0 && !kl) return KLD_ERR_INVALID_ARG;
  if (step > 0 && !gathered) return KLD_ERR_INVALID_ARG;
  if (step < KLD_SHARD_STEPS - 1 && !block_out) return KLD_ERR_INVALID_ARG;
  if (step == KLD_SHARD_STEPS - 1 && !out) return KLD_ERR_INVALID_ARG;
  for (int i = 0; i < nq; ++i)
    if (!(quantiles[i] >= 0.0 && quantiles[i] <= 1.0)) return KLD_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < kld::reduce_shard_workspace_bytes(n)) return KLD_ERR_WORKSPACE;
  if (!aligned(out, 8) || !aligned(workspace, 256) || !aligned(gathered, 16) || !aligned(block_out, 16) ||
      !aligned(kl, 4) || !aligned(ref_argmax, 4) || !aligned(cand_argmax, 4) || !aligned(ref_target_lp, 4) ||
      !aligned(cand_target_lp, 4) || !aligned(dev_status, 4))
    return KLD_ERR_ALIGNMENT;
  kld::ReduceArgs a;
  std::memset(&a, 0, sizeof(a));
  a.kl = kl;
  a.ref_argmax = ref_argmax;
  a.cand_argmax = cand_argmax;
  a.top1 = top1;
  a.ref_lp = ref_target_lp;
  a.cand_lp = cand_target_lp;
  a.mask = mask;
  a.n = n;
  a.nq = nq;
  a.nt = nt;
  for (int i = 0; i < nq; ++i) a.quantiles[i] = quantiles[i];
  for (int i = 0; i < nt; ++i) a.thresholds[i] = thresholds[i];
  a.out = out;
  a.workspace = workspace;
  a.dev_status = dev_status;
  return cuda_status(kld::launch_reduce_shard_step(a, step, n_shards, gathered, block_out,
                                                   static_cast<cudaStream_t>(stream)));
}

size_t kld_paired_workspace_size(int64_t n_ctx, int32_t n_clusters, int32_t n_boot) {
  return kld::paired_workspace_bytes(n_ctx, n_clusters, n_boot);
}

kld_status kld_paired_compare(const float* kl_a, const float* kl_b, const uint8_t* mask, int64_t n_ctx,
                              int32_t ctx_len, const int32_t* cluster, int32_t n_clusters,
                              const int32_t* resample, int32_t n_boot, const double* quantiles, int32_t nq,
                              kld_paired* out, double* boot_stats, void* workspace, size_t workspace_bytes,
                              int32_t* dev_status, void* stream) {
  if (n_ctx < 0 || ctx_len < 1 || n_clusters < 1 || n_boot < 0) return KLD_ERR_INVALID_ARG;
  if (n_ctx > ((int64_t)1 << 40) / ctx_len || n_ctx > INT32_MAX) return KLD_ERR_INVALID_ARG;
  if ((int64_t)n_boot * n_clusters >= ((int64_t)1 << 31)) return KLD_ERR_INVALID_ARG;
  if (nq < 0 || nq > KLD_MAX_QUANTILES || (nq > 0 && !quantiles)) return KLD_ERR_INVALID_ARG;
  for (int i = 0; i < nq; ++i)
    if (!(quantiles[i] >= 0.0 && quantiles[i] <= 1.0)) return KLD_ERR_INVALID_ARG;
  if (!out || (n_ctx > 0 && (!kl_a || !kl_b || !cluster)) || (n_boot > 0 && !resample)) return KLD_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < kld::paired_workspace_bytes(n_ctx, n_clusters, n_boot))
    return KLD_ERR_WORKSPACE;
  if (!aligned(workspace, 256) || !aligned(out, 8) || !aligned(boot_stats, 8) || !aligned(kl_a, 16) ||
      !aligned(kl_b, 16) || !aligned(cluster, 4) || !aligned(resample, 4) || !aligned(dev_status, 4))
    return KLD_ERR_ALIGNMENT;
  kld::PairedArgs a;
  std::memset(&a, 0, sizeof(a));
  a.kl_a = kl_a;
  a.kl_b = kl_b;
  a.mask = mask;
  a.n_ctx = n_ctx;
  a.ctx_len = ctx_len;
  a.cluster = cluster;
  a.n_clusters = n_clusters;
  a.resample = resample;
  a.n_boot = n_boot;
  a.nq = nq;
  for (int i = 0; i < nq; ++i) a.quantiles[i] = quantiles[i];
  a.out = out;
  a.boot_stats = boot_stats;
  a.workspace = workspace;
  a.dev_status = dev_status;
  return cuda_status(kld::launch_paired(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

static_assert(KLD_SHARD_STEPS == kld::kShardSteps, "shard step count");
static_assert(sizeof(kld_stats) == 280, "kld_stats layout changed: update the Python mirror");
static_assert(sizeof(kld_paired) == 144, "kld_paired layout changed: update the Python mirror");
