// Internal launcher interface between the C ABI (kld_api.cpp) and the
// kernels.  Arguments arrive here already validated.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kld.h"

namespace kld {

struct FullVocabArgs {
  const void* x;
  const void* y;
  bool bf16;
  int64_t n_rows, vocab, ld_x, ld_y;
  const int32_t* targets;
  float* kl;
  int32_t* ax;
  int32_t* ay;
  float* lpx;
  float* lpy;
  int32_t* dev_status;
  void* workspace;       // >= full_vocab_workspace_bytes(n_rows)
  int warps_override;    // 0: choose from the problem size
};
// Upper bound on the streaming warps (fixed, so results do not depend on the
// device): two CTAs of eight warps per SM on 148 SMs (each CTA holds its
// warps' 96 KB of load rings).
constexpr int kStreamCtasPerSm = 2;
constexpr int kFullVocabMaxWarps = 148 * kStreamCtasPerSm * 8;
// The sparse-reference and capture streams: at most three CTAs of eight
// persistent warps per SM of a 148-SM part (their row slots are row + warp).
constexpr int kSparseMaxWarps = 148 * 3 * 8;
size_t full_vocab_workspace_bytes(int64_t n_rows);
cudaError_t launch_full_vocab(const FullVocabArgs& a, cudaStream_t stream);
// Rows the library-owned scratch of kld_full_vocab_noalloc can hold.
constexpr int64_t kNoAllocMaxRows = KLD_NOALLOC_MAX_ROWS;
// Device address and size of that scratch on the current device (looked up
// on the first call per device).
cudaError_t noalloc_scratch(void** ptr, size_t* bytes);

struct TopkTailArgs {
  const int32_t* ref_ids;
  const uint16_t* ref_lp;
  const int32_t* cand_ids;
  const uint16_t* cand_lp;
  int64_t n_rows;
  int k;
  int64_t vocab;
  float* kl;
  uint8_t* top1;
  int32_t* n_matched;
  int32_t* dev_status;
};
cudaError_t launch_topk_tail(const TopkTailArgs& a, cudaStream_t stream);

struct SparseRefArgs {
  const void* y;          // candidate logits [n_rows, ld]
  bool bf16;
  int64_t n_rows, vocab, ld;
  const kld_top_entry* ref_top;  // [n_rows, k]
  int k;
  const float* ref_rows;  // [n_rows, 3] or null
  const int32_t* targets;
  float* kl;
  int32_t* argmax;
  uint8_t* top1;
  float* lp_cand;
  float* lp_ref;
  void* workspace;        // >= sparse_ref_workspace_bytes(n_rows, k)
  int32_t* dev_status;
  int warps_override;     // 0: choose from the problem size
};
size_t sparse_ref_workspace_bytes(int64_t n_rows, int k);
cudaError_t launch_sparse_ref(const SparseRefArgs& a, cudaStream_t stream);

struct SparseCaptureArgs {
  const void* x;           // reference logits [n_rows, ld]
  bool bf16;
  int64_t n_rows, vocab, ld;
  int k;
  const int32_t* targets;  // or null
  kld_top_entry* top;      // [n_rows, k]
  float* rows;             // [n_rows, 3]
  void* workspace;         // >= sparse_capture_workspace_bytes(n_rows)
  int32_t* dev_status;
  int force_exact;         // tests only: every row takes the exact path
};
size_t sparse_capture_workspace_bytes(int64_t n_rows);
cudaError_t launch_sparse_capture(const SparseCaptureArgs& a, cudaStream_t stream);

struct SharedHeadArgs {
  const void* h_ref;   // bf16 [n_rows, hidden]
  const void* h_cand;  // bf16 [n_rows, hidden]
  const void* head_w;  // bf16 [vocab, hidden]
  int64_t n_rows, hidden, vocab;
  const int32_t* targets;
  float* kl;
  int32_t* ax;
  int32_t* ay;
  float* lpx;
  float* lpy;
  void* workspace;     // >= shared_head_workspace_bytes(n_rows, vocab)
  int32_t* dev_status;
  int withhold;        // tests only (see shared_head.cu)
};
size_t shared_head_workspace_bytes(int64_t n_rows, int64_t vocab);
cudaError_t launch_shared_head(const SharedHeadArgs& a, cudaStream_t stream);

struct ReduceArgs {
  const float* kl;
  const int32_t* ref_argmax;
  const int32_t* cand_argmax;
  const uint8_t* top1;
  const float* ref_lp;
  const float* cand_lp;
  const uint8_t* mask;
  int64_t n;
  int nq, nt;
  double quantiles[KLD_MAX_QUANTILES];
  float thresholds[KLD_MAX_THRESHOLDS];
  kld_stats* out;
  void* workspace;
  int32_t* dev_status;
  int withhold;  // tests only (see reduce.cu)
};
size_t reduce_workspace_bytes(int64_t n);
cudaError_t launch_reduce(const ReduceArgs& a, cudaStream_t stream);
// Statistics over several shards' positions, one step of a shard (see
// kld_reduce_shard_step): steps 0 .. 3 add this shard's pass histogram (and
// at step 0 its sums) to block_out; steps 1 .. 4 first add up the gathered
// blocks of the previous step; step 4 writes the statistics.
size_t reduce_shard_block_bytes();
size_t reduce_shard_workspace_bytes(int64_t n);
constexpr int kShardSteps = 5;
cudaError_t launch_reduce_shard_step(const ReduceArgs& a, int step, int n_shards, const void* gathered,
                                     void* block_out, cudaStream_t stream);

struct PairedArgs {
  const float* kl_a;
  const float* kl_b;
  const uint8_t* mask;
  int64_t n_ctx;
  int ctx_len;
  const int32_t* cluster;
  int n_clusters;
  const int32_t* resample;
  int n_boot;
  int nq;
  double quantiles[KLD_MAX_QUANTILES];
  kld_paired* out;
  double* boot_stats;  // or null: replicate statistics kept in the workspace
  void* workspace;     // >= paired_workspace_bytes(n_ctx, n_clusters, n_boot)
  int32_t* dev_status;
};
size_t paired_workspace_bytes(int64_t n_ctx, int32_t n_clusters, int32_t n_boot);
cudaError_t launch_paired(const PairedArgs& a, cudaStream_t stream);

}  // namespace kld
