// Top-k + one tail bucket KL, a half-warp per position.
//
// "Qwopus3.8-27B-Coder-Flash: quality-eval reference", section "Method": the
// KL runs over the reference's top-64 ids plus one tail bucket; a reference id
// missing from the candidate's top-64 gets the candidate's leftover mass
// spread evenly over the ids outside the candidate's top-64; top-1 agreement
// is an exact argmax match (the first stored slot, lists being sorted per
// section "Files").
//
// Each 16-lane half of a warp scores one position, so one warp instruction
// advances two positions; lane l of a half holds list slots l, l+16, l+32,
// l+48 of both lists.  Matching: the candidate's ids go into a 128-slot
// open-addressed table in shared memory (key = id, value = first slot holding
// it; atomicMin keeps the first slot of a repeated id), then each reference
// id is looked up.  The table gives the same answer whatever order the lanes
// insert in, so the result is deterministic.  The three masses that feed
// 1 - sum (candidate list, reference list, matched candidate cells) are f64
// butterflies in fixed lane order; the KL terms are f32.
#include <cuda_fp16.h>
#include <math_constants.h>

#include "kld_common.cuh"
#include "launch.h"

namespace kld {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kHalves = 2 * kWarps;  // positions in flight per CTA
constexpr int kPer = 4;              // list slots per lane
constexpr int kSlots = 128;          // >= 2 * 64: probe chains stay short and always end
constexpr uint32_t kEmpty = 0xffffffffu;
constexpr double kQFloor = 1e-12;

__device__ __forceinline__ uint32_t slot_of(uint32_t id) { return (id * 0x9E3779B1u) >> 25; }

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// Butterfly sums inside a 16-lane half (offsets 8, 4, 2, 1 stay in the half).
__device__ __forceinline__ double half_sum(double v) {
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
__device__ __forceinline__ float half_sum(float v) {
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

struct TopkParams {
  const int32_t* ref_ids;
  const uint16_t* ref_lp;
  const int32_t* cand_ids;
  const uint16_t* cand_lp;
  int64_t n_rows;
  int k;
  int vocab;
  float* kl;
  uint8_t* top1;
  int32_t* n_matched;
  int32_t* dev_status;
};

__global__ void __launch_bounds__(kThreads) topk_tail_kernel(const TopkParams p) {
  __shared__ uint32_t table[kHalves][kSlots];
  __shared__ float cand_lp_s[kHalves][64];

  wait_prior_grid();
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15;                       // lane within the half
  const int half = (threadIdx.x >> 4);            // half index in the CTA
  const unsigned half_mask = (lane < 16) ? 0x0000ffffu : 0xffff0000u;
  const int k = p.k;
  const uint32_t V = (uint32_t)p.vocab;
  uint32_t* tab = table[half];
  float* clps = cand_lp_s[half];

  const int64_t n_pairs = (p.n_rows + 1) / 2;
  for (int64_t pair = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); pair < n_pairs;
       pair += (int64_t)gridDim.x * kWarps) {
    const int64_t pos = 2 * pair + (lane >> 4);
    const bool live = pos < p.n_rows;             // the odd tail position's second half idles
    const int64_t base = pos * k;

    int32_t r[kPer], c[kPer];
    float a[kPer], b[kPer];
    bool valid[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int j = hl + 16 * i;
      valid[i] = live && j < k;
      r[i] = valid[i] ? p.ref_ids[base + j] : 0;
      c[i] = valid[i] ? p.cand_ids[base + j] : 0;
      a[i] = valid[i] ? h2f(p.ref_lp[base + j]) : 0.f;
      b[i] = valid[i] ? h2f(p.cand_lp[base + j]) : 0.f;
    }
    bool bad_lane = false;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      bad_lane |= valid[i] && ((uint32_t)r[i] >= V || (uint32_t)c[i] >= V);
    const bool bad = (__ballot_sync(0xffffffffu, bad_lane) & half_mask) != 0;

    // clear this half's table, publish the candidate log-probs
#pragma unroll
    for (int s = hl; s < kSlots; s += 16) tab[s] = kEmpty;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (valid[i]) clps[hl + 16 * i] = b[i];
    __syncwarp();
    if (!bad) {
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (!valid[i]) continue;
        const uint32_t id = (uint32_t)c[i];
        const uint32_t entry = (id << 6) | (uint32_t)(hl + 16 * i);
        uint32_t s = slot_of(id);
        for (int probe = 0; probe < kSlots; ++probe) {
          const uint32_t old = atomicCAS(&tab[s], kEmpty, entry);
          if (old == kEmpty) break;
          if ((old >> 6) == id) {
            atomicMin(&tab[s], entry);
            break;
          }
          s = (s + 1) & (kSlots - 1);
        }
      }
    }
    __syncwarp();

    double c_sum = 0.0, p_sum = 0.0, qm_sum = 0.0;
    float klm = 0.f, pau = 0.f, pu = 0.f;
    int matched = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (!valid[i] || bad) continue;
      c_sum += (double)expf(b[i]);
      const uint32_t id = (uint32_t)r[i];
      int slot = -1;
      uint32_t s = slot_of(id);
      for (int probe = 0; probe < kSlots; ++probe) {
        const uint32_t e = tab[s];
        if (e == kEmpty) break;
        if ((e >> 6) == id) {
          slot = (int)(e & 63u);
          break;
        }
        s = (s + 1) & (kSlots - 1);
      }
      const float pj = expf(a[i]);
      p_sum += (double)pj;
      if (slot >= 0) {
        const float bm = clps[slot];
        qm_sum += (double)expf(bm);
        klm += pj * (a[i] - bm);
        ++matched;
      } else {
        pu += pj;
        pau += pj * a[i];
      }
    }
    c_sum = half_sum(c_sum);
    p_sum = half_sum(p_sum);
    qm_sum = half_sum(qm_sum);
    klm = half_sum(klm);
    pau = half_sum(pau);
    pu = half_sum(pu);
    int m_total = matched;
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) m_total += __shfl_xor_sync(0xffffffffu, m_total, off);

    if (hl == 0 && live) {
      float out;
      if (bad) {
        out = CUDART_NAN_F;
        set_dev_status(p.dev_status, 0x2 /* KLD_DEV_BAD_ID */);
      } else {
        const double leftover = fmax(1.0 - c_sum, 0.0);
        const double spread = leftover / (double)(p.vocab - k);
        const float log_spread = logf((float)fmax(spread, kQFloor));
        const int unmatched = k - m_total;
        const double q_sum = qm_sum + (double)unmatched * spread;
        const double p_tail = 1.0 - p_sum;
        const double q_tail = 1.0 - q_sum;
        float kl = klm + pau - log_spread * pu;
        if (p_tail > 0.0)
          kl += (float)p_tail * (logf((float)p_tail) - logf((float)fmax(q_tail, kQFloor)));
        out = kl;
      }
      p.kl[pos] = out;
      if (p.top1) p.top1[pos] = (uint8_t)(r[0] == c[0]);
      if (p.n_matched) p.n_matched[pos] = bad ? -1 : m_total;
    }
    __syncwarp();  // the tables are cleared again for the next pair
  }
}

}  // namespace

cudaError_t launch_topk_tail(const TopkTailArgs& a, cudaStream_t stream) {
  TopkParams p;
  p.ref_ids = a.ref_ids;
  p.ref_lp = a.ref_lp;
  p.cand_ids = a.cand_ids;
  p.cand_lp = a.cand_lp;
  p.n_rows = a.n_rows;
  p.k = a.k;
  p.vocab = (int)a.vocab;
  p.kl = a.kl;
  p.top1 = a.top1;
  p.n_matched = a.n_matched;
  p.dev_status = a.dev_status;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t pairs = (a.n_rows + 1) / 2;
  const int64_t need = (pairs + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)sms * 8;  // 8 resident CTAs of 256 threads per SM
  const unsigned grid = (unsigned)(need < cap ? need : cap);
  return launch_dependent(topk_tail_kernel, dim3(grid), dim3(kThreads), stream, p);
}

}  // namespace kld
