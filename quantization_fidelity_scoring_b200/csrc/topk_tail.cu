// Top-k + one tail bucket KL, one warp per position.
//
// "Qwopus3.8-27B-Coder-Flash: quality-eval reference", section "Method": the
// KL runs over the reference's top-64 ids plus one tail bucket; a reference id
// missing from the candidate's top-64 gets the candidate's leftover mass
// spread evenly over the ids outside the candidate's top-64; top-1 agreement
// is an exact argmax match (the first stored slot, lists being sorted per
// section "Files").
//
// Matching: the candidate's k ids are inserted into a 128-slot open-address
// table in shared memory (key = id, value = first slot holding it), then each
// reference id is looked up.  The table gives the same answer whatever order
// the lanes insert in, so the result is deterministic.  Mass sums are f64
// butterfly reductions in a fixed lane order.
#include <cuda_fp16.h>
#include <math_constants.h>

#include "kld_common.cuh"
#include "launch.h"

namespace kld {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSlots = 128;  // >= 2 * 64: probe chains stay short and always end
constexpr uint32_t kEmpty = 0xffffffffu;
constexpr double kQFloor = 1e-12;

__device__ __forceinline__ uint32_t slot_of(uint32_t id) { return (id * 0x9E3779B1u) >> 25; }

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
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
  __shared__ uint32_t table[kWarps][kSlots];
  __shared__ float cand_lp_s[kWarps][64];

  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const int k = p.k;
  uint32_t* tab = table[w];
  float* clps = cand_lp_s[w];

  for (int64_t pos = (int64_t)blockIdx.x * kWarps + w; pos < p.n_rows; pos += (int64_t)gridDim.x * kWarps) {
    const int64_t base = pos * k;
    const int j0 = lane, j1 = lane + 32;
    const bool v0 = j0 < k, v1 = j1 < k;
    const int32_t r0 = v0 ? p.ref_ids[base + j0] : 0;
    const int32_t r1 = v1 ? p.ref_ids[base + j1] : 0;
    const int32_t c0 = v0 ? p.cand_ids[base + j0] : 0;
    const int32_t c1 = v1 ? p.cand_ids[base + j1] : 0;
    const float a0 = v0 ? h2f(p.ref_lp[base + j0]) : 0.f;
    const float a1 = v1 ? h2f(p.ref_lp[base + j1]) : 0.f;
    const float b0 = v0 ? h2f(p.cand_lp[base + j0]) : 0.f;
    const float b1 = v1 ? h2f(p.cand_lp[base + j1]) : 0.f;

    const uint32_t V = (uint32_t)p.vocab;
    const bool bad_lane = (v0 && ((uint32_t)r0 >= V || (uint32_t)c0 >= V)) ||
                          (v1 && ((uint32_t)r1 >= V || (uint32_t)c1 >= V));
    const bool bad = __any_sync(0xffffffffu, bad_lane);

    // clear this warp's table, publish candidate log-probs
#pragma unroll
    for (int s = lane; s < kSlots; s += 32) tab[s] = kEmpty;
    if (v0) clps[j0] = b0;
    if (v1) clps[j1] = b1;
    __syncwarp();

    if (!bad) {
      // insert candidate ids; a repeated id keeps its lowest slot
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool valid = h == 0 ? v0 : v1;
        if (!valid) continue;
        const uint32_t id = (uint32_t)(h == 0 ? c0 : c1);
        const uint32_t entry = (id << 6) | (uint32_t)(h == 0 ? j0 : j1);
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

    // per reference slot: matched candidate slot or -1
    double p_sum = 0.0, c_sum = 0.0, qm_sum = 0.0, pu_sum = 0.0, pau_sum = 0.0, klm = 0.0;
    int unmatched = 0, matched = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const bool valid = h == 0 ? v0 : v1;
      if (!valid || bad) continue;
      const uint32_t id = (uint32_t)(h == 0 ? r0 : r1);
      const float a = h == 0 ? a0 : a1;
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
      const double pj = (double)expf(a);
      p_sum += pj;
      if (slot >= 0) {
        const float b = clps[slot];
        qm_sum += (double)expf(b);
        klm += pj * ((double)a - (double)b);
        ++matched;
      } else {
        pu_sum += pj;
        pau_sum += pj * (double)a;
        ++unmatched;
      }
    }
    if (v0) c_sum += (double)expf(b0);
    if (v1) c_sum += (double)expf(b1);

    p_sum = warp_sum(p_sum);
    c_sum = warp_sum(c_sum);
    qm_sum = warp_sum(qm_sum);
    pu_sum = warp_sum(pu_sum);
    pau_sum = warp_sum(pau_sum);
    klm = warp_sum(klm);
    unmatched = __reduce_add_sync(0xffffffffu, unmatched);
    matched = __reduce_add_sync(0xffffffffu, matched);

    if (lane == 0) {
      float out;
      if (bad) {
        out = CUDART_NAN_F;
        set_dev_status(p.dev_status, 0x2 /* KLD_DEV_BAD_ID */);
      } else {
        const double leftover = fmax(1.0 - c_sum, 0.0);
        const double spread = leftover / (double)(p.vocab - k);
        const double log_spread = log(fmax(spread, kQFloor));
        const double q_sum = qm_sum + (double)unmatched * spread;
        const double p_tail = 1.0 - p_sum;
        const double q_tail = 1.0 - q_sum;
        double kl = klm + pau_sum - log_spread * pu_sum;
        if (p_tail > 0.0) kl += p_tail * (log(p_tail) - log(fmax(q_tail, kQFloor)));
        out = (float)kl;
      }
      p.kl[pos] = out;
      if (p.top1) p.top1[pos] = (uint8_t)(r0 == c0);
      if (p.n_matched) p.n_matched[pos] = bad ? -1 : matched;
    }
    __syncwarp();  // the table is cleared again for the next position
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
  const int64_t need = (a.n_rows + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)sms * 8;  // 8 resident CTAs of 256 threads per SM
  const unsigned grid = (unsigned)(need < cap ? need : cap);
  topk_tail_kernel<<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kld
