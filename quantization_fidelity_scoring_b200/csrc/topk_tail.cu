// Top-k + one tail bucket KL, sixteen lanes per position.
//
// "Qwopus3.8-27B-Coder-Flash: quality-eval reference", section "Method": the
// KL runs over the reference's top-64 ids plus one tail bucket; a reference id
// missing from the candidate's top-64 gets the candidate's leftover mass
// spread evenly over the ids outside the candidate's top-64; top-1 agreement
// is an exact argmax match (the first stored slot, lists being sorted per
// section "Files").
//
// Each 16-lane half of a warp scores one position, so one warp instruction
// advances two positions.  Lane l of a half holds list slots 4l .. 4l+3
// (vector loads when k is a multiple of 4; element loads otherwise).
// Matching: the candidate's ids go into a 256-slot open-addressed table in
// shared memory of 32-bit entries (id << 6 | list slot), and their fp16
// log-probs into a per-position array by list slot; the load factor is at
// most 1/4, so almost every insert and lookup finishes at its first probe,
// and the two halves' tables are offset by 16 banks.  The inserts are
// shared-memory compare-and-swaps, which the hardware serialises per lane,
// and with the table traffic they bound this kernel; 64-bit entries that
// carried the log-prob cost 10 % more.  A repeated candidate id keeps its
// lowest slot (atomicMin on the entry).  Results do not depend on the order
// of insertion, so they are deterministic.  The three masses that feed 1 - sum
// (candidate list, reference list, matched candidate cells) are exp on the
// MUFU unit accumulated in f64, in fixed lane order; the KL terms are f32
// and the tail term takes one logarithm of the f64 ratio p_tail / q_tail.
#include <cuda_fp16.h>
#include <math_constants.h>

#include "kld_common.cuh"
#include "launch.h"

namespace kld {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kGroup = 16;                   // lanes per position
constexpr int kPerWarp = 32 / kGroup;        // positions per warp
constexpr int kPer = 64 / kGroup;            // list slots per lane
constexpr int kPositions = kWarps * kPerWarp;
constexpr int kSlots = 256;                  // >= 4 * 64: short probe chains that always end
constexpr int kTableStride = kSlots + 64 + 16;  // 32-bit words: table, then 64 fp16 log-probs (32 words)
constexpr uint32_t kEmpty = ~0u;
constexpr double kQFloor = 1e-12;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t slot_of(uint32_t id) { return (id * 0x9E3779B1u) >> 24; }

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// exp(lp) of a stored log-prob on the MUFU unit (relative error a few units
// in the last place; the sums that use it are f64).
__device__ __forceinline__ float mass(float lp) { return ex2(lp * kLog2e); }

__device__ __forceinline__ float fast_log(float x) {
  float r;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r * kLn2;
}

// Entry: id in bits 6..31, list slot in 0..5.  For equal ids the lower slot
// is the smaller entry.
__device__ __forceinline__ uint32_t pack(uint32_t id, int slot) { return (id << 6) | (uint32_t)slot; }
__device__ __forceinline__ uint32_t entry_id(uint32_t e) { return e >> 6; }

// Butterfly sums inside a 16-lane group (offsets 8, 4, 2, 1 stay in the group).
template <typename T>
__device__ __forceinline__ T group_sum(T v) {
#pragma unroll
  for (int off = kGroup / 2; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
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
  double inv_spread_ids;  // 1 / (vocab - k)
  bool vec;               // aligned rows for vector loads: k % 4 == 0
  float* kl;
  uint8_t* top1;
  int32_t* n_matched;
  int32_t* dev_status;
};

// Load slots 4l .. 4l+3 of one list (ids int32, log-probs as fp16 bits).
__device__ __forceinline__ void load_list(const TopkParams& p, const int32_t* ids, const uint16_t* lps,
                                          int64_t base, int gl, bool live, int32_t (&id)[kPer],
                                          uint16_t (&lp)[kPer], bool (&valid)[kPer]) {
  const int j0 = gl * kPer;
  if (p.vec && live && j0 + kPer <= p.k) {
    const int4 i4 = __ldg(reinterpret_cast<const int4*>(ids + base + j0));
    const uint2 l2 = __ldg(reinterpret_cast<const uint2*>(lps + base + j0));
    id[0] = i4.x;
    id[1] = i4.y;
    id[2] = i4.z;
    id[3] = i4.w;
    lp[0] = (uint16_t)(l2.x & 0xffffu);
    lp[1] = (uint16_t)(l2.x >> 16);
    lp[2] = (uint16_t)(l2.y & 0xffffu);
    lp[3] = (uint16_t)(l2.y >> 16);
#pragma unroll
    for (int t = 0; t < kPer; ++t) valid[t] = true;
    return;
  }
#pragma unroll
  for (int t = 0; t < kPer; ++t) {
    const int j = j0 + t;
    valid[t] = live && j < p.k;
    id[t] = valid[t] ? ids[base + j] : 0;
    lp[t] = valid[t] ? lps[base + j] : (uint16_t)0;
  }
}

__global__ void __launch_bounds__(kThreads) topk_tail_kernel(const TopkParams p) {
  __shared__ __align__(16) uint32_t table[kPositions * kTableStride];

  wait_prior_grid();
  const int lane = threadIdx.x & 31;
  const int gl = lane & (kGroup - 1);             // lane within the group
  const int grp = lane / kGroup;                  // group within the warp
  const int gslot = threadIdx.x / kGroup;         // group index in the CTA
  const unsigned gmask = 0xffffu << (grp * kGroup);
  const int k = p.k;
  const uint32_t V = (uint32_t)p.vocab;
  uint32_t* tab = table + gslot * kTableStride;
  uint16_t* clp = reinterpret_cast<uint16_t*>(tab + kSlots);

  const int64_t n_iter = (p.n_rows + kPerWarp - 1) / kPerWarp;
  for (int64_t it = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); it < n_iter;
       it += (int64_t)gridDim.x * kWarps) {
    const int64_t pos = it * kPerWarp + grp;
    const bool live = pos < p.n_rows;
    const int64_t base = pos * k;

    int32_t r[kPer], c[kPer];
    uint16_t ra[kPer], cb[kPer];
    bool valid[kPer], vc[kPer];
    load_list(p, p.ref_ids, p.ref_lp, base, gl, live, r, ra, valid);
    load_list(p, p.cand_ids, p.cand_lp, base, gl, live, c, cb, vc);

    bool bad_lane = false;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      bad_lane |= valid[i] && ((uint32_t)r[i] >= V || (uint32_t)c[i] >= V);
    const bool bad = (__ballot_sync(0xffffffffu, bad_lane) & gmask) != 0;

    // clear this group's table: 16 lanes x 8 stores of 16 bytes
    {
      uint4* t4 = reinterpret_cast<uint4*>(tab);
#pragma unroll
      for (int s = gl; s < kSlots / 4; s += kGroup) t4[s] = make_uint4(kEmpty, kEmpty, kEmpty, kEmpty);
#pragma unroll
      for (int i = 0; i < kPer; ++i) clp[gl * kPer + i] = cb[i];
    }
    __syncwarp();
    if (!bad) {
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (!valid[i]) continue;
        const uint32_t id = (uint32_t)c[i];
        const uint32_t entry = pack(id, gl * kPer + i);
        uint32_t s = slot_of(id);
        for (int probe = 0; probe < kSlots; ++probe) {
          const uint32_t old = atomicCAS(&tab[s], kEmpty, entry);
          if (old == kEmpty) break;
          if (entry_id(old) == id) {
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
    if (!bad) {
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (!valid[i]) continue;
        const float a = h2f(ra[i]);
        const float pj = mass(a);
        c_sum += (double)mass(h2f(cb[i]));
        p_sum += (double)pj;
        const uint32_t id = (uint32_t)r[i];
        uint32_t s = slot_of(id);
        uint32_t e = tab[s];
        for (int probe = 1; probe < kSlots && e != kEmpty && entry_id(e) != id; ++probe) {
          s = (s + 1) & (kSlots - 1);  // rare at load factor 1/4
          e = tab[s];
        }
        if (e != kEmpty && entry_id(e) == id) {
          const float bm = h2f(clp[e & 63u]);
          qm_sum += (double)mass(bm);
          klm += pj * (a - bm);
          ++matched;
        } else {
          pu += pj;
          pau += pj * a;
        }
      }
    }
    c_sum = group_sum(c_sum);
    p_sum = group_sum(p_sum);
    qm_sum = group_sum(qm_sum);
    klm = group_sum(klm);
    pau = group_sum(pau);
    pu = group_sum(pu);
    matched = group_sum(matched);

    if (gl == 0 && live) {
      float out;
      if (bad) {
        out = CUDART_NAN_F;
        set_dev_status(p.dev_status, 0x2 /* KLD_DEV_BAD_ID */);
      } else {
        const double spread = fmax(1.0 - c_sum, 0.0) * p.inv_spread_ids;
        const float log_spread = fast_log((float)fmax(spread, kQFloor));
        const double q_sum = qm_sum + (double)(k - matched) * spread;
        const double p_tail = 1.0 - p_sum;
        const double q_tail = 1.0 - q_sum;
        float kl = klm + pau - log_spread * pu;
        if (p_tail > 0.0) kl += (float)p_tail * logf((float)(p_tail / fmax(q_tail, kQFloor)));
        out = kl;
      }
      p.kl[pos] = out;
      if (p.top1) p.top1[pos] = (uint8_t)(r[0] == c[0]);
      if (p.n_matched) p.n_matched[pos] = bad ? -1 : matched;
    }
    __syncwarp();  // the tables are cleared again for the next positions
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
  p.inv_spread_ids = 1.0 / (double)(a.vocab - a.k);
  const auto al = [](const void* q, uintptr_t n) { return (reinterpret_cast<uintptr_t>(q) % n) == 0; };
  // 4 ids (16 B) and 4 fp16 log-probs (8 B) per lane: rows aligned when k % 4 == 0
  p.vec = (a.k % 4 == 0) && al(a.ref_ids, 16) && al(a.cand_ids, 16) && al(a.ref_lp, 8) && al(a.cand_lp, 8);
  p.kl = a.kl;
  p.top1 = a.top1;
  p.n_matched = a.n_matched;
  p.dev_status = a.dev_status;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t iters = (a.n_rows + kPerWarp - 1) / kPerWarp;
  const int64_t need = (iters + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)sms * 8;
  const unsigned grid = (unsigned)(need < cap ? need : cap);
  return launch_dependent(topk_tail_kernel, dim3(grid), dim3(kThreads), stream, p);
}

}  // namespace kld
