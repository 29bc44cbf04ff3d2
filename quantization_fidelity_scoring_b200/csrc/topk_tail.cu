// Top-k + one tail bucket KL, eight lanes per position.
//
// "Qwopus3.8-27B-Coder-Flash: quality-eval reference", section "Method": the
// KL runs over the reference's top-64 ids plus one tail bucket; a reference id
// missing from the candidate's top-64 gets the candidate's leftover mass
// spread evenly over the ids outside the candidate's top-64; top-1 agreement
// is an exact argmax match (the first stored slot, lists being sorted per
// section "Files").
//
// Each 8-lane group of a warp scores one position, so one warp instruction
// advances four positions.  Lane l of a group holds list slots 8l .. 8l+7
// (two 16-byte id vectors and one 16-byte log-prob vector when k is a
// multiple of 8; element loads otherwise).
//
// Matching uses a 256-slot linear-probing table per position in shared
// memory, 32-bit entries (id << 6 | list slot) with the top bit marking a
// contested slot: one that an id hashing there failed to take.
//   1. Every candidate id tries its home slot with one compare-and-swap; the
//      eight of a lane are issued back to back and their results read after.
//      A repeated id keeps its lowest list slot (atomicMin).
//   2. The few ids that lost their home slot (about 7 of 64 at load 1/4) are
//      compacted into a per-position list and placed by the group's eight
//      lanes together: mark the home slot contested, then probe onwards.
//   3. Each reference id reads its home slot: its own entry is a match, an
//      empty or uncontested slot means absent (an id stored further on would
//      have contested it), and only a contested slot holding another id goes
//      to a second compacted list that probes onwards.
// The table is a valid linear-probing table whatever the order of the
// inserts, so results do not depend on scheduling.  The masses that feed
// 1 - sum (candidate list, reference list, matched candidate cells) are exp
// on the MUFU unit accumulated in f64 in fixed lane order; the per-cell KL
// terms are f32.  The candidate mass is reduced first, so every lane knows
// the spread mass before the reference cells are scored and each unmatched
// cell adds its spread term directly.
#include <cuda_fp16.h>
#include <math_constants.h>

#include <atomic>

#include "kld_common.cuh"
#include "launch.h"

namespace kld {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kGroup = 8;                    // lanes per position
constexpr int kPerWarp = 32 / kGroup;        // positions per warp
constexpr int kPer = 64 / kGroup;            // list slots per lane
constexpr int kPositions = kWarps * kPerWarp;
constexpr int kSlots = 256;                  // >= 4 * 64: short probe chains that always end
// Per-position shared area in 32-bit words: the table, the candidate fp16
// log-probs by list slot, the pending list, the pending lookups' results.
constexpr int kLpOff = kSlots;
constexpr int kListOff = kLpOff + 64 / 2;
constexpr int kResOff = kListOff + 64;
constexpr int kStride = kResOff + 64 / 4;
constexpr uint32_t kContested = 1u << 31;
constexpr uint32_t kIdBits = 0x7FFFFFC0u;    // the id field of an entry
constexpr uint32_t kEmpty = 0x7FFFFFFFu;     // id field all ones: never a valid id (ids < 2^25 - 1)
constexpr double kQFloor = 1e-12;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t slot_of(uint32_t id) { return (id * 0x9E3779B1u) >> 24; }

// Entry: id in bits 6..30, list slot in 0..5, bit 31 = contested.  For equal
// ids the lower list slot is the smaller entry.
__device__ __forceinline__ uint32_t pack(uint32_t id, int slot) { return (id << 6) | (uint32_t)slot; }
__device__ __forceinline__ uint32_t entry_id(uint32_t e) { return (e & kIdBits) >> 6; }
// True when entry e holds the id whose key (id << 6) is given.
__device__ __forceinline__ bool same_id(uint32_t e, uint32_t key) { return ((e ^ key) & kIdBits) == 0u; }

// exp(lp) of a stored log-prob on the MUFU unit (relative error a few units
// in the last place; the sums that use it are f64).
__device__ __forceinline__ float mass(float lp) { return ex2(lp * kLog2e); }

__device__ __forceinline__ float lg2(float x) {
  float r;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// The two fp16 values packed in w, converted one by one: the conversion is
// exact, fp16 subnormals included (log-probs of near-certain tokens are
// subnormal in fp16), and the same on both sides of a cell.
__device__ __forceinline__ float2 half_pair(uint32_t w) {
  return make_float2(__half2float(__ushort_as_half((unsigned short)(w & 0xffffu))),
                     __half2float(__ushort_as_half((unsigned short)(w >> 16))));
}

// Butterfly sum inside an 8-lane group (offsets 4, 2, 1 stay in the group).
template <typename T>
__device__ __forceinline__ T group_sum(T v) {
#pragma unroll
  for (int off = kGroup / 2; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Exclusive prefix of n over the group's lanes; *total gets the group sum.
__device__ __forceinline__ int group_offset(int n, int gl, int* total) {
  int incl = n;
#pragma unroll
  for (int d = 1; d < kGroup; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d, kGroup);
    if (gl >= d) incl += v;
  }
  *total = __shfl_sync(0xffffffffu, incl, kGroup - 1, kGroup);
  return incl - n;
}

// Lowers the entry at *slot to e's list slot (same id), keeping its
// contested bit.  Every failed swap means another update of the slot landed,
// and a slot sees at most 128 of them (64 inserts, 64 contest marks).
__device__ __forceinline__ void merge_lower(uint32_t* slot, uint32_t e, uint32_t cur) {
  for (int tries = 0; tries < 2 * kSlots; ++tries) {
    const uint32_t want = min(cur & ~kContested, e) | (cur & kContested);
    if (want == cur) return;
    const uint32_t seen = atomicCAS(slot, cur, want);
    if (seen == cur) return;
    cur = seen;
  }
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
  float* kl;
  uint8_t* top1;
  int32_t* n_matched;
  int32_t* dev_status;
};

// Slots 8l .. 8l+7 of one list: ids, and fp16 log-probs packed in pairs.
// Returns the number of valid slots (a prefix of the eight).  kVec: rows
// aligned with k % 8 == 0, so a lane has all eight slots or none.
template <bool kVec>
__device__ __forceinline__ int load_list(const TopkParams& p, const int32_t* ids, const uint16_t* lps,
                                         int64_t base, int j0, bool live, int32_t (&id)[kPer],
                                         uint32_t (&lp)[kPer / 2]) {
  const int nv = live ? max(0, min(kPer, p.k - j0)) : 0;
  if constexpr (kVec) {
    if (nv == kPer) {
      const int4 a = __ldg(reinterpret_cast<const int4*>(ids + base + j0));
      const int4 b = __ldg(reinterpret_cast<const int4*>(ids + base + j0 + 4));
      const uint4 l = __ldg(reinterpret_cast<const uint4*>(lps + base + j0));
      id[0] = a.x; id[1] = a.y; id[2] = a.z; id[3] = a.w;
      id[4] = b.x; id[5] = b.y; id[6] = b.z; id[7] = b.w;
      lp[0] = l.x; lp[1] = l.y; lp[2] = l.z; lp[3] = l.w;
    } else {
#pragma unroll
      for (int t = 0; t < kPer; ++t) id[t] = 0;
#pragma unroll
      for (int t = 0; t < kPer / 2; ++t) lp[t] = 0;
    }
  } else {
#pragma unroll
    for (int t = 0; t < kPer; ++t) id[t] = t < nv ? __ldg(ids + base + j0 + t) : 0;
#pragma unroll
    for (int t = 0; t < kPer / 2; ++t) {
      const uint32_t lo = 2 * t < nv ? __ldg(lps + base + j0 + 2 * t) : 0u;
      const uint32_t hi = 2 * t + 1 < nv ? __ldg(lps + base + j0 + 2 * t + 1) : 0u;
      lp[t] = lo | (hi << 16);
    }
  }
  return nv;
}

template <bool kVec>
__global__ void __launch_bounds__(kThreads) topk_tail_kernel(const TopkParams p) {
  __shared__ __align__(16) uint32_t area[kPositions * kStride];

  wait_prior_grid();
  const int lane = threadIdx.x & 31;
  const int gl = lane & (kGroup - 1);             // lane within the group
  const int grp = lane / kGroup;                  // group within the warp
  const unsigned gmask = 0xffu << (grp * kGroup);
  const int j0 = gl * kPer;                       // first list slot of this lane
  const uint32_t V = (uint32_t)p.vocab;
  uint32_t* tab = area + (threadIdx.x / kGroup) * kStride;
  uint32_t* list = tab + kListOff;
  int8_t* res = reinterpret_cast<int8_t*>(tab + kResOff);
  const uint16_t* clp = reinterpret_cast<const uint16_t*>(tab + kLpOff);

  const int64_t n_iter = (p.n_rows + kPerWarp - 1) / kPerWarp;
  for (int64_t it = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); it < n_iter;
       it += (int64_t)gridDim.x * kWarps) {
    const int64_t pos = it * kPerWarp + grp;
    const bool live = pos < p.n_rows;
    const int64_t base = pos * p.k;

    int32_t r[kPer], c[kPer];
    uint32_t rl[kPer / 2], cl[kPer / 2];
    int nv = load_list<kVec>(p, p.ref_ids, p.ref_lp, base, j0, live, r, rl);
    load_list<kVec>(p, p.cand_ids, p.cand_lp, base, j0, live, c, cl);

    bool bad_lane = false;
#pragma unroll
    for (int t = 0; t < kPer; ++t) bad_lane |= t < nv && ((uint32_t)r[t] >= V || (uint32_t)c[t] >= V);
    const bool bad = (__ballot_sync(0xffffffffu, bad_lane) & gmask) != 0;
    if (bad) nv = 0;
    // slot t of this lane takes part (one predicate for all eight under kVec)
    const bool full = nv == kPer;
    const auto on = [&](int t) { return kVec ? full : t < nv; };

    // clear this position's table (8 lanes x 8 stores of 16 bytes), park the
    // candidate log-probs by list slot
    {
      uint4* t4 = reinterpret_cast<uint4*>(tab);
#pragma unroll
      for (int s = gl; s < kSlots / 4; s += kGroup) t4[s] = make_uint4(kEmpty, kEmpty, kEmpty, kEmpty);
      reinterpret_cast<uint4*>(tab + kLpOff)[gl] = make_uint4(cl[0], cl[1], cl[2], cl[3]);
    }

    // candidate mass, reduced first: the spread mass of unmatched cells
    double c_part = 0.0;
#pragma unroll
    for (int t = 0; t < kPer / 2; ++t) {
      const float2 b = half_pair(cl[t]);
      if (on(2 * t)) c_part += (double)mass(b.x);
      if (on(2 * t + 1)) c_part += (double)mass(b.y);
    }
    __syncwarp();

    // 1. home-slot inserts
    uint32_t lost = 0;
    {
      uint32_t old[kPer];
#pragma unroll
      for (int t = 0; t < kPer; ++t) {
        const uint32_t id = (uint32_t)c[t];
        old[t] = on(t) ? atomicCAS(&tab[slot_of(id)], kEmpty, pack(id, j0 + t)) : kEmpty;
      }
#pragma unroll
      for (int t = 0; t < kPer; ++t) {
        const uint32_t id = (uint32_t)c[t];
        const bool dup = old[t] != kEmpty && same_id(old[t], id << 6);
        if (dup) atomicMin(&tab[slot_of(id)], pack(id, j0 + t));  // repeated id
        lost |= (uint32_t)(old[t] != kEmpty && !dup) << t;
      }
    }
    // 2. displaced inserts, compacted per position
    if (__any_sync(0xffffffffu, lost != 0)) {
      int n_lost;
      int off = group_offset(__popc(lost), gl, &n_lost);
#pragma unroll
      for (int t = 0; t < kPer; ++t)
        if ((lost >> t) & 1u) list[off++] = pack((uint32_t)c[t], j0 + t);
      __syncwarp();
      for (int i = gl; i < n_lost; i += kGroup) {
        const uint32_t e = list[i];
        const uint32_t h = slot_of(entry_id(e));
        atomicOr(&tab[h], kContested);
        uint32_t s = (h + 1) & (kSlots - 1);
        for (int probe = 1; probe < kSlots; ++probe) {
          uint32_t cur = *reinterpret_cast<volatile uint32_t*>(&tab[s]);
          if (cur == kEmpty) {
            cur = atomicCAS(&tab[s], kEmpty, e);
            if (cur == kEmpty) break;
          }
          if (same_id(cur, e)) {
            merge_lower(&tab[s], e, cur);
            break;
          }
          s = (s + 1) & (kSlots - 1);
        }
      }
    }
    const double c_sum = group_sum(c_part);
    const double spread = fmax(1.0 - c_sum, 0.0) * p.inv_spread_ids;
    const float log_spread = lg2((float)fmax(spread, kQFloor)) * kLn2;
    __syncwarp();

    // 3. lookups at the home slot: own entry = match; a contested slot
    // holding another id = keep probing; anything else = absent
    int mt[kPer];
    uint32_t pend = 0;
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const uint32_t id = (uint32_t)r[t];
      const uint32_t e = on(t) ? tab[slot_of(id)] : kEmpty;
      const bool hit = same_id(e, id << 6);
      mt[t] = hit ? (int)(e & 63u) : -1;
      pend |= (uint32_t)(!hit && (e & kContested) != 0u) << t;
    }
    if (__any_sync(0xffffffffu, pend != 0)) {
      int n_pend;
      int off = group_offset(__popc(pend), gl, &n_pend);
#pragma unroll
      for (int t = 0; t < kPer; ++t)
        if ((pend >> t) & 1u) list[off++] = pack((uint32_t)r[t], j0 + t);
      __syncwarp();
      for (int i = gl; i < n_pend; i += kGroup) {
        const uint32_t e = list[i];
        uint32_t s = (slot_of(entry_id(e)) + 1) & (kSlots - 1);
        int found = -1;
        for (int probe = 1; probe < kSlots; ++probe) {
          const uint32_t cur = tab[s];
          if (cur == kEmpty) break;
          if (same_id(cur, e)) {
            found = (int)(cur & 63u);
            break;
          }
          s = (s + 1) & (kSlots - 1);
        }
        res[e & 63u] = (int8_t)found;
      }
      __syncwarp();
#pragma unroll
      for (int t = 0; t < kPer; ++t)
        if ((pend >> t) & 1u) mt[t] = res[j0 + t];
    }

    // reference cells, without branches: an unmatched cell reads slot 0 and
    // takes the spread values instead
    double p_part = 0.0, q_part = 0.0;
    float kl_part = 0.f;
    int matched = 0;
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const float2 ap = half_pair(rl[t / 2]);
      const float a = (t & 1) ? ap.y : ap.x;
      const bool m = mt[t] >= 0;
      const float bm = __half2float(__ushort_as_half(clp[m ? mt[t] : 0]));
      const float pj = mass(a);
      const float lq = m ? bm : log_spread;
      const double qv = m ? (double)mass(bm) : spread;
      if (on(t)) {
        p_part += (double)pj;
        q_part += qv;
        kl_part += pj * (a - lq);
        matched += (int)m;
      }
    }
    p_part = group_sum(p_part);
    q_part = group_sum(q_part);
    kl_part = group_sum(kl_part);
    matched = group_sum(matched);

    if (gl == 0 && live) {
      float out;
      if (bad) {
        out = CUDART_NAN_F;
        set_dev_status(p.dev_status, 0x2 /* KLD_DEV_BAD_ID */);
      } else {
        const double p_tail = 1.0 - p_part;
        const double q_tail = 1.0 - q_part;
        out = kl_part;
        if (p_tail > 0.0) {
          const float pt = (float)p_tail;
          // difference of the base-2 logs first, then the scale: equal tails
          // give exactly 0 (no fused multiply-add can leave a rounding residue)
          const float d2 = lg2(pt) - lg2((float)fmax(q_tail, kQFloor));
          out += pt * (d2 * kLn2);
        }
      }
      p.kl[pos] = out;
      if (p.top1) p.top1[pos] = (uint8_t)(r[0] == c[0]);
      if (p.n_matched) p.n_matched[pos] = bad ? -1 : matched;
    }
    __syncwarp();  // the tables are cleared again for the next positions
  }
}

template <bool kVec>
int resident_blocks() {
  static std::atomic<int> cached[16];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 16) {
    const int v = cached[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int blocks = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, topk_tail_kernel<kVec>, kThreads, 0) != cudaSuccess ||
      blocks < 1)
    blocks = 1;
  if (dev >= 0 && dev < 16) cached[dev].store(blocks, std::memory_order_relaxed);
  return blocks;
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
  // 8 ids (2 x 16 B) and 8 fp16 log-probs (16 B) per lane: rows aligned when k % 8 == 0
  const bool vec = (a.k % 8 == 0) && al(a.ref_ids, 16) && al(a.cand_ids, 16) && al(a.ref_lp, 16) &&
                   al(a.cand_lp, 16);
  p.kl = a.kl;
  p.top1 = a.top1;
  p.n_matched = a.n_matched;
  p.dev_status = a.dev_status;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t iters = (a.n_rows + kPerWarp - 1) / kPerWarp;
  const int64_t need = (iters + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)sms * (vec ? resident_blocks<true>() : resident_blocks<false>());
  const unsigned grid = (unsigned)(need < cap ? need : cap);
  return vec ? launch_dependent(topk_tail_kernel<true>, dim3(grid), dim3(kThreads), stream, p)
             : launch_dependent(topk_tail_kernel<false>, dim3(grid), dim3(kThreads), stream, p);
}

}  // namespace kld
