// Leaderboard reductions over per-position results.
//
// "Qwen3.8-27B Quantization Challenge", "The score": mean KL ranks entries;
// median, p99 and p99.9, top-1 agreement and the perplexity ratio are shown
// beside it.  "Qwen3.8-27B fidelity suite v5", "What is in here": percentiles
// and exact exceedance counts.  "Qwopus3.8-27B-Coder-Flash: quality-eval
// reference", "Method": perplexity = exp(mean NLL of the true next token).
//
// Order statistics are exact: the f32 KL bit patterns are mapped to
// order-preserving 32-bit keys and each requested rank is found by an
// MSB-first radix select over integer histograms.  kld_reduce_stats takes
// the key in three digits of 12, 10 and 10 bits; each pass histograms only
// the keys whose leading digits match a target's prefix so far.  Sums are
// f64 (counts 32-bit integers) in fixed orders: per-thread strided, then
// fixed shuffle trees, then CTA partials in CTA order, so every output is
// bitwise reproducible.
//
// Up to kSmallN positions run in one CTA that keeps the keys in shared
// memory.  Larger inputs take one grid launch per pass after a zeroing
// launch; within a pass every CTA adds its shared-memory histogram to a
// global one and the last CTA to finish (a ticket counter) chooses the next
// digits, so no separate selection launch is needed.  The shard protocol
// (kld_reduce_shard_step) keeps four 8-bit passes, whose 16 KB histograms are
// what the shards exchange.
#include <math_constants.h>

#include "kld_common.cuh"
#include "launch.h"

namespace kld {
namespace {

constexpr int kMaxTargets = 2 * KLD_MAX_QUANTILES;
constexpr int kBatch = 8;                // positions a thread loads before using any

// kld_reduce_stats: digits of 12, 10, 10 bits
constexpr int kTopBits = 12;
constexpr int kTopBins = 1 << kTopBits;  // first-pass histogram (no prefix yet)
constexpr int kLowBits = 10;
constexpr int kLowBins = 1 << kLowBits;  // later passes: one row per distinct prefix
constexpr int kLowHistWords = kMaxTargets * kLowBins;
constexpr int64_t kSmallN = 8192;

// shard protocol: four 8-bit passes
constexpr int kBins = 256;
constexpr int kPasses = 4;
constexpr int kBigThreads = 256;
constexpr int kMaxBigBlocks = 1024;

// Sums of a set of positions.  Counts fit 32 bits: n <= INT32_MAX.
struct Sums {
  double kl, nll_r, nll_c;
  unsigned n, n_nan, agree;
  unsigned exceed[KLD_MAX_THRESHOLDS];
};

// The shard block's sums: 64-bit counts, as shards' counts add up.
struct Partial {
  double kl, nll_r, nll_c;
  long long n, n_nan, agree;
  long long exceed[KLD_MAX_THRESHOLDS];
};

struct ReduceParams {
  const float* kl;
  const int32_t* ra;
  const int32_t* ca;
  const uint8_t* top1;
  const float* lpr;
  const float* lpc;
  const uint8_t* mask;
  long long n;
  int nq, nt;
  double q[KLD_MAX_QUANTILES];
  float thr[KLD_MAX_THRESHOLDS];
  kld_stats* out;
  unsigned* hist;     // shard protocol: [kPasses][kMaxTargets][kBins], the histograms of all positions
  Partial* partials;  // shard protocol: [gridDim of pass 0]
  int32_t* dev_status;
  unsigned* hist_out; // shard protocol: where a pass adds its histogram
  int withhold;       // tests only: the cooperative grid's CTA 0 leaves before the first barrier
};

__device__ __forceinline__ uint32_t f2key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0 sorts with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key2f(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}
// Key 0 is never the key of a non-NaN value (the least, -inf, maps to
// 0x007fffff), so 0 marks "not scored" wherever keys are stored.

// ------------------------------------------------------------ radix select

// Per-target radix-select state, identical in every thread that reads it.
struct Select {
  int nt;                      // number of target ranks
  int nu;                      // number of distinct prefixes
  long long n;                 // scored count
  uint32_t prefix[kMaxTargets];
  long long rem[kMaxTargets];  // rank within the current prefix group
  int uslot[kMaxTargets];      // index of the target's prefix among the distinct ones
  uint32_t uprefix[kMaxTargets];
};

// Targets from the scored count: for every quantile, the lower and upper
// order statistic ranks of linear interpolation at h = (n - 1) q.  Thread 0.
__device__ void select_init(Select& s, const ReduceParams& p, long long n) {
  s.n = n;
  s.nt = (n > 0) ? 2 * p.nq : 0;
  for (int i = 0; i < p.nq && n > 0; ++i) {
    const double h = __dmul_rn((double)(n - 1), p.q[i]);
    long long lo = (long long)floor(h);
    if (lo > n - 1) lo = n - 1;
    if (lo < 0) lo = 0;
    const long long hi = (lo + 1 < n) ? lo + 1 : n - 1;
    s.rem[2 * i] = lo;
    s.rem[2 * i + 1] = hi;
  }
  for (int t = 0; t < s.nt; ++t) s.prefix[t] = 0u;
}

// Group targets by prefix (warp 0): uslot[t] indexes uprefix[] of distinct
// prefixes, numbered in order of their first target.  Call from every thread.
__device__ void select_unique(Select& s) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const unsigned act = __ballot_sync(0xffffffffu, lane < s.nt);
    unsigned leaders = 0;
    if (lane < s.nt) {
      const unsigned same = __match_any_sync(act, s.prefix[lane]);
      const int leader = __ffs(same) - 1;
      leaders = __ballot_sync(act, lane == leader);
      const int my_u = __popc(leaders & ((1u << leader) - 1u));
      s.uslot[lane] = my_u;
      if (lane == leader) s.uprefix[my_u] = s.prefix[lane];
    }
    if (lane == 0) s.nu = __popc(leaders);  // lane 0 is active whenever nt > 0
  }
  __syncthreads();
}

__device__ __forceinline__ unsigned warp_exclusive_scan(unsigned x, int lane) {
  unsigned inc = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  return inc - x;
}

// Advance every target by one digit of kDigitBits bits from histogram rows
// h[u * row_stride + bin] (u: the target's prefix slot).  Warp w takes
// targets w, w + warps, ...  Lane l sums a run of consecutive bins and a
// warp scan of the run totals finds the run holding the target rank; for
// digits wider than 8 bits a second scan over that run's 32 sub-runs
// narrows it to at most 4 bins.  The last bins are walked in registers.
// Call from every thread; regroups the prefixes.
template <int kDigitBits>
__device__ void select_step(Select& s, const unsigned* h, int row_stride) {
  constexpr int kPer = (1 << kDigitBits) / 32;      // bins per lane, first level
  constexpr bool kTwoLevel = kPer > 8;
  constexpr int kSub = kTwoLevel ? kPer / 32 : kPer;  // bins a lane walks
  static_assert(kPer % 4 == 0 && (kSub == 1 || kSub % 4 == 0), "bins are read as 16-byte vectors");
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int t = w; t < s.nt; t += nw) {
    const unsigned* row = h + s.uslot[t] * row_stride;
    const unsigned rem = (unsigned)s.rem[t];
    unsigned c[kSub];
    unsigned run = 0;
#pragma unroll
    for (int k = 0; k < kPer; k += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(row + lane * kPer + k);
      if constexpr (!kTwoLevel) {
        c[k] = v.x;
        c[k + 1] = v.y;
        c[k + 2] = v.z;
        c[k + 3] = v.w;
      }
      run += v.x + v.y + v.z + v.w;
    }
    const unsigned excl = warp_exclusive_scan(run, lane);
    int L = __ffs(__ballot_sync(0xffffffffu, excl + run > rem)) - 1;
    if (L < 0) L = 31;
    unsigned before = __shfl_sync(0xffffffffu, excl, L);
    int first = L * kPer;  // first bin of the run holding the target
    if constexpr (kTwoLevel) {
      const unsigned* sub = row + first + lane * kSub;
      unsigned r2 = 0;
      if constexpr (kSub == 1) {
        c[0] = sub[0];
        r2 = c[0];
      } else {
#pragma unroll
        for (int k = 0; k < kSub; k += 4) {
          const uint4 v = *reinterpret_cast<const uint4*>(sub + k);
          c[k] = v.x;
          c[k + 1] = v.y;
          c[k + 2] = v.z;
          c[k + 3] = v.w;
          r2 += v.x + v.y + v.z + v.w;
        }
      }
      const unsigned e2 = warp_exclusive_scan(r2, lane);
      L = __ffs(__ballot_sync(0xffffffffu, before + e2 + r2 > rem)) - 1;
      if (L < 0) L = 31;
      before += __shfl_sync(0xffffffffu, e2, L);
      first += L * kSub;
    }
    // lane L holds the final bins: walk them
    unsigned acc = before;
    int k = 0;
#pragma unroll
    for (int j = 0; j < kSub - 1; ++j) {
      if (k == j && acc + c[j] <= rem) {
        acc += c[j];
        k = j + 1;
      }
    }
    k = __shfl_sync(0xffffffffu, k, L);
    acc = __shfl_sync(0xffffffffu, acc, L);
    if (lane == 0) {
      s.rem[t] = (long long)(rem - acc);
      s.prefix[t] = (s.prefix[t] << kDigitBits) | (uint32_t)(first + k);
    }
    __syncwarp();
  }
  __syncthreads();
  select_unique(s);
}

// A pass's distinct prefixes in registers; unused slots hold a value no
// prefix takes (prefixes have at most 24 bits).
struct Prefixes {
  uint32_t v[kMaxTargets];
};

__device__ __forceinline__ Prefixes load_prefixes(const Select& s) {
  Prefixes r;
#pragma unroll
  for (int u = 0; u < kMaxTargets; ++u) r.v[u] = (u < s.nu) ? s.uprefix[u] : 0xffffffffu;
  return r;
}

// The slot of the distinct prefix `pre` is, or -1.
__device__ __forceinline__ int prefix_slot(const Prefixes& P, uint32_t pre) {
  int u = -1;
#pragma unroll
  for (int j = kMaxTargets - 1; j >= 0; --j)
    if (P.v[j] == pre) u = j;
  return u;
}

// ---------------------------------------------------------------- sums

__device__ __forceinline__ bool has_agreement(const ReduceParams& p) { return p.ra != nullptr || p.top1 != nullptr; }

// Positions first, first + stride, ... below end, kBatch at a time with
// every load of a batch issued before any is used.  Adds scored positions
// to `acc` and hands every position's index and key (0: not scored) to
// on_pos.
template <class F>
__device__ __forceinline__ void scan_positions(const ReduceParams& p, long long first, long long stride,
                                               long long end, Sums& acc, F&& on_pos) {
  for (long long i0 = first; i0 < end; i0 += kBatch * stride) {
    float v[kBatch], lr[kBatch], lc[kBatch];
    int ra[kBatch], ca[kBatch];
    bool in[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const long long i = i0 + b * stride;
      in[b] = i < end && (!p.mask || p.mask[i]);
      v[b] = in[b] ? p.kl[i] : 0.f;
      lr[b] = (in[b] && p.lpr) ? p.lpr[i] : 0.f;
      lc[b] = (in[b] && p.lpc) ? p.lpc[i] : 0.f;
      ra[b] = (in[b] && p.ra) ? p.ra[i] : -1;
      ca[b] = (in[b] && p.ra) ? p.ca[i] : -2;
      if (in[b] && !p.ra && p.top1) ra[b] = ca[b] = p.top1[i] ? 0 : -1;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const long long i = i0 + b * stride;
      if (i >= end) break;
      uint32_t key = 0u;
      if (in[b]) {
        if (v[b] != v[b]) {
          ++acc.n_nan;
        } else {
          ++acc.n;
          acc.kl += (double)v[b];
          acc.nll_r -= (double)lr[b];
          acc.nll_c -= (double)lc[b];
          acc.agree += (ra[b] >= 0 && ra[b] == ca[b]) ? 1u : 0u;
#pragma unroll
          for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j)
            if (j < p.nt) acc.exceed[j] += (v[b] > p.thr[j]) ? 1u : 0u;
          key = f2key(v[b]);
        }
      }
      on_pos(i, key);
    }
  }
}

// Keys only (kBatch at a time), for passes after the first: on_key(key)
// for the scored positions among first, first + stride, ... below end.
template <class F>
__device__ __forceinline__ void scan_keys(const ReduceParams& p, long long first, long long stride, long long end,
                                          F&& on_key) {
  for (long long i0 = first; i0 < end; i0 += kBatch * stride) {
    float v[kBatch];
    bool in[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const long long i = i0 + b * stride;
      in[b] = i < end && (!p.mask || p.mask[i]);
      v[b] = in[b] ? p.kl[i] : 0.f;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
      if (in[b] && !(v[b] != v[b])) on_key(f2key(v[b]));
  }
}

__device__ __forceinline__ void sums_add(Sums& a, const Sums& b, int nt) {
  a.kl += b.kl;
  a.nll_r += b.nll_r;
  a.nll_c += b.nll_c;
  a.n += b.n;
  a.n_nan += b.n_nan;
  a.agree += b.agree;
#pragma unroll
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j)
    if (j < nt) a.exceed[j] += b.exceed[j];
}

// Fixed-order warp sum: f64 by a shuffle tree (result in lane 0), counts
// by redux (exact, in every lane).
__device__ __forceinline__ void warp_sums(Sums& a, int nt) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a.kl += __shfl_down_sync(0xffffffffu, a.kl, off);
    a.nll_r += __shfl_down_sync(0xffffffffu, a.nll_r, off);
    a.nll_c += __shfl_down_sync(0xffffffffu, a.nll_c, off);
  }
  a.n = __reduce_add_sync(0xffffffffu, a.n);
  a.n_nan = __reduce_add_sync(0xffffffffu, a.n_nan);
  a.agree = __reduce_add_sync(0xffffffffu, a.agree);
#pragma unroll
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j)
    if (j < nt) a.exceed[j] = __reduce_add_sync(0xffffffffu, a.exceed[j]);
}

// Sum of every thread's `a` in a fixed order (warps, then the warp totals
// in warp order), returned to every thread.  sh holds 32 entries.  Call
// from every thread.
__device__ Sums block_sums(Sums a, Sums* sh, int nt) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  warp_sums(a, nt);
  if (lane == 0) sh[w] = a;
  __syncthreads();
  if (w == 0) {
    Sums t{};
    if (lane < nw) t = sh[lane];
    warp_sums(t, nt);
    __syncwarp();
    if (lane == 0) sh[0] = t;
  }
  __syncthreads();
  const Sums r = sh[0];
  __syncthreads();
  return r;
}

__device__ void write_stats(const ReduceParams& p, long long n, long long n_nan, long long agree, double kl,
                            double nll_r, double nll_c, const long long* exceed, const Select& s) {
  kld_stats st;
  const double nan = CUDART_NAN;
  st.n = n;
  st.n_nan = n_nan;
  const bool have_agree = has_agreement(p);
  st.top1_agree = have_agree ? agree : -1;
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j) st.exceed[j] = (j < p.nt) ? exceed[j] : 0;
  st.mean_kl = n ? kl / (double)n : nan;
  st.top1_rate = (have_agree && n) ? (double)agree / (double)n : nan;
  st.ref_mean_nll = (p.lpr && n) ? nll_r / (double)n : nan;
  st.cand_mean_nll = (p.lpc && n) ? nll_c / (double)n : nan;
  st.ref_ppl = exp(st.ref_mean_nll);
  st.cand_ppl = exp(st.cand_mean_nll);
  st.ppl_ratio = st.cand_ppl / st.ref_ppl;
  for (int i = 0; i < KLD_MAX_QUANTILES; ++i) {
    st.q_value[i] = nan;
    st.q_lo[i] = st.q_hi[i] = CUDART_NAN_F;
  }
  for (int i = 0; i < p.nq && n > 0; ++i) {
    const float lo = key2f(s.prefix[2 * i]);
    const float hi = key2f(s.prefix[2 * i + 1]);
    const double h = __dmul_rn((double)(n - 1), p.q[i]);
    const double frac = __dsub_rn(h, floor(h));
    st.q_lo[i] = lo;
    st.q_hi[i] = hi;
    st.q_value[i] = __dadd_rn((double)lo, __dmul_rn(__dsub_rn((double)hi, (double)lo), frac));
  }
  st.nq = p.nq;
  st.nt = p.nt;
  *p.out = st;
}

// ---------------------------------------------------------------- targets

// The statistics from the totals (doubles valid in lane 0, counts in every
// lane) and the targets' order statistics as keys; warp 0, fields written
// by several lanes side by side.
__device__ void write_stats_warp(const ReduceParams& p, const Sums& t, const uint32_t* target_key, int lane) {
  kld_stats* o = p.out;
  const double kl = __shfl_sync(0xffffffffu, t.kl, 0);
  const double nll_r = __shfl_sync(0xffffffffu, t.nll_r, 0);
  const double nll_c = __shfl_sync(0xffffffffu, t.nll_c, 0);
  const long long n = t.n;
  const double nan = CUDART_NAN;
  const double ref_nll = (p.lpr && n) ? nll_r / (double)n : nan;
  const double cand_nll = (p.lpc && n) ? nll_c / (double)n : nan;
  double ppl = nan;
  if (lane == 1) ppl = exp(ref_nll);
  if (lane == 2) ppl = exp(cand_nll);
  const double ref_ppl = __shfl_sync(0xffffffffu, ppl, 1);
  const double cand_ppl = __shfl_sync(0xffffffffu, ppl, 2);
  if (lane == 0) {
    const bool have_agree = has_agreement(p);
    o->n = n;
    o->n_nan = t.n_nan;
    o->top1_agree = have_agree ? (long long)t.agree : -1;
    for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j) o->exceed[j] = (j < p.nt) ? (long long)t.exceed[j] : 0;
    o->mean_kl = n ? kl / (double)n : nan;
    o->top1_rate = (have_agree && n) ? (double)t.agree / (double)n : nan;
    o->ref_mean_nll = ref_nll;
    o->cand_mean_nll = cand_nll;
    o->nq = p.nq;
    o->nt = p.nt;
  } else if (lane == 1) {
    o->ref_ppl = ref_ppl;
  } else if (lane == 2) {
    o->cand_ppl = cand_ppl;
  } else if (lane == 3) {
    o->ppl_ratio = cand_ppl / ref_ppl;
  } else if (lane >= 8 && lane < 8 + KLD_MAX_QUANTILES) {
    const int i = lane - 8;
    if (i < p.nq && n > 0) {
      const float lo = key2f(target_key[2 * i]);
      const float hi = key2f(target_key[2 * i + 1]);
      const double h = __dmul_rn((double)(n - 1), p.q[i]);
      const double frac = __dsub_rn(h, floor(h));
      o->q_lo[i] = lo;
      o->q_hi[i] = hi;
      o->q_value[i] = __dadd_rn((double)lo, __dmul_rn(__dsub_rn((double)hi, (double)lo), frac));
    } else {
      o->q_lo[i] = o->q_hi[i] = CUDART_NAN_F;
      o->q_value[i] = nan;
    }
  }
}

// ---------------------------------------------------------------- one CTA

// Histogram of one select pass over keys[0 .. m) in shared memory (0 = not
// scored): the digit at `shift` of every key (kTop), or of every key whose
// bits above the digit extend a target prefix, in the row of that prefix.
// Keys are loaded four at a time before any is counted.
template <int kDigitBits, bool kTop>
__device__ __forceinline__ void hist_keys(const uint32_t* keys, int m, const Select& sel, int shift, unsigned* hist) {
  constexpr int B = 4;
  Prefixes P;
  if constexpr (!kTop) P = load_prefixes(sel);
  for (int i0 = threadIdx.x; i0 < m; i0 += B * blockDim.x) {
    uint32_t k[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int i = i0 + b * blockDim.x;
      k[b] = (i < m) ? keys[i] : 0u;
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (!k[b]) continue;
      int u = 0;
      if constexpr (!kTop) u = prefix_slot(P, k[b] >> (shift + kDigitBits));
      if (u >= 0) atomicAdd(&hist[(u << kDigitBits) | ((k[b] >> shift) & ((1u << kDigitBits) - 1u))], 1u);
    }
  }
}

constexpr int kSmallThreads = 512;

// All of kld_reduce_stats for n <= kSmallN in one CTA: every thread sums
// its positions and keeps their keys in shared memory; four 8-bit select
// passes follow, each one histogram over all targets' prefixes; warp 0
// writes the statistics.
__global__ void __launch_bounds__(kSmallThreads) reduce_small_kernel(const ReduceParams p) {
  extern __shared__ __align__(16) uint32_t keys[];  // p.n
  __shared__ __align__(16) unsigned hist[kMaxTargets * kBins];
  __shared__ Sums sh[32];
  __shared__ Select sel;
  static_assert(kSmallThreads / 32 <= kMaxTargets, "one first-pass histogram row per warp");
  for (int i = threadIdx.x; i < kMaxTargets * kBins; i += blockDim.x) hist[i] = 0u;
  wait_prior_grid();
  Sums acc{};
  scan_positions(p, threadIdx.x, blockDim.x, p.n, acc, [&](long long i, uint32_t key) { keys[i] = key; });
  const Sums tot = block_sums(acc, sh, p.nt);  // its barriers publish keys[] and the cleared histogram
  if (threadIdx.x == 0) select_init(sel, p, tot.n);
  __syncthreads();
  select_unique(sel);
  const int m = (int)p.n;
  if (sel.nt > 0) {
    // first pass: every warp counts into its own row (the top bytes of KL
    // values fall in a handful of bins), then the rows are added up
    unsigned* row = hist + (threadIdx.x >> 5) * kBins;
    for (int i0 = threadIdx.x; i0 < m; i0 += 4 * blockDim.x) {
      uint32_t k[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) k[b] = (i0 + b * (int)blockDim.x < m) ? keys[i0 + b * blockDim.x] : 0u;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (k[b]) atomicAdd(&row[k[b] >> 24], 1u);
    }
    __syncthreads();
    unsigned c = 0u;
    if (threadIdx.x < kBins)
      for (int r = 0; r < (int)(blockDim.x >> 5); ++r) c += hist[r * kBins + threadIdx.x];
    __syncthreads();
    if (threadIdx.x < kBins) hist[threadIdx.x] = c;
  }
  __syncthreads();
  select_step<8>(sel, hist, kBins);
  for (int pass = 1; pass < kPasses; ++pass) {
    for (int i = threadIdx.x; i < sel.nu * kBins; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    if (sel.nt > 0) hist_keys<8, false>(keys, m, sel, 24 - 8 * pass, hist);
    __syncthreads();
    select_step<8>(sel, hist, kBins);
  }
  if (threadIdx.x < 32) write_stats_warp(p, tot, sel.prefix, threadIdx.x);
}

constexpr size_t kSmallSmemMax = sizeof(uint32_t) * kSmallN;

// ---------------------------------------------------------------- grid

// kld_reduce_stats for n > kSmallN: one cooperative launch (every CTA
// resident at once) over contiguous chunks of positions, one CTA per SM.
// Pass 0 sums the chunk, keeps its keys in shared memory (when the chunk
// fits) and histograms their top 12 bits; passes 1 and 2 histogram the
// next 10 bits of the keys that extend a target's prefix.  After passes 0
// and 1 every CTA adds its histogram into global memory and meets the
// others at a grid barrier (a counter polled with a bounded wait); then
// each CTA reads the whole histogram and takes the next digits itself, so
// no CTA waits for another to publish them.  After pass 2 the last CTA to
// arrive (a ticket) takes the final digits and writes the statistics.

constexpr int kCoopThreads = 512;
constexpr int kCoopKeys = 32768;  // keys a CTA keeps in shared memory (128 KB)
constexpr int kMaxCoopGrid = 1024;
constexpr long long kSpinLimit = 1ll << 21;  // polls before a wait gives up (about a second)
constexpr size_t kCoopSmem = sizeof(unsigned) * (kLowHistWords + kCoopKeys);

struct CoopWs {
  unsigned arrive[4];
  alignas(16) unsigned hist0[kTopBins];
  alignas(16) unsigned hist1[kLowHistWords];
  alignas(16) unsigned hist2[kLowHistWords];
  Sums partials[kMaxCoopGrid];
};

// Cleared before every cooperative launch: its counters and the first
// pass's histogram (the later passes' are cleared inside it).
__global__ void __launch_bounds__(1024) reduce_zero_kernel(CoopWs* g) {
  wait_prior_grid();
  if (threadIdx.x < 4) g->arrive[threadIdx.x] = 0u;
  uint4* h = reinterpret_cast<uint4*>(g->hist0);
  for (int i = threadIdx.x; i < kTopBins / 4; i += blockDim.x) h[i] = make_uint4(0u, 0u, 0u, 0u);
}

__device__ Sums load_sums_cg(const Sums* s, int nt) {
  Sums r{};
  r.kl = __ldcg(&s->kl);
  r.nll_r = __ldcg(&s->nll_r);
  r.nll_c = __ldcg(&s->nll_c);
  r.n = __ldcg(&s->n);
  r.n_nan = __ldcg(&s->n_nan);
  r.agree = __ldcg(&s->agree);
#pragma unroll
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j)
    if (j < nt) r.exceed[j] = __ldcg(&s->exceed[j]);
  return r;
}

// Adds this CTA's histogram (`words` bins) to gh and counts the CTA in at
// `counter`, every thread's global writes fenced first.  Call from every
// thread; returns the counter's value before this CTA's arrival (thread 0).
__device__ unsigned flush_and_arrive(const unsigned* sh_hist, unsigned* gh, int words, unsigned* counter,
                                     unsigned* sh_ticket) {
  for (int i = threadIdx.x; i < words; i += blockDim.x) {
    const unsigned c = sh_hist[i];
    if (c) atomicAdd(&gh[i], c);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) *sh_ticket = atomicAdd(counter, 1u);
  __syncthreads();
  return *sh_ticket;
}

// Grid barrier after flush_and_arrive: thread 0 polls the counter until
// every CTA has arrived (bounded; a timeout is recorded as
// KLD_DEV_TIMEOUT and returns false).  Call from every thread.
__device__ bool grid_wait(const unsigned* counter, int32_t* dev_status, int* sh_ok) {
  if (threadIdx.x == 0) {
    int ok = 0;
    for (long long it = 0; it < kSpinLimit; ++it) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
      if (v >= gridDim.x) {
        ok = 1;
        break;
      }
      __nanosleep(32);
    }
    if (!ok) set_dev_status(dev_status, 0x4 /* KLD_DEV_TIMEOUT */);
    *sh_ok = ok;
  }
  __syncthreads();
  return *sh_ok != 0;
}

__global__ void __launch_bounds__(kCoopThreads, 1) reduce_coop_kernel(const ReduceParams p, CoopWs* g) {
  extern __shared__ __align__(16) unsigned dsm[];
  unsigned* hist = dsm;                  // kTopBins, later nu rows of kLowBins
  uint32_t* keys = dsm + kLowHistWords;  // this CTA's chunk, when it fits
  __shared__ Sums sh[32];
  __shared__ Select sel;
  __shared__ unsigned ticket;
  __shared__ int ok;
  __shared__ unsigned n_scored;

  const long long chunk = (p.n + gridDim.x - 1) / gridDim.x;
  const long long begin = (long long)blockIdx.x * chunk;
  const long long end = (begin + chunk < p.n) ? begin + chunk : p.n;
  const int m = (end > begin) ? (int)(end - begin) : 0;
  const bool cached = chunk <= kCoopKeys;

  for (int i = threadIdx.x; i < kTopBins; i += blockDim.x) hist[i] = 0u;
  if (threadIdx.x == 0) n_scored = 0u;
  {  // the later passes' global histograms, cleared across the grid
    const int vecs = 2 * kLowHistWords / 4;
    uint4* h12 = reinterpret_cast<uint4*>(g->hist1);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < vecs; i += gridDim.x * blockDim.x)
      h12[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();

  // pass 0: sums, keys, top-12-bit histogram
  Sums acc{};
  scan_positions(p, begin + threadIdx.x, blockDim.x, end, acc, [&](long long i, uint32_t key) {
    if (cached) keys[i - begin] = key;
    else if (key) atomicAdd(&hist[key >> (32 - kTopBits)], 1u);
  });
  const Sums cta = block_sums(acc, sh, p.nt);  // its barriers publish keys[] (or complete the histogram)
  if (threadIdx.x == 0) g->partials[blockIdx.x] = cta;
  if (cached) {
    hist_keys<kTopBits, true>(keys, m, sel, 32 - kTopBits, hist);
    __syncthreads();
  }
  // (tests only: CTA 0 never arrives, so every other CTA's bounded wait
  // runs out and reports KLD_DEV_TIMEOUT)
  if (p.withhold && blockIdx.x == 0) return;
  flush_and_arrive(hist, g->hist0, kTopBins, &g->arrive[0], &ticket);
  if (!grid_wait(&g->arrive[0], p.dev_status, &ok)) return;
  {  // every CTA: the whole first-pass histogram, the scored count, the first digits
    unsigned c = 0u;
    for (int i = threadIdx.x; i < kTopBins; i += blockDim.x) {
      const unsigned v = __ldcg(g->hist0 + i);
      hist[i] = v;
      c += v;
    }
    c = __reduce_add_sync(0xffffffffu, c);
    if ((threadIdx.x & 31) == 0) atomicAdd(&n_scored, c);
    __syncthreads();
    if (threadIdx.x == 0) select_init(sel, p, (long long)n_scored);
    __syncthreads();
    select_unique(sel);
    select_step<kTopBits>(sel, hist, kTopBins);
  }

  // passes 1 and 2
  for (int pass = 1; pass <= 2; ++pass) {
    const int shift = (pass == 1) ? kLowBits : 0;  // this pass's digit: key bits [shift, shift + 10)
    const int words = sel.nu * kLowBins;          // nu = 0 when there is no target
    for (int i = threadIdx.x; i < words; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    if (sel.nt > 0) {
      if (cached) {
        hist_keys<kLowBits, false>(keys, m, sel, shift, hist);
      } else {
        const Prefixes P = load_prefixes(sel);
        scan_keys(p, begin + threadIdx.x, blockDim.x, end, [&](uint32_t k) {
          const int u = prefix_slot(P, k >> (shift + kLowBits));
          if (u >= 0) atomicAdd(&hist[u * kLowBins + ((k >> shift) & (kLowBins - 1))], 1u);
        });
      }
    }
    __syncthreads();
    unsigned* gh = (pass == 1) ? g->hist1 : g->hist2;
    const unsigned before = flush_and_arrive(hist, gh, words, &g->arrive[pass], &ticket);
    if (pass == 1) {
      if (!grid_wait(&g->arrive[1], p.dev_status, &ok)) return;
    } else if (before != gridDim.x - 1) {
      return;  // not the last CTA of the final pass
    } else {
      __threadfence();
    }
    for (int i = threadIdx.x; i < words; i += blockDim.x) hist[i] = __ldcg(gh + i);
    __syncthreads();
    select_step<kLowBits>(sel, hist, kLowBins);
  }

  // the last CTA: all sums in CTA order, then the statistics
  Sums s{};
  for (int b = threadIdx.x; b < (int)gridDim.x; b += blockDim.x) sums_add(s, load_sums_cg(&g->partials[b], p.nt), p.nt);
  const Sums tot = block_sums(s, sh, p.nt);
  if (threadIdx.x < 32) write_stats_warp(p, tot, sel.prefix, threadIdx.x);
}

// ---------------------------------------------------------------- shards
//
// Statistics over positions held by several shards: every shard runs four
// 8-bit passes over its own positions, and between passes the shards
// exchange fixed-size blocks (their pass histogram; at the first pass also
// their sums).  Each shard adds the gathered blocks up in shard order, so
// every shard holds the same totals and derives the same select state and
// statistics.

struct ShardBlock {
  Partial partial;
  unsigned hist[kMaxTargets * kBins];
};

__device__ __forceinline__ Partial to_partial(const Sums& s) {
  Partial r;
  r.kl = s.kl;
  r.nll_r = s.nll_r;
  r.nll_c = s.nll_c;
  r.n = s.n;
  r.n_nan = s.n_nan;
  r.agree = s.agree;
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j) r.exceed[j] = s.exceed[j];
  return r;
}

__device__ __forceinline__ void partial_add(Partial& a, const Partial& b) {
  a.kl += b.kl;
  a.nll_r += b.nll_r;
  a.nll_c += b.nll_c;
  a.n += b.n;
  a.n_nan += b.n_nan;
  a.agree += b.agree;
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j) a.exceed[j] += b.exceed[j];
}

// Rebuild the select state from the all-shard histograms of passes < pass.
// Call from every thread of the block.
__device__ void select_replay(Select& s, const ReduceParams& p, int pass) {
  if (threadIdx.x == 0) {
    long long n = 0;
    for (int d = 0; d < kBins; ++d) n += p.hist[d];
    select_init(s, p, n);
  }
  __syncthreads();
  select_unique(s);
  for (int q = 0; q < pass; ++q) select_step<8>(s, p.hist + q * kMaxTargets * kBins, kBins);
}

// One 8-bit pass over this shard's positions, adding its histogram to
// p.hist_out; pass 0 histograms every scored key and writes the CTA's sums.
__global__ void __launch_bounds__(kBigThreads) reduce_pass_kernel(const ReduceParams p, int pass) {
  __shared__ __align__(16) unsigned sh[kMaxTargets * kBins];
  __shared__ Select sel;
  __shared__ Sums sh_w[32];
  for (int i = threadIdx.x; i < kMaxTargets * kBins; i += blockDim.x) sh[i] = 0u;
  wait_prior_grid();
  if (pass > 0) select_replay(sel, p, pass);  // starts with a barrier
  __syncthreads();
  const long long begin = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  int used = kBins;
  if (pass == 0) {
    Sums acc{};
    scan_positions(p, begin, stride, p.n, acc, [&](long long, uint32_t key) {
      if (key) atomicAdd(&sh[key >> 24], 1u);
    });
    const Sums cta = block_sums(acc, sh_w, p.nt);
    if (threadIdx.x == 0) p.partials[blockIdx.x] = to_partial(cta);
  } else {
    used = sel.nu * kBins;
    const int shift = 24 - 8 * pass;
    const Prefixes P = load_prefixes(sel);
    if (sel.nt > 0)
      scan_keys(p, begin, stride, p.n, [&](uint32_t key) {
        const int u = prefix_slot(P, key >> (shift + 8));
        if (u >= 0) atomicAdd(&sh[u * kBins + ((key >> shift) & 0xffu)], 1u);
      });
  }
  __syncthreads();
  for (int i = threadIdx.x; i < used; i += blockDim.x)
    if (sh[i]) atomicAdd(&p.hist_out[i], sh[i]);
}

// this shard's block: histogram cleared (before a pass adds into it)
__global__ void shard_clear_kernel(ShardBlock* blk) {
  wait_prior_grid();
  for (int i = threadIdx.x; i < kMaxTargets * kBins; i += blockDim.x) blk->hist[i] = 0u;
}

// this shard's sums of the first pass: its CTAs' partials, each thread
// adding a strided set in CTA order, then a fixed tree over the threads
__global__ void __launch_bounds__(kBigThreads) shard_fold_kernel(const ReduceParams p, int n_partials,
                                                                 ShardBlock* blk) {
  __shared__ Partial sh[kBigThreads];
  wait_prior_grid();
  Partial t{};
  for (int b = threadIdx.x; b < n_partials; b += blockDim.x) partial_add(t, p.partials[b]);
  sh[threadIdx.x] = t;
  __syncthreads();
  for (int half = blockDim.x / 2; half > 0; half >>= 1) {
    if ((int)threadIdx.x < half) partial_add(sh[threadIdx.x], sh[threadIdx.x + half]);
    __syncthreads();
  }
  if (threadIdx.x == 0) blk->partial = sh[0];
}

// all shards' blocks of pass `pass`: histograms into the totals, in shard
// order (integers: exact); after the first pass also the sums (shard order)
__global__ void shard_gather_kernel(const ReduceParams p, int pass, const ShardBlock* gathered, int n_shards,
                                    Partial* total) {
  wait_prior_grid();
  unsigned* h = p.hist + pass * kMaxTargets * kBins;
  for (int i = threadIdx.x; i < kMaxTargets * kBins; i += blockDim.x) {
    unsigned c = 0u;
    for (int s = 0; s < n_shards; ++s) c += gathered[s].hist[i];
    h[i] = c;
  }
  if (pass == 0 && threadIdx.x == 0) {
    Partial t = gathered[0].partial;
    for (int s = 1; s < n_shards; ++s) partial_add(t, gathered[s].partial);
    *total = t;
  }
}

__global__ void __launch_bounds__(kBigThreads) shard_final_kernel(const ReduceParams p, const Partial* total) {
  wait_prior_grid();
  __shared__ Select sel;
  select_replay(sel, p, kPasses);
  if (threadIdx.x == 0) {
    const Partial& t = *total;
    write_stats(p, t.n, t.n_nan, t.agree, t.kl, t.nll_r, t.nll_c, t.exceed, sel);
  }
}

int big_grid(long long n) {
  long long g = (n + kBigThreads * 8 - 1) / (kBigThreads * 8);
  if (g < 1) g = 1;
  if (g > kMaxBigBlocks) g = kMaxBigBlocks;
  return (int)g;
}

constexpr size_t kShardHistBytes = sizeof(unsigned) * kPasses * kMaxTargets * kBins;

ReduceParams make_params(const ReduceArgs& a) {
  ReduceParams p;
  p.kl = a.kl;
  p.ra = a.ref_argmax;
  p.ca = a.cand_argmax;
  p.top1 = a.top1;
  p.lpr = a.ref_lp;
  p.lpc = a.cand_lp;
  p.mask = a.mask;
  p.n = a.n;
  p.nq = a.nq;
  p.nt = a.nt;
  for (int i = 0; i < KLD_MAX_QUANTILES; ++i) p.q[i] = a.quantiles[i];
  for (int i = 0; i < KLD_MAX_THRESHOLDS; ++i) p.thr[i] = a.thresholds[i];
  p.out = a.out;
  p.hist = nullptr;
  p.partials = nullptr;
  p.dev_status = a.dev_status;
  p.hist_out = nullptr;
  p.withhold = a.withhold;
  return p;
}

// Cooperative grid for n positions: about eight positions per thread, at
// most as many CTAs as can be resident at once.
cudaError_t coop_grid(long long n, int* grid) {
  int dev = 0, sms = 0, occ = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, reduce_coop_kernel, kCoopThreads, kCoopSmem);
  if (e != cudaSuccess) return e;
  long long g = (n + kCoopThreads * kBatch - 1) / (kCoopThreads * kBatch);
  long long cap = (long long)sms * occ;
  if (cap > kMaxCoopGrid) cap = kMaxCoopGrid;
  if (cap < 1) return cudaErrorCooperativeLaunchTooLarge;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  *grid = (int)g;
  return cudaSuccess;
}

cudaError_t launch_coop(const ReduceParams& p, CoopWs* g, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kCoopThreads);
  cfg.dynamicSmemBytes = kCoopSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, reduce_coop_kernel, p, g);
}

}  // namespace

size_t reduce_workspace_bytes(int64_t n) {
  (void)n;
  return sizeof(CoopWs);
}

size_t reduce_shard_block_bytes() { return sizeof(ShardBlock); }

// the shard workspace: pass histograms, CTA sums, the all-shard sums
size_t reduce_shard_workspace_bytes(int64_t n) {
  (void)n;
  return kShardHistBytes + sizeof(Partial) * (kMaxBigBlocks + 1);
}

cudaError_t launch_reduce(const ReduceArgs& a, cudaStream_t stream) {
  const ReduceParams p = make_params(a);
  if (a.n <= kSmallN) {
    cudaError_t e = allow_dynamic_smem<reduce_small_kernel>(kSmallSmemMax);
    if (e != cudaSuccess) return e;
    return launch_dependent_smem(reduce_small_kernel, dim3(1), dim3(kSmallThreads), sizeof(uint32_t) * (size_t)a.n,
                                 stream, p);
  }
  cudaError_t e = allow_dynamic_smem<reduce_coop_kernel>(kCoopSmem);
  int grid = 0;
  if (e == cudaSuccess) e = coop_grid(a.n, &grid);
  if (e != cudaSuccess) return e;
  CoopWs* g = reinterpret_cast<CoopWs*>(a.workspace);
  e = launch_dependent(reduce_zero_kernel, dim3(1), dim3(1024), stream, g);
  if (e != cudaSuccess) return e;
  return launch_coop(p, g, grid, stream);
}

cudaError_t launch_reduce_shard_step(const ReduceArgs& a, int step, int n_shards, const void* gathered,
                                     void* block_out, cudaStream_t stream) {
  ReduceParams p = make_params(a);
  p.hist = reinterpret_cast<unsigned*>(a.workspace);
  p.partials = reinterpret_cast<Partial*>(reinterpret_cast<char*>(a.workspace) + kShardHistBytes);
  Partial* total = p.partials + kMaxBigBlocks;
  ShardBlock* blk = reinterpret_cast<ShardBlock*>(block_out);
  const ShardBlock* all = reinterpret_cast<const ShardBlock*>(gathered);
  const int grid = big_grid(a.n);
  cudaError_t e = cudaSuccess;
  if (step > 0) {  // the previous pass, all shards
    e = launch_dependent(shard_gather_kernel, dim3(1), dim3(1024), stream, p, step - 1, all, n_shards, total);
    if (e != cudaSuccess) return e;
  }
  if (step == kPasses) return launch_dependent(shard_final_kernel, dim3(1), dim3(kBigThreads), stream, p,
                                               (const Partial*)total);
  e = launch_dependent(shard_clear_kernel, dim3(1), dim3(1024), stream, blk);
  if (e != cudaSuccess) return e;
  p.hist_out = blk->hist;
  e = launch_dependent(reduce_pass_kernel, dim3(grid), dim3(kBigThreads), stream, p, step);
  if (e != cudaSuccess || step != 0) return e;
  return launch_dependent(shard_fold_kernel, dim3(1), dim3(kBigThreads), stream, p, grid, blk);
}

}  // namespace kld
