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
// MSB-first radix select, 8 bits per pass (4 passes), with integer
// histograms.  Sums are f64 in fixed orders (per-thread strided, then fixed
// trees), so every output is bitwise reproducible.
//
// Small inputs (n <= kSmallN) run in one CTA with shared-memory histograms;
// larger inputs use a grid of CTAs per pass with global integer histograms.
#include <math_constants.h>

#include "kld_common.cuh"
#include "launch.h"

namespace kld {
namespace {

constexpr int kMaxTargets = 2 * KLD_MAX_QUANTILES;
constexpr int kBins = 256;
constexpr int kPasses = 4;
constexpr int64_t kSmallN = 65536;
constexpr int kBigThreads = 256;
constexpr int kMaxBigBlocks = 1024;
constexpr int kSmallThreads = 512;

struct Partial {  // per-CTA sums of the first pass
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
  unsigned* hist;     // [kPasses][kMaxTargets][kBins]: the histograms of all positions
  Partial* partials;  // [gridDim of pass 0]
  int32_t* dev_status;
  unsigned* hist_out; // where a pass adds its histogram (null: hist's own slot for the pass)
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

// Per-target radix-select state, identical in every thread that derives it.
struct Select {
  int nt;                      // number of target ranks
  long long n;                 // scored count
  uint32_t prefix[kMaxTargets];
  long long rem[kMaxTargets];  // rank within the current prefix group
  int uslot[kMaxTargets];      // index of the target's prefix among the unique ones
  uint32_t uprefix[kMaxTargets];
  int nu;
};

__device__ __forceinline__ bool scored(const ReduceParams& p, long long i, float& v) {
  if (p.mask && !p.mask[i]) return false;
  v = p.kl[i];
  return !(v != v);
}

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

// Group targets by prefix (warp 0): uslot[t] indexes uprefix[] of unique
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

// Advance every target by one 8-bit digit using histogram h[u][bin]: warp w
// takes targets w, w + warps, ...  Lane l holds bins 8l .. 8l+7; a warp scan
// of the lane totals finds the bin holding the target rank.  Call from every
// thread; regroups the prefixes afterwards.
__device__ void select_step(Select& s, const unsigned* h) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int t = w; t < s.nt; t += nw) {
    const unsigned* row = h + s.uslot[t] * kBins + lane * 8;
    unsigned c[8];
    unsigned run = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      run += row[k];
      c[k] = run;  // inclusive prefix within the lane
    }
    unsigned base = run;  // inclusive warp scan of lane totals
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned o = __shfl_up_sync(0xffffffffu, base, off);
      if (lane >= off) base += o;
    }
    base -= run;  // exclusive
    const unsigned long long rem = (unsigned long long)s.rem[t];
    const unsigned hit = __ballot_sync(0xffffffffu, (unsigned long long)base + run > rem);
    const int L = hit ? __ffs(hit) - 1 : 31;
    if (lane == L) {
      int k = 7;
      for (int j = 7; j >= 0; --j)
        if ((unsigned long long)base + c[j] > rem) k = j;
      const unsigned before = base + (k ? c[k - 1] : 0u);
      s.rem[t] = (long long)(rem - before);
      s.prefix[t] = (s.prefix[t] << 8) | (uint32_t)(8 * L + k);
    }
    __syncwarp();
  }
  __syncthreads();
  select_unique(s);
}

// One histogram pass over [begin, end) with stride `stride`, adding into the
// shared-memory histogram sh[u][bin] for elements whose key matches a unique
// prefix of this pass.  Pass 0 histograms every scored element.
__device__ __forceinline__ void hist_pass(const ReduceParams& p, const Select& s, int pass,
                                          long long begin, long long stride, unsigned* sh) {
  const int shift = 24 - 8 * pass;
  for (long long i = begin; i < p.n; i += stride) {
    float v;
    if (!scored(p, i, v)) continue;
    const uint32_t key = f2key(v);
    const uint32_t digit = (key >> shift) & 0xffu;
    if (pass == 0) {
      atomicAdd(&sh[digit], 1u);
    } else {
      const uint32_t pre = key >> (shift + 8);
      for (int u = 0; u < s.nu; ++u) {
        if (s.uprefix[u] == pre) {
          atomicAdd(&sh[u * kBins + digit], 1u);
          break;
        }
      }
    }
  }
}

// Pass-0 sums of one thread (fixed stride order).  Positions are taken four
// at a time with every load issued before any is used, so one memory latency
// covers the batch.
__device__ __forceinline__ void thread_sums(const ReduceParams& p, long long begin, long long stride,
                                            Partial& acc) {
  constexpr int B = 4;
  acc.kl = acc.nll_r = acc.nll_c = 0.0;
  acc.n = acc.n_nan = acc.agree = 0;
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j) acc.exceed[j] = 0;
  for (long long i0 = begin; i0 < p.n; i0 += B * stride) {
    float v[B], lr[B], lc[B];
    int ra[B], ca[B];
    bool in[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const long long i = i0 + b * stride;
      in[b] = i < p.n && (!p.mask || p.mask[i]);
      v[b] = in[b] ? p.kl[i] : 0.f;
      lr[b] = (in[b] && p.lpr) ? p.lpr[i] : 0.f;
      lc[b] = (in[b] && p.lpc) ? p.lpc[i] : 0.f;
      ra[b] = (in[b] && p.ra) ? p.ra[i] : -1;
      ca[b] = (in[b] && p.ra) ? p.ca[i] : -2;
      if (in[b] && !p.ra && p.top1) ra[b] = ca[b] = p.top1[i] ? 0 : -1;
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (!in[b]) continue;
      if (v[b] != v[b]) {
        ++acc.n_nan;
        continue;
      }
      ++acc.n;
      acc.kl += (double)v[b];
      acc.nll_r -= (double)lr[b];
      acc.nll_c -= (double)lc[b];
      acc.agree += (ra[b] >= 0 && ra[b] == ca[b]) ? 1 : 0;
      for (int j = 0; j < p.nt; ++j) acc.exceed[j] += (v[b] > p.thr[j]) ? 1 : 0;
    }
  }
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

__device__ __forceinline__ Partial shfl_down_partial(const Partial& a, int off, int nt) {
  Partial o;
  o.kl = __shfl_down_sync(0xffffffffu, a.kl, off);
  o.nll_r = __shfl_down_sync(0xffffffffu, a.nll_r, off);
  o.nll_c = __shfl_down_sync(0xffffffffu, a.nll_c, off);
  o.n = __shfl_down_sync(0xffffffffu, a.n, off);
  o.n_nan = __shfl_down_sync(0xffffffffu, a.n_nan, off);
  o.agree = __shfl_down_sync(0xffffffffu, a.agree, off);
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j)
    o.exceed[j] = (j < nt) ? __shfl_down_sync(0xffffffffu, a.exceed[j], off) : 0;
  return o;
}

// Fixed-order CTA reduction of per-thread partials: a butterfly in every
// warp, then warp 0 does the same over the warp totals.  Result valid in
// thread 0.  Call from every thread.
__device__ void block_sum(Partial& acc, Partial* sh_warp, int nt) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const Partial o = shfl_down_partial(acc, off, nt);
    if (lane < off) partial_add(acc, o);
  }
  if (lane == 0) sh_warp[w] = acc;
  __syncthreads();
  if (w == 0) {
    Partial t;
    if (lane < nw) {
      t = sh_warp[lane];
    } else {
      t.kl = t.nll_r = t.nll_c = 0.0;
      t.n = t.n_nan = t.agree = 0;
      for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j) t.exceed[j] = 0;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const Partial o = shfl_down_partial(t, off, nt);
      if (lane < off) partial_add(t, o);
    }
    if (lane == 0) acc = t;
  }
  __syncthreads();
}

__device__ void write_stats(const ReduceParams& p, const Partial& tot, const Select& s) {
  kld_stats st;
  const long long n = tot.n;
  const double nan = CUDART_NAN;
  st.n = n;
  st.n_nan = tot.n_nan;
  const bool have_agree = p.ra != nullptr || p.top1 != nullptr;
  st.top1_agree = have_agree ? tot.agree : -1;
  for (int j = 0; j < KLD_MAX_THRESHOLDS; ++j) st.exceed[j] = (j < p.nt) ? tot.exceed[j] : 0;
  st.mean_kl = n ? tot.kl / (double)n : nan;
  st.top1_rate = (have_agree && n) ? (double)tot.agree / (double)n : nan;
  st.ref_mean_nll = (p.lpr && n) ? tot.nll_r / (double)n : nan;
  st.cand_mean_nll = (p.lpc && n) ? tot.nll_c / (double)n : nan;
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

// ---------------------------------------------------------------- one CTA

// Up to kCacheN scored keys stay in shared memory across the passes; key 0
// marks a position that is not scored (only NaN bit patterns map to 0).
constexpr int kCacheN = 6144;

__global__ void __launch_bounds__(kSmallThreads) reduce_small_kernel(const ReduceParams p) {
  __shared__ unsigned sh[kMaxTargets * kBins];
  __shared__ uint32_t keys[kCacheN];
  __shared__ Partial sh_warp[kSmallThreads / 32];
  __shared__ Select sel;

  wait_prior_grid();
  const bool cached = p.n <= kCacheN;
  Partial acc;
  thread_sums(p, threadIdx.x, blockDim.x, acc);
  if (cached) {
    for (int i = threadIdx.x; i < (int)p.n; i += blockDim.x) {
      float v;
      keys[i] = scored(p, i, v) ? f2key(v) : 0u;
    }
  }
  block_sum(acc, sh_warp, p.nt);
  if (threadIdx.x == 0) select_init(sel, p, acc.n);
  __syncthreads();
  select_unique(sel);
  for (int pass = 0; pass < kPasses; ++pass) {
    for (int i = threadIdx.x; i < kMaxTargets * kBins; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
    if (sel.nt > 0) {
      if (cached) {
        const int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < (int)p.n; i += blockDim.x) {
          const uint32_t key = keys[i];
          if (key == 0u) continue;
          const uint32_t digit = (key >> shift) & 0xffu;
          if (pass == 0) {
            atomicAdd(&sh[digit], 1u);
          } else {
            const uint32_t pre = key >> (shift + 8);
            for (int u = 0; u < sel.nu; ++u)
              if (sel.uprefix[u] == pre) {
                atomicAdd(&sh[u * kBins + digit], 1u);
                break;
              }
          }
        }
      } else {
        hist_pass(p, sel, pass, threadIdx.x, blockDim.x, sh);
      }
    }
    __syncthreads();
    select_step(sel, sh);
  }
  if (threadIdx.x == 0) write_stats(p, acc, sel);
}

// ---------------------------------------------------------------- many CTAs

__global__ void reduce_zero_kernel(unsigned* hist) {
  wait_prior_grid();
  for (int i = threadIdx.x; i < kPasses * kMaxTargets * kBins; i += blockDim.x) hist[i] = 0u;
}

// Rebuild the select state from the histograms of passes < pass.  Call
// from every thread of the block.
__device__ void select_replay(Select& s, const ReduceParams& p, int pass) {
  if (threadIdx.x == 0) {
    long long n = 0;
    for (int d = 0; d < kBins; ++d) n += p.hist[d];
    select_init(s, p, n);
  }
  __syncthreads();
  select_unique(s);
  for (int q = 0; q < pass; ++q) select_step(s, p.hist + q * kMaxTargets * kBins);
}

__global__ void __launch_bounds__(kBigThreads) reduce_pass_kernel(const ReduceParams p, int pass) {
  wait_prior_grid();
  __shared__ unsigned sh[kMaxTargets * kBins];
  __shared__ Select sel;
  __shared__ Partial sh_warp[kBigThreads / 32];
  for (int i = threadIdx.x; i < kMaxTargets * kBins; i += blockDim.x) sh[i] = 0u;
  if (pass == 0) {
    if (threadIdx.x == 0) {
      sel.nt = 1;  // histogram every scored element
      sel.nu = 0;
    }
    __syncthreads();
  } else {
    select_replay(sel, p, pass);
  }
  const long long begin = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  if (sel.nt > 0) hist_pass(p, sel, pass, begin, stride, sh);
  if (pass == 0) {
    Partial acc;
    thread_sums(p, begin, stride, acc);
    block_sum(acc, sh_warp, p.nt);
    if (threadIdx.x == 0) p.partials[blockIdx.x] = acc;
  }
  __syncthreads();
  unsigned* g = p.hist_out ? p.hist_out : p.hist + pass * kMaxTargets * kBins;
  const int used = (pass == 0) ? kBins : sel.nu * kBins;
  for (int i = threadIdx.x; i < used; i += blockDim.x)
    if (sh[i]) atomicAdd(&g[i], sh[i]);
}

__global__ void __launch_bounds__(kBigThreads) reduce_final_kernel(const ReduceParams p, int n_partials) {
  wait_prior_grid();
  __shared__ Select sel;
  select_replay(sel, p, kPasses);
  if (threadIdx.x != 0) return;
  Partial tot = p.partials[0];
  for (int b = 1; b < n_partials; ++b) partial_add(tot, p.partials[b]);
  write_stats(p, tot, sel);
}

// ---------------------------------------------------------------- shards
//
// Statistics over positions held by several shards: every shard runs the
// passes of the grid path on its own positions, and between passes the
// shards exchange fixed-size blocks (their pass histogram; at the first
// pass also their sums).  Each shard adds the gathered blocks up in shard
// order, so every shard holds the same totals and derives the same select
// state and statistics.

struct ShardBlock {
  Partial partial;
  unsigned hist[kMaxTargets * kBins];
};

// this shard's block: histogram cleared (before a pass adds into it)
__global__ void shard_clear_kernel(ShardBlock* blk) {
  wait_prior_grid();
  for (int i = threadIdx.x; i < kMaxTargets * kBins; i += blockDim.x) blk->hist[i] = 0u;
}

// this shard's sums of the first pass: its CTAs' partials in CTA order
__global__ void shard_fold_kernel(const ReduceParams p, int n_partials, ShardBlock* blk) {
  wait_prior_grid();
  if (threadIdx.x != 0) return;
  Partial tot = p.partials[0];
  for (int b = 1; b < n_partials; ++b) partial_add(tot, p.partials[b]);
  blk->partial = tot;
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
  if (threadIdx.x == 0) write_stats(p, *total, sel);
}

int big_grid(long long n) {
  long long g = (n + kBigThreads * 8 - 1) / (kBigThreads * 8);
  if (g < 1) g = 1;
  if (g > kMaxBigBlocks) g = kMaxBigBlocks;
  return (int)g;
}

constexpr size_t kHistBytes = sizeof(unsigned) * kPasses * kMaxTargets * kBins;

}  // namespace

size_t reduce_workspace_bytes(int64_t n) {
  (void)n;
  return kHistBytes + sizeof(Partial) * kMaxBigBlocks;
}

size_t reduce_shard_block_bytes() { return sizeof(ShardBlock); }

// the shard workspace: the grid path's, then the all-shard sums
size_t reduce_shard_workspace_bytes(int64_t n) { return reduce_workspace_bytes(n) + sizeof(Partial); }

cudaError_t launch_reduce(const ReduceArgs& a, cudaStream_t stream) {
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
  p.hist = reinterpret_cast<unsigned*>(a.workspace);
  p.partials = reinterpret_cast<Partial*>(reinterpret_cast<char*>(a.workspace) + kHistBytes);
  p.dev_status = a.dev_status;
  p.hist_out = nullptr;

  if (a.n <= kSmallN) return launch_dependent(reduce_small_kernel, dim3(1), dim3(kSmallThreads), stream, p);
  const int grid = big_grid(a.n);
  cudaError_t e = launch_dependent(reduce_zero_kernel, dim3(1), dim3(1024), stream, p.hist);
  for (int pass = 0; pass < kPasses && e == cudaSuccess; ++pass)
    e = launch_dependent(reduce_pass_kernel, dim3(grid), dim3(kBigThreads), stream, p, pass);
  if (e != cudaSuccess) return e;
  return launch_dependent(reduce_final_kernel, dim3(1), dim3(kBigThreads), stream, p, grid);
}

cudaError_t launch_reduce_shard_step(const ReduceArgs& a, int step, int n_shards, const void* gathered,
                                     void* block_out, cudaStream_t stream) {
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
  p.hist = reinterpret_cast<unsigned*>(a.workspace);
  p.partials = reinterpret_cast<Partial*>(reinterpret_cast<char*>(a.workspace) + kHistBytes);
  p.dev_status = a.dev_status;
  Partial* total = reinterpret_cast<Partial*>(reinterpret_cast<char*>(a.workspace) + kHistBytes +
                                              sizeof(Partial) * kMaxBigBlocks);
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
  return launch_dependent(shard_fold_kernel, dim3(1), dim3(32), stream, p, grid, blk);
}

}  // namespace kld
