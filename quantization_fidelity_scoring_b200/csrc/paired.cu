// Paired comparison of two candidates scored against one reference:
// per-context means, per-cluster sums, source-cluster bootstrap replicates
// and exact percentiles of the replicates.
//
// "Qwen3.8-27B fidelity suite v5": the suite's contexts come from source
// clusters ("What is in here"), and two candidates are compared paired per
// context, reported as a difference with a 95 % source-cluster bootstrap
// interval and the contexts each side wins (the sibling-rebuild paragraph
// and the "compare against a published candidate" step).  The page gives
// no formulas; kld.h states the reading implemented here.
//
// Four launches, all deterministic (f64 sums in fixed orders, integer
// counts):
//   ctx      one warp per context: sums of A's and B's counted KL (exact in
//            f64 for ordinary spreads of f32 values), the count, the means
//            and their difference d_c.
//   cluster  one thread per context adds d_c to its cluster's D[k] as a
//            64-bit fixed-point integer (scaled to the largest |d_c|, so the
//            integer sums are exact and their order does not matter) and 1
//            to N[k]; non-finite d_c set flags instead.  More blocks sum
//            chunks of 1024 contexts (means, win and tie counts) for the
//            finish to add in order.
//   boot     one warp per replicate: the draws' D and N gathered and summed.
//   select   one CTA finds the replicates' order statistics at the target
//            ranks exactly (bucketed 64-bit keys, a few passes), then one of
//            its warps writes the result (the finish kernel does that alone
//            when there are no replicates).
#include <math_constants.h>

#include <algorithm>
#include <cfloat>

#include "kld_common.cuh"
#include "launch.h"

namespace kld {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTargets = 2 * KLD_MAX_QUANTILES;
constexpr int kBootThreads = 512;
constexpr int kBootSmemClusters = 2048;  // clusters whose sums a boot CTA keeps in shared memory

constexpr int kTotChunk = 1024;  // contexts per totals block

// Sums over one chunk of counted contexts.
struct PairedPart {
  double sa, sb, sd;  // m_A, m_B, d
  long long n_used, n_pos, a_lower, b_lower, ties;
};

struct PairedTotals {
  unsigned n_valid;  // replicates whose draws hold a counted context
  unsigned pad;
  int shift;         // one unit of the clusters' fixed-point sums is 2^shift
  int pad2;
  double ostat[kMaxTargets];
};

// Flags of a cluster whose contexts include non-finite differences.
constexpr int kFlagPosInf = 1, kFlagNegInf = 2, kFlagNaN = 4;

struct PairedParams {
  const float* a;
  const float* b;
  const uint8_t* mask;
  long long n_ctx;
  int ctx_len;
  const int32_t* cluster;
  int n_clusters;
  const int32_t* resample;
  int n_boot;
  int nq;
  double q[KLD_MAX_QUANTILES];
  kld_paired* out;
  double* boot;  // [n_boot] replicate statistics
  double* ctx_a;
  double* ctx_b;
  double* ctx_d;
  int32_t* ctx_n;
  double* blk_max;    // [ctx blocks] largest finite |d_c| of each block of the context pass
  int n_ctx_blocks;
  long long* Dq;      // [n_clusters] fixed-point sums of d_c
  int32_t* Dflag;     // [n_clusters] kFlag* bits
  long long* Nk;
  PairedPart* parts;  // [ceil(n_ctx / kTotChunk)]
  PairedTotals* tot;
  int32_t* dev_status;
};

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_down_sync(0xffffffffu, x, off);
  return x;  // lane 0
}

__device__ __forceinline__ long long warp_sum(long long x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_down_sync(0xffffffffu, x, off);
  return x;  // lane 0
}

// Rank (0-based, ascending) of target t among n values: quantile t / 2,
// lower (even t) or upper (odd t) order statistic of linear interpolation.
__device__ __forceinline__ long long target_rank(const PairedParams& p, long long n, int t) {
  const double h = __dmul_rn((double)(n - 1), p.q[t >> 1]);
  long long lo = (long long)floor(h);
  if (lo > n - 1) lo = n - 1;
  if (lo < 0) lo = 0;
  if (!(t & 1)) return lo;
  return (lo + 1 < n) ? lo + 1 : n - 1;
}

__device__ __forceinline__ void add_pair(float va, float vb, bool in, double& sa, double& sb, unsigned& cnt) {
  if (in && !(va != va) && !(vb != vb)) {
    sa += (double)va;
    sb += (double)vb;
    ++cnt;
  }
}

__global__ void __launch_bounds__(kThreads) paired_ctx_kernel(const PairedParams p) {
  __shared__ double wmax[kWarps];
  wait_prior_grid();
  if (blockIdx.x == 0 && threadIdx.x == 0) p.tot->n_valid = 0u;
  // the clusters' accumulators start at zero (the cluster pass runs after this kernel)
  for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < p.n_clusters;
       k += (long long)gridDim.x * blockDim.x) {
    p.Dq[k] = 0ll;
    p.Nk[k] = 0ll;
    p.Dflag[k] = 0;
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const long long c = (long long)blockIdx.x * kWarps + w;
  double dmax = 0.0;  // largest finite |d_c| of this warp's context
  if (c < p.n_ctx) {
    const long long base = c * p.ctx_len;
    const float* a = p.a + base;
    const float* b = p.b + base;
    const uint8_t* m = p.mask ? p.mask + base : nullptr;
    const int L = p.ctx_len;
    double sa = 0.0, sb = 0.0;
    unsigned cnt = 0;
    // the row's head up to a 16-byte boundary (both rows share the offset),
    // then 16-byte vectors, then the tail
    const int head = (int)((4 - (base & 3)) & 3) < L ? (int)((4 - (base & 3)) & 3) : L;
    if (lane < head) add_pair(a[lane], b[lane], !m || m[lane], sa, sb, cnt);
    const int nvec = (L - head) >> 2;
    const float4* a4 = reinterpret_cast<const float4*>(a + head);
    const float4* b4 = reinterpret_cast<const float4*>(b + head);
    constexpr int U = 2;  // vectors in flight per lane and row
    for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
      float4 va[U], vb[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + 32 * u;
        if (v < nvec) {
          va[u] = __ldcs(a4 + v);
          vb[u] = __ldcs(b4 + v);
        } else {
          va[u] = vb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + 32 * u;
        const bool live = v < nvec;
        const int i = head + 4 * v;
        add_pair(va[u].x, vb[u].x, live && (!m || m[i]), sa, sb, cnt);
        add_pair(va[u].y, vb[u].y, live && (!m || m[i + 1]), sa, sb, cnt);
        add_pair(va[u].z, vb[u].z, live && (!m || m[i + 2]), sa, sb, cnt);
        add_pair(va[u].w, vb[u].w, live && (!m || m[i + 3]), sa, sb, cnt);
      }
    }
    const int tail0 = head + 4 * nvec;
    if (tail0 + lane < L) add_pair(a[tail0 + lane], b[tail0 + lane], !m || m[tail0 + lane], sa, sb, cnt);
    sa = warp_sum(sa);
    sb = warp_sum(sb);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) {
      const double ma = cnt ? sa / (double)cnt : 0.0;
      const double mb = cnt ? sb / (double)cnt : 0.0;
      const double d = ma - mb;
      p.ctx_n[c] = (int32_t)cnt;
      p.ctx_a[c] = ma;
      p.ctx_b[c] = mb;
      p.ctx_d[c] = d;
      if (cnt && fabs(d) <= DBL_MAX) dmax = fabs(d);
    }
  }
  if (lane == 0) wmax[w] = dmax;
  __syncthreads();
  if (threadIdx.x == 0) {
    double mx = wmax[0];
    for (int j = 1; j < kWarps; ++j) mx = fmax(mx, wmax[j]);
    p.blk_max[blockIdx.x] = mx;
  }
}

// Blocks [0, cluster_blocks): one thread per context adds it to its
// cluster.  Every block first finds the largest finite |d_c| (the same in
// every block) and scales d_c so that the sum over all contexts fits 62 bits:
// the fixed-point sums are then exact and independent of the order of the
// atomics.  Block cluster_blocks on: the totals over all counted contexts.
__global__ void __launch_bounds__(kThreads) paired_cluster_kernel(const PairedParams p, int cluster_blocks) {
  wait_prior_grid();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if ((int)blockIdx.x < cluster_blocks) {
    __shared__ double wmax[kWarps];
    double mx = 0.0;
    for (int j = threadIdx.x; j < p.n_ctx_blocks; j += blockDim.x) mx = fmax(mx, p.blk_max[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) wmax[w] = mx;
    __syncthreads();
    mx = wmax[0];
    for (int j = 1; j < kWarps; ++j) mx = fmax(mx, wmax[j]);
    int lg = 0;
    while ((1ll << lg) < p.n_ctx + 1) ++lg;
    // mx = f 2^e with f in [0.5, 1) (e = 0 when mx = 0); units of 2^shift
    // make every |d_c| < 2^(62 - lg), so the n_ctx terms sum to less than
    // 2^62.  Scaling by a power of two (ldexp) is exact at any magnitude.
    int e = 0;
    frexp(mx, &e);
    const int shift = lg - 62 + e;
    if (blockIdx.x == 0 && threadIdx.x == 0) p.tot->shift = shift;
    for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < p.n_ctx;
         c += (long long)cluster_blocks * blockDim.x) {
      const int k = p.cluster[c];
      if (k < 0 || k >= p.n_clusters || p.ctx_n[c] <= 0) continue;  // bad ids are flagged by the totals
      const double d = p.ctx_d[c];
      if (fabs(d) <= DBL_MAX) {
        atomicAdd(reinterpret_cast<unsigned long long*>(p.Dq + k), (unsigned long long)__double2ll_rn(ldexp(d, -shift)));
      } else {
        atomicOr(p.Dflag + k, d != d ? kFlagNaN : (d > 0.0 ? kFlagPosInf : kFlagNegInf));
      }
      atomicAdd(reinterpret_cast<unsigned long long*>(p.Nk + k), 1ull);
    }
    return;
  }
  // totals of one chunk of kTotChunk contexts: per-thread strided sums,
  // then a fixed tree; the finish kernel adds the chunks in order
  const int chunk = blockIdx.x - cluster_blocks;
  const long long c0 = (long long)chunk * kTotChunk;
  const long long c1 = (c0 + kTotChunk < p.n_ctx) ? c0 + kTotChunk : p.n_ctx;
  double sa = 0.0, sb = 0.0, sd = 0.0;
  long long used = 0, pos = 0, al = 0, bl = 0, ties = 0;
  bool bad = false;
  for (long long c = c0 + threadIdx.x; c < c1; c += blockDim.x) {
    const int k = p.cluster[c];
    if (k < 0 || k >= p.n_clusters) {
      bad = true;
      continue;
    }
    const int n = p.ctx_n[c];
    if (n <= 0) continue;
    const double d = p.ctx_d[c];
    pos += n;
    ++used;
    sa += p.ctx_a[c];
    sb += p.ctx_b[c];
    sd += d;
    al += d < 0.0;
    bl += d > 0.0;
    ties += d == 0.0;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) set_dev_status(p.dev_status, 0x2 /* KLD_DEV_BAD_ID */);
  __shared__ PairedPart sh[kWarps];
  sa = warp_sum(sa);
  sb = warp_sum(sb);
  sd = warp_sum(sd);
  used = warp_sum(used);
  pos = warp_sum(pos);
  al = warp_sum(al);
  bl = warp_sum(bl);
  ties = warp_sum(ties);
  if (lane == 0) sh[w] = PairedPart{sa, sb, sd, used, pos, al, bl, ties};
  __syncthreads();
  if (threadIdx.x == 0) {
    PairedPart t = sh[0];
    for (int j = 1; j < kWarps; ++j) {
      t.sa += sh[j].sa;
      t.sb += sh[j].sb;
      t.sd += sh[j].sd;
      t.n_used += sh[j].n_used;
      t.n_pos += sh[j].n_pos;
      t.a_lower += sh[j].a_lower;
      t.b_lower += sh[j].b_lower;
      t.ties += sh[j].ties;
    }
    p.parts[chunk] = t;
  }
}

// D[k] from its fixed-point sum, or the IEEE sum of its non-finite
// differences (NaN when it holds NaN or both infinities).
__device__ __forceinline__ double cluster_sum(const PairedParams& p, int k, int shift) {
  const int f = p.Dflag[k];
  if (f == 0) return ldexp((double)p.Dq[k], shift);
  if ((f & kFlagNaN) || (f & (kFlagPosInf | kFlagNegInf)) == (kFlagPosInf | kFlagNegInf)) return CUDART_NAN;
  return (f & kFlagPosInf) ? CUDART_INF : -CUDART_INF;
}

// One warp per replicate; the clusters' sums sit in shared memory when
// there are at most kBootSmemClusters of them.  Draws are loaded four per
// lane before their sums are gathered.
__global__ void __launch_bounds__(kBootThreads, 2) paired_boot_kernel(const PairedParams p) {
  __shared__ double sD[kBootSmemClusters];
  __shared__ int sN[kBootSmemClusters];  // counts of contexts, < 2^31
  wait_prior_grid();
  const bool staged = p.n_clusters <= kBootSmemClusters;
  const int shift = p.tot->shift;
  if (staged) {
    for (int k = threadIdx.x; k < p.n_clusters; k += blockDim.x) {
      sD[k] = cluster_sum(p, k, shift);
      sN[k] = (int)p.Nk[k];
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  // a fixed grid (one wave); warps stride over the replicates
  const long long n_warps = (long long)gridDim.x * (kBootThreads / 32);
  bool bad = false;
  for (long long r = (long long)blockIdx.x * (kBootThreads / 32) + (threadIdx.x >> 5); r < p.n_boot;
       r += n_warps) {
    const int32_t* draws = p.resample + r * p.n_clusters;
    const int C = p.n_clusters;
    double D = 0.0;
    long long N = 0;
    // the row's draws: up to three before its first 16-byte boundary and up
    // to three after its last one one by one, the rest as 16-byte vectors,
    // kVecRound per lane issued together (one round trip for rows of up to
    // 32 * 4 * kVecRound draws); nothing outside the row is read
    constexpr int kVecRound = 7;
    const int head = min(C, (int)((4 - ((reinterpret_cast<uintptr_t>(draws) >> 2) & 3)) & 3));
    const int nvec = (C - head) >> 2;
    const int tail = C - head - 4 * nvec;
    const int4* dv = reinterpret_cast<const int4*>(draws + head);
    auto take = [&](int k) {
      if (k < 0 || k >= C) {
        bad = true;
        return;
      }
      if (staged) {
        D += sD[k];
        N += sN[k];
      } else {
        D += cluster_sum(p, k, shift);
        N += __ldg(p.Nk + k);
      }
    };
    if (lane < head) take(__ldcs(draws + lane));
    if (lane < tail) take(__ldcs(draws + head + 4 * nvec + lane));
    for (int v0 = lane; v0 < nvec; v0 += 32 * kVecRound) {
      int4 q[kVecRound];
#pragma unroll
      for (int u = 0; u < kVecRound; ++u) {
        const int v = v0 + 32 * u;
        if (v < nvec) q[u] = __ldcs(dv + v);
      }
#pragma unroll
      for (int u = 0; u < kVecRound; ++u) {
        if (v0 + 32 * u >= nvec) continue;
        take(q[u].x);
        take(q[u].y);
        take(q[u].z);
        take(q[u].w);
      }
    }
    D = warp_sum(D);
    N = warp_sum(N);
    if (lane == 0) p.boot[r] = N ? D / (double)N : CUDART_NAN;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_dev_status(p.dev_status, 0x2 /* KLD_DEV_BAD_ID */);
}

// Exact order statistics of the replicate statistics (NaN left out) at the
// target ranks, in one CTA, on order-preserving 64-bit keys of the doubles.
// The keys in [klo, khi] are spread over kBuckets buckets by the monotone
// map (key - klo) * kBuckets / (khi - klo + 1), which puts klo and khi in
// different buckets and divides the key range ~4096-fold; the bucket holding
// the target rank is either small enough to gather into shared memory and
// rank exactly by pairwise counting, or becomes the next [klo, khi] (its own
// least and greatest key).  64-bit keys need at most six such rounds.
constexpr int kSelThreads = 1024;
constexpr int kBuckets = 4096;
constexpr int kGather = 1024;

constexpr int kSelTargets = 2 * KLD_MAX_QUANTILES;

struct SelShared {
  unsigned hist[kBuckets];
  unsigned long long gather[kGather];
  int gather_bucket[kGather];
  unsigned picked[kBuckets / 32];  // buckets gathered by the shared first pass
  unsigned long long rk[2][32];
  unsigned ru[32];
  unsigned long long answer;
  unsigned n_gather, bucket, before;
  unsigned t_bucket[kSelTargets], t_before[kSelTargets];
  unsigned long long t_answer[kSelTargets];
};

__device__ __forceinline__ unsigned long long dkey(double v) {
  unsigned long long u = (unsigned long long)__double_as_longlong(v);
  if (u == 0x8000000000000000ull) u = 0ull;  // -0 sorts with +0
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ double dval(unsigned long long k) {
  const unsigned long long u = (k & 0x8000000000000000ull) ? (k & 0x7fffffffffffffffull) : ~k;
  return __longlong_as_double((long long)u);
}

__device__ __forceinline__ int key_bucket(unsigned long long k, unsigned long long klo, double scale) {
  const int b = (int)((double)(k - klo) * scale);
  return b < kBuckets - 1 ? b : kBuckets - 1;
}

// Block-wide (min, max) of 64-bit keys; returned to every thread.
__device__ void block_key_range(unsigned long long& mn, unsigned long long& mx, SelShared& S) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, mn, off);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, mx, off);
    mn = a < mn ? a : mn;
    mx = b > mx ? b : mx;
  }
  if (lane == 0) {
    S.rk[0][w] = mn;
    S.rk[1][w] = mx;
  }
  __syncthreads();
  mn = S.rk[0][0];
  mx = S.rk[1][0];
  for (int j = 1; j < nw; ++j) {
    mn = S.rk[0][j] < mn ? S.rk[0][j] : mn;
    mx = S.rk[1][j] > mx ? S.rk[1][j] : mx;
  }
  __syncthreads();
}

constexpr int kStageKeys = 20480;  // replicates whose keys the select keeps in shared memory

// Key of replicate i: from shared memory when staged, else recomputed from
// global memory; 0 (no double's key) marks NaN.
struct KeySrc {
  const double* boot;
  const unsigned long long* staged;  // or null
  __device__ __forceinline__ unsigned long long at(long long i) const {
    if (staged) return staged[i];
    const double v = boot[i];
    return (v == v) ? dkey(v) : 0ull;
  }
};

__device__ void finish_warp(const PairedParams& p, int n_parts);

// (its last step writes the result, so no separate launch is needed)
__global__ void __launch_bounds__(kSelThreads) paired_select_kernel(const PairedParams p, int n_parts) {
  __shared__ SelShared S;
  extern __shared__ __align__(16) unsigned long long sk[];  // kStageKeys keys when staged
  wait_prior_grid();
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  const long long B = p.n_boot;
  const bool staged = B <= kStageKeys;
  // the keys (staged), their range and count; loads four at a time
  unsigned long long kmin = ~0ull, kmax = 0ull;
  unsigned cnt = 0u;
  for (long long i0 = tid; i0 < B; i0 += 4 * blockDim.x) {
    double v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long i = i0 + (long long)u * blockDim.x;
      v[u] = (i < B) ? p.boot[i] : CUDART_NAN;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long i = i0 + (long long)u * blockDim.x;
      const unsigned long long k = (v[u] == v[u]) ? dkey(v[u]) : 0ull;
      if (staged && i < B) sk[i] = k;
      if (k) {
        ++cnt;
        kmin = k < kmin ? k : kmin;
        kmax = k > kmax ? k : kmax;
      }
    }
  }
  block_key_range(kmin, kmax, S);  // its barriers also publish sk[]
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) S.ru[w] = cnt;
  __syncthreads();
  long long n = 0;
  for (int j = 0; j < nw; ++j) n += S.ru[j];
  __syncthreads();
  if (tid == 0) p.tot->n_valid = (unsigned)n;
  if (n == 0) {  // no replicate to rank: the result alone
    __syncthreads();
    if (tid < 32) finish_warp(p, n_parts);
    return;
  }
  const KeySrc src{p.boot, staged ? sk : nullptr};
  const int nt = 2 * p.nq;

  // Shared first pass: one histogram over [kmin, kmax] serves every target;
  // the buckets holding the targets' ranks are gathered together while they
  // fit the gather buffer, and each target is ranked inside its bucket.
  // A target whose bucket does not fit runs the narrowing loop below alone.
  unsigned done = 0u;  // targets answered here (the same in every thread)
  if (kmin == kmax) {
    if (tid == 0)
      for (int t = 0; t < nt; ++t) S.t_answer[t] = kmin;
    done = (1u << nt) - 1u;
    __syncthreads();
  } else {
    const double scale = (double)kBuckets / ((double)(kmax - kmin) + 1.0);
    for (int b = tid; b < kBuckets; b += blockDim.x) S.hist[b] = 0u;
    for (int b = tid; b < kBuckets / 32; b += blockDim.x) S.picked[b] = 0u;
    if (tid == 0) S.n_gather = 0u;
    __syncthreads();
    for (long long i = tid; i < B; i += blockDim.x) {
      const unsigned long long k = src.at(i);
      if (k) atomicAdd(&S.hist[key_bucket(k, kmin, scale)], 1u);
    }
    __syncthreads();
    unsigned c4[4], run = 0u;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      c4[q] = S.hist[4 * tid + q];
      run += c4[q];
    }
    unsigned incl = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) S.ru[w] = incl;
    __syncthreads();
    unsigned wbase = 0u;
    for (int j = 0; j < w; ++j) wbase += S.ru[j];
    const long long before_run = (long long)wbase + incl - run;
    for (int t = 0; t < nt; ++t) {
      const long long r = target_rank(p, n, t);
      if (before_run <= r && r < before_run + (long long)run) {
        long long acc = before_run;
        int q = 0;
        while (q < 3 && acc + (long long)c4[q] <= r) acc += c4[q++];
        S.t_bucket[t] = 4 * tid + q;
        S.t_before[t] = (unsigned)acc;
      }
    }
    __syncthreads();
    // which targets' buckets fit together (every thread decides alike)
    unsigned total = 0u;
    for (int t = 0; t < nt; ++t) {
      const unsigned bk = S.t_bucket[t];
      bool seen = false;
      for (int u = 0; u < t; ++u) seen |= ((done >> u) & 1u) && S.t_bucket[u] == bk;
      if (seen) {
        done |= 1u << t;
      } else if (total + S.hist[bk] <= (unsigned)kGather) {
        total += S.hist[bk];
        done |= 1u << t;
        if (tid == 0) S.picked[bk >> 5] |= 1u << (bk & 31);
      }
    }
    __syncthreads();
    if (done) {
      for (long long i = tid; i < B; i += blockDim.x) {
        const unsigned long long k = src.at(i);
        if (!k) continue;
        const int b = key_bucket(k, kmin, scale);
        if ((S.picked[b >> 5] >> (b & 31)) & 1u) {
          const unsigned at = atomicAdd(&S.n_gather, 1u);
          S.gather[at] = k;
          S.gather_bucket[at] = b;
        }
      }
      __syncthreads();
      const int m = (int)S.n_gather;
      for (int t = 0; t < nt; ++t) {
        if (!((done >> t) & 1u)) continue;
        const int bk = (int)S.t_bucket[t];
        const long long rr = target_rank(p, n, t) - (long long)S.t_before[t];  // rank inside the bucket
        for (int g = tid; g < m; g += blockDim.x) {
          if (S.gather_bucket[g] != bk) continue;
          const unsigned long long k = S.gather[g];
          int less = 0, eq = 0;
          for (int j = 0; j < m; ++j) {
            if (S.gather_bucket[j] != bk) continue;
            const unsigned long long u = S.gather[j];
            less += u < k;
            eq += u == k;
          }
          if (less <= rr && rr < less + eq) S.t_answer[t] = k;  // equal keys write the same value
        }
      }
      __syncthreads();
    }
  }

  for (int t = 0; t < nt; ++t) {
    if ((done >> t) & 1u) {
      if (tid == 0) p.tot->ostat[t] = dval(S.t_answer[t]);
      continue;
    }
    long long r = target_rank(p, n, t);  // rank among all non-NaN values
    unsigned long long klo = kmin, khi = kmax;
    unsigned long long ans;
    for (;;) {
      if (klo == khi) {  // one key left
        ans = klo;
        break;
      }
      const double scale = (double)kBuckets / ((double)(khi - klo) + 1.0);
      for (int b = tid; b < kBuckets; b += blockDim.x) S.hist[b] = 0u;
      if (tid == 0) S.n_gather = 0u;
      __syncthreads();
      for (long long i = tid; i < B; i += blockDim.x) {
        const unsigned long long k = src.at(i);
        if (k && k >= klo && k <= khi) atomicAdd(&S.hist[key_bucket(k, klo, scale)], 1u);
      }
      __syncthreads();
      // the bucket holding rank r: every thread sums 4 buckets, a block scan
      // of those sums, and the thread whose run holds r walks it
      unsigned c4[4], run = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        c4[q] = S.hist[4 * tid + q];
        run += c4[q];
      }
      unsigned incl = run;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (lane == 31) S.ru[w] = incl;
      __syncthreads();
      unsigned wbase = 0u;
      for (int j = 0; j < w; ++j) wbase += S.ru[j];
      const long long before_run = (long long)wbase + incl - run;
      if (before_run <= r && r < before_run + (long long)run) {
        long long acc = before_run;
        int q = 0;
        while (q < 3 && acc + (long long)c4[q] <= r) acc += c4[q++];
        S.bucket = 4 * tid + q;
        S.before = (unsigned)acc;
      }
      __syncthreads();
      const int bk = (int)S.bucket;
      const long long rr = r - (long long)S.before;  // rank inside the bucket
      const unsigned in_bucket = S.hist[bk];
      __syncthreads();
      if (in_bucket <= (unsigned)kGather) {
        for (long long i = tid; i < B; i += blockDim.x) {
          const unsigned long long k = src.at(i);
          if (k && k >= klo && k <= khi && key_bucket(k, klo, scale) == bk) S.gather[atomicAdd(&S.n_gather, 1u)] = k;
        }
        __syncthreads();
        const int m = (int)S.n_gather;
        if (tid < m) {
          const unsigned long long k = S.gather[tid];
          int less = 0, eq = 0;
          for (int j = 0; j < m; ++j) {
            const unsigned long long u = S.gather[j];
            less += u < k;
            eq += u == k;
          }
          if (less <= rr && rr < less + eq) S.answer = k;  // equal keys write the same value
        }
        __syncthreads();
        ans = S.answer;
        __syncthreads();
        break;
      }
      // too many: the bucket's own least and greatest key become [klo, khi]
      unsigned long long bmn = ~0ull, bmx = 0ull;
      for (long long i = tid; i < B; i += blockDim.x) {
        const unsigned long long k = src.at(i);
        if (k && k >= klo && k <= khi && key_bucket(k, klo, scale) == bk) {
          bmn = k < bmn ? k : bmn;
          bmx = k > bmx ? k : bmx;
        }
      }
      block_key_range(bmn, bmx, S);
      r = rr;
      klo = bmn;
      khi = bmx;
    }
    if (tid == 0) p.tot->ostat[t] = dval(ans);
    __syncthreads();
  }
  __syncthreads();  // the statistics above are written; one warp writes the result
  if (tid < 32) finish_warp(p, n_parts);
}

// One warp: the chunks' sums (lane l adds chunks l, l + 32, ... in order,
// then a fixed tree), the interval ends, the result.
// The result, written by one warp: the totals' chunks added in order, the
// interval ends from the replicates' order statistics.
__device__ void finish_warp(const PairedParams& p, int n_parts) {
  const int lane = threadIdx.x & 31;
  const PairedTotals* t = p.tot;
  kld_paired* o = p.out;
  const double nan = CUDART_NAN;
  double sa = 0.0, sb = 0.0, sd = 0.0;
  long long used = 0, pos = 0, al = 0, bl = 0, ties = 0;
  for (int j = lane; j < n_parts; j += 32) {
    const PairedPart& q = p.parts[j];
    sa += q.sa;
    sb += q.sb;
    sd += q.sd;
    used += q.n_used;
    pos += q.n_pos;
    al += q.a_lower;
    bl += q.b_lower;
    ties += q.ties;
  }
  sa = warp_sum(sa);
  sb = warp_sum(sb);
  sd = warp_sum(sd);
  used = __shfl_sync(0xffffffffu, warp_sum(used), 0);
  pos = warp_sum(pos);
  al = warp_sum(al);
  bl = warp_sum(bl);
  ties = warp_sum(ties);
  const long long nb = t->n_valid;
  if (lane == 0) {
    o->n_ctx = used;
    o->n_pos = pos;
    o->a_lower = al;
    o->b_lower = bl;
    o->ties = ties;
    o->n_boot = nb;
    o->mean_a = used ? sa / (double)used : nan;
    o->mean_b = used ? sb / (double)used : nan;
    o->diff = used ? sd / (double)used : nan;
    o->nq = p.nq;
    o->pad = 0;
  }
  if (lane < KLD_MAX_QUANTILES) {
    double v = nan;
    if (lane < p.nq && nb > 0) {
      const double lo = t->ostat[2 * lane], hi = t->ostat[2 * lane + 1];
      const double h = __dmul_rn((double)(nb - 1), p.q[lane]);
      const double frac = __dsub_rn(h, floor(h));
      v = __dadd_rn(lo, __dmul_rn(__dsub_rn(hi, lo), frac));
    }
    o->ci[lane] = v;
  }
}

__global__ void paired_finish_kernel(const PairedParams p, int n_parts) {
  wait_prior_grid();
  finish_warp(p, n_parts);
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

size_t paired_workspace_bytes(int64_t n_ctx, int32_t n_clusters, int32_t n_boot) {
  const size_t nc = n_ctx > 0 ? (size_t)n_ctx : 0;
  const size_t k = n_clusters > 0 ? (size_t)n_clusters : 0;
  const size_t b = n_boot > 0 ? (size_t)n_boot : 0;
  const size_t parts = (nc + kTotChunk - 1) / kTotChunk + 1;
  const size_t blocks = (nc + kWarps - 1) / kWarps + 1;
  return align256(sizeof(PairedTotals)) + align256(sizeof(PairedPart) * parts) + 3 * align256(sizeof(double) * nc) +
         align256(sizeof(int32_t) * nc) + align256(sizeof(double) * blocks) + align256(sizeof(long long) * k) +
         align256(sizeof(int32_t) * k) + align256(sizeof(long long) * k) + align256(sizeof(double) * b);
}

cudaError_t launch_paired(const PairedArgs& a, cudaStream_t stream) {
  PairedParams p;
  p.a = a.kl_a;
  p.b = a.kl_b;
  p.mask = a.mask;
  p.n_ctx = a.n_ctx;
  p.ctx_len = a.ctx_len;
  p.cluster = a.cluster;
  p.n_clusters = a.n_clusters;
  p.resample = a.resample;
  p.n_boot = a.n_boot;
  p.nq = a.nq;
  for (int i = 0; i < KLD_MAX_QUANTILES; ++i) p.q[i] = a.quantiles[i];
  p.out = a.out;
  p.dev_status = a.dev_status;
  char* ws = reinterpret_cast<char*>(a.workspace);
  const size_t nc = (size_t)a.n_ctx, k = (size_t)a.n_clusters, b = (size_t)a.n_boot;
  const int n_parts = (int)((nc + kTotChunk - 1) / kTotChunk);
  p.tot = reinterpret_cast<PairedTotals*>(ws);
  ws += align256(sizeof(PairedTotals));
  p.parts = reinterpret_cast<PairedPart*>(ws);
  ws += align256(sizeof(PairedPart) * (size_t)(n_parts + 1));
  p.ctx_a = reinterpret_cast<double*>(ws);
  ws += align256(sizeof(double) * nc);
  p.ctx_b = reinterpret_cast<double*>(ws);
  ws += align256(sizeof(double) * nc);
  p.ctx_d = reinterpret_cast<double*>(ws);
  ws += align256(sizeof(double) * nc);
  p.ctx_n = reinterpret_cast<int32_t*>(ws);
  ws += align256(sizeof(int32_t) * nc);
  const unsigned ctx_grid = (unsigned)((nc + kWarps - 1) / kWarps);
  p.n_ctx_blocks = ctx_grid > 0 ? (int)ctx_grid : 1;
  p.blk_max = reinterpret_cast<double*>(ws);
  ws += align256(sizeof(double) * (size_t)(p.n_ctx_blocks + 1));
  p.Dq = reinterpret_cast<long long*>(ws);
  ws += align256(sizeof(long long) * k);
  p.Dflag = reinterpret_cast<int32_t*>(ws);
  ws += align256(sizeof(int32_t) * k);
  p.Nk = reinterpret_cast<long long*>(ws);
  ws += align256(sizeof(long long) * k);
  p.boot = a.boot_stats ? a.boot_stats : reinterpret_cast<double*>(ws);

  cudaError_t e = cudaSuccess;
  if (ctx_grid > 0) e = launch_dependent(paired_ctx_kernel, dim3(ctx_grid), dim3(kThreads), stream, p);
  else e = launch_dependent(paired_ctx_kernel, dim3(1), dim3(kThreads), stream, p);  // clears the counter
  if (e != cudaSuccess) return e;
  // one thread per context, at most 128 blocks (grid-stride beyond)
  const int cluster_blocks = (int)std::min<size_t>((nc + kThreads - 1) / kThreads, 128) + (nc == 0 ? 1 : 0);
  e = launch_dependent(paired_cluster_kernel, dim3(cluster_blocks + n_parts), dim3(kThreads), stream, p,
                       cluster_blocks);
  if (e != cudaSuccess) return e;
  if (b > 0) {
    constexpr int kBootWarps = kBootThreads / 32;
    // at most two 512-thread CTAs per SM of a 148-SM part: one wave
    const size_t boot_blocks = std::min<size_t>((b + kBootWarps - 1) / kBootWarps, 2 * 148);
    e = launch_dependent(paired_boot_kernel, dim3((unsigned)boot_blocks), dim3(kBootThreads), stream, p);
    if (e != cudaSuccess) return e;
    e = allow_dynamic_smem<paired_select_kernel>(sizeof(unsigned long long) * kStageKeys);
    if (e != cudaSuccess) return e;
    const size_t smem = (b <= (size_t)kStageKeys) ? sizeof(unsigned long long) * b : 0;
    return launch_dependent_smem(paired_select_kernel, dim3(1), dim3(kSelThreads), smem, stream, p, n_parts);
  }
  return launch_dependent(paired_finish_kernel, dim3(1), dim3(32), stream, p, n_parts);
}

}  // namespace kld
