// Sparse capture of a reference distribution from its full logits.
//
// "Qwen3.8-27B Quantization Challenge", "Golden distributions": per scored
// position the reference keeps its K most likely tokens with f32 log p, most
// likely first, and a row (NLL of the true next token, entropy in nats, tail
// mass summed over the rest of the full row).  Equal log-probs keep the lower
// id first.
//
// Three kernels:
//  1. sample (one CTA per row): 4096 elements of the row in evenly spaced
//     runs of four 16-byte vectors (whole DRAM bursts), 16 per thread; the threshold tau is the 25th largest of the 256 thread
//     maxima, at most the sample's own 25th largest, so about 25 / 4096 of
//     the row is at or above it (~1,500 ids at V = 248,320) while the row's
//     top 512 are all above it unless the sample holds 25 of them (mean 8.4
//     for a random layout: about 1e-7).  tau = -inf when the whole row fits
//     the candidate buffer.
//  2. stream (persistent warps over the flattened (row, 16-byte vector)
//     space): elements >= tau are appended, as (value, id), to the row's
//     candidate buffer; every other element feeds the row's tail mass
//     T = sum e^{x - m} and entropy term B = sum e^{x - m} (x - m) with a
//     warp-uniform running maximum m over all elements.  Neither sum ever
//     holds a candidate, so the tail never comes from 1 - sum of the listed
//     masses (which cancels when they hold all but ~1e-6 of the mass).
//  3. finalize (one CTA per row): exact selection of the K largest among
//     the candidates (bitwise radix select on the value bits, then on the ids
//     of the values tied at the boundary), a bitonic sort of the K, and the
//     outputs.  The listed terms are summed in sorted order and the unlisted
//     candidates in fixed point scaled to the K-th weight, so every sum is
//     exact up to rounding and independent of the order candidates arrived
//     in.  A row whose candidates at or above tau are fewer than K, or
//     overflow the buffer, is redone exactly from the full row by the same
//     CTA (every element a candidate).
#include <cuda_bf16.h>
#include <cfloat>

#include "kld_common.cuh"
#include "launch.h"
#include "stream_common.cuh"

namespace kld {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kVecs = 4;                      // 16-byte vectors per lane per step
constexpr int kStepVecs = 32 * kVecs;
constexpr int kMinVecsPerWarp = 4 * kStepVecs;
constexpr int kStreamCtasPerSm = 3;
constexpr int kMaxStreamWarps = 148 * kStreamCtasPerSm * kWarpsPerCta;
constexpr int kSampleElems = 4096;
constexpr int kSampleRank = 25;
constexpr int kCap = KLD_CAPTURE_CANDIDATES;  // candidates kept per row
constexpr int kFinThreads = 128;     // finish: one CTA per row, 8 rows per SM
constexpr int kSampleThreads = 256;  // sample: 16 sampled values per thread
constexpr int kMaxK = KLD_SPARSE_MAX_K;
constexpr int kStage = 2048;  // candidates a finish CTA keeps in shared memory
constexpr int kTieCap = 256;  // values tied at the K-th that are ranked by counting

// Tail state of one warp over one row piece (16 bytes): running maximum m
// over all elements, and over the non-candidates T = sum e^{x-m},
// B = sum e^{x-m} (x - m).
struct CapPiece {
  float m, T, B;
  int pad;
};

struct CapParams {
  const void* x;
  int64_t ld;          // elements
  int vocab, nvec, n_rows, nwarps;
  int64_t total;       // n_rows * nvec
  int K;
  const int32_t* targets;
  float* tau;          // [n_rows]
  int* count;          // [n_rows] candidates appended (may exceed kCap)
  int2* cand;          // [n_rows][kCap] (f32 value bits, id)
  CapPiece* pieces;    // slot row + warp
  kld_top_entry* top;  // [n_rows, K]
  float* rows;         // [n_rows, 3] NLL, entropy, tail
  int32_t* dev_status;
  int force_exact;     // tests only: every row takes the exact path
};

// Per-warp shared memory of the stream: the 16-byte vectors that hold
// candidates, with their vector index in the row, gathered until the ring
// is full and then unpacked together.
constexpr int kRing = 256;
struct CapRing {
  uint4 vec[kRing];
  int vid[kRing];
};

// Append the elements >= tau of the ring's `fill` vectors to the row's
// candidate buffer.  Lane l takes ring entries l, l + 32, ...: it counts
// their candidates first, one warp scan of those counts gives every lane its
// place, and one atomic reserves the whole flush (the order of a row's
// candidates in the buffer does not matter).
template <bool kBF16>
__device__ void ring_flush(const CapParams& p, CapRing& R, int fill, int row, float tau, int lane) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  constexpr int kGroups = kRing / 32;
  int2* cand = p.cand + (int64_t)row * kCap;
  __syncwarp();
  uint32_t em[kGroups];
  int mine = 0;
#pragma unroll
  for (int g = 0; g < kGroups; ++g) {
    em[g] = 0u;
    const int j = g * 32 + lane;
    if (j < fill) {
      const uint4 v = R.vec[j];
#pragma unroll
      for (int k = 0; k < E / 2; ++k) {
        const float2 pr = El::pair(v, k);
        em[g] |= (pr.x >= tau) ? (1u << (2 * k)) : 0u;
        em[g] |= (pr.y >= tau) ? (1u << (2 * k + 1)) : 0u;
      }
      mine += __popc(em[g]);
    }
  }
  int incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const int tot = __shfl_sync(0xffffffffu, incl, 31);
  int base = 0;
  if (lane == 0 && tot > 0) base = atomicAdd(p.count + row, tot);
  int pos = __shfl_sync(0xffffffffu, base, 0) + incl - mine;
#pragma unroll
  for (int g = 0; g < kGroups; ++g) {
    uint32_t m = em[g];
    if (m == 0u) continue;
    const int j = g * 32 + lane;
    const uint4 v = R.vec[j];
    const int vid = R.vid[j];
    while (m) {
      const int e = __ffs(m) - 1;
      m &= m - 1u;
      const float2 pr = El::pair(v, e >> 1);
      if (pos < kCap) cand[pos] = make_int2(__float_as_int((e & 1) ? pr.y : pr.x), vid * E + e);
      ++pos;
    }
  }
  __syncwarp();
}

// 2. stream vectors [a, b) of one row; returns the piece's tail state
// (identical in every lane) and appends the piece's candidates.
// 1.0f when a >= b, else 0.0f (NaN compares false).
__device__ __forceinline__ float set_ge(float a, float b) {
  float r;
  asm("set.ge.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Both bf16 halves of w raised to at least the lowest finite bf16; NaN stays.
__device__ __forceinline__ uint32_t bf16x2_floor(uint32_t w) {
  uint32_t r;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(0xff7fff7fu));
  return r;
}

// Both bf16 halves of w that are >= the bf16 halves of tau2 moved down by
// the lowest finite bf16 (1.0 or 0.0 per half from the compare, then one
// fused multiply-add); the others unchanged.
__device__ __forceinline__ uint32_t bf16x2_mask_ge(uint32_t w, uint32_t tau2) {
  uint32_t s, r;
  asm("set.ge.bf16x2.bf16x2 %0, %1, %2;" : "=r"(s) : "r"(w), "r"(tau2));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(s), "r"(0xff7fff7fu), "r"(w));
  return r;
}

// Shift that takes a candidate's exponent far below any real one: its
// weight underflows to exactly 0.
constexpr float kMaskShift = 1e30f;

template <bool kBF16>
__device__ CapPiece cap_piece(const CapParams& p, CapRing& R, int row, int a, int b, int lane, float tau) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  constexpr int kElemBytes = kBF16 ? 2 : 4;
  constexpr uint32_t kNegInfWord = kBF16 ? 0xff80ff80u : 0xff800000u;
  const uint4 neg_inf = make_uint4(kNegInfWord, kNegInfWord, kNegInfWord, kNegInfWord);
  const char* yl = reinterpret_cast<const char*>(p.x) + (int64_t)row * p.ld * kElemBytes + (int64_t)(a + lane) * 16;
  int fill = 0;  // vectors in the ring (warp-uniform)

  float m = -CUDART_INF_F;  // warp-uniform
  float2 T2 = make_float2(0.f, 0.f), B2 = T2;
  const int n = b - a;
  const int nsteps = (n + kStepVecs - 1) / kStepVecs;
  auto load_step = [&](int st, uint4 (&v)[kVecs]) {
    const int64_t o = (int64_t)st * kStepVecs * 16;
    if ((st + 1) * kStepVecs <= n) {
#pragma unroll
      for (int q = 0; q < kVecs; ++q) v[q] = ld_stream(yl + o + q * 32 * 16);
    } else {
#pragma unroll
      for (int q = 0; q < kVecs; ++q)
        v[q] = (st * kStepVecs + lane + 32 * q < n) ? ld_stream(yl + o + q * 32 * 16) : neg_inf;
    }
  };
  uint4 nx[kVecs];
  if (nsteps > 0) load_step(0, nx);
  for (int st = 0; st < nsteps; ++st) {
    uint4 v[kVecs];
#pragma unroll
    for (int q = 0; q < kVecs; ++q) v[q] = nx[q];
    if (st + 1 < nsteps) load_step(st + 1, nx);

    float c[kVecs];
    float cm = -CUDART_INF_F;
#pragma unroll
    for (int q = 0; q < kVecs; ++q) {
      c[q] = El::vmax(v[q]);
      cm = fmaxf(cm, c[q]);
    }
    const float CM = warp_max(cm);
    if (CM > m) {  // warp-uniform: a new maximum; rescale both sums to it
      float T = T2.x + T2.y, B = B2.x + B2.y;
      if (m != -CUDART_INF_F) {  // else nothing finite yet: the sums hold 0, or NaN, and stay
        const float sc = ex2((m - CM) * kLog2e);
        B = sc * (B + (m - CM) * T);
        T = sc * T;
      }
      T2 = make_float2(T, 0.f);
      B2 = make_float2(B, 0.f);
      m = CM;
    }

    // candidates: vectors that reach tau go to the warp's ring
    unsigned hitq = 0u;
#pragma unroll
    for (int q = 0; q < kVecs; ++q) hitq |= (c[q] >= tau) ? (1u << q) : 0u;
    const unsigned hm = __ballot_sync(0xffffffffu, hitq != 0u);
    if (hm) {
      // a lane's place in the ring: with at most one hit per lane (the
      // usual case) the count of hitting lanes below it, else a warp scan
      const int nh = __popc(hitq);
      int before, tot;
      if (!__any_sync(0xffffffffu, nh > 1)) {
        before = __popc(hm & ((1u << lane) - 1u));
        tot = __popc(hm);
      } else {
        int incl = nh;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int o = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += o;
        }
        before = incl - nh;
        tot = __shfl_sync(0xffffffffu, incl, 31);
      }
      if (fill + tot > kRing) {
        ring_flush<kBF16>(p, R, fill, row, tau, lane);
        fill = 0;
      }
      int pos = fill + before;
#pragma unroll
      for (int q = 0; q < kVecs; ++q) {
        if ((hitq >> q) & 1u) {
          R.vec[pos] = v[q];
          R.vid[pos] = a + st * kStepVecs + lane + 32 * q;
          ++pos;
        }
      }
      fill += tot;
    }

    // tail and entropy sums over the non-candidates; a row with no finite
    // value yet has only -inf (weight 0) or NaN (poisons T), so any finite
    // offset serves
    const float mo = (m == -CUDART_INF_F) ? 0.f : m;
    const float2 nm = make_float2(-mo, -mo);
    const float2 l2 = make_float2(kLog2e, kLog2e);
    const float2 shove = make_float2(-kMaskShift, -kMaskShift);
    const uint32_t tau2 = kBF16 ? ((__float_as_uint(tau) >> 16) * 0x10001u) : 0u;  // tau is a bf16 value
#pragma unroll
    for (int q = 0; q < kVecs; ++q) {
      uint4 u = v[q];
      if constexpr (kBF16) {
        // a candidate (>= tau) is moved down by the lowest bf16, far below
        // any maximum (weight 0); then whatever is -inf (a -inf logit, or a
        // negative candidate moved past the lowest) is raised to the lowest
        // finite bf16 (NaN kept), so d below is finite and w * d never
        // forms 0 * inf
        u.x = bf16x2_floor(bf16x2_mask_ge(u.x, tau2));
        u.y = bf16x2_floor(bf16x2_mask_ge(u.y, tau2));
        u.z = bf16x2_floor(bf16x2_mask_ge(u.z, tau2));
        u.w = bf16x2_floor(bf16x2_mask_ge(u.w, tau2));
      }
#pragma unroll
      for (int k = 0; k < E / 2; ++k) {
        const float2 X = El::pair(u, k);
        float2 d = __fadd2_rn(X, nm);
        float2 t;
        if constexpr (kBF16) {
          t = __fmul2_rn(d, l2);
        } else {
          // a candidate (X >= tau) is pushed far below the maximum: weight 0
          const float2 c = make_float2(set_ge(X.x, tau), set_ge(X.y, tau));
          t = __fmul2_rn(__ffma2_rn(c, shove, d), l2);
        }
        const float2 w = make_float2(ex2(t.x), ex2(t.y));
        T2 = __fadd2_rn(T2, w);
        if constexpr (!kBF16) {
          d.x = fmaxf(d.x, -FLT_MAX);
          d.y = fmaxf(d.y, -FLT_MAX);
        }
        B2 = __ffma2_rn(w, d, B2);
      }
    }
  }
  if (fill > 0) ring_flush<kBF16>(p, R, fill, row, tau, lane);
  float T = T2.x + T2.y, B = B2.x + B2.y;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    T += __shfl_xor_sync(0xffffffffu, T, off);
    B += __shfl_xor_sync(0xffffffffu, B, off);
  }
  return CapPiece{m, T, B, 0};
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads, kStreamCtasPerSm) cap_stream_kernel(const CapParams p) {
  __shared__ CapRing rings[kWarpsPerCta];
  wait_prior_grid();
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (w >= p.nwarps) return;  // the whole warp leaves together
  int64_t pos = warp_begin(w, p.total, p.nwarps);
  const int64_t end = warp_begin(w + 1, p.total, p.nwarps);
  while (pos < end) {
    const int row = (int)(pos / p.nvec);
    const int64_t row0 = (int64_t)row * p.nvec;
    const int a = (int)(pos - row0);
    const int b = (int)min((int64_t)p.nvec, end - row0);
    const CapPiece pc = cap_piece<kBF16>(p, rings[threadIdx.x >> 5], row, a, b, lane, p.tau[row]);
    if (lane == 0) p.pieces[row + w] = pc;
    pos = row0 + b;
  }
}

// ---------------------------------------------------------------- finalize

// Order-preserving 32-bit key of a non-NaN f32 value (-0 sorts with +0).
__device__ __forceinline__ uint32_t vkey(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float keyv(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Block sums in a fixed order (butterfly in each warp, then the warp totals
// in warp order): every thread gets the same, reproducible result.
template <typename T>
__device__ T block_sum(T v, T* sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  T t = sh[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i) t += sh[i];
  return t;
}

__device__ float block_max(float v, float* sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  float t = sh[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i) t = fmaxf(t, sh[i]);
  return t;
}

// Merge of two pieces' tail states (the larger maximum wins; a side that has
// seen nothing finite holds 0 or NaN and is added as it is).
__device__ __forceinline__ CapPiece piece_merge(const CapPiece& a, const CapPiece& b) {
  const float M = fmaxf(a.m, b.m);
  float T = 0.f, B = 0.f;
  if (a.m == -CUDART_INF_F || M == -CUDART_INF_F) {
    T += a.T;
    B += a.B;
  } else {
    const float s = ex2((a.m - M) * kLog2e);
    T += s * a.T;
    B += s * (a.B + (a.m - M) * a.T);
  }
  if (b.m == -CUDART_INF_F || M == -CUDART_INF_F) {
    T += b.T;
    B += b.B;
  } else {
    const float s = ex2((b.m - M) * kLog2e);
    T += s * b.T;
    B += s * (b.B + (b.m - M) * b.T);
  }
  return CapPiece{M, T, B, 0};
}

// Candidates: the row's streamed ones in its global buffer (read through
// L1 on every pass), then the few of the row's ragged end, in shared memory.
struct BufCands {
  const int2* cand;
  int ns;
  const float* rv;
  const int* ri;
  int n;
  __device__ __forceinline__ float val(int i) const {
    return i < ns ? __int_as_float(__ldg(&cand[i].x)) : rv[i - ns];
  }
  __device__ __forceinline__ int idx(int i) const { return i < ns ? __ldg(&cand[i].y) : ri[i - ns]; }
};

// A row's candidates staged in shared memory (most rows: the finish
// reads every candidate on each of its passes).
struct SmemCands {
  const float* v;
  const int* id;
  int n;
  __device__ __forceinline__ float val(int i) const { return v[i]; }
  __device__ __forceinline__ int idx(int i) const { return id[i]; }
};

// Every element of a row, read from global memory (the exact path).
template <bool kBF16>
struct RowCands {
  const void* row;
  int n;
  __device__ __forceinline__ float val(int i) const { return Elems<kBF16>::load1(row, i); }
  __device__ __forceinline__ int idx(int i) const { return i; }
};

struct FinScratch {  // block-reduction slots for up to 8 warps
  double d[8];
  long long ll[8];
  int i[8];
  float f[8];
  int n_sel;
  unsigned hist[256];
  unsigned digit, rank, eq;
};

// The r-th largest (1-based) of the 32-bit keys of the elements i < n for
// which key(i, k) returns true: an MSB-first radix select, 8 bits per pass,
// with shared-memory histograms (plain atomics: measured faster here than
// aggregating equal digits with __match_any_sync).  Returns the key; eq =
// elements equal to it, rank = its
// rank among them (eq - rank of the equal keys come after position r); rank
// is 0 when fewer than r elements take part.
// Every thread of the CTA calls this.
// kLowBits: the keys' low kLowBits bits are fixed by the sign bit (all 0 for
// a positive value, all 1 for a negative one), as for the key of a bf16 value
// widened to f32; the passes over them, which would put every remaining
// element into one bin, are skipped and the bits filled in.
template <int kLowBits, class KeyFn>
__device__ uint32_t rth_largest(int n, int r, KeyFn key, FinScratch& sc, int& eq, int& rank) {
  static_assert(kLowBits == 0 || kLowBits == 16, "whole 8-bit digits, the sign digit always scanned");
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0u, pmask = 0u;
  for (int shift = 24; shift >= kLowBits; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) sc.hist[b] = 0u;
    __syncthreads();
    for (int i0 = threadIdx.x & ~31; i0 < n; i0 += blockDim.x) {  // warp-uniform trip count
      const int i = i0 + lane;
      uint32_t k = 0u;
      const bool ok = i < n && key(i, k) && (k & pmask) == prefix;
      const unsigned digit = ok ? ((k >> shift) & 255u) : 256u;
      if (ok) atomicAdd(&sc.hist[digit], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l holds bins 255 - 8l .. 248 - 8l (descending); scan from the top
      unsigned c[8], run = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = sc.hist[255 - 8 * lane - j];
        run += c[j];
      }
      unsigned incl = run;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const unsigned base = incl - run;
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= (unsigned)r && base < (unsigned)r);
      if (hit == 0u && lane == 0) {  // fewer than r keys: report rank 0
        sc.digit = 0u;
        sc.rank = 0u;
        sc.eq = 0u;
      }
      if (lane == __ffs(hit) - 1) {
        unsigned before = base, j = 0u, cj = 0u;
        bool found = false;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          if (!found && before + c[jj] >= (unsigned)r) {
            found = true;
            j = (unsigned)jj;
            cj = c[jj];
          } else if (!found) {
            before += c[jj];
          }
        }
        sc.digit = 255u - 8u * lane - j;
        sc.rank = (unsigned)r - before;
        sc.eq = cj;
      }
    }
    __syncthreads();
    prefix |= sc.digit << shift;
    pmask |= 255u << shift;
    r = (int)sc.rank;
  }
  if (kLowBits > 0 && r > 0 && !(prefix & 0x80000000u)) prefix |= (1u << kLowBits) - 1u;
  eq = (int)sc.eq;
  rank = r;
  return prefix;
}

// Sort P = 128 R keys of sel[] descending with the finish CTA's 128
// threads: a bitonic network on registers.  Thread t holds elements
// t R .. t R + R - 1; partners closer than R are in the same thread, up to
// 32 R apart in the same warp (shuffles), farther in another warp (shared
// memory, the only stages with a barrier).
// One stage of partners J < R apart inside a thread (J fixed at compile
// time so the registers are addressed statically).
template <int R, int J, typename Key>
__device__ __forceinline__ void local_stage(Key (&a)[R], int t, int kk) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if ((r ^ J) > r) {
      const bool desc = ((t * R + r) & kk) == 0;
      const Key x = a[r], y = a[r ^ J];
      const bool sw = desc ? (x < y) : (x > y);
      a[r] = sw ? y : x;
      a[r ^ J] = sw ? x : y;
    }
  }
}

template <int R, typename Key>
__device__ void sort_desc(Key* sel) {
  const int t = threadIdx.x;
  Key a[R];
#pragma unroll
  for (int r = 0; r < R; ++r) a[r] = sel[t * R + r];
  constexpr int P = kFinThreads * R;
  for (int kk = 2; kk <= P; kk <<= 1) {
    for (int jj = kk >> 1; jj > 0; jj >>= 1) {
      if (jj < R) {
        if (jj == 1) local_stage<R, 1, Key>(a, t, kk);
        else if (jj == 2) local_stage<R, (R > 2 ? 2 : 1), Key>(a, t, kk);
        else local_stage<R, (R > 4 ? 4 : 1), Key>(a, t, kk);
      } else if (jj / R < 32) {
        const int tm = jj / R;
        const bool lower = (t & tm) == 0;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const Key o = __shfl_xor_sync(0xffffffffu, a[r], tm);
          const bool desc = ((t * R + r) & kk) == 0;
          const Key hi = a[r] > o ? a[r] : o, lo = a[r] > o ? o : a[r];
          a[r] = (lower == desc) ? hi : lo;
        }
      } else {
        const int tm = jj / R;
        const bool lower = (t & tm) == 0;
        __syncthreads();
#pragma unroll
        for (int r = 0; r < R; ++r) sel[t * R + r] = a[r];
        __syncthreads();
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const Key o = sel[(t ^ tm) * R + r];
          const bool desc = ((t * R + r) & kk) == 0;
          const Key hi = a[r] > o ? a[r] : o, lo = a[r] > o ? o : a[r];
          a[r] = (lower == desc) ? hi : lo;
        }
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) sel[t * R + r] = a[r];
  __syncthreads();
}

// 1. one CTA per row: tau = the kSampleRank-th largest of kSampleElems
// evenly spaced elements (counted with multiplicity); also clears the row's
// candidate count.
template <bool kBF16>
__global__ void __launch_bounds__(kSampleThreads) cap_sample_kernel(const CapParams p) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  constexpr int kSampleVecs = kSampleElems / E;  // 512 (bf16) or 1024 (f32)
  __shared__ float tmax[kSampleThreads];
  __shared__ FinScratch sc;
  wait_prior_grid();
  const int row = blockIdx.x;
  if (threadIdx.x == 0) p.count[row] = 0;
  if ((int64_t)p.nvec * E <= kCap || p.nvec < kSampleVecs) {
    if (threadIdx.x == 0) p.tau[row] = -CUDART_INF_F;  // every element fits the buffer
    return;
  }
  const char* xrow = reinterpret_cast<const char*>(p.x) + (int64_t)row * p.ld * (kBF16 ? 2 : 4);
  // each thread keeps the largest of its sampled values; the kSampleRank-th
  // largest of those maxima is at most the sample's own kSampleRank-th
  // largest (a subset's), so tau only errs low: more candidates, never fewer
  float mx = -CUDART_INF_F;
  // the sample is kSampleVecs / 4 runs of 4 vectors (64 bytes, 64-byte
  // aligned), evenly spaced: whole DRAM bursts rather than 16 bytes of each
  constexpr int kRuns = kSampleVecs / 4;
  for (int s = threadIdx.x; s < kSampleVecs; s += kSampleThreads) {
    const int64_t run0 = (((int64_t)(s >> 2) * p.nvec) / kRuns) & ~int64_t(3);
    const int64_t vec = run0 + (s & 3);
    mx = fmaxf(mx, El::vmax(*reinterpret_cast<const uint4*>(xrow + vec * 16)));
  }
  tmax[threadIdx.x] = mx;
  __syncthreads();
  int eq = 0, rank = 0;
  const uint32_t kk = rth_largest<kBF16 ? 16 : 0>(kSampleThreads, kSampleRank, [&](int i, uint32_t& k) {
    const float v = tmax[i];
    k = vkey(v);
    return v == v;  // NaN (an invalid row) takes no part
  }, sc, eq, rank);
  // too few sampled values to rank (NaN): every element becomes a candidate,
  // which sends the row down the exact path
  if (threadIdx.x == 0) p.tau[row] = rank > 0 ? keyv(kk) : -CUDART_INF_F;
}

// The outputs of one row from its candidates `src` and, on the streaming
// path, the tail state (mT, T, B) of every element that is not a candidate
// (mT = -inf and T = B = 0 when every element is a candidate).  Every
// thread of the CTA calls this.
template <bool kBF16, class Src>
__device__ void capture_finish(const CapParams& p, int row, const Src& src, float mT, float T, float B,
                               unsigned long long* sel, FinScratch& sc) {
  const int tid = threadIdx.x;
  const int K = p.K;
  const int n = src.n;
  const char* xrow = reinterpret_cast<const char*>(p.x) + (int64_t)row * p.ld * (kBF16 ? 2 : 4);
  kld_top_entry* top = p.top + (int64_t)row * K;
  float* out = p.rows + (int64_t)row * 3;

  // the row's maximum; NaN or +inf anywhere makes the row invalid
  float lm = -CUDART_INF_F;
  int bad = 0;
  for (int i = tid; i < n; i += kFinThreads) {
    const float v = src.val(i);
    bad |= (v != v) || (v == CUDART_INF_F);
    lm = fmaxf(lm, v);
  }
  bad = __syncthreads_or(bad);
  const float m = fmaxf(block_max(lm, sc.f), mT);
  if (bad || T != T || B != B || !(m > -CUDART_INF_F) || m == CUDART_INF_F) {
    for (int j = tid; j < K; j += kFinThreads) top[j] = kld_top_entry{-1, CUDART_NAN_F};
    if (tid == 0) {
      out[0] = out[1] = out[2] = CUDART_NAN_F;
      if (p.targets) {
        const int t = p.targets[row];
        if (t < 0 || t >= p.vocab) set_dev_status(p.dev_status, 0x1 /* KLD_DEV_BAD_TARGET */);
      }
    }
    return;
  }

  // the K-th largest value, and which of the values tied with it join
  // (the lowest ids first): pre, then ids up to id_cut among the ties
  int eq = 0, need = 0;
  const uint32_t pre = rth_largest<kBF16 ? 16 : 0>(n, K, [&](int i, uint32_t& k) {
    k = vkey(src.val(i));
    return true;
  }, sc, eq, need);
  uint32_t id_cut = 0xffffffffu;
  if (need < eq && eq <= kTieCap) {
    // the usual case: a few values tied at the K-th.  Collect their ids
    // (sel is free until the gather below) and take the need-th lowest by
    // counting, for each, the tied ids below it (ids are distinct)
    uint32_t* ties = reinterpret_cast<uint32_t*>(sel);
    if (tid == 0) sc.n_sel = 0;
    __syncthreads();
    for (int i0 = tid & ~31; i0 < n; i0 += kFinThreads) {  // warp-uniform: one reservation per warp
      const int i = i0 + (tid & 31);
      const bool tie = i < n && vkey(src.val(i)) == pre;
      const unsigned tb = __ballot_sync(0xffffffffu, tie);
      int base = 0;
      if ((tid & 31) == 0 && tb) base = atomicAdd(&sc.n_sel, __popc(tb));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (tie) ties[base + __popc(tb & ((1u << (tid & 31)) - 1u))] = (uint32_t)src.idx(i);
    }
    __syncthreads();
    for (int t = tid; t < eq; t += kFinThreads) {
      const uint32_t id = ties[t];
      int below = 0;
      for (int u = 0; u < eq; ++u) below += ties[u] < id ? 1 : 0;
      if (below == need - 1) sc.digit = id;  // exactly one tied id has this rank
    }
    __syncthreads();
    id_cut = sc.digit;
    __syncthreads();  // sc and sel are reused below
  } else if (need < eq) {
    int eq2 = 0, r2 = 0;
    id_cut = ~rth_largest<0>(n, need, [&](int i, uint32_t& k) {
      k = ~(uint32_t)src.idx(i);
      return vkey(src.val(i)) == pre;
    }, sc, eq2, r2);
  }

  // gather the K selected as descending-sortable keys and sort them.  For
  // bf16 values the key's low 16 bits are fixed by its sign, so a 32-bit
  // sort key holds the value's top 16 key bits over 0xffff - gather slot,
  // and the ids stay in a table by gather slot; values tied in the sorted
  // order are put in id order when the outputs are written.  For f32 values
  // the keys are 64-bit: value key over ~id.
  uint32_t* sel32 = reinterpret_cast<uint32_t*>(sel);  // [P] keys (bf16)
  uint32_t* slot_id = sel32 + kMaxK;                    // [K] ids by gather slot (bf16)
  if (tid == 0) sc.n_sel = 0;
  int P = kFinThreads;
  while (P < K) P <<= 1;
  for (int j = K + tid; j < P; j += kFinThreads) {
    if constexpr (kBF16) sel32[j] = 0u;  // below every real key: its low half is at least 0xfc00
    else sel[j] = 0ull;
  }
  __syncthreads();
  for (int i0 = tid & ~31; i0 < n; i0 += kFinThreads) {  // warp-uniform: one slot reservation per warp
    const int i = i0 + (tid & 31);
    uint32_t k = 0u, id = 0u;
    bool take = false;
    if (i < n) {
      k = vkey(src.val(i));
      id = (uint32_t)src.idx(i);
      take = k > pre || (k == pre && id <= id_cut);
    }
    const unsigned takers = __ballot_sync(0xffffffffu, take);
    int base = 0;
    if ((tid & 31) == 0 && takers) base = atomicAdd(&sc.n_sel, __popc(takers));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (take) {
      const int at = base + __popc(takers & ((1u << (tid & 31)) - 1u));
      if (at < K) {
        if constexpr (kBF16) {
          sel32[at] = (k & 0xffff0000u) | (0xffffu - (uint32_t)at);
          slot_id[at] = id;
        } else {
          sel[at] = ((unsigned long long)k << 32) | (unsigned long long)(~id);
        }
      }
    }
  }
  __syncthreads();
  // sort, descending: P = 128 R >= K slots (the padding keys are 0)
  if constexpr (kBF16) {
    if (P <= kFinThreads) sort_desc<1>(sel32);
    else if (P <= 2 * kFinThreads) sort_desc<2>(sel32);
    else if (P <= 4 * kFinThreads) sort_desc<4>(sel32);
    else sort_desc<8>(sel32);
  } else {
    if (P <= kFinThreads) sort_desc<1>(sel);
    else if (P <= 2 * kFinThreads) sort_desc<2>(sel);
    else if (P <= 4 * kFinThreads) sort_desc<4>(sel);
    else sort_desc<8>(sel);
  }
  // the 32-bit value key at sorted position j
  const auto key_at = [&](int j) -> uint32_t {
    if constexpr (kBF16) {
      const uint32_t hi = sel32[j] & 0xffff0000u;
      return (hi & 0x80000000u) ? hi : (hi | 0xffffu);  // a negative value's low key bits are all ones
    } else {
      return (uint32_t)(sel[j] >> 32);
    }
  };

  // listed terms in sorted order (a fixed share per thread): the largest
  // has weight exactly 1 and is left out of s1 so that log S = log1p(S - 1).
  // Weights are ex2 on the MUFU unit (relative error ~1e-7), sums f64.
  const double md = (double)m;
  double s1 = 0.0, b1 = 0.0;
  for (int j = tid; j < K; j += kFinThreads) {
    const float d = keyv(key_at(j)) - m;
    const float w = ex2(d * kLog2e);
    if (j > 0) s1 += (double)w;
    if (w > 0.f) b1 += (double)w * (double)d;
  }
  s1 = block_sum(s1, sc.d);
  b1 = block_sum(b1, sc.d);

  // candidates left out of the list: every one weighs at most the K-th
  // weight wK, so their sums go to 64-bit fixed point scaled to that bound
  // (exact integer sums: the order candidates arrived in does not matter)
  // (the K-th listed value is pre; the listed ids tied with it are those up to id_cut)
  const uint32_t kkey = pre, kid = id_cut;
  const float dKf = keyv(kkey) - m;
  const double dK = (double)dKf;
  const double wK = (double)ex2(dKf * kLog2e);
  double s_ns = 0.0, b_ns = 0.0;
  if (wK > 0.0 && n > K) {
    int lg = 0;
    while ((1 << lg) < n + 1) ++lg;
    const double unit = ldexp(1.0, 62 - lg);                    // n * unit < 2^62
    const double bw = (dK <= -1.0) ? wK * -dK : exp(-1.0);    // max of w |d| over d <= dK
    const double to_w = unit / wK, to_b = unit / bw;
    long long aw = 0, ab = 0;
    for (int i = tid; i < n; i += kFinThreads) {
      const float v = src.val(i);
      const uint32_t k = vkey(v);
      const uint32_t id = (uint32_t)src.idx(i);
      if (k > kkey || (k == kkey && id <= kid)) continue;       // listed
      const float df = v - m;
      const float wf = ex2(df * kLog2e);
      if (wf > 0.f) {
        const double w = (double)wf;
        aw += __double2ll_rn(w * to_w);
        ab += __double2ll_rn(w * -(double)df * to_b);
      }
    }
    aw = block_sum(aw, sc.ll);
    ab = block_sum(ab, sc.ll);
    s_ns = (double)aw / unit * wK;
    b_ns = -(double)ab / unit * bw;
  }

  // the streamed tail, moved to the row's maximum
  double Ts = 0.0, Bs = 0.0;
  if (mT == -CUDART_INF_F) {
    Ts = (double)T;
    Bs = (double)B;
  } else {
    const double e = exp((double)mT - md);
    Ts = e * (double)T;
    Bs = e * ((double)B + ((double)mT - md) * (double)T);
  }
  const double s_minus_1 = s1 + s_ns + Ts;
  const double logS = log1p(s_minus_1);
  const double S = 1.0 + s_minus_1;

  for (int j = tid; j < K; j += kFinThreads) {
    const double v = (double)keyv(key_at(j));
    if constexpr (kBF16) {
      // position j holds one of a run of equal values in gather order: the
      // run's ids go out ascending
      const uint32_t e = sel32[j], v16 = e >> 16;
      const uint32_t id = slot_id[0xffffu - (e & 0xffffu)];
      int lo = j, hi = j + 1;
      while (lo > 0 && (sel32[lo - 1] >> 16) == v16) --lo;
      while (hi < K && (sel32[hi] >> 16) == v16) ++hi;
      int at = lo;
      for (int u = lo; u < hi; ++u) at += slot_id[0xffffu - (sel32[u] & 0xffffu)] < id ? 1 : 0;
      top[at] = kld_top_entry{(int32_t)id, (float)((v - md) - logS)};
    } else {
      top[j] = kld_top_entry{(int32_t)(~(uint32_t)sel[j]), (float)((v - md) - logS)};
    }
  }
  if (tid == 0) {
    float nll = CUDART_NAN_F;
    if (p.targets) {
      const int t = p.targets[row];
      if (t >= 0 && t < p.vocab) nll = (float)(logS - ((double)Elems<kBF16>::load1(xrow, t) - md));
      else set_dev_status(p.dev_status, 0x1 /* KLD_DEV_BAD_TARGET */);
    }
    out[0] = nll;
    out[1] = (float)(logS - (b1 + b_ns + Bs) / S);
    out[2] = (float)((s_ns + Ts) / S);
  }
}

// 3. one CTA per row.
template <bool kBF16>
__global__ void __launch_bounds__(kFinThreads, 8) cap_finalize_kernel(const CapParams p) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  __shared__ unsigned long long sel[kMaxK];
  __shared__ FinScratch sc;
  __shared__ CapPiece merged;
  __shared__ float rv[8];
  __shared__ int ri[8];
  __shared__ float stage_v[kStage];
  __shared__ int stage_i[kStage];
  wait_prior_grid();
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const char* xrow = reinterpret_cast<const char*>(p.x) + (int64_t)row * p.ld * (kBF16 ? 2 : 4);

  // the streamed tail state: the row's pieces merged in index order (warp 0)
  if (tid < 32) {
    const int lane = tid;
    CapPiece acc{-CUDART_INF_F, 0.f, 0.f, 0};
    if (p.nvec > 0) {
      const int64_t f = (int64_t)row * p.nvec;
      const int w0 = warp_of(f, p.total, p.nwarps);
      const int w1 = warp_of(f + p.nvec - 1, p.total, p.nwarps);
      for (int c = w0; c <= w1; c += 32) {
        const int w = c + lane;
        CapPiece s = (w <= w1) ? p.pieces[row + w] : CapPiece{-CUDART_INF_F, 0.f, 0.f, 0};
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const CapPiece o{__shfl_xor_sync(0xffffffffu, s.m, off), __shfl_xor_sync(0xffffffffu, s.T, off),
                           __shfl_xor_sync(0xffffffffu, s.B, off), 0};
          s = (lane & off) ? piece_merge(o, s) : piece_merge(s, o);
        }
        acc = (c == w0) ? s : piece_merge(acc, s);
      }
    }
    if (lane == 0) merged = acc;
  }

  // candidates: the streamed ones, then the ragged end of the row
  const int cnt = p.count[row];
  const int ns = min(cnt, kCap);
  const int ragged = p.vocab - p.nvec * E;
  const float tau = p.tau[row];
  int ge = 0;
  if (tid < ragged) {
    const int id = p.nvec * E + tid;
    const float v = El::load1(xrow, id);
    rv[tid] = v;
    ri[tid] = id;
    ge = v >= tau ? 1 : 0;
  }
  ge = __syncthreads_count(ge);
  const bool exact = p.force_exact || cnt > kCap || ns + ge < p.K;
  if (!exact && ns + ragged <= kStage) {
    const int2* cand = p.cand + (int64_t)row * kCap;
    for (int i = tid; i < ns; i += kFinThreads) {
      const int2 c = __ldg(cand + i);
      stage_v[i] = __int_as_float(c.x);
      stage_i[i] = c.y;
    }
    if (tid < ragged) {
      stage_v[ns + tid] = rv[tid];
      stage_i[ns + tid] = ri[tid];
    }
    __syncthreads();
    capture_finish<kBF16>(p, row, SmemCands{stage_v, stage_i, ns + ragged}, merged.m, merged.T, merged.B, sel, sc);
  } else if (!exact) {
    capture_finish<kBF16>(p, row, BufCands{p.cand + (int64_t)row * kCap, ns, rv, ri, ns + ragged}, merged.m,
                          merged.T, merged.B, sel, sc);
  } else {
    // every element of the row is a candidate; nothing was left to the tail
    capture_finish<kBF16>(p, row, RowCands<kBF16>{xrow, p.vocab}, -CUDART_INF_F, 0.f, 0.f, sel, sc);
  }
}

int stream_warps(int64_t total) {
  int64_t w = total / kMinVecsPerWarp;
  if (w < 1) w = 1;
  if (w > kMaxStreamWarps) w = kMaxStreamWarps;
  return (int)w;
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

size_t sparse_capture_workspace_bytes(int64_t n_rows) {
  return align256(sizeof(float) * n_rows) + align256(sizeof(int) * n_rows) +
         align256(sizeof(CapPiece) * (n_rows + kMaxStreamWarps)) + sizeof(int2) * (size_t)n_rows * kCap;
}

cudaError_t launch_sparse_capture(const SparseCaptureArgs& a, cudaStream_t stream) {
  const int E = a.bf16 ? 8 : 4;
  CapParams p;
  p.x = a.x;
  p.ld = a.ld;
  p.vocab = (int)a.vocab;
  p.nvec = (int)(a.vocab / E);
  p.n_rows = (int)a.n_rows;
  p.total = a.n_rows * (int64_t)p.nvec;
  p.nwarps = stream_warps(p.total);
  p.K = a.k;
  p.targets = a.targets;
  char* ws = reinterpret_cast<char*>(a.workspace);
  p.tau = reinterpret_cast<float*>(ws);
  ws += align256(sizeof(float) * a.n_rows);
  p.count = reinterpret_cast<int*>(ws);
  ws += align256(sizeof(int) * a.n_rows);
  p.pieces = reinterpret_cast<CapPiece*>(ws);
  ws += align256(sizeof(CapPiece) * (a.n_rows + kMaxStreamWarps));
  p.cand = reinterpret_cast<int2*>(ws);
  p.top = a.top;
  p.rows = a.rows;
  p.dev_status = a.dev_status;
  p.force_exact = a.force_exact;

  cudaError_t e;
  if (a.bf16) e = launch_dependent(cap_sample_kernel<true>, dim3((unsigned)a.n_rows), dim3(kSampleThreads), stream, p);
  else e = launch_dependent(cap_sample_kernel<false>, dim3((unsigned)a.n_rows), dim3(kSampleThreads), stream, p);
  if (e != cudaSuccess) return e;
  if (p.total > 0) {
    const unsigned grid = (unsigned)((p.nwarps + kWarpsPerCta - 1) / kWarpsPerCta);
    if (a.bf16) e = launch_dependent(cap_stream_kernel<true>, dim3(grid), dim3(kThreads), stream, p);
    else e = launch_dependent(cap_stream_kernel<false>, dim3(grid), dim3(kThreads), stream, p);
    if (e != cudaSuccess) return e;
  }
  if (a.bf16) return launch_dependent(cap_finalize_kernel<true>, dim3((unsigned)a.n_rows), dim3(kFinThreads), stream, p);
  return launch_dependent(cap_finalize_kernel<false>, dim3((unsigned)a.n_rows), dim3(kFinThreads), stream, p);
}

}  // namespace kld
