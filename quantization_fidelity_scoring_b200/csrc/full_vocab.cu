// Full-vocabulary scoring: one streaming pass over both logit rows.
//
// Per row the reference logits x and candidate logits y are read once from
// HBM with 128-bit non-allocating loads; a cluster of CTAs splits the row.
// Each warp walks 32 consecutive 16-byte vectors (two per lane) per step and
// keeps an online log-sum-exp state (kld_common.cuh) whose running maximum
// and argmax are warp-uniform: one redux.sync finds the step's maximum, and
// only a step that raises it (a handful per warp per row) takes the branch
// that rescales, locates the new argmax and leaves it out of the sum.  Every
// other step is two ex2 per element pair on paired f32x2 arithmetic.  Warp
// states merge across the CTA's warps and then across the cluster's CTAs
// through distributed shared memory, in fixed orders.
//
// Sources: "Qwen3.8-27B Quantization Challenge", sections "How the
// references were made" (full 248,320-token distribution in f32) and "The
// score" (KL over cells); "Qwopus3.8-27B-Coder-Flash: quality-eval
// reference", "Method" (exact argmax top-1, perplexity from the true-token
// log-prob).
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cfloat>

#include "kld_common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace kld {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct FullVocabParams {
  const void* x;
  const void* y;
  int64_t ld_x, ld_y;  // elements
  int vocab;
  int cl;              // CTAs per row (cluster size)
  const int32_t* targets;
  float* kl;
  int32_t* ax;
  int32_t* ay;
  float* lpx;
  float* lpy;
  int32_t* dev_status;
};

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Element access on raw 16-byte vectors.  bf16: a 32-bit word holds
// elements (2k, 2k+1) in its low and high halves, so a pair widens to f32
// with one shift and one mask.  f32: the vector is four elements.
template <bool kBF16>
struct Elems;

template <>
struct Elems<true> {
  static constexpr int E = 8;
  __device__ __forceinline__ static float2 pair(const uint4& v, int k) {
    const uint32_t w = k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
  __device__ __forceinline__ static float vmax(const uint4& v) {
    uint32_t a, b, m;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(v.x), "r"(v.y));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(b) : "r"(v.z), "r"(v.w));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(b));
    return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
  }
  __device__ __forceinline__ static float load1(const void* base, int64_t i) {
    const unsigned short b = reinterpret_cast<const unsigned short*>(base)[i];
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
};

template <>
struct Elems<false> {
  static constexpr int E = 4;
  __device__ __forceinline__ static float2 pair(const uint4& v, int k) {
    return k == 0 ? make_float2(__uint_as_float(v.x), __uint_as_float(v.y))
                  : make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
  __device__ __forceinline__ static float vmax(const uint4& v) {
    return fmaxf(fmaxf(__uint_as_float(v.x), __uint_as_float(v.y)),
                 fmaxf(__uint_as_float(v.z), __uint_as_float(v.w)));
  }
  __device__ __forceinline__ static float load1(const void* base, int64_t i) {
    return reinterpret_cast<const float*>(base)[i];
  }
};

// One step of a lane: two consecutive-in-warp vectors of each side.
struct StepRaw {
  uint4 x0, y0, x1, y1;
};

// Order-preserving map between floats and signed ints, so that a warp-wide
// float maximum is one redux.sync.max.s32 (NaN is mapped to -inf first).
__device__ __forceinline__ int ordered_key(float f) {
  const int i = __float_as_int(f != f ? -CUDART_INF_F : f);
  return i ^ ((i >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float key_value(int k) { return __int_as_float(k ^ ((k >> 31) & 0x7fffffff)); }

__device__ __forceinline__ float warp_max(float v) {
  return key_value(__reduce_max_sync(0xffffffffu, ordered_key(v)));
}

// Warp-uniform side state: the maximum m and its index a are the same in
// every lane; each lane keeps its own share r of sum_{i != a} exp(z_i - m).
struct WarpSide {
  float m;
  int a;
  float r;
};

// A step whose warp maximum cm beats the running maximum: rescale every
// lane's share to the new maximum, hand the old maximum's own term (1 before
// the rescale) to lane 0, and locate the first occurrence of the new maximum
// in index order (lanes hold consecutive vectors; a lane's first vector comes
// before its second; c0/c1 are the lane's per-vector maxima).  Returns the
// rescale factor; `excl` is the element slot (0 .. 2E-1) this lane leaves
// out of r.
template <bool kBF16>
__device__ __forceinline__ float side_new_max(WarpSide& s, float cm, const uint4& v0, const uint4& v1, float c0,
                                              float c1, int i0, int i1, int lane, int& excl) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  excl = -1;
  if (!(cm > s.m)) return 1.f;
  const float sc = (s.a < 0) ? 0.f : ex2((s.m - cm) * kLog2e);
  s.r = s.r * sc + ((lane == 0 && s.a >= 0) ? sc : 0.f);
  const unsigned b0 = __ballot_sync(0xffffffffu, c0 == cm);
  const unsigned b1 = __ballot_sync(0xffffffffu, c1 == cm);
  const int part = b0 ? 0 : 1;
  const int src = __ffs(b0 ? b0 : b1) - 1;
  int idx = 0;
  if (lane == src) {
    const uint4& v = part ? v1 : v0;
    int j = E - 1;
#pragma unroll
    for (int k = E / 2 - 1; k >= 0; --k) {
      const float2 q = El::pair(v, k);
      if (q.y == cm) j = 2 * k + 1;
      if (q.x == cm) j = 2 * k;
    }
    excl = part * E + j;
    idx = (part ? i1 : i0) + j;
  }
  s.a = __shfl_sync(0xffffffffu, idx, src);
  s.m = cm;
  return sc;
}

// Accumulate one step: weights exp(z - m) on paired f32x2 arithmetic.  With
// kMasked, the slots ex_x / ex_y (the new argmaxes) are weighed as -inf so
// they stay out of r; the reference argmax's own A term, 1 * (x - y), is
// added by the caller.
template <bool kBF16, bool kMasked>
__device__ __forceinline__ void accumulate(const StepRaw& raw, float mx, float my, int ex_x, int ex_y,
                                           float2& rx2, float2& ry2, float2& a2) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  const float2 nmx = make_float2(-mx, -mx);
  const float2 nmy = make_float2(-my, -my);
  const float2 l2 = make_float2(kLog2e, kLog2e);
  const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int vec = 0; vec < 2; ++vec) {
#pragma unroll
    for (int k = 0; k < E / 2; ++k) {
      const float2 X = El::pair(vec ? raw.x1 : raw.x0, k);
      const float2 Y = El::pair(vec ? raw.y1 : raw.y0, k);
      float2 XW = X, YW = Y;
      if (kMasked) {
        const int j = vec * E + 2 * k;
        if (ex_x == j) XW.x = -CUDART_INF_F;
        if (ex_x == j + 1) XW.y = -CUDART_INF_F;
        if (ex_y == j) YW.x = -CUDART_INF_F;
        if (ex_y == j + 1) YW.y = -CUDART_INF_F;
      }
      const float2 tx = __fmul2_rn(__fadd2_rn(XW, nmx), l2);
      const float2 ty = __fmul2_rn(__fadd2_rn(YW, nmy), l2);
      const float2 ex = make_float2(ex2(tx.x), ex2(tx.y));
      const float2 ey = make_float2(ex2(ty.x), ex2(ty.y));
      rx2 = __fadd2_rn(rx2, ex);
      ry2 = __fadd2_rn(ry2, ey);
      float2 d = __ffma2_rn(Y, neg1, X);
      d.x = fmaxf(d.x, -FLT_MAX);
      d.y = fmaxf(d.y, -FLT_MAX);
      a2 = __ffma2_rn(ex, d, a2);
    }
  }
}

// The exact A term 1 * (x - y) of the element in slot j of this lane's step.
template <bool kBF16>
__device__ __forceinline__ float slot_diff(const StepRaw& raw, int j) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  float d = 0.f;
#pragma unroll
  for (int vec = 0; vec < 2; ++vec)
#pragma unroll
    for (int k = 0; k < E / 2; ++k) {
      const float2 X = El::pair(vec ? raw.x1 : raw.x0, k);
      const float2 Y = El::pair(vec ? raw.y1 : raw.y0, k);
      if (j == vec * E + 2 * k) d = X.x - Y.x;
      if (j == vec * E + 2 * k + 1) d = X.y - Y.y;
    }
  return fmaxf(d, -FLT_MAX);
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads) full_vocab_kernel(const FullVocabParams p) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;  // elements per 16-byte vector
  constexpr int kElemBytes = kBF16 ? 2 : 4;
  constexpr uint32_t kNegInfWord = kBF16 ? 0xff80ff80u : 0xff800000u;

  const int cl = p.cl;
  const int row = blockIdx.x / cl;
  const int rank = blockIdx.x % cl;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;

  const char* xrow = reinterpret_cast<const char*>(p.x) + (int64_t)row * p.ld_x * kElemBytes;
  const char* yrow = reinterpret_cast<const char*>(p.y) + (int64_t)row * p.ld_y * kElemBytes;

  const int nvec = p.vocab / E;
  const int seg_begin = (int)(((int64_t)nvec * rank) / cl);
  const int seg_end = (int)(((int64_t)nvec * (rank + 1)) / cl);
  const int steps = (seg_end - seg_begin + 2 * kThreads - 1) / (2 * kThreads);
  const int lane_base = seg_begin + warp * 32 + lane;
  const uint4 neg_inf = make_uint4(kNegInfWord, kNegInfWord, kNegInfWord, kNegInfWord);

  auto load_step = [&](int st, StepRaw& r) {
    const int v0 = lane_base + st * 2 * kThreads;
    const int v1 = v0 + kThreads;
    r.x0 = v0 < seg_end ? ld_stream(xrow + (int64_t)v0 * 16) : neg_inf;
    r.y0 = v0 < seg_end ? ld_stream(yrow + (int64_t)v0 * 16) : neg_inf;
    r.x1 = v1 < seg_end ? ld_stream(xrow + (int64_t)v1 * 16) : neg_inf;
    r.y1 = v1 < seg_end ? ld_stream(yrow + (int64_t)v1 * 16) : neg_inf;
  };

  WarpSide sx{-CUDART_INF_F, -1, 0.f}, sy{-CUDART_INF_F, -1, 0.f};
  float2 rx2 = make_float2(0.f, 0.f), ry2 = rx2, a2 = rx2;

  StepRaw cur;
  if (steps > 0) load_step(0, cur);
  for (int st = 0; st < steps; ++st) {
    // the next step's loads are in flight while this step computes
    StepRaw nxt;
    if (st + 1 < steps) load_step(st + 1, nxt);

    const float cx0 = El::vmax(cur.x0), cx1 = El::vmax(cur.x1);
    const float cy0 = El::vmax(cur.y0), cy1 = El::vmax(cur.y1);
    const float CMX = warp_max(fmaxf(cx0, cx1));
    const float CMY = warp_max(fmaxf(cy0, cy1));

    if (!((CMX > sx.m) || (CMY > sy.m) || (sx.a < 0) || (sy.a < 0))) {  // warp-uniform
      accumulate<kBF16, false>(cur, sx.m, sy.m, -1, -1, rx2, ry2, a2);
    } else {
      // a new maximum on either side, or a side still without a finite
      // value: fold the paired sums, move to the new maxima, weigh with the
      // new argmaxes masked out of r
      sx.r += rx2.x + rx2.y;
      sy.r += ry2.x + ry2.y;
      float A = a2.x + a2.y;
      const int i0 = (lane_base + st * 2 * kThreads) * E;
      const int i1 = i0 + kThreads * E;
      int ex_x, ex_y;
      const float scx = side_new_max<kBF16>(sx, CMX, cur.x0, cur.x1, cx0, cx1, i0, i1, lane, ex_x);
      side_new_max<kBF16>(sy, CMY, cur.y0, cur.y1, cy0, cy1, i0, i1, lane, ex_y);
      A *= scx;
      if (ex_x >= 0) A += slot_diff<kBF16>(cur, ex_x);
      rx2 = ry2 = make_float2(0.f, 0.f);
      a2 = make_float2(A, 0.f);
      // a side with no finite value yet has only -inf (weight 0) or NaN
      // (poisons r, marking the row invalid); any finite offset serves
      accumulate<kBF16, true>(cur, sx.a < 0 ? 0.f : sx.m, sy.a < 0 ? 0.f : sy.m, ex_x, ex_y, rx2, ry2, a2);
    }
    if (st + 1 < steps) cur = nxt;
  }

  // warp state: uniform maxima, lane shares summed in a fixed butterfly
  RowState s;
  s.x.m = sx.m;
  s.x.a = sx.a;
  s.y.m = sy.m;
  s.y.a = sy.a;
  float rxs = sx.r + (rx2.x + rx2.y);
  float rys = sy.r + (ry2.x + ry2.y);
  float as = a2.x + a2.y;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    rxs += __shfl_xor_sync(0xffffffffu, rxs, off);
    rys += __shfl_xor_sync(0xffffffffu, rys, off);
    as += __shfl_xor_sync(0xffffffffu, as, off);
  }
  s.x.r = rxs;
  s.y.r = rys;
  s.A = as;
  s.bad = 0;

  __shared__ RowState warp_states[kWarps];
  __shared__ RowState cta_state;
  if (lane == 0) warp_states[warp] = s;
  __syncthreads();
  if (tid == 0) {
    RowState c = warp_states[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) c = row_merge(c, warp_states[w]);
    // ragged tail (vocab not a multiple of E): the row's last ids, pushed
    // one by one in index order into the last CTA's state
    if (rank == cl - 1) {
      for (int i = nvec * E; i < p.vocab; ++i) {
        const float xv = El::load1(xrow, i), yv = El::load1(yrow, i);
        float wx, scx, wy, scy;
        side_push(c.x, xv, i, wx, scx, c.bad);
        side_push(c.y, yv, i, wy, scy, c.bad);
        c.A = c.A * scx + wx * fmaxf(xv - yv, -FLT_MAX);
      }
    }
    cta_state = c;
  }

  if (cl > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && tid == 0) {
      RowState c = *cluster.map_shared_rank(&cta_state, 0);
      for (int r = 1; r < cl; ++r) c = row_merge(c, *cluster.map_shared_rank(&cta_state, r));
      cta_state = c;
    }
    cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
  } else {
    __syncthreads();
  }
  if (rank != 0 || tid != 0) return;

  const RowState fin = cta_state;
  bool have_t = false;
  float xt = 0.f, yt = 0.f;
  if (p.targets) {
    const int tg = p.targets[row];
    if (tg >= 0 && tg < p.vocab) {
      have_t = true;
      xt = El::load1(xrow, tg);
      yt = El::load1(yrow, tg);
    } else {
      set_dev_status(p.dev_status, 0x1 /* KLD_DEV_BAD_TARGET */);
    }
  }
  const RowOut o = row_finish(fin, have_t, xt, yt);
  p.kl[row] = o.kl;
  if (p.ax) p.ax[row] = o.ax;
  if (p.ay) p.ay[row] = o.ay;
  if (p.lpx) p.lpx[row] = o.lp_x;
  if (p.lpy) p.lpy[row] = o.lp_y;
}

int choose_cluster(int nvec) {
  // about 32 vectors per thread per CTA, at most 8 CTAs (portable cluster)
  const int per_cta = kThreads * 32;
  int cl = (nvec + per_cta - 1) / per_cta;
  if (cl < 1) cl = 1;
  if (cl > 8) cl = 8;
  return cl;
}

}  // namespace

cudaError_t launch_full_vocab(const FullVocabArgs& a, cudaStream_t stream) {
  FullVocabParams p;
  p.x = a.x;
  p.y = a.y;
  p.ld_x = a.ld_x;
  p.ld_y = a.ld_y;
  p.vocab = (int)a.vocab;
  p.targets = a.targets;
  p.kl = a.kl;
  p.ax = a.ax;
  p.ay = a.ay;
  p.lpx = a.lpx;
  p.lpy = a.lpy;
  p.dev_status = a.dev_status;
  const int E = a.bf16 ? 8 : 4;
  p.cl = a.cluster_override > 0 ? a.cluster_override : choose_cluster((int)(a.vocab / E));

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.n_rows * p.cl), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.bf16) return cudaLaunchKernelEx(&cfg, full_vocab_kernel<true>, p);
  return cudaLaunchKernelEx(&cfg, full_vocab_kernel<false>, p);
}

}  // namespace kld
