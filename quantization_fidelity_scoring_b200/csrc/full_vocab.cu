// Full-vocabulary scoring: one streaming pass over both logit rows.
//
// Per row the reference logits x and candidate logits y are read once from
// HBM with 128-bit non-allocating loads.  Each thread folds its strided
// 16-byte vectors into an online log-sum-exp state (kld_common.cuh) for
// both sides plus the cross term A; a vector whose maximum does not beat the
// running maxima takes the fast path (two ex2 per element pair, paired f32x2
// arithmetic), otherwise every element is pushed exactly (new maximum,
// argmax, rescale).  States merge by warp butterfly, then across the CTA's
// warps, then across the CTAs of a thread-block cluster through distributed
// shared memory, all in fixed orders.
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

template <bool kBF16>
struct Elems;

template <>
struct Elems<true> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static float load1(const void* base, int64_t i) {
    const unsigned short b = reinterpret_cast<const unsigned short*>(base)[i];
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
};

template <>
struct Elems<false> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static float load1(const void* base, int64_t i) {
    return reinterpret_cast<const float*>(base)[i];
  }
};

// Per-thread accumulation: an exact RowState plus paired fast-path sums that
// are folded into it before any rescale and at the end.
struct ThreadAcc {
  RowState s;
  float2 rx2, ry2, a2;
};

__device__ __forceinline__ void fold(ThreadAcc& t) {
  t.s.x.r += t.rx2.x + t.rx2.y;
  t.s.y.r += t.ry2.x + t.ry2.y;
  t.s.A += t.a2.x + t.a2.y;
  t.rx2 = t.ry2 = t.a2 = make_float2(0.f, 0.f);
}

__device__ __forceinline__ void push_exact(ThreadAcc& t, float xv, float yv, int i) {
  float wx, sx, wy, sy;
  side_push(t.s.x, xv, i, wx, sx, t.s.bad);
  side_push(t.s.y, yv, i, wy, sy, t.s.bad);
  t.s.A = t.s.A * sx + wx * fmaxf(xv - yv, -FLT_MAX);
}

template <int E>
__device__ __forceinline__ void push_chunk(ThreadAcc& t, const float (&xs)[E], const float (&ys)[E], int i0) {
  float cmx = xs[0], cmy = ys[0];
#pragma unroll
  for (int j = 1; j < E; ++j) {
    cmx = fmaxf(cmx, xs[j]);
    cmy = fmaxf(cmy, ys[j]);
  }
  if (cmx > t.s.x.m || cmy > t.s.y.m || t.s.x.a < 0 || t.s.y.a < 0) {
    fold(t);
#pragma unroll
    for (int j = 0; j < E; ++j) push_exact(t, xs[j], ys[j], i0 + j);
    return;
  }
  const float2 nmx = make_float2(-t.s.x.m, -t.s.x.m);
  const float2 nmy = make_float2(-t.s.y.m, -t.s.y.m);
  const float2 l2 = make_float2(kLog2e, kLog2e);
  const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int k = 0; k < E / 2; ++k) {
    const float2 X = make_float2(xs[2 * k], xs[2 * k + 1]);
    const float2 Y = make_float2(ys[2 * k], ys[2 * k + 1]);
    const float2 tx = __fmul2_rn(__fadd2_rn(X, nmx), l2);
    const float2 ty = __fmul2_rn(__fadd2_rn(Y, nmy), l2);
    const float2 ex = make_float2(ex2(tx.x), ex2(tx.y));
    const float2 ey = make_float2(ex2(ty.x), ex2(ty.y));
    t.rx2 = __fadd2_rn(t.rx2, ex);
    t.ry2 = __fadd2_rn(t.ry2, ey);
    float2 d = __ffma2_rn(Y, neg1, X);
    d.x = fmaxf(d.x, -FLT_MAX);
    d.y = fmaxf(d.y, -FLT_MAX);
    t.a2 = __ffma2_rn(ex, d, t.a2);
  }
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads) full_vocab_kernel(const FullVocabParams p) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  constexpr int kElemBytes = kBF16 ? 2 : 4;

  const int cl = p.cl;
  const int row = blockIdx.x / cl;
  const int rank = blockIdx.x % cl;
  const int tid = threadIdx.x;

  const char* xrow = reinterpret_cast<const char*>(p.x) + (int64_t)row * p.ld_x * kElemBytes;
  const char* yrow = reinterpret_cast<const char*>(p.y) + (int64_t)row * p.ld_y * kElemBytes;

  const int nvec = p.vocab / E;
  const int seg_begin = (int)(((int64_t)nvec * rank) / cl);
  const int seg_end = (int)(((int64_t)nvec * (rank + 1)) / cl);

  ThreadAcc t;
  t.s = row_empty();
  t.rx2 = t.ry2 = t.a2 = make_float2(0.f, 0.f);

  int v = seg_begin + tid;
  for (; v + kThreads < seg_end; v += 2 * kThreads) {
    const uint4 X0 = ld_stream(xrow + (int64_t)v * 16);
    const uint4 Y0 = ld_stream(yrow + (int64_t)v * 16);
    const uint4 X1 = ld_stream(xrow + (int64_t)(v + kThreads) * 16);
    const uint4 Y1 = ld_stream(yrow + (int64_t)(v + kThreads) * 16);
    float xs[E], ys[E];
    El::unpack(X0, xs);
    El::unpack(Y0, ys);
    push_chunk<E>(t, xs, ys, v * E);
    El::unpack(X1, xs);
    El::unpack(Y1, ys);
    push_chunk<E>(t, xs, ys, (v + kThreads) * E);
  }
  if (v < seg_end) {
    const uint4 X0 = ld_stream(xrow + (int64_t)v * 16);
    const uint4 Y0 = ld_stream(yrow + (int64_t)v * 16);
    float xs[E], ys[E];
    El::unpack(X0, xs);
    El::unpack(Y0, ys);
    push_chunk<E>(t, xs, ys, v * E);
  }
  fold(t);
  // ragged tail (vocab not a multiple of E): the last CTA's first threads,
  // after their vectors, so each thread still sees increasing indices
  const int tail = p.vocab - nvec * E;
  if (rank == cl - 1 && tid < tail) {
    const int i = nvec * E + tid;
    push_exact(t, El::load1(xrow, i), El::load1(yrow, i), i);
  }

  RowState s = warp_merge_row(t.s);

  __shared__ RowState warp_states[kWarps];
  __shared__ RowState cta_state;
  const int warp = tid >> 5;
  if ((tid & 31) == 0) warp_states[warp] = s;
  __syncthreads();
  if (tid == 0) {
    RowState c = warp_states[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) c = row_merge(c, warp_states[w]);
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
  // about 16 vectors per thread per CTA, at most 8 CTAs (portable cluster)
  const int per_cta = kThreads * 16;
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
