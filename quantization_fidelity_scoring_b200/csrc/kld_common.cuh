// Shared device helpers for the libkld kernels (sm_100a).
//
// Online log-sum-exp state.  For one side (reference x or candidate y) of one
// row, a partial state over a set of vocabulary ids I is
//     m = max_{i in I} z_i,   a = lowest i in I with z_i = m,
//     r = sum_{i in I, i != a} exp(z_i - m)
// so that sum_{i in I} exp(z_i - m) = 1 + r.  Keeping the maximum's own term
// out of r lets log S = log1p(r) be formed without cancellation even when the
// top id holds almost all of the mass (a near-certain token), which the
// relative target log-prob bound needs.  The reference side also carries
//     A = sum_{i in I} exp(x_i - m_x) (x_i - y_i)
// from which KL = A / S_x - (m_x - m_y) + log S_y - log S_x, the expansion of
// sum_i p_i (log p_i - log q_i) with log p_i = x_i - m_x - log S_x.
// ("Qwen3.8-27B Quantization Challenge", "The score".)
//
// An empty state has a = -1 (m = -inf, r = 0).  `bad` records a NaN seen on a
// path that would otherwise drop it.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <mutex>

namespace kld {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2(float t) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
  return r;
}

struct Side {
  float m;
  float r;
  int a;
};

__device__ __forceinline__ Side side_empty() { return Side{-CUDART_INF_F, 0.f, -1}; }

// Fold one element (index i, value v) into a side state, in increasing
// index order.  Returns the weight exp(v - m_new) of the element relative to
// the new maximum (1 for a new maximum) and the factor the previous sums were
// rescaled by, so the reference side can update A.
__device__ __forceinline__ void side_push(Side& s, float v, int i, float& w, float& scale, int& bad) {
  if (v > s.m) {
    // new maximum: old maximum joins r, every old term is rescaled
    scale = (s.a < 0) ? 0.f : ex2((s.m - v) * kLog2e);
    s.r = (s.a < 0) ? 0.f : (1.f + s.r) * scale;
    s.m = v;
    s.a = i;
    w = 1.f;
  } else {
    scale = 1.f;
    if (s.a < 0) {
      // nothing finite seen yet: v is -inf (weight 0) or NaN
      w = 0.f;
      bad |= (v != v);
    } else {
      w = ex2((v - s.m) * kLog2e);
      s.r += w;
    }
  }
}

// Merge two partial states of one side.  Returns the factor that the state
// with the smaller maximum was scaled by (for the reference side's A), and
// which operand won (0: s1 keeps its maximum, 1: s2's maximum wins).
__device__ __forceinline__ Side side_merge(const Side& s1, const Side& s2, float& scale_other, int& winner) {
  if (s2.a < 0) { scale_other = 0.f; winner = 0; return s1; }
  if (s1.a < 0) { scale_other = 0.f; winner = 1; return s2; }
  const bool first = (s1.m > s2.m) || (s1.m == s2.m && s1.a < s2.a);
  const Side& big = first ? s1 : s2;
  const Side& small = first ? s2 : s1;
  const float sc = ex2((small.m - big.m) * kLog2e);
  scale_other = sc;
  winner = first ? 0 : 1;
  return Side{big.m, big.r + (1.f + small.r) * sc, big.a};
}

// Row state: both sides, the cross term A (scaled like the reference side)
// and a NaN flag.
struct RowState {
  Side x, y;
  float A;
  int bad;
};

__device__ __forceinline__ RowState row_empty() {
  RowState s;
  s.x = side_empty();
  s.y = side_empty();
  s.A = 0.f;
  s.bad = 0;
  return s;
}

__device__ __forceinline__ RowState row_merge(const RowState& p, const RowState& q) {
  RowState o;
  float scx, scy;
  int wx, wy;
  o.x = side_merge(p.x, q.x, scx, wx);
  o.y = side_merge(p.y, q.y, scy, wy);
  // A follows the reference side's maximum
  if (p.x.a < 0) o.A = q.A;
  else if (q.x.a < 0) o.A = p.A;
  else o.A = (wx == 0) ? (p.A + q.A * scx) : (q.A + p.A * scx);
  o.bad = p.bad | q.bad;
  return o;
}

__device__ __forceinline__ RowState shfl_xor_row(const RowState& s, int lane_mask) {
  RowState o;
  o.x.m = __shfl_xor_sync(0xffffffffu, s.x.m, lane_mask);
  o.x.r = __shfl_xor_sync(0xffffffffu, s.x.r, lane_mask);
  o.x.a = __shfl_xor_sync(0xffffffffu, s.x.a, lane_mask);
  o.y.m = __shfl_xor_sync(0xffffffffu, s.y.m, lane_mask);
  o.y.r = __shfl_xor_sync(0xffffffffu, s.y.r, lane_mask);
  o.y.a = __shfl_xor_sync(0xffffffffu, s.y.a, lane_mask);
  o.A = __shfl_xor_sync(0xffffffffu, s.A, lane_mask);
  o.bad = __shfl_xor_sync(0xffffffffu, s.bad, lane_mask);
  return o;
}

// Butterfly merge across a warp.  Every lane ends with the same state; the
// merge order depends only on lane ids, so the result is deterministic, and
// it is symmetric in x and y.  Lane order is preserved (lower lanes first)
// at every level so that equal maxima keep the lowest index.
__device__ __forceinline__ RowState warp_merge_row(RowState s) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    RowState o = shfl_xor_row(s, off);
    s = (lane & off) ? row_merge(o, s) : row_merge(s, o);
  }
  return s;
}

// Final per-row outputs from a merged state, in f64.
struct RowOut {
  float kl, lp_x, lp_y;
  int ax, ay;
};

__device__ __forceinline__ bool row_valid(const RowState& s) {
  return !s.bad && s.x.a >= 0 && s.y.a >= 0 && !isinf(s.x.m) && !isinf(s.y.m) &&
         !isnan(s.x.r) && !isnan(s.y.r);
}

__device__ __forceinline__ RowOut row_finish(const RowState& s, bool have_target, float xt, float yt) {
  RowOut o;
  if (!row_valid(s)) {
    o.kl = CUDART_NAN_F;
    o.lp_x = o.lp_y = CUDART_NAN_F;
    o.ax = o.ay = -1;
    return o;
  }
  const double lsx = log1p((double)s.x.r);
  const double lsy = log1p((double)s.y.r);
  const double kl = (double)s.A / (1.0 + (double)s.x.r) - ((double)s.x.m - (double)s.y.m) + (lsy - lsx);
  // In a valid row A can only turn NaN through 0 * inf: a candidate logit of
  // -inf where the reference weight underflowed f32 but p_i > 0 exactly.
  o.kl = (s.A != s.A) ? CUDART_INF_F : (float)kl;
  o.ax = s.x.a;
  o.ay = s.y.a;
  if (have_target) {
    o.lp_x = (float)(((double)xt - (double)s.x.m) - lsx);
    o.lp_y = (float)(((double)yt - (double)s.y.m) - lsy);
  } else {
    o.lp_x = o.lp_y = CUDART_NAN_F;
  }
  return o;
}

__device__ __forceinline__ void set_dev_status(int32_t* dev_status, int bits) {
  if (dev_status) atomicOr(reinterpret_cast<int*>(dev_status), bits);
}

// Programmatic dependent launch.  A kernel launched with launch_dependent()
// may be scheduled while the previous kernel on the stream is still
// finishing, which hides its launch latency; it must call
// wait_prior_grid() before touching memory the previous kernels use (the
// wait returns at once when the kernel was launched the ordinary way).
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Raises a kernel's dynamic shared-memory limit (required above 48 KB) on
// the current device, once per device and kernel.
template <auto Kernel>
inline cudaError_t allow_dynamic_smem(size_t bytes) {
  static std::mutex mu;
  static unsigned long long done = 0ull;  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && ((done >> dev) & 1ull)) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev < 64) done |= 1ull << dev;
  return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent_smem(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem_bytes,
                                  cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t stream,
                             Args&&... args) {
  return launch_dependent_smem(kernel, grid, block, 0, stream, static_cast<Args&&>(args)...);
}

}  // namespace kld
