// Fused shared-head scoring on the 5th-generation tensor cores.
//
// "Qwen3.8-27B fidelity suite v5", opening paragraph: the KL is computed from
// final hidden states pushed through one shared BF16 LM head, so reference
// and candidate logits are x = W h_ref and y = W h_cand with the same W.
// "Qwen3.8-27B Quantization Challenge", "How the references were made": the
// distribution is computed in f32.  Here the logits are accumulated in f32 in
// tensor memory and consumed there: they never reach HBM.
//
// Tiling.  A tile is 64 positions x 256 vocabulary ids.  Its 128 MMA rows
// stack the 64 reference hidden states over the same 64 candidate hidden
// states, so one 128x256x16 tcgen05.mma per K step produces both sides'
// logits of the tile from one W tile.  K advances 64 at a time through a
// 4-stage ring that TMA fills (128-byte swizzle, no multicast); the
// accumulator is double-buffered in TMEM (2 x 256 columns) so the epilogue
// of one tile overlaps the MMAs of the next.
//
// Warp roles (192 threads, one CTA per SM): warp 0 issues TMA, warp 1 owns
// TMEM and issues MMAs, warps 2..5 are the epilogue.  TMEM lane quarters
// 0,1 hold reference rows and 2,3 candidate rows, so each epilogue thread
// owns one position of one side: it takes the tile maximum in a first pass
// over its lane, then weighs every logit in a second pass.  Candidate threads
// hand their logits to the reference threads through shared memory, 32
// columns at a time, for the cross term A = sum exp(x - m_x)(x - y).
//
// Each tile's per-position state (max, argmax, sum of the other weights, A;
// kld_common.cuh) goes to the workspace; a merge kernel combines a
// position's tiles in vocabulary order.  Persistent CTAs walk the tiles
// round-robin in an order that sweeps 32 position blocks together along the
// vocabulary, so concurrently resident CTAs share W tiles and the group's
// hidden states through L2.  Every wait is bounded; a timeout sets
// KLD_DEV_TIMEOUT, drains what is in flight and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cfloat>

#include "kld_common.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace kld {
namespace {

constexpr int kPos = 64;         // positions per tile
constexpr int kBM = 2 * kPos;    // MMA rows: reference then candidate
constexpr int kBN = 256;         // vocabulary ids per tile
constexpr int kBK = 64;          // K per stage: one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kGroup = 32;       // position blocks swept together
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kChunk = 32;       // TMEM columns per load
constexpr int kChunks = kBN / kChunk;
constexpr int kXStride = kChunk + 1;  // exchange row stride in floats
constexpr uint32_t kStageA = kBM * kBK * 2;
constexpr uint32_t kStageB = kBN * kBK * 2;
constexpr uint32_t kTmemCols = 2 * kBN;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kBM, kBN);

constexpr size_t kSmemStages = (size_t)kStages * (kStageA + kStageB);
constexpr size_t kSmemX = (size_t)2 * kPos * kXStride * sizeof(float);
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 1;
constexpr size_t kSmemBytes = 1024 + kSmemStages + kSmemX + kNumBars * 8 + 16;

struct HeadParams {
  int n_rows, hidden, vocab;
  int nb, nt, kblocks;
  int64_t ntiles;
  float4* px;  // [nt][n_rows] reference side: max, sum of other weights, argmax bits, A
  float4* py;  // [nt][n_rows] candidate side: max, sum, argmax bits, 0
  float2* tv;  // [n_rows] target logits (x_t, y_t)
  const int32_t* targets;
  int32_t* dev_status;
  int withhold;  // tests only: skip the first TMA fill so every wait times out
};

__device__ __forceinline__ void tile_coords(int64_t i, int nb, int nt, int& pb, int& vt) {
  const int64_t per_group = (int64_t)kGroup * nt;
  const int g = (int)(i / per_group);
  const int64_t j = i - (int64_t)g * per_group;
  const int gsize = min(kGroup, nb - g * kGroup);
  vt = (int)(j / gsize);
  pb = g * kGroup + (int)(j % gsize);
}

__device__ __forceinline__ void timed_out(int* abort_flag, int32_t* dev_status) {
  atomicExch(abort_flag, 1);
  set_dev_status(dev_status, 0x4 /* KLD_DEV_TIMEOUT */);
}

__global__ void __launch_bounds__(kThreads, 1)
    head_kernel(const __grid_constant__ CUtensorMap tm_ref, const __grid_constant__ CUtensorMap tm_cand,
                const __grid_constant__ CUtensorMap tm_w, const HeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + (size_t)kStages * kStageA;
  float* xbuf = reinterpret_cast<float*>(smem + kSmemStages);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemStages + kSmemX);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* xfull = tempty + 2;
  uint64_t* xempty = xfull + 2;
  uint64_t* mma_done = xempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], kEpiThreads);
      ptx::mbar_init(&xfull[b], kPos);
      ptx::mbar_init(&xempty[b], kPos);
    }
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_ref);
      ptx::prefetch_tmap(&tm_cand);
      ptx::prefetch_tmap(&tm_w);
      int stage = 0;
      uint32_t phase = 0;
      int used = 0;  // stages ever filled (to drain at the end)
      for (int64_t i = blockIdx.x; i < p.ntiles && !*abort_flag; i += gridDim.x) {
        int pb, vt;
        tile_coords(i, p.nb, p.nt, pb, vt);
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1, kWaitNs)) {
            timed_out(const_cast<int*>(abort_flag), p.dev_status);
            break;
          }
          if (!(p.withhold && i == blockIdx.x && kb == 0)) {
            ptx::mbar_arrive_expect_tx(&full[stage], kStageA + kStageB);
            uint8_t* a = sA + (size_t)stage * kStageA;
            ptx::tma_load_2d(a, &tm_ref, kb * kBK, pb * kPos, &full[stage]);
            ptx::tma_load_2d(a + kStageA / 2, &tm_cand, kb * kBK, pb * kPos, &full[stage]);
            ptx::tma_load_2d(sB + (size_t)stage * kStageB, &tm_w, kb * kBK, vt * kBN, &full[stage]);
          }
          if (used < kStages) ++used;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every issued copy lands before the CTA may exit: the last fill of
      // each stage s sits in the phase before the current one
      for (int k = 0; k < used; ++k) {
        stage = (stage + kStages - 1) % kStages;
        if (stage == kStages - 1) phase ^= 1;
        ptx::mbar_wait(&full[stage], phase, kWaitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool issued = false;
      for (int64_t i = blockIdx.x; i < p.ntiles && !*abort_flag; i += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!ptx::mbar_wait(&tempty[buf], (use & 1) ^ 1, kWaitNs)) {
          timed_out(const_cast<int*>(abort_flag), p.dev_status);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * kBN);
        bool ok = true;
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!ptx::mbar_wait(&full[stage], phase, kWaitNs)) {
            timed_out(const_cast<int*>(abort_flag), p.dev_status);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t adesc = ptx::sw128_kmajor_desc(ptx::smem_addr(sA + (size_t)stage * kStageA));
          const uint64_t bdesc = ptx::sw128_kmajor_desc(ptx::smem_addr(sB + (size_t)stage * kStageB));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // 16 bf16 = 32 bytes = 2 descriptor units
            ptx::umma_bf16(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, (kb | k) != 0 ? 1u : 0u);
          ptx::umma_commit(&empty[stage]);  // frees the stage once these MMAs are done
          issued = true;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        ptx::umma_commit(&tfull[buf]);
      }
      // nothing may still write TMEM when it is released
      if (issued) {
        ptx::umma_commit(mma_done);
        ptx::mbar_wait(mma_done, 0, kWaitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;          // TMEM lane quarter of this warp
    const bool is_x = q < 2;         // quarters 0,1: reference rows
    const int pos = (q & 1) * 32 + lane;
    int local = 0;
    uint32_t chunk_no = 0;
    for (int64_t i = blockIdx.x; i < p.ntiles; i += gridDim.x, ++local) {
      if (__any_sync(0xffffffffu, *abort_flag)) break;  // leave as a whole warp
      int pb, vt;
      tile_coords(i, p.nb, p.nt, pb, vt);
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&tfull[buf], use & 1, kWaitNs))) {
        timed_out(const_cast<int*>(abort_flag), p.dev_status);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kBN);
      const int col0 = vt * kBN;
      const int nvalid = min(kBN, p.vocab - col0);
      const int row = pb * kPos + pos;
      const int tloc = (p.targets && row < p.n_rows) ? p.targets[row] - col0 : -1;

      // pass 1: the tile maximum of this position and side
      float m = -CUDART_INF_F;
      for (int c = 0; c < kChunks; ++c) {
        float v[kChunk];
        ptx::tmem_ld32(tbase + c * kChunk, v);
#pragma unroll
        for (int j = 0; j < kChunk; ++j)
          if (c * kChunk + j < nvalid) m = fmaxf(m, v[j]);
      }
      // pass 2: weights relative to the maximum; the first maximal id is the
      // tile's argmax and stays out of r
      float r = 0.f, A = 0.f, tval = 0.f;
      int a = -1;
      bool ok = true;
      for (int c = 0; c < kChunks; ++c, ++chunk_no) {
        float v[kChunk];
        ptx::tmem_ld32(tbase + c * kChunk, v);
#pragma unroll
        for (int j = 0; j < kChunk; ++j)
          if (c * kChunk + j >= nvalid) v[j] = -CUDART_INF_F;
        const int xb = (int)(chunk_no & 1);
        const uint32_t xu = chunk_no >> 1;
        float* xrow = xbuf + (size_t)(xb * kPos + pos) * kXStride;
        if (!is_x) {
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(&xempty[xb], (xu & 1) ^ 1, kWaitNs))) {
            timed_out(const_cast<int*>(abort_flag), p.dev_status);
            ok = false;
            break;
          }
#pragma unroll
          for (int j = 0; j < kChunk; ++j) xrow[j] = v[j];
          ptx::mbar_arrive(&xfull[xb]);
        }
        float w[kChunk];
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
          w[j] = ex2((v[j] - m) * kLog2e);
          const bool first = (a < 0) && (v[j] == m);
          if (first) a = col0 + c * kChunk + j;
          r += first ? 0.f : w[j];
        }
        if (is_x) {
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(&xfull[xb], xu & 1, kWaitNs))) {
            timed_out(const_cast<int*>(abort_flag), p.dev_status);
            ok = false;
            break;
          }
#pragma unroll
          for (int j = 0; j < kChunk; ++j) A += w[j] * fmaxf(v[j] - xrow[j], -FLT_MAX);
          ptx::mbar_arrive(&xempty[xb]);
        }
        if ((unsigned)(tloc - c * kChunk) < (unsigned)kChunk) {
#pragma unroll
          for (int j = 0; j < kChunk; ++j)
            if (tloc - c * kChunk == j) tval = v[j];
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&tempty[buf]);
      if (!ok) break;
      if (row < p.n_rows) {
        const float4 st = make_float4(m, r, __int_as_float(a), is_x ? A : 0.f);
        (is_x ? p.px : p.py)[(int64_t)vt * p.n_rows + row] = st;
        if (tloc >= 0 && tloc < nvalid) {
          if (is_x) p.tv[row].x = tval;
          else p.tv[row].y = tval;
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// One warp per position: merge its tiles in vocabulary order, then form the
// outputs from the merged state and the target logits.
__global__ void __launch_bounds__(256) head_merge_kernel(const HeadParams p, float* kl, int32_t* ax, int32_t* ay,
                                                         float* lpx, float* lpy) {
  wait_prior_grid();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= p.n_rows) return;
  // the target logits first: their loads overlap the merge
  const int tg = p.targets ? p.targets[row] : -1;
  const bool have_t = p.targets && tg >= 0 && tg < p.vocab;
  const float2 t2 = have_t ? p.tv[row] : make_float2(0.f, 0.f);
  RowState acc = row_empty();
  for (int c = 0; c < p.nt; c += 32) {
    const int t = c + lane;
    RowState s = row_empty();
    if (t < p.nt) {
      const float4 x = p.px[(int64_t)t * p.n_rows + row];
      const float4 y = p.py[(int64_t)t * p.n_rows + row];
      s.x = Side{x.x, x.y, __float_as_int(x.z)};
      s.y = Side{y.x, y.y, __float_as_int(y.z)};
      s.A = x.w;
    }
    s = warp_merge_row(s);
    acc = (c == 0) ? s : row_merge(acc, s);
  }
  if (lane != 0) return;
  if (p.targets && !have_t) set_dev_status(p.dev_status, 0x1 /* KLD_DEV_BAD_TARGET */);
  const RowOut o = row_finish(acc, have_t, t2.x, t2.y);
  kl[row] = o.kl;
  if (ax) ax[row] = o.ax;
  if (ay) ay[row] = o.ay;
  if (lpx) lpx[row] = o.lp_x;
  if (lpy) lpy[row] = o.lp_y;
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

cudaError_t encode_fn(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  if (!cached) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || f == nullptr) return cudaErrorNotSupported;
    cached = reinterpret_cast<EncodeTiledFn>(f);
  }
  *fn = cached;
  return cudaSuccess;
}

// 2-D bf16 map over a row-major [rows, cols] matrix, box = box_rows x 64 columns.
cudaError_t make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn fn;
  const cudaError_t e = encode_fn(&fn);
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

struct Layout {
  size_t px, py, tv, total;
};

Layout workspace_layout(int64_t n_rows, int64_t vocab) {
  const int64_t nt = (vocab + kBN - 1) / kBN;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  Layout l;
  l.px = 0;
  l.py = up(l.px + (size_t)nt * n_rows * sizeof(float4));
  l.tv = up(l.py + (size_t)nt * n_rows * sizeof(float4));
  l.total = up(l.tv + (size_t)n_rows * sizeof(float2));
  return l;
}

}  // namespace

size_t shared_head_workspace_bytes(int64_t n_rows, int64_t vocab) { return workspace_layout(n_rows, vocab).total; }

cudaError_t launch_shared_head(const SharedHeadArgs& a, cudaStream_t stream) {
  CUtensorMap tm_ref, tm_cand, tm_w;
  cudaError_t e = make_map(&tm_ref, a.h_ref, a.n_rows, a.hidden, kPos);
  if (e == cudaSuccess) e = make_map(&tm_cand, a.h_cand, a.n_rows, a.hidden, kPos);
  if (e == cudaSuccess) e = make_map(&tm_w, a.head_w, a.vocab, a.hidden, kBN);
  if (e != cudaSuccess) return e;

  const Layout l = workspace_layout(a.n_rows, a.vocab);
  char* ws = reinterpret_cast<char*>(a.workspace);
  HeadParams p;
  p.n_rows = (int)a.n_rows;
  p.hidden = (int)a.hidden;
  p.vocab = (int)a.vocab;
  p.nb = (int)((a.n_rows + kPos - 1) / kPos);
  p.nt = (int)((a.vocab + kBN - 1) / kBN);
  p.kblocks = (int)((a.hidden + kBK - 1) / kBK);
  p.ntiles = (int64_t)p.nb * p.nt;
  p.px = reinterpret_cast<float4*>(ws + l.px);
  p.py = reinterpret_cast<float4*>(ws + l.py);
  p.tv = reinterpret_cast<float2*>(ws + l.tv);
  p.targets = a.targets;
  p.dev_status = a.dev_status;
  p.withhold = a.withhold;

  int dev = 0, sms = 148;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = allow_dynamic_smem<head_kernel>(kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = p.ntiles < sms ? p.ntiles : sms;
  head_kernel<<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(tm_ref, tm_cand, tm_w, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned mgrid = (unsigned)((a.n_rows + 7) / 8);
  return launch_dependent(head_merge_kernel, dim3(mgrid), dim3(256), stream, p, a.kl, a.ax, a.ay, a.lpx, a.lpy);
}

}  // namespace kld
