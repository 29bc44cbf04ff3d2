// Full-vocabulary scoring: one streaming pass over both logit rows.
//
// The rows' 16-byte vectors, flattened in (row, vector) order, are split
// evenly over a fixed set of persistent warps.  Each warp streams its range
// two vectors per lane per side per step, copied by the lane itself with
// 16-byte cp.async into a per-warp shared-memory ring five steps ahead of
// the step it reads (no registers held for loads in flight), and keeps an
// online log-sum-exp state (kld_common.cuh) whose running maximum and argmax are
// warp-uniform: one redux.sync finds a step's maximum, and only a step that
// raises it (a handful per row piece) takes the branch that rescales,
// locates the new argmax and leaves it out of the sum.  Every other step is
// two ex2 per element pair on paired f32x2 arithmetic.  A warp writes one
// partial state per row it touches to the workspace; a second kernel merges
// each row's pieces in index order (one warp per row), adds the ragged tail
// and forms the outputs.  No barrier is shared between warps of the
// streaming kernel, and every merge order is fixed, so results are bitwise
// reproducible.
//
// Sources: "Qwen3.8-27B Quantization Challenge", sections "How the
// references were made" (full 248,320-token distribution in f32) and "The
// score" (KL over cells); "Qwopus3.8-27B-Coder-Flash: quality-eval
// reference", "Method" (exact argmax top-1, perplexity from the true-token
// log-prob).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cfloat>
#include <mutex>

#include "kld_common.cuh"
#include "launch.h"
#include "stream_common.cuh"

namespace kld {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kStepVecs = 64;                    // vectors a warp covers per step
constexpr int kMinVecsPerWarp = 8 * kStepVecs;   // below this, use fewer warps
constexpr int kMaxStreamWarps = kFullVocabMaxWarps;
constexpr int kFlushSteps = 16;                  // steps whose sums meet before joining the row's

// Partial state of one warp over one row piece (32 bytes).
struct Piece {
  float mx, rx;
  int ax;
  float my, ry;
  int ay;
  float A;
  int pad;
};

struct StreamParams {
  const void* x;
  const void* y;
  int64_t ld_x, ld_y;  // elements
  int nvec;            // full 16-byte vectors per row
  int nwarps;
  int64_t total;       // n_rows * nvec
  Piece* pieces;       // slot row + warp
};

struct MergeParams {
  const void* x;
  const void* y;
  int64_t ld_x, ld_y;
  int vocab, nvec, n_rows, nwarps;
  int64_t total;
  const Piece* pieces;
  const int32_t* targets;
  float* kl;
  int32_t* ax;
  int32_t* ay;
  float* lpx;
  float* lpy;
  int32_t* dev_status;
};

// One step of a lane: two consecutive-in-warp vectors of each side.
struct StepRaw {
  uint4 x0, y0, x1, y1;
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

// Accumulate one step: weights exp(z - m) 2^-rho on paired f32x2 arithmetic
// (see Offset; cx, cy are the sides' offsets c).  With
// kMasked, the slots ex_x / ex_y (the new argmaxes) are weighed as -inf so
// they stay out of r; the reference argmax's own A term, 1 * (x - y), is
// added by the caller.
template <bool kBF16, bool kMasked, bool kExact>
__device__ __forceinline__ void accumulate(const StepRaw& raw, float cx, float cy, int ex_x, int ex_y,
                                           float2& rx2, float2& ry2, float2& a2) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  const float2 nmx = make_float2(cx, cx);
  const float2 nmy = make_float2(cy, cy);
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
      // x log2(e) + c, one rounding (exact offsets: (x - m) log2(e))
      const float2 tx = kExact ? __fmul2_rn(__fadd2_rn(XW, nmx), l2) : __ffma2_rn(XW, l2, nmx);
      const float2 ty = kExact ? __fmul2_rn(__fadd2_rn(YW, nmy), l2) : __ffma2_rn(YW, l2, nmy);
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


// Stream vectors [a, b) of one row; returns the warp's partial state
// (identical in every lane).
// 16-byte asynchronous copy global -> shared (cached in L2 only), and the
// group bookkeeping of such copies
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((unsigned)__cvta_generic_to_shared(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_four() { asm volatile("cp.async.wait_group 4;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
constexpr int kRingSteps = 6;  // steps a warp's ring holds: the one read, five in flight

template <bool kBF16>
__device__ __forceinline__ Piece stream_piece(const char* xrow, const char* yrow, int a, int b, int lane,
                                              uint4* ring) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  constexpr uint32_t kNegInfWord = kBF16 ? 0xff80ff80u : 0xff800000u;
  const uint4 neg_inf = make_uint4(kNegInfWord, kNegInfWord, kNegInfWord, kNegInfWord);

  // Sums on two levels of f32: lanes add each step's weights into rx2, ry2,
  // a2 (formed with the sides' offsets), which join the side's r and aA
  // (times the offsets' fix) every kFlushSteps steps and whenever a maximum
  // moves.  No f32 sum then has more than about a hundred terms however long
  // the row: a row's thousands of terms in one running sum lost up to 1e-5 of
  // a target log-prob.
  WarpSide sx{-CUDART_INF_F, -1, 0.f}, sy{-CUDART_INF_F, -1, 0.f};
  Offset ox{0.f, 1.f, false}, oy{0.f, 1.f, false};
  float2 rx2 = make_float2(0.f, 0.f), ry2 = rx2, a2 = rx2;
  float aA = 0.f;
  int since = 0;
  auto fold = [&]() {
    sx.r += (rx2.x + rx2.y) * ox.fix;
    sy.r += (ry2.x + ry2.y) * oy.fix;
    aA += (a2.x + a2.y) * ox.fix;
    rx2 = ry2 = a2 = make_float2(0.f, 0.f);
    since = 0;
  };

  const int n = b - a;
  const int nfull = n / kStepVecs;
  const char* xl = xrow + (int64_t)(a + lane) * 16;
  const char* yl = yrow + (int64_t)(a + lane) * 16;

  auto step = [&](const StepRaw& cur, int st) {
    const float CMX = warp_max(El::vmax2(cur.x0, cur.x1));
    const float CMY = warp_max(El::vmax2(cur.y0, cur.y1));
    if (!((CMX > sx.m) || (CMY > sy.m) || (sx.a < 0) || (sy.a < 0))) {  // warp-uniform
      if (!ox.exact) accumulate<kBF16, false, false>(cur, ox.c, oy.c, -1, -1, rx2, ry2, a2);
      else accumulate<kBF16, false, true>(cur, ox.c, oy.c, -1, -1, rx2, ry2, a2);
    } else {
      // the per-vector maxima locate a new maximum (rare: computed only here)
      const float cx0 = El::vmax(cur.x0), cx1 = El::vmax(cur.x1);
      const float cy0 = El::vmax(cur.y0), cy1 = El::vmax(cur.y1);
      // a new maximum on either side, or a side still without a finite
      // value: fold the step sums in, move to the new maxima, weigh the step
      // with the new argmaxes masked out of r
      fold();
      const int i0 = (a + st * kStepVecs + lane) * E;
      const int i1 = i0 + 32 * E;
      int ex_x, ex_y;
      const float scx = side_new_max<kBF16>(sx, CMX, cur.x0, cur.x1, cx0, cx1, i0, i1, lane, ex_x);
      side_new_max<kBF16>(sy, CMY, cur.y0, cur.y1, cy0, cy1, i0, i1, lane, ex_y);
      aA *= scx;
      if (ex_x >= 0) aA += slot_diff<kBF16>(cur, ex_x);
      // a side with no finite value yet has only -inf (weight 0) or NaN
      // (poisons r, marking the row invalid); any finite offset serves
      offsets_of(sx, sy, ox, oy);
      if (!ox.exact) accumulate<kBF16, true, false>(cur, ox.c, oy.c, ex_x, ex_y, rx2, ry2, a2);
      else accumulate<kBF16, true, true>(cur, ox.c, oy.c, ex_x, ex_y, rx2, ry2, a2);
    }
    if (++since == kFlushSteps) fold();  // warp-uniform
  };

  // full steps: each lane copies its four 16-byte vectors of step st + 5
  // into the warp's shared-memory ring (cp.async: no registers held) before
  // step st is processed, so five steps of loads are in flight per warp
  auto issue = [&](int s) {
    const int64_t o = (int64_t)s * kStepVecs * 16;
    uint4* r = ring + (s % kRingSteps) * 4 * 32 + lane;
    cp_async16(r, xl + o);
    cp_async16(r + 32, yl + o);
    cp_async16(r + 64, xl + o + 32 * 16);
    cp_async16(r + 96, yl + o + 32 * 16);
  };
  StepRaw A;
  int st = 0;
  if (nfull > 0) issue(0);
  cp_async_commit();
  if (nfull > 1) issue(1);
  cp_async_commit();
  if (nfull > 2) issue(2);
  cp_async_commit();
  if (nfull > 3) issue(3);
  cp_async_commit();
  if (nfull > 4) issue(4);
  cp_async_commit();
  for (; st < nfull; ++st) {
    cp_async_wait_four();  // every group but the four newest has landed: step st is in the ring
    const uint4* r = ring + (st % kRingSteps) * 4 * 32 + lane;
    A.x0 = r[0];
    A.y0 = r[32];
    A.x1 = r[64];
    A.y1 = r[96];
    if (st + 5 < nfull) issue(st + 5);  // into the slot read one step ago
    cp_async_commit();
    step(A, st);
  }
  cp_async_wait_all();
  // ragged last step: lanes past b read -inf
  if (st * kStepVecs < n) {
    const int v0 = st * kStepVecs + lane, v1 = v0 + 32;
    const int64_t o = (int64_t)st * kStepVecs * 16;
    A.x0 = v0 < n ? ld_stream(xl + o) : neg_inf;
    A.y0 = v0 < n ? ld_stream(yl + o) : neg_inf;
    A.x1 = v1 < n ? ld_stream(xl + o + 32 * 16) : neg_inf;
    A.y1 = v1 < n ? ld_stream(yl + o + 32 * 16) : neg_inf;
    step(A, st);
  }

  fold();
  float rxs = sx.r;
  float rys = sy.r;
  float as = aA;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    rxs += __shfl_xor_sync(0xffffffffu, rxs, off);
    rys += __shfl_xor_sync(0xffffffffu, rys, off);
    as += __shfl_xor_sync(0xffffffffu, as, off);
  }
  return Piece{sx.m, rxs, sx.a, sy.m, rys, sy.a, as, 0};
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads, kStreamCtasPerSm) stream_kernel(const StreamParams p) {
  constexpr int kElemBytes = kBF16 ? 2 : 4;
  extern __shared__ __align__(16) uint4 rings_dyn[];
  uint4 (*rings)[kRingSteps * 4 * 32] = reinterpret_cast<uint4 (*)[kRingSteps * 4 * 32]>(rings_dyn);
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
    const char* xrow = reinterpret_cast<const char*>(p.x) + (int64_t)row * p.ld_x * kElemBytes;
    const char* yrow = reinterpret_cast<const char*>(p.y) + (int64_t)row * p.ld_y * kElemBytes;
    const Piece pc = stream_piece<kBF16>(xrow, yrow, a, b, lane, rings[threadIdx.x >> 5]);
    if (lane == 0) p.pieces[row + w] = pc;
    pos = row0 + b;
  }
}

__device__ __forceinline__ RowState piece_state(const Piece& pc) {
  RowState s;
  s.x = Side{pc.mx, pc.rx, pc.ax};
  s.y = Side{pc.my, pc.ry, pc.ay};
  s.A = pc.A;
  s.bad = 0;
  return s;
}

// One warp per row: merge the row's pieces in warp (= index) order, push the
// ragged tail ids, gather the target logits and write the outputs.
template <bool kBF16>
__global__ void __launch_bounds__(kThreads) merge_kernel(const MergeParams p) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  constexpr int kElemBytes = kBF16 ? 2 : 4;
  wait_prior_grid();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (row >= p.n_rows) return;
  const char* xrow = reinterpret_cast<const char*>(p.x) + (int64_t)row * p.ld_x * kElemBytes;
  const char* yrow = reinterpret_cast<const char*>(p.y) + (int64_t)row * p.ld_y * kElemBytes;

  // the target logits first: their two dependent loads overlap the merge
  bool have_t = false, bad_t = false;
  float xt = 0.f, yt = 0.f;
  if (p.targets) {
    const int tg = p.targets[row];
    if (tg >= 0 && tg < p.vocab) {
      have_t = true;
      xt = El::load1(xrow, tg);
      yt = El::load1(yrow, tg);
    } else {
      bad_t = true;
    }
  }

  RowState acc = row_empty();
  if (p.nvec > 0) {
    const int64_t f = (int64_t)row * p.nvec;
    const int w0 = warp_of(f, p.total, p.nwarps);
    const int w1 = warp_of(f + p.nvec - 1, p.total, p.nwarps);
    for (int c = w0; c <= w1; c += 32) {
      const int w = c + lane;
      RowState s = (w <= w1) ? piece_state(p.pieces[row + w]) : row_empty();
      s = warp_merge_row(s);
      acc = (c == w0) ? s : row_merge(acc, s);
    }
  }
  if (lane != 0) return;
  for (int i = p.nvec * E; i < p.vocab; ++i) {
    const float xv = El::load1(xrow, i), yv = El::load1(yrow, i);
    float wx, scx, wy, scy;
    side_push(acc.x, xv, i, wx, scx, acc.bad);
    side_push(acc.y, yv, i, wy, scy, acc.bad);
    acc.A = acc.A * scx + wx * fmaxf(xv - yv, -FLT_MAX);
  }
  if (bad_t) set_dev_status(p.dev_status, 0x1 /* KLD_DEV_BAD_TARGET */);
  const RowOut o = row_finish(acc, have_t, xt, yt);
  p.kl[row] = o.kl;
  if (p.ax) p.ax[row] = o.ax;
  if (p.ay) p.ay[row] = o.ay;
  if (p.lpx) p.lpx[row] = o.lp_x;
  if (p.lpy) p.lpy[row] = o.lp_y;
}

int stream_warps(int64_t total, int override_warps) {
  if (override_warps > 0) {
    int64_t w = override_warps < kMaxStreamWarps ? override_warps : kMaxStreamWarps;
    return (int)(w < total ? w : (total > 0 ? total : 1));
  }
  int64_t w = total / kMinVecsPerWarp;
  if (w < 1) w = 1;
  if (w > kMaxStreamWarps) w = kMaxStreamWarps;
  return (int)w;
}

// Library-owned scratch for kld_full_vocab_noalloc: room for the row pieces
// of up to kNoAllocMaxRows rows.  Every device that loads this module holds
// it until the process exits; all calls on a device share it.
constexpr int64_t kNoAllocRows = kNoAllocMaxRows;
static __device__ __align__(256) unsigned char g_noalloc_scratch[sizeof(Piece) * (kNoAllocRows + kMaxStreamWarps)];

}  // namespace

namespace {

// A process-unique id of the context current on this thread (a context made
// again after a device reset gets a new one).  False when there is no
// current context or the driver cannot tell.
bool current_context_id(unsigned long long* id) {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t noalloc_scratch(void** ptr, size_t* bytes) {
  // Host code cannot use g_noalloc_scratch's name as a device address: look
  // the address up with the device current and cache it, per device, for the
  // context it was found in; a different context (e.g. after a device reset)
  // looks it up again.
  constexpr int kMaxDevices = 64;
  struct Entry {
    unsigned long long ctx_id;
    void* ptr;
  };
  static std::mutex mu;
  static Entry cached[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(mu);
  if (!have_id || cached[dev].ptr == nullptr || cached[dev].ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the device's context current if it was not
    if (e != cudaSuccess) return e;
    if (!have_id) have_id = current_context_id(&id);
    cached[dev] = Entry{have_id ? id : 0ull, have_id ? p : nullptr};  // unknown context: look up every call
    *ptr = p;
  } else {
    *ptr = cached[dev].ptr;
  }
  *bytes = sizeof(g_noalloc_scratch);
  return cudaSuccess;
}

size_t full_vocab_workspace_bytes(int64_t n_rows) {
  return sizeof(Piece) * (size_t)(n_rows + kMaxStreamWarps);
}

cudaError_t launch_full_vocab(const FullVocabArgs& a, cudaStream_t stream) {
  const int E = a.bf16 ? 8 : 4;
  const int nvec = (int)(a.vocab / E);
  const int64_t total = a.n_rows * (int64_t)nvec;
  const int nwarps = stream_warps(total, a.warps_override);
  Piece* pieces = reinterpret_cast<Piece*>(a.workspace);
  if (total > 0) {
    StreamParams sp{a.x, a.y, a.ld_x, a.ld_y, nvec, nwarps, total, pieces};
    const unsigned grid = (unsigned)((nwarps + kWarpsPerCta - 1) / kWarpsPerCta);
    constexpr size_t kRingBytes = sizeof(uint4) * kWarpsPerCta * kRingSteps * 4 * 32;
    if (a.bf16) {
      cudaError_t e0 = allow_dynamic_smem<stream_kernel<true>>(kRingBytes);
      if (e0 != cudaSuccess) return e0;
      stream_kernel<true><<<grid, kThreads, kRingBytes, stream>>>(sp);
    } else {
      cudaError_t e0 = allow_dynamic_smem<stream_kernel<false>>(kRingBytes);
      if (e0 != cudaSuccess) return e0;
      stream_kernel<false><<<grid, kThreads, kRingBytes, stream>>>(sp);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  MergeParams mp{a.x, a.y, a.ld_x, a.ld_y, (int)a.vocab, nvec, (int)a.n_rows, nwarps, total, pieces,
                 a.targets, a.kl, a.ax, a.ay, a.lpx, a.lpy, a.dev_status};
  const unsigned mgrid = (unsigned)((a.n_rows + kWarpsPerCta - 1) / kWarpsPerCta);
  if (a.bf16) return launch_dependent(merge_kernel<true>, dim3(mgrid), dim3(kThreads), stream, mp);
  return launch_dependent(merge_kernel<false>, dim3(mgrid), dim3(kThreads), stream, mp);
}

}  // namespace kld
