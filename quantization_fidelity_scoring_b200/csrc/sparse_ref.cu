// Candidate full logits against a sparse reference: KL over the reference's
// K listed ids plus one tail cell.
//
// "Qwen3.8-27B Quantization Challenge", "Golden distributions": the
// reference keeps, per position, its K most likely ids with f32 log p (most
// likely first) and the tail mass of the rest of its full row.  "The score":
// the candidate's q = softmax(y) over the whole vocabulary is coarsened onto
// the K listed ids plus one cell holding the rest of q's mass, and
// KL(p || q) = sum over cells p_c (log p_c - log q_c).
//
// The tail cell is not formed as 1 - sum_R q: when the listed ids hold all
// but ~1e-6 of the mass that difference cancels down to the rounding error
// of the row sum.  Instead the streaming pass masks the listed ids out of
// the row, so its online state (running max, argmax, sum of the other
// weights; kld_common.cuh) covers the unlisted ids only and yields the tail
// mass T directly, and the merge forms, in f64,
//     m = max(tail max, listed max),  S = sum_R e^{y_j - m} + T e^{m_T - m},
//     log q_j = y_j - m - log S,       q_tail = T e^{m_T - m} / S.
//
// Pass 1 (persistent warps over the flattened (row, 16-byte vector) space,
// as the full-vocabulary kernel): for each row piece a warp buckets the
// listed ids that fall in the piece by streaming step (a counting sort in
// shared memory, 256 steps at a time); a repeated id shows up twice in one
// bucket and flags the row.  A step that holds listed ids is staged through
// shared memory, where up to 32 of its ids at once have their logits written
// to the workspace and replaced by -inf, before the step's maximum and
// weights are taken.  Pass 2 (one warp per row) merges the pieces in index
// order, adds the ragged end of the row, reads the listed logits and forms
// the outputs.
#include <cuda_bf16.h>
#include <cfloat>

#include "kld_common.cuh"
#include "launch.h"
#include "stream_common.cuh"

namespace kld {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kMergeThreads = 128;           // one warp per row, four rows per CTA
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kVecs = 4;                         // 16-byte vectors per lane per step
constexpr int kStepVecs = 32 * kVecs;            // vectors per warp step
constexpr int kMinVecsPerWarp = 4 * kStepVecs;
constexpr int kStreamCtasPerSm = 3;
constexpr int kMaxStreamWarps = 148 * kStreamCtasPerSm * kWarpsPerCta;
constexpr int kWin = 256;                        // steps per bucket window
constexpr int kFlushSteps = 16;                  // steps whose sums meet before joining the piece's
constexpr int kMaxK = KLD_SPARSE_MAX_K;
constexpr int kFlagRepeat = 1;
constexpr uint32_t kSkip = 0x80000000u;
constexpr double kQFloor = 1e-12;

// Tail state of one warp over one row piece (16 bytes).
struct TailPiece {
  float m, r;
  int a;
  int flags;
};

struct StreamParams {
  const void* y;
  int64_t ld;     // elements
  int nvec;       // full 16-byte vectors per row
  int nwarps;
  int64_t total;  // n_rows * nvec
  const int2* top;  // [n_rows, K] (id, f32 log-prob bits)
  int K;
  float* gy;         // [n_rows, K] listed logits
  TailPiece* pieces; // slot row + warp
};

struct MergeParams {
  const void* y;
  int64_t ld;
  int vocab, nvec, n_rows, nwarps;
  int64_t total;
  const TailPiece* pieces;
  const int2* top;
  int K;
  const float* gy;
  const float* ref_rows;  // [n_rows, 3] or null
  const int32_t* targets;
  float* kl;
  int32_t* argmax;
  uint8_t* top1;
  float* lp_cand;
  float* lp_ref;
  int32_t* dev_status;
};

// Per-warp shared memory (6 KB): the bucketed list of a window, and either
// the bucket counts (while the list is built) or one step's vectors (while
// the listed elements of that step are captured and masked).
struct WarpLists {
  // (step in window << 20) | (element in step << 10) | list slot, and
  // kSkip on the later copies of a repeated id
  uint32_t entry[kMaxK];
  union {
    uint32_t count[kWin + 1];
    uint4 stage[kStepVecs];
  };
};
static_assert(sizeof(uint32_t) * (kWin + 1) <= sizeof(uint4) * kStepVecs, "counts fit in the stage");

// Weights exp(y - m) 2^-rho of a lane's step (one paired FMA per pair for
// the exponent, y log2 e + c; see Offset; with kExact (y - m) log2 e),
// added to r2.  With kMasked the
// element slot `excl` (a new argmax) is weighed as -inf.
template <bool kBF16, bool kMasked, bool kExact>
__device__ __forceinline__ void accumulate(const uint4 (&v)[kVecs], float c, int excl, float2& r2) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  const float2 nm = make_float2(c, c);
  const float2 l2 = make_float2(kLog2e, kLog2e);
#pragma unroll
  for (int q = 0; q < kVecs; ++q) {
#pragma unroll
    for (int k = 0; k < E / 2; ++k) {
      float2 Y = El::pair(v[q], k);
      if (kMasked) {
        if (excl == q * E + 2 * k) Y.x = -CUDART_INF_F;
        if (excl == q * E + 2 * k + 1) Y.y = -CUDART_INF_F;
      }
      const float2 t = kExact ? __fmul2_rn(__fadd2_rn(Y, nm), l2) : __ffma2_rn(Y, l2, nm);
      r2 = __fadd2_rn(r2, make_float2(ex2(t.x), ex2(t.y)));
    }
  }
}

// Bucket the listed ids of elements [elo, ehi) by step (kStepVecs * E
// elements each) for the window's steps; returns the number of entries and
// sets `repeat` when an id is listed twice.  Entries of one step are
// contiguous; their order inside a step is not fixed and does not matter.
__device__ int build_window(WarpLists& L, const int2* top, int K, int64_t elo, int64_t ehi, int step_elems,
                            int lane, bool& repeat) {
  for (int s = lane; s <= kWin; s += 32) L.count[s] = 0u;
  __syncwarp();
  for (int j = lane; j < K; j += 32) {
    const int64_t id = top[j].x;
    if (id >= elo && id < ehi) atomicAdd(&L.count[(int)((id - elo) / step_elems)], 1u);
  }
  __syncwarp();
  // exclusive scan of count[0 .. kWin): lane l owns steps 8l .. 8l+7
  uint32_t c[kWin / 32];
  uint32_t run = 0;
#pragma unroll
  for (int i = 0; i < kWin / 32; ++i) {
    c[i] = L.count[lane * (kWin / 32) + i];
    run += c[i];
  }
  uint32_t incl = run;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const int total = (int)__shfl_sync(0xffffffffu, incl, 31);
  uint32_t base = incl - run;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < kWin / 32; ++i) {
    L.count[lane * (kWin / 32) + i] = base;  // now the write cursor of the step
    base += c[i];
  }
  __syncwarp();
  for (int j = lane; j < K; j += 32) {
    const int64_t id = top[j].x;
    if (id >= elo && id < ehi) {
      const int64_t rel = id - elo;
      const int s = (int)(rel / step_elems);
      const uint32_t pos = atomicAdd(&L.count[s], 1u);
      L.entry[pos] = ((uint32_t)s << 20) | ((uint32_t)(rel - (int64_t)s * step_elems) << 10) | (uint32_t)j;
    }
  }
  __syncwarp();
  // a repeated id lands twice in one bucket: compare every entry with the
  // later entries of its bucket (count[s] now holds the bucket's end) and
  // mark the later copies, which then record -inf instead of the logit so
  // the row's sums hold the id once
  bool rep = false;
  for (int i = lane; i < total; i += 32) {
    const uint32_t key = (L.entry[i] >> 10) & 0x3ffffu;
    const int end = (int)L.count[key >> 10];
    for (int t = i + 1; t < end; ++t) {
      if (((L.entry[t] >> 10) & 0x3ffffu) == key) {
        rep = true;
        atomicOr(&L.entry[t], kSkip);
      }
    }
  }
  repeat = __any_sync(0xffffffffu, rep);
  __syncwarp();
  return total;
}

// Stream vectors [a, b) of one row with its listed ids masked out; returns
// the warp's tail state (identical in every lane).
template <bool kBF16>
__device__ TailPiece stream_piece(const StreamParams& p, WarpLists& L, int row, int a, int b, int lane) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  constexpr int kStepElems = kStepVecs * E;
  constexpr uint32_t kNegInfWord = kBF16 ? 0xff80ff80u : 0xff800000u;
  const uint4 neg_inf = make_uint4(kNegInfWord, kNegInfWord, kNegInfWord, kNegInfWord);
  constexpr int kElemBytes = kBF16 ? 2 : 4;
  const char* yrow = reinterpret_cast<const char*>(p.y) + (int64_t)row * p.ld * kElemBytes;
  const int2* top = p.top + (int64_t)row * p.K;
  float* gy = p.gy + (int64_t)row * p.K;

  // r2 holds the lane's step weights (formed with the offset o) for at most
  // kFlushSteps steps, then joins s.r times o.fix: no f32 sum gets more than
  // about a hundred terms however long the row
  WarpSide s{-CUDART_INF_F, -1, 0.f};
  Offset o{0.f, 1.f, false};
  float2 r2 = make_float2(0.f, 0.f);
  int since = 0;
  auto fold = [&]() {
    s.r += (r2.x + r2.y) * o.fix;
    r2 = make_float2(0.f, 0.f);
    since = 0;
  };
  int flags = 0;
  const int n = b - a;
  const int nsteps = (n + kStepVecs - 1) / kStepVecs;
  const char* yl = yrow + (int64_t)(a + lane) * 16;

  for (int w0 = 0; w0 < nsteps; w0 += kWin) {
    const int64_t elo = (int64_t)(a + w0 * kStepVecs) * E;
    const int wend = min(nsteps, w0 + kWin);
    const int64_t ehi = (int64_t)min(b, a + wend * kStepVecs) * E;
    bool repeat;
    const int cnt = build_window(L, top, p.K, elo, ehi, kStepElems, lane, repeat);
    flags |= repeat ? kFlagRepeat : 0;
    int ptr = 0;
    // one step of loads stays in flight while the previous step is processed
    auto load_step = [&](int st, uint4 (&v)[kVecs]) {
      const int64_t o = (int64_t)st * kStepVecs * 16;
      if ((st + 1) * kStepVecs <= n) {
#pragma unroll
        for (int q = 0; q < kVecs; ++q) v[q] = ld_stream(yl + o + q * 32 * 16);
      } else {
#pragma unroll
        for (int q = 0; q < kVecs; ++q) v[q] = (st * kStepVecs + lane + 32 * q < n) ? ld_stream(yl + o + q * 32 * 16)
                                                                                   : neg_inf;
      }
    };
    uint4 nx[kVecs];
    load_step(w0, nx);
    for (int st = w0; st < wend; ++st) {
      uint4 v[kVecs];
#pragma unroll
      for (int q = 0; q < kVecs; ++q) v[q] = nx[q];
      if (st + 1 < wend) load_step(st + 1, nx);
      // listed ids of this step: stage the step's vectors so that element
      // `off` of the step has a fixed shared-memory address (vector v of the
      // step is lane v % 32's vector v / 32), capture and mask up to 32 ids
      // at once, and reload
      if (ptr < cnt && (int)((L.entry[ptr] >> 20) & 0xffu) == st - w0) {
#pragma unroll
        for (int q = 0; q < kVecs; ++q) L.stage[lane + 32 * q] = v[q];
        __syncwarp();
        for (;;) {
          const int i = ptr + lane;
          const uint32_t e = (i < cnt) ? L.entry[i] : 0xffffffffu;
          const bool act = (i < cnt) && (int)((e >> 20) & 0xffu) == st - w0;
          if (act && (e & kSkip)) {
            gy[e & 1023u] = -CUDART_INF_F;
          } else if (act) {
            const int off = (int)((e >> 10) & 1023u);
            if (kBF16) {
              unsigned short* el = reinterpret_cast<unsigned short*>(L.stage) + off;
              gy[e & 1023u] = __uint_as_float((uint32_t)*el << 16);
              *el = (unsigned short)0xff80u;
            } else {
              uint32_t* el = reinterpret_cast<uint32_t*>(L.stage) + off;
              gy[e & 1023u] = __uint_as_float(*el);
              *el = 0xff800000u;
            }
          }
          const int nact = __popc(__ballot_sync(0xffffffffu, act));
          ptr += nact;
          if (nact < 32) break;
        }
        __syncwarp();
#pragma unroll
        for (int q = 0; q < kVecs; ++q) v[q] = L.stage[lane + 32 * q];
      }
      float c[kVecs];
      float cm = -CUDART_INF_F;
#pragma unroll
      for (int q = 0; q < kVecs; ++q) {
        c[q] = El::vmax(v[q]);
        cm = fmaxf(cm, c[q]);
      }
      const float CM = warp_max(cm);
      if (!(CM > s.m)) {  // warp-uniform: the common step
        if (!o.exact) accumulate<kBF16, false, false>(v, o.c, -1, r2);
        else accumulate<kBF16, false, true>(v, o.c, -1, r2);
        if (++since == kFlushSteps) fold();
        continue;
      }
      // a new maximum: fold the pair sums, rescale to the new maximum, hand
      // the old maximum's own term to lane 0, find the first occurrence
      fold();
      const float sc = (s.a < 0) ? 0.f : ex2((s.m - CM) * kLog2e);
      s.r = s.r * sc + ((lane == 0 && s.a >= 0) ? sc : 0.f);
      int part = kVecs - 1, src = 0;
#pragma unroll
      for (int q = kVecs - 1; q >= 0; --q) {
        const unsigned bq = __ballot_sync(0xffffffffu, c[q] == CM);
        if (bq) {
          part = q;
          src = __ffs(bq) - 1;
        }
      }
      int idx = 0, excl = -1;
      if (lane == src) {
        uint4 vv = v[0];
#pragma unroll
        for (int q = 1; q < kVecs; ++q)
          if (q == part) vv = v[q];
        int jj = E - 1;
#pragma unroll
        for (int k = E / 2 - 1; k >= 0; --k) {
          const float2 pr = El::pair(vv, k);
          if (pr.y == CM) jj = 2 * k + 1;
          if (pr.x == CM) jj = 2 * k;
        }
        excl = part * E + jj;
        idx = (a + st * kStepVecs + src + 32 * part) * E + jj;
      }
      s.a = __shfl_sync(0xffffffffu, idx, src);
      s.m = CM;
      o = offset_of(s);
      if (!o.exact) accumulate<kBF16, true, false>(v, o.c, excl, r2);
      else accumulate<kBF16, true, true>(v, o.c, excl, r2);
    }
    __syncwarp();  // the lists are rebuilt for the next window
  }
  fold();
  float rs = s.r;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
  flags = __reduce_or_sync(0xffffffffu, flags);
  return TailPiece{s.m, rs, s.a, flags};
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads, kStreamCtasPerSm) sparse_stream_kernel(const StreamParams p) {
  __shared__ WarpLists lists[kWarpsPerCta];
  const int lane = threadIdx.x & 31;
  const int wl = threadIdx.x >> 5;
  const int w = blockIdx.x * kWarpsPerCta + wl;
  if (w >= p.nwarps) return;  // the whole warp leaves together
  int64_t pos = warp_begin(w, p.total, p.nwarps);
  const int64_t end = warp_begin(w + 1, p.total, p.nwarps);
  while (pos < end) {
    const int row = (int)(pos / p.nvec);
    const int64_t row0 = (int64_t)row * p.nvec;
    const int a = (int)(pos - row0);
    const int b = (int)min((int64_t)p.nvec, end - row0);
    const TailPiece pc = stream_piece<kBF16>(p, lists[wl], row, a, b, lane);
    if (lane == 0) p.pieces[row + w] = pc;
    pos = row0 + b;
  }
}

// Merge of two tail states in index order (lower first on equal maxima).
__device__ __forceinline__ TailPiece tail_merge(const TailPiece& p, const TailPiece& q) {
  float sc;
  int win;
  const Side s = side_merge(Side{p.m, p.r, p.a}, Side{q.m, q.r, q.a}, sc, win);
  return TailPiece{s.m, s.r, s.a, p.flags | q.flags};
}

__device__ __forceinline__ TailPiece shfl_xor_tail(const TailPiece& s, int mask) {
  return TailPiece{__shfl_xor_sync(0xffffffffu, s.m, mask), __shfl_xor_sync(0xffffffffu, s.r, mask),
                   __shfl_xor_sync(0xffffffffu, s.a, mask), __shfl_xor_sync(0xffffffffu, s.flags, mask)};
}

__device__ __forceinline__ TailPiece warp_merge_tail(TailPiece s) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const TailPiece o = shfl_xor_tail(s, off);
    s = (lane & off) ? tail_merge(o, s) : tail_merge(s, o);
  }
  return s;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// One warp per row.
template <bool kBF16>
__global__ void __launch_bounds__(kMergeThreads) sparse_merge_kernel(const MergeParams p) {
  using El = Elems<kBF16>;
  constexpr int E = El::E;
  constexpr int kElemBytes = kBF16 ? 2 : 4;
  __shared__ float ys[kMergeWarps][kMaxK];   // listed ids, then listed logits
  __shared__ float lps[kMergeWarps][kMaxK];  // listed reference log-probs
  const int lane = threadIdx.x & 31;
  const int wl = threadIdx.x >> 5;
  const int row = blockIdx.x * kMergeWarps + wl;
  const bool live = row < p.n_rows;
  const char* yrow = reinterpret_cast<const char*>(p.y) + (int64_t)row * p.ld * kElemBytes;
  const int2* top = p.top + (int64_t)row * p.K;
  const float* gy = p.gy + (int64_t)row * p.K;
  float* ysw = ys[wl];
  float* lpw = lps[wl];
  const int64_t listed_end = (int64_t)p.nvec * E;  // ids below this were captured by the stream

  // Before the streaming pass is waited for, only its inputs are read: the
  // target logit (two dependent loads) and the reference entries, whose
  // validity is checked here
  const int tgt = (live && p.lp_cand) ? p.targets[row] : -1;
  const bool tgt_ok = tgt >= 0 && tgt < p.vocab;
  const float y_tgt = (p.lp_cand && tgt_ok) ? El::load1(yrow, tgt) : 0.f;
  bool bad = false;   // an id outside [0, V), or a repeated id
  if (live) {
#pragma unroll 8
    for (int j = lane; j < p.K; j += 32) {
      const int2 t = top[j];
      bad |= t.x < 0 || t.x >= p.vocab;
      ysw[j] = __int_as_float(t.x);
      lpw[j] = __int_as_float(t.y);
    }
  }
  wait_prior_grid();
  if (!live) return;

  // tail state of the unlisted ids covered by the stream
  TailPiece acc{-CUDART_INF_F, 0.f, -1, 0};
  if (p.nvec > 0) {
    const int64_t f = (int64_t)row * p.nvec;
    const int w0 = warp_of(f, p.total, p.nwarps);
    const int w1 = warp_of(f + p.nvec - 1, p.total, p.nwarps);
    for (int c = w0; c <= w1; c += 32) {
      const int w = c + lane;
      TailPiece s = (w <= w1) ? p.pieces[row + w] : TailPiece{-CUDART_INF_F, 0.f, -1, 0};
      s = warp_merge_tail(s);
      acc = (c == w0) ? s : tail_merge(acc, s);
    }
  }

  // listed logits (the stream captured those below listed_end); the listed maximum
  bool nan = false;
  float lm = -CUDART_INF_F;
#pragma unroll 8
  for (int j = lane; j < p.K; j += 32) {
    const int id = __float_as_int(ysw[j]);
    const float g = gy[j];
    float y = -CUDART_INF_F;
    if (id >= 0 && id < p.vocab) y = (id < listed_end) ? g : El::load1(yrow, id);
    nan |= (y != y);
    lm = fmaxf(lm, y);
    ysw[j] = y;
  }
  __syncwarp();
  bad = __any_sync(0xffffffffu, bad) || (acc.flags & kFlagRepeat);

  // ragged end of the row: ids at or past listed_end, pushed in index order
  // by lane 0 unless listed; a listed id there is checked for repeats
  int tail_nan = 0;
  if (listed_end < p.vocab) {
    for (int64_t i = listed_end; i < p.vocab; ++i) {
      int hits = 0;
      for (int j = lane; j < p.K; j += 32) hits += (top[j].x == i) ? 1 : 0;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) hits += __shfl_xor_sync(0xffffffffu, hits, off);
      bad |= hits > 1;
      if (lane == 0 && hits == 0) {
        float w, sc;
        Side s{acc.m, acc.r, acc.a};
        side_push(s, El::load1(yrow, i), (int)i, w, sc, tail_nan);
        acc.m = s.m;
        acc.r = s.r;
        acc.a = s.a;
      }
    }
    acc.m = __shfl_sync(0xffffffffu, acc.m, 0);
    acc.r = __shfl_sync(0xffffffffu, acc.r, 0);
    acc.a = __shfl_sync(0xffffffffu, acc.a, 0);
    tail_nan = __shfl_sync(0xffffffffu, tail_nan, 0);
  }

  // overall maximum and its lowest index
  const float m_listed = key_value(__reduce_max_sync(0xffffffffu, ordered_key(lm)));
  const bool have_tail = acc.a >= 0;
  const float m = have_tail ? fmaxf(acc.m, m_listed) : m_listed;
  int cand = INT32_MAX;
  for (int j = lane; j < p.K; j += 32) {
    if (ysw[j] != m) continue;
    const int id = top[j].x;
    if (id >= 0 && id < cand) cand = id;
  }
  cand = __reduce_min_sync(0xffffffffu, cand);
  if (have_tail && acc.m == m && acc.a < cand) cand = acc.a;
  nan = __any_sync(0xffffffffu, nan) || tail_nan || (acc.r != acc.r);
  const bool valid = !nan && !isinf(m) && cand != INT32_MAX;

  // S = sum_R e^{y_j - m} + T, with T the tail mass relative to m.  The
  // listed weights are ex2 on the MUFU unit (relative error ~1e-7; a
  // maximum's weight is exactly 1, so log S keeps its relative accuracy for
  // near-certain rows), summed in f64.
  double sw = 0.0;
#pragma unroll 4
  for (int j = lane; j < p.K; j += 32) {
    const float y = ysw[j];
    sw += (y == m) ? 1.0 : (double)ex2((y - m) * kLog2e);
  }
  sw = warp_sum(sw);
  const double T = have_tail ? (1.0 + (double)acc.r) * exp((double)acc.m - (double)m) : 0.0;
  const double S = sw + T;
  const double logS = log(S);

  // p_j also from ex2 for the KL terms (in f64 where ex2 underflows, so that
  // every p_j > 0 counts: against a candidate -inf it makes the KL +inf);
  // without a stored tail the reference's tail mass is 1 - sum p_j, which
  // cancels: that sum takes p_j in f64
  const bool need_psum = p.ref_rows == nullptr;
  double kl = 0.0, psum = 0.0;
#pragma unroll 4
  for (int j = lane; j < p.K; j += 32) {
    const float lpf = lpw[j];
    const double lp = (double)lpf;
    const float pf = ex2(lpf * kLog2e);
    const double pj = pf > 0.f ? (double)pf : exp(lp);
    if (need_psum) psum += exp(lp);
    if (pj > 0.0) kl += pj * (lp - (((double)ysw[j] - (double)m) - logS));
  }
  kl = warp_sum(kl);
  psum = warp_sum(psum);

  if (lane != 0) return;
  float out = CUDART_NAN_F;
  if (valid && !bad) {
    const double p_tail = p.ref_rows ? (double)p.ref_rows[(int64_t)row * 3 + 2] : 1.0 - psum;
    if (p_tail > 0.0) kl += p_tail * (log(p_tail) - log(fmax(T / S, kQFloor)));
    out = (float)kl;
  }
  if (bad) set_dev_status(p.dev_status, 0x2 /* KLD_DEV_BAD_ID */);
  p.kl[row] = out;
  const int am = valid ? cand : -1;
  if (p.argmax) p.argmax[row] = am;
  if (p.top1) p.top1[row] = (uint8_t)(valid && top[0].x == am);
  if (p.lp_cand) {
    float lpc = CUDART_NAN_F;
    if (tgt_ok) {
      if (valid) lpc = (float)(((double)y_tgt - (double)m) - logS);
    } else {
      set_dev_status(p.dev_status, 0x1 /* KLD_DEV_BAD_TARGET */);
    }
    p.lp_cand[row] = lpc;
  }
  if (p.lp_ref) p.lp_ref[row] = -p.ref_rows[(int64_t)row * 3 + 0];
}

int stream_warps(int64_t total, int override_warps) {
  if (override_warps > 0) {
    const int64_t w = override_warps < kMaxStreamWarps ? override_warps : kMaxStreamWarps;
    return (int)(w < total ? w : (total > 0 ? total : 1));
  }
  int64_t w = total / kMinVecsPerWarp;
  if (w < 1) w = 1;
  if (w > kMaxStreamWarps) w = kMaxStreamWarps;
  return (int)w;
}

}  // namespace

size_t sparse_ref_workspace_bytes(int64_t n_rows, int k) {
  const size_t pieces = sizeof(TailPiece) * (size_t)(n_rows + kMaxStreamWarps);
  const size_t gy = sizeof(float) * (size_t)n_rows * (size_t)k;
  return ((pieces + 255) / 256) * 256 + gy;
}

cudaError_t launch_sparse_ref(const SparseRefArgs& a, cudaStream_t stream) {
  const int E = a.bf16 ? 8 : 4;
  const int nvec = (int)(a.vocab / E);
  const int64_t total = a.n_rows * (int64_t)nvec;
  const int nwarps = stream_warps(total, a.warps_override);
  TailPiece* pieces = reinterpret_cast<TailPiece*>(a.workspace);
  const size_t pieces_bytes = ((sizeof(TailPiece) * (size_t)(a.n_rows + kMaxStreamWarps) + 255) / 256) * 256;
  float* gy = reinterpret_cast<float*>(reinterpret_cast<char*>(a.workspace) + pieces_bytes);
  const int2* top = reinterpret_cast<const int2*>(a.ref_top);
  if (total > 0) {
    StreamParams sp{a.y, a.ld, nvec, nwarps, total, top, a.k, gy, pieces};
    const unsigned grid = (unsigned)((nwarps + kWarpsPerCta - 1) / kWarpsPerCta);
    if (a.bf16) sparse_stream_kernel<true><<<grid, kThreads, 0, stream>>>(sp);
    else sparse_stream_kernel<false><<<grid, kThreads, 0, stream>>>(sp);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  MergeParams mp{a.y, a.ld, (int)a.vocab, nvec, (int)a.n_rows, nwarps, total, pieces, top, a.k, gy,
                 a.ref_rows, a.targets, a.kl, a.argmax, a.top1, a.lp_cand, a.lp_ref, a.dev_status};
  const unsigned mgrid = (unsigned)((a.n_rows + kMergeWarps - 1) / kMergeWarps);
  if (total == 0) {  // no streaming pass: the merge reads its inputs at once, so no early launch
    if (a.bf16) sparse_merge_kernel<true><<<mgrid, kMergeThreads, 0, stream>>>(mp);
    else sparse_merge_kernel<false><<<mgrid, kMergeThreads, 0, stream>>>(mp);
    return cudaGetLastError();
  }
  if (a.bf16) return launch_dependent(sparse_merge_kernel<true>, dim3(mgrid), dim3(kMergeThreads), stream, mp);
  return launch_dependent(sparse_merge_kernel<false>, dim3(mgrid), dim3(kMergeThreads), stream, mp);
}

}  // namespace kld
