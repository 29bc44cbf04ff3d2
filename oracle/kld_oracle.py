"""Plain f64 CPU oracle for teacher-forced KL(reference || candidate) scoring.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may call it.  It shares no code with the CUDA path: every
quantity is recomputed here from its definition, in float64, with numpy
library primitives (max, exp, log, sum, sort, matmul) as the only building
blocks.  Inputs are converted exactly to float64 (bf16, fp16 and f32 all
embed exactly in f64) before any arithmetic.

Sources (web pages, cited by title and section):

* "Qwen3.8-27B Quantization Challenge" (dataset card), sections
  "How the references were made" (each position's full 248,320-token
  distribution in f32), "Golden distributions" (NLL, entropy in nats),
  "The score" (KL(p||q) = sum_i p_i (log p_i - log q_i); mean, median, p99,
  p99.9, top-1 agreement, perplexity ratio).
* "Qwen3.8-27B fidelity suite v5", opening paragraph (KLD = KL(BF16 ||
  candidate) from final hidden states through one shared BF16 LM head) and
  "What is in here" (per-shard tail reports: percentiles and exact
  exceedance counts).
* "Qwopus3.8-27B-Coder-Flash: quality-eval reference", sections "Files"
  (top-64 ids + fp16 log-probs sorted, f32 target log-prob) and "Method"
  (top-64 + one tail bucket, uniform spread of the candidate's leftover mass,
  exact argmax top-1, perplexity = exp(mean NLL)).
* "Qwen3.8-27B IQ8R (GPTQ int8, Hadamard-rotated) - radiance container",
  section "Quality" (mean KLD, KLD 99%, KLD 99.9%, top-1 agreement).

Readings where the pages are silent:

* Natural logarithms (entropy is reported in nats).
* 0 * log 0 = 0: vocabulary entries with p_i = 0 contribute nothing.
* p_i > 0 with a candidate logit of -inf gives KL = +inf.
* A row containing NaN or +inf, or no finite logit at all, is invalid:
  KL = NaN, argmax = -1, target log-probs = NaN.
* KL is reported as computed, never clamped at zero.
* Argmax ties resolve to the lowest vocabulary index.
* Tail bucket: p_tail = 1 - sum_R p clamped at 0 (a non-positive tail has
  no term); leftover = 1 - sum_C c clamped at 0; every candidate cell used
  inside a logarithm (the spread cell and q_tail) is floored at Q_FLOOR.
* Percentiles use linear interpolation between order statistics, the
  convention of numpy's default quantile: h = (n - 1) q,
  v = s[floor h] + (s[floor h + 1] - s[floor h]) (h - floor h).
* NaN KL values are excluded from every reduction and counted.
"""
from __future__ import annotations

import math

import numpy as np

# Floor applied to candidate-side tail cells before taking a logarithm
# (a reading: the pages do not say what happens when the leftover is zero).
Q_FLOOR = 1e-12


# ---------------------------------------------------------------------------
# exact input conversions
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact bf16 -> float64: a bf16 value is the upper half of an f32."""
    b = np.ascontiguousarray(np.asarray(bits).view(np.uint16))
    f32 = (b.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return f32.astype(np.float64)


def as_f64(a) -> np.ndarray:
    """Exact conversion of an f16/f32/f64 numpy array to float64."""
    a = np.asarray(a)
    if a.dtype not in (np.float16, np.float32, np.float64):
        raise TypeError(f"unsupported dtype {a.dtype}; convert bf16 via bf16_bits_to_f64")
    return a.astype(np.float64)


# ---------------------------------------------------------------------------
# full-vocabulary scoring
# ---------------------------------------------------------------------------

def _row_is_valid(z: np.ndarray) -> bool:
    if np.isnan(z).any() or np.isposinf(z).any():
        return False
    return bool(np.isfinite(z).any())


def log_softmax(z: np.ndarray) -> np.ndarray:
    """log p_i = z_i - log sum_j exp(z_j), computed around the row maximum m
    as (z_i - m) - log sum_j exp(z_j - m).

    "Qwen3.8-27B Quantization Challenge", "How the references were made":
    the model's distribution over the whole vocabulary is the softmax of its
    logits.  The caller has checked that z holds a finite maximum.
    """
    m = np.max(z)
    log_s = math.log(float(np.sum(np.exp(z - m))))
    return (z - m) - log_s          # z - m first: m + log_s would lose log_s when |m| is huge


def full_vocab_row(x: np.ndarray, y: np.ndarray, target: int | None = None) -> dict:
    """Score one position from full reference logits x and candidate logits y.

    KL(p || q) = sum_i p_i (log p_i - log q_i) with p = softmax(x),
    q = softmax(y) over the whole vocabulary ("Qwen3.8-27B Quantization
    Challenge", "The score"; the full 248,320-token distribution of "How the
    references were made").  Top-1 agreement compares exact argmaxes
    ("Qwopus3.8-27B-Coder-Flash: quality-eval reference", "Method").  The
    target log-probability log p_t is the negated NLL of the true next token
    ("Golden distributions"; perplexity in "Method").
    """
    x = as_f64(x)
    y = as_f64(y)
    out = dict(kl=math.nan, ref_argmax=-1, cand_argmax=-1,
               ref_target_lp=math.nan, cand_target_lp=math.nan)
    if x.shape != y.shape or x.ndim != 1:
        raise ValueError("x and y must be 1-D and of equal length")
    if not (_row_is_valid(x) and _row_is_valid(y)):
        return out
    lp = log_softmax(x)
    lq = log_softmax(y)
    p = np.exp(lp)
    live = p > 0.0                        # 0 * log 0 = 0
    terms = p[live] * (lp[live] - lq[live])   # lq = -inf with p > 0 gives +inf
    out["kl"] = float(np.sum(terms))
    out["ref_argmax"] = int(np.argmax(x))     # first (lowest) index of the max
    out["cand_argmax"] = int(np.argmax(y))
    if target is not None:
        t = int(target)
        if 0 <= t < x.shape[0]:
            out["ref_target_lp"] = float(lp[t])
            out["cand_target_lp"] = float(lq[t])
    return out


def full_vocab(X: np.ndarray, Y: np.ndarray, targets=None) -> dict:
    """full_vocab_row over every row of X, Y ([n, V], already float64-exact)."""
    X = np.asarray(X)
    Y = np.asarray(Y)
    n = X.shape[0]
    kl = np.full(n, np.nan)
    ra = np.full(n, -1, dtype=np.int64)
    ca = np.full(n, -1, dtype=np.int64)
    rt = np.full(n, np.nan)
    ct = np.full(n, np.nan)
    for i in range(n):
        t = None if targets is None else int(targets[i])
        r = full_vocab_row(X[i], Y[i], t)
        kl[i], ra[i], ca[i] = r["kl"], r["ref_argmax"], r["cand_argmax"]
        rt[i], ct[i] = r["ref_target_lp"], r["cand_target_lp"]
    return dict(kl=kl, ref_argmax=ra, cand_argmax=ca, ref_target_lp=rt, cand_target_lp=ct)


# ---------------------------------------------------------------------------
# shared LM head
# ---------------------------------------------------------------------------

def shared_head_logits(H: np.ndarray, W: np.ndarray) -> np.ndarray:
    """logits[n, v] = sum_k H[n, k] W[v, k] in float64.

    "Qwen3.8-27B fidelity suite v5", opening paragraph: both models' final
    hidden states go through one shared BF16 LM head, so the head is the same
    matrix for reference and candidate.  H and W hold the exact bf16 values
    converted to float64; the product is formed in float64 (logits are not
    rounded back to bf16).
    """
    return np.asarray(H, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T


def shared_head(H_ref, H_cand, W, targets=None, v_chunk: int = 1 << 15) -> dict:
    """Score positions from reference and candidate hidden states ([n, K])
    through one head W ([V, K]): logits for both sides, then full_vocab.

    The logits are built in vocabulary chunks of v_chunk rows of W so that
    the float64 copy of a 248,320 x 5120 head never exists at once; the
    chunking only partitions the matmul's output columns.
    """
    H_ref = np.asarray(H_ref, dtype=np.float64)
    H_cand = np.asarray(H_cand, dtype=np.float64)
    n = H_ref.shape[0]
    V = W.shape[0]
    X = np.empty((n, V))
    Y = np.empty((n, V))
    for v0 in range(0, V, v_chunk):
        Wc = np.asarray(W[v0:v0 + v_chunk], dtype=np.float64)
        X[:, v0:v0 + v_chunk] = H_ref @ Wc.T
        Y[:, v0:v0 + v_chunk] = H_cand @ Wc.T
    res = full_vocab(X, Y, targets)
    res["ref_logits"] = X
    res["cand_logits"] = Y
    return res


def logit_error_bound(H_row: np.ndarray, W_row, unit_roundoff=2.0 ** -24) -> float:
    """gamma_K * sum_k |h_k w_k|: the standard bound on the error of an
    f32-accumulated dot product of length K (Higham, "Accuracy and Stability
    of Numerical Algorithms", Sec. 3.1)."""
    h = np.abs(np.asarray(H_row, dtype=np.float64))
    return H_row.shape[0] * unit_roundoff * float(h @ np.abs(np.asarray(W_row, dtype=np.float64)))


def argmax_ambiguous(logits_row: np.ndarray, H_row: np.ndarray, W, unit_roundoff=2.0 ** -24) -> bool:
    """True when the row's top-2 logits are closer than twice the standard
    f32 dot-product error bound gamma_K * sum_k |h_k w_vk| (gamma_K = K u,
    Higham, "Accuracy and Stability of Numerical Algorithms", Sec. 3.1).
    On such a row an f32-accumulated argmax may legitimately differ from
    the float64 one, so the bit-exact argmax comparison skips it."""
    z = np.asarray(logits_row, dtype=np.float64)
    order = np.argsort(-z, kind="stable")
    i1, i2 = int(order[0]), int(order[1])
    K = H_row.shape[0]
    gamma = K * unit_roundoff
    h = np.abs(np.asarray(H_row, dtype=np.float64))
    b1 = gamma * float(h @ np.abs(np.asarray(W[i1], dtype=np.float64)))
    b2 = gamma * float(h @ np.abs(np.asarray(W[i2], dtype=np.float64)))
    return (z[i1] - z[i2]) < 2.0 * (b1 + b2)


# ---------------------------------------------------------------------------
# top-k + one tail bucket
# ---------------------------------------------------------------------------

def topk_tail_row(ref_ids, ref_lp, cand_ids, cand_lp, vocab: int) -> dict:
    """KL over the reference's top-k ids plus one tail bucket, one position.

    "Qwopus3.8-27B-Coder-Flash: quality-eval reference", "Method": the sum
    runs over the reference's top-64 ids plus one tail bucket; a reference
    id missing from the candidate's top-64 receives the candidate's leftover
    probability mass spread evenly over the vocabulary ids outside the
    candidate's top-64; top-1 agreement is an exact argmax match, read from
    the first stored slot because "Files" stores the lists sorted.
    Stored log-probs are used directly as log p and log q of listed ids.
    """
    ref_ids = [int(v) for v in ref_ids]
    cand_ids = [int(v) for v in cand_ids]
    rlp = as_f64(np.asarray(ref_lp))
    clp = as_f64(np.asarray(cand_lp))
    k = len(ref_ids)
    if len(cand_ids) != k or not (0 < k < vocab):
        raise ValueError("need equal list lengths and 0 < k < vocab")
    c = np.exp(clp)
    leftover = max(1.0 - float(np.sum(c)), 0.0)
    spread = leftover / (vocab - k)
    log_spread = math.log(max(spread, Q_FLOOR))

    first_slot = {}
    for s, cid in enumerate(cand_ids):          # first occurrence wins
        first_slot.setdefault(cid, s)

    p = np.exp(rlp)
    q = np.empty(k)
    logq = np.empty(k)
    matched = 0
    for j, rid in enumerate(ref_ids):
        s = first_slot.get(rid)
        if s is None:
            q[j] = spread
            logq[j] = log_spread
        else:
            q[j] = c[s]
            logq[j] = clp[s]
            matched += 1
    kl = float(np.sum(p * (rlp - logq)))
    p_tail = 1.0 - float(np.sum(p))
    q_tail = 1.0 - float(np.sum(q))
    if p_tail > 0.0:
        kl += p_tail * (math.log(p_tail) - math.log(max(q_tail, Q_FLOOR)))
    return dict(kl=kl, top1=int(ref_ids[0] == cand_ids[0]), n_matched=matched)


def topk_tail(ref_ids, ref_lp, cand_ids, cand_lp, vocab: int, chunk: int = 8192) -> dict:
    """topk_tail_row for every position of [n, k] arrays.

    Same arithmetic, applied to a chunk of positions at once: matching is the
    plain [n, k, k] equality table (first matching candidate slot wins), and
    every sum runs along the k axis.
    """
    ref_ids = np.asarray(ref_ids).astype(np.int64)
    cand_ids = np.asarray(cand_ids).astype(np.int64)
    rlp_all = np.asarray(ref_lp)
    clp_all = np.asarray(cand_lp)
    n, k = ref_ids.shape
    if cand_ids.shape != (n, k) or not (0 < k < vocab):
        raise ValueError("need [n, k] arrays with 0 < k < vocab")
    kl = np.empty(n)
    top1 = np.empty(n, dtype=np.uint8)
    n_matched = np.empty(n, dtype=np.int64)
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        rid, cid = ref_ids[a:b], cand_ids[a:b]
        rlp = as_f64(rlp_all[a:b])
        clp = as_f64(clp_all[a:b])
        c = np.exp(clp)
        leftover = np.maximum(1.0 - np.sum(c, axis=1), 0.0)
        spread = leftover / (vocab - k)
        log_spread = np.log(np.maximum(spread, Q_FLOOR))
        eq = rid[:, :, None] == cid[:, None, :]            # [m, j, s]
        found = eq.any(axis=2)
        slot = np.argmax(eq, axis=2)                        # first True
        q_m = np.take_along_axis(c, slot, axis=1)
        lq_m = np.take_along_axis(clp, slot, axis=1)
        q = np.where(found, q_m, spread[:, None])
        logq = np.where(found, lq_m, log_spread[:, None])
        p = np.exp(rlp)
        row = np.sum(p * (rlp - logq), axis=1)
        p_tail = 1.0 - np.sum(p, axis=1)
        q_tail = 1.0 - np.sum(q, axis=1)
        safe_pt = np.where(p_tail > 0.0, p_tail, 1.0)
        lq_tail = np.log(np.maximum(q_tail, Q_FLOOR))
        tail = np.where(p_tail > 0.0, p_tail * (np.log(safe_pt) - lq_tail), 0.0)
        kl[a:b] = row + tail
        top1[a:b] = (rid[:, 0] == cid[:, 0]).astype(np.uint8)
        n_matched[a:b] = found.sum(axis=1)
    return dict(kl=kl, top1=top1, n_matched=n_matched)


# ---------------------------------------------------------------------------
# candidate full logits against a sparse reference (the challenge score)
# ---------------------------------------------------------------------------

def sparse_ref_row(y, ref_ids, ref_lp, p_tail=None, target=None) -> dict:
    """KL over the reference's K listed ids plus one tail cell, from the
    candidate's full logits y, one position.

    "Qwen3.8-27B Quantization Challenge", "Golden distributions": the
    reference is stored sparse, as its K most likely ids with f32 log p (most
    likely first) and, per row, the tail mass 1 - sum exp(top lp) summed
    over the rest of the full row.  "The score": the candidate's q =
    softmax(y) is coarsened onto the reference's K + 1 cells (the K listed
    ids, and one cell holding all the rest of q's mass) and
    KL(p || q) = sum over cells p_c (log p_c - log q_c).  Top-1 agreement is
    an argmax match; the reference's argmax is its first listed id.

    p_tail defaults to 1 - sum_R p when the row's stored tail mass is not
    given.  Listed ids are distinct (a top-K of one distribution); an id
    outside [0, V) or a repeated id makes the position invalid (KL NaN).
    """
    y = as_f64(y)
    V = y.shape[0]
    ids = np.asarray(ref_ids).astype(np.int64)
    lp = as_f64(np.asarray(ref_lp))
    K = ids.shape[0]
    out = dict(kl=math.nan, cand_argmax=-1, top1=0, cand_target_lp=math.nan)
    if not 0 < K <= V or lp.shape != (K,):
        raise ValueError("need 0 < K <= V listed ids with one log-prob each")
    if not _row_is_valid(y):
        return out
    lq_all = log_softmax(y)
    out["cand_argmax"] = int(np.argmax(y))
    out["top1"] = int(int(ids[0]) == out["cand_argmax"])
    if target is not None and 0 <= int(target) < V:
        out["cand_target_lp"] = float(lq_all[int(target)])
    if np.any((ids < 0) | (ids >= V)) or np.unique(ids).shape[0] != K:
        return out
    p = np.exp(lp)
    live = p > 0.0                                  # 0 * log 0 = 0
    kl = float(np.sum(p[live] * (lp[live] - lq_all[ids][live])))
    rest = np.ones(V, dtype=bool)
    rest[ids] = False
    q_tail = float(np.sum(np.exp(lq_all[rest])))    # the rest of q's mass
    pt = (1.0 - float(np.sum(p))) if p_tail is None else float(p_tail)
    if pt > 0.0:
        kl += pt * (math.log(pt) - math.log(max(q_tail, Q_FLOOR)))
    out["kl"] = kl
    return out


def sparse_ref(Y, ref_ids, ref_lp, p_tail=None, targets=None) -> dict:
    """sparse_ref_row for every position: Y [n, V] candidate logits
    (float64-exact), ref_ids / ref_lp [n, K], p_tail [n] or None."""
    Y = np.asarray(Y)
    n = Y.shape[0]
    kl = np.full(n, np.nan)
    ca = np.full(n, -1, dtype=np.int64)
    top1 = np.zeros(n, dtype=np.uint8)
    ct = np.full(n, np.nan)
    for i in range(n):
        r = sparse_ref_row(Y[i], ref_ids[i], ref_lp[i], None if p_tail is None else p_tail[i],
                           None if targets is None else int(targets[i]))
        kl[i], ca[i], top1[i], ct[i] = r["kl"], r["cand_argmax"], r["top1"], r["cand_target_lp"]
    return dict(kl=kl, cand_argmax=ca, top1=top1, cand_target_lp=ct)


# ---------------------------------------------------------------------------
# sparse capture of a reference distribution
# ---------------------------------------------------------------------------

def sparse_capture_row(x, k: int, target=None) -> dict:
    """The sparse record of one position, from the reference's full logits x.

    "Qwen3.8-27B Quantization Challenge", "Golden distributions": per scored
    position the reference keeps its k most likely tokens with their f32 log
    p, most likely first, and a row of (NLL of the true next token, entropy
    in nats, tail mass 1 - sum exp(top lp) summed over the rest of the full
    row).  Equal log-probs keep the lower id first (a reading: the page does
    not order ties).  A row holding NaN or +inf, or no finite logit, gives ids
    -1 and NaN everywhere else.
    """
    x = as_f64(x)
    V = x.shape[0]
    if not 0 < k <= V:
        raise ValueError("need 0 < k <= V")
    out = dict(ids=np.full(k, -1, dtype=np.int64), lp=np.full(k, np.nan), nll=math.nan,
               entropy=math.nan, tail=math.nan)
    if not _row_is_valid(x):
        return out
    lp = log_softmax(x)
    order = np.lexsort((np.arange(V), -lp))        # by log-prob descending, then id ascending
    top = order[:k]
    p = np.exp(lp)
    live = p > 0.0                                  # 0 * log 0 = 0
    rest = np.ones(V, dtype=bool)
    rest[top] = False
    out["ids"] = top.astype(np.int64)
    out["lp"] = lp[top]
    out["entropy"] = -math.fsum((p[live] * lp[live]).tolist())
    out["tail"] = math.fsum(p[rest].tolist())
    if target is not None and 0 <= int(target) < V:
        out["nll"] = -float(lp[int(target)])
    return out


def sparse_capture(X, k: int, targets=None) -> dict:
    """sparse_capture_row for every row of X [n, V] (float64-exact): ids and
    lp [n, k], rows [n, 3] = (NLL, entropy, tail)."""
    X = np.asarray(X)
    n = X.shape[0]
    ids = np.empty((n, k), dtype=np.int64)
    lp = np.empty((n, k))
    rows = np.empty((n, 3))
    for i in range(n):
        r = sparse_capture_row(X[i], k, None if targets is None else int(targets[i]))
        ids[i], lp[i] = r["ids"], r["lp"]
        rows[i] = (r["nll"], r["entropy"], r["tail"])
    return dict(ids=ids, lp=lp, rows=rows)


# ---------------------------------------------------------------------------
# reductions
# ---------------------------------------------------------------------------

def exact_mean(vals: np.ndarray) -> float:
    """Correctly rounded mean (math.fsum), with IEEE results for infinite
    members: +inf and -inf together give NaN, one kind alone gives itself."""
    if vals.shape[0] == 0:
        return math.nan
    try:
        return math.fsum(vals.tolist()) / vals.shape[0]
    except ValueError:      # both +inf and -inf present
        return math.nan


def quantile_linear(sorted_vals: np.ndarray, q: float) -> tuple[float, float, float]:
    """Linear-interpolation percentile of an ascending array.

    Returns (value, lower order statistic, upper order statistic).
    h = (n - 1) q; value = s[lo] + (s[hi] - s[lo]) (h - lo), lo = floor h,
    hi = min(lo + 1, n - 1).
    """
    n = sorted_vals.shape[0]
    if n == 0:
        return math.nan, math.nan, math.nan
    h = (n - 1) * float(q)
    lo = int(math.floor(h))
    hi = min(lo + 1, n - 1)
    s_lo = float(sorted_vals[lo])
    s_hi = float(sorted_vals[hi])
    frac = h - lo
    return s_lo + (s_hi - s_lo) * frac, s_lo, s_hi


def reduce_stats(kl, ref_argmax=None, cand_argmax=None, top1=None,
                 ref_target_lp=None, cand_target_lp=None, mask=None,
                 quantiles=(0.5, 0.99, 0.999), thresholds=()) -> dict:
    """Leaderboard reductions over per-position results.

    "Qwen3.8-27B Quantization Challenge", "The score": mean KL ranks entries;
    the median, p99 and p99.9 KL, top-1 agreement and the perplexity ratio
    are reported beside it.  "Qwopus3.8-27B-Coder-Flash: quality-eval
    reference", "Method": perplexity = exp(mean NLL of the true next token).
    "Qwen3.8-27B fidelity suite v5", "What is in here": percentiles and exact
    exceedance counts.  The optional mask selects which positions are scored
    (e.g. only assistant-written positions, as in the IQ8R card's "Quality").

    The set of scored positions is mask & (KL is not NaN); NaN KLs are
    counted in n_nan.  The mean uses an exactly rounded sum (math.fsum).
    """
    kl = np.asarray(kl, dtype=np.float32)
    n_all = kl.shape[0]
    sel = np.ones(n_all, dtype=bool) if mask is None else np.asarray(mask).astype(bool)
    isnan = np.isnan(kl)
    valid = sel & ~isnan
    vals = kl[valid].astype(np.float64)
    n = int(vals.shape[0])
    out = dict(n=n, n_nan=int(np.sum(sel & isnan)))
    out["mean_kl"] = exact_mean(vals)
    s = np.sort(kl[valid])
    qv, qlo, qhi = [], [], []
    for q in quantiles:
        v, lo, hi = quantile_linear(s, q)
        qv.append(v)
        qlo.append(lo)
        qhi.append(hi)
    out["q_value"], out["q_lo"], out["q_hi"] = qv, qlo, qhi
    if top1 is not None:
        agree = np.asarray(top1).astype(bool)
    elif ref_argmax is not None and cand_argmax is not None:
        ra = np.asarray(ref_argmax)
        ca = np.asarray(cand_argmax)
        agree = (ra == ca) & (ra >= 0)
    else:
        agree = None
    if agree is not None:
        cnt = int(np.sum(agree & valid))
        out["top1_agree"] = cnt
        out["top1_rate"] = cnt / n if n else math.nan
    for name, arr in (("ref", ref_target_lp), ("cand", cand_target_lp)):
        if arr is None:
            continue
        nll = -np.asarray(arr, dtype=np.float32)[valid].astype(np.float64)
        out[f"{name}_mean_nll"] = exact_mean(nll)
        out[f"{name}_ppl"] = math.exp(out[f"{name}_mean_nll"]) if n else math.nan
    if "ref_ppl" in out and "cand_ppl" in out:
        out["ppl_ratio"] = out["cand_ppl"] / out["ref_ppl"]
    out["exceed"] = [int(np.sum(valid & (kl > np.float32(t)))) for t in thresholds]
    return out


# ---------------------------------------------------------------------------
# paired comparison of two candidates (per-context differences, cluster
# bootstrap)
# ---------------------------------------------------------------------------

def paired_compare(kl_a, kl_b, ctx_len: int, cluster, resample, quantiles=(0.025, 0.975), mask=None) -> dict:
    """Paired per-context comparison of two candidates scored against one
    reference, with a source-cluster bootstrap interval.

    "Qwen3.8-27B fidelity suite v5": the suite's contexts are grouped into
    source clusters ("What is in here"); two candidates are compared "paired
    per context" and the difference is reported with a 95 % source-cluster
    bootstrap interval, together with how many contexts each side wins and
    the ties (the sibling-rebuild paragraph and the "compare against a
    published candidate" step).

    Readings (the page gives no formulas):
    * kl_a, kl_b hold n_ctx contexts of ctx_len positions each, context-major.
      A position counts when mask is set (all when None) and neither KL is
      NaN; a context counts when it has at least one such position.
    * Per counted context c: mean_a(c), mean_b(c) are exact means of its
      counted positions and d_c = mean_a(c) - mean_b(c).
    * The reported difference is the mean of d_c over counted contexts;
      mean_a / mean_b likewise.  a_lower / b_lower / ties count the contexts
      with d_c < 0 / d_c > 0 / d_c == 0.
    * Bootstrap replicate r draws the clusters resample[r, 0..C-1] (with
      repetition; C = number of clusters) and takes every counted context of
      each drawn cluster: stat_r = sum_j D[j] / sum_j N[j] over the draws,
      with D[k] = sum of d_c and N[k] = number of counted contexts in cluster
      k.  A replicate whose draws hold no counted context is NaN and left
      out.  The interval ends are the linear-interpolation percentiles of the
      replicates (the convention of reduce_stats).
    The random draws are an input: the page does not say how they are made.
    """
    a = np.asarray(kl_a, dtype=np.float32).reshape(-1, ctx_len)
    b = np.asarray(kl_b, dtype=np.float32).reshape(-1, ctx_len)
    n_ctx = a.shape[0]
    use = ~(np.isnan(a) | np.isnan(b))
    if mask is not None:
        use &= np.asarray(mask).astype(bool).reshape(-1, ctx_len)
    cluster = np.asarray(cluster, dtype=np.int64)
    n_clusters = int(np.asarray(resample).shape[1]) if np.asarray(resample).ndim == 2 else 0
    ctx_a, ctx_b, ctx_n = [], [], []
    for c in range(n_ctx):
        va = a[c][use[c]].astype(np.float64)
        vb = b[c][use[c]].astype(np.float64)
        ctx_n.append(int(va.shape[0]))
        ctx_a.append(exact_mean(va))
        ctx_b.append(exact_mean(vb))
    counted = [c for c in range(n_ctx) if ctx_n[c] > 0]
    d = {c: ctx_a[c] - ctx_b[c] for c in counted}
    out = dict(n_ctx=len(counted), n_pos=int(sum(ctx_n)))
    out["mean_a"] = exact_mean(np.array([ctx_a[c] for c in counted]))
    out["mean_b"] = exact_mean(np.array([ctx_b[c] for c in counted]))
    out["diff"] = exact_mean(np.array([d[c] for c in counted]))
    out["a_lower"] = sum(1 for c in counted if d[c] < 0)
    out["b_lower"] = sum(1 for c in counted if d[c] > 0)
    out["ties"] = sum(1 for c in counted if d[c] == 0)
    D = [[] for _ in range(n_clusters)]
    N = [0] * n_clusters
    for c in counted:
        D[cluster[c]].append(d[c])
        N[cluster[c]] += 1
    stats = []
    for draws in np.asarray(resample, dtype=np.int64):
        terms, cnt = [], 0
        for k in draws:
            terms.extend(D[k])
            cnt += N[k]
        stats.append(math.fsum(terms) / cnt if cnt else math.nan)
    stats = np.array(stats, dtype=np.float64)
    out["boot"] = stats
    ok = np.sort(stats[~np.isnan(stats)])
    out["n_boot"] = int(ok.shape[0])
    out["ci"] = [quantile_linear(ok, q)[0] for q in quantiles]
    out["ctx_mean_a"] = np.array(ctx_a)
    out["ctx_mean_b"] = np.array(ctx_b)
    out["ctx_n"] = np.array(ctx_n)
    return out
