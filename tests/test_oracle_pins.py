"""Pins for the f64 oracle: closed forms, invariants, brute force and library
routines that do not share the oracle's own formulas.

Every pin is a function of the oracle module, so the same pins also run
against mutated copies of the oracle (a sign flipped, a term dropped, an
index moved): each planted mistake must make at least one pin fail.
"""
import importlib.util
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle.kld_oracle as ORACLE

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_SRC = os.path.join(ROOT, "oracle", "kld_oracle.py")


def _close(a, b, rtol=1e-10, atol=1e-12):
    return abs(a - b) <= atol + rtol * abs(b)


# ---------------------------------------------------------------------------
# full-vocabulary pins
# ---------------------------------------------------------------------------

def pin_self_is_zero(O):
    rng = np.random.default_rng(1)
    for V in (2, 7, 1000):
        x = rng.normal(0, 3, V)
        r = O.full_vocab_row(x, x.copy(), 0)
        assert r["kl"] == 0.0
        assert r["ref_argmax"] == r["cand_argmax"] == int(np.argmax(x))


def pin_nonnegative(O):
    rng = np.random.default_rng(2)
    for _ in range(50):
        V = int(rng.integers(2, 300))
        x = rng.normal(0, 2, V)
        y = x + rng.normal(0, rng.uniform(0.01, 3), V)
        assert O.full_vocab_row(x, y)["kl"] >= -1e-14


def pin_one_hot_vs_uniform(O):
    for V in (2, 10, 4096, 248_320):
        x = np.full(V, -np.inf)
        x[V // 3] = 0.0
        r = O.full_vocab_row(x, np.zeros(V), V // 3)
        assert _close(r["kl"], math.log(V), rtol=1e-13)
        assert r["ref_argmax"] == V // 3 and r["cand_argmax"] == 0
        assert r["ref_target_lp"] == 0.0
        assert _close(r["cand_target_lp"], -math.log(V), rtol=1e-13)


def pin_two_point(O):
    rng = np.random.default_rng(3)
    for _ in range(20):
        a, b, c, d = rng.normal(0, 2, 4)
        p = 1.0 / (1.0 + math.exp(b - a))
        q = 1.0 / (1.0 + math.exp(d - c))
        want = p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))
        got = O.full_vocab_row(np.array([a, b]), np.array([c, d]))["kl"]
        assert _close(got, want, rtol=1e-9, atol=1e-15)


def pin_geometric(O):
    # x_i = a i, y_i = b i: truncated geometric distributions with ratio
    # r = e^a; Z(a) = (1 - r^V) / (1 - r), E_p[i] = r/(1-r) - V r^V/(1-r^V),
    # KL = (a - b) E_p[i] - ln Z(a) + ln Z(b).
    for (a, b, V) in ((-0.3, -0.25, 50), (-0.05, -0.2, 400), (0.1, -0.1, 30)):
        i = np.arange(V, dtype=np.float64)
        ra, rb = math.exp(a), math.exp(b)
        Za = (1 - ra ** V) / (1 - ra)
        Zb = (1 - rb ** V) / (1 - rb)
        Ei = ra / (1 - ra) - V * ra ** V / (1 - ra ** V)
        want = (a - b) * Ei - math.log(Za) + math.log(Zb)
        r = O.full_vocab_row(a * i, b * i, V - 1)
        assert _close(r["kl"], want, rtol=1e-10)
        # log p_{V-1} = a (V-1) - ln Z(a); log q_{V-1} = b (V-1) - ln Z(b)
        assert _close(r["ref_target_lp"], a * (V - 1) - math.log(Za), rtol=1e-12)
        assert _close(r["cand_target_lp"], b * (V - 1) - math.log(Zb), rtol=1e-12)


def pin_single_logit_shift(O):
    # y = x + c e_j  =>  KL(p || q) = ln(1 - p_j + p_j e^c) - c p_j
    rng = np.random.default_rng(4)
    for _ in range(20):
        V = int(rng.integers(3, 500))
        x = rng.normal(0, 1.5, V)
        j = int(rng.integers(0, V))
        c = float(rng.normal(0, 2))
        y = x.copy()
        y[j] += c
        e = np.exp(x - x.max())
        pj = e[j] / e.sum()
        want = math.log(1 - pj + pj * math.exp(c)) - c * pj
        assert _close(O.full_vocab_row(x, y)["kl"], want, rtol=1e-9, atol=1e-15)


def pin_shift_and_permutation(O):
    rng = np.random.default_rng(5)
    V = 777
    x = rng.normal(0, 2, V)
    y = x + rng.normal(0, 0.3, V)
    base = O.full_vocab_row(x, y, 5)
    sh = O.full_vocab_row(x + 3.7, y - 2.1, 5)
    assert _close(sh["kl"], base["kl"], rtol=1e-10)
    assert _close(sh["ref_target_lp"], base["ref_target_lp"], rtol=1e-12)
    perm = rng.permutation(V)
    pr = O.full_vocab_row(x[perm], y[perm], int(np.argmax(perm == 5)))
    assert _close(pr["kl"], base["kl"], rtol=1e-10)
    assert perm[pr["ref_argmax"]] == base["ref_argmax"]
    assert _close(pr["ref_target_lp"], base["ref_target_lp"], rtol=1e-12)


def pin_argmax_lowest_index(O):
    x = np.array([1.0, 3.0, 2.0, 3.0, 3.0])
    y = np.array([5.0, 0.0, 5.0, 5.0, -1.0])
    r = O.full_vocab_row(x, y)
    assert r["ref_argmax"] == 1 and r["cand_argmax"] == 0


def pin_huge_logits_keep_the_normaliser(O):
    # ties at a maximum near the largest f32 value: log p of each of the k
    # tied ids is -ln k exactly, whatever the magnitude of the maximum
    for base in (3.0e38, -3.0e38, 1.0e30, 0.0):
        V = 50
        x = np.full(V, -3.3e38 if base > -3.0e38 else -3.4e38)
        y = x.copy()
        x[[3, 7, 11]] = base
        y[[3, 7, 11, 20]] = base
        r = O.full_vocab_row(x, y, 7)
        assert _close(r["ref_target_lp"], -math.log(3), rtol=1e-14)
        assert _close(r["cand_target_lp"], -math.log(4), rtol=1e-14)
        assert _close(r["kl"], math.log(4 / 3), rtol=1e-12)


def pin_uniform_target(O):
    for V in (3, 4096):
        r = O.full_vocab_row(np.zeros(V), np.full(V, 2.5), 1)
        assert _close(r["ref_target_lp"], -math.log(V), rtol=1e-13)
        assert abs(r["kl"]) < 1e-15


def pin_non_finite(O):
    V = 16
    x = np.linspace(-2, 2, V)
    bad = x.copy()
    bad[3] = np.nan
    for a, b in ((bad, x), (x, bad)):
        r = O.full_vocab_row(a, b, 1)
        assert math.isnan(r["kl"]) and r["ref_argmax"] == -1 and math.isnan(r["ref_target_lp"])
    pinf = x.copy()
    pinf[0] = np.inf
    assert math.isnan(O.full_vocab_row(pinf, x)["kl"])
    assert math.isnan(O.full_vocab_row(np.full(V, -np.inf), x)["kl"])
    # a masked reference id (x = -inf) contributes nothing, even against -inf
    xm = x.copy()
    xm[2] = -np.inf
    ym = x.copy()
    ym[2] = -np.inf
    assert abs(O.full_vocab_row(xm, ym)["kl"]) < 1e-15
    # the candidate gives zero mass where the reference has some: KL = +inf
    yz = x.copy()
    yz[7] = -np.inf
    assert O.full_vocab_row(x, yz)["kl"] == math.inf


def pin_bf16_conversion(O):
    # bf16 bit patterns of a few exactly known values
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x7F80, 0xFF80, 0x3E80, 0x4049], dtype=np.uint16)
    want = [1.0, -2.0, 0.0, math.inf, -math.inf, 0.25, 3.140625]
    assert list(O.bf16_bits_to_f64(bits)) == want


# ---------------------------------------------------------------------------
# top-k + tail bucket pins
# ---------------------------------------------------------------------------

def _brute_force_tail_kl(ref_ids, ref_lp, cand_ids, cand_lp, V):
    """Materialise the candidate's distribution over all V ids from the
    rule (listed ids keep their mass, the leftover is spread evenly over the
    other V - k ids), then coarsen both sides onto the reference's k cells
    plus one cell holding every other id, by enumeration."""
    k = len(ref_ids)
    q_full = [None] * V
    for s, cid in enumerate(cand_ids):
        if q_full[cid] is None:
            q_full[cid] = math.exp(cand_lp[s])
    listed = sum(math.exp(v) for v in cand_lp)
    fill = max(1.0 - listed, 0.0) / (V - k)
    q_full = [fill if v is None else v for v in q_full]
    p_cells = [math.exp(v) for v in ref_lp]
    q_cells = [q_full[r] for r in ref_ids]
    p_rest = 1.0 - sum(p_cells)
    q_rest = sum(q_full[v] for v in range(V) if v not in set(ref_ids))
    kl = 0.0
    for p, q in zip(p_cells, q_cells):
        kl += p * math.log(p / q)
    if p_rest > 0:
        kl += p_rest * math.log(p_rest / q_rest)
    return kl


def pin_tail_brute_force(O):
    rng = np.random.default_rng(6)
    for _ in range(300):
        V = int(rng.integers(3, 17))
        k = int(rng.integers(1, min(8, V - 1) + 1))
        # full distributions so that every listed mass is consistent
        p = rng.dirichlet(np.full(V, 0.7))
        q = rng.dirichlet(np.full(V, 0.7))
        ref_ids = rng.permutation(V)[:k]
        cand_ids = rng.permutation(V)[:k]
        ref_lp = np.log(p[ref_ids])
        cand_lp = np.log(q[cand_ids])
        want = _brute_force_tail_kl(list(ref_ids), list(ref_lp), list(cand_ids), list(cand_lp), V)
        got = O.topk_tail_row(ref_ids, ref_lp, cand_ids, cand_lp, V)
        assert _close(got["kl"], want, rtol=1e-9, atol=1e-13), (V, k, got, want)
        assert got["n_matched"] == len(set(ref_ids) & set(cand_ids))
        assert got["top1"] == int(ref_ids[0] == cand_ids[0])
        vec = O.topk_tail(ref_ids[None], ref_lp[None], cand_ids[None], cand_lp[None], V)
        assert _close(vec["kl"][0], want, rtol=1e-9, atol=1e-13)
        assert vec["n_matched"][0] == got["n_matched"]


def pin_tail_lower_bound(O):
    # "The score": coarsening onto cells gives a lower bound on the full KL.
    # When the candidate's top-k holds every reference top-k id, the tail
    # rule is an exact coarsening, so tail KL <= full KL must hold.
    rng = np.random.default_rng(7)
    hits = 0
    for _ in range(200):
        V = int(rng.integers(20, 200))
        k = int(rng.integers(2, 12))
        x = rng.normal(0, 2, V)
        y = x + rng.normal(0, 0.05, V)
        lp = x - (x.max() + math.log(np.exp(x - x.max()).sum()))
        lq = y - (y.max() + math.log(np.exp(y - y.max()).sum()))
        R = np.argsort(-lp, kind="stable")[:k]
        C = np.argsort(-lq, kind="stable")[:k]
        if not set(R) <= set(C):
            continue
        hits += 1
        t = O.topk_tail_row(R, lp[R], C, lq[C], V)["kl"]
        f = O.full_vocab_row(x, y)["kl"]
        assert t <= f + 1e-13
        # with the ids equal the tail rule is the exact two-level coarsening
        pr = 1 - np.exp(lp[R]).sum()
        qr = 1 - np.exp(lq[R]).sum()
        exact = float(np.sum(np.exp(lp[R]) * (lp[R] - lq[R]))) + pr * math.log(pr / qr)
        assert _close(t, exact, rtol=1e-9, atol=1e-14)
    assert hits > 20


def pin_tail_spread_cases(O):
    # one unmatched id: q = leftover / (V - k), exactly
    V, k = 10, 2
    ref_ids = np.array([0, 1])
    cand_ids = np.array([0, 5])
    ref_lp = np.log(np.array([0.5, 0.25]))
    cand_lp = np.log(np.array([0.4, 0.2]))
    spread = 0.4 / 8
    want = 0.5 * math.log(0.5 / 0.4) + 0.25 * math.log(0.25 / spread) \
        + 0.25 * math.log(0.25 / (1 - 0.4 - spread))
    assert _close(O.topk_tail_row(ref_ids, ref_lp, cand_ids, cand_lp, V)["kl"], want, rtol=1e-12)
    # duplicate candidate id: the first slot is the match
    r = O.topk_tail_row(np.array([3, 1]), np.log([0.5, 0.1]), np.array([3, 3]),
                        np.log([0.3, 0.2]), 20)
    assert r["n_matched"] == 1
    q_tail = 1 - 0.3 - 0.5 / 18
    want = 0.5 * math.log(0.5 / 0.3) + 0.1 * math.log(0.1 / (0.5 / 18)) + 0.4 * math.log(0.4 / q_tail)
    assert _close(r["kl"], want, rtol=1e-12)


def pin_tail_duplicates_vectorised(O):
    # the hand-computed duplicate case through the [n, k] function: the
    # candidate lists id 3 twice (0.3 then 0.2) and the first slot is the match
    want = 0.5 * math.log(0.5 / 0.3) + 0.1 * math.log(0.1 / (0.5 / 18)) + 0.4 * math.log(0.4 / (1 - 0.3 - 0.5 / 18))
    r = O.topk_tail(np.array([[3, 1], [1, 3]]), np.log([[0.5, 0.1], [0.1, 0.5]]), np.array([[3, 3], [3, 3]]),
                    np.log([[0.3, 0.2], [0.3, 0.2]]), 20)
    assert _close(r["kl"][0], want, rtol=1e-12) and _close(r["kl"][1], want, rtol=1e-12)
    assert list(r["n_matched"]) == [1, 1] and list(r["top1"]) == [1, 0]
    # random lists drawn with repetition (distinct log-probs at repeated ids):
    # the [n, k] function agrees with the per-position one, which the brute
    # force and the hand-computed cases pin
    rng = np.random.default_rng(9)
    n, k, V = 200, 12, 40
    ri = rng.integers(0, 16, (n, k))
    ci = rng.integers(0, 16, (n, k))
    assert any(len(set(row)) < k for row in ci)
    rl = np.log(rng.dirichlet(np.ones(k + 4), n)[:, :k])
    cl = np.log(rng.dirichlet(np.ones(k + 4), n)[:, :k])
    vec = O.topk_tail(ri, rl, ci, cl, V, chunk=64)
    for i in range(n):
        row = O.topk_tail_row(ri[i], rl[i], ci[i], cl[i], V)
        assert _close(vec["kl"][i], row["kl"], rtol=1e-12, atol=1e-15)
        assert vec["n_matched"][i] == row["n_matched"] and vec["top1"][i] == row["top1"]


def pin_tail_self(O):
    rng = np.random.default_rng(8)
    ids = np.stack([rng.permutation(1000)[:64] for _ in range(50)])
    lp = np.sort(np.log(rng.dirichlet(np.ones(80), 50)[:, :64]), axis=1)[:, ::-1].astype(np.float16)
    r = O.topk_tail(ids, lp, ids, lp, 1000)
    assert np.all(r["kl"] == 0.0) and np.all(r["top1"] == 1) and np.all(r["n_matched"] == 64)


# ---------------------------------------------------------------------------
# candidate full logits against a sparse reference (K + 1 cells)
# ---------------------------------------------------------------------------

def _softmax_loop(y):
    e = [math.exp(v) for v in y]
    s = sum(e)
    return [v / s for v in e]


def _brute_force_cells_kl(p, q, listed):
    """KL between p and q coarsened onto the listed singletons plus one cell
    holding every other id, by enumerating the cells."""
    cells = [[i] for i in listed] + [[i for i in range(len(p)) if i not in set(listed)]]
    kl = 0.0
    for c in cells:
        P = sum(p[i] for i in c)
        Q = sum(q[i] for i in c)
        if P > 0:
            kl += P * math.log(P / Q)
    return kl


def pin_sparse_brute_force(O):
    rng = np.random.default_rng(21)
    for trial in range(300):
        V = int(rng.integers(2, 17))
        K = int(rng.integers(1, V + 1))
        p = list(rng.dirichlet(np.full(V, 0.6)))
        y = list(rng.normal(0, 1.5, V))
        q = _softmax_loop(y)
        listed = sorted(range(V), key=lambda i: -p[i])[:K]
        lp = np.log([p[i] for i in listed])
        tail = sum(p[i] for i in range(V) if i not in set(listed))
        want = _brute_force_cells_kl(p, q, listed)
        given = O.sparse_ref_row(np.array(y), np.array(listed), lp, tail)
        assert _close(given["kl"], want, rtol=1e-9, atol=1e-13), (V, K, given, want)
        if trial % 3 == 0:   # stored tail absent: 1 - sum of the listed masses
            dflt = O.sparse_ref_row(np.array(y), np.array(listed), lp)
            assert _close(dflt["kl"], want, rtol=1e-9, atol=1e-12)
        assert given["cand_argmax"] == max(range(V), key=lambda i: (y[i], -i))
        assert given["top1"] == int(listed[0] == given["cand_argmax"])


def pin_sparse_all_ids_is_full_kl(O):
    # listing every id makes the coarsening the identity: the full KL
    rng = np.random.default_rng(22)
    for V in (5, 64, 1000):
        x = rng.normal(0, 2, V)
        y = x + rng.normal(0, 0.3, V)
        m = x.max()
        lp = x - (m + math.log(math.fsum(np.exp(x - m))))
        ids = rng.permutation(V)
        r = O.sparse_ref_row(y, ids, lp[ids], 0.0)
        f = O.full_vocab_row(x, y)
        assert _close(r["kl"], f["kl"], rtol=1e-10, atol=1e-15)
        assert r["cand_argmax"] == f["cand_argmax"]


def pin_sparse_lower_bound_and_self(O):
    rng = np.random.default_rng(23)
    for _ in range(50):
        V = int(rng.integers(50, 400))
        K = int(rng.integers(1, 40))
        x = rng.normal(0, 2, V)
        y = x + rng.normal(0, 0.2, V)
        m = x.max()
        lp = x - (m + math.log(math.fsum(np.exp(x - m))))
        ids = np.argsort(-lp, kind="stable")[:K]
        rest = np.setdiff1d(np.arange(V), ids)
        tail = math.fsum(np.exp(lp[rest]))
        s = O.sparse_ref_row(y, ids, lp[ids], tail)["kl"]
        assert s <= O.full_vocab_row(x, y)["kl"] + 1e-13     # coarsening lowers KL
        assert abs(O.sparse_ref_row(x, ids, lp[ids], tail)["kl"]) < 1e-13   # q = p


def pin_sparse_binary_closed_form(O):
    # V = 2, K = 1: cells {a} and {b}; KL = binary KL of p and sigmoid(y_a - y_b)
    for p, ya, yb in ((0.7, 0.3, -0.4), (0.99, 2.0, 1.0), (0.2, -1.0, 3.0)):
        q = 1.0 / (1.0 + math.exp(yb - ya))
        want = p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))
        r = O.sparse_ref_row(np.array([ya, yb]), np.array([0]), np.array([math.log(p)]), 1 - p, target=1)
        assert _close(r["kl"], want, rtol=1e-12)
        assert _close(r["cand_target_lp"], math.log(1 - q), rtol=1e-12)


def pin_sparse_edge_cases(O):
    y = np.zeros(8)
    lp = np.log([0.5, 0.25])
    assert math.isnan(O.sparse_ref_row(y, np.array([0, 8]), lp, 0.25)["kl"])      # id out of range
    assert math.isnan(O.sparse_ref_row(y, np.array([3, 3]), lp, 0.25)["kl"])      # repeated id
    bad = y.copy()
    bad[5] = np.nan
    r = O.sparse_ref_row(bad, np.array([0, 1]), lp, 0.25)
    assert math.isnan(r["kl"]) and r["cand_argmax"] == -1
    ninf = y.copy()
    ninf[1] = -np.inf                                  # p > 0 on a cell with q = 0
    assert O.sparse_ref_row(ninf, np.array([0, 1]), lp, 0.25)["kl"] == math.inf
    # no tail term when the stored tail is not positive; uniform q = 1/8
    r = O.sparse_ref_row(y, np.array([2, 6]), np.log([0.75, 0.25]), 0.0, target=4)
    assert _close(r["kl"], 0.75 * math.log(0.75 * 8) + 0.25 * math.log(0.25 * 8), rtol=1e-12)
    assert _close(r["cand_target_lp"], -math.log(8), rtol=1e-14)
    assert r["cand_argmax"] == 0 and r["top1"] == 0   # uniform row: lowest index wins


# ---------------------------------------------------------------------------
# sparse capture of a reference distribution
# ---------------------------------------------------------------------------

def pin_capture_uniform_and_peak(O):
    # uniform row: ties keep the lowest ids, every lp = -ln V, entropy ln V,
    # tail (V - k) / V, NLL ln V
    for V, k in ((10, 3), (64, 64), (1000, 17)):
        r = O.sparse_capture_row(np.full(V, 2.5), k, target=V - 1)
        assert list(r["ids"]) == list(range(k))
        assert np.allclose(r["lp"], -math.log(V), rtol=0, atol=1e-14)
        assert _close(r["entropy"], math.log(V)) and _close(r["nll"], math.log(V))
        assert _close(r["tail"], (V - k) / V, atol=1e-15)
    # one raised logit: p0 = e^c / (e^c + V - 1)
    V, c = 50, 3.0
    x = np.zeros(V)
    x[7] = c
    p0 = math.exp(c) / (math.exp(c) + V - 1)
    q = 1.0 / (math.exp(c) + V - 1)
    r = O.sparse_capture_row(x, 2, target=7)
    assert list(r["ids"]) == [7, 0]
    assert _close(r["lp"][0], math.log(p0)) and _close(r["lp"][1], math.log(q))
    assert _close(r["entropy"], -(p0 * math.log(p0) + (V - 1) * q * math.log(q)))
    assert _close(r["tail"], (V - 2) * q) and _close(r["nll"], -math.log(p0))


def pin_capture_brute_force(O):
    import scipy.stats
    rng = np.random.default_rng(31)
    for _ in range(200):
        V = int(rng.integers(2, 40))
        k = int(rng.integers(1, V + 1))
        x = np.round(rng.normal(0, 2, V), 1)          # rounding makes ties common
        p = _softmax_loop(list(x))
        want = sorted(range(V), key=lambda i: (-p[i], i))[:k]
        t = int(rng.integers(0, V))
        r = O.sparse_capture_row(x, k, target=t)
        # ids equal where the probabilities differ; equal logits give exactly equal lp
        assert [x[i] for i in r["ids"]] == [x[i] for i in want]
        assert sorted(r["ids"][np.array([x[i] for i in r["ids"]]) == x[want[-1]]]) == list(r["ids"][
            np.array([x[i] for i in r["ids"]]) == x[want[-1]]])
        assert np.allclose(np.exp(r["lp"]), [p[i] for i in r["ids"]], rtol=1e-12, atol=0)
        assert _close(r["entropy"], float(scipy.stats.entropy(p)), rtol=1e-10, atol=1e-14)
        assert _close(r["tail"], sum(p[i] for i in range(V) if i not in set(r["ids"])), rtol=1e-10, atol=1e-15)
        assert _close(r["nll"], -math.log(p[t]))


def pin_capture_round_trip(O):
    # a candidate identical to the captured reference scores 0 against it,
    # and the listed masses plus the tail make 1
    rng = np.random.default_rng(32)
    for _ in range(20):
        V, k = int(rng.integers(20, 300)), int(rng.integers(1, 20))
        x = rng.normal(0, 3, V)
        r = O.sparse_capture_row(x, k)
        assert abs(O.sparse_ref_row(x, r["ids"], r["lp"], r["tail"])["kl"]) < 1e-13
        assert _close(math.fsum(np.exp(r["lp"]).tolist()) + r["tail"], 1.0, atol=1e-14)
    bad = O.sparse_capture_row(np.array([0.0, np.nan, 1.0]), 2, target=0)
    assert list(bad["ids"]) == [-1, -1] and math.isnan(bad["tail"]) and math.isnan(bad["nll"])
    ninf = O.sparse_capture_row(np.array([0.0, -np.inf, 1.0]), 3, target=1)
    assert list(ninf["ids"]) == [2, 0, 1] and ninf["nll"] == math.inf and ninf["tail"] == 0.0


# ---------------------------------------------------------------------------
# reductions
# ---------------------------------------------------------------------------

def pin_quantiles(O):
    rng = np.random.default_rng(9)
    for n in (1, 2, 3, 10, 1001, 2047):
        kl = rng.exponential(1e-3, n).astype(np.float32)
        qs = (0.0, 0.5, 0.9, 0.99, 0.999, 1.0)
        st = O.reduce_stats(kl, quantiles=qs)
        want = np.quantile(kl.astype(np.float64), qs, method="linear")
        for got, w in zip(st["q_value"], want):
            assert _close(got, float(w), rtol=1e-15, atol=0)
        s = sorted(kl.tolist())
        for q, lo, hi in zip(qs, st["q_lo"], st["q_hi"]):
            h = (n - 1) * q
            assert lo == s[int(math.floor(h))]
            assert hi == s[min(int(math.floor(h)) + 1, n - 1)]


def pin_mean_and_counts(O):
    rng = np.random.default_rng(10)
    n = 3000
    kl = rng.exponential(0.01, n).astype(np.float32)
    kl[::97] = np.nan
    mask = rng.random(n) < 0.8
    ra = rng.integers(0, 5, n)
    ca = rng.integers(0, 5, n)
    rt = -rng.exponential(2.0, n).astype(np.float32)
    ct = -rng.exponential(2.1, n).astype(np.float32)
    thr = (0.0, 0.01, 0.05)
    st = O.reduce_stats(kl, ra, ca, None, rt, ct, mask, quantiles=(0.5,), thresholds=thr)
    sel = [i for i in range(n) if mask[i] and not math.isnan(kl[i])]
    assert st["n"] == len(sel)
    assert st["n_nan"] == sum(1 for i in range(n) if mask[i] and math.isnan(kl[i]))
    exact = sum((Fraction(float(kl[i])) for i in sel), Fraction(0)) / len(sel)
    assert st["mean_kl"] == float(exact)
    assert st["top1_agree"] == sum(1 for i in sel if ra[i] == ca[i])
    for t, c in zip(thr, st["exceed"]):
        assert c == sum(1 for i in sel if kl[i] > np.float32(t))
    nll_r = float(sum((Fraction(-float(rt[i])) for i in sel), Fraction(0)) / len(sel))
    assert _close(st["ref_ppl"], math.exp(nll_r), rtol=1e-15)


def pin_mean_infinities(O):
    assert math.isnan(O.reduce_stats(np.array([np.inf, -np.inf, 1.0], np.float32))["mean_kl"])
    assert O.reduce_stats(np.array([np.inf, 2.0], np.float32))["mean_kl"] == math.inf
    assert O.reduce_stats(np.array([-np.inf, 2.0], np.float32))["mean_kl"] == -math.inf


def pin_uniform_perplexity(O):
    # A uniform reference over V ids has perplexity V.
    V = 4096
    res = O.full_vocab(np.zeros((5, V)), np.zeros((5, V)), np.arange(5))
    st = O.reduce_stats(res["kl"], res["ref_argmax"], res["cand_argmax"], None,
                        res["ref_target_lp"], res["cand_target_lp"])
    assert _close(st["ref_ppl"], V, rtol=1e-6)
    assert st["top1_rate"] == 1.0 and st["ppl_ratio"] == 1.0


# ---------------------------------------------------------------------------
# shared head
# ---------------------------------------------------------------------------

def pin_shared_head_matmul(O):
    rng = np.random.default_rng(11)
    n, K, V = 3, 5, 7
    H = rng.normal(size=(n, K))
    W = rng.normal(size=(V, K))
    L = O.shared_head_logits(H, W)
    for i in range(n):
        for v in range(V):
            acc = 0.0
            for k in range(K):
                acc += H[i, k] * W[v, k]
            assert _close(L[i, v], acc, rtol=1e-12, atol=1e-14)
    res = O.shared_head(H, H.copy(), W, np.zeros(n, dtype=np.int64), v_chunk=3)
    assert np.all(res["kl"] == 0.0)
    res2 = O.shared_head(H, H + 0.1, W, np.zeros(n, dtype=np.int64), v_chunk=3)
    for i in range(n):
        assert _close(res2["kl"][i], O.full_vocab_row(H[i] @ W.T, (H[i] + 0.1) @ W.T)["kl"], rtol=1e-12)


def pin_logit_error_bound_closed_form(O):
    # K = 2, h = (1, -2), w = (3, 0.5): sum |h_k w_k| = 3 + 1 = 4 and
    # gamma_2 = 2 u, so the bound is 8 u = 2^-21 at u = 2^-24, exactly.
    assert O.logit_error_bound(np.array([1.0, -2.0]), np.array([3.0, 0.5])) == 2.0 ** -21
    # K = 3 with cancelling products: |h.w| = 0 but sum |h_k w_k| = 6, so
    # the bound is gamma_3 * 6 = 18 u (a bound on |h.w| alone would be 0)
    assert O.logit_error_bound(np.array([1.0, 1.0, 1.0]), np.array([2.0, -3.0, 1.0])) == 18.0 * 2.0 ** -24
    # the unit roundoff is a parameter: bf16 (u = 2^-8), K = 1, |h w| = 0.75
    assert O.logit_error_bound(np.array([-0.5]), np.array([1.5]), unit_roundoff=2.0 ** -8) == 0.75 * 2.0 ** -8


def pin_argmax_ambiguous_threshold(O):
    # K = 1, h = (1): logits are the head's single column w_v.  With top two
    # logits 1 and 1 - d, the bounds are u and u (1 - d), so the row is
    # ambiguous exactly when d < 2 (u + u (1 - d)), i.e. d < 4u / (1 + 2u).
    u = 2.0 ** -24
    edge = 4 * u / (1 + 2 * u)
    h = np.array([1.0])
    for d, amb in ((edge * 0.98, True), (edge * 1.02, False), (0.0, True), (0.5, False)):
        W = np.array([[0.0], [1.0], [-3.0], [1.0 - d]])
        z = W @ h
        assert bool(O.argmax_ambiguous(z, h, W)) is amb, (d, amb)
    # K = 2, h = (1, 1), rows (3, -2) -> 1 and (2, -1 - d) -> 1 - d: the sums
    # of |h_k w_k| are 5 and 3 + d, so the threshold is 2 * 2u * (8 + d)
    # ~ 2^-19, far above the 2 * 2u * (2 - d) that |h.w| alone would give.
    h = np.array([1.0, 1.0])
    for d, amb in ((2.0 ** -20, True), (2.0 ** -19 * 1.01, False), (2.0 ** -19 * 0.99, True)):
        W = np.array([[3.0, -2.0], [0.0, 0.0], [2.0, -1.0 - d]])
        z = W @ h
        assert bool(O.argmax_ambiguous(z, h, W)) is amb, (d, amb)
    # the top two are found by value, whatever their positions
    W = np.array([[0.0, 0.0], [2.0, -1.0 - 2.0 ** -20], [-1.0, 0.0], [3.0, -2.0]])
    assert bool(O.argmax_ambiguous(W @ h, h, W)) is True


def pin_argmax_ambiguous_covers_f32_sums(O):
    # Sequential float32 sums of float32 products, in several orders: any row
    # whose f32 argmax differs from the float64 one must be flagged.  Each
    # row plants a near-twin of its leading head row, at logit gaps from
    # 1e-7 to 1 (log-uniform).
    rng = np.random.default_rng(21)
    K, V, n = 256, 6, 120
    f32 = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)
    flips = flagged = 0
    for _ in range(n):
        h = f32(rng.normal(0, 1, K))
        W = f32(rng.normal(0, 0.05, (V, K)))
        W[0] = f32(W[0] + 0.25 * np.sign(h))             # a clear leader ...
        j = int(np.argmax(np.abs(h)))
        W[1] = W[0].copy()                               # ... and a near-twin
        W[1, j] = f32(W[0, j] + rng.choice([-1.0, 1.0]) * 10 ** rng.uniform(-7, 0) / abs(h[j]))
        z = W @ h
        best = int(np.argmax(z))
        amb = bool(O.argmax_ambiguous(z, h, W))
        flagged += amb
        prods = (W * h).astype(np.float32)               # the correctly rounded f32 products
        sums = []
        for order in (np.arange(K), np.arange(K)[::-1], rng.permutation(K)):
            acc = np.zeros(V, dtype=np.float32)
            for k in order:
                acc = acc + prods[:, k]
            sums.append(acc)
        # blocks of 16 summed first, then the block sums in order
        blocks = prods.reshape(V, K // 16, 16).sum(axis=2, dtype=np.float32)
        acc = np.zeros(V, dtype=np.float32)
        for b in range(K // 16):
            acc = acc + blocks[:, b]
        sums.append(acc)
        for acc in sums:
            if int(np.argmax(acc)) != best:
                flips += 1
                assert amb, ("an f32 argmax differs on a row not flagged ambiguous", z[0] - z[1])
    assert flips > 0            # the planted gaps do reach f32's rounding
    assert 0 < flagged < n      # and the bound separates wide gaps from narrow ones


# ---------------------------------------------------------------------------
# paired comparison
# ---------------------------------------------------------------------------

def _paired_case(seed, n_ctx=5, L=4, C=3, nan=True):
    rng = np.random.default_rng(seed)
    a = rng.lognormal(-6, 1.5, (n_ctx, L)).astype(np.float32)
    b = (a * rng.uniform(0.7, 1.4, (n_ctx, L))).astype(np.float32)
    if nan:
        a[0, 1] = np.nan
        b[2, 3] = np.nan
    mask = np.ones((n_ctx, L), dtype=np.uint8)
    mask[1, 0] = 0
    cluster = np.array([k % C for k in range(n_ctx)])
    return a, b, mask, cluster


def pin_paired_brute_force(O):
    # every draw of 3 clusters out of 3 (27 replicates), replicate statistics
    # from cluster multiplicities in exact rationals
    a, b, mask, cluster = _paired_case(20)
    n_ctx, L = a.shape
    C = 3
    draws = np.array([[i, j, k] for i in range(C) for j in range(C) for k in range(C)])
    r = O.paired_compare(a, b, L, cluster, draws, quantiles=(0.1, 0.5, 0.9), mask=mask)
    d = {}
    for c in range(n_ctx):
        keep = [i for i in range(L) if mask[c, i] and not (math.isnan(a[c, i]) or math.isnan(b[c, i]))]
        if keep:
            ma = sum(Fraction(float(a[c, i])) for i in keep) / len(keep)
            mb = sum(Fraction(float(b[c, i])) for i in keep) / len(keep)
            d[c] = ma - mb
    assert r["n_ctx"] == len(d)
    assert _close(r["diff"], float(sum(d.values()) / len(d)), rtol=1e-14, atol=0)
    assert r["a_lower"] == sum(1 for v in d.values() if v < 0)
    assert r["b_lower"] == sum(1 for v in d.values() if v > 0)
    for row, got in zip(draws, r["boot"]):
        mult = np.bincount(row, minlength=C)
        num = sum(mult[cluster[c]] * d[c] for c in d)
        den = sum(mult[cluster[c]] for c in d)
        assert _close(got, float(num / den), rtol=1e-13, atol=0)
    want = np.quantile(r["boot"], (0.1, 0.5, 0.9), method="linear")
    for got, w in zip(r["ci"], want):
        assert _close(got, float(w), rtol=1e-14, atol=1e-300)


def pin_paired_identical(O):
    a, _, mask, cluster = _paired_case(21, n_ctx=9, L=6)
    rs = np.random.default_rng(22).integers(0, 3, (40, 3))
    r = O.paired_compare(a, a.copy(), 6, cluster, rs, mask=mask)
    assert r["diff"] == 0.0 and r["ties"] == r["n_ctx"] and r["a_lower"] == r["b_lower"] == 0
    assert r["ci"] == [0.0, 0.0] and r["mean_a"] == r["mean_b"]


def pin_paired_constant_shift(O):
    # values on a 2^-10 grid: every mean and difference is exact
    rng = np.random.default_rng(23)
    b = (rng.integers(1, 1000, (8, 8)) / 1024.0).astype(np.float32)
    a = b + np.float32(2.0 ** -8)
    rs = rng.integers(0, 4, (30, 4))
    r = O.paired_compare(a, b, 8, np.arange(8) % 4, rs)
    assert r["diff"] == 2.0 ** -8 and r["a_lower"] == 0 and r["b_lower"] == 8
    assert all(v == 2.0 ** -8 for v in r["boot"]) and r["ci"] == [2.0 ** -8, 2.0 ** -8]


def pin_paired_each_cluster_once(O):
    # a replicate that draws every cluster once is the full sample
    a, b, mask, cluster = _paired_case(24, n_ctx=12, L=5, C=4)
    rs = np.array([np.random.default_rng(s).permutation(4) for s in range(10)])
    r = O.paired_compare(a, b, 5, cluster, rs, mask=mask)
    for v in r["boot"]:
        assert _close(v, r["diff"], rtol=1e-14, atol=0)


def pin_paired_swap(O):
    # B against A: the difference and the interval change sign, wins swap
    a, b, mask, cluster = _paired_case(25, n_ctx=10, L=7, C=4)
    rs = np.random.default_rng(26).integers(0, 4, (101, 4))
    r = O.paired_compare(a, b, 7, cluster, rs, quantiles=(0.025, 0.975), mask=mask)
    s2 = O.paired_compare(b, a, 7, cluster, rs, quantiles=(0.025, 0.975), mask=mask)
    assert s2["diff"] == -r["diff"] and s2["a_lower"] == r["b_lower"] and s2["b_lower"] == r["a_lower"]
    assert _close(s2["ci"][0], -r["ci"][1], rtol=1e-12, atol=1e-18)
    assert _close(s2["ci"][1], -r["ci"][0], rtol=1e-12, atol=1e-18)


def pin_paired_context_bootstrap(O):
    # one context per cluster and no dropped positions: an ordinary bootstrap
    # of the per-context differences
    rng = np.random.default_rng(27)
    a = rng.lognormal(-6, 1, (20, 9)).astype(np.float32)
    b = rng.lognormal(-6, 1, (20, 9)).astype(np.float32)
    rs = rng.integers(0, 20, (50, 20))
    r = O.paired_compare(a, b, 9, np.arange(20), rs)
    d = a.astype(np.float64).mean(axis=1) - b.astype(np.float64).mean(axis=1)
    for row, got in zip(rs, r["boot"]):
        assert _close(got, float(np.mean(d[row])), rtol=1e-12, atol=0)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(ORACLE)


def test_golden_bf16_self_scores():
    """Reference vs itself: mean KLD 0 and top-1 agreement 100% (golden)."""
    path = os.path.join(ROOT, "tests", "golden", "bf16_self_scores.txt")
    with open(path) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    mean_kld, top1 = float(rows[0][0]), float(rows[0][1])
    rng = np.random.default_rng(12)
    X = rng.normal(0, 2, (16, 4096))
    res = ORACLE.full_vocab(X, X.copy(), rng.integers(0, 4096, 16))
    st = ORACLE.reduce_stats(res["kl"], res["ref_argmax"], res["cand_argmax"])
    assert st["mean_kl"] == mean_kld and st["top1_rate"] == top1
    ids = np.stack([rng.permutation(4096)[:64] for _ in range(16)])
    lp = np.sort(np.log(rng.dirichlet(np.ones(100), 16)[:, :64]), axis=1)[:, ::-1]
    tr = ORACLE.topk_tail(ids, lp, ids, lp, 4096)
    st2 = ORACLE.reduce_stats(tr["kl"], top1=tr["top1"])
    assert st2["mean_kl"] == mean_kld and st2["top1_rate"] == top1


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin
# ---------------------------------------------------------------------------

MUTANTS = [
    ("KL direction reversed", "terms = p[live] * (lp[live] - lq[live])",
     "terms = np.exp(lq[live]) * (lq[live] - lp[live])"),
    ("log-softmax sign", "return (z - m) - log_s", "return (z - m) + log_s"),
    ("normaliser without max", "return (z - m) - log_s", "return z - log_s"),
    ("argmax picks the last tie", "out[\"ref_argmax\"] = int(np.argmax(x))",
     "out[\"ref_argmax\"] = int(x.shape[0] - 1 - np.argmax(x[::-1]))"),
    ("candidate target from the reference", "out[\"cand_target_lp\"] = float(lq[t])",
     "out[\"cand_target_lp\"] = float(lp[t])"),
    ("spread over V instead of V - k", "spread = leftover / (vocab - k)\n    log_spread",
     "spread = leftover / vocab\n    log_spread"),
    ("tail term dropped", "kl += p_tail * (math.log(p_tail) - math.log(max(q_tail, Q_FLOOR)))",
     "kl += 0.0"),
    ("unmatched ids get the whole leftover", "            q[j] = spread\n            logq[j] = log_spread",
     "            q[j] = leftover\n            logq[j] = math.log(max(leftover, Q_FLOOR))"),
    ("q_tail from the reference side", "q_tail = 1.0 - float(np.sum(q))", "q_tail = 1.0 - float(np.sum(p))"),
    ("percentile index n q", "h = (n - 1) * float(q)", "h = n * float(q) - 0.5"),
    ("mean over all positions", "out[\"mean_kl\"] = exact_mean(vals)",
     "out[\"mean_kl\"] = exact_mean(kl.astype(np.float64))"),
    ("tail cell keeps listed ids", "rest[ids] = False", "rest[ids[:1]] = False"),
    ("sparse tail term dropped", "kl += pt * (math.log(pt) - math.log(max(q_tail, Q_FLOOR)))", "kl += 0.0"),
    ("listed cells scored against p", "kl = float(np.sum(p[live] * (lp[live] - lq_all[ids][live])))",
     "kl = float(np.sum(p[live] * (lp[live] - lp[live])))"),
    ("default tail from the candidate", "pt = (1.0 - float(np.sum(p)))",
     "pt = (1.0 - float(np.sum(np.exp(lq_all[ids]))))"),
    ("reference top-1 from the last listed id", "out[\"top1\"] = int(int(ids[0]) == out[\"cand_argmax\"])",
     "out[\"top1\"] = int(int(ids[-1]) == out[\"cand_argmax\"])"),
    ("capture tail from the listed ids", "out[\"tail\"] = math.fsum(p[rest].tolist())",
     "out[\"tail\"] = math.fsum(p[top].tolist())"),
    ("capture entropy sign", "out[\"entropy\"] = -math.fsum((p[live] * lp[live]).tolist())",
     "out[\"entropy\"] = math.fsum((p[live] * lp[live]).tolist())"),
    ("capture ties keep the higher id", "order = np.lexsort((np.arange(V), -lp))",
     "order = np.lexsort((-np.arange(V), -lp))"),
    ("capture NLL sign", "out[\"nll\"] = -float(lp[int(target)])", "out[\"nll\"] = float(lp[int(target)])"),
    ("paired difference reversed", "d = {c: ctx_a[c] - ctx_b[c] for c in counted}",
     "d = {c: ctx_b[c] - ctx_a[c] for c in counted}"),
    ("replicate divides by clusters drawn", "stats.append(math.fsum(terms) / cnt if cnt else math.nan)",
     "stats.append(math.fsum(terms) / len(draws) if cnt else math.nan)"),
    ("paired positions keep B's NaNs", "use = ~(np.isnan(a) | np.isnan(b))", "use = ~np.isnan(a)"),
    ("ties counted for A", "out[\"a_lower\"] = sum(1 for c in counted if d[c] < 0)",
     "out[\"a_lower\"] = sum(1 for c in counted if d[c] <= 0)"),
    ("transposed head", "return np.asarray(H, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T",
     "return (np.asarray(W, dtype=np.float64) @ np.asarray(H, dtype=np.float64).T).T[:, ::-1]"),
    ("vectorised top-k: last matching slot wins", "slot = np.argmax(eq, axis=2)",
     "slot = k - 1 - np.argmax(eq[:, :, ::-1], axis=2)"),
    ("per-position top-k: last matching slot wins", "first_slot.setdefault(cid, s)", "first_slot[cid] = s"),
    ("error bound without the length factor",
     "return H_row.shape[0] * unit_roundoff * float(h @ np.abs(np.asarray(W_row, dtype=np.float64)))",
     "return unit_roundoff * float(h @ np.abs(np.asarray(W_row, dtype=np.float64)))"),
    ("error bound from |h.w|",
     "return H_row.shape[0] * unit_roundoff * float(h @ np.abs(np.asarray(W_row, dtype=np.float64)))",
     "return H_row.shape[0] * unit_roundoff * abs(float(np.asarray(H_row) @ np.asarray(W_row)))"),
    ("ambiguity threshold ten times too wide", "return (z[i1] - z[i2]) < 2.0 * (b1 + b2)",
     "return (z[i1] - z[i2]) < 20.0 * (b1 + b2)"),
    ("ambiguity threshold without the factor two", "return (z[i1] - z[i2]) < 2.0 * (b1 + b2)",
     "return (z[i1] - z[i2]) < (b1 + b2)"),
    ("ambiguity bound from |h.w|",
     "b1 = gamma * float(h @ np.abs(np.asarray(W[i1], dtype=np.float64)))\n"
     "    b2 = gamma * float(h @ np.abs(np.asarray(W[i2], dtype=np.float64)))",
     "b1 = gamma * abs(float(np.asarray(H_row) @ np.asarray(W[i1])))\n"
     "    b2 = gamma * abs(float(np.asarray(H_row) @ np.asarray(W[i2])))"),
    ("ambiguity against the lowest logit", "i1, i2 = int(order[0]), int(order[1])",
     "i1, i2 = int(order[0]), int(order[-1])"),
]


def _load_mutant(old, new):
    with open(ORACLE_SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutant anchor not unique / missing: {old!r}"
    spec = importlib.util.spec_from_loader("oracle_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new):
    mod = _load_mutant(old, new)
    failures = 0
    for pin in PINS:
        try:
            pin(mod)
        except Exception:
            failures += 1
    assert failures > 0, f"no pin catches: {name}"
