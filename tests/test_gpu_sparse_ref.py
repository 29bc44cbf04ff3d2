"""Candidate full logits against a sparse top-K reference (K + 1 cells), on
the GPU against the f64 oracle."""
import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from oracle import kld_oracle as O
from quantization_fidelity_scoring_b200 import _lib
from synth import workloads as W
from tests.helpers import assert_kl_close, assert_lp_close, to_f64

pytestmark = pytest.mark.gpu


def run(cand, ref_top, ref_rows=None, targets=None, **kw):
    st = torch.zeros(1, dtype=torch.int32, device=cand.device)
    res = kq.kld_sparse_ref_score(cand, ref_top, ref_rows, targets, dev_status=st, **kw)
    torch.cuda.synchronize()
    res["status"] = int(st.item())
    return res


def padded(t, per16):
    """A copy of [n, V] rows in storage whose row stride is a multiple of 16 bytes."""
    ld = -(-t.shape[1] // per16) * per16
    base = t.new_zeros((t.shape[0], ld))
    base[:, :t.shape[1]] = t
    return base[:, :t.shape[1]]


def oracle(cand, ref_top, ref_rows, targets, rows=None, chunk=128):
    n = cand.shape[0]
    rows = np.arange(n) if rows is None else np.asarray(rows)
    ids = ref_top[:, :, 0].cpu().numpy()
    lp = ref_top[:, :, 1].contiguous().view(torch.float32).cpu().numpy().astype(np.float64)
    tail = None if ref_rows is None else ref_rows[:, 2].cpu().numpy().astype(np.float64)
    T = None if targets is None else targets.cpu().numpy()
    out = {k: [] for k in ("kl", "cand_argmax", "top1", "cand_target_lp")}
    for a in range(0, len(rows), chunk):
        r = rows[a:a + chunk]
        Y = to_f64(cand[torch.as_tensor(r, device=cand.device)])
        w = O.sparse_ref(Y, ids[r], lp[r], None if tail is None else tail[r], None if T is None else T[r])
        for k in out:
            out[k].append(w[k])
    return {k: np.concatenate(v) for k, v in out.items()}


def check(res, want, rows=None, targets=True):
    n = res["kl"].shape[0]
    rows = np.arange(n) if rows is None else np.asarray(rows)
    assert_kl_close(res["kl"].cpu().numpy()[rows], want["kl"])
    assert np.array_equal(res["cand_argmax"].cpu().numpy()[rows], want["cand_argmax"])
    assert np.array_equal(res["top1"].cpu().numpy()[rows], want["top1"])
    if targets:
        assert_lp_close(res["cand_target_lp"].cpu().numpy()[rows], want["cand_target_lp"], "cand lp")


@pytest.mark.parametrize("n,V,K,dtype", [
    (64, 4096, 512, torch.float32),
    (33, 1003, 64, torch.bfloat16),       # ragged end of the row: 3 ids past the last full vector
    (16, 300, 300, torch.float32),        # every id listed: the tail cell is empty
    (40, 5000, 1, torch.bfloat16),
    (7, 262_147, 1024, torch.bfloat16),
    (9, 70_001, 777, torch.float32),
])
def test_small_shapes_all_rows(cuda_device, n, V, K, dtype):
    d = W.sparse_ref_window(seed=W.SEED_BASE + 2000 + V + K, device=cuda_device, n_rows=n, vocab=V, k=K,
                            dtype=dtype)
    cand = padded(d["cand"], 8 if dtype == torch.bfloat16 else 4)
    res = run(cand, d["ref_top"], d["ref_rows"], d["targets"])
    assert res["status"] == 0
    check(res, oracle(cand, d["ref_top"], d["ref_rows"], d["targets"]))
    assert torch.equal(res["ref_target_lp"], -d["ref_rows"][:, 0])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("warps", [1, 2, 5, 37, 4736])
def test_warp_splits(cuda_device, dtype, warps):
    """One warp per several rows (f32 rows span two bucket windows), down to
    many pieces per row merged in index order."""
    d = W.sparse_ref_window(seed=W.SEED_BASE + 2100, device=cuda_device, n_rows=5, vocab=W.VOCAB, k=512,
                            dtype=dtype)
    res = run(d["cand"], d["ref_top"], d["ref_rows"], d["targets"], warps=warps)
    assert res["status"] == 0
    check(res, oracle(d["cand"], d["ref_top"], d["ref_rows"], d["targets"]))


def test_full_size_window_all_rows(cuda_device):
    """2047 positions x 248,320 bf16 against 512-id references: every row."""
    d = W.sparse_ref_window(device=cuda_device)
    res = run(d["cand"], d["ref_top"], d["ref_rows"], d["targets"])
    assert res["status"] == 0
    want = oracle(d["cand"], d["ref_top"], d["ref_rows"], d["targets"])
    check(res, want)
    assert np.all(np.isfinite(want["kl"]))


def test_without_stored_tail(cuda_device):
    d = W.sparse_ref_window(seed=W.SEED_BASE + 2200, device=cuda_device, n_rows=50, vocab=20_000, k=256)
    res = run(d["cand"], d["ref_top"], None, d["targets"])
    assert res["status"] == 0 and res["ref_target_lp"] is None
    check(res, oracle(d["cand"], d["ref_top"], None, d["targets"]))


def test_deterministic(cuda_device):
    d = W.sparse_ref_window(seed=W.SEED_BASE + 2300, device=cuda_device, n_rows=300, vocab=50_000, k=512)
    a = run(d["cand"], d["ref_top"], d["ref_rows"], d["targets"])
    b = run(d["cand"], d["ref_top"], d["ref_rows"], d["targets"])
    for k in ("kl", "cand_argmax", "top1", "cand_target_lp"):
        assert torch.equal(a[k], b[k]), k


def test_edge_rows(cuda_device):
    """Repeated and out-of-range ids, NaN and infinities, ties across the
    listed / unlisted boundary, ids packed into one streaming step."""
    V, K = 4096, 64
    d = W.sparse_ref_window(seed=W.SEED_BASE + 2400, device=cuda_device, n_rows=12, vocab=V, k=K,
                            dtype=torch.float32)
    cand, top, rows, tg = d["cand"].clone(), d["ref_top"].clone(), d["ref_rows"], d["targets"].clone()
    top[0, 5, 0] = top[0, 9, 0]                    # repeated id
    top[1, 3, 0] = V                               # id out of range
    cand[2, int((set(range(V)) - set(top[2, :, 0].tolist())).pop())] = float("nan")   # NaN, unlisted
    cand[3, int(top[3, 7, 0])] = float("nan")      # NaN, listed
    cand[4, int(top[4, 2, 0])] = float("-inf")     # p > 0 on a cell with q = 0
    tg[5] = V + 3                                  # target out of range
    cand[7, 11] = float("inf")
    # row 8: the maximum at a listed id and, lower, at an unlisted id
    hi = float(cand[8].max()) + 1.0
    lst = sorted(top[8, :, 0].tolist())
    unl = min(set(range(V)) - set(lst))
    cand[8, lst[-1]] = hi
    cand[8, unl] = hi
    # row 9: the same tie with the listed id lower
    lst9 = top[9, :, 0].tolist()
    lo_listed = min(lst9)
    unl9 = max(set(range(V)) - set(lst9))
    hi9 = float(cand[9].max()) + 1.0
    cand[9, lo_listed] = hi9
    cand[9, unl9] = hi9
    # row 10: listed ids 100 .. 163, all inside the first streaming step
    top[10, :, 0] = torch.arange(100, 100 + K, device=cuda_device, dtype=torch.int32)
    # row 11: a listed id with p = e^-100 (below the f32 range, not f64's)
    # where the candidate logit is -inf: KL = +inf
    top[11, K - 1, 1] = torch.tensor([-100.0], dtype=torch.float32).view(torch.int32).item()
    cand[11, int(top[11, K - 1, 0])] = float("-inf")
    res = run(cand, top, rows, tg)
    assert res["status"] == (_lib.KLD_DEV_BAD_ID | _lib.KLD_DEV_BAD_TARGET)
    want = oracle(cand, top, rows, tg)
    check(res, want)
    kl = res["kl"].cpu().numpy()
    assert np.isnan(kl[[0, 1, 2, 3, 7]]).all() and kl[4] == np.inf and kl[11] == np.inf
    assert res["cand_argmax"][8].item() == unl and res["cand_argmax"][9].item() == lo_listed
    assert np.isnan(res["cand_target_lp"][5].item())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_candidate_logits_near_the_largest_finite_values(cuda_device, dtype):
    """Candidate rows whose maximum is large: near the largest finite value
    (where y log2 e overflows f32), around 2^20 (where the one-FMA exponent
    gives way to (y - m) log2 e) and past 2^31: ties at the maximum among
    the listed ids, an unlisted one, values just below it, the rest far
    below.  Every y_i - m stays finite in f32, as the kernel's domain
    requires."""
    V, K = 5000, 64
    # (candidate maximum, fill value)
    cases = [(3.0e38, 1.0e37), (-3.0e38, -3.3e38), (1.0e38, -1.0e38), (-1.0e38, -2.0e38), (8.4e37, -8.0e37),
             (-8.4e37, -1.0e38), (1.0e9, -1.0e9), (-3.0e9, -3.1e9), (1.0e6, 1.0e6 - 40.0), (1.048e6, 1.0e6),
             (3.0e6, 2.9e6), (-1.0e6, -1.0e6 - 30.0)]
    d = W.sparse_ref_window(seed=W.SEED_BASE + 2500, device=cuda_device, n_rows=len(cases), vocab=V, k=K,
                            dtype=torch.float32)
    rng = np.random.default_rng(2500)
    top, rows, tg = d["ref_top"], d["ref_rows"], d["targets"].clone()
    cand = np.empty((len(cases), V))
    for i, (m, fill) in enumerate(cases):
        y = np.full(V, fill)
        some = rng.choice(V, 150, replace=False)
        y[some[:100]] = rng.uniform(fill, fill + 0.5 * (m - fill), 100)
        y[some[100:]] = m - rng.uniform(0.0, 12.0, 50)    # just below the maximum
        listed = top[i, :, 0].cpu().numpy()
        unlisted = np.setdiff1d(np.arange(V), listed)
        y[listed[[0, 5, 9]]] = m
        y[unlisted[i]] = m
        cand[i] = y
        tg[i] = int(listed[0]) if i % 2 == 0 else int(unlisted[i + 1])
    cand = torch.tensor(cand, dtype=torch.float32).to(dtype).to(cuda_device)
    res = run(cand, top, rows, tg)
    assert res["status"] == 0
    want = oracle(cand, top, rows, tg)
    check(res, want)
    assert np.isfinite(want["kl"]).all()
