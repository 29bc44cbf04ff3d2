"""Sparse capture of reference rows (top-K ids + log-probs, NLL, entropy,
tail mass) on the GPU against the f64 oracle."""
import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from oracle import kld_oracle as O
from oracle.pool import OraclePool
from quantization_fidelity_scoring_b200 import _lib
from synth import workloads as W
from tests.helpers import to_f64

pytestmark = pytest.mark.gpu

# entropy and tail come from f32 sums over the row (relative error ~1e-6)
H_RTOL, H_ATOL = 1e-5, 1e-7
TAIL_RTOL, TAIL_ATOL = 1e-4, 1e-12
LP_RTOL, LP_ATOL = 1e-5, 1e-9


def run(x, k, targets=None, **kw):
    st = torch.zeros(1, dtype=torch.int32, device=x.device)
    res = kq.kld_sparse_capture(x, k, targets, dev_status=st, **kw)
    torch.cuda.synchronize()
    res["status"] = int(st.item())
    return res


def padded(t, per16):
    ld = -(-t.shape[1] // per16) * per16
    base = t.new_zeros((t.shape[0], ld))
    base[:, :t.shape[1]] = t
    return base[:, :t.shape[1]]


def compare(res, want, rows):
    """Library capture outputs on `rows` against the oracle's for those rows."""
    ids = res["ids"].cpu().numpy()[rows]
    lp = res["lp"].cpu().numpy().astype(np.float64)[rows]
    out = res["rows"].cpu().numpy().astype(np.float64)[rows]
    assert np.array_equal(ids, want["ids"]), "ids differ"
    w_lp, g_lp = want["lp"], lp
    assert np.array_equal(np.isnan(g_lp), np.isnan(w_lp))
    ok = ~np.isnan(w_lp)
    assert np.all(np.abs(g_lp[ok] - w_lp[ok]) <= LP_RTOL * np.abs(w_lp[ok]) + LP_ATOL), "lp"
    g, w = out, want["rows"]
    assert np.array_equal(np.isnan(g), np.isnan(w))
    ok = ~np.isnan(w)
    inf = np.isinf(w)
    assert np.array_equal(np.isinf(g), inf) and np.array_equal(g[inf], w[inf])  # a target at -inf: NLL +inf
    ok &= ~inf
    for col, rt, at in ((0, LP_RTOL, LP_ATOL), (1, H_RTOL, H_ATOL), (2, TAIL_RTOL, TAIL_ATOL)):
        m = ok[:, col]
        err = np.abs(g[m, col] - w[m, col])
        assert np.all(err <= rt * np.abs(w[m, col]) + at), (col, err.max())


def check(res, x, k, targets, rows=None, chunk=64):
    n = x.shape[0]
    rows = np.arange(n) if rows is None else np.asarray(rows)
    T = None if targets is None else targets.cpu().numpy()[rows]
    for a in range(0, len(rows), chunk):
        r = rows[a:a + chunk]
        X = to_f64(x[torch.as_tensor(r, device=x.device)])
        compare(res, O.sparse_capture(X, k, None if T is None else T[a:a + chunk]), r)


@pytest.mark.parametrize("n,V,k,dtype", [
    (64, 4096, 512, torch.float32),      # the whole row fits the candidate buffer
    (33, 1003, 64, torch.bfloat16),      # ragged end of the row
    (16, 300, 300, torch.float32),       # every id listed
    (40, 5000, 1, torch.bfloat16),
    (9, 70_001, 777, torch.float32),     # sampled threshold
    (8, 262_147, 1024, torch.bfloat16),  # sampled threshold, ragged end, K at its limit
    (6, 90_001, 777, torch.bfloat16),    # 32-bit sort keys with 247 padding slots
    (10, 4096, 512, torch.bfloat16),     # the whole row fits the buffer, bf16
])
@pytest.mark.parametrize("exact", [False, True])
def test_shapes_all_rows(cuda_device, n, V, k, dtype, exact):
    d = W.window_full_vocab(seed=W.SEED_BASE + 3000 + V + k, device=cuda_device, n_rows=n,
                            vocab=-(-V // 8) * 8, dtype=dtype)
    x = padded(d["ref"][:, :V].contiguous(), 8 if dtype == torch.bfloat16 else 4)
    tg = torch.remainder(d["targets"], V).to(torch.int32)
    res = run(x, k, tg, exact=exact)
    assert res["status"] == 0
    check(res, x, k, tg)


def test_full_size_window_all_rows(cuda_device):
    """2047 positions x 248,320 bf16, K = 512: every row against the oracle
    (one oracle process per host core), every row's listed masses plus tail
    making 1."""
    d = W.window_full_vocab(device=cuda_device)
    res = run(d["ref"], 512, d["targets"])
    assert res["status"] == 0
    with OraclePool() as pool:
        staged = {"X": pool.stage("x", d["ref"], "bf16"), "targets": pool.stage("t", d["targets"], "int")}
        want = pool.run("sparse_capture", staged, d["ref"].shape[0], rows_per_job=4, k=512)
    compare(res, want, np.arange(d["ref"].shape[0]))
    mass = torch.exp(res["lp"].double()).sum(1) + res["rows"][:, 2].double()
    assert torch.all(torch.abs(mass - 1.0) < 1e-5)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_ties_nonfinite_and_bad_target(cuda_device, dtype):
    V, k = 70_001, 64
    d = W.window_full_vocab(seed=W.SEED_BASE + 3100, device=cuda_device, n_rows=8, vocab=70_008,
                            dtype=torch.float32)
    x = padded(d["ref"][:, :V].contiguous().to(dtype), 8 if dtype == torch.bfloat16 else 4)
    tg = torch.remainder(d["targets"], V).to(torch.int32)
    x[0] = 1.5                                      # every logit equal: the k lowest ids
    x[1, ::3] = x[1].max() + 1.0                    # 23,334 ties at the top: more than the buffer
    x[2, 5] = float("nan")
    x[3, 7] = float("inf")
    x[4] = float("-inf")                            # no finite logit
    x[5, ::2] = float("-inf")                       # half the row -inf
    x[6, 100:200] = x[6, 50]                        # ties at an arbitrary level
    tg[7] = V + 5
    res = run(x, k, tg)
    assert res["status"] == _lib.KLD_DEV_BAD_TARGET
    check(res, x, k, tg)
    assert res["ids"][0].tolist() == list(range(k))
    assert res["ids"][1].tolist() == list(range(0, 3 * k, 3))
    assert (res["ids"][2:5] == -1).all()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_long_tie_runs(cuda_device, dtype):
    """K = 1024 with long runs of equal values: a whole row equal, 600 equal
    values at the top, 300 values tied at the K-th (more than are ranked by
    counting), and runs of 40 equal values all through the list."""
    V, k = 70_001, 1024
    d = W.window_full_vocab(seed=W.SEED_BASE + 3200, device=cuda_device, n_rows=4, vocab=70_008,
                            dtype=torch.float32)
    x = padded(d["ref"][:, :V].contiguous().to(dtype), 8 if dtype == torch.bfloat16 else 4)
    tg = torch.remainder(d["targets"], V).to(torch.int32)
    x[0] = -2.0
    x[1, 1000:1600] = x[1].max() + 1.0
    srt = torch.sort(x[2].float(), descending=True).values
    kth = float(srt[k - 1])
    x[2, (x[2].float() == kth)] = kth - 1.0          # clear the natural ties there ...
    x[2, 20_000:20_300] = kth                         # ... and plant 300 of them
    order = torch.argsort(x[3].float(), descending=True)[:k]
    x[3, order] = torch.repeat_interleave(x[3, order[::40]], 40)[:k]   # runs of 40 equal values
    res = run(x, k, tg)
    assert res["status"] == 0
    check(res, x, k, tg)


def test_round_trip_through_the_score(cuda_device):
    """A candidate equal to the captured reference scores 0 against it."""
    d = W.window_full_vocab(seed=W.SEED_BASE + 3200, device=cuda_device, n_rows=64, vocab=50_000)
    cap = run(d["ref"], 512, d["targets"])
    sc = kq.kld_sparse_ref_score(d["ref"], cap["top"], cap["rows"], d["targets"])
    torch.cuda.synchronize()
    assert torch.all(sc["kl"].abs() < 1e-5)
    assert torch.all(sc["top1"] == 1)
    assert torch.allclose(sc["ref_target_lp"], sc["cand_target_lp"], rtol=1e-5, atol=1e-6)


def test_deterministic(cuda_device):
    d = W.window_full_vocab(seed=W.SEED_BASE + 3300, device=cuda_device, n_rows=100, vocab=100_000)
    a = run(d["ref"], 512, d["targets"])
    b = run(d["ref"], 512, d["targets"])
    assert torch.equal(a["top"], b["top"]) and torch.equal(a["rows"], b["rows"])
