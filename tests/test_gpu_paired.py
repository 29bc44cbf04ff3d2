"""Paired comparison with a cluster bootstrap on the GPU against the oracle:
counts exact, means and replicate statistics within f64 summation error,
interval ends the exact percentiles of the replicates."""
import math

import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from oracle import kld_oracle as O
from synth import workloads as W

pytestmark = pytest.mark.gpu

QS = (0.025, 0.975)


def run(d, quantiles=QS, mask=None, status=None):
    boot = torch.empty(d["resample"].shape[0], dtype=torch.float64, device=d["kl_a"].device)
    r = kq.kld_paired_compare(d["kl_a"], d["kl_b"], d["cluster"], d["resample"], quantiles, mask,
                              boot_stats=boot, dev_status=status)
    return r, boot.cpu().numpy()


def oracle(d, quantiles=QS, mask=None):
    L = d["kl_a"].shape[1]
    return O.paired_compare(d["kl_a"].cpu().numpy(), d["kl_b"].cpu().numpy(), L, d["cluster"].cpu().numpy(),
                            d["resample"].cpu().numpy(), quantiles,
                            None if mask is None else mask.cpu().numpy())


def close(g, w, scale, rtol=1e-12):
    if math.isnan(w):
        return math.isnan(g)
    return abs(g - w) <= rtol * max(abs(w), scale)


def compare(r, boot, want, quantiles=QS):
    for k in ("n_ctx", "n_pos", "a_lower", "b_lower", "ties", "n_boot"):
        assert r[k] == want[k], k
    counted = want["ctx_n"] > 0
    scale = float(np.max(np.abs(want["ctx_mean_a"][counted]))) if want["n_ctx"] else 1.0
    for k in ("mean_a", "mean_b", "diff"):
        assert close(r[k], want[k], scale), (k, r[k], want[k])
    dscale = float(np.max(np.abs(want["ctx_mean_a"] - want["ctx_mean_b"])[counted])) if want["n_ctx"] else 1.0
    wb = want["boot"]
    assert np.array_equal(np.isnan(boot), np.isnan(wb))
    ok = ~np.isnan(wb)
    assert np.all(np.abs(boot[ok] - wb[ok]) <= 1e-12 * dscale)
    # the interval ends: exact percentiles of the GPU's own replicates, and
    # within summation error of the oracle's
    vals = np.sort(boot[ok])
    for q, g, w in zip(quantiles, r["ci"], want["ci"]):
        assert g == O.quantile_linear(vals, q)[0] or (math.isnan(g) and vals.size == 0)
        assert close(g, w, dscale)


@pytest.mark.parametrize("n_ctx,L,C,B", [(1, 1, 1, 1), (37, 53, 7, 300), (64, 129, 64, 257), (300, 31, 1, 100),
                                          (40, 12, 6, 25_000), (3000, 5, 2500, 150), (9000, 3, 40, 60)])
def test_against_oracle(cuda_device, n_ctx, L, C, B):
    d = W.paired_candidates(seed=90 + n_ctx, device=cuda_device, n_ctx=n_ctx, ctx_len=L, n_clusters=C,
                            n_boot=B)
    r, boot = run(d)
    compare(r, boot, oracle(d))


def test_crowded_interval_buckets(cuda_device):
    """One context far above the rest makes its cluster dominate every
    replicate that draws it: the replicates bunch into a few narrow bands of
    a wide range, so the buckets holding the interval ends overflow the
    gather buffer and the select narrows them; 25,000 replicates also leave
    the keys unstaged."""
    d = W.paired_candidates(seed=93, device=cuda_device, n_ctx=400, ctx_len=16, n_clusters=40, n_boot=25_000)
    d["kl_a"][5] += 1e6
    for q in ((0.025, 0.975), (0.0, 0.3, 0.5, 0.7, 1.0)):
        r, boot = run(d, quantiles=q)
        compare(r, boot, oracle(d, quantiles=q), quantiles=q)


def test_mask_and_nan(cuda_device):
    d = W.paired_candidates(seed=95, device=cuda_device, n_ctx=41, ctx_len=77, n_clusters=9, n_boot=211)
    d["kl_a"][3, ::5] = float("nan")
    d["kl_b"][7, ::3] = float("nan")
    d["kl_a"][11] = float("nan")                 # a context with nothing counted
    g = torch.Generator(device=cuda_device).manual_seed(96)
    mask = (torch.rand(d["kl_a"].shape, generator=g, device=cuda_device) < 0.8).to(torch.uint8)
    mask[20] = 0                                  # another one
    r, boot = run(d, quantiles=(0.0, 0.05, 0.5, 0.95, 1.0), mask=mask)
    want = oracle(d, quantiles=(0.0, 0.05, 0.5, 0.95, 1.0), mask=mask)
    assert want["n_ctx"] == 39
    compare(r, boot, want, quantiles=(0.0, 0.05, 0.5, 0.95, 1.0))


def test_identical_candidates(cuda_device):
    d = W.paired_candidates(seed=97, device=cuda_device, n_ctx=100, ctx_len=300, n_clusters=13, n_boot=500)
    d["kl_b"] = d["kl_a"].clone()
    r, boot = run(d)
    assert r["diff"] == 0.0 and r["ties"] == 100 and r["a_lower"] == r["b_lower"] == 0
    assert r["ci"] == [0.0, 0.0] and np.all(boot == 0.0)


def test_no_context_counted(cuda_device):
    d = W.paired_candidates(seed=98, device=cuda_device, n_ctx=5, ctx_len=4, n_clusters=2, n_boot=10)
    d["kl_a"][:] = float("nan")
    r, boot = run(d)
    assert r["n_ctx"] == 0 and r["n_boot"] == 0 and math.isnan(r["diff"])
    assert all(math.isnan(v) for v in r["ci"]) and np.all(np.isnan(boot))


def test_out_of_range_ids_are_flagged(cuda_device):
    d = W.paired_candidates(seed=99, device=cuda_device, n_ctx=20, ctx_len=8, n_clusters=4, n_boot=30)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    d["cluster"][3] = 4                           # one past the last cluster
    d["resample"][5, 1] = -1
    run(d, status=status)
    assert status.item() & 0x2


def test_suite_size_sampled(cuda_device):
    """The bench workload (5,120 contexts x 2,047 positions, 842 clusters,
    10,000 replicates): per-context means from the oracle for every context,
    the cluster sums and 200 sampled replicates recomputed from them."""
    d = W.paired_candidates(seed=W.seed_for(8), device=cuda_device)
    r, boot = run(d)
    a = d["kl_a"].cpu().numpy()
    b = d["kl_b"].cpu().numpy()
    cl = d["cluster"].cpu().numpy()
    rs = d["resample"].cpu().numpy()
    ma = np.array([O.exact_mean(row.astype(np.float64)) for row in a])
    mb = np.array([O.exact_mean(row.astype(np.float64)) for row in b])
    dd = ma - mb
    assert r["n_ctx"] == a.shape[0] and r["n_pos"] == a.size
    assert r["a_lower"] == int(np.sum(dd < 0)) and r["b_lower"] == int(np.sum(dd > 0))
    assert close(r["diff"], O.exact_mean(dd), float(np.max(np.abs(dd))))
    C = d["n_clusters"]
    D = [math.fsum(dd[cl == k].tolist()) for k in range(C)]
    N = np.bincount(cl, minlength=C)
    scale = float(np.max(np.abs(dd)))
    for i in np.random.default_rng(0).choice(rs.shape[0], 200, replace=False):
        want = math.fsum(D[k] for k in rs[i]) / int(N[rs[i]].sum())
        assert abs(boot[i] - want) <= 1e-12 * scale
    vals = np.sort(boot)
    assert r["ci"] == [O.quantile_linear(vals, q)[0] for q in QS]
    assert r["ci"][0] < r["diff"] < r["ci"][1]


def test_infinite_and_undefined_context_means(cuda_device):
    """A context whose A mean is +inf (a position with infinite KL) gives
    +inf replicates wherever its cluster is drawn; a context with +inf on
    both sides has an undefined difference (NaN), which poisons the
    replicates that draw it.  Counts and the exact percentiles still match
    the oracle."""
    d = W.paired_candidates(seed=93, device=cuda_device, n_ctx=30, ctx_len=20, n_clusters=10, n_boot=400)
    d["kl_a"][2, 5] = float("inf")
    d["kl_a"][17, 3] = float("inf")
    d["kl_b"][17, 9] = float("inf")
    qs = (0.0, 0.1, 0.5, 0.9, 1.0)
    r, boot = run(d, quantiles=qs)
    want = oracle(d, quantiles=qs)
    assert np.isinf(boot).any() and np.isnan(boot).any()
    for key in ("n_ctx", "n_pos", "n_boot"):
        assert r[key] == want[key], key
    ok = ~np.isnan(want["boot"])
    assert np.array_equal(np.isnan(boot), ~ok)
    fin = ok & np.isfinite(want["boot"])
    assert np.array_equal(np.isinf(boot[ok]), np.isinf(want["boot"][ok]))
    dscale = float(np.nanmax(np.abs(want["boot"][fin])))
    assert np.all(np.abs(boot[fin] - want["boot"][fin]) <= 1e-12 * dscale)
    vals = np.sort(boot[ok])
    for q, g, wv in zip(qs, r["ci"], want["ci"]):
        e = O.quantile_linear(vals, q)[0]
        assert (g == e) or (math.isnan(g) and math.isnan(e))
        assert (math.isnan(g) and math.isnan(wv)) or g == wv or abs(g - wv) <= 1e-12 * dscale
