"""Reductions on the GPU against the oracle: order statistics bit-exact on
the same f32 array, counts exact, sums within f64 rounding."""
import math

import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from oracle import kld_oracle as O

pytestmark = pytest.mark.gpu

QS = (0.0, 0.5, 0.99, 0.999, 1.0, 0.25, 0.9, 0.75)
THR = (0.0, 1e-4, 1e-3, 1e-2, 0.1, 1.0, 10.0, -1.0)


def make(n, seed, nan_every=0, dup=False):
    rng = np.random.default_rng(seed)
    kl = rng.lognormal(-7, 2.0, n).astype(np.float32)
    kl[rng.random(n) < 0.01] *= -1e-3            # tiny negative values (rounding)
    if dup:
        kl = np.round(kl * 1e3).astype(np.float32) / np.float32(1e3)   # many ties
    if nan_every:
        kl[::nan_every] = np.nan
    ra = rng.integers(-1, 50, n).astype(np.int32)
    ca = np.where(rng.random(n) < 0.9, ra, rng.integers(0, 50, n)).astype(np.int32)
    lr = (-rng.exponential(2.0, n)).astype(np.float32)
    lc = (lr - rng.exponential(0.05, n)).astype(np.float32)
    mask = (rng.random(n) < 0.85).astype(np.uint8)
    return kl, ra, ca, lr, lc, mask


def compare(st, want):
    assert st["n"] == want["n"] and st["n_nan"] == want["n_nan"]
    if want["n"]:
        assert abs(st["mean_kl"] - want["mean_kl"]) <= 1e-12 * abs(want["mean_kl"]) + 1e-300
    else:
        assert math.isnan(st["mean_kl"])
    for g, w in zip(st["q_lo"], want["q_lo"]):
        assert (g == w) or (math.isnan(g) and math.isnan(w))
    for g, w in zip(st["q_hi"], want["q_hi"]):
        assert (g == w) or (math.isnan(g) and math.isnan(w))
    for g, w in zip(st["q_value"], want["q_value"]):
        assert (g == w) or (math.isnan(g) and math.isnan(w))
    if "top1_agree" in want:
        assert st["top1_agree"] == want["top1_agree"]
    assert list(st["exceed"]) == want["exceed"]
    for key in ("ref_ppl", "cand_ppl", "ppl_ratio"):
        if key in want and want["n"]:
            assert abs(st[key] - want[key]) <= 1e-12 * abs(want[key])


@pytest.mark.parametrize("n", [1, 2, 3, 100, 2047, 8192, 8193, 65536, 65537, 300_001, 1_048_064, 5_000_000])
def test_against_oracle(cuda_device, n):
    kl, ra, ca, lr, lc, mask = make(n, seed=n, nan_every=53)
    T = lambda a: torch.tensor(a, device=cuda_device)
    st = kq.kld_reduce_stats(T(kl), T(ra), T(ca), None, T(lr), T(lc), T(mask), QS, THR)
    want = O.reduce_stats(kl, ra, ca, None, lr, lc, mask, quantiles=QS, thresholds=THR)
    compare(st, want)


@pytest.mark.parametrize("n", [5000, 200_000])
def test_ties_no_mask_top1_flags(cuda_device, n):
    kl, _, _, _, _, _ = make(n, seed=7 + n, dup=True)
    flags = (np.arange(n) % 3 == 0).astype(np.uint8)
    T = lambda a: torch.tensor(a, device=cuda_device)
    st = kq.kld_reduce_stats(T(kl), top1=T(flags), quantiles=QS, thresholds=THR[:3])
    want = O.reduce_stats(kl, top1=flags, quantiles=QS, thresholds=THR[:3])
    compare(st, want)
    assert st["top1_agree"] == int(flags.sum())


def test_special_values(cuda_device):
    kl = np.array([np.inf, 0.0, -0.0, 1e-30, np.nan, 5.0, -np.inf, 1e-45], dtype=np.float32)
    T = lambda a: torch.tensor(a, device=cuda_device)
    st = kq.kld_reduce_stats(T(kl), quantiles=QS)
    want = O.reduce_stats(kl, quantiles=QS)
    assert st["n"] == 7 and st["n_nan"] == 1 and st["top1_agree"] == -1
    assert math.isnan(st["mean_kl"]) and math.isnan(want["mean_kl"])   # +inf and -inf together
    for key in ("q_lo", "q_hi", "q_value"):
        for g, w in zip(st[key], want[key]):
            assert (g == w) or (math.isnan(g) and math.isnan(w)), key


def test_empty_and_all_nan(cuda_device):
    for kl in (np.zeros(0, np.float32), np.full(10, np.nan, np.float32)):
        st = kq.kld_reduce_stats(torch.tensor(kl, device=cuda_device), quantiles=(0.5,), thresholds=(0.1,))
        assert st["n"] == 0 and math.isnan(st["mean_kl"]) and math.isnan(st["q_value"][0])
        assert st["exceed"] == [0]


def test_deterministic_large(cuda_device):
    kl, ra, ca, lr, lc, mask = make(2_000_000, seed=99)
    T = lambda a: torch.tensor(a, device=cuda_device)
    args = (T(kl), T(ra), T(ca), None, T(lr), T(lc), T(mask), QS, THR)
    a = kq.kld_reduce_stats(*args)
    b = kq.kld_reduce_stats(*args)
    assert a == b or all((a[k] == b[k]) or (a[k] != a[k] and b[k] != b[k]) for k in a)


def test_grid_barrier_timeout_is_reported(cuda_device):
    """The cooperative reduction's grid barriers are bounded waits: with one
    CTA withheld (a test hook) the others give up, report KLD_DEV_TIMEOUT and
    return; the next call on the same context and workspace is correct."""
    import ctypes
    from quantization_fidelity_scoring_b200 import _lib
    n = 100_000
    kl, ra, ca, lr, lc, mask = make(n, seed=6, nan_every=17)
    T = lambda a: torch.tensor(a, device=cuda_device)
    dk, dra, dca, dlr, dlc, dm = (T(a) for a in (kl, ra, ca, lr, lc, mask))
    ws = torch.empty(kq.kld_reduce_workspace_size(n), dtype=torch.uint8, device=cuda_device)
    out = torch.zeros(280, dtype=torch.uint8, device=cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    qs = (ctypes.c_double * len(QS))(*QS)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = _lib.load().kld_reduce_stats_withhold(p(dk), p(dra), p(dca), None, p(dlr), p(dlc), p(dm), n,
                                               ctypes.cast(qs, ctypes.c_void_p), len(QS), None, 0, p(out), p(ws),
                                               ws.numel(), p(status),
                                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() & 0x4                     # KLD_DEV_TIMEOUT
    st = kq.kld_reduce_stats(dk, dra, dca, None, dlr, dlc, dm, QS, THR, workspace=ws)
    compare(st, O.reduce_stats(kl, ra, ca, None, lr, lc, mask, quantiles=QS, thresholds=THR))
