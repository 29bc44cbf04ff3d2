"""Shared helpers for the GPU parity tests: exact device -> f64 conversion
and the tolerance checks of the scoring contract."""
import math

import numpy as np
import torch

from oracle import kld_oracle as O

# |KL_gpu - KL_oracle| <= KL_ATOL + KL_RTOL * |KL_oracle|
KL_ATOL = 1e-5
KL_RTOL = 1e-3
# |lp_gpu - lp_oracle| <= LP_RTOL * |lp_oracle| (+ a 1e-9 floor for lp == 0)
LP_RTOL = 1e-5
LP_ATOL = 1e-9


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a device tensor (bf16, f16 or f32)."""
    c = t.detach().cpu()
    if c.dtype == torch.bfloat16:
        return O.bf16_bits_to_f64(c.view(torch.int16).numpy().view(np.uint16))
    return O.as_f64(c.numpy())


def assert_kl_close(gpu, ref, what="kl"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape
    nan_g, nan_r = np.isnan(gpu), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r), f"{what}: NaN pattern differs"
    inf_g, inf_r = np.isinf(gpu), np.isinf(ref)
    assert np.array_equal(inf_g, inf_r) and np.array_equal(gpu[inf_g], ref[inf_r]), f"{what}: inf differs"
    ok = ~(nan_r | inf_r)
    err = np.abs(gpu[ok] - ref[ok])
    bound = KL_ATOL + KL_RTOL * np.abs(ref[ok])
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {ok.sum()} outside tolerance; worst "
                           f"err {err.max():.3e} at ref {ref[ok][np.argmax(err)]:.6e}")
    return float(err.max()) if err.size else 0.0


def assert_lp_close(gpu, ref, what="lp"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    nan_g, nan_r = np.isnan(gpu), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r), f"{what}: NaN pattern differs"
    ok = ~nan_r
    err = np.abs(gpu[ok] - ref[ok])
    bound = LP_RTOL * np.abs(ref[ok]) + LP_ATOL
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} outside tolerance; worst rel "
                           f"{np.max(err / np.maximum(np.abs(ref[ok]), 1e-30)):.3e}")


def check_full_vocab(res: dict, X: np.ndarray, Y: np.ndarray, T, rows=None):
    """Compare library outputs on `rows` (all when None) with the oracle."""
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    want = O.full_vocab(X, Y, None if T is None else np.asarray(T))
    kl = res["kl"].cpu().numpy()[rows]
    assert_kl_close(kl, want["kl"])
    if res.get("ref_argmax") is not None:
        assert np.array_equal(res["ref_argmax"].cpu().numpy()[rows], want["ref_argmax"])
        assert np.array_equal(res["cand_argmax"].cpu().numpy()[rows], want["cand_argmax"])
    if T is not None:
        assert_lp_close(res["ref_target_lp"].cpu().numpy()[rows], want["ref_target_lp"], "ref lp")
        assert_lp_close(res["cand_target_lp"].cpu().numpy()[rows], want["cand_target_lp"], "cand lp")
    return want


def finite_mean(a):
    a = np.asarray(a, dtype=np.float64)
    a = a[~np.isnan(a)]
    return math.fsum(a.tolist()) / max(len(a), 1)
