"""Fused shared-head scoring (tcgen05 tensor cores) against the f64 oracle.

Logits are accumulated in f32 on the tensor cores and in float64 by the
oracle, so an argmax can legitimately differ where the top two logits are
closer than the f32 dot-product error bound.  Where the oracle's argmax is
provably unique the GPU's must equal it; elsewhere the GPU's choice must lie
within that bound of the true maximum.
"""
import ctypes

import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from oracle import kld_oracle as O
from quantization_fidelity_scoring_b200 import _lib
from synth import workloads as W
from tests.helpers import assert_kl_close, assert_lp_close, to_f64

pytestmark = pytest.mark.gpu


def run(d, **kw):
    st = torch.zeros(1, dtype=torch.int32, device=d["h_ref"].device)
    res = kq.kld_from_hidden_shared_head(d["h_ref"], d["h_cand"], d["W"], d["targets"], dev_status=st, **kw)
    torch.cuda.synchronize()
    res["status"] = int(st.item())
    return res


def check(res, d, rows=None):
    n = d["h_ref"].shape[0]
    rows = np.arange(n) if rows is None else np.asarray(rows)
    idx = torch.as_tensor(rows, device=d["h_ref"].device)
    H = to_f64(d["h_ref"][idx])
    Hc = to_f64(d["h_cand"][idx])
    Wf = d["W"].float().cpu().numpy()          # exact bf16 values, f32 storage
    T = d["targets"].cpu().numpy()[rows]
    want = O.shared_head(H, Hc, Wf, T)
    assert_kl_close(res["kl"].cpu().numpy()[rows], want["kl"])
    assert_lp_close(res["ref_target_lp"].cpu().numpy()[rows], want["ref_target_lp"], "ref lp")
    assert_lp_close(res["cand_target_lp"].cpu().numpy()[rows], want["cand_target_lp"], "cand lp")
    ra = res["ref_argmax"].cpu().numpy()[rows]
    ca = res["cand_argmax"].cpu().numpy()[rows]
    exact = 0
    for i in range(len(rows)):
        for got, logits, h, name in ((ra[i], want["ref_logits"][i], H[i], "ref"),
                                     (ca[i], want["cand_logits"][i], Hc[i], "cand")):
            best = int(np.argmax(logits))
            if not O.argmax_ambiguous(logits, h, Wf):
                assert got == best, (name, rows[i], got, best)        # unique: bit-exact
                exact += 1
            else:
                # several ids are within the f32 error of the top logit: the
                # GPU's choice must be one of them
                slack = 2.0 * (O.logit_error_bound(h, Wf[best]) + O.logit_error_bound(h, Wf[got]))
                assert logits[got] >= logits[best] - slack, (name, rows[i], got, best)
    assert exact >= len(rows)      # at least half of the argmaxes are provably unique
    return want


@pytest.mark.parametrize("n,K,V", [(64, 256, 4096), (100, 200, 1000), (1, 64, 300), (130, 520, 2048 + 17)])
def test_small_shapes_all_rows(cuda_device, n, K, V):
    d = W.shared_head_states(seed=W.SEED_BASE + 1300 + n + K, device=cuda_device, n_rows=n, hidden=K, vocab=V)
    res = run(d)
    assert res["status"] == 0
    check(res, d)


def test_two_position_groups(cuda_device):
    """More than 32 position blocks: tiles from two groups, rows sampled."""
    d = W.shared_head_states(seed=W.SEED_BASE + 1400, device=cuda_device, n_rows=64 * 33 + 5, hidden=128,
                             vocab=3000)
    res = run(d)
    assert res["status"] == 0
    rows = np.unique(np.concatenate([np.arange(0, d["h_ref"].shape[0], 23), [d["h_ref"].shape[0] - 1]]))
    check(res, d, rows)


def test_identical_hidden_states_give_zero(cuda_device):
    d = W.shared_head_states(seed=W.SEED_BASE + 1500, device=cuda_device, n_rows=200, hidden=512, vocab=5000)
    d["h_cand"] = d["h_ref"].clone()
    res = run(d)
    assert torch.all(res["kl"] == 0.0)
    assert torch.equal(res["ref_argmax"], res["cand_argmax"])
    assert torch.equal(res["ref_target_lp"], res["cand_target_lp"])


def test_deterministic(cuda_device):
    d = W.shared_head_states(seed=W.SEED_BASE + 1600, device=cuda_device, n_rows=256, hidden=1024, vocab=20_000)
    a, b = run(d), run(d)
    for k in ("kl", "ref_argmax", "cand_argmax", "ref_target_lp", "cand_target_lp"):
        assert torch.equal(a[k], b[k]), k


def test_full_size_sampled(cuda_device):
    """8192 positions x 5120 hidden through a 248,320 x 5120 head: 256 seeded
    rows against the oracle (its f64 logits cost 5.1 GFLOP per row), every
    row finite."""
    d = W.shared_head_states(device=cuda_device)
    res = run(d)
    assert res["status"] == 0
    n = d["h_ref"].shape[0]
    g = torch.Generator().manual_seed(11)
    rows = np.unique(np.concatenate([torch.randperm(n - 2, generator=g)[:254].numpy() + 1, [0, n - 1]]))
    assert len(rows) == 256
    check(res, d, rows)
    kl = res["kl"].cpu().numpy()
    assert np.all(np.isfinite(kl)) and kl.min() >= -1e-5


def test_bounded_wait_reports_timeout(cuda_device):
    """A TMA fill that never arrives: every wait gives up, the kernel returns
    with KLD_DEV_TIMEOUT, and the device stays usable."""
    d = W.shared_head_states(seed=W.SEED_BASE + 1700, device=cuda_device, n_rows=64, hidden=128, vocab=1024)
    n, K = d["h_ref"].shape
    V = d["W"].shape[0]
    kl = torch.empty(n, dtype=torch.float32, device=cuda_device)
    ws = torch.empty(kq.kld_shared_head_workspace_size(n, K, V), dtype=torch.uint8, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = _lib.load().kld_from_hidden_shared_head_withhold(
        p(d["h_ref"]), p(d["h_cand"]), p(d["W"]), n, K, V, p(kl), p(ws), ws.numel(), p(st),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.KLD_OK
    torch.cuda.synchronize()
    assert st.item() & _lib.KLD_DEV_TIMEOUT
    res = run(d)                       # the context still works
    assert res["status"] == 0
    check(res, d)
