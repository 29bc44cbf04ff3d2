"""kld_full_vocab_noalloc: the entry for callers that cannot allocate.

Some callers of this library cannot allocate device memory where they score
(their framework owns all device memory through its own pool, they run at
their memory limit, or they must not risk the synchronisation an allocation
can cause), so they cannot pass kld_full_vocab a workspace.  The no-alloc
entry uses a fixed array inside the library instead.  These tests call it
through the C ABI and compare it with kld_full_vocab on the same inputs and
with the f64 oracle, for calls in a row (the array keeps the previous call's
contents, which must not leak into the next call), including one call at the
largest row count the array holds.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from quantization_fidelity_scoring_b200 import _lib
from oracle.pool import OraclePool
from synth import workloads as W
from tests.helpers import assert_kl_close, assert_lp_close, check_full_vocab, to_f64

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_noalloc(ref, cand, targets, status):
    n, V = ref.shape
    dev = ref.device
    out = dict(kl=torch.empty(n, dtype=torch.float32, device=dev),
               ref_argmax=torch.empty(n, dtype=torch.int32, device=dev),
               cand_argmax=torch.empty(n, dtype=torch.int32, device=dev),
               ref_target_lp=torch.empty(n, dtype=torch.float32, device=dev),
               cand_target_lp=torch.empty(n, dtype=torch.float32, device=dev))
    dtype = _lib.KLD_BF16 if ref.dtype == torch.bfloat16 else _lib.KLD_F32
    lib = _lib.load()
    st = lib.kld_full_vocab_noalloc(_p(ref), _p(cand), dtype, n, V, ref.stride(0), cand.stride(0),
                                    _p(targets), _p(out["kl"]), _p(out["ref_argmax"]),
                                    _p(out["cand_argmax"]), _p(out["ref_target_lp"]),
                                    _p(out["cand_target_lp"]), _p(status),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def check_against_workspace_entry(got, d):
    want = kq.kld_full_vocab(d["ref"], d["cand"], d["targets"])
    torch.cuda.synchronize()
    assert_kl_close(got["kl"].cpu().numpy(), want["kl"].cpu().numpy().astype(np.float64))
    assert torch.equal(got["ref_argmax"], want["ref_argmax"])
    assert torch.equal(got["cand_argmax"], want["cand_argmax"])
    assert_lp_close(got["ref_target_lp"].cpu().numpy(), want["ref_target_lp"].cpu().numpy())
    assert_lp_close(got["cand_target_lp"].cpu().numpy(), want["cand_target_lp"].cpu().numpy())


def test_noalloc_matches_workspace_entry_and_oracle_twice(cuda_device):
    inputs = [W.window_full_vocab(seed=W.SEED_BASE + 1201, device=cuda_device, n_rows=300,
                                  vocab=W.VOCAB, dtype=torch.bfloat16),
              W.window_full_vocab(seed=W.SEED_BASE + 1202, device=cuda_device, n_rows=77,
                                  vocab=50_000, dtype=torch.float32)]
    for d in inputs:  # two calls in a row, different shapes, shared library scratch
        status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        st, got = call_noalloc(d["ref"], d["cand"], d["targets"], status)
        assert st == _lib.KLD_OK
        torch.cuda.synchronize()
        assert status.item() == 0
        check_against_workspace_entry(got, d)
        check_full_vocab(got, to_f64(d["ref"]), to_f64(d["cand"]), d["targets"].cpu().numpy())


def test_noalloc_at_its_row_limit(cuda_device):
    """KLD_NOALLOC_MAX_ROWS rows of 8,192 bf16 logits: the split then uses
    the most streaming warps and the most chunks, so the array's pieces are
    filled to the last slot.  Every row against the oracle, then a smaller
    call on the same array."""
    n = _lib.KLD_NOALLOC_MAX_ROWS
    d = W.window_full_vocab(seed=W.SEED_BASE + 1203, device=cuda_device, n_rows=n, vocab=8192,
                            dtype=torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    st, got = call_noalloc(d["ref"], d["cand"], d["targets"], status)
    assert st == _lib.KLD_OK
    torch.cuda.synchronize()
    assert status.item() == 0
    check_against_workspace_entry(got, d)
    with OraclePool() as pool:
        staged = {"X": pool.stage("x", d["ref"], "bf16"), "Y": pool.stage("y", d["cand"], "bf16"),
                  "targets": pool.stage("t", d["targets"], "int")}
        want = pool.run("full_vocab", staged, n, rows_per_job=256)
    assert_kl_close(got["kl"].cpu().numpy(), want["kl"])
    assert np.array_equal(got["ref_argmax"].cpu().numpy(), want["ref_argmax"])
    assert np.array_equal(got["cand_argmax"].cpu().numpy(), want["cand_argmax"])
    assert_lp_close(got["ref_target_lp"].cpu().numpy(), want["ref_target_lp"], "ref lp")
    assert_lp_close(got["cand_target_lp"].cpu().numpy(), want["cand_target_lp"], "cand lp")
    # a smaller call right after, on the array the full one left behind
    small = W.window_full_vocab(seed=W.SEED_BASE + 1204, device=cuda_device, n_rows=5, vocab=4096,
                                dtype=torch.float32)
    st, got = call_noalloc(small["ref"], small["cand"], small["targets"], status)
    assert st == _lib.KLD_OK
    torch.cuda.synchronize()
    assert status.item() == 0
    check_full_vocab(got, to_f64(small["ref"]), to_f64(small["cand"]), small["targets"].cpu().numpy())


def test_noalloc_refuses_more_rows_than_its_array(cuda_device):
    ref = torch.zeros((1, 64), device=cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    lib = _lib.load()
    # the row count is checked before anything is launched, so these small
    # tensors are never read as if they held that many rows
    st = lib.kld_full_vocab_noalloc(_p(ref), _p(ref), _lib.KLD_F32, _lib.KLD_NOALLOC_MAX_ROWS + 1, 64,
                                    64, 64, None, _p(status), None, None, None, None, None, None)
    assert st == _lib.KLD_ERR_UNSUPPORTED
