"""The Python binding has no host path: every entry point refuses CPU
tensors with an error before anything is launched (runs without a GPU)."""
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq


def test_host_tensors_are_refused():
    x = torch.zeros(2, 64)
    xb = x.to(torch.bfloat16)
    ids = torch.zeros(2, 8, dtype=torch.int32)
    lp = torch.zeros(2, 8, dtype=torch.float16)
    kl = torch.zeros(8)
    calls = [
        lambda: kq.kld_full_vocab(x, x),
        lambda: kq.kld_full_vocab(xb, xb),
        lambda: kq.kld_topk_tail(ids, lp, ids, lp, 100),
        lambda: kq.kld_sparse_ref_score(xb, torch.zeros(2, 4, 2, dtype=torch.int32)),
        lambda: kq.kld_sparse_capture(xb, 4),
        lambda: kq.kld_from_hidden_shared_head(xb, xb, xb),
        lambda: kq.kld_reduce_stats(kl),
        lambda: kq.kld_paired_compare(x, x, torch.zeros(2, dtype=torch.int32),
                                      torch.zeros(3, 1, dtype=torch.int32)),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()


def test_library_loads_without_a_gpu():
    lib = kq.load_library()
    assert lib.kld_version() >= 100
    assert kq.kld_reduce_workspace_size(10) > 0
    assert kq.kld_paired_workspace_size(10, 3, 5) > 0
