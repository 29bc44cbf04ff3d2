"""Statistics over several shards' positions (histogram exchange) on the
GPU: every shard ends with the same statistics, equal to the oracle's over
all positions together (order statistics and counts exact)."""
import socket

import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from oracle import kld_oracle as O
from quantization_fidelity_scoring_b200 import _lib
from tests.test_gpu_reduce import QS, THR, compare, make

pytestmark = pytest.mark.gpu


def shard_stats(parts, device, quantiles=QS, thresholds=THR):
    """Run the shard steps for every shard on one device, gathering the
    blocks between steps as an all-gather would."""
    S = len(parts)
    bb = kq.kld_reduce_shard_block_bytes()
    blocks = [torch.empty(bb, dtype=torch.uint8, device=device) for _ in range(S)]
    outs = [torch.empty(280, dtype=torch.uint8, device=device) for _ in range(S)]
    ws = [torch.empty(kq.kld_reduce_shard_workspace_size(p[0].shape[0]), dtype=torch.uint8, device=device)
          for p in parts]
    gathered = None
    for step in range(_lib.KLD_SHARD_STEPS):
        last = step == _lib.KLD_SHARD_STEPS - 1
        for i, (kl, ra, ca, lr, lc, mask) in enumerate(parts):
            kq.kld_reduce_shard_step(step, S, gathered, None if last else blocks[i], kl, ra, ca, None, lr, lc,
                                     mask, quantiles, thresholds, out=outs[i] if last else None, workspace=ws[i])
        if not last:
            gathered = torch.cat(blocks)
    torch.cuda.synchronize()
    return outs


def to_dev(arrs, device):
    return [torch.as_tensor(a, device=device) for a in arrs]


@pytest.mark.parametrize("sizes", [(1000, 0, 2500), (5, 7), (1,), (70_000, 130_000, 3, 65_536)])
def test_shards_match_the_whole(cuda_device, sizes):
    n = sum(sizes)
    kl, ra, ca, lr, lc, mask = make(n, seed=40 + n, nan_every=97)
    cuts = np.cumsum((0,) + sizes)
    parts = [to_dev((kl[a:b], ra[a:b], ca[a:b], lr[a:b], lc[a:b], mask[a:b]), cuda_device)
             for a, b in zip(cuts[:-1], cuts[1:])]
    outs = shard_stats(parts, cuda_device)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])            # every shard holds the same statistics
    st = kq.stats_from_device(outs[0])
    want = O.reduce_stats(kl, ra, ca, None, lr, lc, mask, quantiles=QS, thresholds=THR)
    compare(st, want)
    # the single-call reduction over the concatenation: the same counts and order statistics
    whole = kq.kld_reduce_stats(*to_dev((kl, ra, ca), cuda_device), None,
                                *to_dev((lr, lc, mask), cuda_device), quantiles=QS, thresholds=THR)
    for key in ("n", "n_nan", "top1_agree", "exceed", "q_lo", "q_hi"):
        assert np.array_equal(np.asarray(st[key], dtype=np.float64), np.asarray(whole[key], dtype=np.float64),
                              equal_nan=True), key


def test_ties_across_shards(cuda_device):
    """Many equal values split over shards: order statistics still exact."""
    kl, ra, ca, lr, lc, mask = make(60_000, seed=41, dup=True)
    parts = [to_dev(tuple(a[i::3] for a in (kl, ra, ca, lr, lc, mask)), cuda_device) for i in range(3)]
    st = kq.stats_from_device(shard_stats(parts, cuda_device)[0])
    compare(st, O.reduce_stats(kl, ra, ca, None, lr, lc, mask, quantiles=QS, thresholds=THR))


def test_one_rank_process_group(cuda_device):
    """The cross-rank helper on a one-rank NCCL group: the same statistics
    as the single-call reduction."""
    import torch.distributed as dist
    from quantization_fidelity_scoring_b200 import shards
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=cuda_device)
    try:
        kl, ra, ca, lr, lc, mask = to_dev(make(10_000, seed=42, nan_every=31), cuda_device)
        st = shards.reduce_stats_across_ranks(kl, ra, ca, None, lr, lc, mask, quantiles=QS, thresholds=THR)
        whole = kq.kld_reduce_stats(kl, ra, ca, None, lr, lc, mask, quantiles=QS, thresholds=THR)
        for key in ("n", "n_nan", "top1_agree", "exceed", "q_lo", "q_hi"):
            assert np.array_equal(np.asarray(st[key], dtype=np.float64), np.asarray(whole[key], dtype=np.float64),
                                  equal_nan=True), key
        assert abs(st["mean_kl"] - whole["mean_kl"]) <= 1e-12 * abs(whole["mean_kl"])
    finally:
        dist.destroy_process_group()
