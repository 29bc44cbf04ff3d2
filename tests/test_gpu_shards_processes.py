"""The shard protocol across processes: two ranks in a gloo group, each
running the library's shard steps (kld_reduce_shard_step) on its own part of
the positions on cuda:0, with the blocks moved between steps by
torch.distributed ("Qwen3.8-27B fidelity suite v5", "What is in here": tail
reports over two shards' positions).

Both ranks must end with byte-identical statistics, equal to the oracle's
over all positions: order statistics and counts exact, sums within 1e-12.
The ranks' kernels never wait on one another (the exchange is on the host),
so sharing one GPU between the two processes is safe.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import kld_oracle as O
from tests.test_gpu_reduce import QS, THR, compare, make

pytestmark = pytest.mark.gpu

NAMES = ("kl", "ra", "ca", "lr", "lc", "mask")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, data_dir, cuts):
    from datetime import timedelta

    import torch.distributed as dist

    import quantization_fidelity_scoring_b200 as kq
    from quantization_fidelity_scoring_b200 import shards
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        dev = torch.device("cuda:0")
        torch.cuda.set_device(dev)
        kq.load_library()
        a, b = cuts[rank], cuts[rank + 1]
        arrs = [torch.as_tensor(np.load(os.path.join(data_dir, f"{k}.npy"))[a:b], device=dev) for k in NAMES]
        kl, ra, ca, lr, lc, mask = arrs
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        out = shards.reduce_stats_across_ranks(kl, ra, ca, None, lr, lc, mask, QS, THR, dev_status=status,
                                               to_host=False)
        torch.cuda.synchronize()
        with open(os.path.join(data_dir, f"out{rank}.bin"), "wb") as f:
            f.write(out.cpu().numpy().tobytes())
        with open(os.path.join(data_dir, f"status{rank}.txt"), "w") as f:
            f.write(str(int(status.item())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n,cut", [(300_000, 123_457), (40_001, 0), (9, 5)])
def test_two_processes_agree_with_the_oracle(cuda_device, tmp_path, n, cut):
    import quantization_fidelity_scoring_b200 as kq
    arrays = make(n, seed=60 + n, nan_every=113)
    for k, a in zip(NAMES, arrays):
        np.save(tmp_path / f"{k}.npy", a)
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), (0, cut, n)), nprocs=world,
                       start_method="spawn")
    outs = [(tmp_path / f"out{r}.bin").read_bytes() for r in range(world)]
    assert outs[0] == outs[1]                           # identical statistics on both ranks
    assert all((tmp_path / f"status{r}.txt").read_text() == "0" for r in range(world))
    st = kq.stats_from_device(torch.frombuffer(bytearray(outs[0]), dtype=torch.uint8))
    kl, ra, ca, lr, lc, mask = arrays
    compare(st, O.reduce_stats(kl, ra, ca, None, lr, lc, mask, quantiles=QS, thresholds=THR))
