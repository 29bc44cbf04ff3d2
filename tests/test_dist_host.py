"""Host logic of the multi-rank bench path, on CPU with two gloo ranks.

With N GPUs every rank scores its own window (weak scaling): ranks draw
distinct inputs, the timed duration is the slowest rank's, and the reported
rate counts every rank's positions.  The reference arm runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
        w, r, lr = bench.rank_env()
        slow = 1.5 + rank                     # rank 1 is the slow one
        res = {
            "env": [w, r, lr],
            "max": bench.max_over_ranks(slow, torch.device("cpu"), world),
            "seed": bench.window_seed(rank),
            "rate": bench.whole_job_rate(2047, world, 10, bench.max_over_ranks(slow, torch.device("cpu"), world)),
        }
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_slowest_time(tmp_path):
    world, port = 2, free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    for r, x in enumerate(res):
        assert x["env"] == [world, r, r]
        assert x["max"] == 2.5                       # the slowest rank, on every rank
        assert x["rate"] == pytest.approx(2047 * world * 10 / 2.5)
    assert res[0]["seed"] != res[1]["seed"]          # each rank scores its own window


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, torch.device("cpu"), 1) == 3.0
    assert bench.whole_job_rate(100, 1, 4, 2.0) == 200.0


def test_reference_arm_under_torchrun_prints_once(tmp_path):
    """Two ranks under torchrun: rank 0 prints one JSON line, rank 1 exits 0
    without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-seconds", "1"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    p = subprocess.run(cmd, cwd=str(tmp_path), env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0 and line["higher_is_better"] is True


class _StampStep:
    """Stands in for the library's shard step on CPU: writes (rank, step)
    into this rank's block and checks the blocks gathered from the previous
    step came from every rank, in rank order."""
    block_bytes = 64

    def __init__(self, rank, world):
        self.rank, self.world, self.seen = rank, world, []

    def __call__(self, step, n_shards, gathered, block_out, *arrays, out=None, workspace=None, **kw):
        assert n_shards == self.world
        if step > 0:
            g = gathered.view(self.world, self.block_bytes)
            for r in range(self.world):
                assert g[r, 0].item() == r and g[r, 1].item() == step - 1, (step, r, g[r, :2])
            self.seen.append(step)
        if block_out is not None:
            block_out.zero_()
            block_out[0], block_out[1] = self.rank, step
        else:
            out.fill_(7)


def _shard_main(rank, world, port, out_dir):
    from quantization_fidelity_scoring_b200 import shards
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        fake = _StampStep(rank, world)
        kl = torch.zeros(5 + rank)
        out = shards.reduce_stats_across_ranks(kl, step_fn=fake)
        with open(os.path.join(out_dir, f"shard{rank}.json"), "w") as f:
            json.dump({"seen": fake.seen, "out": int(out[0].item())}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shard_exchange_two_gloo_ranks(tmp_path):
    """The sharded statistics' exchange: after every step each rank holds
    every rank's block, in rank order, and the last step runs everywhere."""
    world, port = 2, free_port()
    mp.start_processes(_shard_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    for r in range(world):
        res = json.loads((tmp_path / f"shard{r}.json").read_text())
        assert res["seen"] == [1, 2, 3, 4] and res["out"] == 7
