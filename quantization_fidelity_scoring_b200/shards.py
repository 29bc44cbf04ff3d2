"""Statistics over positions held by several ranks.

Host-side sequencing only: every rank runs the library's shard steps
(kld_reduce_shard_step) on its own per-position arrays, and after each step
the ranks all-gather their fixed-size blocks, so no rank ever sends its
per-position arrays.  Every rank ends with identical statistics over all
ranks' positions ("Qwen3.8-27B fidelity suite v5", "What is in here": tail
reports over two shards' positions).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api
from ._lib import KLD_SHARD_STEPS


def reduce_stats_across_ranks(kl, ref_argmax=None, cand_argmax=None, top1=None, ref_target_lp=None,
                              cand_target_lp=None, mask=None, quantiles=(0.5, 0.99, 0.999), thresholds=(), *,
                              group=None, workspace=None, out=None, dev_status=None, stream=None,
                              step_fn=None, to_host: bool = True):
    """The kld_reduce_stats statistics of every rank's positions together.

    Collective: every rank of `group` calls this with the same quantiles and
    thresholds.  With NCCL the blocks move device to device; with gloo (which
    gathers host tensors) a rank's device block goes through host memory.
    `step_fn` replaces the library step (tests of the exchange on hosts
    without a GPU)."""
    step_fn = api.kld_reduce_shard_step if step_fn is None else step_fn
    world = dist.get_world_size(group)
    dev = kl.device
    bb = api.kld_reduce_shard_block_bytes() if step_fn is api.kld_reduce_shard_step else step_fn.block_bytes
    block = torch.empty(bb, dtype=torch.uint8, device=dev)
    gathered = [torch.empty(world * bb, dtype=torch.uint8, device=dev) for _ in range(2)]
    via_host = dev.type == "cuda" and dist.get_backend(group) == "gloo"
    if via_host:
        host_block = torch.empty(bb, dtype=torch.uint8)
        host_gathered = torch.empty(world * bb, dtype=torch.uint8)
    if workspace is None and step_fn is api.kld_reduce_shard_step:
        workspace = torch.empty(api.kld_reduce_shard_workspace_size(kl.shape[0]), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty(280, dtype=torch.uint8, device=dev)
    for step in range(KLD_SHARD_STEPS):
        last = step == KLD_SHARD_STEPS - 1
        step_fn(step, world, gathered[(step + 1) % 2] if step else None, None if last else block, kl, ref_argmax,
                cand_argmax, top1, ref_target_lp, cand_target_lp, mask, quantiles, thresholds,
                out=out if last else None, workspace=workspace, dev_status=dev_status, stream=stream)
        if not last:
            # alternate buffers, so a step never overwrites the blocks it is still reading
            if via_host:
                if stream is not None:
                    stream.synchronize()
                host_block.copy_(block)          # waits for the step on the current stream
                dist.all_gather_into_tensor(host_gathered, host_block, group=group)
                gathered[step % 2].copy_(host_gathered)
                if stream is not None:           # the next step reads it on `stream`
                    stream.wait_stream(torch.cuda.current_stream(dev))
            else:
                dist.all_gather_into_tensor(gathered[step % 2], block, group=group)
    if not to_host:
        return out
    return api.stats_from_device(out) if step_fn is api.kld_reduce_shard_step else out
