"""Python binding of libkld: torch tensors in, C ABI call, tensors out.

Argument marshalling only.  Every number is computed by the CUDA kernels
behind the C ABI (include/kld.h); torch provides device memory and the
current stream.  Functions carry the C names.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib


class KldError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _lib.load()
        msg = lib.kld_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != _lib.KLD_OK:
        raise KldError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(name, t, dtype=None, ndim=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D")


def _out(t, n, dtype, device):
    return torch.empty(n, dtype=dtype, device=device) if t is None else t


_DTYPES = {torch.float32: _lib.KLD_F32, torch.bfloat16: _lib.KLD_BF16}


def kld_full_vocab(ref: torch.Tensor, cand: torch.Tensor, targets: torch.Tensor | None = None, *,
                   argmax: bool = True, kl=None, ref_argmax=None, cand_argmax=None,
                   ref_target_lp=None, cand_target_lp=None, workspace=None, dev_status=None,
                   stream=None, warps: int = 0) -> dict:
    """Full-vocabulary KL / argmax / target log-probs of [n, V] logit rows
    (f32 or bf16, unit stride along V).  Outputs and the workspace are
    allocated when not given.  `warps` forces the number of streaming warps
    (tests of the piece merge)."""
    _need_cuda("ref", ref, ndim=2)
    _need_cuda("cand", cand, ndim=2)
    if ref.dtype != cand.dtype or ref.dtype not in _DTYPES:
        raise ValueError("ref and cand must both be float32 or both bfloat16")
    if ref.shape != cand.shape:
        raise ValueError("ref and cand shapes differ")
    if ref.stride(1) != 1 or cand.stride(1) != 1:
        raise ValueError("logit rows must be contiguous along the vocabulary")
    n, V = ref.shape
    dev = ref.device
    if targets is not None:
        _need_cuda("targets", targets, torch.int32, 1)
    kl = _out(kl, n, torch.float32, dev)
    if argmax:
        ref_argmax = _out(ref_argmax, n, torch.int32, dev)
        cand_argmax = _out(cand_argmax, n, torch.int32, dev)
    if targets is not None:
        ref_target_lp = _out(ref_target_lp, n, torch.float32, dev)
        cand_target_lp = _out(cand_target_lp, n, torch.float32, dev)
    lib = _lib.load()
    if workspace is None:
        workspace = torch.empty(lib.kld_full_vocab_workspace_size(n), dtype=torch.uint8, device=dev)
    args = (_ptr(ref), _ptr(cand), _DTYPES[ref.dtype], n, V, ref.stride(0), cand.stride(0),
            _ptr(targets), _ptr(kl), _ptr(ref_argmax), _ptr(cand_argmax), _ptr(ref_target_lp),
            _ptr(cand_target_lp), _ptr(workspace), workspace.numel(), _ptr(dev_status),
            _stream_handle(stream))
    if warps:
        st = lib.kld_full_vocab_split(*args, warps)
    else:
        st = lib.kld_full_vocab(*args)
    _check(st, "kld_full_vocab")
    return dict(kl=kl, ref_argmax=ref_argmax, cand_argmax=cand_argmax,
                ref_target_lp=ref_target_lp, cand_target_lp=cand_target_lp)


def kld_topk_tail(ref_ids, ref_lp, cand_ids, cand_lp, vocab: int, *, kl=None, top1=None,
                  n_matched=None, want_matched: bool = False, dev_status=None, stream=None) -> dict:
    """Top-k + tail-bucket KL and top-1 of [..., k] id (int32) / log-prob
    (float16) lists, contiguous."""
    for name, t, dt in (("ref_ids", ref_ids, torch.int32), ("cand_ids", cand_ids, torch.int32),
                        ("ref_lp", ref_lp, torch.float16), ("cand_lp", cand_lp, torch.float16)):
        _need_cuda(name, t, dt)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.shape != ref_ids.shape:
            raise ValueError("all four lists must have the same shape")
    k = ref_ids.shape[-1]
    n = ref_ids.numel() // k if k else 0
    dev = ref_ids.device
    kl = _out(kl, n, torch.float32, dev)
    top1 = _out(top1, n, torch.uint8, dev)
    if want_matched:
        n_matched = _out(n_matched, n, torch.int32, dev)
    lib = _lib.load()
    st = lib.kld_topk_tail(_ptr(ref_ids), _ptr(ref_lp), _ptr(cand_ids), _ptr(cand_lp), n, k, vocab,
                           _ptr(kl), _ptr(top1), _ptr(n_matched), _ptr(dev_status),
                           _stream_handle(stream))
    _check(st, "kld_topk_tail")
    return dict(kl=kl, top1=top1, n_matched=n_matched)


def kld_sparse_ref_score(cand: torch.Tensor, ref_top: torch.Tensor, ref_rows=None, targets=None, *,
                         kl=None, cand_argmax=None, top1=None, cand_target_lp=None, ref_target_lp=None,
                         workspace=None, dev_status=None, stream=None, warps: int = 0) -> dict:
    """Challenge score of candidate logit rows [n, V] (f32 or bf16, unit
    stride along V) against a sparse reference: ref_top int32 [n, k, 2]
    holding (id, f32 log-prob bits) pairs, contiguous; ref_rows f32 [n, 3]
    (NLL, entropy, tail mass) or None.  Outputs and the workspace are
    allocated when not given.  `warps` forces the number of streaming warps
    (tests of long pieces and of the piece merge)."""
    _need_cuda("cand", cand, ndim=2)
    if cand.dtype not in _DTYPES:
        raise ValueError("cand must be float32 or bfloat16")
    if cand.stride(1) != 1:
        raise ValueError("logit rows must be contiguous along the vocabulary")
    _need_cuda("ref_top", ref_top, torch.int32, 3)
    n, V = cand.shape
    if ref_top.shape[0] != n or ref_top.shape[2] != 2 or not ref_top.is_contiguous():
        raise ValueError("ref_top must be a contiguous int32 [n, k, 2] tensor")
    k = ref_top.shape[1]
    if ref_rows is not None:
        _need_cuda("ref_rows", ref_rows, torch.float32, 2)
        if tuple(ref_rows.shape) != (n, 3) or not ref_rows.is_contiguous():
            raise ValueError("ref_rows must be a contiguous float32 [n, 3] tensor")
    dev = cand.device
    kl = _out(kl, n, torch.float32, dev)
    cand_argmax = _out(cand_argmax, n, torch.int32, dev)
    top1 = _out(top1, n, torch.uint8, dev)
    if targets is not None:
        _need_cuda("targets", targets, torch.int32, 1)
        cand_target_lp = _out(cand_target_lp, n, torch.float32, dev)
    if ref_rows is not None:
        ref_target_lp = _out(ref_target_lp, n, torch.float32, dev)
    lib = _lib.load()
    if workspace is None:
        workspace = torch.empty(lib.kld_sparse_ref_workspace_size(n, k), dtype=torch.uint8, device=dev)
    args = (_ptr(cand), _DTYPES[cand.dtype], n, V, cand.stride(0), _ptr(ref_top), k, _ptr(ref_rows),
            _ptr(targets), _ptr(kl), _ptr(cand_argmax), _ptr(top1), _ptr(cand_target_lp), _ptr(ref_target_lp),
            _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream_handle(stream))
    st = lib.kld_sparse_ref_score_split(*args, warps) if warps else lib.kld_sparse_ref_score(*args)
    _check(st, "kld_sparse_ref_score")
    return dict(kl=kl, cand_argmax=cand_argmax, top1=top1, cand_target_lp=cand_target_lp,
                ref_target_lp=ref_target_lp)


def kld_sparse_ref_workspace_size(n_rows: int, k: int) -> int:
    return int(_lib.load().kld_sparse_ref_workspace_size(n_rows, k))


def kld_sparse_capture(logits: torch.Tensor, k: int, targets=None, *, top=None, rows=None, workspace=None,
                       dev_status=None, stream=None, exact: bool = False) -> dict:
    """Sparse record of reference logit rows [n, V] (f32 or bf16, unit
    stride along V): top int32 [n, k, 2] of (id, f32 log-prob bits), most
    likely first, and rows f32 [n, 3] of (NLL, entropy, tail mass).  Outputs
    and the workspace are allocated when not given.  `exact` sends every row
    down the exact path (tests)."""
    _need_cuda("logits", logits, ndim=2)
    if logits.dtype not in _DTYPES:
        raise ValueError("logits must be float32 or bfloat16")
    if logits.stride(1) != 1:
        raise ValueError("logit rows must be contiguous along the vocabulary")
    n, V = logits.shape
    dev = logits.device
    if targets is not None:
        _need_cuda("targets", targets, torch.int32, 1)
    top = torch.empty((n, k, 2), dtype=torch.int32, device=dev) if top is None else top
    rows = torch.empty((n, 3), dtype=torch.float32, device=dev) if rows is None else rows
    lib = _lib.load()
    if workspace is None:
        workspace = torch.empty(max(lib.kld_sparse_capture_workspace_size(n, k), 1), dtype=torch.uint8, device=dev)
    fn = lib.kld_sparse_capture_exact if exact else lib.kld_sparse_capture
    st = fn(_ptr(logits), _DTYPES[logits.dtype], n, V, logits.stride(0), k, _ptr(targets), _ptr(top), _ptr(rows),
            _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream_handle(stream))
    _check(st, "kld_sparse_capture")
    return dict(top=top, ids=top[:, :, 0], lp=top[:, :, 1].view(torch.float32), rows=rows)


def kld_sparse_capture_workspace_size(n_rows: int, k: int) -> int:
    return int(_lib.load().kld_sparse_capture_workspace_size(n_rows, k))


def kld_from_hidden_shared_head(h_ref, h_cand, head_w, targets=None, *, argmax: bool = True, kl=None,
                                ref_argmax=None, cand_argmax=None, ref_target_lp=None, cand_target_lp=None,
                                workspace=None, dev_status=None, stream=None) -> dict:
    """Full-vocabulary scores of hidden states [n, K] (bf16) through one
    head W [V, K] (bf16), all contiguous.  Outputs and the workspace are
    allocated when not given."""
    for name, t in (("h_ref", h_ref), ("h_cand", h_cand), ("head_w", head_w)):
        _need_cuda(name, t, torch.bfloat16, 2)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if h_ref.shape != h_cand.shape or head_w.shape[1] != h_ref.shape[1]:
        raise ValueError("shape mismatch between hidden states and head")
    n, K = h_ref.shape
    V = head_w.shape[0]
    dev = h_ref.device
    if targets is not None:
        _need_cuda("targets", targets, torch.int32, 1)
    kl = _out(kl, n, torch.float32, dev)
    if argmax:
        ref_argmax = _out(ref_argmax, n, torch.int32, dev)
        cand_argmax = _out(cand_argmax, n, torch.int32, dev)
    if targets is not None:
        ref_target_lp = _out(ref_target_lp, n, torch.float32, dev)
        cand_target_lp = _out(cand_target_lp, n, torch.float32, dev)
    lib = _lib.load()
    if workspace is None:
        workspace = torch.empty(lib.kld_shared_head_workspace_size(n, K, V), dtype=torch.uint8, device=dev)
    st = lib.kld_from_hidden_shared_head(_ptr(h_ref), _ptr(h_cand), _ptr(head_w), n, K, V, _ptr(targets),
                                         _ptr(kl), _ptr(ref_argmax), _ptr(cand_argmax), _ptr(ref_target_lp),
                                         _ptr(cand_target_lp), _ptr(workspace), workspace.numel(),
                                         _ptr(dev_status), _stream_handle(stream))
    _check(st, "kld_from_hidden_shared_head")
    return dict(kl=kl, ref_argmax=ref_argmax, cand_argmax=cand_argmax, ref_target_lp=ref_target_lp,
                cand_target_lp=cand_target_lp)


def kld_shared_head_workspace_size(n_rows: int, hidden: int, vocab: int) -> int:
    return int(_lib.load().kld_shared_head_workspace_size(n_rows, hidden, vocab))


def kld_full_vocab_workspace_size(n_rows: int) -> int:
    return int(_lib.load().kld_full_vocab_workspace_size(n_rows))


def kld_reduce_workspace_size(n: int) -> int:
    return int(_lib.load().kld_reduce_workspace_size(n))


def stats_to_dict(raw: _lib.KldStats) -> dict:
    d = {f: getattr(raw, f) for f, _ in raw._fields_}
    for f in ("exceed", "q_value", "q_lo", "q_hi"):
        d[f] = list(d[f])
    d["q_value"] = d["q_value"][:raw.nq]
    d["q_lo"] = d["q_lo"][:raw.nq]
    d["q_hi"] = d["q_hi"][:raw.nq]
    d["exceed"] = d["exceed"][:raw.nt]
    return d


def kld_reduce_stats(kl, ref_argmax=None, cand_argmax=None, top1=None, ref_target_lp=None,
                     cand_target_lp=None, mask=None, quantiles=(0.5, 0.99, 0.999), thresholds=(), *,
                     out=None, workspace=None, dev_status=None, stream=None, to_host: bool = True):
    """Mean / percentiles / top-1 / perplexity / exceedance over n positions.

    Returns a dict (synchronising on the copy) when to_host, else the device
    buffer holding the kld_stats struct."""
    _need_cuda("kl", kl, torch.float32, 1)
    n = kl.shape[0]
    dev = kl.device
    for name, t, dt in (("ref_argmax", ref_argmax, torch.int32), ("cand_argmax", cand_argmax, torch.int32),
                        ("top1", top1, torch.uint8), ("ref_target_lp", ref_target_lp, torch.float32),
                        ("cand_target_lp", cand_target_lp, torch.float32), ("mask", mask, torch.uint8)):
        _need_cuda(name, t, dt, 1)
        if t is not None and t.shape[0] != n:
            raise ValueError(f"{name} length differs from kl")
    lib = _lib.load()
    if workspace is None:
        workspace = torch.empty(lib.kld_reduce_workspace_size(n), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty(ctypes.sizeof(_lib.KldStats), dtype=torch.uint8, device=dev)
    qs = (ctypes.c_double * max(len(quantiles), 1))(*quantiles)
    ts = (ctypes.c_float * max(len(thresholds), 1))(*thresholds)
    st = lib.kld_reduce_stats(_ptr(kl), _ptr(ref_argmax), _ptr(cand_argmax), _ptr(top1),
                              _ptr(ref_target_lp), _ptr(cand_target_lp), _ptr(mask), n,
                              ctypes.cast(qs, ctypes.c_void_p), len(quantiles),
                              ctypes.cast(ts, ctypes.c_void_p), len(thresholds), _ptr(out),
                              _ptr(workspace), workspace.numel(), _ptr(dev_status),
                              _stream_handle(stream))
    _check(st, "kld_reduce_stats")
    if not to_host:
        return out
    host = out.cpu()
    raw = _lib.KldStats.from_buffer_copy(bytes(host.numpy().tobytes()))
    return stats_to_dict(raw)


def kld_paired_workspace_size(n_ctx: int, n_clusters: int, n_boot: int) -> int:
    return int(_lib.load().kld_paired_workspace_size(n_ctx, n_clusters, n_boot))


def paired_from_device(buf) -> dict:
    raw = _lib.KldPaired.from_buffer_copy(bytes(buf.cpu().numpy().tobytes()))
    out = {k: getattr(raw, k) for k in ("n_ctx", "n_pos", "a_lower", "b_lower", "ties", "n_boot",
                                        "mean_a", "mean_b", "diff", "nq")}
    out["ci"] = list(raw.ci)[:raw.nq]
    return out


def kld_paired_compare(kl_a, kl_b, cluster, resample, quantiles=(0.025, 0.975), mask=None, *, boot_stats=None,
                       out=None, workspace=None, dev_status=None, stream=None, to_host: bool = True):
    """Paired per-context comparison of candidates A and B with a
    source-cluster bootstrap interval (kld_paired_compare in include/kld.h).

    kl_a, kl_b: f32 [n_ctx, ctx_len]; mask: u8 of the same shape or None;
    cluster: int32 [n_ctx]; resample: int32 [n_boot, n_clusters], the
    bootstrap draws.  Returns a dict when to_host, else the device buffer
    holding the kld_paired struct."""
    _need_cuda("kl_a", kl_a, torch.float32, 2)
    _need_cuda("kl_b", kl_b, torch.float32, 2)
    _need_cuda("mask", mask, torch.uint8, 2)
    _need_cuda("cluster", cluster, torch.int32, 1)
    _need_cuda("resample", resample, torch.int32, 2)
    _need_cuda("boot_stats", boot_stats, torch.float64, 1)
    n_ctx, ctx_len = kl_a.shape
    if kl_b.shape != kl_a.shape or (mask is not None and mask.shape != kl_a.shape):
        raise ValueError("kl_b and mask must have kl_a's shape")
    if cluster.shape[0] != n_ctx:
        raise ValueError("cluster needs one id per context")
    n_boot, n_clusters = resample.shape
    if boot_stats is not None and boot_stats.shape[0] != n_boot:
        raise ValueError("boot_stats needs one entry per replicate")
    for name, t in (("kl_a", kl_a), ("kl_b", kl_b), ("mask", mask), ("resample", resample)):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    lib = _lib.load()
    dev = kl_a.device
    if workspace is None:
        workspace = torch.empty(lib.kld_paired_workspace_size(n_ctx, n_clusters, n_boot), dtype=torch.uint8,
                                device=dev)
    if out is None:
        out = torch.empty(ctypes.sizeof(_lib.KldPaired), dtype=torch.uint8, device=dev)
    qs = (ctypes.c_double * max(len(quantiles), 1))(*quantiles)
    st = lib.kld_paired_compare(_ptr(kl_a), _ptr(kl_b), _ptr(mask), n_ctx, ctx_len, _ptr(cluster), n_clusters,
                                _ptr(resample), n_boot, ctypes.cast(qs, ctypes.c_void_p), len(quantiles),
                                _ptr(out), _ptr(boot_stats), _ptr(workspace), workspace.numel(),
                                _ptr(dev_status), _stream_handle(stream))
    _check(st, "kld_paired_compare")
    return paired_from_device(out) if to_host else out


def kld_reduce_shard_block_bytes() -> int:
    return int(_lib.load().kld_reduce_shard_block_bytes())


def kld_reduce_shard_workspace_size(n: int) -> int:
    return int(_lib.load().kld_reduce_shard_workspace_size(n))


def kld_reduce_shard_step(step: int, n_shards: int, gathered, block_out, kl, ref_argmax=None, cand_argmax=None,
                          top1=None, ref_target_lp=None, cand_target_lp=None, mask=None,
                          quantiles=(0.5, 0.99, 0.999), thresholds=(), *, out=None, workspace, dev_status=None,
                          stream=None) -> None:
    """One step of the sharded statistics (see kld_reduce_shard_step in
    include/kld.h).  gathered / block_out / out / workspace are device byte
    tensors; every array argument is as in kld_reduce_stats."""
    _need_cuda("kl", kl, torch.float32, 1)
    n = kl.shape[0]
    for name, t, dt in (("ref_argmax", ref_argmax, torch.int32), ("cand_argmax", cand_argmax, torch.int32),
                        ("top1", top1, torch.uint8), ("ref_target_lp", ref_target_lp, torch.float32),
                        ("cand_target_lp", cand_target_lp, torch.float32), ("mask", mask, torch.uint8)):
        _need_cuda(name, t, dt, 1)
        if t is not None and t.shape[0] != n:
            raise ValueError(f"{name} length differs from kl")
    qs = (ctypes.c_double * max(len(quantiles), 1))(*quantiles)
    ts = (ctypes.c_float * max(len(thresholds), 1))(*thresholds)

    def present(t):
        # an input that is given but empty (a shard with no positions) must
        # still read as present, like the same input on the other shards;
        # with n == 0 the library never dereferences it
        if t is None:
            return None
        return _ptr(t) if t.numel() else ctypes.c_void_p(workspace.data_ptr())

    st = _lib.load().kld_reduce_shard_step(step, n_shards, _ptr(gathered), _ptr(block_out), present(kl),
                                           present(ref_argmax), present(cand_argmax), present(top1),
                                           present(ref_target_lp), present(cand_target_lp), present(mask), n,
                                           ctypes.cast(qs, ctypes.c_void_p),
                                           len(quantiles), ctypes.cast(ts, ctypes.c_void_p), len(thresholds),
                                           _ptr(out), _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                           _stream_handle(stream))
    _check(st, "kld_reduce_shard_step")


def stats_from_device(out) -> dict:
    """The kld_stats struct in a device byte tensor, as a dict (synchronises)."""
    raw = _lib.KldStats.from_buffer_copy(bytes(out.cpu().numpy().tobytes()))
    return stats_to_dict(raw)
