"""Seeded synthetic workloads with the shapes of the scored data.

This module only draws inputs.  It computes no KL, no argmax agreement and
no reduction: the library under test and the f64 oracle each do that from
the tensors returned here.  Everything is drawn with a seeded
``torch.Generator`` on the requested device, so a test or benchmark that
needs the oracle copies the exact device bytes back to the host.

Shapes follow the pages: V = 248,320 vocabulary entries ("Qwen3.8-27B
Quantization Challenge", "How the references were made"); 2,047 scored
positions per 2,048-token window ("Qwen3.8-27B fidelity suite v5", "What is
in here"; "Qwopus3.8-27B-Coder-Flash: quality-eval reference", "Method");
top-64 ids + fp16 log-probs sorted descending and f32 target log-probs over
512 windows ("Qwopus...", "Files"); final hidden states of width 5120 and
one bf16 LM head ("Qwen3.8-27B fidelity suite v5", "What is in here" and
"What we preserve"); a sparse reference of the 512 most likely ids with f32
log-probs, most likely first, and per row (NLL, entropy, tail mass)
("Qwen3.8-27B Quantization Challenge", "Golden distributions").  No corpus,
model or capture is reproduced: the distributions below stand in for them.

Reference rows are Gumbel-perturbed Zipf(s = 1.1) log-weights over a
per-row pseudo-random assignment of ranks to vocabulary ids, scaled by
ALPHA so that the top-64 ids hold about 95% of the mass (the average
coverage reported in "Qwopus...", "Method").
"""
from __future__ import annotations

import math

import torch

VOCAB = 248_320
ZIPF_S = 1.1
SEED_BASE = 0x5EED0000
TOPK = 64
HIDDEN = 5120
SPARSE_K = 512

# rank -> vocabulary id bijection: id = (rank * RANK_MUL + offset) mod V.
# 7919 is prime and does not divide 248,320 = 2^9 * 5 * 97.
RANK_MUL = 7919

# Scale of the Zipf/Gumbel log-weights.  Found by calibrate_alpha() (64-row
# sample, V = 248,320, top-64 mass 0.95) and checked by a CPU test.
ALPHA = 1.435
# Candidate noise (logit units) in the top-64 workload, found by
# calibrate_topk_sigma() for a mean top-64 id overlap of ~90%.
TOPK_SIGMA = 0.386


def seed_for(config: int) -> int:
    return SEED_BASE + config


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _gumbel(shape, g, device) -> torch.Tensor:
    u = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    u.clamp_(min=2.0 ** -24, max=1.0 - 2.0 ** -24)
    return -torch.log(-torch.log(u))


def _zipf_logw(vocab: int, device) -> torch.Tensor:
    r = torch.arange(vocab, device=device, dtype=torch.float32)
    return -ZIPF_S * torch.log1p(r)


def _ranks_of_ids(offsets: torch.Tensor, vocab: int) -> torch.Tensor:
    """Rank of every vocabulary id for each row's bijection ([rows, V] int64)."""
    inv = pow(RANK_MUL, -1, vocab)
    v = torch.arange(vocab, device=offsets.device, dtype=torch.int64)[None, :]
    return torch.remainder((v - offsets[:, None]) % vocab * inv, vocab)


def _ids_of_ranks(ranks: torch.Tensor, offsets: torch.Tensor, vocab: int) -> torch.Tensor:
    return torch.remainder(ranks.to(torch.int64) * RANK_MUL + offsets[:, None], vocab)


def zipf_gumbel_rows(n_rows: int, vocab: int, g, device, alpha: float = ALPHA,
                     rank_space: bool = False):
    """f32 [n_rows, vocab] reference logits alpha * (Zipf log-weight + Gumbel).

    In rank space column r holds rank r; otherwise columns are vocabulary ids
    and each row's ranks follow its own bijection.  Returns (logits, offsets).
    """
    offsets = torch.randint(0, vocab, (n_rows,), generator=g, device=device, dtype=torch.int64)
    noise = _gumbel((n_rows, vocab), g, device)
    logw = _zipf_logw(vocab, device)
    if rank_space:
        base = logw[None, :] + noise
    else:
        base = logw[_ranks_of_ids(offsets, vocab)] + noise
    return base.mul_(alpha), offsets


def calibrate_alpha(vocab: int = VOCAB, k: int = TOPK, target: float = 0.95,
                    rows: int = 64, seed: int = SEED_BASE, device="cpu") -> float:
    """Bisection for the scale that gives a mean top-k mass of `target`."""
    g = _gen(seed, device)
    z, _ = zipf_gumbel_rows(rows, vocab, g, device, alpha=1.0, rank_space=True)
    z = z.double()
    top = torch.topk(z, k, dim=1).values            # order does not depend on alpha > 0
    lo, hi = 0.1, 20.0
    for _ in range(60):
        a = 0.5 * (lo + hi)
        mass = torch.exp(torch.logsumexp(a * top, 1) - torch.logsumexp(a * z, 1)).mean().item()
        lo, hi = (a, hi) if mass < target else (lo, a)
    return 0.5 * (lo + hi)


def top1_planted_tiny(seed: int = seed_for(1), device="cpu", n_rows: int = 64,
                      vocab: int = 4096) -> dict:
    """Tiny full-vocabulary workload (64 x 4096, f32): ref ~ N(0, 2^2) with a
    +8 peak planted at a seeded index per row, candidate = ref + N(0, 0.05^2),
    uniform seeded target ids."""
    g = _gen(seed, device)
    ref = 2.0 * torch.randn((n_rows, vocab), generator=g, device=device)
    peak = torch.randint(0, vocab, (n_rows,), generator=g, device=device)
    ref[torch.arange(n_rows, device=device), peak] += 8.0
    cand = ref + 0.05 * torch.randn((n_rows, vocab), generator=g, device=device)
    targets = torch.randint(0, vocab, (n_rows,), generator=g, device=device, dtype=torch.int32)
    return dict(ref=ref.contiguous(), cand=cand.contiguous(), targets=targets)


def window_full_vocab(seed: int = seed_for(2), device="cpu", n_rows: int = 2047,
                      vocab: int = VOCAB, dtype=torch.bfloat16, sigma: float = 0.02,
                      chunk: int = 256) -> dict:
    """One scored window of full-vocabulary logits (2047 x 248,320, bf16 by
    default): ref = Zipf/Gumbel rows, candidate = ref + N(0, sigma^2) before
    rounding to `dtype`, target ids drawn from softmax(ref) by Gumbel-max."""
    g = _gen(seed, device)
    ref = torch.empty((n_rows, vocab), device=device, dtype=dtype)
    cand = torch.empty_like(ref)
    targets = torch.empty(n_rows, device=device, dtype=torch.int32)
    for a in range(0, n_rows, chunk):
        b = min(n_rows, a + chunk)
        r32, _ = zipf_gumbel_rows(b - a, vocab, g, device)
        c32 = r32 + sigma * torch.randn(r32.shape, generator=g, device=device)
        ref[a:b] = r32.to(dtype)
        cand[a:b] = c32.to(dtype)
        pick = ref[a:b].float() + _gumbel(r32.shape, g, device)
        targets[a:b] = torch.argmax(pick, dim=1).to(torch.int32)
        del r32, c32, pick
    return dict(ref=ref, cand=cand, targets=targets)


def batched_full_vocab(seed: int = seed_for(3), device="cpu", n_rows: int = 16 * 2047,
                       vocab: int = VOCAB, sigma_lo: float = 0.005, sigma_hi: float = 0.1,
                       forced_frac: float = 0.01, chunk: int = 256) -> dict:
    """Batched full-vocabulary logits (16 windows x 2047 rows, f32): same
    reference generator; candidate noise sigma per row ~ U(sigma_lo,
    sigma_hi); a seeded 1% of rows get the candidate's logit at the
    reference's second-ranked id raised to the candidate's value at the
    reference argmax + 1.0, so their argmaxes differ."""
    g = _gen(seed, device)
    ref = torch.empty((n_rows, vocab), device=device, dtype=torch.float32)
    cand = torch.empty_like(ref)
    targets = torch.empty(n_rows, device=device, dtype=torch.int32)
    sig = sigma_lo + (sigma_hi - sigma_lo) * torch.rand(n_rows, generator=g, device=device)
    n_forced = int(round(forced_frac * n_rows))
    forced = torch.randperm(n_rows, generator=g, device=device)[:n_forced]
    is_forced = torch.zeros(n_rows, dtype=torch.bool, device=device)
    is_forced[forced] = True
    for a in range(0, n_rows, chunk):
        b = min(n_rows, a + chunk)
        r32, _ = zipf_gumbel_rows(b - a, vocab, g, device)
        ref[a:b] = r32
        cand[a:b] = r32 + sig[a:b, None] * torch.randn(r32.shape, generator=g, device=device)
        pick = r32 + _gumbel(r32.shape, g, device)
        targets[a:b] = torch.argmax(pick, dim=1).to(torch.int32)
        rows = torch.nonzero(is_forced[a:b]).flatten()
        if rows.numel():
            top2 = torch.topk(r32[rows], 2, dim=1).indices
            ra = a + rows
            cand[ra, top2[:, 1]] = cand[ra, top2[:, 0]] + 1.0
        del r32, pick
    return dict(ref=ref, cand=cand, targets=targets, forced_rows=forced.sort().values)


def topk_tail_windows(seed: int = seed_for(4), device="cpu", windows: int = 512,
                      positions: int = 2047, vocab: int = VOCAB, k: int = TOPK,
                      sigma: float = TOPK_SIGMA, chunk: int = 1024) -> dict:
    """Top-k lists of a reference and a perturbed candidate ([W, P, k] int32
    ids + fp16 log-probs sorted descending, f32 target log-probs [W, P]).

    Each position is drawn as a full rank-space row (Zipf/Gumbel), the
    candidate adds N(0, sigma^2) to every logit, each side keeps its own
    top-k with log-probs relative to its full-row normaliser, and ranks map
    to vocabulary ids through the row's bijection.  The true next token is
    drawn from the reference row by Gumbel-max."""
    g = _gen(seed, device)
    n = windows * positions
    ref_ids = torch.empty((n, k), device=device, dtype=torch.int32)
    cand_ids = torch.empty_like(ref_ids)
    ref_lp = torch.empty((n, k), device=device, dtype=torch.float16)
    cand_lp = torch.empty_like(ref_lp)
    ref_t = torch.empty(n, device=device, dtype=torch.float32)
    cand_t = torch.empty_like(ref_t)
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        r, off = zipf_gumbel_rows(b - a, vocab, g, device, rank_space=True)
        c = r + sigma * torch.randn(r.shape, generator=g, device=device)
        r_norm = torch.logsumexp(r, dim=1, keepdim=True)
        c_norm = torch.logsumexp(c, dim=1, keepdim=True)
        rv, ri = torch.topk(r, k, dim=1)
        cv, ci = torch.topk(c, k, dim=1)
        ref_ids[a:b] = _ids_of_ranks(ri, off, vocab).to(torch.int32)
        cand_ids[a:b] = _ids_of_ranks(ci, off, vocab).to(torch.int32)
        ref_lp[a:b] = (rv - r_norm).to(torch.float16)
        cand_lp[a:b] = (cv - c_norm).to(torch.float16)
        t = torch.argmax(r + _gumbel(r.shape, g, device), dim=1, keepdim=True)
        ref_t[a:b] = (torch.gather(r, 1, t) - r_norm).squeeze(1)
        cand_t[a:b] = (torch.gather(c, 1, t) - c_norm).squeeze(1)
        del r, c
    shape3 = (windows, positions, k)
    return dict(ref_ids=ref_ids.view(shape3), ref_lp=ref_lp.view(shape3),
                cand_ids=cand_ids.view(shape3), cand_lp=cand_lp.view(shape3),
                ref_target_lp=ref_t.view(windows, positions),
                cand_target_lp=cand_t.view(windows, positions), vocab=vocab)


def calibrate_topk_sigma(vocab: int = VOCAB, k: int = TOPK, target: float = 0.90,
                         rows: int = 64, seed: int = SEED_BASE, device="cpu") -> float:
    """Bisection for the candidate noise giving a mean top-k id overlap of `target`."""
    lo, hi = 0.0, 4.0
    for _ in range(24):
        s = 0.5 * (lo + hi)
        g = _gen(seed, device)
        r, _ = zipf_gumbel_rows(rows, vocab, g, device, rank_space=True)
        c = r + s * torch.randn(r.shape, generator=g, device=device)
        ri = torch.topk(r, k, dim=1).indices
        ci = torch.topk(c, k, dim=1).indices
        ov = (ri[:, :, None] == ci[:, None, :]).any(2).float().mean().item()
        lo, hi = (s, hi) if ov > target else (lo, s)
    return 0.5 * (lo + hi)


def shared_head_states(seed: int = seed_for(5), device="cpu", n_rows: int = 8192,
                       hidden: int = HIDDEN, vocab: int = VOCAB, noise: float = 0.01,
                       w_std: float = 0.02, chunk: int = 8192) -> dict:
    """Final hidden states and one shared head: h_ref ~ N(0, 1) bf16 [n, K],
    h_cand = bf16(h_ref + N(0, noise^2)), W = bf16(N(0, w_std^2)) [V, K],
    uniform target ids."""
    g = _gen(seed, device)
    h32 = torch.randn((n_rows, hidden), generator=g, device=device)
    h_ref = h32.to(torch.bfloat16)
    h_cand = (h32 + noise * torch.randn(h32.shape, generator=g, device=device)).to(torch.bfloat16)
    del h32
    W = torch.empty((vocab, hidden), device=device, dtype=torch.bfloat16)
    for a in range(0, vocab, chunk):
        b = min(vocab, a + chunk)
        W[a:b] = (w_std * torch.randn((b - a, hidden), generator=g, device=device)).to(torch.bfloat16)
    targets = torch.randint(0, vocab, (n_rows,), generator=g, device=device, dtype=torch.int32)
    return dict(h_ref=h_ref, h_cand=h_cand, W=W, targets=targets)


def sparse_ref_window(seed: int = seed_for(6), device="cpu", n_rows: int = 2047, vocab: int = VOCAB,
                      k: int = SPARSE_K, dtype=torch.bfloat16, sigma: float = 0.05,
                      chunk: int = 256) -> dict:
    """A sparse reference and a candidate's full logits for one window.

    Reference, per row: a tail mass p_tail with log10 p_tail ~ U(-10, -3)
    (median ~3e-7: the pages put the median below 1e-6 at 512 ids), and k
    listed probabilities proportional to (j + 1)^-s e^{0.3 g_j} (g Gumbel,
    s ~ U(1.5, 4) per row), sorted descending and summing to 1 - p_tail.
    Listed ids are ranks 0 .. k-1 mapped through the row's id bijection, so
    they are distinct; with k = vocab every id is listed and p_tail = 0.  ref_top is int32 [n, k, 2]: (id, f32 log-prob bits).
    ref_rows is f32 [n, 3]: (NLL of the target, 0.0 in place of the entropy,
    which the score does not read, p_tail).

    Candidate full logits, per row: listed ids get log p_j + N(0, sigma^2),
    the other ids log(p_tail c / (V - k)) + N(0, 1) with c = e^{N(0, 0.5^2)},
    all shifted by U(-5, 5); 1% of rows swap the candidate values of the two
    most likely listed ids.  Targets are drawn from the listed distribution
    by Gumbel-max (an unlisted uniform id with probability p_tail)."""
    g = _gen(seed, device)
    n = n_rows
    ref_top = torch.empty((n, k, 2), device=device, dtype=torch.int32)
    ref_rows = torch.zeros((n, 3), device=device, dtype=torch.float32)
    cand = torch.empty((n, vocab), device=device, dtype=dtype)
    targets = torch.empty(n, device=device, dtype=torch.int32)
    j = torch.arange(k, device=device, dtype=torch.float32)
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        m = b - a
        log_tail = math.log(10.0) * (-10.0 + 7.0 * torch.rand(m, generator=g, device=device, dtype=torch.float64))
        if k >= vocab:          # every id listed: nothing is left for the tail
            log_tail = torch.full_like(log_tail, -math.inf)
        steep = 1.5 + 2.5 * torch.rand((m, 1), generator=g, device=device)
        logw = -steep * torch.log1p(j)[None, :] + 0.3 * _gumbel((m, k), g, device)
        logw = torch.sort(logw.double(), dim=1, descending=True).values
        lp = logw - torch.logsumexp(logw, dim=1, keepdim=True) + torch.log1p(-torch.exp(log_tail))[:, None]
        lp32 = lp.float()
        off = torch.randint(0, vocab, (m,), generator=g, device=device, dtype=torch.int64)
        ids = _ids_of_ranks(torch.arange(k, device=device)[None, :].expand(m, k), off, vocab)
        ref_top[a:b, :, 0] = ids.to(torch.int32)
        ref_top[a:b, :, 1] = lp32.view(torch.int32)
        ref_rows[a:b, 2] = torch.exp(log_tail).float()

        shift = -5.0 + 10.0 * torch.rand((m, 1), generator=g, device=device)
        c_tail = log_tail + 0.5 * torch.randn(m, generator=g, device=device, dtype=torch.float64)
        rest = (c_tail - math.log(max(vocab - k, 1))).float()[:, None]
        y = rest + torch.randn((m, vocab), generator=g, device=device)
        listed = lp32 + sigma * torch.randn((m, k), generator=g, device=device)
        swap = torch.rand(m, generator=g, device=device) < 0.01
        if k > 1 and bool(swap.any()):
            top2 = listed[swap, :2].flip(1)
            listed[swap, :2] = top2
        y.scatter_(1, ids, listed)
        cand[a:b] = (y + shift).to(dtype)

        pick = torch.argmax(lp32 + _gumbel((m, k), g, device), dim=1)
        t = torch.gather(ids, 1, pick[:, None]).squeeze(1)
        nll = -torch.gather(lp32, 1, pick[:, None]).squeeze(1)
        in_tail = torch.rand(m, generator=g, device=device, dtype=torch.float64) < torch.exp(log_tail)
        if bool(in_tail.any()):
            r = torch.randint(k, vocab, (m,), generator=g, device=device)
            t = torch.where(in_tail, _ids_of_ranks(r[:, None], off, vocab).squeeze(1), t)
            nll = torch.where(in_tail, (math.log(vocab - k) - log_tail).float(), nll)
        targets[a:b] = t.to(torch.int32)
        ref_rows[a:b, 0] = nll
        del y, listed
    return dict(cand=cand, ref_top=ref_top, ref_ids=ref_top[:, :, 0], ref_lp=ref_top[:, :, 1].view(torch.float32),
                ref_rows=ref_rows, targets=targets, vocab=vocab)


def position_results(seed: int = seed_for(7), device="cpu", n: int = 2047) -> dict:
    """Per-position results of one window, as the full-vocabulary pass
    leaves them, for timing the statistics alone: KL log-normal around
    e^-7 (a spread of e^±2), argmaxes over 50 ids agreeing 90% of the
    time, target log-probs -Exp(mean 2) for the reference and -Exp(mean
    0.05) lower for the candidate."""
    g = _gen(seed, device)
    kl = torch.exp(-7.0 + 2.0 * torch.randn(n, generator=g, device=device)).float()
    ra = torch.randint(0, 50, (n,), generator=g, device=device, dtype=torch.int32)
    other = torch.randint(0, 50, (n,), generator=g, device=device, dtype=torch.int32)
    ca = torch.where(torch.rand(n, generator=g, device=device) < 0.9, ra, other)
    lpr = 2.0 * torch.log1p(-torch.rand(n, generator=g, device=device))
    lpc = lpr + 0.05 * torch.log1p(-torch.rand(n, generator=g, device=device))
    return dict(kl=kl, ra=ra, ca=ca, lpr=lpr.float(), lpc=lpc.float())


def paired_candidates(seed: int = seed_for(8), device="cpu", n_ctx: int = 5120, ctx_len: int = 2047,
                      n_clusters: int = 842, n_boot: int = 10_000) -> dict:
    """Two candidates' per-position KL over one suite, its source clusters
    and bootstrap draws ("Qwen3.8-27B fidelity suite v5", "What is in
    here": 5,120 contexts of 2,047 scored positions over 842 source
    clusters).

    kl_a: f32 [n_ctx, ctx_len], log-normal around e^-7.5 with a spread of
    e^±2 (means near the pages' 5e-4), scaled per context by e^{N(0, 0.5^2)};
    kl_b = kl_a * e^{N(0, 0.1^2)} per position.  Contexts go to clusters in
    contiguous runs of uneven length (every cluster gets at least one).
    resample: int32 [n_boot, n_clusters], uniform draws of cluster ids."""
    g = _gen(seed, device)
    base = -7.5 + 0.5 * torch.randn((n_ctx, 1), generator=g, device=device)
    kl_a = torch.exp(base + 2.0 * torch.randn((n_ctx, ctx_len), generator=g, device=device)).float()
    kl_b = (kl_a * torch.exp(0.1 * torch.randn((n_ctx, ctx_len), generator=g, device=device))).float()
    cut = torch.randperm(max(n_ctx - 1, 1), generator=g, device=device)[:n_clusters - 1] + 1
    starts = torch.zeros(n_ctx, dtype=torch.int32, device=device)
    if n_ctx > 1 and n_clusters > 1:
        starts[cut.clamp(max=n_ctx - 1)] = 1
    cluster = (torch.cumsum(starts, 0) % max(n_clusters, 1)).to(torch.int32)
    resample = torch.randint(0, n_clusters, (n_boot, n_clusters), generator=g, device=device, dtype=torch.int32)
    return dict(kl_a=kl_a, kl_b=kl_b, cluster=cluster, resample=resample, n_clusters=n_clusters)
