"""The seeded generators produce the statistics their recipe promises."""
import torch

from synth import workloads as W


def test_alpha_gives_95_percent_top64_mass():
    g = W._gen(W.SEED_BASE + 99, "cpu")
    z, _ = W.zipf_gumbel_rows(24, W.VOCAB, g, "cpu", rank_space=True)
    z = z.double()
    mass = torch.exp(torch.logsumexp(torch.topk(z, 64, dim=1).values, 1) - torch.logsumexp(z, 1))
    assert 0.93 < mass.mean().item() < 0.97


def test_topk_overlap_near_90_percent():
    d = W.topk_tail_windows(seed=W.SEED_BASE + 98, windows=1, positions=48)
    ri = d["ref_ids"].reshape(-1, 64)
    ci = d["cand_ids"].reshape(-1, 64)
    ov = (ri[:, :, None] == ci[:, None, :]).any(2).float().mean().item()
    assert 0.86 < ov < 0.94
    lp = d["ref_lp"].reshape(-1, 64).float()
    assert torch.all(lp[:, :-1] >= lp[:, 1:])          # sorted descending
    assert torch.all((ri >= 0) & (ri < W.VOCAB))
    assert all(len(set(r.tolist())) == 64 for r in ri)  # distinct ids per row


def test_rank_bijection():
    V = 1000
    off = torch.tensor([0, 17, 999])
    ranks = W._ranks_of_ids(off, V)
    for row in range(3):
        assert sorted(ranks[row].tolist()) == list(range(V))
        ids = W._ids_of_ranks(ranks[row][None], off[row:row + 1], V)[0]
        assert torch.equal(ids, torch.arange(V))


def test_seeded_reproducible():
    a = W.window_full_vocab(n_rows=3, vocab=512)
    b = W.window_full_vocab(n_rows=3, vocab=512)
    assert torch.equal(a["ref"], b["ref"]) and torch.equal(a["targets"], b["targets"])
    c = W.batched_full_vocab(n_rows=200, vocab=300)
    f = c["forced_rows"]
    assert f.numel() == 2
    assert torch.all(c["cand"][f].argmax(1) != c["ref"][f].argmax(1))
