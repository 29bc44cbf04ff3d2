"""Top-k + tail-bucket scoring on the GPU against the f64 oracle."""
import math

import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from oracle import kld_oracle as O
from synth import workloads as W
from tests.helpers import assert_kl_close, to_f64

pytestmark = pytest.mark.gpu


def run(ri, rl, ci, cl, vocab):
    st = torch.zeros(1, dtype=torch.int32, device=ri.device)
    res = kq.kld_topk_tail(ri, rl, ci, cl, vocab, want_matched=True, dev_status=st)
    torch.cuda.synchronize()
    res["status"] = int(st.item())
    return res


def check(res, ri, rl, ci, cl, vocab):
    k = ri.shape[-1]
    want = O.topk_tail(ri.reshape(-1, k).cpu().numpy(), rl.reshape(-1, k).cpu().numpy(),
                       ci.reshape(-1, k).cpu().numpy(), cl.reshape(-1, k).cpu().numpy(), vocab)
    assert_kl_close(res["kl"].cpu().numpy(), want["kl"])
    assert np.array_equal(res["top1"].cpu().numpy(), want["top1"])
    assert np.array_equal(res["n_matched"].cpu().numpy(), want["n_matched"])
    return want


def test_full_size_windows(cuda_device):
    """512 windows x 2047 positions x top-64: every position against the oracle."""
    d = W.topk_tail_windows(device=cuda_device)
    res = run(d["ref_ids"], d["ref_lp"], d["cand_ids"], d["cand_lp"], d["vocab"])
    assert res["status"] == 0
    want = check(res, d["ref_ids"], d["ref_lp"], d["cand_ids"], d["cand_lp"], d["vocab"])
    assert 0.85 < want["n_matched"].mean() / 64 < 0.95


@pytest.mark.parametrize("k", [1, 2, 8, 16, 31, 32, 33, 40, 63, 64])
def test_list_lengths(cuda_device, k):
    d = W.topk_tail_windows(seed=W.SEED_BASE + 600 + k, device=cuda_device, windows=3, positions=257,
                            vocab=50_000, k=k, sigma=0.3)
    res = run(d["ref_ids"], d["ref_lp"], d["cand_ids"], d["cand_lp"], 50_000)
    check(res, d["ref_ids"], d["ref_lp"], d["cand_ids"], d["cand_lp"], 50_000)


def test_unaligned_rows(cuda_device):
    """k = 64 lists that start 4 bytes (ids) and 2 bytes (log-probs) past a
    16-byte boundary take the element-load path: same results as the oracle."""
    d = W.topk_tail_windows(seed=W.SEED_BASE + 650, device=cuda_device, windows=2, positions=301,
                            vocab=50_000, k=64, sigma=0.3)
    shifted = []
    for name in ("ref_ids", "ref_lp", "cand_ids", "cand_lp"):
        a = d[name].reshape(-1, 64)
        buf = torch.empty(a.numel() + 8, dtype=a.dtype, device=cuda_device)
        view = buf[1:1 + a.numel()].view(a.shape)
        view.copy_(a)
        assert view.data_ptr() % 16 != 0
        shifted.append(view)
    res = run(*shifted, 50_000)
    check(res, *shifted, 50_000)


def test_small_vocab_brute_force_cases(cuda_device):
    """V <= 16, k <= 8: random lists from valid full distributions."""
    rng = np.random.default_rng(11)
    for V in range(3, 17):
        for k in range(1, min(8, V - 1) + 1):
            n = 64
            p = rng.dirichlet(np.full(V, 0.7), n)
            q = rng.dirichlet(np.full(V, 0.7), n)
            ri = np.stack([rng.permutation(V)[:k] for _ in range(n)]).astype(np.int32)
            ci = np.stack([rng.permutation(V)[:k] for _ in range(n)]).astype(np.int32)
            rl = np.log(np.take_along_axis(p, ri, 1)).astype(np.float16)
            cl = np.log(np.take_along_axis(q, ci, 1)).astype(np.float16)
            t = [torch.tensor(a, device=cuda_device) for a in (ri, rl, ci, cl)]
            res = run(*t, V)
            check(res, *t, V)


def test_duplicates_bad_ids_and_degenerate_mass(cuda_device):
    k, V = 8, 100
    ri = np.tile(np.arange(k, dtype=np.int32), (6, 1))
    ci = np.tile(np.arange(k, dtype=np.int32)[::-1].copy(), (6, 1))
    rl = np.tile(np.log(np.full(k, 0.1)), (6, 1)).astype(np.float16)
    cl = rl.copy()
    ci[1, :] = 3                       # every candidate slot repeats one id
    ci[2, 0] = 500                     # id outside the vocabulary -> NaN + status
    cl[3, :] = np.float16(np.log(0.2))  # candidate lists hold more than all the mass
    rl[4, :] = np.float16(np.log(0.2))  # reference tail mass negative -> no tail term
    cl[5, :] = np.float16(-np.inf)      # candidate gives the listed ids zero mass
    t = [torch.tensor(a, device=cuda_device) for a in (ri, rl, ci, cl)]
    res = run(*t, V)
    assert res["status"] == 0x2
    kl = res["kl"].cpu().numpy()
    assert math.isnan(kl[2]) and res["n_matched"][2].item() == -1
    keep = [0, 1, 3, 4, 5]
    want = O.topk_tail(ri[keep], rl[keep], ci[keep], cl[keep], V)
    assert_kl_close(kl[keep], want["kl"])
    assert np.array_equal(res["n_matched"].cpu().numpy()[keep], want["n_matched"])


def test_self_is_zero_and_top1(cuda_device):
    d = W.topk_tail_windows(seed=W.SEED_BASE + 700, device=cuda_device, windows=2, positions=1000)
    res = run(d["ref_ids"], d["ref_lp"], d["ref_ids"].clone(), d["ref_lp"].clone(), d["vocab"])
    assert torch.all(res["kl"] == 0.0) and torch.all(res["top1"] == 1)
    assert torch.all(res["n_matched"] == 64)


def test_lower_bound_against_full_vocab(cuda_device):
    """Where the candidate's top-k holds all the reference's top-k ids, the tail
    rule is an exact coarsening and its KL cannot exceed the full KL
    ("Qwen3.8-27B Quantization Challenge", "The score")."""
    V, k, n = 8192, 64, 256
    d = W.window_full_vocab(seed=W.SEED_BASE + 800, device=cuda_device, n_rows=n, vocab=V,
                            dtype=torch.float32, sigma=0.01)
    full = kq.kld_full_vocab(d["ref"], d["cand"])
    lp = torch.log_softmax(d["ref"].double(), 1)
    lq = torch.log_softmax(d["cand"].double(), 1)
    rv, ri = torch.topk(lp, k, 1)
    cv, ci = torch.topk(lq, k, 1)
    res = run(ri.int().contiguous(), rv.half().contiguous(), ci.int().contiguous(), cv.half().contiguous(), V)
    contained = torch.tensor([set(a.tolist()) <= set(b.tolist()) for a, b in zip(ri.cpu(), ci.cpu())])
    assert contained.sum() > n // 2
    tail_kl = res["kl"].cpu()[contained]
    full_kl = full["kl"].cpu()[contained]
    # fp16 storage moves each listed log-prob by at most 2^-11 of itself, which
    # bounds how far the coarse KL can move: sum_j p_j (|a_j| + |b_j|) 2^-11
    p = rv.exp().cpu()[contained]
    slack = (p * (rv.abs().cpu()[contained] + cv.abs().cpu()[contained])).sum(1) * 2.0 ** -11
    assert torch.all(tail_kl.double() <= full_kl.double() + slack + 1e-6)


def test_deterministic(cuda_device):
    d = W.topk_tail_windows(seed=W.SEED_BASE + 900, device=cuda_device, windows=4, positions=2047)
    a = run(d["ref_ids"], d["ref_lp"], d["cand_ids"], d["cand_lp"], d["vocab"])
    b = run(d["ref_ids"], d["ref_lp"], d["cand_ids"], d["cand_lp"], d["vocab"])
    assert torch.equal(a["kl"], b["kl"]) and torch.equal(a["n_matched"], b["n_matched"])


def _table_slot(ids):
    """The shared-memory table slot the kernel's matching hashes an id to (a
    property of the implementation, used only to build colliding inputs)."""
    ids = np.asarray(ids, dtype=np.uint64)
    return ((ids * np.uint64(0x9E3779B1)) & np.uint64(0xFFFFFFFF)) >> np.uint64(24)


def test_colliding_candidate_ids(cuda_device):
    """Candidate lists whose ids all hash to one table slot (the longest
    probe chains the matching can meet), with repeated ids among them, next
    to a list of ordinary ids: every case matches the oracle."""
    V, k = (1 << 25) - 1, 64                     # the largest vocabulary the library takes
    rng = np.random.default_rng(11)
    pool = rng.choice(V, 1 << 20, replace=False).astype(np.int64)
    h = _table_slot(pool)
    same = pool[h == h[0]][:k]
    assert same.shape[0] == k
    rows = []
    for r in range(6):
        cand = rng.choice(same, k, replace=True) if r % 2 else rng.permutation(same)
        if r == 4:
            cand = rng.choice(V, k, replace=False)          # an ordinary row in the same launch
        ref = np.where(rng.random(k) < 0.7, cand[rng.permutation(k)], rng.choice(V, k))
        rows.append((ref.astype(np.int32), cand.astype(np.int32)))
    ri = np.stack([a for a, _ in rows])
    ci = np.stack([b for _, b in rows])
    lp = np.sort(np.log(rng.dirichlet(np.ones(80), (6,))[:, :k]), axis=1)[:, ::-1].astype(np.float16)
    cl = np.sort(np.log(rng.dirichlet(np.ones(80), (6,))[:, :k]), axis=1)[:, ::-1].astype(np.float16)
    t = [torch.tensor(np.ascontiguousarray(a), device=cuda_device) for a in (ri, lp, ci, cl)]
    res = run(*t, V)
    assert res["status"] == 0
    check(res, *t, V)
