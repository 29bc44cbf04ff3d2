"""Full-vocabulary scoring on the GPU against the f64 oracle."""
import math

import numpy as np
import pytest
import torch

import quantization_fidelity_scoring_b200 as kq
from oracle import kld_oracle as O
from oracle.pool import OraclePool, concat
from synth import workloads as W
from tests.helpers import assert_kl_close, assert_lp_close, check_full_vocab, to_f64

pytestmark = pytest.mark.gpu


def run(ref, cand, targets=None, **kw):
    st = torch.zeros(1, dtype=torch.int32, device=ref.device)
    res = kq.kld_full_vocab(ref, cand, targets, dev_status=st, **kw)
    torch.cuda.synchronize()
    res["status"] = int(st.item())
    return res


def ragged(seed, device, n_rows, vocab, dtype, sigma=0.05):
    """Rows of `vocab` logits in storage padded to a 16-byte row stride."""
    per16 = 8 if dtype == torch.bfloat16 else 4
    ld = -(-vocab // per16) * per16
    d = W.window_full_vocab(seed=seed, device=device, n_rows=n_rows, vocab=ld, dtype=dtype, sigma=sigma)
    tg = torch.remainder(d["targets"], vocab).to(torch.int32)
    return d["ref"][:, :vocab], d["cand"][:, :vocab], tg


def same_layout_copy(t):
    """A copy of a row-strided view that keeps its (padded) row stride."""
    base = t.new_empty((t.shape[0], t.stride(0)))
    base[:, :t.shape[1]] = t
    return base[:, :t.shape[1]]


def test_tiny_planted_peak(cuda_device):
    d = W.top1_planted_tiny(device=cuda_device)
    res = run(d["ref"], d["cand"], d["targets"])
    assert res["status"] == 0
    check_full_vocab(res, to_f64(d["ref"]), to_f64(d["cand"]), d["targets"].cpu().numpy())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("vocab", [1, 3, 7, 8, 9, 4096 + 8, 4099, 40_003, 262_147])
def test_ragged_vocab(cuda_device, dtype, vocab):
    ref, cand, tg = ragged(W.SEED_BASE + 100 + vocab, cuda_device, 37, vocab, dtype)
    res = run(ref, cand, tg)
    check_full_vocab(res, to_f64(ref), to_f64(cand), tg.cpu().numpy())


@pytest.mark.parametrize("warps", [1, 2, 3, 7, 20, 64, 500, 4736])
def test_warp_split_and_padded_rows(cuda_device, warps):
    """Rows cut into pieces at every position a warp range can end, merged back."""
    V, ld = 30_011, 30_016
    d = W.window_full_vocab(seed=W.SEED_BASE + 200, device=cuda_device, n_rows=21, vocab=ld,
                            dtype=torch.bfloat16, sigma=0.03)
    ref, cand = d["ref"][:, :V], d["cand"][:, :V]
    tg = torch.remainder(d["targets"], V).to(torch.int32)
    res = run(ref, cand, tg, warps=warps)
    check_full_vocab(res, to_f64(ref), to_f64(cand), tg.cpu().numpy())


def test_one_window_bf16_full_size(cuda_device):
    """One scored window (2047 x 248,320, bf16): every row against the oracle."""
    d = W.window_full_vocab(device=cuda_device)
    res = run(d["ref"], d["cand"], d["targets"])
    assert res["status"] == 0
    X, Y = to_f64(d["ref"]), to_f64(d["cand"])
    check_full_vocab(res, X, Y, d["targets"].cpu().numpy())


def oracle_streamed(ref, cand, targets, kind, chunk_rows=512):
    """The f64 oracle over every row of device inputs too large for the host
    at once: row chunks (~1 GB at 512 rows of 248,320 f32 per side) are
    copied back and staged while the previous chunk is scored by one oracle
    process per host core."""
    n = ref.shape[0]
    parts, pending = [], None
    with OraclePool() as pool:
        for i, a in enumerate(range(0, n, chunk_rows)):
            b, tag = min(n, a + chunk_rows), i % 2
            staged = {"X": pool.stage(f"x{tag}", ref[a:b], kind), "Y": pool.stage(f"y{tag}", cand[a:b], kind),
                      "targets": pool.stage(f"t{tag}", targets[a:b], "int")}
            job = pool.run_async("full_vocab", staged, b - a, rows_per_job=8)
            if pending is not None:
                parts.append(concat(pending.get()))   # the chunk staged two rounds ago is free again
            pending = job
        parts.append(concat(pending.get()))
    return {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}


def test_batched_f32_full_size_all_rows(cuda_device):
    """16 windows x 2047 rows of f32 logits (65 GB): every one of the 32,752
    rows against the oracle, and every row whose candidate argmax was forced
    to differ does differ."""
    d = W.batched_full_vocab(device=cuda_device)
    res = run(d["ref"], d["cand"], d["targets"])
    assert res["status"] == 0
    want = oracle_streamed(d["ref"], d["cand"], d["targets"], "f32")
    assert_kl_close(res["kl"].cpu().numpy(), want["kl"])
    ra = res["ref_argmax"].cpu().numpy()
    ca = res["cand_argmax"].cpu().numpy()
    assert np.array_equal(ra, want["ref_argmax"]) and np.array_equal(ca, want["cand_argmax"])
    assert_lp_close(res["ref_target_lp"].cpu().numpy(), want["ref_target_lp"], "ref lp")
    assert_lp_close(res["cand_target_lp"].cpu().numpy(), want["cand_target_lp"], "cand lp")
    forced = d["forced_rows"].cpu().numpy()
    assert len(forced) > 0 and np.all(ra[forced] != ca[forced])
    kl = res["kl"].cpu().numpy()
    assert np.all(np.isfinite(kl)) and kl.min() >= -1e-5


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_identical_inputs_give_exact_zero(cuda_device, dtype):
    ref, _, tg = ragged(W.SEED_BASE + 300, cuda_device, 64, 100_003, dtype)
    for warps in (0, 1, 3, 64, 1000):
        res = run(ref, same_layout_copy(ref), tg, warps=warps)
        assert torch.all(res["kl"] == 0.0)
        assert torch.equal(res["ref_argmax"], res["cand_argmax"])
        assert torch.equal(res["ref_target_lp"], res["cand_target_lp"])


def test_deterministic(cuda_device):
    d = W.window_full_vocab(seed=W.SEED_BASE + 400, device=cuda_device, n_rows=300, vocab=W.VOCAB)
    outs = [run(d["ref"], d["cand"], d["targets"]) for _ in range(3)]
    for o in outs[1:]:
        for k in ("kl", "ref_argmax", "cand_argmax", "ref_target_lp", "cand_target_lp"):
            assert torch.equal(o[k], outs[0][k]), k
    # other splits give the same argmaxes and KLs within the contract
    other = run(d["ref"], d["cand"], d["targets"], warps=333)
    assert torch.equal(other["ref_argmax"], outs[0]["ref_argmax"])
    assert torch.allclose(other["kl"], outs[0]["kl"], rtol=1e-4, atol=1e-6)


def test_many_pieces_per_row(cuda_device):
    """Few rows, many warps: a row spans more than 32 pieces (chunked merge)."""
    d = W.window_full_vocab(seed=W.SEED_BASE + 450, device=cuda_device, n_rows=3, vocab=W.VOCAB)
    res = run(d["ref"], d["cand"], d["targets"], warps=150)
    check_full_vocab(res, to_f64(d["ref"]), to_f64(d["cand"]), d["targets"].cpu().numpy())


def test_closed_forms_on_gpu(cuda_device):
    V = 248_320
    # one-hot vs uniform: KL = ln V
    x = torch.full((2, V), -math.inf, device=cuda_device)
    x[0, 12345] = 0.0
    x[1, V - 1] = 3.0
    y = torch.zeros((2, V), device=cuda_device)
    t = torch.tensor([12345, 5], dtype=torch.int32, device=cuda_device)
    res = run(x, y, t)
    assert abs(res["kl"][0].item() - math.log(V)) <= 1e-5 + 1e-3 * math.log(V)
    assert res["ref_argmax"].tolist() == [12345, V - 1]
    assert res["cand_argmax"].tolist() == [0, 0]
    assert res["ref_target_lp"][0].item() == 0.0
    assert math.isinf(res["ref_target_lp"][1].item())      # p_t = 0 exactly
    assert abs(res["cand_target_lp"][0].item() + math.log(V)) <= 1e-5 * math.log(V)
    # ties: lowest index wins
    x = torch.zeros((1, 1000), device=cuda_device)
    x[0, [17, 400, 999]] = 5.0
    res = run(x, x.flip(1).contiguous())
    assert res["ref_argmax"].item() == 17 and res["cand_argmax"].item() == 0


def test_non_finite_rows(cuda_device):
    V = 5000
    rng = np.random.default_rng(3)
    X = rng.normal(0, 2, (8, V)).astype(np.float32)
    Y = (X + rng.normal(0, 0.1, (8, V))).astype(np.float32)
    X[0, 17] = np.nan                       # NaN in the reference
    Y[1, 4000] = np.nan                     # NaN in the candidate
    X[2, 5] = np.inf                        # +inf
    X[3, :] = -np.inf                       # no finite reference logit
    X[4, :2500] = -np.inf                   # masked reference ids
    Y[4, :100] = -np.inf                    # ... also masked in the candidate
    Y[5, int(np.argmax(X[5]))] = -np.inf    # candidate gives zero mass to the top id
    X[6, :4990] = -np.inf                   # leading -inf run in every thread's first chunk
    Y[6, :4990] = -np.inf
    ref = torch.tensor(X, device=cuda_device)
    cand = torch.tensor(Y, device=cuda_device)
    tg = torch.tensor([0, 1, 2, 3, 4000, 6, 4995, -1], dtype=torch.int32, device=cuda_device)
    res = run(ref, cand, tg)
    assert res["status"] & 0x1                              # target -1 reported
    want = O.full_vocab(X.astype(np.float64), Y.astype(np.float64), None)
    assert_kl_close(res["kl"].cpu().numpy(), want["kl"])
    assert np.array_equal(res["ref_argmax"].cpu().numpy(), want["ref_argmax"])
    assert np.array_equal(res["cand_argmax"].cpu().numpy(), want["cand_argmax"])
    assert math.isnan(res["ref_target_lp"][7].item())
    for r in (0, 1, 2, 3):
        assert res["ref_argmax"][r].item() == -1 and math.isnan(res["kl"][r].item())
    assert res["kl"][5].item() == math.inf


def test_bad_target_reported(cuda_device):
    d = W.window_full_vocab(seed=W.SEED_BASE + 500, device=cuda_device, n_rows=4, vocab=1000)
    tg = torch.tensor([0, 999, 1000, -5], dtype=torch.int32, device=cuda_device)
    res = run(d["ref"], d["cand"], tg)
    assert res["status"] == 0x1
    lp = res["ref_target_lp"].cpu().numpy()
    assert np.isfinite(lp[:2]).all() and np.isnan(lp[2:]).all()
    assert torch.isfinite(res["kl"]).all()


def test_near_certain_target_relative_error(cuda_device):
    """A near-certain token: log p_t ~ -1e-6 must still be within 1e-5 relative."""
    V = 248_320
    rng = np.random.default_rng(5)
    X = rng.normal(-30, 1, (4, V)).astype(np.float32)
    X[:, 99] = 0.0
    Y = (X + rng.normal(0, 0.01, (4, V))).astype(np.float32)
    ref = torch.tensor(X, device=cuda_device)
    cand = torch.tensor(Y, device=cuda_device)
    tg = torch.full((4,), 99, dtype=torch.int32, device=cuda_device)
    res = run(ref, cand, tg)
    want = O.full_vocab(X.astype(np.float64), Y.astype(np.float64), np.full(4, 99))
    assert np.all(np.abs(want["ref_target_lp"]) < 1e-4)
    assert_lp_close(res["ref_target_lp"].cpu().numpy(), want["ref_target_lp"])
    assert_lp_close(res["cand_target_lp"].cpu().numpy(), want["cand_target_lp"])
    assert_kl_close(res["kl"].cpu().numpy(), want["kl"])


def test_empty_batch(cuda_device):
    ref = torch.empty((0, 100), device=cuda_device)
    res = kq.kld_full_vocab(ref, ref.clone())
    assert res["kl"].numel() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_logits_near_the_largest_finite_values(cuda_device, dtype):
    """Rows whose maximum is large: near the largest finite value (where
    x log2 e overflows f32), around 2^20 (where the one-FMA exponent gives
    way to (x - m) log2 e) and past 2^31 (where it could not work at all):
    ties at the maximum, values just below it, the rest far below, both
    signs, the candidate's maximum equal to or above the reference's.  Every
    id's difference x_i - y_i, and every x_i - m, stays finite in f32, as the
    kernel's domain requires."""
    V = 5000
    rng = np.random.default_rng(123)
    # (reference maximum, candidate maximum, fill value)
    cases = [(3.0e38, 3.0e38, 1.0e37), (-3.0e38, -3.0e38, -3.3e38), (3.0e38, 3.2e38, 1.0e37),
             (1.0e38, 1.0e38, -1.0e38), (-1.0e38, -1.0e38, -2.0e38), (8.4e37, 8.4e37, -8.0e37),
             (-8.4e37, -8.0e37, -1.0e38), (1.0e9, 1.0e9, -1.0e9), (-3.0e9, -3.0e9 + 512, -3.1e9),
             (1.0e6, 1.0e6 + 2.0, 1.0e6 - 40.0), (1.048e6, 1.048e6, 1.0e6), (3.0e6, 3.0e6, 2.9e6),
             (-1.0e6, -1.0e6, -1.0e6 - 30.0)]
    rows_x, rows_y, tgs = [], [], []
    for i, (bx, by, fill) in enumerate(cases):
        x = np.full(V, fill, dtype=np.float64)
        some = rng.choice(V, 150, replace=False)
        x[some[:100]] = rng.uniform(fill, fill + 0.5 * (bx - fill), 100)
        x[some[100:]] = bx - rng.uniform(0.0, 12.0, 50)   # just below the maximum (ties where it is coarse)
        y = x.copy()
        tx = rng.choice(V, 3, replace=False)
        x[tx] = bx
        y[tx] = bx                            # x's maxima are in y too ...
        ty = rng.choice(V, 2, replace=False)
        y[ty] = by                            # ... with ties (or a larger maximum) of its own
        rows_x.append(x)
        rows_y.append(y)
        tgs.append(int(tx[0]) if i % 2 == 0 else int(rng.integers(0, V)))
    X = torch.tensor(np.array(rows_x), dtype=torch.float32).to(dtype).to(cuda_device)
    Y = torch.tensor(np.array(rows_y), dtype=torch.float32).to(dtype).to(cuda_device)
    tg = torch.tensor(tgs, dtype=torch.int32, device=cuda_device)
    res = run(X, Y, tg)
    assert res["status"] == 0
    want = check_full_vocab(res, to_f64(X), to_f64(Y), tg.cpu().numpy())
    assert np.isfinite(want["kl"]).all()
