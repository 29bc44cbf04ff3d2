"""The oracle's process pool gives exactly the results of calling the oracle
directly (it only stages inputs and hands out row ranges)."""
import numpy as np
import torch

from oracle import kld_oracle as O
from oracle.pool import OraclePool


def test_pool_matches_direct_calls():
    rng = np.random.default_rng(0)
    n, V = 37, 3000
    x = torch.randn(n, V).mul(2).to(torch.bfloat16)
    y = (x.float() + 0.05 * torch.randn(n, V)).to(torch.bfloat16)
    t = torch.as_tensor(rng.integers(0, V, n).astype(np.int32))
    xf = rng.normal(0, 1, (n, V)).astype(np.float32)
    bits = lambda a: a.view(torch.int16).numpy().view(np.uint16)
    with OraclePool(cores=3) as pool:
        st = {"X": pool.stage("x", x, "bf16"), "Y": pool.stage("y", y, "bf16"), "targets": pool.stage("t", t, "int")}
        got = pool.run("full_vocab", st, n, rows_per_job=5)
        part = pool.run("full_vocab", st, 11, rows_per_job=4, start=20)
        cap = pool.run("sparse_capture", {"X": pool.stage("xf", xf, "f32")}, n, k=9)
    want = O.full_vocab(O.bf16_bits_to_f64(bits(x)), O.bf16_bits_to_f64(bits(y)), t.numpy())
    for k in want:
        assert np.array_equal(got[k], want[k], equal_nan=True), k
        assert np.array_equal(part[k], want[k][20:31], equal_nan=True), k
    wc = O.sparse_capture(xf.astype(np.float64), 9)
    for k in wc:
        assert np.array_equal(cap[k], wc[k], equal_nan=True), k
