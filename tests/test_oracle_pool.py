"""The process-pool driver of the full-size GPU tests (``tests/oracle_pool.py``) returns what
the oracle's whole-batch functions return, on CPU inputs (no GPU needed)."""
import numpy as np

import workloads as W
from oracle import mlra_oracle as O
from tests import oracle_pool


def _args(inp):
    return (inp["q"].double().numpy(), inp["w_uk"].double().numpy(), inp["w_uv"].double().numpy(),
            inp["pool"].float().numpy(), inp["page_table"].numpy(), inp["seq_lens"].numpy())


def test_pool_matches_whole_batch_oracle():
    w = W.scaled(W.WORKLOADS["mlra4_h128_b128_ragged1k_32k"], batch=5, len_range=(0, 700), h=16, seed=3)
    inp = W.make_workload(w, device="cpu")
    inp["seq_lens"][1] = 0
    out, lse = oracle_pool.oracle_workload(w, inp, workers=2)
    ref = O.decode(*_args(inp), w.k, w.d_r)
    np.testing.assert_allclose(out, ref["out"], rtol=1e-10, atol=1e-12)
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref["lse"]))
    live = np.isfinite(ref["lse"])
    np.testing.assert_allclose(lse[live], ref["lse"][live], rtol=1e-12)


def test_pool_matches_whole_batch_oracle_summed():
    w = W.scaled(W.WORKLOADS["mlra2sum_h128_b64_n4096"], batch=3, seq_len=None, len_range=(1, 300), h=8, seed=4)
    inp = W.make_workload(w, device="cpu")
    out, lse = oracle_pool.oracle_workload(w, inp, workers=2)
    ref = O.decode_summed(*_args(inp), w.k, w.d_r)
    np.testing.assert_allclose(out, ref["out"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref["lse"], rtol=1e-12)
