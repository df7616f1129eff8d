"""k-way tensor-parallel decoding, one rank at a time on one GPU.

Under k-way tensor parallelism of an MLRA-k layer, rank j holds the cache columns of block j
plus the shared RoPE key, the up-projections of head group j and that group's query heads, and
runs plain latent attention (k = 1) over its shard; the head groups' outputs are then
concatenated ("Multi-Head Low-Rank Attention: Making Compressed Attention Actually
Parallelizable", *Core Mechanism*: each device loads only its latent head's cache and the
results get combined). Here the k ranks' decodes run one after another through the C ABI on
the same GPU, each on its own shard, and the concatenated heads must match the oracle's MLRA-k
result for the whole layer. The ranks share nothing and never wait on one another.
"""
import pytest
import torch

import rank_latent_kv_mlra_b200 as M
import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

CASES = {
    "mlra4_tp4": W.scaled(W.WORKLOADS["mlra4_h128_b32_n8192"], batch=3, seq_len=None, len_range=(1, 1500),
                          seed=41),
    "mlra2_tp2": W.scaled(W.WORKLOADS["mlra2_h128_b64_n4096"], batch=3, seq_len=None, len_range=(100, 1300),
                          seed=42),
}


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    M.load_library()


@pytest.mark.parametrize("name", list(CASES))
def test_rank_shards_concatenate_to_the_layer_output(name):
    """Each rank's shard is cut by the library's tp helpers and decoded by tp.RankDecode."""
    from rank_latent_kv_mlra_b200 import tp
    w = CASES[name]
    inp = W.make_workload(w, device="cuda")
    outs, lses = [], []
    for j in range(w.k):
        rank = tp.RankDecode(j, w.k, w.h, w.d_h, w.d_c, w.d_r, inp["w_uk"], inp["w_uv"])
        pool_j = tp.shard_pool(inp["pool"], j, w.k, w.d_c)
        q_j = tp.shard_heads(inp["q"], j, w.k, 1)
        out = torch.full((w.batch, w.h // w.k, w.d_h), float("nan"), device="cuda")
        lse = torch.full((w.batch, w.h // w.k), float("nan"), device="cuda")
        ws = rank.decode(q_j, pool_j, inp["page_table"], inp["seq_lens"], out, lse)
        torch.cuda.synchronize()
        assert M.mlra_get_status(ws) == 0
        outs.append(out)
        lses.append(lse)
        del rank
    out = torch.cat(outs, dim=1).cpu().numpy()
    lse = torch.cat(lses, dim=1).cpu().numpy()
    ref = G.oracle_full(w, inp)
    G.assert_parity(out, ref["out"], f"{name}: concatenated rank outputs")
    live = ref["lse"] > -1e300
    assert abs(lse[live] - ref["lse"][live]).max() < G.TOL_LSE_ABS
