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


def rank_shard(w, inp, j):
    """Rank j's inputs: cache columns [c_j | k^R] (a page pool of its own), the head group's
    query rows and up-projections. Test-side data layout only."""
    d_b, hb = w.d_c // w.k, w.h // w.k
    pool = torch.cat([inp["pool"][..., j * d_b:(j + 1) * d_b], inp["pool"][..., w.d_c:]], dim=-1).contiguous()
    return {
        "pool": pool,
        "page_table": inp["page_table"],
        "seq_lens": inp["seq_lens"],
        "q": inp["q"][:, j * hb:(j + 1) * hb].contiguous(),
        "w_uk": inp["w_uk"][j * hb:(j + 1) * hb].contiguous(),
        "w_uv": inp["w_uv"][j * hb:(j + 1) * hb].contiguous(),
    }


@pytest.mark.parametrize("name", list(CASES))
def test_rank_shards_concatenate_to_the_layer_output(name):
    w = CASES[name]
    inp = W.make_workload(w, device="cuda")
    d_b, hb = w.d_c // w.k, w.h // w.k
    outs, lses = [], []
    for j in range(w.k):
        sh = rank_shard(w, inp, j)
        hdl = M.mlra_create(hb, w.d_h, d_b, w.d_r, 1, sh["w_uk"], sh["w_uv"],
                            softmax_scale=1.0 / (w.d_h + w.d_r) ** 0.5)
        out, lse, ws = G.run_decode(hdl, sh)
        assert M.mlra_get_status(ws) == 0
        outs.append(out)
        lses.append(lse)
        del hdl
    out = torch.cat(outs, dim=1).cpu().numpy()
    lse = torch.cat(lses, dim=1).cpu().numpy()
    ref = G.oracle_full(w, inp)
    G.assert_parity(out, ref["out"], f"{name}: concatenated rank outputs")
    live = ref["lse"] > -1e300
    assert abs(lse[live] - ref["lse"][live]).max() < G.TOL_LSE_ABS
