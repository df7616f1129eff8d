"""k-way tensor parallelism across processes, on CPU with the gloo backend (k = 2 and 4).

Each rank cuts its shard out of the full layer with the library's tp helpers (block j's cache
columns plus the RoPE key, head group j's queries and up-projections), computes its heads on
the shard, and the ranks all-gather their outputs with tp.gather_heads. On CPU the per-rank
attention is the float64 oracle (the kernels need a B200); what is under test is the sharding,
the choice of head group, the softmax scale a rank must use, and the order of the gather. Rank
0 checks the assembled heads against the oracle's result for the whole MLRA-k layer.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import workloads as W
        from oracle import mlra_oracle as O
        from rank_latent_kv_mlra_b200 import tp
        base = W.WORKLOADS["mlra4_h128_b32_n8192" if world == 4 else "mlra2_h128_b64_n4096"]
        w = W.scaled(base, batch=3, seq_len=None, len_range=(1, 400), h=16, seed=90 + world)
        inp = W.make_workload(w, device="cpu")
        # rank j's shard, cut by the library's helpers
        pool_j = tp.shard_pool(inp["pool"], rank, world, w.d_c)
        q_j = tp.shard_heads(inp["q"], rank, world, 1)
        wuk_j = tp.shard_heads(inp["w_uk"], rank, world, 0)
        wuv_j = tp.shard_heads(inp["w_uv"], rank, world, 0)
        # the rank's heads: plain latent attention (k = 1) with the layer's softmax scale
        res = O.decode(q_j.double().numpy(), wuk_j.double().numpy(), wuv_j.double().numpy(),
                       pool_j.float().numpy(), inp["page_table"].numpy(), inp["seq_lens"].numpy(), 1, w.d_r,
                       scale=O.default_scale(w.d_h, w.d_r))
        full = tp.gather_heads(torch.from_numpy(res["out"]))
        if rank == 0:
            ref = O.decode(inp["q"].double().numpy(), inp["w_uk"].double().numpy(), inp["w_uv"].double().numpy(),
                           inp["pool"].float().numpy(), inp["page_table"].numpy(), inp["seq_lens"].numpy(), w.k,
                           w.d_r)
            out["max_abs"] = float(np.abs(full.numpy() - ref["out"]).max())
            out["shape"] = tuple(full.shape)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_tensor_parallel_ranks_gather_the_layer(world):
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out["shape"][1] == 16
    assert out["max_abs"] < 1e-12, out["max_abs"]
