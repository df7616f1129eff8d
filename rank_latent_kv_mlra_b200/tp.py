"""k-way tensor-parallel decoding of an MLRA-k layer across k processes (one GPU each).

Under tensor parallelism each device of an MLRA-k layer holds one latent block of the cache
plus the shared RoPE key, serves that block's head group with its own up-projections, and the
head groups' outputs are then combined ("Multi-Head Low-Rank Attention: Making Compressed
Attention Actually Parallelizable", Core Mechanism; "Multi-Head Low-Rank Attention", abstract:
4-way tensor parallelism). Rank j's share of the work is plain latent attention (k = 1) over
[c_j | k^R] with h/k heads, which the library runs as it is; the exchange is one all-gather of
the ranks' [batch][h/k][d_h] outputs, concatenated in group order.

This module only moves data: it cuts the full layer's tensors into rank shards (device-side
indexing), creates rank j's handle, and gathers head outputs over a torch.distributed process
group (NCCL over NVLink on GPUs). Every step of the attention itself runs in the library's
kernels (rank_latent_kv_mlra_b200.mlra_decode).
"""
from __future__ import annotations

import math

import torch

from . import mlra_create, mlra_decode


def shard_pool(pool: torch.Tensor, j: int, k: int, d_c: int) -> torch.Tensor:
    """Rank j's cache: columns [c_j | k^R] of every cached row, [pages][page_size][d_c/k + d_r]."""
    d_b = d_c // k
    return torch.cat([pool[..., j * d_b:(j + 1) * d_b], pool[..., d_c:]], dim=-1).contiguous()


def shard_heads(t: torch.Tensor, j: int, k: int, dim: int) -> torch.Tensor:
    """Rank j's slice of a per-head tensor along `dim` (head group j: heads [j*h/k, (j+1)*h/k))."""
    hb = t.shape[dim] // k
    return t.narrow(dim, j * hb, hb).contiguous()


def shard_rows(rows: torch.Tensor, j: int, k: int, d_c: int) -> torch.Tensor:
    """Rank j's part of new cache rows [n][d_c + d_r] (for appending): [c_j | k^R]."""
    return shard_pool(rows, j, k, d_c)


class RankDecode:
    """Rank j's decode under k-way tensor parallelism: a k = 1 handle over [c_j | k^R] with the
    layer's h/k heads of group j. The softmax scale is the layer's (1/sqrt(d_h + d_r) unless
    given), not the one a k = 1 handle of width d_c/k would pick."""

    def __init__(self, j: int, k: int, h: int, d_h: int, d_c: int, d_r: int, w_uk: torch.Tensor,
                 w_uv: torch.Tensor, softmax_scale: float = 0.0):
        self.j, self.k, self.h, self.d_h, self.d_c, self.d_r = j, k, h, d_h, d_c, d_r
        scale = softmax_scale if softmax_scale > 0 else 1.0 / math.sqrt(d_h + d_r)
        self.w_uk = shard_heads(w_uk, j, k, 0)
        self.w_uv = shard_heads(w_uv, j, k, 0)
        self.handle = mlra_create(h // k, d_h, d_c // k, d_r, 1, self.w_uk, self.w_uv, softmax_scale=scale)

    def decode(self, q_local, pool_shard, page_table, seq_lens, out_local, lse=None, workspace=None,
               stream=None):
        """q_local [batch][h/k][d_h + d_r] (group j's query rows), pool_shard from shard_pool."""
        return mlra_decode(self.handle, q_local, pool_shard, page_table, seq_lens, out_local, lse,
                           workspace=workspace, stream=stream)


def gather_heads(out_local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of every rank's [batch][h/k][d_h] output into the layer's [batch][h][d_h],
    head groups in rank order (rank j = group j)."""
    import torch.distributed as dist
    k = dist.get_world_size(group)
    B, hb, d = out_local.shape
    parts = torch.empty((k * B, hb, d), dtype=out_local.dtype, device=out_local.device)
    dist.all_gather_into_tensor(parts, out_local.contiguous(), group=group)  # rank-major along dim 0
    return parts.view(k, B, hb, d).permute(1, 0, 2, 3).reshape(B, k * hb, d)
