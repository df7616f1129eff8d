"""Seeded synthetic workloads for MLRA decode attention over a paged latent cache.

This module only draws inputs. It holds none of the attention arithmetic, so both the
float64 oracle (``oracle/``) and the CUDA path can be fed from it without sharing any of
the method's code.

What a workload holds (all tensors on the requested device):

* ``seq_lens``   int32 [B]: context length n_b of each sequence.
* ``page_table`` int32 [B][max_pages]: logical page i of sequence b -> physical page id.
  Entries past a sequence's last page are -1.
* ``pool``       bf16 [num_pages][64][d_c + d_r] (uint8 E4M3 bytes for an ``e4m3`` cache,
  each meaning ``E4M3_SCALE * e4m3(byte)``): the paged latent cache. Row layout per
  token is ``[c_1 | ... | c_k | k^R]`` (k latent blocks of d_c/k, then the decoupled RoPE
  key). Slots past n_b in a sequence's last page hold NaN, so a kernel that lets unused
  slots leak into its result fails loudly.
* ``q``          [B][h][d_h + d_r]: per-head query, content part q^C then RoPE part q^R
  (already rotated). fp32 for the tiny workload, bf16 otherwise.
* ``w_uk``, ``w_uv`` bf16 [h][d_c/k][d_h]: per-head up-projections, stored the way the
  ai360xpert "Multi-Head Latent Attention" page stores them ((H, d_c, d_head), "Show Me
  the Code"), restricted to the head's latent block.

Distributions (the pages fix none of them for decode):
cache rows and queries N(0,1), weights N(0,1)/sqrt(fan_in) with fan_in = d_c/k (the input
width of the c -> K/V map). The tiny workload also scales activations by 1/sqrt(width).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

PAGE_SIZE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    k: int                 # latent blocks (1 = plain MLA)
    h: int                 # query heads
    d_h: int               # head dim
    d_c: int               # latent width (all blocks)
    d_r: int               # decoupled RoPE key width
    batch: int
    seq_len: Optional[int] = None          # fixed context length
    len_range: Optional[tuple] = None      # (lo, hi) inclusive, uniform integers
    seed: int = 0
    paging: str = "permuted"               # "permuted" | "contiguous"
    tiny_scaling: bool = False             # activations / sqrt(width)
    q_dtype: str = "bf16"                  # "bf16" | "f32"
    summed: bool = False                   # every head attends to every block; outputs summed
    cache: str = "bf16"                    # "bf16" | "e4m3" (one byte per cached element)

    @property
    def d_b(self) -> int:
        return self.d_c // self.k


# The five decode workloads: names say what they are and their sizes.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("mlra4_h8_b1_n256_f32", k=4, h=8, d_h=32, d_c=128, d_r=16, batch=1,
                 seq_len=256, seed=0, paging="contiguous", tiny_scaling=True, q_dtype="f32"),
        Workload("mlra4_h128_b32_n8192", k=4, h=128, d_h=128, d_c=512, d_r=64, batch=32,
                 seq_len=8192, seed=1),
        Workload("mlra2_h128_b64_n4096", k=2, h=128, d_h=128, d_c=512, d_r=64, batch=64,
                 seq_len=4096, seed=2),
        Workload("mlra4_h128_b8_n131072", k=4, h=128, d_h=128, d_c=512, d_r=64, batch=8,
                 seq_len=131072, seed=3),
        Workload("mlra4_h128_b128_ragged1k_32k", k=4, h=128, d_h=128, d_c=512, d_r=64,
                 batch=128, len_range=(1024, 32768), seed=4),
        Workload("mla_h128_b128_ragged1k_32k", k=1, h=128, d_h=128, d_c=512, d_r=64,
                 batch=128, len_range=(1024, 32768), seed=4),
        # the summed-blocks reading of MLRA-4 on the h=128, batch-32, context-8192 shapes
        Workload("mlra4sum_h128_b32_n8192", k=4, h=128, d_h=128, d_c=512, d_r=64, batch=32,
                 seq_len=8192, seed=5, summed=True),
        # the summed-blocks reading of MLRA-2 (two blocks of 256, all 128 heads on each) on
        # the batch-64, context-4096 shapes
        Workload("mlra2sum_h128_b64_n4096", k=2, h=128, d_h=128, d_c=512, d_r=64, batch=64,
                 seq_len=4096, seed=7, summed=True),
        # the headline shapes over an E4M3 cache (latent and RoPE columns scaled by 2^-5)
        Workload("mlra4fp8_h128_b32_n8192", k=4, h=128, d_h=128, d_c=512, d_r=64, batch=32,
                 seq_len=8192, seed=8, cache="e4m3"),
        # One rank's share under 4-way tensor parallelism of the model above (h = 128,
        # d_c = 512, d_r = 64): an MLRA-4 rank holds one block plus the RoPE key and its 32
        # heads; an MLA rank holds the whole latent and 32 heads. Batch 64 keeps either cache
        # larger than L2.
        Workload("tp4rank_mlra4_h32_b64_n8192", k=1, h=32, d_h=128, d_c=128, d_r=64, batch=64,
                 seq_len=8192, seed=6),
        Workload("tp4rank_mla_h32_b64_n8192", k=1, h=32, d_h=128, d_c=512, d_r=64, batch=64,
                 seq_len=8192, seed=6),
    ]
}

HEADLINE = "mlra4_h128_b32_n8192"

# Scales of the E4M3 workloads' caches: a cached byte e means E4M3_SCALE * e4m3(e). With N(0,1)
# values the largest magnitude in a 2.5 GB cache stays far below 448 * 2^-5 = 14.
E4M3_SCALE = 2.0 ** -5


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller batches / contexts for tests)."""
    return dataclasses.replace(w, **changes)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def draw_seq_lens(w: Workload, device="cpu") -> torch.Tensor:
    if w.seq_len is not None:
        return torch.full((w.batch,), w.seq_len, dtype=torch.int32, device=device)
    lo, hi = w.len_range
    g = _gen("cpu", w.seed * 7919 + 13)
    lens = torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int64)
    return lens.to(torch.int32).to(device)


def make_page_table(seq_lens: torch.Tensor, paging: str, seed: int, device="cpu",
                    extra_pages: int = 0):
    """Assign physical pages to every (sequence, logical page).

    Returns (page_table int32 [B][max_pages] with -1 padding, num_pages).
    ``extra_pages`` appends never-referenced pages to the pool (they hold NaN).
    """
    lens = seq_lens.to("cpu", torch.int64)
    pages_per_seq = (lens + PAGE_SIZE - 1) // PAGE_SIZE
    used = int(pages_per_seq.sum())
    num_pages = used + extra_pages
    max_pages = max(1, int(pages_per_seq.max()) if len(lens) else 1)
    if paging == "contiguous":
        phys = torch.arange(used, dtype=torch.int64)
    elif paging == "permuted":
        phys = torch.randperm(num_pages, generator=_gen("cpu", seed * 104729 + 7))[:used]
    else:
        raise ValueError(paging)
    table = torch.full((len(lens), max_pages), -1, dtype=torch.int32)
    off = 0
    for b, p in enumerate(pages_per_seq.tolist()):
        table[b, :p] = phys[off:off + p].to(torch.int32)
        off += p
    return table.to(device), num_pages


def make_workload(w: Workload, device="cpu", seq_lens: Optional[torch.Tensor] = None,
                  extra_pages: int = 0, keep_f32: bool = False) -> dict:
    """Draw every input of workload ``w`` on ``device`` from its seed.

    The same (workload, device) always gives the same tensors. CPU and CUDA draws differ
    (different generators); a test feeds one draw to both sides.
    """
    if seq_lens is None:
        seq_lens = draw_seq_lens(w, device)
    seq_lens = seq_lens.to(device=device, dtype=torch.int32)
    page_table, num_pages = make_page_table(seq_lens, w.paging, w.seed, device, extra_pages)
    g = _gen(device, w.seed)
    D = w.d_c + w.d_r
    d_b = w.d_b

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=torch.float32)

    c_scale = 1.0 / math.sqrt(d_b) if w.tiny_scaling else 1.0
    r_scale = 1.0 / math.sqrt(w.d_r) if w.tiny_scaling else 1.0
    pool32 = randn(max(num_pages, 1), PAGE_SIZE, D)
    pool32[..., :w.d_c] *= c_scale
    pool32[..., w.d_c:] *= r_scale
    # Unused slots of each sequence's last page (and never-referenced pages) hold NaN.
    lens_cpu = seq_lens.to("cpu", torch.int64)
    pt_cpu = page_table.to("cpu")
    referenced = torch.zeros(max(num_pages, 1), dtype=torch.bool)
    for b, n in enumerate(lens_cpu.tolist()):
        p = (n + PAGE_SIZE - 1) // PAGE_SIZE
        if p:
            referenced[pt_cpu[b, :p].long()] = True
            tail = n - (p - 1) * PAGE_SIZE
            if tail < PAGE_SIZE:
                pool32[int(pt_cpu[b, p - 1]), tail:, :] = float("nan")
    pool32[~referenced.to(device)] = float("nan")

    qc_scale = 1.0 / math.sqrt(w.d_h) if w.tiny_scaling else 1.0
    qr_scale = 1.0 / math.sqrt(w.d_r) if w.tiny_scaling else 1.0
    q32 = randn(w.batch, w.h, w.d_h + w.d_r)
    q32[..., :w.d_h] *= qc_scale
    q32[..., w.d_h:] *= qr_scale
    w_scale = 1.0 / math.sqrt(d_b)
    # [h][d_b][d_h], or [k][h][d_b][d_h] (one pair of matrices per block and head) when summed
    wshape = (w.k, w.h, d_b, w.d_h) if w.summed else (w.h, d_b, w.d_h)
    w_uk32 = randn(*wshape) * w_scale
    w_uv32 = randn(*wshape) * w_scale

    if w.cache == "e4m3":
        # stored bytes: nearest E4M3 value of v / scale (torch's float8_e4m3fn conversion; no
        # value reaches its range limit at this scale); NaN slots stay NaN (0x7F)
        pool = (pool32 / E4M3_SCALE).to(torch.float8_e4m3fn).view(torch.uint8)
    else:
        pool = pool32.to(torch.bfloat16)
    out = {
        "workload": w,
        "seq_lens": seq_lens,
        "page_table": page_table,
        "num_pages": num_pages,
        "pool": pool,
        "q": q32 if w.q_dtype == "f32" else q32.to(torch.bfloat16),
        "w_uk": w_uk32.to(torch.bfloat16),
        "w_uv": w_uv32.to(torch.bfloat16),
    }
    if keep_f32:
        out.update(pool_f32=pool32, q_f32=q32, w_uk_f32=w_uk32, w_uv_f32=w_uv32)
    else:
        del pool32
    return out


def logical_rows(inputs: dict, b: int) -> torch.Tensor:
    """Rows [n_b][d_c + d_r] of sequence b, gathered through the page table (bf16)."""
    n = int(inputs["seq_lens"][b])
    pt = inputs["page_table"][b].to(torch.int64)
    t = torch.arange(n, device=pt.device)
    return inputs["pool"][pt[t // PAGE_SIZE], t % PAGE_SIZE]


# The step before decoding (each sequence's new cache row) needs the model width, which the
# decode workloads do not fix: DeepSeek-V2's hidden size, matching the h = 128, d_c = 512
# DeepSeek-V2-like attention shapes.
PRODUCER_D_MODEL = 5120


def make_producer_inputs(w: Workload, inputs: dict, d_model: int = PRODUCER_D_MODEL,
                         seed: Optional[int] = None) -> dict:
    """Inputs of the new-row step for workload ``w``'s batch, on the device of ``inputs``:
    hidden states x [batch][d_model] ~ N(0,1) and w_down [d_c + d_r][d_model] ~
    N(0,1)/sqrt(d_model) (fan_in = d_model), both bf16, and one position per sequence drawn
    uniformly from the slots its page-table row covers."""
    device = inputs["pool"].device
    s = (w.seed if seed is None else seed) * 31 + 17
    g = _gen(device, s)
    x = torch.randn(w.batch, d_model, generator=g, device=device).to(torch.bfloat16)
    w_down = (torch.randn(w.d_c + w.d_r, d_model, generator=g, device=device) / math.sqrt(d_model)).to(
        torch.bfloat16)
    cap = (inputs["page_table"] >= 0).sum(dim=1).to("cpu", torch.int64) * PAGE_SIZE
    u = torch.rand(w.batch, generator=_gen("cpu", s + 1), dtype=torch.float64)
    positions = torch.minimum((u * cap).long(), cap - 1).clamp(min=0).to(torch.int32)
    return {"x": x, "w_down": w_down, "positions": positions.to(device), "d_model": d_model}
