"""Float64 CPU oracle for the step before the decode path: one new token's cache row.

TEST INFRASTRUCTURE ONLY. Only ``tests/`` and the CPU-baseline leg of ``bench.py`` may import
this module. The CUDA library never calls it and shares no code with it.

What it computes (plain definitions, float64):

* the latent of the new token, all k blocks at once: ``c = x W^DKV`` (the down-projection of
  the token's hidden state; lesty.tech MLA article, section 4, and "Multi-Head Low-Rank
  Attention: Making Compressed Attention Actually Parallelizable", Core Mechanism: the input is
  projected into the latent representations, one block per latent head);
* its decoupled RoPE key: ``k^R = RoPE_pos(x W^KR)`` (lesty.tech section 4: the positional key
  is derived from the hidden state and rotated), shared by every head;
* the row ``[c | k^R]`` is stored in slot ``pos % 64`` of page ``page_table[b][pos // 64]``, the
  same addressing the decode oracle reads (``mlra_oracle.gather_rows``).

The weights are stored ``w_down[r][d]`` with one row per output feature (latent features
first, then the RoPE key features), so ``y[r] = sum_d w_down[r][d] x[d]``.

Readings where the pages are silent: the rotation follows RoFormer (the
pages cite it; its Section 3.4): feature pairs ``(2i, 2i+1)`` of the RoPE key are rotated by
the angle ``pos * theta_i`` with ``theta_i = base^(-2i / d_r)``, base 10000 unless given, i.e.
the pair read as the complex number ``v[2i] + 1j * v[2i+1]`` is multiplied by
``exp(1j * pos * theta_i)``. The position is the token's index in its sequence (0-based).

Parity status: every function is pinned by ``tests/test_oracle_producer.py``.
"""
from __future__ import annotations

import numpy as np

PAGE_SIZE = 64
ROPE_BASE = 10000.0


def rope_frequencies(d_r: int, base: float = ROPE_BASE) -> np.ndarray:
    """theta_i = base^(-2i/d_r) for the d_r/2 feature pairs."""
    i = np.arange(d_r // 2, dtype=np.float64)
    return base ** (-2.0 * i / d_r)


def rope(v, pos, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate each feature pair (2i, 2i+1) of ``v`` (last axis, even width) by pos * theta_i."""
    v = np.asarray(v, dtype=np.float64)
    ang = float(pos) * rope_frequencies(v.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = v[..., 0::2], v[..., 1::2]
    out = np.empty_like(v)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def project_row(x_b, w_down, d_c: int, d_r: int, pos, base: float = ROPE_BASE) -> np.ndarray:
    """The cache row [c | k^R] of one token with hidden state x_b at position pos."""
    y = np.asarray(w_down, dtype=np.float64) @ np.asarray(x_b, dtype=np.float64)
    assert y.shape[0] == d_c + d_r
    y[d_c:] = rope(y[d_c:], pos, base)
    return y


def project_append(x, w_down, d_c: int, d_r: int, positions, page_table, base: float = ROPE_BASE):
    """Rows for a batch of new tokens and where each goes: (rows [B][d_c + d_r], pages [B],
    slots [B])."""
    x = np.asarray(x, dtype=np.float64)
    rows = np.stack([project_row(x[b], w_down, d_c, d_r, positions[b], base) for b in range(x.shape[0])])
    pages = np.array([page_table[b][int(positions[b]) // PAGE_SIZE] for b in range(x.shape[0])])
    slots = np.array([int(positions[b]) % PAGE_SIZE for b in range(x.shape[0])])
    return rows, pages, slots


def bytes_per_step(batch: int, d_model: int, d_c: int, d_r: int) -> int:
    """Algorithmic bytes: the bf16 weights and hidden states read once, the bf16 rows written,
    one position and one page-table entry read per token."""
    d_out = d_c + d_r
    return 2 * d_out * d_model + 2 * batch * d_model + 2 * batch * d_out + 8 * batch
