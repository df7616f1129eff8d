"""Float64 CPU oracle for MLRA decode attention over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module. The CUDA library never calls it and shares no
code with it.

What it computes (plain definitions, float64, one head at a time):

Multi-Head Low-Rank Attention keeps one latent ``c = [c_1 | ... | c_k]`` per token, cut into k
independent blocks, plus one decoupled RoPE key ``k^R`` shared by all heads. Head group j
(heads ``[j*h/k, (j+1)*h/k)``) attends only to block ``c_j``
("Multi-Head Low-Rank Attention: Making Compressed Attention Actually Parallelizable",
Core Mechanism and Key Concepts: four latent heads, each serving eight of the original heads;
"Multi-Head Low-Rank Attention" abstract: partitionable latent states). k = 1 is plain MLA.

For head h of group j and a context of n tokens:

* explicit form ("Multi-Head Latent Attention", How It Actually Works / The two projections):
  ``K_h[t] = W^UK_h c_j[t]``, ``V_h[t] = W^UV_h c_j[t]``;
* score (lesty.tech MLA article, section 4, decoupled RoPE: content dot plus positional dot):
  ``s_t = scale * (q^C_h . K_h[t] + q^R_h . k^R[t])``;
* ``p = softmax(s)``, ``o_h = sum_t p_t V_h[t]``, ``lse_h = log sum_t exp(s_t)``;
* absorbed form (lesty.tech section 5, "On-The-Fly Matrix Absorption"; ai360xpert "Absorbing
  the up-projection"): ``q~_h = (W^UK_h)^T q^C_h`` scored directly against ``c_j``,
  ``o~_h = sum_t p_t c_j[t]``, then one up-projection ``o_h = W^UV_h o~_h``.

Weights are stored ``[h][d_b][d_h]`` (the ai360xpert code's ``(H, d_c, d_head)`` convention,
restricted to the head's block of width d_b = d_c/k), so ``K_h[t][d] = sum_c c[t][c] W[h][c][d]``.

Readings where the pages are silent:
* softmax scale: ``1/sqrt(d_h + d_r)`` unless given;
* k^R is one vector per token, shared by every head and block, cached already rotated;
* every head has its own q^R_h; RoPE is applied upstream.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py`` (the
summed-blocks functions by ``tests/test_oracle_summed.py``; the per-sequence forms
``decode_sequence`` and ``decode_summed_sequence`` against torch SDPA like the per-head ones)
except ``plan_segments``, whose rule
is not from the pages (they have no split-KV scheme); it is pinned by hand-worked golden
cases and by invariants (coverage, disjointness, quota).
"""
from __future__ import annotations

import math
from typing import List, NamedTuple

import numpy as np

PAGE_SIZE = 64
TILE_TOKENS = 128  # split granularity: two pages


def default_scale(d_h: int, d_r: int) -> float:
    """Softmax scale: 1/sqrt of the un-absorbed per-head key width [k^C_h | k^R]."""
    return 1.0 / math.sqrt(d_h + d_r)


def head_block(head: int, h: int, k: int) -> int:
    """Latent block j that head ``head`` attends to: contiguous groups of h/k heads."""
    return head // (h // k)


def gather_rows(pool: np.ndarray, page_table: np.ndarray, b: int, n: int) -> np.ndarray:
    """Cache rows [n][d_c + d_r] of sequence b: token t lives at page table entry t // 64,
    slot t % 64 (PagedAttention-style paging, as the MLRA index page's bibliography cites)."""
    t = np.arange(n)
    pages = np.asarray(page_table[b])[t // PAGE_SIZE].astype(np.int64)
    return np.asarray(pool[pages, t % PAGE_SIZE], dtype=np.float64)


def _split(rows: np.ndarray, j: int, d_c: int, k: int):
    d_b = d_c // k
    return rows[:, j * d_b:(j + 1) * d_b], rows[:, d_c:]


def _softmax_stats(s: np.ndarray):
    m = s.max()
    e = np.exp(s - m)
    l = e.sum()
    return e / l, m + math.log(l)


def attend_head_explicit(qc, qr, w_uk_h, w_uv_h, c_j, kr, scale):
    """One head, explicit reconstruction. Returns (o_h [d_h], lse)."""
    K = c_j @ w_uk_h                      # [n, d_h]
    V = c_j @ w_uv_h                      # [n, d_h]
    s = scale * (K @ qc + kr @ qr)        # [n]
    p, lse = _softmax_stats(s)
    return p @ V, lse


def attend_head_absorbed(qc, qr, w_uk_h, w_uv_h, c_j, kr, scale):
    """One head, absorbed form. Returns (o_h [d_h], o_latent [d_b], lse)."""
    q_lat = w_uk_h @ qc                   # [d_b] = (W^UK_h)^T q^C_h in the [d_b][d_h] storage
    s = scale * (c_j @ q_lat + kr @ qr)
    p, lse = _softmax_stats(s)
    o_lat = p @ c_j                       # [d_b]
    return o_lat @ w_uv_h, o_lat, lse


def decode(q, w_uk, w_uv, pool, page_table, seq_lens, k, d_r, scale=None, form="absorbed"):
    """Full decode step for every sequence and head.

    q: [B][h][d_h + d_r]; w_uk, w_uv: [h][d_b][d_h]; pool: [pages][64][d_c + d_r];
    page_table: [B][max_pages]; seq_lens: [B].
    Returns dict with ``out`` [B][h][d_h], ``lse`` [B][h] (natural log) and, for the absorbed
    form, ``latent`` [B][h][d_b]. An empty sequence gives out = 0, latent = 0, lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    pool = np.asarray(pool, dtype=np.float64)
    B, h, qw = q.shape
    d_h = qw - d_r
    d_b = w_uk.shape[1]
    d_c = d_b * k
    if scale is None:
        scale = default_scale(d_h, d_r)
    out = np.zeros((B, h, d_h))
    lse = np.full((B, h), -np.inf)
    latent = np.zeros((B, h, d_b))
    for b in range(B):
        n = int(seq_lens[b])
        if n == 0:
            continue
        rows = gather_rows(pool, page_table, b, n)
        for hd in range(h):
            j = head_block(hd, h, k)
            c_j, kr = _split(rows, j, d_c, k)
            qc, qr = q[b, hd, :d_h], q[b, hd, d_h:]
            if form == "explicit":
                out[b, hd], lse[b, hd] = attend_head_explicit(qc, qr, w_uk[hd], w_uv[hd], c_j, kr, scale)
            else:
                out[b, hd], latent[b, hd], lse[b, hd] = attend_head_absorbed(
                    qc, qr, w_uk[hd], w_uv[hd], c_j, kr, scale)
    res = {"out": out, "lse": lse}
    if form != "explicit":
        res["latent"] = latent
    return res


def decode_heads(q, w_uk, w_uv, rows, seq_heads, k, d_r, scale=None):
    """Absorbed-form result for a list of heads of ONE sequence whose rows are given.

    Used for sampled checks at full size: rows [n][d_c + d_r] (float64), seq_heads: head ids.
    Returns (out [len][d_h], latent [len][d_b], lse [len]).
    """
    q = np.asarray(q, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    h = w_uk.shape[0]
    d_b = w_uk.shape[1]
    d_c = d_b * k
    d_h = q.shape[-1] - d_r
    if scale is None:
        scale = default_scale(d_h, d_r)
    outs, lats, lses = [], [], []
    for hd in seq_heads:
        j = head_block(hd, h, k)
        c_j, kr = _split(rows, j, d_c, k)
        o, lat, l = attend_head_absorbed(q[hd, :d_h], q[hd, d_h:], w_uk[hd], w_uv[hd], c_j, kr, scale)
        outs.append(o)
        lats.append(lat)
        lses.append(l)
    return np.array(outs), np.array(lats), np.array(lses)


def decode_sequence(q_b, w_uk, w_uv, rows, k, d_r, scale=None):
    """Absorbed-form result for EVERY head of one sequence whose rows are given, with the
    heads of each latent block stacked so that one matrix product serves them all (used for
    the elementwise checks at full size, where one head at a time would re-read the rows h
    times). Same definitions as ``attend_head_absorbed``; for block j and its heads G_j:

      Q~_j = [(W^UK_h)^T q^C_h]_{h in G_j}                      [|G_j|][d_b]
      S_j  = scale * (c_j Q~_j^T + k^R (Q^R_j)^T)               [n][|G_j|]
      P_j  = softmax of each column of S_j;  lse_h = log sum_t exp(S_j[t][h])
      o~_h = (P_j^T c_j)[h];  o_h = W^UV_h o~_h

    q_b: [h][d_h + d_r]; w_uk, w_uv: [h][d_b][d_h]; rows: [n][d_c + d_r].
    Returns (out [h][d_h], latent [h][d_b], lse [h]); n = 0 gives zeros and -inf."""
    q_b = np.asarray(q_b, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    h, qw = q_b.shape
    d_h = qw - d_r
    d_b = w_uk.shape[1]
    d_c = d_b * k
    if scale is None:
        scale = default_scale(d_h, d_r)
    out = np.zeros((h, d_h))
    latent = np.zeros((h, d_b))
    lse = np.full(h, -np.inf)
    if rows.shape[0] == 0:
        return out, latent, lse
    hb = h // k
    for j in range(k):
        g = slice(j * hb, (j + 1) * hb)
        c_j, kr = _split(rows, j, d_c, k)
        q_lat = np.einsum("hcd,hd->hc", w_uk[g], q_b[g, :d_h])      # [hb][d_b]
        S = scale * (c_j @ q_lat.T + kr @ q_b[g, d_h:].T)          # [n][hb]
        m = S.max(axis=0)
        E = np.exp(S - m)
        l = E.sum(axis=0)
        P = E / l
        lse[g] = m + np.log(l)
        latent[g] = P.T @ c_j                                      # [hb][d_b]
        out[g] = np.einsum("hc,hcd->hd", latent[g], w_uv[g])
    return out, latent, lse


def decode_summed_sequence(q_b, w_uk, w_uv, rows, k, d_r, scale=None, attn_scale=None):
    """``decode_summed`` for every head of one sequence whose rows are given, each block's
    heads stacked into one matrix product (as in ``decode_sequence``, but every head sees
    every block through its own W^UK_{j,h}, W^UV_{j,h}). w_uk, w_uv: [k][h][d_b][d_h].
    Returns (out [h][d_h], lse [k][h])."""
    q_b = np.asarray(q_b, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    h, qw = q_b.shape
    d_h = qw - d_r
    d_b = w_uk.shape[2]
    d_c = d_b * k
    if scale is None:
        scale = default_scale(d_h, d_r)
    if attn_scale is None:
        attn_scale = default_attn_scale(k)
    out = np.zeros((h, d_h))
    lse = np.full((k, h), -np.inf)
    if rows.shape[0] == 0:
        return out, lse
    for j in range(k):
        c_j, kr = _split(rows, j, d_c, k)
        q_lat = np.einsum("hcd,hd->hc", w_uk[j], q_b[:, :d_h])
        S = scale * (c_j @ q_lat.T + kr @ q_b[:, d_h:].T)
        m = S.max(axis=0)
        E = np.exp(S - m)
        l = E.sum(axis=0)
        lse[j] = m + np.log(l)
        lat = (E / l).T @ c_j
        out += attn_scale * np.einsum("hc,hcd->hd", lat, w_uv[j])
    return out, lse


# ---------------------------------------------------------------------------------------
# Summed-blocks reading: every head attends to every latent block with its own pair of
# matrices per block, each block under its own softmax, and the head's output is the sum of
# the k per-block outputs times alpha_attn. This is the reading that the MLRA index page's
# Table 2 (MLRA-4: 4nh(d_c/4) + 2nh d_h^R FLOPs per device, all h heads on each device's
# block) and the alpha_attn column of its model tables (MLRA-2: sqrt(2)/2, MLRA-4: 1/2) point
# to; the partitioned reading above is the default one.
# ---------------------------------------------------------------------------------------

def default_attn_scale(k: int) -> float:
    """alpha_attn when none is given: 1/sqrt(k). The MLRA index page's appendix model tables
    print sqrt(2)/2 for MLRA-2 and 1/2 for MLRA-4 (in its extracted text every caption sits
    below its own table's row, so each of these rows follows the caption of the table before)."""
    return 1.0 / math.sqrt(k)


def decode_summed(q, w_uk, w_uv, pool, page_table, seq_lens, k, d_r, scale=None, attn_scale=None,
                  form="absorbed"):
    """Full decode step under the summed-blocks reading.

    q: [B][h][d_h + d_r]; w_uk, w_uv: [k][h][d_b][d_h]; the rest as in ``decode``.
    ``out[b][h] = attn_scale * sum_j W^UV_{j,h} softmax_t(s_{j,h,t}) c_j[t]`` with
    ``s_{j,h,t} = scale * (q^C_h . W^UK_{j,h} c_j[t] + q^R_h . k^R[t])``.
    Returns ``out`` [B][h][d_h], ``lse`` [B][k][h] (each block's softmax, natural log) and, for
    the absorbed form, ``latent`` [B][k][h][d_b]. An empty sequence gives zeros and lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    pool = np.asarray(pool, dtype=np.float64)
    B, h, qw = q.shape
    d_h = qw - d_r
    d_b = w_uk.shape[2]
    d_c = d_b * k
    if scale is None:
        scale = default_scale(d_h, d_r)
    if attn_scale is None:
        attn_scale = default_attn_scale(k)
    out = np.zeros((B, h, d_h))
    lse = np.full((B, k, h), -np.inf)
    latent = np.zeros((B, k, h, d_b))
    for b in range(B):
        n = int(seq_lens[b])
        if n == 0:
            continue
        rows = gather_rows(pool, page_table, b, n)
        for j in range(k):
            c_j, kr = _split(rows, j, d_c, k)
            for hd in range(h):
                qc, qr = q[b, hd, :d_h], q[b, hd, d_h:]
                if form == "explicit":
                    o, lse[b, j, hd] = attend_head_explicit(qc, qr, w_uk[j, hd], w_uv[j, hd], c_j, kr, scale)
                else:
                    o, latent[b, j, hd], lse[b, j, hd] = attend_head_absorbed(
                        qc, qr, w_uk[j, hd], w_uv[j, hd], c_j, kr, scale)
                out[b, hd] += attn_scale * o
    res = {"out": out, "lse": lse}
    if form != "explicit":
        res["latent"] = latent
    return res


def decode_summed_heads(q, w_uk, w_uv, rows, seq_heads, k, d_r, scale=None, attn_scale=None):
    """``decode_summed`` for a list of heads of ONE sequence whose rows are given (sampled
    checks at full size). Returns (out [len][d_h], lse [len][k])."""
    q = np.asarray(q, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    d_b = w_uk.shape[2]
    d_c = d_b * k
    d_h = q.shape[-1] - d_r
    if scale is None:
        scale = default_scale(d_h, d_r)
    if attn_scale is None:
        attn_scale = default_attn_scale(k)
    outs, lses = [], []
    for hd in seq_heads:
        o_sum = np.zeros(d_h)
        l = np.zeros(k)
        for j in range(k):
            c_j, kr = _split(rows, j, d_c, k)
            o, _, l[j] = attend_head_absorbed(q[hd, :d_h], q[hd, d_h:], w_uk[j, hd], w_uv[j, hd], c_j, kr, scale)
            o_sum += attn_scale * o
        outs.append(o_sum)
        lses.append(l)
    return np.array(outs), np.array(lses)


# ---------------------------------------------------------------------------------------
# Split-KV plan and log-sum-exp merge. The pages describe no split scheme; this is the
# rule the library documents, restated here so the plan can be checked bit for bit.
# ---------------------------------------------------------------------------------------

class Segment(NamedTuple):
    b: int            # sequence
    group: int        # CTA group that processes it
    tile_begin: int   # first 128-token tile of sequence b (inclusive)
    tile_end: int     # last tile (exclusive)
    slot: int         # partial-result slot = b + group


def plan_segments(seq_lens, groups: int) -> List[Segment]:
    """Cut the flattened (sequence, 128-token tile) list into ``groups`` equal runs.

    tiles_b = ceil(n_b / 128); T = sum tiles_b; quota = ceil(T / groups); group g takes the
    flattened tiles [g*quota, min((g+1)*quota, T)); a run that crosses a sequence boundary
    becomes one segment per sequence. Slot b + g is unique because b and g never decrease
    along the flattened order.
    """
    tiles = [(int(n) + TILE_TOKENS - 1) // TILE_TOKENS for n in seq_lens]
    T = sum(tiles)
    if T == 0:
        return []
    quota = (T + groups - 1) // groups
    starts = []
    acc = 0
    for t in tiles:
        starts.append(acc)
        acc += t
    segs = []
    for g in range((T + quota - 1) // quota):
        lo, hi = g * quota, min((g + 1) * quota, T)
        for b, t in enumerate(tiles):
            s0, s1 = starts[b], starts[b] + t
            a, e = max(lo, s0), min(hi, s1)
            if a < e:
                segs.append(Segment(b, g, a - s0, e - s0, b + g))
    return segs


def partial_head(q_row, w_uk_h, c_j, kr, scale, t0, t1):
    """Latent partial of one head over tokens [t0, t1): (o~ normalised, lse natural log)."""
    d_h = w_uk_h.shape[1]
    q_lat = w_uk_h @ q_row[:d_h]
    s = scale * (c_j[t0:t1] @ q_lat + kr[t0:t1] @ q_row[d_h:])
    p, lse = _softmax_stats(s)
    return p @ c_j[t0:t1], lse


def merge_partials(parts):
    """Log-sum-exp merge of [(o~_s, lse_s)] into (o~, lse)."""
    lses = np.array([l for _, l in parts])
    m = lses.max()
    lse = m + math.log(np.exp(lses - m).sum())
    o = sum(np.exp(l - lse) * o_s for o_s, l in parts)
    return o, lse


# ---------------------------------------------------------------------------------------
# Counters (bytes and FLOPs of the decode path)
# ---------------------------------------------------------------------------------------

def cache_elems_per_token(d_c: int, d_r: int) -> int:
    """Latent-cache elements per token: d_c + d_r (Table 1 'KV Cache' column for MLA)."""
    return d_c + d_r


def loading_per_token_per_device(d_c: int, d_r: int, k: int, devices: int) -> float:
    """Elements each device loads per token when the k blocks are spread over ``devices``
    (devices <= k, devices | k): its d_c*(k/devices)/k latent share plus the shared k^R.
    k = 1 gives MLA's d_c + d_r at every device count (Table 1)."""
    blocks_here = max(1, k // devices)
    return d_c * blocks_here / k + d_r


def flops_per_token(h: int, d_c: int, d_r: int, k: int) -> int:
    """Attention FLOPs per cached token for one decode query: each head does a dot product
    over its block plus k^R (2*(d_b + d_r)) and a weighted sum over its block (2*d_b)."""
    d_b = d_c // k
    return h * (4 * d_b + 2 * d_r)


def mha_cache_elems_per_token(h: int, d_h: int) -> int:
    """Standard MHA caches K and V for every head: 2*h*d_h elements per token."""
    return 2 * h * d_h
