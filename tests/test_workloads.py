"""The synthetic inputs (workloads.py) have the structure the benchmark configurations state:
lengths, page placement, NaN-poisoned unused slots, value scales and determinism. CPU only."""
import math

import numpy as np
import pytest
import torch

import workloads as W


def test_every_configured_workload_has_consistent_shapes():
    for name, w in W.WORKLOADS.items():
        assert w.d_c % w.k == 0 and w.h % w.k == 0, name
        assert (w.seq_len is None) != (w.len_range is None), name
        lens = W.draw_seq_lens(w)
        assert lens.dtype == torch.int32 and lens.shape == (w.batch,)
        if w.seq_len is not None:
            assert int(lens.min()) == int(lens.max()) == w.seq_len
        else:
            lo, hi = w.len_range
            assert lo <= int(lens.min()) and int(lens.max()) <= hi


def test_headline_shapes():
    w = W.WORKLOADS[W.HEADLINE]
    assert (w.k, w.h, w.d_h, w.d_c, w.d_r, w.batch, w.seq_len) == (4, 128, 128, 512, 64, 32, 8192)


@pytest.mark.parametrize("paging", ["permuted", "contiguous"])
def test_page_table_places_every_page_once(paging):
    lens = torch.tensor([0, 1, 63, 64, 65, 1000, 4096], dtype=torch.int32)
    table, num_pages = W.make_page_table(lens, paging, seed=3, extra_pages=5)
    pages = [(int(n) + 63) // 64 for n in lens]
    assert num_pages == sum(pages) + 5
    assert table.shape == (len(lens), max(pages))
    used = []
    for b, p in enumerate(pages):
        row = table[b].tolist()
        assert all(x >= 0 for x in row[:p]) and all(x == -1 for x in row[p:])
        used += row[:p]
    assert len(set(used)) == len(used) and all(0 <= x < num_pages for x in used)
    if paging == "contiguous":
        assert used == list(range(sum(pages)))
    else:
        assert used != sorted(used)


def test_unused_slots_and_pages_hold_nan():
    w = W.scaled(W.WORKLOADS[W.HEADLINE], batch=3, seq_len=None, len_range=(1, 300), h=8, d_h=16,
                 d_c=64, d_r=16, seed=11)
    inp = W.make_workload(w, extra_pages=2)
    pool = inp["pool"].float()
    referenced = set()
    for b in range(w.batch):
        n = int(inp["seq_lens"][b])
        p = (n + 63) // 64
        ids = inp["page_table"][b, :p].tolist()
        referenced |= set(ids)
        rows = W.logical_rows(inp, b).float()
        assert rows.shape == (n, w.d_c + w.d_r) and torch.isfinite(rows).all()
        tail = n - (p - 1) * 64
        assert torch.isnan(pool[ids[-1], tail:]).all()
    for pg in range(inp["num_pages"]):
        if pg not in referenced:
            assert torch.isnan(pool[pg]).all()


def test_draws_are_deterministic_and_scaled():
    w = W.scaled(W.WORKLOADS[W.HEADLINE], batch=2, seq_len=256, h=8, d_h=16, d_c=64, d_r=16)
    a, b = W.make_workload(w, keep_f32=True), W.make_workload(w, keep_f32=True)
    for key in ("seq_lens", "page_table", "pool", "q", "w_uk", "w_uv"):
        assert torch.equal(a[key].view(torch.uint8) if a[key].is_floating_point() else a[key],
                           b[key].view(torch.uint8) if b[key].is_floating_point() else b[key]), key
    # cache and query N(0, 1); weights N(0, 1) / sqrt(d_b)
    rows = torch.cat([W.logical_rows(a, i).float() for i in range(2)])
    assert abs(float(rows.std()) - 1.0) < 0.05 and abs(float(rows.mean())) < 0.05
    assert abs(float(a["w_uk_f32"].std()) * math.sqrt(w.d_b) - 1.0) < 0.05
    assert a["w_uk"].shape == (w.h, w.d_b, w.d_h)


def test_tiny_workload_scales_activations_and_keeps_f32_query():
    w = W.WORKLOADS["mlra4_h8_b1_n256_f32"]
    inp = W.make_workload(w, keep_f32=True)
    assert inp["q"].dtype == torch.float32
    rows = W.logical_rows({**inp, "pool": inp["pool_f32"]}, 0)
    # latent columns scaled by 1/sqrt(d_b), RoPE columns by 1/sqrt(d_r)
    assert abs(float(rows[:, :w.d_c].std()) * math.sqrt(w.d_b) - 1.0) < 0.1
    assert abs(float(rows[:, w.d_c:].std()) * math.sqrt(w.d_r) - 1.0) < 0.15


def test_e4m3_cache_bytes_are_the_scaled_values():
    w = W.scaled(W.WORKLOADS["mlra4fp8_h128_b32_n8192"], batch=2, seq_len=200, h=8, d_h=16, d_c=64,
                 d_r=16)
    inp = W.make_workload(w, keep_f32=True)
    assert inp["pool"].dtype == torch.uint8
    for b in range(2):
        got = W.logical_rows(inp, b).view(torch.float8_e4m3fn).float() * W.E4M3_SCALE
        ref = W.logical_rows({**inp, "pool": inp["pool_f32"]}, b)
        # one E4M3 rounding: within half a unit in the last place (3 mantissa bits)
        rel = ((got - ref).abs() / ref.abs().clamp_min(1e-3)).max()
        assert float(rel) <= 2.0 ** -4 + 1e-6
