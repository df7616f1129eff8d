"""Pins for the float64 oracle: each test checks it against something other than itself.

* torch's scaled_dot_product_attention (an independent attention routine, run in float64)
  on explicitly reconstructed per-head keys and values;
* brute-force pure-Python loops on tiny inputs (no numpy linear algebra);
* closed forms: a length-1 context returns the up-projected value exactly;
* algebraic identities the pages state: absorbed == explicit reconstruction;
* the pages' printed numbers: Table 1 / Table 2 of "Multi-Head Low-Rank Attention"
  (thelatestinai.com) and the ai360xpert "Multi-Head Latent Attention" code example;
* invariants of the method: block independence, page placement, key order;
* hand-worked split plans.

The last group plants mistakes in the oracle (on the CPU) and checks that a pin catches each.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import mlra_oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_case(rng, B=2, h=8, k=4, d_h=16, d_b=24, d_r=8, lens=(37, 130), permute=True):
    """Small float64 case with d_b != d_h so a transposed weight cannot pass silently."""
    d_c = d_b * k
    lens = np.array(lens[:B])
    pages = [(n + 63) // 64 for n in lens]
    num_pages = sum(pages) + 2
    phys = rng.permutation(num_pages) if permute else np.arange(num_pages)
    pt = np.full((B, max(pages)), -1, dtype=np.int64)
    off = 0
    for b, p in enumerate(pages):
        pt[b, :p] = phys[off:off + p]
        off += p
    pool = rng.standard_normal((num_pages, 64, d_c + d_r))
    q = rng.standard_normal((B, h, d_h + d_r))
    w_uk = rng.standard_normal((h, d_b, d_h)) / math.sqrt(d_b)
    w_uv = rng.standard_normal((h, d_b, d_h)) / math.sqrt(d_b)
    return dict(q=q, w_uk=w_uk, w_uv=w_uv, pool=pool, page_table=pt, seq_lens=lens,
                k=k, d_r=d_r, d_c=d_c, d_h=d_h, h=h)


def _run(case, **kw):
    return O.decode(case["q"], case["w_uk"], case["w_uv"], case["pool"], case["page_table"],
                    case["seq_lens"], case["k"], case["d_r"], **kw)


# ---------------------------------------------------------------------------------------
# Against an independent attention routine
# ---------------------------------------------------------------------------------------

def _sdpa_reference(case, scale):
    """Per head: K_h = [c_j W^UK_h | k^R], V_h = c_j W^UV_h (ai360xpert 'The two projections';
    lesty.tech section 4 decoupled key), attention by torch SDPA in float64."""
    q, pool, pt = case["q"], case["pool"], case["page_table"]
    B, h, _ = q.shape
    d_h, d_r, k, d_c = case["d_h"], case["d_r"], case["k"], case["d_c"]
    d_b = d_c // k
    out = np.zeros((B, h, d_h))
    for b in range(B):
        n = int(case["seq_lens"][b])
        idx = torch.arange(n)
        rows = torch.from_numpy(pool)[torch.from_numpy(pt[b])[idx // 64], idx % 64]
        for hd in range(h):
            j = hd // (h // k)
            c_j = rows[:, j * d_b:(j + 1) * d_b]
            K = torch.cat([c_j @ torch.from_numpy(case["w_uk"][hd]), rows[:, d_c:]], dim=1)
            V = c_j @ torch.from_numpy(case["w_uv"][hd])
            Q = torch.from_numpy(q[b, hd]).reshape(1, 1, 1, -1)
            o = torch.nn.functional.scaled_dot_product_attention(
                Q, K[None, None], V[None, None], scale=scale)
            out[b, hd] = o.reshape(-1).numpy()
    return out


@pytest.mark.parametrize("k", [1, 2, 4])
def test_matches_torch_sdpa_on_reconstructed_heads(k):
    rng = np.random.default_rng(10 + k)
    case = _rand_case(rng, k=k, d_b=96 // k)
    scale = 0.37
    ref = _sdpa_reference(case, scale)
    for form in ("absorbed", "explicit"):
        got = _run(case, scale=scale, form=form)["out"]
        np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def _per_sequence(case, scale):
    """decode_sequence over every sequence of a case (rows gathered like the GPU tests do)."""
    B, h = case["q"].shape[:2]
    out = np.zeros((B, h, case["d_h"]))
    lse = np.zeros((B, h))
    for b in range(B):
        rows = O.gather_rows(case["pool"], case["page_table"], b, int(case["seq_lens"][b]))
        out[b], _, lse[b] = O.decode_sequence(case["q"][b], case["w_uk"], case["w_uv"], rows, case["k"],
                                              case["d_r"], scale=scale)
    return out, lse


@pytest.mark.parametrize("k", [1, 2, 4])
def test_per_sequence_form_matches_torch_sdpa(k):
    """The all-heads-at-once form against the same independent SDPA reference, and its lse
    against scipy's logsumexp of explicitly formed scores."""
    from scipy.special import logsumexp
    rng = np.random.default_rng(20 + k)
    case = _rand_case(rng, k=k, d_b=96 // k, lens=(1, 200))
    out, lse = _per_sequence(case, 0.29)
    np.testing.assert_allclose(out, _sdpa_reference(case, 0.29), rtol=1e-11, atol=1e-12)
    d_h, d_c, h = case["d_h"], case["d_c"], case["h"]
    d_b = d_c // k
    for b in range(2):
        rows = O.gather_rows(case["pool"], case["page_table"], b, int(case["seq_lens"][b]))
        for hd in range(h):
            j = hd // (h // k)
            s = 0.29 * (rows[:, j * d_b:(j + 1) * d_b] @ case["w_uk"][hd] @ case["q"][b, hd, :d_h]
                        + rows[:, d_c:] @ case["q"][b, hd, d_h:])
            assert abs(lse[b, hd] - logsumexp(s)) < 1e-12


def test_per_sequence_form_empty_sequence():
    rng = np.random.default_rng(5)
    case = _rand_case(rng)
    out, lat, lse = O.decode_sequence(case["q"][0], case["w_uk"], case["w_uv"], np.zeros((0, case["d_c"] + 8)),
                                      case["k"], case["d_r"])
    assert np.all(out == 0) and np.all(lat == 0) and np.all(np.isneginf(lse))


def test_planted_mistake_in_per_sequence_form_is_caught(monkeypatch):
    real_split = O._split
    monkeypatch.setattr(O, "_split", lambda rows, j, d_c, k: real_split(rows, (j + 1) % k, d_c, k))
    with pytest.raises(AssertionError):
        test_per_sequence_form_matches_torch_sdpa(4)


def test_absorbed_equals_explicit_reconstruction():
    """Absorption is exact (ai360xpert: reconstruction is exact; lesty.tech section 5)."""
    rng = np.random.default_rng(1)
    case = _rand_case(rng)
    a = _run(case, form="absorbed")
    e = _run(case, form="explicit")
    np.testing.assert_allclose(a["out"], e["out"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(a["lse"], e["lse"], rtol=1e-13)


# ---------------------------------------------------------------------------------------
# Brute force on tiny inputs (pure Python loops)
# ---------------------------------------------------------------------------------------

def _brute(case, scale):
    q, pool, pt = case["q"], case["pool"], case["page_table"]
    B, h, _ = q.shape
    d_h, d_r, k, d_c = case["d_h"], case["d_r"], case["k"], case["d_c"]
    d_b = d_c // k
    out = [[None] * h for _ in range(B)]
    lse = [[None] * h for _ in range(B)]
    lat = [[None] * h for _ in range(B)]
    for b in range(B):
        n = int(case["seq_lens"][b])
        rows = []
        for t in range(n):
            page = int(pt[b][t // 64])
            rows.append([float(x) for x in pool[page][t % 64]])
        for hd in range(h):
            j = hd // (h // k)
            Wk, Wv = case["w_uk"][hd], case["w_uv"][hd]
            scores = []
            for t in range(n):
                c = rows[t][j * d_b:(j + 1) * d_b]
                kr = rows[t][d_c:]
                s = 0.0
                for d in range(d_h):
                    kc = 0.0
                    for ci in range(d_b):
                        kc += c[ci] * Wk[ci][d]
                    s += q[b][hd][d] * kc
                for r in range(d_r):
                    s += q[b][hd][d_h + r] * kr[r]
                scores.append(scale * s)
            m = max(scores)
            e = [math.exp(s - m) for s in scores]
            tot = sum(e)
            lse[b][hd] = m + math.log(tot)
            o = [0.0] * d_h
            la = [0.0] * d_b
            for t in range(n):
                c = rows[t][j * d_b:(j + 1) * d_b]
                p = e[t] / tot
                for ci in range(d_b):
                    la[ci] += p * c[ci]
                for d in range(d_h):
                    v = 0.0
                    for ci in range(d_b):
                        v += c[ci] * Wv[ci][d]
                    o[d] += p * v
            out[b][hd] = o
            lat[b][hd] = la
    return np.array(out), np.array(lse), np.array(lat)


def test_brute_force_tiny():
    rng = np.random.default_rng(2)
    case = _rand_case(rng, B=2, h=4, k=2, d_h=5, d_b=6, d_r=3, lens=(3, 70))
    scale = 0.41
    bo, bl, blat = _brute(case, scale)
    got = _run(case, scale=scale)
    np.testing.assert_allclose(got["out"], bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(got["lse"], bl, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(got["latent"], blat, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------------------
# Closed forms and special cases
# ---------------------------------------------------------------------------------------

def test_length_one_context_returns_up_projected_value():
    """One token: p = 1, so o_h = W^UV_h c_j[0] and lse = s_0, whatever the query."""
    rng = np.random.default_rng(3)
    case = _rand_case(rng, lens=(1, 1))
    res = _run(case, scale=0.5)
    d_b, k, h, d_c = case["d_c"] // case["k"], case["k"], case["h"], case["d_c"]
    for b in range(2):
        row = case["pool"][case["page_table"][b, 0], 0]
        for hd in range(h):
            j = hd // (h // k)
            c = row[j * d_b:(j + 1) * d_b]
            exp_out = np.einsum("cd,c->d", case["w_uv"][hd], c)
            np.testing.assert_allclose(res["out"][b, hd], exp_out, rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(res["latent"][b, hd], c, rtol=0, atol=0)


def test_peaked_softmax_selects_one_token():
    """A query aligned with one token's RoPE key by a huge margin returns that token's value."""
    rng = np.random.default_rng(4)
    case = _rand_case(rng, B=1, lens=(90,))
    d_h, d_r = case["d_h"], case["d_r"]
    target = 57
    row = case["pool"][case["page_table"][0, target // 64], target % 64]
    case["q"][0, :, :d_h] = 0.0
    case["q"][0, :, d_h:] = 1e4 * row[case["d_c"]:]
    res = _run(case, scale=1.0)
    d_b = case["d_c"] // case["k"]
    for hd in range(case["h"]):
        j = hd // (case["h"] // case["k"])
        np.testing.assert_allclose(res["latent"][0, hd], row[j * d_b:(j + 1) * d_b], atol=1e-12)


def test_empty_sequence():
    rng = np.random.default_rng(5)
    case = _rand_case(rng, lens=(0, 5))
    case["page_table"][0, :] = -1
    res = _run(case)
    assert np.all(res["out"][0] == 0) and np.all(np.isneginf(res["lse"][0]))
    assert np.all(np.isfinite(res["out"][1]))


def test_default_scale_is_inverse_sqrt_of_decoupled_key_width():
    assert O.default_scale(128, 64) == 1.0 / math.sqrt(192)


# ---------------------------------------------------------------------------------------
# Invariants of the method
# ---------------------------------------------------------------------------------------

def test_block_independence():
    """Perturbing block j changes exactly the heads of group j (the latent heads 'do not
    talk to each other', alanhou.org summary, Core Mechanism / Key Concepts)."""
    rng = np.random.default_rng(6)
    case = _rand_case(rng)
    base = _run(case)["out"]
    k, h, d_b = case["k"], case["h"], case["d_c"] // case["k"]
    for j in range(k):
        pert = dict(case)
        pert["pool"] = case["pool"].copy()
        pert["pool"][..., j * d_b:(j + 1) * d_b] += rng.standard_normal(
            pert["pool"][..., j * d_b:(j + 1) * d_b].shape)
        out = _run(pert)["out"]
        group = slice(j * h // k, (j + 1) * h // k)
        changed = np.any(out != base, axis=(0, 2))
        assert changed[group].all()
        mask = np.ones(h, bool)
        mask[group] = False
        assert not changed[mask].any()


@pytest.mark.parametrize("k", [2, 4])
def test_tensor_parallel_shards_reproduce_the_layer(k):
    """k-way tensor parallelism (alanhou.org summary, Core Mechanism: each device loads only its
    latent head's cache, computes its subset of heads, and the results are combined): rank j
    runs plain latent attention (k = 1) over [c_j | k^R] with head group j's query and
    matrices; concatenating the ranks' heads gives the MLRA-k layer's output and lse."""
    rng = np.random.default_rng(20 + k)
    case = _rand_case(rng, k=k, d_b=48 // k * 2)
    full = _run(case, scale=0.4)
    h, d_b, d_c = case["h"], case["d_c"] // k, case["d_c"]
    hb = h // k
    outs, lses = [], []
    for j in range(k):
        shard = np.concatenate([case["pool"][..., j * d_b:(j + 1) * d_b], case["pool"][..., d_c:]], axis=-1)
        g = slice(j * hb, (j + 1) * hb)
        r = O.decode(case["q"][:, g], case["w_uk"][g], case["w_uv"][g], shard, case["page_table"],
                     case["seq_lens"], 1, case["d_r"], scale=0.4)
        outs.append(r["out"])
        lses.append(r["lse"])
    np.testing.assert_allclose(np.concatenate(outs, axis=1), full["out"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(np.concatenate(lses, axis=1), full["lse"], rtol=1e-13, atol=1e-14)


def test_page_placement_and_key_order_invariance():
    rng = np.random.default_rng(7)
    case = _rand_case(rng, permute=False)
    base = _run(case)
    # same logical rows in a different physical placement
    perm = rng.permutation(case["pool"].shape[0])
    moved = dict(case)
    moved["pool"] = np.empty_like(case["pool"])
    moved["pool"][perm] = case["pool"]
    moved["page_table"] = np.where(case["page_table"] >= 0, perm[case["page_table"]], -1)
    np.testing.assert_array_equal(_run(moved)["out"], base["out"])
    # reversing the keys of sequence 1 (a softmax is a set function of its keys)
    n = int(case["seq_lens"][1])
    rows = O.gather_rows(case["pool"], case["page_table"], 1, n)[::-1]
    rev = dict(case)
    rev["pool"] = case["pool"].copy()
    for t in range(n):
        rev["pool"][case["page_table"][1, t // 64], t % 64] = rows[t]
    np.testing.assert_allclose(_run(rev)["out"][1], base["out"][1], rtol=1e-12, atol=1e-13)


def test_gather_matches_workload_indexing():
    """The oracle's page walk agrees with torch advanced indexing on a generated workload."""
    inp = W.make_workload(W.scaled(W.WORKLOADS["mlra4_h128_b32_n8192"], batch=3, seq_len=200,
                                   h=8, d_h=16, d_c=64, d_r=16))
    pool = inp["pool"].float().numpy()
    for b in range(3):
        got = O.gather_rows(pool, inp["page_table"].numpy(), b, 200)
        ref = W.logical_rows(inp, b).float().numpy()
        np.testing.assert_array_equal(got, ref)


# ---------------------------------------------------------------------------------------
# Split plan and log-sum-exp merge
# ---------------------------------------------------------------------------------------

def test_plan_golden_cases():
    for case in _golden("plan_cases.json")["cases"]:
        segs = O.plan_segments(case["seq_lens"], case["groups"])
        assert [list(s) for s in segs] == case["segments"], case


@pytest.mark.parametrize("seed", range(5))
def test_plan_invariants(seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 5000, size=rng.integers(1, 40))
    lens[rng.random(len(lens)) < 0.2] = 0
    groups = int(rng.integers(1, 80))
    segs = O.plan_segments(lens, groups)
    tiles = [(n + 127) // 128 for n in lens]
    covered = {b: [] for b in range(len(lens))}
    slots = set()
    per_group = {}
    for s in segs:
        covered[s.b].append((s.tile_begin, s.tile_end))
        assert s.slot == s.b + s.group and s.slot not in slots
        slots.add(s.slot)
        per_group[s.group] = per_group.get(s.group, 0) + s.tile_end - s.tile_begin
        assert s.group < groups
    for b, t in enumerate(tiles):
        ranges = sorted(covered[b])
        pos = 0
        for a, e in ranges:
            assert a == pos and e > a
            pos = e
        assert pos == t
    if per_group:
        quota = (sum(tiles) + groups - 1) // groups
        assert max(per_group.values()) <= quota
    assert max(slots, default=-1) < len(lens) + groups


def test_split_merge_equals_unsplit():
    rng = np.random.default_rng(8)
    case = _rand_case(rng, B=2, lens=(700, 1000))
    scale = 0.3
    ref = _run(case, scale=scale)
    segs = O.plan_segments(case["seq_lens"], groups=5)
    assert len(segs) > 2
    d_h, k, h, d_c = case["d_h"], case["k"], case["h"], case["d_c"]
    for b in range(2):
        n = int(case["seq_lens"][b])
        rows = O.gather_rows(case["pool"], case["page_table"], b, n)
        for hd in range(h):
            j = O.head_block(hd, h, k)
            c_j, kr = rows[:, j * (d_c // k):(j + 1) * (d_c // k)], rows[:, d_c:]
            parts = [O.partial_head(case["q"][b, hd], case["w_uk"][hd], c_j, kr, scale,
                                    s.tile_begin * 128, min(s.tile_end * 128, n))
                     for s in segs if s.b == b]
            lat, lse = O.merge_partials(parts)
            np.testing.assert_allclose(lat, ref["latent"][b, hd], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse, ref["lse"][b, hd], rtol=1e-13)


# ---------------------------------------------------------------------------------------
# The pages' printed numbers
# ---------------------------------------------------------------------------------------

def test_table1_kv_loading():
    g = _golden("kv_cache_tables.json")
    sh = g["table1_shapes"]
    d_h = sh["d_h"]
    for dev, val in g["table1_loading_per_token_per_device_in_dh"]["MLA"].items():
        assert O.loading_per_token_per_device(sh["d_c"], sh["d_r"], 1, int(dev)) == val * d_h
    assert O.cache_elems_per_token(sh["d_c"], sh["d_r"]) == 576
    for dev, val in g["table1_loading_per_token_per_device_in_dh"]["MHA"].items():
        assert O.mha_cache_elems_per_token(sh["mha_heads"], d_h) / int(dev) == val * d_h


def test_table2_counters():
    g = _golden("kv_cache_tables.json")
    m = g["table2_MLA"]
    a = m["at"]
    assert a["n"] * O.flops_per_token(a["h"], a["d_c"], a["d_r"], 1) == m["numerator_value"]
    assert 2 * a["n"] * O.cache_elems_per_token(a["d_c"], a["d_r"]) == m["denominator_value"]
    d = g["table2_MLRA4_denominator"]
    assert 2 * d["at"]["n"] * O.loading_per_token_per_device(
        d["at"]["d_c"], d["at"]["d_r"], 4, 4) == d["value"]


def test_ai360xpert_cache_example():
    g = _golden("ai360xpert_cache_example.json")
    ex = g["code_example"]
    assert O.mha_cache_elems_per_token(ex["H"], ex["d_head"]) == ex["standard_cache_floats_per_token"]
    assert O.cache_elems_per_token(ex["d_c"], 0) == ex["mla_cache_floats_per_token"]
    assert ex["standard_cache_floats_per_token"] // ex["mla_cache_floats_per_token"] == ex["reduction"]
    # shapes of the reconstructed K and V with weights stored (H, d_c, d_head)
    rng = np.random.default_rng(9)
    c = rng.standard_normal(ex["d_c"])
    w = rng.standard_normal((ex["H"], ex["d_c"], ex["d_head"]))
    # a one-token context returns V_h[0] exactly; stacking heads gives V's printed shape
    V = np.stack([O.attend_head_explicit(np.zeros(ex["d_head"]), np.zeros(0), w[hd], w[hd],
                                         c[None], np.zeros((1, 0)), 1.0)[0]
                  for hd in range(ex["H"])])
    assert list(V.shape) == ex["V_shape"]
    ds = g["deepseek_v2"]
    assert O.mha_cache_elems_per_token(ds["H"], ds["d_head"]) == ds["standard_floats"]
    assert ds["standard_floats"] // ds["mla_floats"] == ds["reduction"]


# ---------------------------------------------------------------------------------------
# Planted mistakes: each must be caught by one of the pins above
# ---------------------------------------------------------------------------------------

def _mutant_drop_rope(qc, qr, w_uk_h, w_uv_h, c_j, kr, scale):
    q_lat = w_uk_h @ qc
    s = scale * (c_j @ q_lat)
    p, lse = O._softmax_stats(s)
    o_lat = p @ c_j
    return o_lat @ w_uv_h, o_lat, lse


def _mutant_sign(qc, qr, w_uk_h, w_uv_h, c_j, kr, scale):
    q_lat = w_uk_h @ qc
    s = scale * (c_j @ q_lat - kr @ qr)
    p, lse = O._softmax_stats(s)
    o_lat = p @ c_j
    return o_lat @ w_uv_h, o_lat, lse


def _mutant_reversed_uv_rows(qc, qr, w_uk_h, w_uv_h, c_j, kr, scale):
    q_lat = w_uk_h @ qc
    s = scale * (c_j @ q_lat + kr @ qr)
    p, lse = O._softmax_stats(s)
    o_lat = p @ c_j
    return o_lat @ w_uv_h[::-1], o_lat, lse


@pytest.mark.parametrize("mutant", [_mutant_drop_rope, _mutant_sign, _mutant_reversed_uv_rows])
def test_planted_mistakes_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(O, "attend_head_absorbed", mutant)
    with pytest.raises(AssertionError):
        test_matches_torch_sdpa_on_reconstructed_heads(4)


def test_planted_block_index_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(O, "head_block", lambda head, h, k: head % k)
    with pytest.raises(AssertionError):
        test_block_independence()


def test_planted_page_index_mistake_is_caught(monkeypatch):
    def bad_gather(pool, page_table, b, n):
        rows = np.empty((n, pool.shape[-1]))
        for t in range(n):
            rows[t] = pool[int(page_table[b, t // 64]), (t * 7) % 64]
        return rows
    monkeypatch.setattr(O, "gather_rows", bad_gather)
    with pytest.raises(AssertionError):
        test_gather_matches_workload_indexing()
