"""Pins for the oracle's summed-blocks reading (every head attends to every latent block with
its own matrices per block; the per-block outputs are summed times alpha_attn), each against
something other than the oracle itself:

* torch's scaled_dot_product_attention in float64 on explicitly reconstructed per-(block,
  head) keys and values, summed and scaled by hand;
* brute-force pure-Python loops on a tiny case;
* scipy's logsumexp of explicitly formed scores for the per-block lse;
* the identity the method states for k = 1 (one block, alpha_attn = 1: plain MLA).

The last tests plant mistakes in the oracle (on the CPU) and check that a pin catches each.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import mlra_oracle as O


def _rand_case(rng, B=2, h=6, k=4, d_h=16, d_b=24, d_r=8, lens=(37, 130)):
    d_c = d_b * k
    lens = np.array(lens[:B])
    pages = [(n + 63) // 64 for n in lens]
    num_pages = sum(pages) + 1
    phys = rng.permutation(num_pages)
    pt = np.full((B, max(pages)), -1, dtype=np.int64)
    off = 0
    for b, p in enumerate(pages):
        pt[b, :p] = phys[off:off + p]
        off += p
    pool = rng.standard_normal((num_pages, 64, d_c + d_r))
    q = rng.standard_normal((B, h, d_h + d_r))
    w_uk = rng.standard_normal((k, h, d_b, d_h)) / math.sqrt(d_b)
    w_uv = rng.standard_normal((k, h, d_b, d_h)) / math.sqrt(d_b)
    return dict(q=q, w_uk=w_uk, w_uv=w_uv, pool=pool, page_table=pt, seq_lens=lens, k=k, d_r=d_r,
                d_c=d_c, d_h=d_h, h=h)


def _run(case, **kw):
    return O.decode_summed(case["q"], case["w_uk"], case["w_uv"], case["pool"], case["page_table"],
                           case["seq_lens"], case["k"], case["d_r"], **kw)


def _rows(case, b):
    n = int(case["seq_lens"][b])
    t = np.arange(n)
    return case["pool"][case["page_table"][b][t // 64], t % 64]


def _sdpa_reference(case, scale, attn_scale):
    q = case["q"]
    B, h, _ = q.shape
    d_h, d_r, k, d_c = case["d_h"], case["d_r"], case["k"], case["d_c"]
    d_b = d_c // k
    out = np.zeros((B, h, d_h))
    for b in range(B):
        rows = torch.from_numpy(_rows(case, b))
        for hd in range(h):
            Q = torch.from_numpy(q[b, hd]).reshape(1, 1, 1, -1)
            for j in range(k):
                c_j = rows[:, j * d_b:(j + 1) * d_b]
                K = torch.cat([c_j @ torch.from_numpy(case["w_uk"][j, hd]), rows[:, d_c:]], dim=1)
                V = c_j @ torch.from_numpy(case["w_uv"][j, hd])
                o = torch.nn.functional.scaled_dot_product_attention(Q, K[None, None], V[None, None], scale=scale)
                out[b, hd] += attn_scale * o.reshape(-1).numpy()
    return out


@pytest.mark.parametrize("k", [1, 2, 4])
def test_summed_matches_torch_sdpa(k):
    rng = np.random.default_rng(40 + k)
    case = _rand_case(rng, k=k, d_b=96 // k)
    for form in ("absorbed", "explicit"):
        got = _run(case, scale=0.31, attn_scale=0.7, form=form)["out"]
        np.testing.assert_allclose(got, _sdpa_reference(case, 0.31, 0.7), rtol=1e-11, atol=1e-12)
    # default alpha_attn and default scale: the printed model-table values (MLRA-2 sqrt(2)/2,
    # MLRA-4 1/2), and 1 for a single block (plain MLA has no alpha_attn)
    printed = {1: 1.0, 2: math.sqrt(2) / 2, 4: 0.5}
    got = _run(case)["out"]
    ref = _sdpa_reference(case, O.default_scale(case["d_h"], case["d_r"]), printed[k])
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("k", [2, 4])
def test_summed_per_sequence_form_matches_torch_sdpa(k):
    """decode_summed_sequence (every head of a sequence at once) against the independent SDPA
    reference, at a given and at the default alpha_attn."""
    rng = np.random.default_rng(60 + k)
    case = _rand_case(rng, k=k, d_b=96 // k, lens=(3, 190))
    printed = {2: math.sqrt(2) / 2, 4: 0.5}
    for alpha in (0.8, None):
        ref = _sdpa_reference(case, 0.33, printed[k] if alpha is None else alpha)
        for b in range(2):
            rows = _rows(case, b)
            out, lse = O.decode_summed_sequence(case["q"][b], case["w_uk"], case["w_uv"], rows, k, case["d_r"],
                                                scale=0.33, attn_scale=alpha)
            np.testing.assert_allclose(out, ref[b], rtol=1e-11, atol=1e-12)
            assert lse.shape == (k, case["h"])


def test_summed_lse_per_block_matches_logsumexp():
    rng = np.random.default_rng(3)
    case = _rand_case(rng)
    res = _run(case, scale=0.5)
    d_h, d_c, k = case["d_h"], case["d_c"], case["k"]
    d_b = d_c // k
    for b in range(2):
        rows = _rows(case, b)
        for j in range(k):
            c_j, kr = rows[:, j * d_b:(j + 1) * d_b], rows[:, d_c:]
            for hd in range(case["h"]):
                K = c_j @ case["w_uk"][j, hd]
                s = 0.5 * (K @ case["q"][b, hd, :d_h] + kr @ case["q"][b, hd, d_h:])
                assert abs(res["lse"][b, j, hd] - logsumexp(s)) < 1e-12


def test_summed_brute_force_tiny():
    rng = np.random.default_rng(5)
    case = _rand_case(rng, B=1, h=2, k=2, d_h=3, d_b=4, d_r=2, lens=(5,))
    scale, alpha = 0.9, 0.6
    got = _run(case, scale=scale, attn_scale=alpha)["out"]
    d_h, d_r, k, d_c = case["d_h"], case["d_r"], case["k"], case["d_c"]
    d_b = d_c // k
    rows = [[float(x) for x in r] for r in _rows(case, 0)]
    for hd in range(case["h"]):
        qc = [float(x) for x in case["q"][0, hd, :d_h]]
        qr = [float(x) for x in case["q"][0, hd, d_h:]]
        o = [0.0] * d_h
        for j in range(k):
            Wk, Wv = case["w_uk"][j, hd], case["w_uv"][j, hd]
            scores, vals = [], []
            for r in rows:
                c = r[j * d_b:(j + 1) * d_b]
                K = [sum(c[i] * float(Wk[i][d]) for i in range(d_b)) for d in range(d_h)]
                V = [sum(c[i] * float(Wv[i][d]) for i in range(d_b)) for d in range(d_h)]
                s = sum(qc[d] * K[d] for d in range(d_h)) + sum(qr[d] * r[d_c + d] for d in range(d_r))
                scores.append(scale * s)
                vals.append(V)
            m = max(scores)
            e = [math.exp(s - m) for s in scores]
            z = sum(e)
            for d in range(d_h):
                o[d] += alpha * sum(e[t] * vals[t][d] for t in range(len(rows))) / z
        np.testing.assert_allclose(got[0, hd], o, rtol=1e-12, atol=1e-13)


def test_summed_k1_without_scaling_is_plain_mla():
    """k = 1 and alpha_attn = 1: the one block is the whole latent (MLA), whichever reading."""
    rng = np.random.default_rng(7)
    case = _rand_case(rng, k=1, d_b=48)
    got = _run(case, attn_scale=1.0)
    ref = O.decode(case["q"], case["w_uk"][0], case["w_uv"][0], case["pool"], case["page_table"],
                   case["seq_lens"], 1, case["d_r"])
    np.testing.assert_allclose(got["out"], ref["out"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(got["lse"][:, 0], ref["lse"], rtol=1e-13)


def test_default_attn_scale_matches_the_printed_model_tables():
    """alpha_attn when none is given reproduces both printed MLRA values: sqrt(2)/2 for MLRA-2
    and 1/2 for MLRA-4 (the appendix rows that follow the GTA and MLRA-2 captions, each caption
    sitting below its own table's row in the page text)."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "model_tables.json")))
    for name in ("MLRA-2", "MLRA-4"):
        row = g["alpha_attn"][name]
        assert math.isclose(O.default_attn_scale(row["k"]), row["value"], rel_tol=1e-15), name
    # 1/k would give the MLRA-2 value 1/2 but the MLRA-4 value 1/4: both rows are needed.
    assert not math.isclose(1.0 / 4, g["alpha_attn"]["MLRA-4"]["value"])


def test_summed_empty_sequence():
    rng = np.random.default_rng(9)
    case = _rand_case(rng)
    case["seq_lens"] = np.array([0, 70])
    res = _run(case)
    assert np.all(res["out"][0] == 0) and np.all(np.isneginf(res["lse"][0]))
    assert np.all(np.isfinite(res["out"][1]))


# ---------------------------------------------------------------------------------------
# Planted mistakes (in the oracle, on the CPU) that a pin above must catch
# ---------------------------------------------------------------------------------------

def test_planted_missing_alpha_is_caught(monkeypatch):
    monkeypatch.setattr(O, "default_attn_scale", lambda k: 1.0)
    with pytest.raises(AssertionError):
        test_summed_matches_torch_sdpa(4)


def test_planted_wrong_block_is_caught(monkeypatch):
    real_split = O._split
    monkeypatch.setattr(O, "_split", lambda rows, j, d_c, k: real_split(rows, (j + 1) % k, d_c, k))
    with pytest.raises(AssertionError):
        test_summed_matches_torch_sdpa(4)


def test_planted_missing_rope_term_is_caught(monkeypatch):
    def no_rope(qc, qr, w_uk_h, w_uv_h, c_j, kr, scale):
        q_lat = w_uk_h @ qc
        p, lse = O._softmax_stats(scale * (c_j @ q_lat))
        o_lat = p @ c_j
        return o_lat @ w_uv_h, o_lat, lse
    monkeypatch.setattr(O, "attend_head_absorbed", no_rope)
    with pytest.raises(AssertionError):
        test_summed_matches_torch_sdpa(2)
