"""GPU parity for the step before decoding (each sequence's new cache row: down-projection,
RoPE key, page slot) through the C ABI, against the float64 producer oracle.

The stored bf16 rows are compared with the oracle's float64 rows (bf16 rounding of the value
plus fp32 accumulation: relative 2^-8), every other byte of the pool must be unchanged, and a
decode step over the appended context must match the decode oracle.
"""
import numpy as np
import pytest
import torch

import rank_latent_kv_mlra_b200 as M
import workloads as W
from oracle import producer_oracle as P
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

HEAD = W.WORKLOADS["mlra4_h128_b32_n8192"]
CASES = {
    "small_2slices": (W.scaled(HEAD, batch=3, seq_len=None, len_range=(1, 1500), seed=51), 256),
    "batch100_3slices": (W.scaled(HEAD, batch=100, seq_len=None, len_range=(1, 700), seed=52), 384),
    "batch300_3tiles": (W.scaled(HEAD, batch=300, seq_len=None, len_range=(1, 300), seed=55), 256),
    "mlra2_small": (W.scaled(W.WORKLOADS["mlra2_h128_b64_n4096"], batch=5, seq_len=None, len_range=(1, 900),
                             seed=53), 512),
    "headline_d5120": (HEAD, W.PRODUCER_D_MODEL),
}


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    M.load_library()


def _bits(t):
    return t.view(torch.int16)


def _run(w, inp, pr, **kw):
    hdl = G.make_handle(w, inp)
    ws = M.mlra_project_append(hdl, pr["x"], pr["w_down"], pr["positions"], inp["pool"], inp["page_table"], **kw)
    torch.cuda.synchronize()
    return M.mlra_get_status(ws)


def _oracle_rows(w, inp, pr, base=P.ROPE_BASE):
    return P.project_append(pr["x"].double().cpu().numpy(), pr["w_down"].double().cpu().numpy(), w.d_c, w.d_r,
                            pr["positions"].cpu().numpy(), inp["page_table"].cpu().numpy(), base)


@pytest.mark.parametrize("name", list(CASES))
def test_rows_match_oracle_and_nothing_else_changes(name):
    w, d_model = CASES[name]
    inp = W.make_workload(w, device="cuda")
    pr = W.make_producer_inputs(w, inp, d_model=d_model)
    before = inp["pool"].clone()
    assert _run(w, inp, pr) == 0
    rows, pages, slots = _oracle_rows(w, inp, pr)
    pool = inp["pool"]
    got = pool[torch.as_tensor(pages, device="cuda").long(), torch.as_tensor(slots, device="cuda").long()]
    got = got.float().cpu().numpy()
    err = np.abs(got - rows)
    bound = np.abs(rows) * 2.0 ** -8 + 1e-5
    assert (err <= bound).all(), float((err - bound).max())
    # every other slot is untouched (bitwise, NaN slots included)
    mask = torch.ones(pool.shape[:2], dtype=torch.bool, device="cuda")
    mask[torch.as_tensor(pages, device="cuda").long(), torch.as_tensor(slots, device="cuda").long()] = False
    assert torch.equal(_bits(pool)[mask], _bits(before)[mask])


def test_rope_base_is_applied():
    w, d_model = CASES["small_2slices"]
    inp = W.make_workload(w, device="cuda")
    pr = W.make_producer_inputs(w, inp, d_model=d_model)
    assert _run(w, inp, pr, rope_base=500.0) == 0
    rows, pages, slots = _oracle_rows(w, inp, pr, base=500.0)
    got = inp["pool"][torch.as_tensor(pages).long().cuda(), torch.as_tensor(slots).long().cuda()].float().cpu().numpy()
    assert (np.abs(got - rows) <= np.abs(rows) * 2.0 ** -8 + 1e-5).all()


def test_out_of_range_position_and_page_are_reported_and_not_written():
    w, d_model = CASES["small_2slices"]
    inp = W.make_workload(w, device="cuda")
    pr = W.make_producer_inputs(w, inp, d_model=d_model)
    before = inp["pool"].clone()
    cap = inp["page_table"].shape[1] * 64
    bad = pr["positions"].clone()
    bad[1] = cap  # one past the page-table row
    assert _run(w, inp, dict(pr, positions=bad)) == -7  # MLRA_ERR_SEQ_LEN
    # sequences 0 and 2 are written, nothing else changes
    rows, pages, slots = _oracle_rows(w, inp, pr)
    keep = torch.ones(inp["pool"].shape[:2], dtype=torch.bool, device="cuda")
    for b in (0, 2):
        keep[int(pages[b]), int(slots[b])] = False
    assert torch.equal(_bits(inp["pool"])[keep], _bits(before)[keep])
    # a page id outside the pool
    inp2 = W.make_workload(w, device="cuda")
    pt = inp2["page_table"].clone()
    p0 = int(pr["positions"][0]) // 64
    pt[0, p0] = inp2["pool"].shape[0]
    before2 = inp2["pool"].clone()
    assert _run(w, dict(inp2, page_table=pt), pr) == -4  # MLRA_ERR_PAGE_OOB
    rows2, pages2, slots2 = _oracle_rows(w, inp2, pr)
    keep = torch.ones(inp2["pool"].shape[:2], dtype=torch.bool, device="cuda")
    for b in (1, 2):
        keep[int(pages2[b]), int(slots2[b])] = False
    assert torch.equal(_bits(inp2["pool"])[keep], _bits(before2)[keep])


def test_decode_reads_the_appended_row():
    """Append each sequence's next token (position n_b) and decode over n_b + 1 tokens."""
    w = W.scaled(HEAD, batch=4, seq_len=None, len_range=(1, 900), seed=54)
    inp = W.make_workload(w, device="cuda")
    cap = (inp["page_table"] >= 0).sum(dim=1) * 64
    room = inp["seq_lens"] < cap
    assert room.any()
    pr = W.make_producer_inputs(w, inp, d_model=256)
    pos = torch.where(room, inp["seq_lens"], pr["positions"])
    pr["positions"] = pos.to(torch.int32)
    assert _run(w, inp, pr) == 0
    inp["seq_lens"] = torch.where(room, inp["seq_lens"] + 1, inp["seq_lens"]).to(torch.int32)
    out, lse, ws = G.run_decode(G.make_handle(w, inp), inp)
    assert M.mlra_get_status(ws) == 0
    ref = G.oracle_full(w, inp)
    G.assert_parity(out.cpu().numpy(), ref["out"], "decode after append")


def test_e4m3_cache_rows():
    """New rows into an E4M3 cache: each stored byte is the E4M3 value nearest to row / scale
    (the GPU rounds its fp32 sum, the oracle its float64 value, so a value within the fp32
    accumulation error of a rounding midpoint may take the neighbouring code: one E4M3 step at
    most); nothing else in the pool changes."""
    from oracle import fp8_cache_oracle as F
    w = W.scaled(W.WORKLOADS["mlra4fp8_h128_b32_n8192"], batch=5, seq_len=None, len_range=(1, 700), seed=56)
    inp = W.make_workload(w, device="cuda")
    pr = W.make_producer_inputs(w, inp, d_model=384)
    before = inp["pool"].clone()
    assert _run(w, inp, pr) == 0
    rows, pages, slots = _oracle_rows(w, inp, pr)
    pool = inp["pool"]
    pi, si = torch.as_tensor(pages, device="cuda").long(), torch.as_tensor(slots, device="cuda").long()
    got = pool[pi, si].cpu().numpy()
    deq = F.e4m3_decode_array(got) * W.E4M3_SCALE
    assert np.all(np.abs(deq - rows) <= np.abs(rows) * 2.0 ** -3 + W.E4M3_SCALE * 2.0 ** -9)
    exact = F.quantize_rows(rows, w.d_c, W.E4M3_SCALE, W.E4M3_SCALE)
    assert np.mean(got == exact) > 0.99
    mask = torch.ones(pool.shape[:2], dtype=torch.bool, device="cuda")
    mask[pi, si] = False
    assert torch.equal(pool[mask], before[mask])
