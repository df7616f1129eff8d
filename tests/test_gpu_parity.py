"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Each stage is checked on its own as well as end to end:
  absorbed query (workspace) -> split partials (workspace) -> merged latent -> output.
Reduced sizes and the full workload sizes (the launch configuration the benchmark times)
both compare every output element and every lse against the oracle.
"""
import math

import numpy as np
import pytest
import torch

import rank_latent_kv_mlra_b200 as M
import workloads as W
from oracle import mlra_oracle as O
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    M.load_library()


def _small(name, **kw):
    return W.scaled(W.WORKLOADS[name], **kw)


# reduced workloads: several tiles, a ragged tail, several splits per sequence
SMALL = {
    "tiny_full": W.WORKLOADS["mlra4_h8_b1_n256_f32"],
    "mlra4_small": _small("mlra4_h128_b32_n8192", batch=3, seq_len=None, len_range=(1, 1500), seed=11),
    "mlra2_small": _small("mlra2_h128_b64_n4096", batch=3, seq_len=None, len_range=(100, 1300), seed=12),
    "mlra4_ragged_small": _small("mlra4_h128_b128_ragged1k_32k", batch=6, len_range=(1, 2000), seed=13),
    "mla_small": _small("mla_h128_b128_ragged1k_32k", batch=5, len_range=(1, 1500), seed=14),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_absorbed_query_matches_oracle(name):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    _, _, ws = G.run_decode(hdl, inp)
    v = G.workspace_views(hdl, ws, w.batch)
    exp = G.expected_q_pack(w, inp, v["info"]["heads_per_cta"], v["info"]["ctas_per_group"],
                            v["info"]["softmax_scale"])
    got = v["q_pack"].double().cpu()
    hb = w.h // w.k
    real = torch.zeros(got.shape[1:3], dtype=torch.bool)
    for hd in range(w.h):
        j, r = divmod(hd, hb)
        real[j * (got.shape[1] // w.k) + r // got.shape[2], r % got.shape[2]] = True
    # bf16 rounding of a float64 product: relative 2^-8 of the largest entry per row
    diff = (got - exp).abs()[:, real]
    bound = exp.abs()[:, real].amax(dim=-1, keepdim=True) * 2.0 ** -7 + 1e-6
    assert (diff <= bound).all(), float((diff - bound).max())
    # rows of a head chunk narrower than the MMA are not written (the decode never reads them)


@pytest.mark.parametrize("name", ["tiny_full", "tiny_h12"])
def test_padded_query_rows_are_never_read(name):
    """h/k below the decode MMA's N: the padding rows of the packed query are left unwritten
    and must not reach any output. The workspace is filled with NaN bytes first."""
    w = SMALL["tiny_full"] if name == "tiny_full" else _small("mlra4_h8_b1_n256_f32", h=12, seed=15)
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    info = M.mlra_get_info(hdl)
    assert w.h // w.k < info["heads_per_cta"]
    ws = M.alloc_workspace(hdl, w.batch, "cuda")
    ws.fill_(0xFF)
    out, lse, ws = G.run_decode(hdl, inp, workspace=ws)
    assert M.mlra_get_status(ws) == 0
    G.assert_parity(out.cpu().numpy(), G.oracle_full(w, inp)["out"], f"{name} with a NaN-filled workspace")


@pytest.mark.parametrize("name", list(SMALL))
def test_latent_output_matches_oracle(name):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    lat, lse, ws = G.run_decode(hdl, inp, latent=True)
    assert M.mlra_get_status(ws) == 0
    ref = G.oracle_full(w, inp)
    G.assert_parity(lat.cpu().numpy(), ref["latent"], f"{name} latent")
    G.assert_parity(lse.cpu().numpy(), ref["lse"], f"{name} lse", tol_max=G.TOL_LSE_ABS, tol_mean=2e-3,
                    tol_rel=1e-3)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_output_matches_oracle(name, out_dtype):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    out, lse, ws = G.run_decode(hdl, inp, out_dtype=out_dtype)
    assert M.mlra_get_status(ws) == 0
    ref = G.oracle_full(w, inp)
    G.assert_parity(out.float().cpu().numpy(), ref["out"], f"{name} out")
    G.assert_parity(lse.cpu().numpy(), ref["lse"], f"{name} lse", tol_max=G.TOL_LSE_ABS, tol_mean=2e-3,
                    tol_rel=1e-3)


@pytest.mark.parametrize("name", ["mlra4_small", "mla_small"])
def test_split_partials_match_oracle(name):
    """Every (segment, head) partial the decode kernel writes equals the oracle's partial
    over the same token range (the plan is checked bit-exact separately)."""
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    _, _, ws = G.run_decode(hdl, inp, latent=True)
    v = G.workspace_views(hdl, ws, w.batch)
    segs = O.plan_segments(inp["seq_lens"].cpu().tolist(), v["info"]["groups"])
    pool = inp["pool"].float().cpu().numpy()
    pt = inp["page_table"].cpu().numpy()
    q = inp["q"].double().cpu().numpy()
    wuk = inp["w_uk"].double().cpu().numpy()
    scale = O.default_scale(w.d_h, w.d_r)
    o_part = v["o_part"].cpu().numpy()
    lse_part = v["lse_part"].cpu().numpy()
    worst = 0.0
    for s in segs:
        n = int(inp["seq_lens"][s.b])
        rows = O.gather_rows(pool, pt, s.b, n)
        for hd in range(0, w.h, 7):
            j = O.head_block(hd, w.h, w.k)
            c_j, kr = rows[:, j * w.d_b:(j + 1) * w.d_b], rows[:, w.d_c:]
            o, l = O.partial_head(q[s.b, hd], wuk[hd], c_j, kr, scale, s.tile_begin * 128,
                                  min(s.tile_end * 128, n))
            worst = max(worst, float(np.abs(o_part[s.slot, hd] - o).max()))
            assert abs(lse_part[s.slot, hd] * math.log(2) - l) < 2e-2, (s, hd)
    assert worst < 2e-2, worst


@pytest.mark.parametrize("name", ["mlra4_small", "mlra2_small", "mla_small", "tiny_full"])
def test_plan_is_bit_exact(name):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    groups = M.mlra_get_info(hdl)["groups"]
    rng = np.random.default_rng(5)
    # batches up to 256 take the warp-level plan, larger ones the block-wide scans
    cases = [inp["seq_lens"].cpu().tolist(), [0, 0, 5], [8192] * 32, list(rng.integers(0, 40000, 128)),
             list(rng.integers(0, 3000, 256)), list(rng.integers(0, 3000, 257)), [1] * 300]
    for lens in cases:
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        got, n = M.mlra_plan(hdl, sl, pt_stride=1024)
        exp = O.plan_segments(lens, groups)
        assert n == len(exp)
        assert got == [tuple(s) for s in exp]


def test_page_placement_is_bit_exact():
    """The same logical cache under two physical page placements gives identical bits."""
    w = SMALL["mlra4_small"]
    a = W.make_workload(W.scaled(w, paging="contiguous"), device="cuda")
    b = dict(a)
    perm = torch.randperm(a["pool"].shape[0], generator=torch.Generator().manual_seed(3)).cuda()
    pool = torch.empty_like(a["pool"])
    pool[perm] = a["pool"]
    b["pool"] = pool
    pt = a["page_table"].long()
    b["page_table"] = torch.where(pt >= 0, perm[pt.clamp(min=0)], pt).to(torch.int32)
    hdl = G.make_handle(w, a)
    out_a, lse_a, _ = G.run_decode(hdl, a)
    out_b, lse_b, _ = G.run_decode(hdl, b)
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)


def test_block_independence_is_bit_exact():
    w = SMALL["mlra4_small"]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    base, _, _ = G.run_decode(hdl, inp)
    hb = w.h // w.k
    for j in range(w.k):
        pert = dict(inp)
        pert["pool"] = inp["pool"].clone()
        pert["pool"][..., j * w.d_b:(j + 1) * w.d_b] *= -1.5
        out, _, _ = G.run_decode(hdl, pert)
        changed = (out != base).flatten(2).any(-1).any(0).cpu()
        assert changed[j * hb:(j + 1) * hb].all()
        mask = torch.ones(w.h, dtype=torch.bool)
        mask[j * hb:(j + 1) * hb] = False
        assert not changed[mask].any()


def test_peaked_softmax_returns_one_token_exactly():
    """A query that singles out one token by a huge RoPE score makes the latent output equal
    that token's block (bf16 values, reproduced exactly in fp32)."""
    w = SMALL["mlra4_small"]
    inp = W.make_workload(W.scaled(w, seq_len=700, len_range=None), device="cuda")
    target = 517
    rows = W.logical_rows(inp, 1)
    q = inp["q"].clone()
    q[1, :, :w.d_h] = 0
    q[1, :, w.d_h:] = (rows[target, w.d_c:].float() * 64).to(q.dtype)
    inp["q"] = q
    hdl = G.make_handle(w, inp)
    lat, _, _ = G.run_decode(hdl, inp, latent=True)
    for hd in range(w.h):
        j = hd // (w.h // w.k)
        exp = rows[target, j * w.d_b:(j + 1) * w.d_b].float()
        assert torch.equal(lat[1, hd], exp), hd


def test_empty_and_single_token_sequences():
    w = W.scaled(SMALL["mlra4_small"], batch=4)
    lens = torch.tensor([0, 1, 129, 0], dtype=torch.int32)
    inp = W.make_workload(w, device="cuda", seq_lens=lens)
    hdl = G.make_handle(w, inp)
    out, lse, ws = G.run_decode(hdl, inp)
    assert M.mlra_get_status(ws) == 0
    assert torch.all(out[0] == 0) and torch.all(out[3] == 0)
    assert torch.all(torch.isneginf(lse[0])) and torch.all(torch.isneginf(lse[3]))
    ref = G.oracle_full(w, inp)
    G.assert_parity(out.cpu().numpy()[1:3], ref["out"][1:3], "single/short")


@pytest.mark.parametrize("batch", [257, 300])
def test_batches_past_the_warp_plan(batch):
    """Batches above 256 sequences take the block-wide planner in the decode and combine
    kernels (and two 128-row batch tiles plus a ragged third in the projections)."""
    w = W.scaled(SMALL["mlra4_small"], h=32, batch=batch, len_range=(0, 260), seed=60 + batch)
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    out, lse, ws = G.run_decode(hdl, inp)
    assert M.mlra_get_status(ws) == 0
    ref = G.oracle_full(w, inp)
    G.assert_parity(out.cpu().numpy(), ref["out"], f"batch {batch}")
    live = ref["lse"] > -1e300
    assert np.abs(lse.cpu().numpy()[live] - ref["lse"][live]).max() < G.TOL_LSE_ABS
    assert np.all(np.isneginf(lse.cpu().numpy()[~live]))


def test_page_id_out_of_range_is_reported():
    w = SMALL["mlra4_small"]
    inp = W.make_workload(w, device="cuda")
    inp["page_table"] = inp["page_table"].clone()
    inp["page_table"][0, 0] = inp["num_pages"] + 5
    hdl = G.make_handle(w, inp)
    _, _, ws = G.run_decode(hdl, inp)
    assert M.mlra_get_status(ws) == -4
    # the context is still usable and a clean call resets the status
    inp2 = W.make_workload(w, device="cuda")
    _, _, ws2 = G.run_decode(hdl, inp2, workspace=ws)
    assert M.mlra_get_status(ws2) == 0


def test_append_cache_rounds_and_places_rows():
    w = SMALL["tiny_full"]
    inp = W.make_workload(w, device="cuda", keep_f32=True)
    hdl = G.make_handle(w, inp)
    pool = torch.zeros_like(inp["pool"])
    n = int(inp["seq_lens"][0])
    pos = torch.arange(n, dtype=torch.int32, device="cuda")
    ids = torch.zeros(n, dtype=torch.int32, device="cuda")
    rows32 = W.logical_rows({**inp, "pool": inp["pool_f32"]}, 0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.mlra_append_cache(hdl, pool, inp["page_table"], ids, pos, rows32[:, :w.d_c].contiguous(),
                        rows32[:, w.d_c:].contiguous(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = W.logical_rows({**inp, "pool": pool}, 0)
    assert torch.equal(got, rows32.to(torch.bfloat16))
    # a row aimed at a page outside the pool is skipped and reported
    bad_pt = inp["page_table"].clone()
    bad_pt[0, 0] = 10 ** 6
    M.mlra_append_cache(hdl, pool, bad_pt, ids[:1], pos[:1], rows32[:1, :w.d_c].contiguous(),
                        rows32[:1, w.d_c:].contiguous(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -4


def test_tiny_workload_with_fp32_inputs_against_unrounded_oracle():
    """The tiny workload's fp32 inputs: the library rounds them to bf16 (cache via append, q in
    the absorb kernel); the error against the oracle on the unrounded fp32 values stays within
    the bf16 bar as well."""
    w = SMALL["tiny_full"]
    inp = W.make_workload(w, device="cuda", keep_f32=True)
    hdl = G.make_handle(w, inp)
    out, _, _ = G.run_decode(hdl, inp)
    ref = O.decode(inp["q_f32"].double().cpu().numpy(), inp["w_uk_f32"].double().cpu().numpy(),
                   inp["w_uv_f32"].double().cpu().numpy(), inp["pool_f32"].double().cpu().numpy(),
                   inp["page_table"].cpu().numpy(), inp["seq_lens"].cpu().numpy(), w.k, w.d_r)
    G.assert_parity(out.cpu().numpy(), ref["out"], "tiny vs unrounded fp32 oracle")


# ------------------------------------------------------------------------------------------
# Full workload sizes, every output element against the oracle
# ------------------------------------------------------------------------------------------
FULL = [n for n in W.WORKLOADS if n != "mlra4_h8_b1_n256_f32" and not W.WORKLOADS[n].summed]


@pytest.mark.parametrize("name", FULL)
def test_full_size_every_element(name):
    """The benchmark's launch configuration on the whole workload: every (sequence, head, d)
    output and every lse against the oracle (computed one sequence per task in a process
    pool)."""
    from tests import oracle_pool
    w = W.WORKLOADS[name]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    out, lse, ws = G.run_decode(hdl, inp, out_dtype=torch.float32)
    assert M.mlra_get_status(ws) == 0
    ref_out, ref_lse = oracle_pool.oracle_workload(w, inp)
    e = G.assert_parity(out.cpu().numpy(), ref_out, f"{name} out")
    dl = np.abs(lse.cpu().numpy() - ref_lse)
    print(f"{name}: max_abs={e['max_abs']:.3e} mean_abs={e['mean_abs']:.3e} rel_rms={e['rel_rms']:.3e} "
          f"lse_max_abs={dl.max():.3e}")
    assert dl.max() < G.TOL_LSE_ABS


@pytest.mark.parametrize("where", [1, 2])
def test_bounded_wait_times_out_cleanly(where):
    """A decode with one wait made to run out after the given limit: (1) the decode kernel's
    producer withholds every CTA's first tile; (2) one absorb CTA other than the one that
    clears the status word never issues its MMA. Every role drains and leaves, the status word
    reads MLRA_ERR_TIMEOUT (the early error survives the clear), and the context stays usable
    for the next call."""
    import time
    w = SMALL["mlra4_small"]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    out = torch.zeros(w.batch, w.h, w.d_h, device="cuda")
    ws = M.alloc_workspace(hdl, w.batch)
    t0 = time.time()
    M.mlra_test_decode_stalled(hdl, inp["q"], inp["pool"], inp["page_table"], inp["seq_lens"], out, ws,
                               wait_limit_ns=2_000_000, where=where)
    torch.cuda.synchronize()
    assert M.mlra_get_status(ws) == -5  # MLRA_ERR_TIMEOUT
    assert time.time() - t0 < 10
    got, _, ws2 = G.run_decode(hdl, inp)
    assert M.mlra_get_status(ws2) == 0
    G.assert_parity(got.cpu().numpy(), G.oracle_full(w, inp)["out"], "decode after a timed-out call")
