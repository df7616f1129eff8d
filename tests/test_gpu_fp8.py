"""GPU parity for decode over an E4M3 (FP8) latent cache through the C ABI, against the float64
oracle on the dequantized cache (``oracle/fp8_cache_oracle.py``).

The E4M3 kernels carry the query and P each as two E4M3 terms (about 7 significant bits, close
to bf16's 8), so the bf16 path's bar applies: max-abs 2e-2, mean-abs 2e-3, relative RMS 1e-2,
lse max-abs 2e-2. Writes into the cache (append, new rows) are bit-exact against the oracle's
encoder where the value to encode is the same on both sides.
"""
import numpy as np
import pytest
import torch

import rank_latent_kv_mlra_b200 as M
import workloads as W
from oracle import fp8_cache_oracle as F
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

FULL = W.WORKLOADS["mlra4fp8_h128_b32_n8192"]
SMALL = {
    "fp8_small": W.scaled(FULL, batch=3, seq_len=None, len_range=(1, 1500), seed=81),
    "fp8_ragged": W.scaled(FULL, batch=9, seq_len=None, len_range=(1, 3000), seed=82),
    "fp8_batch300": W.scaled(FULL, batch=300, seq_len=None, len_range=(0, 400), seed=83),
}


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    M.load_library()


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_fp8_output_matches_oracle(name, out_dtype):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    out, lse, ws = G.run_decode(hdl, inp, out_dtype=out_dtype)
    assert M.mlra_get_status(ws) == 0
    ref = G.oracle_full(w, inp)
    G.assert_parity(out.float().cpu().numpy(), ref["out"], f"{name} out ({out_dtype})")
    got_l = lse.cpu().numpy()
    live = np.isfinite(ref["lse"])
    assert np.array_equal(np.isneginf(got_l), ~live)
    assert np.abs(got_l[live] - ref["lse"][live]).max() < G.TOL_LSE_ABS


def test_fp8_latent_matches_oracle():
    w = SMALL["fp8_ragged"]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    lat, _, ws = G.run_decode(hdl, inp, latent=True)
    assert M.mlra_get_status(ws) == 0
    G.assert_parity(lat.cpu().numpy(), G.oracle_full(w, inp)["latent"], "fp8 latent")


def test_fp8_peaked_scores():
    """Queries times 8: a few tokens dominate, so the running maximum is raised often."""
    w = SMALL["fp8_small"]
    inp = W.make_workload(w, device="cuda")
    inp["q"] = (inp["q"].float() * 8).to(torch.bfloat16)
    hdl = G.make_handle(w, inp)
    out, _, ws = G.run_decode(hdl, inp)
    assert M.mlra_get_status(ws) == 0
    G.assert_parity(out.cpu().numpy(), G.oracle_full(w, inp)["out"], "fp8 peaked")


def test_fp8_plan_is_bit_exact():
    from oracle import mlra_oracle as O
    w = SMALL["fp8_small"]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    info = M.mlra_get_info(hdl)
    rng = np.random.default_rng(84)
    for lens in ([8192] * 32, list(rng.integers(0, 40000, 100)), list(rng.integers(0, 300, 257))):
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        got, n = M.mlra_plan(hdl, sl, pt_stride=1024)
        exp = O.plan_segments(lens, info["groups"])
        assert n == len(exp) and got == [tuple(s) for s in exp]


def test_fp8_full_size_every_element():
    from tests import oracle_pool
    w = FULL
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    out, lse, ws = G.run_decode(hdl, inp)
    assert M.mlra_get_status(ws) == 0
    ref_out, ref_lse = oracle_pool.oracle_workload(w, inp, e4m3_scales=(W.E4M3_SCALE, W.E4M3_SCALE))
    e = G.assert_parity(out.cpu().numpy(), ref_out, f"{w.name} out")
    dl = np.abs(lse.cpu().numpy() - ref_lse)
    print(f"{w.name}: max_abs={e['max_abs']:.3e} mean_abs={e['mean_abs']:.3e} rel_rms={e['rel_rms']:.3e} "
          f"lse_max_abs={dl.max():.3e}")
    assert dl.max() < G.TOL_LSE_ABS


@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
def test_fp8_append_is_bit_exact(in_dtype):
    """New rows are stored as the oracle's encoder stores them (power-of-two scales, so v / scale
    is exact on both sides), into their slots only; out-of-range values saturate."""
    w = SMALL["fp8_small"]
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    pool = inp["pool"].clone()
    rng = np.random.default_rng(85)
    B = w.batch
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    pos = torch.tensor([int(rng.integers(0, int(n))) for n in inp["seq_lens"].tolist()], dtype=torch.int32,
                       device="cuda")
    rows = torch.from_numpy(rng.standard_normal((B, w.d_c + w.d_r)).astype(np.float32) * 3)
    rows[0, :4] = torch.tensor([1e4, -1e4, 20.0, -0.0])  # saturation, a tie region, signed zero
    rows = rows.to(in_dtype).cuda()
    before = pool.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.mlra_append_cache(hdl, pool, inp["page_table"], ids, pos, rows[:, :w.d_c].contiguous(),
                        rows[:, w.d_c:].contiguous(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    exp = F.quantize_rows(rows.double().cpu().numpy(), w.d_c, W.E4M3_SCALE, W.E4M3_SCALE)
    pt = inp["page_table"].cpu().numpy()
    got = pool.cpu().numpy()
    mask = np.ones(got.shape[:2], dtype=bool)
    for b in range(B):
        p_ = int(pos[b])
        page, slot = pt[b, p_ // 64], p_ % 64
        assert np.array_equal(got[page, slot], exp[b]), b
        mask[page, slot] = False
    assert np.array_equal(got[mask], before.cpu().numpy()[mask])
