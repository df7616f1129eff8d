"""GPU parity for the summed-blocks reading (every head attends to every latent block, per-block
softmax, outputs summed times alpha_attn) through the C ABI, against the float64 oracle's
``decode_summed``. Reduced and full sizes (MLRA-4: batch 32, context 8192; MLRA-2: batch 64,
context 4096; h = 128) compare every element."""
import numpy as np
import pytest
import torch

import rank_latent_kv_mlra_b200 as M
import workloads as W
from oracle import mlra_oracle as O
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

FULL = W.WORKLOADS["mlra4sum_h128_b32_n8192"]
SMALL = {
    "mlra4sum_small": W.scaled(FULL, batch=3, seq_len=None, len_range=(1, 1500), seed=31),
    "mlra2sum_small": W.scaled(W.WORKLOADS["mlra2sum_h128_b64_n4096"], batch=3, seq_len=None,
                               len_range=(1, 1300), seed=33),
    "tiny_summed": W.scaled(W.WORKLOADS["mlra4_h8_b1_n256_f32"], summed=True, batch=2, seq_len=None,
                            len_range=(100, 300), seed=32),
}


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    M.load_library()


def _handle(w, inp, attn_scale=0.0):
    return M.mlra_create(w.h, w.d_h, w.d_c, w.d_r, w.k, inp["w_uk"], inp["w_uv"], blocks_summed=True,
                         attn_scale=attn_scale)


def _oracle(w, inp, attn_scale=None):
    return O.decode_summed(inp["q"].double().cpu().numpy(), inp["w_uk"].double().cpu().numpy(),
                           inp["w_uv"].double().cpu().numpy(), inp["pool"].float().cpu().numpy(),
                           inp["page_table"].cpu().numpy(), inp["seq_lens"].cpu().numpy(), w.k, w.d_r,
                           attn_scale=attn_scale)


def _run(hdl, w, inp, out_dtype=torch.float32):
    out = torch.full((w.batch, w.h, w.d_h), float("nan"), device="cuda", dtype=out_dtype)
    lse = torch.full((w.batch, w.k * w.h), float("nan"), device="cuda")
    ws = M.mlra_decode(hdl, inp["q"], inp["pool"], inp["page_table"], inp["seq_lens"], out, lse)
    torch.cuda.synchronize()
    assert M.mlra_get_status(ws) == 0
    return out, lse


def _lse_check(lse_gpu, lse_ref, w):
    got = lse_gpu.cpu().numpy().reshape(w.batch, w.k, w.h)
    live = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(got), ~live)
    assert np.abs(got[live] - lse_ref[live]).max() < G.TOL_LSE_ABS


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_summed_output_matches_oracle(name, out_dtype):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    out, lse = _run(_handle(w, inp), w, inp, out_dtype)
    ref = _oracle(w, inp)
    G.assert_parity(out.float().cpu().numpy(), ref["out"], f"{name} out ({out_dtype})")
    _lse_check(lse, ref["lse"], w)


@pytest.mark.parametrize("name", ["mlra4sum_small", "mlra2sum_small"])
def test_summed_attn_scale_is_applied(name):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    out, _ = _run(_handle(w, inp, attn_scale=0.6), w, inp)
    G.assert_parity(out.cpu().numpy(), _oracle(w, inp, attn_scale=0.6)["out"], "alpha_attn 0.6")


@pytest.mark.parametrize("name", ["mlra4sum_small", "mlra2sum_small"])
def test_summed_latent_per_block_matches_oracle(name):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    hdl = _handle(w, inp)
    lat = torch.full((w.batch, w.k * w.h, w.d_b), float("nan"), device="cuda")
    lse = torch.full((w.batch, w.k * w.h), float("nan"), device="cuda")
    ws = M.mlra_decode_latent(hdl, inp["q"], inp["pool"], inp["page_table"], inp["seq_lens"], lat, lse)
    torch.cuda.synchronize()
    assert M.mlra_get_status(ws) == 0
    ref = _oracle(w, inp)
    G.assert_parity(lat.cpu().numpy().reshape(w.batch, w.k, w.h, w.d_b), ref["latent"], "summed latent")
    _lse_check(lse, ref["lse"], w)


@pytest.mark.parametrize("name", ["mlra4sum_small", "mlra2sum_small"])
def test_summed_plan_is_bit_exact(name):
    w = SMALL[name]
    inp = W.make_workload(w, device="cuda")
    hdl = _handle(w, inp)
    info = M.mlra_get_info(hdl)
    per = info["ctas_per_group"]
    assert per == w.k * (w.h // info["heads_per_cta"]) and info["groups"] == info["num_sms"] // per
    rng = np.random.default_rng(8)
    for lens in (inp["seq_lens"].cpu().tolist(), [8192] * 32, list(rng.integers(0, 40000, 100))):
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        got, n = M.mlra_plan(hdl, sl, pt_stride=1024)
        exp = O.plan_segments(lens, info["groups"])
        assert n == len(exp) and got == [tuple(s) for s in exp]


@pytest.mark.parametrize("name", ["mlra4sum_h128_b32_n8192", "mlra2sum_h128_b64_n4096"])
def test_summed_full_size_every_element(name):
    """Full size, every output element and every per-block lse against the oracle."""
    from tests import oracle_pool
    w = W.WORKLOADS[name]
    inp = W.make_workload(w, device="cuda")
    out, lse = _run(_handle(w, inp), w, inp)
    ref_out, ref_lse = oracle_pool.oracle_workload(w, inp)
    e = G.assert_parity(out.cpu().numpy(), ref_out, f"{name} out")
    dl = np.abs(lse.cpu().numpy().reshape(w.batch, w.k, w.h) - ref_lse)
    print(f"{name}: max_abs={e['max_abs']:.3e} mean_abs={e['mean_abs']:.3e} rel_rms={e['rel_rms']:.3e} "
          f"lse_max_abs={dl.max():.3e}")
    assert dl.max() < G.TOL_LSE_ABS
