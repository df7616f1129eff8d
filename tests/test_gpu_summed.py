"""GPU parity for the summed-blocks reading (every head attends to every latent block, per-block
softmax, outputs summed times alpha_attn) through the C ABI, against the float64 oracle's
``decode_summed``. Reduced sizes compare every element; the full-size workload (h = 128, batch 32, context 8192)
compares sampled heads."""
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


def test_summed_attn_scale_is_applied():
    w = SMALL["mlra4sum_small"]
    inp = W.make_workload(w, device="cuda")
    out, _ = _run(_handle(w, inp, attn_scale=0.6), w, inp)
    G.assert_parity(out.cpu().numpy(), _oracle(w, inp, attn_scale=0.6)["out"], "alpha_attn 0.6")


def test_summed_latent_per_block_matches_oracle():
    w = SMALL["mlra4sum_small"]
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


def test_summed_plan_is_bit_exact():
    w = SMALL["mlra4sum_small"]
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


def test_summed_full_size_sampled():
    w = FULL
    inp = W.make_workload(w, device="cuda")
    out, lse = _run(_handle(w, inp), w, inp)
    assert not torch.isnan(out).any()
    rng = np.random.default_rng(17)
    bs = sorted(set([0, w.batch - 1] + list(rng.integers(0, w.batch, 2))))
    heads = sorted(set([0, w.h - 1] + list(rng.integers(0, w.h, 5))))
    q = inp["q"].double().cpu().numpy()
    wuk = inp["w_uk"].double().cpu().numpy()
    wuv = inp["w_uv"].double().cpu().numpy()
    lse_np = lse.cpu().numpy().reshape(w.batch, w.k, w.h)
    for b in bs:
        rows = W.logical_rows(inp, b).double().cpu().numpy()
        o_ref, l_ref = O.decode_summed_heads(q[b], wuk, wuv, rows, heads, w.k, w.d_r)
        G.assert_parity(np.stack([out[b, hd].cpu().numpy() for hd in heads]), o_ref, f"seq {b} sampled")
        assert np.abs(lse_np[b][:, heads].T - l_ref).max() < G.TOL_LSE_ABS
