"""Helpers shared by the GPU tests: run the library on a workload, read its workspace, and
compare against the float64 oracle. Nothing here computes attention on the GPU side; the
oracle side is ``oracle/``.
"""
import math

import numpy as np
import torch

import rank_latent_kv_mlra_b200 as M
import workloads as W
from oracle import mlra_oracle as O

# Parity bar for bf16 cache / fp32 accumulate outputs (elementwise against the oracle).
TOL_MAX_ABS = 2e-2
TOL_MEAN_ABS = 2e-3
TOL_REL_RMS = 1e-2     # ||gpu - oracle||_2 / ||oracle||_2
TOL_LSE_ABS = 2e-2


def make_handle(w: W.Workload, inputs: dict):
    fp8 = dict(cache_fp8=True, latent_scale=W.E4M3_SCALE, rope_scale=W.E4M3_SCALE) if w.cache == "e4m3" else {}
    return M.mlra_create(w.h, w.d_h, w.d_c, w.d_r, w.k, inputs["w_uk"], inputs["w_uv"], **fp8)


def run_decode(handle, inputs: dict, out_dtype=torch.float32, latent=False, workspace=None):
    q = inputs["q"]
    B, h = q.shape[0], q.shape[1]
    cfg = handle.cfg
    lse = torch.full((B, h), float("nan"), device=q.device)
    if latent:
        out = torch.full((B, h, cfg.d_c // cfg.k), float("nan"), device=q.device)
        ws = M.mlra_decode_latent(handle, q, inputs["pool"], inputs["page_table"], inputs["seq_lens"],
                                  out, lse, workspace=workspace)
    else:
        out = torch.full((B, h, cfg.d_h), float("nan"), device=q.device, dtype=out_dtype)
        ws = M.mlra_decode(handle, q, inputs["pool"], inputs["page_table"], inputs["seq_lens"], out, lse,
                           workspace=workspace)
    torch.cuda.synchronize()
    return out, lse, ws


def workspace_views(handle, ws: torch.Tensor, batch: int):
    """Views of the decode workspace (layout of mlra_api.cu's carve())."""
    info = M.mlra_get_info(handle)
    cfg = handle.cfg
    d_b = cfg.d_c // cfg.k
    np_ = info["heads_per_cta"]
    nsub = info["ctas_per_group"]
    a = lambda x: (x + 255) // 256 * 256
    off = 256
    qb = batch * nsub * np_ * (d_b + cfg.d_rope) * 2
    q_pack = ws[off:off + qb].view(torch.bfloat16).view(batch, nsub, np_, d_b + cfg.d_rope)
    off += a(qb)
    slots = batch + info["groups"]
    ob = slots * cfg.h * d_b * 4
    o_part = ws[off:off + ob].view(torch.float32).view(slots, cfg.h, d_b)
    off += a(ob)
    lb = slots * cfg.h * 4
    lse_part = ws[off:off + lb].view(torch.float32).view(slots, cfg.h)
    return {"status": ws[:4].view(torch.int32), "q_pack": q_pack, "o_part": o_part, "lse_part": lse_part,
            "info": info}


def oracle_full(w: W.Workload, inputs: dict):
    """Oracle on the exact values the GPU reads (bf16-rounded cache and weights, or the E4M3
    cache's bytes; q as given)."""
    args = (inputs["q"].double().cpu().numpy(), inputs["w_uk"].double().cpu().numpy(),
            inputs["w_uv"].double().cpu().numpy())
    rest = (inputs["page_table"].cpu().numpy(), inputs["seq_lens"].cpu().numpy(), w.k, w.d_r)
    if w.cache == "e4m3":
        from oracle import fp8_cache_oracle as F
        return F.decode_fp8(*args, inputs["pool"].cpu().numpy(), *rest, W.E4M3_SCALE, W.E4M3_SCALE)
    return O.decode(*args, inputs["pool"].float().cpu().numpy(), *rest)


def errors(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(got - ref)
    return {
        "max_abs": float(d.max()) if d.size else 0.0,
        "mean_abs": float(d.mean()) if d.size else 0.0,
        "rel_rms": float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)),
        "nan": int(np.isnan(got).sum()),
    }


def assert_parity(got, ref, what: str, tol_max=TOL_MAX_ABS, tol_mean=TOL_MEAN_ABS, tol_rel=TOL_REL_RMS):
    e = errors(got, ref)
    ok = e["nan"] == 0 and e["max_abs"] <= tol_max and e["mean_abs"] <= tol_mean and e["rel_rms"] <= tol_rel
    assert ok, f"{what}: {e}"
    return e


def expected_q_pack(w: W.Workload, inputs: dict, np_: int, nsub: int, scale: float):
    """Absorbed query as the decode kernel expects it, from a float64 oracle product."""
    q = inputs["q"].double().cpu()
    wuk = inputs["w_uk"].double().cpu()
    B, h = q.shape[0], q.shape[1]
    hb = h // w.k
    chunks = nsub // w.k
    alpha = scale * math.log2(math.e)
    out = torch.zeros(B, nsub, np_, w.d_b + w.d_r, dtype=torch.float64)
    for hd in range(h):
        j, r = divmod(hd, hb)
        sub, row = j * chunks + r // np_, r % np_
        out[:, sub, row, :w.d_b] = alpha * torch.einsum("cd,bd->bc", wuk[hd], q[:, hd, :w.d_h])
        out[:, sub, row, w.d_b:] = alpha * q[:, hd, w.d_h:]
    return out


def sampled_heads(w: W.Workload, inputs: dict, pairs, rows_cache=None):
    """Oracle (out, latent, lse) for sampled (b, head) pairs, one sequence at a time."""
    res = {}
    by_b = {}
    for b, hd in pairs:
        by_b.setdefault(b, []).append(hd)
    q = inputs["q"].double().cpu().numpy()
    wuk = inputs["w_uk"].double().cpu().numpy()
    wuv = inputs["w_uv"].double().cpu().numpy()
    pt = inputs["page_table"].cpu().numpy()
    for b, heads in by_b.items():
        n = int(inputs["seq_lens"][b])
        # rows of sequence b only, gathered by the oracle's own page walk on a host copy of the
        # pages this sequence uses
        pages = pt[b, :(n + 63) // 64]
        sub_pool = inputs["pool"][torch.as_tensor(pages, device=inputs["pool"].device).long()].float().cpu().numpy()
        local_pt = np.arange(len(pages))[None, :]
        rows = O.gather_rows(sub_pool, local_pt, 0, n)
        o, lat, lse = O.decode_heads(q[b], wuk, wuv, rows, heads, w.k, w.d_r)
        for i, hd in enumerate(heads):
            res[(b, hd)] = (o[i], lat[i], lse[i])
    return res
