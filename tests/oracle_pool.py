"""Whole-workload oracle results for the full-size GPU parity tests.

The float64 oracle (``oracle/``) runs one sequence per task in a pool of worker processes.
Workers are started with ``spawn`` (a worker forked from a process that has used CUDA can
hang), get the query and weights once through the pool initializer, and receive each
sequence's pages as raw bf16 bits; they gather the sequence's rows with the oracle's own
page walk over those pages and call the oracle's per-sequence form. Nothing here computes
attention itself.
"""
import contextlib
import multiprocessing as mp
import os

import numpy as np

_G = {}


def _bf16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: a bf16 is the top half of an fp32)."""
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _init(q, w_uk, w_uv, k, d_r, summed, e4m3_scales):
    _G.update(q=q, w_uk=w_uk, w_uv=w_uv, k=k, d_r=d_r, summed=summed, e4m3_scales=e4m3_scales)


def _task(args):
    from oracle import mlra_oracle as O
    b, pages, n = args
    if _G["e4m3_scales"] is not None:  # E4M3 bytes, dequantized by the FP8-cache oracle
        from oracle import fp8_cache_oracle as F
        ls, rs = _G["e4m3_scales"]
        pool = F.dequantize_pool(pages, pages.shape[-1] - _G["d_r"], ls, rs)
    else:
        pool = _bf16_bits_to_f64(pages)
    rows = O.gather_rows(pool, np.arange(pool.shape[0])[None, :], 0, n)
    if _G["summed"]:
        out, lse = O.decode_summed_sequence(_G["q"][b], _G["w_uk"], _G["w_uv"], rows, _G["k"], _G["d_r"])
    else:
        out, _, lse = O.decode_sequence(_G["q"][b], _G["w_uk"], _G["w_uv"], rows, _G["k"], _G["d_r"])
    return b, out, lse


@contextlib.contextmanager
def _single_threaded_blas():
    keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
    old = {key: os.environ.get(key) for key in keys}
    for key in keys:
        os.environ[key] = "1"
    try:
        yield
    finally:
        for key, v in old.items():
            if v is None:
                os.environ.pop(key, None)
            else:
                os.environ[key] = v


def oracle_workload(w, inputs, workers=None, e4m3_scales=None):
    """Oracle (out [B][h][d_h], lse) for every sequence and head of workload ``w`` (lse is
    [B][h], or [B][k][h] for the summed reading), on the exact values the GPU reads (bf16, or
    E4M3 bytes with the (latent, RoPE) scales ``e4m3_scales``)."""
    import torch  # the parent holds the inputs as torch tensors (possibly on the GPU)
    if e4m3_scales is None and getattr(w, "cache", "bf16") == "e4m3":
        import workloads
        e4m3_scales = (workloads.E4M3_SCALE, workloads.E4M3_SCALE)
    q = inputs["q"].double().cpu().numpy()
    w_uk = inputs["w_uk"].double().cpu().numpy()
    w_uv = inputs["w_uv"].double().cpu().numpy()
    lens = inputs["seq_lens"].cpu().numpy()
    pt = inputs["page_table"]
    pool = inputs["pool"]
    B, h = q.shape[:2]
    d_h = q.shape[2] - w.d_r

    def tasks():
        for b in range(B):
            n = int(lens[b])
            npg = (n + 63) // 64
            idx = pt[b, :npg].long()
            if pool.dtype == torch.uint8:
                pages = pool[idx].contiguous().cpu().numpy()
            else:
                pages = pool[idx].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
            yield b, pages, n

    out = np.zeros((B, h, d_h))
    lse = np.full((B, w.k, h) if w.summed else (B, h), -np.inf)
    workers = workers or max(1, min(16, os.cpu_count() or 1))
    ctx = mp.get_context("spawn")
    with _single_threaded_blas():
        pool_proc = ctx.Pool(workers, initializer=_init,
                             initargs=(q, w_uk, w_uv, w.k, w.d_r, w.summed, e4m3_scales))
    try:
        for b, o, l in pool_proc.imap_unordered(_task, tasks(), chunksize=1):
            out[b] = o
            lse[b] = l
    finally:
        pool_proc.close()
        pool_proc.join()
    return out, lse
