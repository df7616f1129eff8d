"""Benchmark of one MLRA decode step (query absorption, split-KV latent attention, log-sum-exp
combine + W^UV up-projection) on the MLRA-4 workload h=128, d_h=128, d_c=512 (4 blocks of
128), d_r=64, batch 32, context 8192, bf16 paged cache (64-token pages, seeded permutation).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Prints one JSON line. The metric is the latent-cache stream rate of a whole decode step:
cache bytes of the step / step time (GB/s), with the step time in ms_per_step. Under
torchrun (N > 1) every rank runs its own replica of the workload (weak scaling; the path
has no data exchange) and rank 0 reports the total over ranks / the slowest rank's time.

`--impl reference` times the float64 oracle (oracle/) on this host's cores: each step is a
bounded sample of the same workload (a few (sequence, head) pairs), scaled to the metric by
the fraction of the workload it covers.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MLRA-4 decode attn: achieved HBM GB/s (% of peak), µs/step at B=32, n=8192"
UNIT = "GB/s"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


def cache_bytes(w: W.Workload, seq_lens) -> int:
    """Algorithmic bytes of the latent-cache stream of one step: each cached token's row
    [c | k^R] read once (2 bytes per element in bf16, 1 in E4M3) plus one 4-byte page-table
    entry per 64 tokens."""
    toks = int(sum(int(n) for n in seq_lens))
    pages = int(sum((int(n) + 63) // 64 for n in seq_lens))
    return toks * (w.d_c + w.d_r) * (1 if w.cache == "e4m3" else 2) + pages * 4


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_peak():
    """Dense bf16 tensor peak (burst figure: the decode kernel is timed on its own)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def decode_flops(w, seq_lens):
    """Algorithmic FLOPs of the decode kernel: per cached token and per (virtual) head, the
    score over d_b + d_r columns and the P.C accumulation over d_b, 2 FLOPs per MAC. A head
    sees one block (partitioned) or all k blocks (summed)."""
    d_b = w.d_c // w.k
    heads = w.h * w.k if w.summed else w.h
    return float(sum(int(n) for n in seq_lens)) * heads * (2 * (d_b + w.d_r) + 2 * d_b)


def decode_shape_name(w):
    """The decode kernel shape (`using Dec...` in mlra_api.cu) a workload runs on."""
    d_b = w.d_c // w.k
    if w.cache == "e4m3":
        return "DecMlra4F8"
    if d_b == 32:
        return "DecTiny"
    if d_b == 128:
        return "DecMlra4Sum" if w.summed else "DecMlra4"
    if d_b == 256:
        return "DecMlra2"
    return "DecMla"


def kernel_source_hash(w):
    """Hash of the decode kernel code workload `w` runs: common.cuh, decode.cuh and the line of
    mlra_api.cu that fixes its shape (comments and blank lines left out, so a comment edit or
    another shape's change does not invalidate a recorded ncu capture)."""
    h = hashlib.sha256()
    shape = decode_shape_name(w)
    for f in ["common.cuh", "decode.cuh", "mlra_api.cu"]:
        with open(os.path.join(ROOT, "rank_latent_kv_mlra_b200", "csrc", f), encoding="utf-8") as fh:
            for line in fh:
                code = line.split("//", 1)[0].rstrip()
                if code and (f != "mlra_api.cu" or code.startswith(f"using {shape} ")):
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic(workload_name):
    """DRAM bytes per launch of the decode kernel from a committed ncu summary, if the code of
    the kernel the workload runs has not changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    ent = rec.get("workloads", {}).get(workload_name)
    if ent is None or ent.get("kernel_source_hash") != kernel_source_hash(W.WORKLOADS[workload_name]):
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons sampled during the measured legs.

    Read-only NVML queries from a background thread every ~1 ms (the decode step takes tens of
    microseconds, so the sampler runs from the first warm-up step to the end of the profiled
    leg, and `under_load` counts the samples taken while the GPU was not idle); `nvidia-smi
    -lms 100` in a subprocess is the fallback when NVML cannot be loaded."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device):
        self.device = torch.device(device)
        self.samples = []
        self.max_mhz = None
        self.thread = None
        self.stop_flag = False
        self.smi = None

    def _nvml_handle(self):
        """The NVML handle of this process's CUDA device, matched by UUID (NVML enumerates
        every GPU of the machine, whatever CUDA_VISIBLE_DEVICES hides)."""
        import pynvml
        pynvml.nvmlInit()
        want = str(torch.cuda.get_device_properties(self.device).uuid).lower().replace("gpu-", "")
        for i in range(pynvml.nvmlDeviceGetCount()):
            h = pynvml.nvmlDeviceGetHandleByIndex(i)
            u = pynvml.nvmlDeviceGetUUID(h)
            u = (u.decode() if isinstance(u, bytes) else str(u)).lower().replace("gpu-", "")
            if u == want:
                return pynvml, h
        raise RuntimeError("no NVML device with this CUDA device's UUID")

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
        except Exception:
            self._start_smi()
            return
        self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        bits = {name: getattr(nv, attr) for name, attr in self.REASONS}
        idle = nv.nvmlClocksEventReasonGpuIdle

        def run():
            while not self.stop_flag:
                try:
                    mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    r = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                    self.samples.append((mhz, r & idle != 0, [n for n, b in bits.items() if r & b]))
                except Exception:
                    pass
                time.sleep(0.001)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def _start_smi(self):
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.gpu_idle,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        try:
            self.fh = tempfile.TemporaryFile(mode="w+")
            idx = self.device.index or 0
            self.smi = subprocess.Popen(["nvidia-smi", f"--id={idx}", f"--query-gpu={fields}",
                                         "--format=csv,noheader,nounits", "-lms", "100"],
                                        stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.smi = None

    def _stop_smi(self):
        self.smi.terminate()
        try:
            self.smi.wait(timeout=5)
        except Exception:
            self.smi.kill()
        self.fh.seek(0)
        names = [n for n, _ in self.REASONS]
        for line in self.fh:
            p = [x.strip() for x in line.split(",")]
            if len(p) < 7:
                continue
            try:
                mhz, self.max_mhz = float(p[0]), float(p[1])
            except ValueError:
                continue
            self.samples.append((mhz, p[2].lower() == "active",
                                 [n for n, v in zip(names, p[3:7]) if v.lower() == "active"]))

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
        elif self.smi is not None:
            self._stop_smi()
        else:
            return None
        if not self.samples:
            return None
        load = [s for s in self.samples if not s[1]] or self.samples
        reasons = sorted({r for s in load for r in s[2]})
        return {"sm_mhz": statistics.median(s[0] for s in load), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "samples_under_load": len(load),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


def config_of(w, world, nbytes):
    """The workload description both arms print (identical keys, so the lines compare)."""
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seq_len,
            "len_range": list(w.len_range) if w.len_range else None, "h": w.h, "d_h": w.d_h,
            "d_c": w.d_c, "d_r": w.d_r, "k": w.k, "page_size": 64, "paging": w.paging,
            "reading": "summed" if w.summed else "partitioned", "cache": w.cache, "l2": "inputs larger than L2",
            "parallelism": f"replicas{world}", "cache_bytes_per_step": nbytes}


def dist_setup(impl):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if impl == "ours" else "gloo"
        if impl == "ours":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------------------
# float64 oracle on host cores
# ---------------------------------------------------------------------------------------

def oracle_sample_rate(w, inp, pairs_per_step, steps, warmup):
    """Times the oracle as it stands on (sequence, head) pairs of the workload; returns
    (GB/s-equivalent, seconds per step, threads)."""
    from oracle import mlra_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        threads = 1
    seq_lens = inp["seq_lens"].cpu().numpy()
    q = inp["q"].double().cpu().numpy()
    wuk = inp["w_uk"].double().cpu().numpy()
    wuv = inp["w_uv"].double().cpu().numpy()
    pt = inp["page_table"].cpu().numpy()
    rng = np.random.default_rng(0)
    total_heads = w.batch * w.h
    full_bytes = cache_bytes(w, seq_lens)
    sub_pools = {}

    def rows_of(b):
        if b not in sub_pools:
            n = int(seq_lens[b])
            pages = pt[b, :(n + 63) // 64]
            sp = inp["pool"][torch.as_tensor(pages, device=inp["pool"].device).long()]
            if w.cache == "e4m3":
                from oracle import fp8_cache_oracle as F
                sp = F.dequantize_pool(sp.cpu().numpy(), w.d_c, W.E4M3_SCALE, W.E4M3_SCALE)
            else:
                sp = sp.float().cpu().numpy()
            sub_pools[b] = O.gather_rows(sp, np.arange(len(pages))[None, :], 0, n)
        return sub_pools[b]

    def step():
        for _ in range(pairs_per_step):
            b = int(rng.integers(0, w.batch))
            hd = int(rng.integers(0, w.h))
            if w.summed:
                O.decode_summed_heads(q[b], wuk, wuv, rows_of(b), [hd], w.k, w.d_r)
            else:
                O.decode_heads(q[b], wuk, wuv, rows_of(b), [hd], w.k, w.d_r)

    for _ in range(warmup):
        step()
    # gathering rows is the oracle's page walk; it is timed too, per sequence first seen
    sub_pools.clear()
    t0, c0 = time.perf_counter(), time.process_time()
    for _ in range(steps):
        step()
    dt, cpu = time.perf_counter() - t0, time.process_time() - c0
    bytes_done = full_bytes * (pairs_per_step * steps) / total_heads
    # threads the oracle actually kept busy: process CPU time over wall time (its BLAS pool may
    # be larger, but one small matrix-vector product at a time leaves most of it idle)
    cores = round(max(1.0, cpu / dt), 1)
    return bytes_done / dt / 1e9, dt / steps, cores, threads


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = W.make_workload(w, device=dev)
    rate, sec_per_step, cores, pool_threads = oracle_sample_rate(w, inp, 1, args.steps, args.warmup)
    nbytes = cache_bytes(w, inp["seq_lens"].cpu().tolist())
    line = {
        "impl": "reference",
        "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec_per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world, nbytes),
        "cpu_baseline": {"value": rate, "unit": UNIT, "cores": cores, "blas_pool_threads": pool_threads,
                         "kind": "oracle",
                         "sample": "each step: the float64 oracle on one random (sequence, head) pair "
                                   f"of the {w.name} workload; value scaled by the fraction of the "
                                   "workload's heads covered; cores = process CPU time / wall time"},
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------
# our CUDA path
# ---------------------------------------------------------------------------------------

# the other benchmark configurations, timed in the same run as the headline (decode step and
# kernels); each is a fresh workload on the device
EXTRA_WORKLOADS = ["mlra2_h128_b64_n4096", "mlra4_h128_b8_n131072", "mlra4_h128_b128_ragged1k_32k",
                   "mla_h128_b128_ragged1k_32k", "mlra4sum_h128_b32_n8192", "mlra2sum_h128_b64_n4096",
                   "mlra4fp8_h128_b32_n8192"]


def make_handle(M, w, inp):
    fp8 = dict(cache_fp8=True, latent_scale=W.E4M3_SCALE, rope_scale=W.E4M3_SCALE) if w.cache == "e4m3" else {}
    return M.mlra_create(w.h, w.d_h, w.d_c, w.d_r, w.k, inp["w_uk"], inp["w_uv"], blocks_summed=w.summed, **fp8)


def time_decode(M, w, inp, hdl, dev, steps, warmup):
    """Whole-step time (CUDA events around `steps` back-to-back calls, kernels chained by
    programmatic dependent launch) and per-kernel times (mlra_decode_profiled: events between
    the kernels, no overlap), after a status-checked call and `warmup` untimed steps."""
    out = torch.empty(w.batch, w.h, w.d_h, device=dev, dtype=torch.bfloat16)
    ws = M.alloc_workspace(hdl, w.batch, dev)
    stream = torch.cuda.current_stream(dev)
    args_dec = (hdl, inp["q"], inp["pool"], inp["page_table"], inp["seq_lens"], out)
    M.mlra_decode(*args_dec, workspace=ws)
    torch.cuda.synchronize()
    status = M.mlra_get_status(ws)
    if status != 0:
        raise RuntimeError(f"{w.name}: decode status {status}")
    for _ in range(warmup):
        M.mlra_decode(*args_dec, workspace=ws)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        M.mlra_decode(*args_dec, workspace=ws)
    ev1.record(stream)
    torch.cuda.synchronize()
    step_ms = ev0.elapsed_time(ev1) / steps
    kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        M.mlra_decode_profiled(*args_dec, kevs[i], workspace=ws)
    torch.cuda.synchronize()
    k_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in kevs) / steps for i in range(3)]
    return {"step_ms": step_ms, "k_ms": k_ms, "out": out, "ws": ws, "args": args_dec, "stream": stream}


def roofline_of(w, seq_lens, decode_ms):
    """Roofline of the decode kernel: HBM for the partitioned reading (below the ridge), the
    bf16 tensor peak for the summed one (k times the MMA work per cached byte)."""
    nbytes = cache_bytes(w, seq_lens)
    peak, peak_kind = measured_hbm_peak()
    tpeak, tpeak_kind = measured_bf16_peak()
    achieved = nbytes / (decode_ms * 1e-3) / 1e9
    flops = decode_flops(w, seq_lens)
    tflops = flops / (decode_ms * 1e-3) / 1e12
    if w.summed:
        return {"bound": "tensor", "achieved": tflops, "peak": tpeak, "unit": "TFLOP/s", "frac": tflops / tpeak,
                "peak_kind": f"{tpeak_kind} dense bf16 (burst)", "flops_per_launch": flops,
                "hbm_achieved_gbs": achieved, "hbm_frac": achieved / peak,
                "kernel": "mlra_decode_kernel (split-KV latent attention, summed blocks)",
                "traffic": recorded_traffic(w.name)}
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_kind": f"{peak_kind} copy bandwidth", "bytes_per_launch": nbytes,
            "tensor_tflops": tflops, "tensor_frac": tflops / tpeak,
            "kernel": "mlra_decode_kernel (split-KV latent attention)", "traffic": recorded_traffic(w.name)}


def run_ours(args, world, rank, local):
    import rank_latent_kv_mlra_b200 as M

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = W.WORKLOADS[args.workload]
    inp = W.make_workload(w, device=dev)
    hdl = make_handle(M, w, inp)
    B = w.batch
    seq_lens = inp["seq_lens"].cpu().tolist()
    nbytes = cache_bytes(w, seq_lens)

    clocks = ClockSampler(dev)
    clocks.start()
    barrier(world)
    r = time_decode(M, w, inp, hdl, dev, args.steps, args.warmup)
    barrier(world)
    step_ms, k_ms, out, ws, stream = r["step_ms"], r["k_ms"], r["out"], r["ws"], r["stream"]
    clk = clocks.stop()

    # End to end through the public API: every step uploads its query and lengths from pinned
    # host memory and reads its output back into pinned host memory, inside the timed region.
    # Steps are pipelined the way a serving loop runs them: uploads on one copy stream,
    # downloads on another and two device buffer sets, so the copies of one step overlap the
    # kernels of its neighbours (events order upload -> kernels -> download, and a buffer set is
    # reused only after the step that last used it has finished with it).
    NB = 2
    q_host = inp["q"].cpu().pin_memory()
    sl_host = inp["seq_lens"].cpu().pin_memory()
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(NB)]
    q_dev = [torch.empty_like(inp["q"]) for _ in range(NB)]
    sl_dev = [torch.empty_like(inp["seq_lens"]) for _ in range(NB)]
    outs = [torch.empty_like(out) for _ in range(NB)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(NB)]
    ev_dec = [torch.cuda.Event() for _ in range(NB)]
    ev_down = [torch.cuda.Event() for _ in range(NB)]

    def e2e_step(i, cur):
        k = i % NB
        with torch.cuda.stream(up):
            if i >= NB:
                up.wait_event(ev_dec[k])  # the kernels of step i - NB have read q_dev[k]
            q_dev[k].copy_(q_host, non_blocking=True)
            sl_dev[k].copy_(sl_host, non_blocking=True)
            ev_up[k].record(up)
        cur.wait_event(ev_up[k])
        if i >= NB:
            cur.wait_event(ev_down[k])  # step i - NB's output has been read back
        M.mlra_decode(hdl, q_dev[k], inp["pool"], inp["page_table"], sl_dev[k], outs[k], workspace=ws,
                      stream=cur)
        ev_dec[k].record(cur)
        with torch.cuda.stream(down):
            down.wait_event(ev_dec[k])
            out_host[k].copy_(outs[k], non_blocking=True)
            ev_down[k].record(down)

    def e2e_steps_on(cur, n):
        # fork the copy streams from `cur`, run n pipelined steps, join them back into `cur`
        fork = torch.cuda.Event()
        fork.record(cur)
        up.wait_event(fork)
        down.wait_event(fork)
        for i in range(n):
            e2e_step(i, cur)
        cur.wait_event(ev_up[(n - 1) % NB])
        cur.wait_event(ev_down[(n - 1) % NB])

    def e2e_run(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_steps_on(stream, n)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    e2e_run(max(3, args.warmup // 10))
    e2e_steps = max(10, args.steps // 4)
    e2e_ms = e2e_run(e2e_steps)
    # copy bandwidths alone, for reading the e2e figure (the uploads bound it when they take
    # longer than the kernels)
    def copy_gbs(dst, src, strm, n=20):
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(strm):
            c0.record(strm)
            for _ in range(n):
                dst.copy_(src, non_blocking=True)
            c1.record(strm)
        torch.cuda.synchronize()
        return n * src.numel() * src.element_size() / (c0.elapsed_time(c1) * 1e-3) / 1e9
    h2d_gbs = copy_gbs(q_dev[0], q_host, up)
    d2h_gbs = copy_gbs(out_host[0], outs[0], down)
    # the pipelined steps computed the same output as the plain call
    assert torch.equal(out_host[(e2e_steps - 1) % NB], out.cpu())

    # the same step through mlra_decode_noalloc (the library's fixed device scratch instead of
    # a caller's workspace), timed the same way as the main leg
    # (only where the batch fits the fixed 16 MiB scratch; larger ones are refused up front)
    na_out = torch.empty_like(out)
    na_args = (hdl, inp["q"], inp["pool"], inp["page_table"], inp["seq_lens"], na_out)
    na_steps = max(20, args.steps // 4)
    try:
        M.mlra_decode_noalloc(*na_args)
        noalloc_fits = True
    except M.MlraError as ex:
        if M.STATUS.get(ex.code) != "MLRA_ERR_SCRATCH_LIMIT":
            raise
        noalloc_fits = False
    noalloc_ms = float("nan")
    if noalloc_fits:
        for _ in range(3):
            M.mlra_decode_noalloc(*na_args)
        n0, n1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n0.record(stream)
        for _ in range(na_steps):
            M.mlra_decode_noalloc(*na_args)
        n1.record(stream)
        torch.cuda.synchronize()
        noalloc_ms = n0.elapsed_time(n1) / na_steps
        assert torch.equal(na_out, out)

    # the other configurations, each timed the same way in this run
    extra = {}
    if not args.headline_only:
        del inp, r
        for name in EXTRA_WORKLOADS:
            we = W.WORKLOADS[name]
            ie = W.make_workload(we, device=dev)
            he = make_handle(M, we, ie)
            sl = ie["seq_lens"].cpu().tolist()
            # about 0.2 s of timed steps per configuration, at least 20
            n = max(20, min(args.steps, int(0.2e6 / max(1.0, cache_bytes(we, sl) / 4.0e6))))
            re_ = time_decode(M, we, ie, he, dev, n, max(3, min(args.warmup, 20)))
            st = max_over_ranks(re_["step_ms"], world, dev)
            km = [max_over_ranks(x, world, dev) for x in re_["k_ms"]]
            rf = roofline_of(we, sl, km[1])
            extra[name] = {"cache": we.cache, "steps": n, "step_us": st * 1e3, "decode_us": km[1] * 1e3,
                           "absorb_us": km[0] * 1e3, "combine_uproj_us": km[2] * 1e3,
                           "cache_bytes_per_step": cache_bytes(we, sl),
                           "step_gbs": cache_bytes(we, sl) / (st * 1e-3) / 1e9,
                           "roofline": {k2: rf[k2] for k2 in ("bound", "achieved", "peak", "unit", "frac")},
                           "hbm_frac": rf.get("hbm_frac", rf["frac"])}
            del ie, re_, he
            torch.cuda.empty_cache()

    step_ms_max = max_over_ranks(step_ms, world, dev)
    e2e_ms_max = max_over_ranks(e2e_ms, world, dev)
    noalloc_ms_max = max_over_ranks(noalloc_ms, world, dev) if noalloc_fits else None
    k_ms = [max_over_ranks(x, world, dev) for x in k_ms]
    if rank != 0:
        return

    peak, peak_kind = measured_hbm_peak()
    value = world * nbytes / (step_ms_max * 1e-3) / 1e9
    roofline = roofline_of(w, seq_lens, k_ms[1])
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms_max, "us_per_step": step_ms_max * 1e3,
        "pct_of_hbm_peak": 100.0 * value / world / peak,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": f"synthetic (seeded; inputs larger than L2: the {nbytes / 1e6:.0f} MB cache stream evicts the 126 MB L2 each step)",
        "config": config_of(w, world, nbytes),
        "kernels_ms": {"absorb": k_ms[0], "decode": k_ms[1], "combine_uproj": k_ms[2]},
        "roofline": roofline,
        "e2e": {"value": world * nbytes / (e2e_ms_max * 1e-3) / 1e9, "unit": UNIT,
                "ms_per_step": e2e_ms_max,
                "h2d_bytes_per_step": q_host.numel() * q_host.element_size() + sl_host.numel() * 4,
                "d2h_bytes_per_step": out_host[0].numel() * out_host[0].element_size(),
                "pipelined": "uploads, kernels and downloads of consecutive steps overlap on three streams",
                "h2d_gbs_alone": h2d_gbs, "d2h_gbs_alone": d2h_gbs},
        "noalloc": ({"us_per_step": noalloc_ms_max * 1e3, "steps": na_steps,
                     "note": "mlra_decode_noalloc on the same inputs (fixed library scratch, no workspace)"}
                    if noalloc_fits else {"us_per_step": None, "note": "batch too large for the fixed scratch"}),
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
    }
    if clk and clk.get("sm_mhz"):
        # step time scaled to the maximum SM clock: how the number would move with the clock
        line["us_x_mhz"] = step_ms_max * 1e3 * clk["sm_mhz"]
    if extra:
        line["workloads"] = extra
    if world == 1 and not args.no_cpu_baseline:
        # a summed-blocks head attends to all k blocks: k times the oracle work per pair
        pairs = max(1, args.cpu_pairs // (w.k if w.summed else 1))
        rate, sec, cores, pool_threads = oracle_sample_rate(w, inp_for_cpu(w, dev), pairs, 1, 0)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "blas_pool_threads": pool_threads,
                                "kind": "oracle",
                                "sample": f"float64 oracle on {pairs} random (sequence, head) pairs of "
                                          f"{w.name} ({sec:.1f} s), scaled by the fraction of the "
                                          "workload's heads covered; cores = process CPU time / wall time"}
    print(json.dumps(line), flush=True)


def inp_for_cpu(w, dev):
    """The headline workload again (same seed, same values) for the CPU baseline."""
    return W.make_workload(w, device=dev)


def run_tp(args, world, rank, local):
    """k-way tensor parallelism of the workload's MLRA-k layer across the torchrun ranks
    (world size = k): rank j decodes latent block j's cache shard for head group j, and the
    ranks all-gather their heads (NCCL) every step. Timed on the device, max over ranks; value =
    the whole layer's cache bytes per step / step time."""
    import rank_latent_kv_mlra_b200 as M
    from rank_latent_kv_mlra_b200 import tp

    w = W.WORKLOADS[args.workload]
    if world != w.k or w.summed or w.cache != "bf16":
        raise SystemExit(f"--tp needs world size = k ({w.k}) and a partitioned bf16 workload")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = W.make_workload(w, device=dev)  # same seed on every rank: the same layer
    rd = tp.RankDecode(rank, w.k, w.h, w.d_h, w.d_c, w.d_r, inp["w_uk"], inp["w_uv"])
    pool = tp.shard_pool(inp["pool"], rank, w.k, w.d_c)
    q = tp.shard_heads(inp["q"], rank, w.k, 1)
    pt, sl = inp["page_table"], inp["seq_lens"]
    nbytes = cache_bytes(w, sl.cpu().tolist())
    del inp
    torch.cuda.empty_cache()
    out = torch.empty(w.batch, w.h // w.k, w.d_h, device=dev, dtype=torch.bfloat16)
    ws = M.alloc_workspace(rd.handle, w.batch, dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        rd.decode(q, pool, pt, sl, out, workspace=ws)
        return tp.gather_heads(out)

    step()
    torch.cuda.synchronize()
    if M.mlra_get_status(ws) != 0:
        raise RuntimeError(f"rank {rank}: decode status {M.mlra_get_status(ws)}")
    for _ in range(args.warmup):
        step()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": nbytes / (ms * 1e-3) / 1e9, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "us_per_step": ms * 1e3,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded)",
        "config": dict(config_of(w, world, nbytes), parallelism=f"tp{world}"),
        "gpu_launches": 3 * args.steps,
    }), flush=True)


def producer_bytes(w, batch, d_model):
    """Algorithmic bytes of the new-row step: bf16 weights [d_c + d_r][d_model] and hidden
    states read once, bf16 rows written, one position and one page-table entry per token."""
    d_out = w.d_c + w.d_r
    return 2 * d_out * d_model + 2 * batch * d_model + 2 * batch * d_out + 8 * batch


def run_producer(args, world, rank, local):
    """Times the step before decoding (each sequence's new cache row: down-projection, RoPE
    key, page slot) on the workload's batch with d_model = workloads.PRODUCER_D_MODEL. Its
    inputs (about 6 MB) fit in L2, so L2 is flushed (a 256 MB write) before every timed step
    and each step is timed alone with CUDA events."""
    import rank_latent_kv_mlra_b200 as M

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = W.WORKLOADS[args.workload]
    inp = W.make_workload(w, device=dev)
    pr = W.make_producer_inputs(w, inp)
    hdl = M.mlra_create(w.h, w.d_h, w.d_c, w.d_r, w.k, inp["w_uk"], inp["w_uv"], blocks_summed=w.summed)
    d_model = pr["d_model"]
    ws = torch.empty(M.mlra_project_workspace_size(hdl, w.batch, d_model), dtype=torch.uint8, device=dev)
    call = lambda: M.mlra_project_append(hdl, pr["x"], pr["w_down"], pr["positions"], inp["pool"],
                                         inp["page_table"], workspace=ws)
    call()
    torch.cuda.synchronize()
    if M.mlra_get_status(ws) != 0:
        raise RuntimeError(f"producer status {M.mlra_get_status(ws)}")
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        call()
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    stream = torch.cuda.current_stream(dev)
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    ms = max_over_ranks(ms, world, dev)
    if rank != 0:
        return
    nbytes = producer_bytes(w, w.batch, d_model)
    peak, peak_kind = measured_hbm_peak()
    gbs = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({
        "metric": "new cache rows (x W^DKV | RoPE(x W^KR), stored in their page slots): achieved HBM GB/s",
        "value": world * gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "us_per_step": ms * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; L2 flushed by a 256 MB write before each step)",
        "config": {"workload": w.name, "batch": w.batch, "d_model": d_model, "d_c": w.d_c, "d_r": w.d_r,
                   "l2": "flushed before every timed step"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "peak_kind": f"{peak_kind} copy bandwidth", "bytes_per_step": nbytes,
                     "kernel": "mlra_down_proj_kernel + mlra_rope_append_kernel", "traffic": None},
        "gpu_launches": 2 * args.steps, "clocks": clk,
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.HEADLINE, choices=list(W.WORKLOADS))
    ap.add_argument("--cpu-pairs", type=int, default=15000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip timing the other configurations (the `workloads` key)")
    ap.add_argument("--producer", action="store_true",
                    help="time the step before decoding (the new cache rows) instead of the decode step")
    ap.add_argument("--tp", action="store_true",
                    help="k-way tensor parallelism of the layer across the torchrun ranks (world size = k)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup(args.impl)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.producer:
            run_producer(args, world, rank, local)
        elif args.tp:
            run_tp(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
