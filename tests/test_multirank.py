"""The multi-process plumbing of bench.py on CPU with the gloo backend (world size 2): the
reference arm under torchrun prints one line from rank 0 only, and the cross-rank helpers take
the maximum over ranks. The decode path itself runs one independent replica per GPU and has
no exchange, so nothing else crosses ranks."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "3", "--warmup", "3", "--workload", "mlra4_h8_b1_n256_f32"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=240)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0
    # the reference line describes its workload with the same keys as the GPU arm's line
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    w = W.WORKLOADS["mlra4_h8_b1_n256_f32"]
    ours = bench.config_of(w, 2, line["config"]["cache_bytes_per_step"])
    assert line["config"] == ours


def _rank_main(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        sys.path.insert(0, ROOT)
        import bench
        bench.barrier(2)
        out[rank] = bench.max_over_ranks(1.5 + rank, 2, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(port, out), nprocs=2, start_method="spawn", join=True)
    assert dict(out) == {0: 2.5, 1: 2.5}
