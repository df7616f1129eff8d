"""Builds libmlra.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m rank_latent_kv_mlra_b200.build [--verbose-ptxas]

The CUDA runtime is linked statically and the driver's tensor-map encoder is resolved at
run time, so the library loads on a machine without a GPU driver (its symbols can be
checked there); compute calls need a B200.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmlra.so")
SOURCES = [os.path.join(HERE, "csrc", "mlra_api.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))] + [
    os.path.join(ROOT, "include", "mlra.h")]


def nvcc_command(ptxas_verbose=False):
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", LIB] + SOURCES
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force=False, ptxas_verbose=False):
    if not force and up_to_date():
        return LIB
    cmd = nvcc_command(ptxas_verbose)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libmlra.so")
    if ptxas_verbose:
        sys.stderr.write(res.stderr)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
