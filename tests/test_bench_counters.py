"""The algorithmic byte and FLOP counts that bench.py divides by kernel time, against the
figures the pages state.

* Bytes: one cached token is d_c + d_r bf16 elements, 4.5 d_h at d_c = 4 d_h, d_r = d_h / 2
  (MLA row of Table 1 of "Multi-Head Low-Rank Attention" (thelatestinai.com)), read once per
  step, plus one 4-byte page id per 64 tokens.
* FLOPs at k = 1: Table 2's MLA numerator, 4 n h d_c + 2 n h d_r per step.
* FLOPs at k > 1: each head sees one block of d_c / k columns (partitioned), or all k blocks
  (summed, k times the work; Table 2's MLRA-4 column, 4 n h d_c / 4 + 2 n h d_r per device,
  times the 4 devices).
"""
import os

import bench
import workloads as W


def test_cache_bytes_per_token_is_table1_mla_row():
    w = W.WORKLOADS["mlra4_h128_b32_n8192"]
    assert w.d_c == 4 * w.d_h and w.d_r == w.d_h // 2
    assert bench.cache_bytes(w, [64]) == 64 * int(4.5 * w.d_h) * 2 + 4
    assert bench.cache_bytes(w, [8192] * 32) == 301_989_888 + 32 * 128 * 4


def test_decode_flops_k1_is_table2_mla_numerator():
    w = W.WORKLOADS["mla_h128_b128_ragged1k_32k"]
    n = 1000
    assert w.k == 1
    assert bench.decode_flops(w, [n]) == 4 * n * w.h * w.d_c + 2 * n * w.h * w.d_r


def test_decode_flops_partitioned_and_summed():
    w = W.WORKLOADS["mlra4_h128_b32_n8192"]
    n = 8192
    per_token = w.h * (4 * w.d_c // w.k + 2 * w.d_r)
    assert per_token == 81_920
    assert bench.decode_flops(w, [n]) == n * per_token
    ws = W.WORKLOADS["mlra4sum_h128_b32_n8192"]
    assert ws.summed and ws.k == 4
    # Table 2, MLRA-4: 4 n h (d_c / 4) + 2 n h d_r per device, one block per device, 4 devices
    per_device = 4 * n * ws.h * (ws.d_c // 4) + 2 * n * ws.h * ws.d_r
    assert bench.decode_flops(ws, [n]) == 4 * per_device


def test_producer_bytes_match_the_oracle_count():
    from oracle import producer_oracle as P
    w = W.WORKLOADS["mlra4_h128_b32_n8192"]
    for batch, d_model in [(32, 5120), (3, 256), (300, 384)]:
        assert bench.producer_bytes(w, batch, d_model) == P.bytes_per_step(batch, d_model, w.d_c, w.d_r)


def test_kernel_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    """A recorded ncu traffic figure stays attached to the decode kernel code it was measured
    on: comment and blank-line edits and another shape's line keep the hash, a code edit
    changes it."""
    import shutil
    src = os.path.join(bench.ROOT, "rank_latent_kv_mlra_b200", "csrc")
    dst = tmp_path / "rank_latent_kv_mlra_b200" / "csrc"
    dst.mkdir(parents=True)
    for f in ("common.cuh", "decode.cuh", "mlra_api.cu"):
        shutil.copy(os.path.join(src, f), dst / f)
    w = W.WORKLOADS[W.HEADLINE]
    base = bench.kernel_source_hash(w)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_source_hash(w) == base
    with open(dst / "decode.cuh", "a") as fh:
        fh.write("\n// a comment\n\n")
    assert bench.kernel_source_hash(w) == base
    api = (dst / "mlra_api.cu").read_text()
    other = [l for l in api.splitlines() if l.startswith("using DecMla ")][0]
    (dst / "mlra_api.cu").write_text(api.replace(other, other.replace("DecodeShape<", "DecodeShape< ")))
    assert bench.kernel_source_hash(w) == base  # another shape's line
    with open(dst / "decode.cuh", "a") as fh:
        fh.write("static_assert(true, \"\");\n")
    assert bench.kernel_source_hash(w) != base


def test_recorded_traffic_is_reported_only_for_captured_workloads():
    assert bench.recorded_traffic("mlra2sum_h128_b64_n4096") is None
