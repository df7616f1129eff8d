"""mlra_decode_noalloc (through the C ABI) against mlra_decode on the same inputs.

The no-allocation variant keeps its scratch in one fixed device array that every call shares
and that keeps the previous call's contents, so two calls in a row are checked, the second on
a different batch, lengths and seed: anything read from stale scratch would show up there.
This file is named to be collected last; it builds its own inputs and runs alone as well.
"""
import numpy as np
import pytest
import torch

import rank_latent_kv_mlra_b200 as M
import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

HEADLINE = W.WORKLOADS["mlra4_h128_b32_n8192"]

# two consecutive calls: different batch sizes, length mixes and seeds
CALLS = [
    W.scaled(HEADLINE, batch=5, seq_len=None, len_range=(1, 3000), seed=21),
    W.scaled(HEADLINE, batch=12, seq_len=None, len_range=(0, 1400), seed=22),
]


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    M.load_library()


def _outputs(hdl, inp, batch, h, d_h, noalloc):
    out = torch.full((batch, h, d_h), float("nan"), device="cuda")
    lse = torch.full((batch, h), float("nan"), device="cuda")
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    args = (hdl, inp["q"], inp["pool"], inp["page_table"], inp["seq_lens"], out, lse)
    if noalloc:
        M.mlra_decode_noalloc(*args, status=status)
    else:
        ws = M.mlra_decode(*args)
        status.copy_(ws[:4].view(torch.int32))
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy(), int(status.item())


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    # one handle (the first workload's weights) for every call, as a serving loop holds it
    inputs = [W.make_workload(w, device="cuda") for w in CALLS]
    hdl = G.make_handle(CALLS[0], inputs[0])
    results = [_outputs(hdl, inp, w.batch, w.h, w.d_h, noalloc=True) for w, inp in zip(CALLS, inputs)]
    for w, inp, (out, lse, status) in zip(CALLS, inputs, results):
        ref_out, ref_lse, ref_status = _outputs(hdl, inp, w.batch, w.h, w.d_h, noalloc=False)
        assert status == 0 and ref_status == 0
        assert not np.isnan(out).any()
        e = G.errors(out, ref_out)
        assert e["max_abs"] <= G.TOL_MAX_ABS and e["mean_abs"] <= G.TOL_MEAN_ABS, e
        live = inp["seq_lens"].cpu().numpy() > 0
        assert np.isneginf(lse[~live]).all()
        assert np.abs(lse[live] - ref_lse[live]).max() <= G.TOL_LSE_ABS


def test_noalloc_rejects_batch_beyond_scratch():
    w = W.scaled(HEADLINE, batch=1, seq_len=64, len_range=None)
    inp = W.make_workload(w, device="cuda")
    hdl = G.make_handle(w, inp)
    # largest batch the 16 MiB scratch holds, and one past it, per mlra_workspace_size
    limit = 16 << 20
    fits = max(b for b in range(1, 400) if M.mlra_workspace_size(hdl, b) <= limit)
    big = fits + 1
    q = torch.zeros(big, w.h, w.d_h + w.d_r, dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros(big, 1, dtype=torch.int32, device="cuda")
    sl = torch.zeros(big, dtype=torch.int32, device="cuda")
    out = torch.full((big, w.h, w.d_h), 7.0, device="cuda")
    with pytest.raises(M.MlraError) as ei:
        M.mlra_decode_noalloc(hdl, q, inp["pool"], pt, sl, out)
    assert ei.value.code == -8
    torch.cuda.synchronize()
    assert (out == 7.0).all()  # nothing was launched
