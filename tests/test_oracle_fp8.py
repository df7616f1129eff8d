"""Pins for the FP8 (E4M3) cache oracle, each against something other than the oracle:

* the format's definition: closed-form values of named codes (zero, the smallest subnormal,
  the smallest normal, one, the largest finite value, NaN);
* torch's float8_e4m3fn conversion (an independent library routine) on every code and on
  random values, ties included;
* round trips and saturation;
* the bf16-cache decode on rows whose values E4M3 holds exactly.

The last tests plant mistakes in the oracle (on the CPU) and check that a pin catches each.
"""
import math

import numpy as np
import pytest
import torch

from oracle import fp8_cache_oracle as F
from oracle import mlra_oracle as O


def test_named_codes():
    assert F.e4m3_decode(0x00) == 0.0
    assert math.copysign(1.0, F.e4m3_decode(0x80)) == -1.0
    assert F.e4m3_decode(0x01) == 2.0 ** -9          # smallest subnormal: 2^-6 * 1/8
    assert F.e4m3_decode(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert F.e4m3_decode(0x08) == 2.0 ** -6          # smallest normal
    assert F.e4m3_decode(0x38) == 1.0                # exponent 7 = bias
    assert F.e4m3_decode(0x3C) == 1.5
    assert F.e4m3_decode(0x7E) == 448.0              # largest finite: 2^8 * 1.75
    assert F.e4m3_decode(0xFE) == -448.0
    assert math.isnan(F.e4m3_decode(0x7F)) and math.isnan(F.e4m3_decode(0xFF))
    assert F.e4m3_decode(0x78) == 256.0              # exponent 15 is a normal exponent here


def test_every_code_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = F.e4m3_decode_array(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(got[~nan], ref[~nan])


def test_encoder_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(3000) * 40, rng.standard_normal(1000) * 0.01,
                        rng.uniform(-463, 463, 1000)])
    # midpoints between neighbouring codes exercise ties-to-even
    vals = F.e4m3_decode_array(np.arange(0x7F))
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([x, mids, -mids])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.e4m3_encode_array(x)
    assert np.array_equal(got, ref), np.nonzero(got != ref)[0][:10]


def test_encoder_round_trip_and_saturation():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert F.e4m3_encode(F.e4m3_decode(c)) == c
    assert F.e4m3_encode(1e6) == 0x7E and F.e4m3_encode(-1e6) == 0xFE
    assert F.e4m3_encode(464.0) == 0x7E          # torch maps this to NaN; satfinite keeps 448
    assert F.e4m3_encode(float("nan")) == 0x7F
    assert F.e4m3_encode(2.0 ** -10) == 0x00     # tie between 0 and 2^-9: even code 0
    assert F.e4m3_encode(3 * 2.0 ** -10) == 0x02  # tie between codes 1 and 2


def _exact_case(rng, k=4, B=2, h=8, d_h=16, d_b=24, d_r=8, lens=(70, 150)):
    """A small cache whose rows are E4M3 values times the scales, so dequantizing gives them
    back exactly and the bf16-cache oracle on the float rows is the reference."""
    d_c = d_b * k
    lens = np.array(lens[:B])
    pages = [(n + 63) // 64 for n in lens]
    num_pages = sum(pages) + 1
    phys = rng.permutation(num_pages)
    pt = np.full((B, max(pages)), -1, dtype=np.int64)
    off = 0
    for b, p in enumerate(pages):
        pt[b, :p] = phys[off:off + p]
        off += p
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    codes = rng.choice(finite, size=(num_pages, 64, d_c + d_r)).astype(np.uint8)
    ls, rs = 0.03125, 0.0078125
    rows = F.e4m3_decode_array(codes)
    rows[..., :d_c] *= ls
    rows[..., d_c:] *= rs
    q = rng.standard_normal((B, h, d_h + d_r))
    w_uk = rng.standard_normal((h, d_b, d_h)) / math.sqrt(d_b)
    w_uv = rng.standard_normal((h, d_b, d_h)) / math.sqrt(d_b)
    return dict(codes=codes, rows=rows, ls=ls, rs=rs, q=q, w_uk=w_uk, w_uv=w_uv, pt=pt, lens=lens,
                k=k, d_r=d_r, d_c=d_c)


def test_decode_fp8_equals_bf16_decode_on_exact_rows():
    c = _exact_case(np.random.default_rng(1))
    got = F.decode_fp8(c["q"], c["w_uk"], c["w_uv"], c["codes"], c["pt"], c["lens"], c["k"], c["d_r"],
                       c["ls"], c["rs"])
    ref = O.decode(c["q"], c["w_uk"], c["w_uv"], c["rows"], c["pt"], c["lens"], c["k"], c["d_r"])
    np.testing.assert_array_equal(got["out"], ref["out"])
    np.testing.assert_array_equal(got["lse"], ref["lse"])


def test_quantize_rows_inverts_dequantize():
    c = _exact_case(np.random.default_rng(2), lens=(10, 20))
    rows = c["rows"][:2]
    back = F.quantize_rows(rows, c["d_c"], c["ls"], c["rs"])
    assert np.array_equal(back, c["codes"][:2])


def test_quantization_error_is_within_half_an_ulp():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(4000) * 1.5     # |x| / s stays below 448 (no saturation)
    s = 8.0 / 448
    deq = F.e4m3_decode_array(F.e4m3_encode_array(x / s)) * s
    # relative half-ulp of a 3-bit mantissa, absolute half of the subnormal step below 2^-6
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10)
    assert np.all(np.abs(deq - x) <= bound * (1 + 1e-12))


# ---------------------------------------------------------------------------------------
# Planted mistakes (in the oracle, on the CPU) that a pin above must catch
# ---------------------------------------------------------------------------------------

def test_planted_wrong_bias_is_caught(monkeypatch):
    bad = np.array([F.e4m3_decode(c) * (2.0 if (c >> 3) & 0xF else 1.0) for c in range(256)])
    monkeypatch.setattr(F, "_TABLE", bad)
    with pytest.raises(AssertionError):
        test_every_code_matches_torch()


def test_planted_swapped_scales_are_caught(monkeypatch):
    real = F.dequantize_pool
    monkeypatch.setattr(F, "dequantize_pool", lambda p, d_c, ls, rs: real(p, d_c, rs, ls))
    with pytest.raises(AssertionError):
        test_decode_fp8_equals_bf16_decode_on_exact_rows()


def test_planted_ties_away_from_zero_is_caught(monkeypatch):
    def away(x):
        if math.isnan(x):
            return F.E4M3_NAN
        sign = 0x80 if x < 0 else 0
        a = min(abs(x), F.E4M3_MAX)
        i = int(np.searchsorted(F._POS_VALUES, a))
        if i < len(F._POS_VALUES) and F._POS_VALUES[i] == a:
            return sign | i
        return sign | (i if F._POS_VALUES[i] - a <= a - F._POS_VALUES[i - 1] else i - 1)
    monkeypatch.setattr(F, "e4m3_encode", away)
    with pytest.raises(AssertionError):
        test_encoder_matches_torch_in_range()
