"""Pins for the producer oracle (the new token's cache row: down-projection, RoPE key,
placement), each against something other than the oracle's own formula:

* the complex form of the rotation (RoFormer Section 3.4.2: a feature pair as a complex number
  multiplied by exp(i m theta)), evaluated with numpy complex arithmetic;
* closed forms: position 0 is the identity, the first pair turns by exactly pos radians, the
  last pair by pos * base^(-(d_r-2)/d_r);
* the property RoPE is built for (RoFormer Section 3.2): the dot product of a query rotated to
  m and a key rotated to n depends only on m - n;
* composition and norm preservation of rotations;
* pure-Python loops for the projection on a tiny case;
* the decode oracle's own page addressing reads back what was placed.

The last tests plant mistakes in the oracle (on the CPU) and check that a pin catches each.
"""
import math

import numpy as np
import pytest

from oracle import mlra_oracle as MO
from oracle import producer_oracle as P


def test_position_zero_is_identity():
    v = np.random.default_rng(0).standard_normal((3, 64))
    np.testing.assert_array_equal(P.rope(v, 0), v)


@pytest.mark.parametrize("pos", [1, 7, 8191, 131071])
def test_rotation_is_complex_multiplication(pos):
    rng = np.random.default_rng(pos)
    d_r = 64
    v = rng.standard_normal(d_r)
    z = v[0::2] + 1j * v[1::2]
    i = np.arange(d_r // 2)
    w = z * np.exp(1j * pos * 10000.0 ** (-2.0 * i / d_r))
    got = P.rope(v, pos)
    np.testing.assert_allclose(got[0::2], w.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got[1::2], w.imag, rtol=1e-12, atol=1e-12)


def test_first_pair_turns_by_pos_radians_and_last_pair_by_its_frequency():
    d_r = 64
    e0 = np.zeros(d_r)
    e0[0] = 1.0
    for pos in (1, 3, 100):
        r = P.rope(e0, pos)
        assert abs(r[0] - math.cos(pos)) < 1e-15 and abs(r[1] - math.sin(pos)) < 1e-15
    # the last pair's frequency is base^(-(d_r-2)/d_r): a quarter turn at pos = (pi/2) / theta
    theta = 10000.0 ** (-(d_r - 2) / d_r)
    el = np.zeros(d_r)
    el[d_r - 2] = 1.0
    r = P.rope(el, (math.pi / 2) / theta)
    assert abs(r[d_r - 2]) < 1e-12 and abs(r[d_r - 1] - 1.0) < 1e-12


def test_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in [(5, 2), (1000, 997), (40000, 39997)]:
        a = P.rope(q, m) @ P.rope(k, n)
        b = P.rope(q, m - n) @ k
        assert abs(a - b) < 1e-9 * (abs(b) + 1)


def test_rotations_compose_and_preserve_norms():
    rng = np.random.default_rng(4)
    v = rng.standard_normal(64)
    np.testing.assert_allclose(P.rope(P.rope(v, 17), 25), P.rope(v, 42), rtol=1e-12, atol=1e-12)
    pairs = v[0::2] ** 2 + v[1::2] ** 2
    r = P.rope(v, 12345)
    np.testing.assert_allclose(r[0::2] ** 2 + r[1::2] ** 2, pairs, rtol=1e-12)


def test_projection_brute_force_tiny():
    rng = np.random.default_rng(5)
    d_model, d_c, d_r = 5, 6, 4
    x = rng.standard_normal(d_model)
    w = rng.standard_normal((d_c + d_r, d_model))
    got = P.project_row(x, w, d_c, d_r, 0)
    for r in range(d_c + d_r):
        s = 0.0
        for d in range(d_model):
            s += float(w[r][d]) * float(x[d])
        assert abs(got[r] - s) < 1e-12
    # at a nonzero position only the RoPE part moves, by the complex form
    got3 = P.project_row(x, w, d_c, d_r, 3)
    np.testing.assert_allclose(got3[:d_c], got[:d_c], rtol=0, atol=0)
    z = (got[d_c::2][:d_r // 2] + 1j * got[d_c + 1::2][:d_r // 2]) * np.exp(
        1j * 3 * 10000.0 ** (-2.0 * np.arange(d_r // 2) / d_r))
    np.testing.assert_allclose(got3[d_c::2], z.real, atol=1e-12)
    np.testing.assert_allclose(got3[d_c + 1::2], z.imag, atol=1e-12)


def test_placed_rows_read_back_through_the_decode_addressing():
    rng = np.random.default_rng(6)
    B, d_model, d_c, d_r = 3, 8, 12, 4
    pages_per_seq = 3
    num_pages = B * pages_per_seq + 2
    pt = rng.permutation(num_pages)[:B * pages_per_seq].reshape(B, pages_per_seq)
    pool = np.full((num_pages, 64, d_c + d_r), np.nan)
    x = rng.standard_normal((B, d_model))
    w = rng.standard_normal((d_c + d_r, d_model))
    positions = np.array([0, 70, 191])
    rows, pages, slots = P.project_append(x, w, d_c, d_r, positions, pt)
    for b in range(B):
        pool[pages[b], slots[b]] = rows[b]
    for b in range(B):
        got = MO.gather_rows(pool, pt, b, int(positions[b]) + 1)[int(positions[b])]
        np.testing.assert_array_equal(got, rows[b])


def test_bytes_per_step():
    # 576 x 5120 bf16 weights, 32 tokens of 5120 bf16, 32 rows of 1152 B, 8 B per token
    assert P.bytes_per_step(32, 5120, 512, 64) == 2 * 576 * 5120 + 2 * 32 * 5120 + 32 * 1152 + 256


# ---------------------------------------------------------------------------------------
# Planted mistakes (in the oracle, on the CPU) that a pin above must catch
# ---------------------------------------------------------------------------------------

def _rope_wrong_sign(v, pos, base=P.ROPE_BASE):
    v = np.asarray(v, dtype=np.float64)
    ang = float(pos) * P.rope_frequencies(v.shape[-1], base)
    out = np.empty_like(v)
    out[..., 0::2] = v[..., 0::2] * np.cos(ang) + v[..., 1::2] * np.sin(ang)
    out[..., 1::2] = -v[..., 0::2] * np.sin(ang) + v[..., 1::2] * np.cos(ang)
    return out


def _rope_rotate_half(v, pos, base=P.ROPE_BASE):
    v = np.asarray(v, dtype=np.float64)
    h = v.shape[-1] // 2
    ang = float(pos) * P.rope_frequencies(v.shape[-1], base)
    out = np.empty_like(v)
    out[..., :h] = v[..., :h] * np.cos(ang) - v[..., h:] * np.sin(ang)
    out[..., h:] = v[..., :h] * np.sin(ang) + v[..., h:] * np.cos(ang)
    return out


def test_planted_wrong_sign_is_caught(monkeypatch):
    monkeypatch.setattr(P, "rope", _rope_wrong_sign)
    with pytest.raises(AssertionError):
        test_rotation_is_complex_multiplication(7)


def test_planted_rotate_half_pairing_is_caught(monkeypatch):
    monkeypatch.setattr(P, "rope", _rope_rotate_half)
    with pytest.raises(AssertionError):
        test_rotation_is_complex_multiplication(7)


def test_planted_wrong_frequency_is_caught(monkeypatch):
    monkeypatch.setattr(P, "rope_frequencies", lambda d_r, base=P.ROPE_BASE: base ** (-np.arange(d_r // 2) / d_r))
    with pytest.raises(AssertionError):
        test_first_pair_turns_by_pos_radians_and_last_pair_by_its_frequency()
