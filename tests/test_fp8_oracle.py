"""Pins of the e4m3 oracle (no GPU) against the format and a library routine.

* every one of the 256 codes decodes to the value torch's float8_e4m3fn dtype gives it (NaN at
  S.1111.111), with the format's landmarks: 448 the largest finite, 2^-6 the smallest normal, 2^-9
  the smallest subnormal;
* rounding: in-range values round as torch's float8_e4m3fn cast does (round to nearest even),
  every finite code round-trips, exact midpoints go to the even mantissa, and values beyond ±448
  saturate to ±448;
* per-tensor quantisation: the element of largest magnitude maps to ±448 exactly and q·dq stays
  within half a grid step (relative 2^-4) of x;
* the product of decoded codes against a plain triple loop on a tiny case.
"""
import numpy as np
import pytest
import torch

from oracle import fp8_oracle as F8


def test_decode_matches_torch_and_the_format_landmarks():
    codes = np.arange(256, dtype=np.uint8)
    got = F8.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.nanmax(got) == 448.0 and got[0x7E] == 448.0 and np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert got[0x08] == 2.0 ** -6 and got[0x01] == 2.0 ** -9 and got[0x80] == 0.0


def test_round_matches_torch_in_range_and_saturates_beyond():
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    y = np.clip(y, -448, 448).astype(np.float32)
    got = F8.e4m3_round(y)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(got, ref)
    assert np.array_equal(F8.e4m3_round(np.array([449.0, 1e6, -500.0])), np.array([448.0, 448.0, -448.0]))


def test_codes_round_trip_and_ties_go_to_even():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = F8.e4m3_decode(codes)
    back = F8.e4m3_encode(vals)
    # +0 and −0 both decode to 0: compare values for those, codes for the rest
    nz = vals != 0
    assert np.array_equal(back[nz], codes[nz])
    # midpoints between neighbours: 1 + 1/16 lies between 1 (mantissa 0) and 1.125 (mantissa 1)
    assert F8.e4m3_round(np.array([1.0625]))[0] == 1.0
    assert F8.e4m3_round(np.array([1.1875]))[0] == 1.25      # between 1.125 (odd) and 1.25 (even)
    assert F8.e4m3_round(np.array([2.0 ** -10]))[0] == 0.0    # half the smallest subnormal → 0 (even)
    assert F8.e4m3_round(np.array([3 * 2.0 ** -10]))[0] == 2.0 ** -8  # 1.5 subnormal steps → 2 steps


def test_per_tensor_quantisation_bounds():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(10000) * 0.3).astype(np.float32)
    x[1234] = -2.5
    q, dq = F8.quantize_per_tensor(x)
    assert F8.e4m3_decode(q[1234:1235])[0] == -448.0
    xr = F8.e4m3_decode(q) * float(dq)
    # the grid's relative half-spacing is 2^-4 for normal values; tiny values: half a subnormal step
    assert np.all(np.abs(xr - x) <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * float(dq)) + 1e-12)
    q0, dq0 = F8.quantize_per_tensor(np.zeros(8, np.float32))
    assert np.all(q0 == 0) and dq0 == 1.0


def test_product_against_a_triple_loop():
    rng = np.random.default_rng(2)
    qa = rng.integers(0, 256, (3, 5)).astype(np.uint8)
    qb = rng.integers(0, 256, (4, 5)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0
    qb[(qb & 0x7F) == 0x7F] = 0
    got = F8.gemm_e4m3(qa, qb, 0.5, 0.25, alpha=2.0)
    da, db = F8.e4m3_decode(qa), F8.e4m3_decode(qb)
    for i in range(3):
        for j in range(4):
            s = 0.0
            for k in range(5):
                s += da[i, k] * db[j, k]
            assert got[i, j] == pytest.approx(2.0 * 0.5 * 0.25 * s, rel=1e-15, abs=1e-300)
