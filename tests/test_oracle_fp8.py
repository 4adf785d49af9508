"""Pins for the oracle's quantised latent cache (FP8 E4M3 codes, one scale per token).

What pins it, other than the oracle itself:
* the E4M3 format's definition checked against a library routine: torch's float8_e4m3fn
  conversions, in both directions, on every code and on random values;
* the format's printed constants (largest finite 448, smallest normal 2^-6, smallest
  subnormal 2^-9, NaN at 0x7F/0xFF);
* brute force: the chosen code is the nearest of all 254 finite codes (ties to the even one);
* exact special cases: every finite value encodes to itself, midpoints go to the even code,
  anything past 448 saturates, the row maximum lands on ±448, a zero row has scale 0;
* the rounding error bound of a 3-bit mantissa (half an ulp: 2^-4 relative for normal values).
"""

import numpy as np
import torch

from oracle import mla_oracle as O


def _torch_values(codes):
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_e4m3_values_match_torch_and_format_constants():
    codes = np.arange(256)
    v = O.e4m3_value(codes)
    t = _torch_values(codes)
    assert np.array_equal(np.isnan(v), np.isnan(t))
    assert np.array_equal(v[~np.isnan(v)], t[~np.isnan(t)])
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.isnan(v).sum() == 2
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert v[0x01] == 2.0 ** -9 and v[0x08] == 2.0 ** -6 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x38] == 1.0   # exponent field 7 = bias, mantissa 0
    assert np.all(np.diff(v[:127]) > 0)


def test_e4m3_encode_round_trip_ties_and_saturation():
    finite = np.array([c for c in range(256) if c & 0x7F != 0x7F])
    vals = O.e4m3_value(finite)
    assert np.array_equal(O.e4m3_encode(vals), finite.astype(np.uint8))
    grid = O.e4m3_value(np.arange(127))
    mids = (grid[:-1] + grid[1:]) / 2               # exact in float64 and float32
    assert np.all(mids.astype(np.float32).astype(np.float64) == mids)
    got = O.e4m3_encode(mids)
    lo, hi = np.arange(126), np.arange(1, 127)
    assert np.array_equal(got, np.where(lo % 2 == 0, lo, hi).astype(np.uint8))
    up = np.nextafter(mids.astype(np.float32), np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(mids.astype(np.float32), np.float32(0)).astype(np.float64)
    assert np.array_equal(O.e4m3_encode(up), hi.astype(np.uint8))
    assert np.array_equal(O.e4m3_encode(dn), lo.astype(np.uint8))
    assert np.array_equal(O.e4m3_encode(-mids), (np.where(lo % 2 == 0, lo, hi) | 0x80).astype(np.uint8))
    big = np.array([448.0, 448.5, 463.9, 464.0, 480.0, 1e6, 3.4e38])
    assert np.all(O.e4m3_encode(big) == 0x7E) and np.all(O.e4m3_encode(-big) == 0xFE)
    tiny = np.array([0.0, 2.0 ** -11, 2.0 ** -10])   # 2^-10 is the tie between 0 and 2^-9: even = 0
    assert np.array_equal(O.e4m3_encode(tiny), np.zeros(3, np.uint8))
    assert np.array_equal(O.e4m3_encode(-tiny), np.full(3, 0x80, np.uint8))
    assert O.e4m3_encode(np.array([2.0 ** -10 * 1.0001]))[0] == 1


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(3)
    mag = np.exp2(rng.uniform(-12, np.log2(440.0), 200_000))
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    ours = O.e4m3_encode(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_is_nearest_by_brute_force():
    rng = np.random.default_rng(4)
    x = (np.exp2(rng.uniform(-11, 9.2, 3000)) * rng.choice([-1.0, 1.0], 3000)).astype(np.float32)
    finite = [c for c in range(256) if c & 0x7F != 0x7F]
    for xi, ci in zip(x.astype(np.float64), O.e4m3_encode(x.astype(np.float64))):
        best, best_d = None, None
        for c in finite:
            d = abs(float(O.e4m3_value(c)) - (min(abs(xi), 448.0) * (1 if xi >= 0 else -1)))
            if best is None or d < best_d or (d == best_d and c % 2 == 0 and best % 2 == 1):
                if d == best_d and (c & 0x7F) == 0 and (best & 0x7F) == 0:
                    continue   # +0 and -0 tie: the sign of x decides, checked below
                best, best_d = c, d
        if O.e4m3_value(best) == 0.0:
            best = 0x80 if xi < 0 else 0x00
        assert int(ci) == best, (xi, int(ci), best)


def test_quantize_rows_scale_max_code_and_error_bound():
    rng = np.random.default_rng(5)
    rows = np.concatenate([rng.standard_normal((40, 576)),
                           rng.standard_normal((8, 576)) * np.exp2(rng.uniform(-20, 20, (8, 1)))])
    rows = rows.astype(np.float32)
    codes, scales = O.quantize_rows_e4m3(rows)
    amax = np.abs(rows).max(axis=1)
    assert scales.dtype == np.float32
    assert np.array_equal(scales, (torch.from_numpy(amax) / 448.0).numpy())
    i_max = np.abs(rows).argmax(axis=1)
    top = codes[np.arange(rows.shape[0]), i_max]
    assert np.all((top & 0x7F) == 0x7E)
    deq = O.dequantize_rows_e4m3(codes, scales)
    v = rows.astype(np.float64)
    rel_part = np.abs(v) >= 2.0 ** -6 * scales[:, None]
    err = np.abs(deq - v)
    # half an ulp of the 3-bit mantissa, plus the float32 rounding of v / scale
    assert np.all(err[rel_part] <= (2.0 ** -4 + 2.0 ** -22) * np.abs(v[rel_part]))
    sub = ~rel_part
    assert np.all(err[sub] <= (2.0 ** -10 + 2.0 ** -22) * np.broadcast_to(scales[:, None], v.shape)[sub])
    # float32 division, then the nearest code: the same codes from torch's own float32 ops
    q32 = (torch.from_numpy(rows) / torch.from_numpy(scales)[:, None])
    assert np.array_equal(codes, q32.to(torch.float8_e4m3fn).view(torch.uint8).numpy())


def test_quantize_zero_row_and_signed_zeros():
    rows = np.zeros((2, 64), np.float32)
    rows[1, ::2] = -0.0
    codes, scales = O.quantize_rows_e4m3(rows)
    assert np.all(scales == 0)
    assert np.all(O.dequantize_rows_e4m3(codes, scales) == 0)
    assert np.all(codes[0] == 0) and np.all(codes[1, ::2] == 0x80)


def test_gather_rows_fp8_follows_block_table():
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 126, (5, 4, 8)).astype(np.uint8)
    scales = rng.uniform(0.5, 2.0, (5, 4)).astype(np.float32)
    bt = np.array([3, 0, 4])
    rows = O.gather_rows_fp8(codes, scales, bt, 10, page_size=4)
    for j in range(10):
        page, slot = bt[j // 4], j % 4
        for d in range(8):
            assert rows[j, d] == float(O.e4m3_value(codes[page, slot, d])) * float(scales[page, slot])
