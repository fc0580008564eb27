"""Pins for the oracle's NVFP4 encoding (CPU only).

Each check ties the oracle to something other than itself: hand-worked bytes,
closed-form descriptions of the rounding, torch's own float8 conversion, exact
arithmetic on lossless inputs and the error bound of round-to-nearest.
"""
import json
import os
import struct

import numpy as np
import pytest
import torch

from oracle import nvfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _f32_from_bits(bits):
    return np.asarray(bits, dtype=np.uint32).view(np.float32)


def _all_bf16_values():
    """Every bfloat16 bit pattern, as fp32 (NaNs dropped)."""
    b = (np.arange(1 << 16, dtype=np.uint32) << 16)
    v = b.view(np.float32)
    return v[~np.isnan(v)]


# --- E2M1 --------------------------------------------------------------------

def _e2m1_closed_form(y):
    """Round-to-nearest-even onto {0,.5,1,1.5,2,3,4,6} written as the seven
    decision thresholds (the midpoints; a midpoint goes to the even code)."""
    a = np.minimum(np.abs(y.astype(np.float64)), 6.0)
    a = np.where(np.isnan(a), 0.0, a)
    mag = ((a > 0.25).astype(np.uint8) + (a >= 0.75) + (a > 1.25) + (a >= 1.75)
           + (a > 2.5) + (a >= 3.5) + (a > 5.0)).astype(np.uint8)
    return mag | (np.signbit(y).astype(np.uint8) << 3)


def _e2m1_brute(y):
    """Argmin of |a - v| over the whole value table, ties to the even code."""
    a = np.minimum(np.abs(y.astype(np.float64)), 6.0)
    a = np.where(np.isnan(a), 0.0, a)
    vals = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    d = np.abs(a[:, None] - vals[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = np.where(d == best, np.arange(8) % 2, 9)        # even first
    cand = cand * 16 + np.arange(8)
    mag = (np.argmin(cand, axis=1)).astype(np.uint8)
    return mag | (np.signbit(y).astype(np.uint8) << 3)


def _e2m1_probe_values():
    vals = [_all_bf16_values()]
    # dense fp32 neighbourhoods of every grid point and midpoint
    pts = np.array([0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7], F32)
    bits = pts.view(np.uint32).astype(np.int64)
    offs = np.arange(-64, 65)
    nb = (bits[:, None] + offs[None, :]).ravel()
    nb = nb[(nb >= 0) & (nb < 0x7F800000)].astype(np.uint32)
    v = nb.view(np.float32)
    vals += [v, -v]
    # random fp32 bit patterns across all exponents
    rng = np.random.default_rng(1)
    r = rng.integers(0, 1 << 32, size=1 << 18, dtype=np.uint64).astype(np.uint32).view(np.float32)
    vals.append(r[~np.isnan(r)])
    return np.concatenate(vals).astype(F32)


def test_e2m1_matches_closed_form_and_brute_force():
    y = _e2m1_probe_values()
    got = nvfp4.e2m1_encode(y)
    np.testing.assert_array_equal(got, _e2m1_closed_form(y))
    sub = y[:: max(1, y.size // 200_000)]
    np.testing.assert_array_equal(nvfp4.e2m1_encode(sub), _e2m1_brute(sub))


def test_e2m1_decode_table():
    # sign-magnitude 1-2-1 format, bias 1: value = (-1)^s 2^(e-1) (1 + m/2), e > 0
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        v = (m * 0.5) if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
        assert nvfp4.e2m1_decode(np.array([code]))[0] == (-v if s else v)


def test_e2m1_known_ties_and_signs():
    y = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.0, -1e-30, 1e9, -1e9], F32)
    np.testing.assert_array_equal(nvfp4.e2m1_encode(y),
                                  [0, 2, 2, 4, 4, 6, 6, 8, 8, 7, 15])


# --- E4M3 ---------------------------------------------------------------------

def test_e4m3_decode_matches_torch_float8():
    codes = torch.arange(0x7F, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    np.testing.assert_array_equal(nvfp4.e4m3_decode(codes.numpy()), ref)


def _e4m3_probe_values():
    v = _all_bf16_values()
    v = np.abs(v[np.isfinite(v)])
    tab = nvfp4.E4M3_VALUES
    mids = ((tab[1:] + tab[:-1]) / 2).astype(F32)
    bits = np.concatenate([tab.astype(F32), mids]).view(np.uint32).astype(np.int64)
    nb = (bits[:, None] + np.arange(-8, 9)[None, :]).ravel()
    nb = nb[(nb >= 0) & (nb < 0x7F800000)].astype(np.uint32)
    rng = np.random.default_rng(2)
    r = rng.uniform(0, 470, size=1 << 16).astype(F32)
    return np.concatenate([v, nb.view(np.float32), r]).astype(F32)


def test_e4m3_encode_matches_torch_float8_below_overflow():
    s = _e4m3_probe_values()
    inside = s < 464.0                      # torch does not saturate beyond
    ref = torch.from_numpy(s[inside]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(nvfp4.e4m3_encode(s[inside]), ref)
    assert np.all(nvfp4.e4m3_encode(s[~inside]) == 0x7E)   # satfinite


def test_e4m3_known_values():
    s = np.array([0.84375, 0.8333333, 1.0, 3.0, 448.0, 1e6, 2.0 ** -9, 2.0 ** -10, 0.0], F32)
    np.testing.assert_array_equal(nvfp4.e4m3_encode(s),
                                  [0x36, 0x35, 0x38, 0x44, 0x7E, 0x7E, 0x01, 0x00, 0x00])


# --- block quantisation -----------------------------------------------------

def _load_cases():
    with open(os.path.join(GOLDEN, "nvfp4_hand_examples.json")) as f:
        return json.load(f)["cases"]


def _row(vals):
    return np.array([[float(v) for v in r] for r in vals], F32)


@pytest.mark.parametrize("case", _load_cases(), ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    x = _row(case["x"])
    g = _f32_from_bits([int(case["g_bits"], 16)])[0]
    if case["kind"] == "weight":
        codes, scales, g_got = nvfp4.quantize_weight(x)
        assert np.float32(g_got).view(np.uint32) == np.float32(g).view(np.uint32)
    else:
        codes, scales = nvfp4.quantize(x, g)
    assert [r.tobytes().hex() for r in codes] == case["codes_hex"]
    assert [r.tobytes().hex() for r in scales] == case["scales_hex"]


def test_pack_order_low_nibble_even_index():
    q = np.array([[1, 2, 3, 4]], np.uint8)
    assert nvfp4.pack_codes(q).tobytes() == bytes([0x21, 0x43])
    np.testing.assert_array_equal(nvfp4.unpack_codes(nvfp4.pack_codes(q)), q)


def _lossless_matrix(rng, n, k, g):
    """Blocks of E2M1 grid values (each with a +-6) times an E4M3 value times
    g; one block uses 448 so that the tensor amax is 6 * 448 * g."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    v = grid[rng.integers(0, 8, size=(n, k // 16, 16))] * rng.choice([-1, 1], size=(n, k // 16, 16))
    v[:, :, 0] = 6.0 * rng.choice([-1, 1], size=(n, k // 16))
    normal = nvfp4.E4M3_VALUES[8:]                # normal-range block scales
    s = rng.choice(normal, size=(n, k // 16))
    s[0, 0] = 448.0
    return (v * s[:, :, None] * g).reshape(n, k).astype(F32), s


@pytest.mark.parametrize("g", [1.0, 2.0 ** -7, 2.0 ** 3])
def test_lossless_inputs_round_trip_exactly(g):
    rng = np.random.default_rng(3)
    x, s = _lossless_matrix(rng, 8, 256, g)
    codes, scales, g_got = nvfp4.quantize_weight(x)
    assert g_got == np.float32(g)
    np.testing.assert_array_equal(nvfp4.e4m3_decode(scales), s.astype(F32))
    np.testing.assert_array_equal(nvfp4.dequantize(codes, scales, g_got), x)


def test_block_max_maps_to_six_and_idempotence():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((64, 512)) * rng.uniform(0.01, 10, size=(64, 1))).astype(F32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    codes, scales, g = nvfp4.quantize_weight(x)
    q = nvfp4.unpack_codes(codes).reshape(64, 32, 16)
    s = nvfp4.e4m3_decode(scales)
    xb = np.abs(x.reshape(64, 32, 16))
    # for blocks whose scale is a normal E4M3 number, the ratio amax / (S*6)
    # lies in [1/1.0625, 1.0625] and the block maximum rounds to code +-6
    normal = s >= 2.0 ** -6
    imax = np.argmax(xb, axis=2)
    top = np.take_along_axis(q, imax[:, :, None], axis=2)[:, :, 0] & 7
    assert np.all(top[normal] == 7)
    # quantise(dequantise(q)) == q for those blocks
    xd = nvfp4.dequantize(codes, scales, g)
    c2, s2 = nvfp4.quantize(xd, g)
    rows_ok = np.all(normal, axis=1)
    np.testing.assert_array_equal(c2[rows_ok], codes[rows_ok])
    np.testing.assert_array_equal(s2[rows_ok], scales[rows_ok])


def test_error_bound_half_step():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((32, 1024)) * 0.02).astype(F32)
    x[rng.random(x.shape) < 0.01] *= 25
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    codes, scales, g = nvfp4.quantize_weight(x)
    xd = nvfp4.dequantize(codes, scales, g).astype(np.float64)
    q = nvfp4.unpack_codes(codes) & 7
    S = np.repeat((nvfp4.e4m3_decode(scales).astype(np.float64) * float(g)), 16, axis=1)
    step = np.select([q < 4, q < 6], [0.5, 1.0], 2.0)
    y = np.abs(x.astype(np.float64)) / np.where(S == 0, 1, S)
    err = np.abs(x - xd)
    inner = y <= 6.0
    # half a grid step times S, plus the fp32 roundings of S, 1/S, y, and S*q
    slack = 4 * np.finfo(np.float32).eps * np.abs(x)
    assert np.all(err[inner] <= 0.5 * step[inner] * S[inner] + slack[inner] + 1e-30)
    sat = ~inner
    assert np.all(err[sat] <= np.abs(x[sat]) - 6 * S[sat] + slack[sat] + 1e-30)


def test_zero_tensor():
    codes, scales, g = nvfp4.quantize_weight(np.zeros((2, 32), F32))
    assert g == 0 and not codes.any() and not scales.any()


def test_bf16_round_matches_torch_for_fp32_inputs():
    rng = np.random.default_rng(6)
    v = rng.standard_normal(1 << 16).astype(F32) * 10.0 ** rng.integers(-5, 5, size=1 << 16)
    ref = torch.from_numpy(v.astype(F32)).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(nvfp4.bf16_round(v), ref)


def test_bf16_round_single_rounding_of_fp64():
    # 1 + 2^-8 + 2^-30: an fp32 first rounding would drop 2^-30 and make this
    # an exact tie (-> 1.0); one rounding of the fp64 value goes up.
    v = np.array([1 + 2.0 ** -8 + 2.0 ** -30], np.float64)
    assert nvfp4.bf16_round(v)[0] == np.float32(1 + 2.0 ** -7)
