"""Device conversions and the router's sigmoid against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

from _util import capi, host, require_cuda
from oracle import moe, nvfp4
from test_oracle_nvfp4 import _e2m1_probe_values, _e4m3_probe_values

pytestmark = pytest.mark.gpu


def test_e2m1_hardware_rounding_equals_midpoint_rule_on_every_fp32():
    require_cuda()
    c = capi()
    n, ex = c.nvfp4_test_e2m1_sweep(0, 1 << 32)
    assert n == 0, f"{n} fp32 patterns convert differently, e.g. 0x{ex:08x}"


def test_e2m1_device_codes_match_oracle():
    require_cuda()
    c = capi()
    y = _e2m1_probe_values()
    hw, sw = c.nvfp4_test_e2m1(torch.from_numpy(y).cuda())
    ref = nvfp4.e2m1_encode(y)
    bad = np.nonzero(host(hw) != ref)[0]
    assert bad.size == 0, f"{bad.size} differ, e.g. y={y[bad[:5]]} gpu={host(hw)[bad[:5]]} oracle={ref[bad[:5]]}"
    np.testing.assert_array_equal(host(sw), ref)


def test_e4m3_device_codes_match_oracle():
    require_cuda()
    c = capi()
    s = _e4m3_probe_values()
    s = np.concatenate([s, np.array([0.0, 1e30, np.inf, 448.0, 464.0, 470.0], np.float32)])
    codes, val = c.nvfp4_test_e4m3(torch.from_numpy(s).cuda())
    np.testing.assert_array_equal(host(codes), nvfp4.e4m3_encode(s))
    np.testing.assert_array_equal(host(val), nvfp4.e4m3_decode(nvfp4.e4m3_encode(s)))


def test_router_sigmoid_bit_exact():
    require_cuda()
    c = capi()
    rng = np.random.default_rng(7)
    bf = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    bf = bf[np.isfinite(bf) & (np.abs(bf) < 120)]
    l = np.concatenate([rng.uniform(-100, 100, 1 << 20).astype(np.float32),
                        rng.standard_normal(1 << 18).astype(np.float32) * 3, bf,
                        np.array([0.0, -0.0, 80.0, -80.0, 88.0, -88.0, 1e-30], np.float32)])
    got = host(c.nvfp4_test_sigmoid(torch.from_numpy(l).cuda()))
    ref = moe.sigmoid_f32(l)
    bad = np.nonzero(got.view(np.uint32) != ref.view(np.uint32))[0]
    assert bad.size == 0, f"{bad.size} differ, e.g. l={l[bad[:4]]} gpu={got[bad[:4]]} oracle={ref[bad[:4]]}"


def _scale_div_g_values():
    """Global scales g that span the quotient's range: weights' and
    activations' usual 1e-6..1e2, the edges of the three-instruction path
    (6 g = 2^-60 and 2^100, one ulp either side), zero, subnormal and huge."""
    rng = np.random.default_rng(21)
    g = list(np.float32(10.0) ** rng.uniform(-12, 6, 300).astype(np.float32))
    g += [np.float32(np.float32(a) / np.float32(2688)) for a in (0.02, 0.1, 0.5, 1.0, 20.0, 448.0, 3.3e4)]
    for d in (2.0 ** -60, 2.0 ** 100):
        d32 = np.float32(d)
        for nd in (np.nextafter(d32, np.float32(0)), d32, np.nextafter(d32, np.float32(np.inf))):
            g.append(np.float32(nd / np.float32(6)))
    g += [np.float32(0), np.float32(1e-41), np.float32(1e-39), np.float32(1e37), np.float32(3e38)]
    return np.array(g, np.float32)


def test_block_scale_division_matches_ieee_division():
    """The quantisers compute s_raw = amax / (6 g) with Markstein's
    correction of the product by the correctly rounded reciprocal (three
    instructions) where 6 g lies in [2^-60, 2^100].  Only the quotient's E4M3
    code is used.  Against CUDA's IEEE division: the same E4M3 code
    everywhere, and the same quotient, bit for bit, on [2^-20, 464).  Below
    2^-20 (far under half the smallest E4M3 value, 2^-10, so the code is 0
    either way) the method's exactness conditions do not hold for subnormal
    operands; at 464 and above every quotient saturates to the code of 448.
    amax runs over every finite non-negative bf16 value (the weight and
    activation quantisers take the max of bf16 inputs) and over random fp32
    values (the intermediate h is fp32)."""
    require_cuda()
    c = capi()
    gs = _scale_div_g_values()
    bf16_vals = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    rng = np.random.default_rng(22)
    f32_vals = (rng.integers(0, 0x7F800000, 1 << 16, dtype=np.uint32)).view(np.float32)
    for vals in (bf16_vals, f32_vals):
        a = np.tile(vals, len(gs))
        g = np.repeat(gs, len(vals))
        ql, qi, cl, ci = (t.cpu().numpy() for t in c.nvfp4_test_block_scale_div(torch.from_numpy(a).cuda(),
                                                                                  torch.from_numpy(g).cuda()))
        below = qi < np.float32(464)
        exact = below & (qi >= np.float32(2.0 ** -20))
        bad = exact & (ql.view(np.uint32) != qi.view(np.uint32))
        assert not bad.any(), (f"{int(bad.sum())} quotients differ, e.g. amax={a[bad][0]!r} g={g[bad][0]!r}: "
                               f"{ql[bad][0]!r} vs {qi[bad][0]!r}")
        np.testing.assert_array_equal(cl, ci)
        assert np.all(ql[~below] >= np.float32(448))
        assert exact.sum() > 0.05 * len(a)          # over a million pairs in the exact range
