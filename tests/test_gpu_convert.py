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
