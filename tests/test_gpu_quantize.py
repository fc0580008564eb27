"""Activation and weight quantisers against the oracle, bit for bit."""
import json
import os

import numpy as np
import pytest
import torch

from _util import capi, host, require_cuda, staged_to_canonical, tiled_rows, tiled_to_canonical
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import nvfp4

pytestmark = pytest.mark.gpu
F32 = np.float32


def _bf16(shape, seed, name, std=1.0, outlier_p=0.0):
    x = workloads.random_floats(shape, seed, name, std=std)
    if outlier_p:
        m = workloads.random_floats(shape, seed, name + "/m").abs() > 3.29   # ~0.1%
        x = torch.where(m, x * 20, x)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("layout", ["canonical", "tiled"])
@pytest.mark.parametrize("rows,cols", [(1, 64), (37, 512), (300, 1024), (129, 6144)])
@pytest.mark.parametrize("g_mode", ["calibrated", "saturating", "zero"])
def test_activation_quantiser_matches_oracle(layout, rows, cols, g_mode):
    require_cuda()
    c = capi()
    x = _bf16((rows, cols), 11, f"act{rows}x{cols}", outlier_p=0.001)
    xf = x.float().numpy()
    amax = F32(np.abs(xf).max())
    g = {"calibrated": F32(amax / F32(2688)), "saturating": F32(amax / F32(2688 * 8)), "zero": F32(0)}[g_mode]
    codes, scales = c.nvfp4_quantize_act(x.cuda(), torch.tensor([g]).cuda(), layout)
    rc, rs = nvfp4.quantize(xf, g)
    np.testing.assert_array_equal(host(codes), rc)
    s = host(scales)
    if layout == "tiled":
        np.testing.assert_array_equal(tiled_to_canonical(s, rows, cols), rs)
        rp = (rows + 127) // 128 * 128
        assert not tiled_to_canonical(s, rp, cols)[rows:].any()     # padding rows hold scale 0
    else:
        np.testing.assert_array_equal(s, rs)


def test_activation_quantiser_hand_examples():
    require_cuda()
    c = capi()
    with open(os.path.join(os.path.dirname(__file__), "golden", "nvfp4_hand_examples.json")) as f:
        cases = [cc for cc in json.load(f)["cases"] if cc["kind"] == "activation"]
    for case in cases:
        x = np.array([[float(v) for v in r] for r in case["x"]], F32)
        x = np.pad(x, ((0, 0), (0, 64 - x.shape[1])))
        g = np.array([int(case["g_bits"], 16)], np.uint32).view(F32)
        codes, scales = c.nvfp4_quantize_act(torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(g).cuda())
        nb = len(case["codes_hex"][0]) // 2
        assert host(codes)[0, :nb].tobytes().hex() == case["codes_hex"][0]
        assert host(scales)[0, : len(case["scales_hex"][0]) // 2].tobytes().hex() == case["scales_hex"][0]


@pytest.mark.parametrize("layout", ["canonical", "tiled", "staged"])
def test_weight_quantiser_matches_oracle(layout):
    require_cuda()
    c = capi()
    w = _bf16((4, 256, 512), 12, "wq", std=0.02)
    w[2] = 0                                        # an all-zero matrix
    w[3] = torch.where(workloads.random_floats((256, 512), 12, "wq3").abs() > 2.6, w[3] * 25, w[3])
    codes, scales, g = c.nvfp4_quantize_weights(w.cuda(), layout)
    wf = w.float().numpy()
    sc = host(scales)
    for m in range(4):
        rc, rs, rg = nvfp4.quantize_weight(wf[m])
        assert host(g)[m].view(np.uint32) == np.float32(rg).view(np.uint32), m
        got = staged_to_canonical(host(codes)[m], 256, 512) if layout == "staged" else host(codes)[m]
        np.testing.assert_array_equal(got, rc)
        if layout != "canonical":
            np.testing.assert_array_equal(tiled_to_canonical(sc, 4 * 256, 512)[m * 256:(m + 1) * 256], rs)
        else:
            np.testing.assert_array_equal(sc[m], rs)


def test_weight_quantiser_tiny_layer():
    require_cuda()
    c = capi()
    cfg = workloads.CONFIGS["tiny"]
    gate, up, down = workloads.stacked_expert_weights(cfg)
    for w in (gate, up, down):
        codes, scales, g = c.nvfp4_quantize_weights(w.cuda(), "tiled")
        n, rows, cols = w.shape
        for m in range(n):
            rc, rs, rg = nvfp4.quantize_weight(w[m].float().numpy())
            assert host(g)[m] == rg
            np.testing.assert_array_equal(host(codes)[m], rc)
            np.testing.assert_array_equal(tiled_to_canonical(host(scales), n * rows, cols)[m * rows:(m + 1) * rows],
                                          rs)


def test_weight_quantiser_full_layer_sampled():
    """The offline quantiser on the full 80-expert layer (3.0e9 parameters),
    as the benchmark runs it (staged codes, tiled scales): every global scale
    checked, and 16 rows of six matrices compared code by code."""
    require_cuda()
    c = capi()
    cfg = workloads.CONFIGS["quantiser"]
    gate, up, down = workloads.stacked_expert_weights(cfg, device="cuda")
    rng = np.random.default_rng(0)
    for name, w in (("gate", gate), ("up", up), ("down", down)):
        codes, scales, g = c.nvfp4_quantize_weights(w, "staged")
        torch.cuda.synchronize()
        n, rows, cols = w.shape
        amax = w.abs().amax(dim=(1, 2)).float().cpu().numpy()       # exact (a max of bf16 values)
        ref_g = (amax.astype(F32) / F32(2688)).astype(F32)
        np.testing.assert_array_equal(host(g), ref_g)
        for m in rng.choice(n, 2, replace=False):
            r = np.sort(rng.choice(rows, 16, replace=False))
            rc, rs = nvfp4.quantize(w[m, r].float().cpu().numpy(), ref_g[m])
            np.testing.assert_array_equal(staged_to_canonical(host(codes[m]), rows, cols)[r], rc)
            sc = tiled_rows(host(scales), m * rows + r, cols)
            np.testing.assert_array_equal(sc, rs)
        del codes, scales
    del gate, up, down
    torch.cuda.empty_cache()
