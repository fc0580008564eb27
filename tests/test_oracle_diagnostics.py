"""Pins of the block-scale distortion statistics (oracle/diagnostics.py).

The statistics follow the NetsPresso AQ article, section "Why 4-Bit
Quantization of MoE Models Is Hard: Outliers in the Final Two Layers"
(outliers |w| > 0.1; their effect on the block scale and on neighbouring
weights).  Pinned by a hand-worked example, by a per-block scalar restatement
on random tensors, by a lossless case and by invariants that hold for any
tensor."""
import json
import os

import numpy as np
import pytest

from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import diagnostics, nvfp4

F32 = np.float32
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "block_stats_hand_example.json")


def test_hand_worked_example():
    ex = json.load(open(GOLDEN))
    w = np.array(ex["w"], dtype=F32)[None, :]
    codes, scales, g = nvfp4.quantize_weight(w)
    assert float(g) == ex["expected_g"]
    np.testing.assert_array_equal(scales[0], ex["expected_scales"])
    st = diagnostics.block_stats(w, codes, scales, g, ex["tau"])
    for f in diagnostics.INT_FIELDS:
        assert st[f] == ex["expected"][f], f
    for f in diagnostics.FIELDS[len(diagnostics.INT_FIELDS):]:
        assert st[f] == pytest.approx(ex["expected"][f], rel=1e-14, abs=0), f
    # the neighbours of the outlier are wiped out; the clean blocks keep ~2^-5
    e = ex["expected"]
    assert diagnostics.relative_rms(st, "neighbours") == 1.0
    assert diagnostics.relative_rms(st, "clean") == pytest.approx((e["sse_clean"] / e["sum_sq_clean"]) ** 0.5,
                                                                  rel=1e-12)


def _scalar_stats(w, codes, scales, g, tau):
    """The same statistics block by block with Python scalars."""
    q = nvfp4.unpack_codes(codes)
    acc = dict.fromkeys(diagnostics.FIELDS, 0)
    n, k = w.shape
    for r in range(n):
        for b in range(k // 16):
            s = int(scales[r, b])
            sval = float(nvfp4.E4M3_VALUES[s]) if s < 0x7F else float("nan")
            S = F32(F32(sval) * F32(g))
            inv = F32(0) if S == 0 else F32(F32(1) / S)
            vals = [float(w[r, 16 * b + i]) for i in range(16)]
            outl = [abs(v) > float(F32(tau)) for v in vals]
            has = any(outl)
            acc["blocks"] += 1
            acc["outlier_blocks"] += int(has)
            acc["zero_scale_blocks"] += int(s == 0)
            acc["subnormal_scale_blocks"] += int(1 <= s <= 7)
            for i, v in enumerate(vals):
                c = int(q[r, 16 * b + i])
                mag = float(nvfp4.E2M1_VALUES[c & 7])
                dq = float(F32(F32(mag * sval) * F32(g))) * (-1.0 if c & 8 else 1.0)
                e2, s2 = (v - dq) ** 2, v * v
                acc["elements"] += 1
                acc["outliers"] += int(outl[i])
                acc["saturated_elements"] += int(abs(float(F32(F32(v) * inv))) > 6.0)
                acc["sum_sq"] += s2
                acc["sse"] += e2
                if has and not outl[i]:
                    acc["neighbours"] += 1
                    acc["sum_sq_neighbours"] += s2
                    acc["sse_neighbours"] += e2
                if not has:
                    acc["clean"] += 1
                    acc["sum_sq_clean"] += s2
                    acc["sse_clean"] += e2
    return acc


@pytest.mark.parametrize("outlier_p", [0.0, 0.05])
def test_matches_a_per_block_restatement(outlier_p):
    cfg = workloads.LayerConfig("diag", T=1, H=64, I=48, E=1, k=1, w_outlier_p=outlier_p, gen_device="cpu")
    g_, u_, d_ = workloads.expert_weights(cfg, 0, 7, device="cpu")
    w = g_.float().numpy()
    codes, scales, g = nvfp4.quantize_weight(w)
    st = diagnostics.block_stats(w, codes, scales, g)
    ref = _scalar_stats(w, codes, scales, g, 0.1)
    for f in diagnostics.INT_FIELDS:
        assert st[f] == ref[f], f
    for f in diagnostics.FIELDS[len(diagnostics.INT_FIELDS):]:
        assert st[f] == pytest.approx(ref[f], rel=1e-12, abs=1e-300), f
    if outlier_p:
        assert st["outliers"] > 0 and st["outlier_blocks"] > 0


def test_lossless_tensor_has_no_error():
    # on-grid values under a power-of-two global scale quantise exactly
    rng = np.random.default_rng(3)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=F32)
    v = grid[rng.integers(0, 8, size=(8, 64))] * np.where(rng.random((8, 64)) < 0.5, -1, 1).astype(F32)
    v[:, ::16] = 6.0                          # every block reaches 6
    g = F32(2.0 ** -8)                        # block amax 6 g: s = 1, S = g, inv = 2^8, all exact
    w = (v * g).astype(F32)
    codes, scales = nvfp4.quantize(w, g)
    assert np.all(scales == 0x38)
    st = diagnostics.block_stats(w, codes, scales, g, tau=10.0)
    assert st["sse"] == 0.0 and st["outliers"] == 0 and st["saturated_elements"] == 0
    assert st["clean"] == st["elements"] == w.size


def test_invariants_on_an_outlier_heavy_tensor():
    cfg = workloads.LayerConfig("diag", T=1, H=256, I=128, E=1, k=1, w_outlier_p=0.01, gen_device="cpu")
    w = workloads.expert_weights(cfg, 0, 11, device="cpu")[0].float().numpy()
    codes, scales, g = nvfp4.quantize_weight(w)
    st = diagnostics.block_stats(w, codes, scales, g)
    assert st["elements"] == st["outliers"] + st["neighbours"] + st["clean"]
    assert st["clean"] == 16 * (st["blocks"] - st["outlier_blocks"])
    assert st["sse"] >= st["sse_neighbours"] + st["sse_clean"] - 1e-18
    assert st["sum_sq"] >= st["sum_sq_neighbours"] + st["sum_sq_clean"]
    # the page's point: neighbours of outliers lose far more than clean blocks
    assert diagnostics.relative_rms(st, "neighbours") > 3 * diagnostics.relative_rms(st, "clean")
