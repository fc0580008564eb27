"""Block-scale distortion statistics on the GPU against the oracle.

The inputs (w and its NVFP4 encoding) come from the seeded generator and the
oracle's quantiser, so the oracle and the GPU read the same bytes.  Counts
must agree exactly.  The GPU sums each block in fp32 (the oracle sums every
term in fp64), so the sums agree within the fp32 rounding of 16-term block
sums: 2e-6 relative."""
import json
import os

import numpy as np
import pytest
import torch

from _util import canonical_to_staged, canonical_to_tiled, capi, require_cuda
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import diagnostics, nvfp4

pytestmark = pytest.mark.gpu
F32 = np.float32
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "block_stats_hand_example.json")


def _run(c, mats, layout, tau=0.1):
    """mats: list of (w fp32 [rows, cols] bf16-exact, codes, scales canonical, g)."""
    rows, cols = mats[0][0].shape
    w = torch.from_numpy(np.stack([m[0] for m in mats])).to(torch.bfloat16).cuda()
    if layout == "staged":
        codes = torch.from_numpy(np.stack([canonical_to_staged(m[1], rows, cols) for m in mats])).cuda()
    else:
        codes = torch.from_numpy(np.stack([m[1] for m in mats])).cuda()
    sc = np.concatenate([m[2] for m in mats])
    if layout != "canonical":
        sc = canonical_to_tiled(sc)
    scales = torch.from_numpy(np.ascontiguousarray(sc)).cuda()
    g = torch.tensor([float(m[3]) for m in mats], dtype=torch.float32).cuda()
    st = c.nvfp4_block_stats_compute(w, codes, scales, g, layout, tau)
    return c.block_stats_to_dicts(st)


def _compare(got, ref):
    for f in diagnostics.INT_FIELDS:
        assert got[f] == ref[f], (f, got[f], ref[f])
    for f in diagnostics.FIELDS[len(diagnostics.INT_FIELDS):]:
        assert got[f] == pytest.approx(ref[f], rel=2e-6, abs=1e-300), f


def test_hand_worked_example():
    require_cuda()
    c = capi()
    ex = json.load(open(GOLDEN))
    w = np.array(ex["w"], dtype=F32)[None, :]
    codes, scales, g = nvfp4.quantize_weight(w)
    got = _run(c, [(w, codes, scales, g)], "canonical", ex["tau"])[0]
    _compare(got, ex["expected"])


# (layout, shape) pairs: the staged layout needs cols % 256 == 0, so the
# 128-column shape runs in the other two layouts only
_SHAPES = [(128, 256, 3, 0.01), (256, 128, 2, 0.0), (384, 512, 1, 0.05)]
_CASES = [(lay, *shape) for lay in ("canonical", "tiled", "staged") for shape in _SHAPES
          if lay != "staged" or shape[1] % 256 == 0]


@pytest.mark.parametrize("layout,rows,cols,n,outlier_p", _CASES)
def test_matches_oracle(layout, rows, cols, n, outlier_p):
    require_cuda()
    c = capi()
    cfg = workloads.LayerConfig("diag", T=1, H=cols, I=rows, E=n, k=1, w_outlier_p=outlier_p, gen_device="cpu")
    mats = []
    for e in range(n):
        w = workloads.expert_weights(cfg, e, 5, device="cpu")[0].float().numpy()   # gate [rows, cols]
        codes, scales, g = nvfp4.quantize_weight(w)
        mats.append((w, codes, scales, g))
    got = _run(c, mats, layout)
    for m, gm in zip(mats, got):
        _compare(gm, diagnostics.block_stats(*m))


def test_zero_tensor_and_ragged_share():
    # an all-zero matrix (scale 0 everywhere) next to a tiny one that leaves
    # most threads without a block
    require_cuda()
    c = capi()
    z = np.zeros((1, 16), dtype=F32)
    codes, scales, g = nvfp4.quantize_weight(z)
    got = _run(c, [(z, codes, scales, g)], "canonical")[0]
    _compare(got, diagnostics.block_stats(z, codes, scales, g))
    assert got["zero_scale_blocks"] == 1 and got["sse"] == 0.0


def test_host_side_checks():
    require_cuda()
    c = capi()
    w = torch.zeros((1, 128, 40), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros((1, 128, 20), dtype=torch.uint8, device="cuda")
    sc = torch.zeros(128 * 3, dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    with pytest.raises(c.Nvfp4Error):
        c.nvfp4_block_stats_compute(w, codes, sc, g, "canonical")
