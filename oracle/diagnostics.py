"""Block-scale distortion statistics of an NVFP4 tensor (test infrastructure only).

Source
------
"[NetsPresso AQ Deep Dive] How to Quantize the K-EXAONE-236B Model to 4-Bit
(NVFP4)", section "Why 4-Bit Quantization of MoE Models Is Hard: Outliers in
the Final Two Layers".  It measures the share of expert weights whose
magnitude exceeds 0.1, and it states that concentrated outliers distort the
NVFP4 block scale and degrade the precision of the neighbouring weights in the
same block.

The statistics below make those two statements measurable for one
quantised tensor (w, codes, scales, g).  The pages give no formulas, so the
definitions are readings (listed in the design notes):

* outlier: an element with |w| > tau (tau = 0.1 on the page);
* outlier block: a 16-element block that holds at least one outlier;
* neighbour: a non-outlier element of an outlier block;
* clean element: an element of a block without outliers;
* error: w - dequantize(codes, scales, g), with the fp32 products of the
  double-scale structure (oracle.nvfp4.dequantize), squared and summed in fp64;
* zero / subnormal scale block: scale code 0 / codes 1..7 (E4M3 subnormals);
* saturated element: |y| > 6 where y = fl32(w * inv) and inv = fl32(1 / S),
  S = fl32(E4M3(s) * g): the quantiser's own scaled value, beyond the E2M1
  range, which the conversion clamps to 6.

Integer fields are exact counts; the fp64 sums are exact up to summation
order.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4

F32 = np.float32
BLOCK = nvfp4.BLOCK

#: The fields, in the order the C structure of the library declares them.
FIELDS = ("elements", "outliers", "blocks", "outlier_blocks", "zero_scale_blocks", "subnormal_scale_blocks",
          "saturated_elements", "neighbours", "clean", "sum_sq", "sse", "sum_sq_neighbours", "sse_neighbours",
          "sum_sq_clean", "sse_clean")
INT_FIELDS = FIELDS[:9]


def block_stats(w: np.ndarray, codes: np.ndarray, scales: np.ndarray, g, tau: float = 0.1) -> dict:
    """Statistics of one tensor: ``w`` [N, K] (the values that were quantised),
    ``codes`` [N, K/2] and ``scales`` [N, K/16] (canonical layout), global
    scale ``g``; ``tau`` is the outlier threshold."""
    w = np.asarray(w, dtype=F32)
    n, k = w.shape
    g = F32(g)
    tau = F32(tau)
    wb = w.reshape(n, k // BLOCK, BLOCK)
    dq = nvfp4.dequantize(codes, scales, g).reshape(n, k // BLOCK, BLOCK)
    err2 = (wb.astype(np.float64) - dq.astype(np.float64)) ** 2
    sq = wb.astype(np.float64) ** 2

    out = np.abs(wb) > tau
    out_block = np.any(out, axis=2)
    neighbour = (~out) & out_block[:, :, None]
    clean = ~out_block[:, :, None] & np.ones_like(out)

    s = np.asarray(scales, dtype=np.uint8)
    S = (nvfp4.e4m3_decode(s) * g).astype(F32)
    with np.errstate(divide="ignore"):
        inv = np.where(S == 0, F32(0), (F32(1.0) / S).astype(F32)).astype(F32)
    y = (wb * inv[:, :, None]).astype(F32)

    return {
        "elements": int(w.size),
        "outliers": int(out.sum()),
        "blocks": int(n * (k // BLOCK)),
        "outlier_blocks": int(out_block.sum()),
        "zero_scale_blocks": int((s == 0).sum()),
        "subnormal_scale_blocks": int(((s >= 1) & (s <= 7)).sum()),
        "saturated_elements": int((np.abs(y) > F32(6.0)).sum()),
        "neighbours": int(neighbour.sum()),
        "clean": int(clean.sum()),
        "sum_sq": float(sq.sum()),
        "sse": float(err2.sum()),
        "sum_sq_neighbours": float(sq[neighbour].sum()),
        "sse_neighbours": float(err2[neighbour].sum()),
        "sum_sq_clean": float(sq[clean].sum()),
        "sse_clean": float(err2[clean].sum()),
    }


def relative_rms(stats: dict, part: str = "") -> float:
    """sqrt(sse / sum_sq) of the whole tensor (part ""), of the neighbours
    ("neighbours") or of the clean elements ("clean"); 0 for an empty part."""
    suffix = f"_{part}" if part else ""
    den = stats["sum_sq" + suffix]
    return float(np.sqrt(stats["sse" + suffix] / den)) if den > 0 else 0.0
