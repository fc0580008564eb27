"""NVFP4 encoding, written out from its definition (test infrastructure only).

Sources
-------
* "K-EXAONE-152B-A23B-REAP-80E-NVFP4" model card, section "Quantization Setup":
  weights are FP4 E2M1 in groups of 16 with FP8 E4M3 block scales, activations
  are dynamically quantised to FP4 under calibrated global scales, weights use
  round-to-nearest (RTN) and each routed expert Linear is quantised on its own.
* "[NetsPresso AQ Deep Dive] How to Quantize the K-EXAONE-236B Model to 4-Bit
  (NVFP4)", section "The Standard NVFP4 Serving Spec": NVFP4 combines a global
  scale with a block scale (a double-scale structure).

Readings taken where the pages are silent (each is one line of the design
notes):

R1  global scale of a weight tensor  g = amax(|w|) / (6 * 448), in fp32, so
    that the largest block scale lands on the top of the E4M3 range.
R2  scale arithmetic, in fp32 with one rounding per operation:
      d = 6 g;  s_raw = amax_block / d (0 if d == 0);  s = E4M3(s_raw);
      S = s * g;  inv = 1 / S (0 if S == 0);  y = x * inv;  q = E2M1(y).
R3  E4M3 conversion: round to nearest, ties to the even code, saturate to 448,
    subnormals kept, the sign bit always 0 (block scales are magnitudes).
R4  E2M1 conversion: nearest value of {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the
    even code, magnitudes beyond 6 saturate to 6.
R5  the sign of y is kept in bit 3, including for -0 and tiny negatives.
R6  two codes per byte, the element with the even index in the low nibble.
R7  an all-zero block (or tensor) has scale code 0 and codes 0 / 8.

Every conversion below is the definition (a search over the finite values of
the format), not a bit trick; the tests pin these searches against closed
forms, hand-worked bytes and the error bound.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32

# ---------------------------------------------------------------------------
# The two element formats, as value tables indexed by code.
# ---------------------------------------------------------------------------

#: E2M1 magnitudes for codes 0..7 (sign in bit 3).  1 sign, 2 exponent and
#: 1 mantissa bit, exponent bias 1, no inf/NaN: {0, 0.5} are the subnormal /
#: zero codes, then 1, 1.5, 2, 3, 4, 6.
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def _e4m3_value(code: int) -> float:
    """Value of a non-negative E4M3 code (1 sign, 4 exponent bits with bias 7,
    3 mantissa bits; code 0x7F is NaN and not a finite value)."""
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0:
        return m * 2.0 ** -9            # subnormal: m/8 * 2^(1-7)
    return (1.0 + m / 8.0) * 2.0 ** (e - 7)


#: Values of the finite non-negative E4M3 codes 0x00..0x7E (0x7E = 448).
E4M3_VALUES = np.array([_e4m3_value(c) for c in range(0x7F)], dtype=np.float64)
E4M3_MAX = 448.0
E2M1_MAX = 6.0


def _nearest_code(a: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest table value to each |a|; an exact tie between two
    neighbours goes to the even index.  ``table`` is increasing, so neighbours
    differ in the last index bit and "even index" is "even mantissa"."""
    a = np.asarray(a, dtype=np.float64)
    # the two table values that bracket a (a is clamped into the table range)
    hi = np.clip(np.searchsorted(table, a, side="left"), 1, table.size - 1)
    lo = hi - 1
    d_lo = a - table[lo]                                     # exact in fp64
    d_hi = table[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    return np.where(take_hi, hi, lo).astype(np.uint8)


def e2m1_encode(y: np.ndarray) -> np.ndarray:
    """fp32 -> 4-bit E2M1 code (R4, R5).  Follows the E2M1 element format of the
    model card's "Quantization Setup" ("Weights: FP4 E2M1")."""
    y = np.asarray(y, dtype=F32)
    a = np.abs(y).astype(np.float64)
    a = np.minimum(a, E2M1_MAX)                              # satfinite
    a = np.where(np.isnan(a), 0.0, a)
    mag = _nearest_code(a, E2M1_VALUES)
    sign = np.signbit(y).astype(np.uint8)
    return (mag | (sign << 3)).astype(np.uint8)


def e2m1_decode(q: np.ndarray) -> np.ndarray:
    """4-bit code -> value (exact in fp32)."""
    q = np.asarray(q, dtype=np.uint8)
    v = E2M1_VALUES[q & 7]
    return np.where(q & 8, -v, v).astype(F32)


def e4m3_encode(s: np.ndarray) -> np.ndarray:
    """Non-negative fp32 -> E4M3 block-scale code (R3).  Follows "Block scales:
    FP8 E4M3" in the model card's "Quantization Setup"."""
    a = np.asarray(s, dtype=F32).astype(np.float64)
    a = np.where(np.isnan(a), 0.0, np.abs(a))
    a = np.minimum(a, E4M3_MAX)                              # satfinite
    return _nearest_code(a, E4M3_VALUES)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """E4M3 code (0x00..0x7E) -> value (exact in fp32)."""
    return E4M3_VALUES[np.asarray(code, dtype=np.uint8) & 0x7F].astype(F32)


# ---------------------------------------------------------------------------
# Block quantisation (R2): one fp32 global scale per tensor, one E4M3 scale
# per 16 consecutive elements along K, one E2M1 code per element.
# ---------------------------------------------------------------------------

BLOCK = 16
GLOBAL_DIVISOR = F32(6.0 * 448.0)     # 2688: E2M1 max times E4M3 max (R1)
_ROW_CHUNK = 1024                     # rows per pass (memory bound, no effect on results)


def weight_global_scale(w: np.ndarray) -> np.float32:
    """Per-tensor fp32 global scale of an RTN-quantised weight (R1).

    The NetsPresso article's "double-scale structure" gives the global scale;
    the model card quantises "at per-expert Linear granularity", so ``w`` is
    one expert matrix."""
    amax = F32(np.max(np.abs(np.asarray(w, dtype=F32)))) if np.size(w) else F32(0)
    return F32(amax / GLOBAL_DIVISOR)


def quantize(x: np.ndarray, g) -> tuple[np.ndarray, np.ndarray]:
    """Quantise rows of ``x`` [N, K] (K % 16 == 0) under global scale ``g``.

    Returns (codes uint8 [N, K/2], scales uint8 [N, K/16]) in the canonical
    row-major layout.  Steps R2 in order, one fp32 rounding per operation.
    """
    x = np.asarray(x, dtype=F32)
    if x.ndim != 2 or x.shape[1] % BLOCK:
        raise ValueError("quantize expects [N, K] with K a multiple of 16")
    n, k = x.shape
    if n > _ROW_CHUNK:                       # bound the working memory only
        parts = [quantize(x[i:i + _ROW_CHUNK], g) for i in range(0, n, _ROW_CHUNK)]
        return (np.concatenate([p[0] for p in parts]),
                np.concatenate([p[1] for p in parts]))
    g = F32(g)
    d = F32(F32(6.0) * g)
    xb = x.reshape(n, k // BLOCK, BLOCK)
    amax_b = np.max(np.abs(xb), axis=2)                       # exact
    with np.errstate(divide="ignore", invalid="ignore"):
        s_raw = np.where(d == 0, F32(0), (amax_b / d).astype(F32)).astype(F32)
    s = e4m3_encode(s_raw)
    S = (e4m3_decode(s) * g).astype(F32)
    with np.errstate(divide="ignore"):
        inv = np.where(S == 0, F32(0), (F32(1.0) / S).astype(F32)).astype(F32)
    y = (xb * inv[:, :, None]).astype(F32)
    q = e2m1_encode(y).reshape(n, k)
    return pack_codes(q), s


def quantize_weight(w: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.float32]:
    """Offline RTN quantisation of one expert matrix (model card, "Quantization
    Setup": "Round-to-nearest weight quantization", "Routed expert weights were
    quantized at per-expert Linear granularity").  Returns codes, scales, g."""
    g = weight_global_scale(w)
    codes, scales = quantize(w, g)
    return codes, scales, g


def pack_codes(q: np.ndarray) -> np.ndarray:
    """[N, K] 4-bit codes -> [N, K/2] bytes, even index in the low nibble (R6)."""
    q = np.asarray(q, dtype=np.uint8)
    return (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(b: np.ndarray) -> np.ndarray:
    """[N, K/2] bytes -> [N, K] 4-bit codes (R6)."""
    b = np.asarray(b, dtype=np.uint8)
    q = np.empty((b.shape[0], b.shape[1] * 2), dtype=np.uint8)
    q[:, 0::2] = b & 0xF
    q[:, 1::2] = b >> 4
    return q


def dequantize(codes: np.ndarray, scales: np.ndarray, g) -> np.ndarray:
    """x_hat = (val(q) * s) * g, each product rounded to fp32 (the inner product
    is exact).  The double-scale structure of the NetsPresso article."""
    q = unpack_codes(codes)
    n, k = q.shape
    v = e2m1_decode(q).reshape(n, k // BLOCK, BLOCK)
    s = e4m3_decode(scales)[:, :, None]
    return ((v * s).astype(F32) * F32(g)).astype(F32).reshape(n, k)


def dequantize_unscaled(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """val(q) * s as exact fp64 (no global scale): the operand a block-scaled
    matrix product consumes before the global scales are applied."""
    q = unpack_codes(codes)
    n, k = q.shape
    v = e2m1_decode(q).astype(np.float64).reshape(n, k // BLOCK, BLOCK)
    s = e4m3_decode(scales).astype(np.float64)[:, :, None]
    return (v * s).reshape(n, k)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 or fp64 values to the nearest bfloat16 (ties to even), once,
    returned as fp32.  bfloat16 keeps 8 significant bits of an fp32 exponent
    range; frexp/ldexp keep this a single rounding for fp64 input."""
    v = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(v)                      # v = m * 2^e, 0.5 <= |m| < 1
    r = np.rint(m * 256.0) / 256.0          # 8 significant bits, half to even
    return np.ldexp(r, e).astype(F32)
