"""Routed-expert MoE layer with NVFP4 W4A4 experts (test infrastructure only).

Sources
-------
* "K-EXAONE-152B-A23B-REAP-80E-BF16" model card, section "Pruning Setup":
  router parameters are ``gate.weight`` and ``e_score_correction_bias``; routing
  is renormalised sigmoid routing with sigmoid-and-bias routing weights and a
  ``routed_scaling_factor``.
* "K-EXAONE-152B-A23B-REAP-80E-NVFP4" model card, section "Quantization Setup":
  the router (``mlp.gate``) stays BF16; routed experts are NVFP4 W4A4 with
  activations dynamically quantised under calibrated global scales.

Readings taken where the pages are silent:

R8  one caller-supplied fp32 global scale per activation tensor: g1 for the
    layer input x, g2 for the intermediate h.
R9  routing arithmetic: logits L = x W_g^T (fp64 sum rounded to fp32), plus an
    optional per-expert offset (a synthetic knob that skews expert loads, not
    part of the method); sigma(l) = 1 / (1 + E(-l)) with E the fp32 exp of
    ``exp_f32`` below; selection by c = sigma + b (bias for selection only),
    the k largest c, ties to the lower expert index, output in descending c;
    weights w_j = (sigma_j / sum) * rsf with sum the fp32 sum of the selected
    sigmas in output order.  No group-limited selection, no epsilon.
R10 gate and up are separate expert Linears with separate global scales.
R11 h = silu(gate) * up is formed in fp64 and rounded once to fp32 before it
    is re-quantised (no bf16 rounding).
R12 the routing weight scales each expert's down-projection output; the
    combine sums the k weighted rows of a token in slot order.
R13 each expert's rows are padded to a multiple of 128; padded rows hold no
    token (perm = -1) and never reach the output.
R16 activation global scales, beyond R8 (the extension "per-expert
    activation global scales plus an on-device dynamic amax mode"): g1 and g2
    may instead be one fp32 per expert, the rows of expert e quantised under
    g1[e] and g2[e]; in the dynamic modes g1 is derived from the batch itself
    with the weight rule R1, g1 = fl32(amax / 2688), over the whole batch x
    ("dynamic") or over the tokens routed to each expert ("dynamic_expert";
    an expert without tokens gets 0).  h keeps a caller-supplied g2.
R19 the shared expert (the model cards keep "shared experts" in BF16; their
    size is not on the pages): one SiLU-gated MLP of the routed experts'
    shape, bf16 weights gate_s, up_s [I_s, H] and down_s [H, I_s], applied to
    every token: y_s = down_s (bf16(silu(gate_s x) * up_s x)), the
    intermediate rounded once to bf16 (the operand of a bf16 matmul); the
    layer output is bf16(y_s + sum_j w_j y_j).
"""
from __future__ import annotations

import math

import numpy as np

from . import nvfp4

F32 = np.float32
ROW_TILE = 128

# ---------------------------------------------------------------------------
# fp32 exp built from IEEE operations only (R9): Cody & Waite argument
# reduction by ln 2, then the degree-7 Taylor polynomial of e^r in Horner form.
# The constants are derived here from ln 2 and 1/j!; nothing else is assumed.
# ---------------------------------------------------------------------------
LOG2E = F32(1.0 / math.log(2.0))
LN2_HI = F32(45426.0 / 65536.0)                 # ln 2 to 16 significant bits
LN2_LO = F32(math.log(2.0) - 45426.0 / 65536.0)  # the remainder
EXP_COEF = [F32(1.0 / math.factorial(j)) for j in range(8)]
EXP_CLAMP = F32(80.0)


def exp_f32(v: np.ndarray) -> np.ndarray:
    """e^v in fp32 with one rounding per IEEE operation, no fused multiply-add.

    n = rint(v log2 e); r = (v - n ln2_hi) - n ln2_lo; p(r) = sum_j r^j / j!
    by Horner; result p * 2^n (2^n built exactly).  |v| is clamped to 80 so
    2^n stays a normal fp32 number."""
    v = np.clip(np.asarray(v, dtype=F32), -EXP_CLAMP, EXP_CLAMP).astype(F32)
    n = np.rint((v * LOG2E).astype(F32)).astype(F32)
    r = ((v - (n * LN2_HI).astype(F32)).astype(F32) - (n * LN2_LO).astype(F32)).astype(F32)
    p = np.full_like(r, EXP_COEF[7])
    for j in range(6, -1, -1):
        p = ((p * r).astype(F32) + EXP_COEF[j]).astype(F32)
    two_n = np.ldexp(F32(1.0), n.astype(np.int32)).astype(F32)
    return (p * two_n).astype(F32)


def sigmoid_f32(l: np.ndarray) -> np.ndarray:
    """sigma(l) = 1 / (1 + e^-l) in fp32 (R9)."""
    e = exp_f32(-np.asarray(l, dtype=F32))
    return (F32(1.0) / (F32(1.0) + e).astype(F32)).astype(F32)


def router_logits(x: np.ndarray, router_weight: np.ndarray,
                  logit_offset: np.ndarray | None = None) -> np.ndarray:
    """L = x W_g^T, accumulated in fp64 and rounded to fp32 (router kept BF16,
    model card "Quantization Setup": "Router modules, including mlp.gate").
    ``logit_offset`` [E] is added in fp32 when given (synthetic load skew)."""
    L = (np.asarray(x, np.float64) @ np.asarray(router_weight, np.float64).T).astype(F32)
    if logit_offset is not None:
        L = (L + np.asarray(logit_offset, F32)[None, :]).astype(F32)
    return L


def route(logits: np.ndarray, bias: np.ndarray, k: int, rsf: float):
    """Top-k sigmoid-plus-bias routing with renormalised, scaled weights (R9).

    Follows "Routing behavior" in the BF16 model card's "Pruning Setup":
    renormalised sigmoid routing, sigmoid-and-bias routing weights,
    routed_scaling_factor.  Returns (topk_idx int32 [T,k], topk_w fp32 [T,k])."""
    logits = np.asarray(logits, F32)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    sig = sigmoid_f32(logits)
    c = (sig + np.asarray(bias, F32)[None, :]).astype(F32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), F32)
    experts = np.arange(E)
    for t in range(T):
        order = np.lexsort((experts, -c[t].astype(np.float64)))   # c desc, index asc
        sel = order[:k]
        idx[t] = sel
        s_sel = sig[t, sel]
        total = F32(0.0)
        for j in range(k):
            total = F32(total + s_sel[j])
        w[t] = ((s_sel / total).astype(F32) * F32(rsf)).astype(F32)
    return idx, w


def permute(topk_idx: np.ndarray, num_experts: int, tile: int = ROW_TILE):
    """Token permutation by expert (R13).

    Pairs (token t, slot j) are ordered by expert, then token, then slot; each
    expert's segment is padded to a multiple of ``tile`` rows.  Returns
    (expert_offsets int32 [E+1], perm int32 [rows], inv_perm int32 [T,k]) with
    perm = -1 on padded rows and rows = expert_offsets[E]."""
    topk_idx = np.asarray(topk_idx, np.int64)
    T, k = topk_idx.shape
    counts = np.bincount(topk_idx.ravel(), minlength=num_experts)[:num_experts]
    padded = -(-counts // tile) * tile
    offsets = np.zeros(num_experts + 1, np.int64)
    offsets[1:] = np.cumsum(padded)
    perm = np.full(int(offsets[-1]), -1, np.int32)
    inv_perm = np.empty((T, k), np.int32)
    fill = offsets[:-1].copy()
    for t in range(T):                      # token order, then slot order
        for j in range(k):
            e = topk_idx[t, j]
            perm[fill[e]] = t
            inv_perm[t, j] = fill[e]
            fill[e] += 1
    return offsets.astype(np.int32), perm, inv_perm


# ---------------------------------------------------------------------------
# Expert GEMMs on quantised operands.
# ---------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z), fp64."""
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(-z))


def block_scaled_matmul(a_codes, a_scales, b_codes, b_scales) -> np.ndarray:
    """sum_k (qa sa)(qb sb) in fp64: a block-scaled FP4 product before global
    scales.  A [M, K] against B [N, K] (both K-contiguous) -> [M, N]."""
    A = nvfp4.dequantize_unscaled(a_codes, a_scales)
    B = nvfp4.dequantize_unscaled(b_codes, b_scales)
    return A @ B.T


def expert_gate_up(a_codes, a_scales, g1, gate, up):
    """Grouped GEMM1 for one expert.  ``gate``/``up`` are (codes, scales, g).

    Returns (gate fp64 [M, I], up fp64 [M, I], h fp32 [M, I]) with
    h = silu(gate) * up (R10, R11)."""
    gate_acc = block_scaled_matmul(a_codes, a_scales, gate[0], gate[1])
    up_acc = block_scaled_matmul(a_codes, a_scales, up[0], up[1])
    gate_v = gate_acc * (float(g1) * float(gate[2]))
    up_v = up_acc * (float(g1) * float(up[2]))
    h = (silu(gate_v) * up_v).astype(F32)
    return gate_v, up_v, h


def expert_down(h_codes, h_scales, g2, down) -> np.ndarray:
    """Grouped GEMM2 for one expert: y = dq(h) dq(W2)^T, fp64 [M, H]."""
    acc = block_scaled_matmul(h_codes, h_scales, down[0], down[1])
    return acc * (float(g2) * float(down[2]))


def activation_scales(x, g1, num_experts, topk_idx_all=None):
    """The x global scale(s) of R8/R16: a scalar or [E] array as given, or
    derived from the batch ``x`` ([T, H], all tokens) for "dynamic" (one
    scalar) and "dynamic_expert" (one per expert over the tokens that
    ``topk_idx_all`` [T, k] routes to it)."""
    if isinstance(g1, str):
        x = np.abs(np.asarray(x, F32))
        if g1 == "dynamic":
            return F32(F32(x.max() if x.size else 0) / nvfp4.GLOBAL_DIVISOR)
        if g1 == "dynamic_expert":
            tmax = x.max(axis=1) if x.size else np.zeros(x.shape[0], F32)
            g = np.zeros(num_experts, F32)
            for e in range(num_experts):
                t = np.nonzero(np.any(topk_idx_all == e, axis=1))[0]
                g[e] = F32(F32(tmax[t].max()) / nvfp4.GLOBAL_DIVISOR) if t.size else F32(0)
            return g
        raise ValueError(f"unknown activation scale mode {g1!r}")
    return np.asarray(g1, F32) if np.ndim(g1) else F32(g1)


def _scale_of(g, e):
    """The global scale of expert e: g itself when per tensor, g[e] when per expert."""
    return F32(g[e]) if np.ndim(g) else F32(g)


def shared_expert(x, shared) -> np.ndarray:
    """R19: y_s [N, H] fp64 for rows x [N, H]; ``shared`` = (gate [I_s, H],
    up [I_s, H], down [H, I_s]) holding bf16 values."""
    gate, up, down = (np.asarray(t, np.float64) for t in shared)
    xd = np.asarray(x, np.float64)
    h = silu(xd @ gate.T) * (xd @ up.T)
    return nvfp4.bf16_round(h).astype(np.float64) @ down.T


def moe_layer(x, router_weight, bias, k, rsf, experts, g1, g2,
              logit_offset=None, tokens=None, logits=None, topk_idx_all=None, shared=None):
    """The NVFP4 W4A4 routed-expert layer for the tokens ``tokens`` (all if None).

    ``experts(e)`` returns ((gate codes, scales, g), (up ...), (down ...)) for
    expert e, canonical layouts.  ``g1`` is the x global scale: a scalar (R8),
    an [E] array, or "dynamic" / "dynamic_expert" (R16); ``g2`` (for h) is a
    scalar or an [E] array.  The rows of expert e are quantised under its
    scales.  Returns a dict with ``out`` (bf16 values as fp32, [len(tokens),
    H]), the routing, each token's per-slot h and y, and the scales used.

    Because routing is per token, evaluating a subset of tokens is exact; the
    dynamic modes take their amax over the whole batch ``x``, and
    "dynamic_expert" needs the routing of every token (``topk_idx_all``,
    computed here when not given).  ``shared`` adds the shared expert (R19)."""
    x = np.asarray(x, F32)
    T, H = x.shape
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    if logits is None:
        logits = router_logits(x[tok], router_weight, logit_offset)
    topk_idx, topk_w = route(logits, bias, k, rsf)
    E = len(bias)
    if isinstance(g1, str) and g1 == "dynamic_expert" and topk_idx_all is None:
        topk_idx_all = route(router_logits(x, router_weight, logit_offset), bias, k, rsf)[0]
    g1 = activation_scales(x, g1, E, topk_idx_all)
    g2 = np.asarray(g2, F32) if np.ndim(g2) else F32(g2)
    per_expert_x = np.ndim(g1) > 0
    if not per_expert_x:
        a_codes, a_scales = nvfp4.quantize(x[tok], g1)
    else:
        a_codes = a_scales = None
    cache = {}
    out = np.zeros((len(tok), H), np.float64)
    h_all, y_all = {}, {}
    for e in np.unique(topk_idx):
        rows = np.nonzero(topk_idx == e)
        ti, sj = rows
        if e not in cache:
            cache[e] = experts(int(e))
        gate, up, down = cache[e]
        g1e, g2e = _scale_of(g1, e), _scale_of(g2, e)
        if per_expert_x:
            ac, asc = nvfp4.quantize(x[tok[ti]], g1e)
        else:
            ac, asc = a_codes[ti], a_scales[ti]
        _, _, h = expert_gate_up(ac, asc, g1e, gate, up)
        hc, hs = nvfp4.quantize(h, g2e)
        y = expert_down(hc, hs, g2e, down)
        for r in range(len(ti)):
            out[ti[r]] += float(topk_w[ti[r], sj[r]]) * y[r]
            h_all[(int(tok[ti[r]]), int(sj[r]))] = h[r]
            y_all[(int(tok[ti[r]]), int(sj[r]))] = y[r]
    if shared is not None:
        out += shared_expert(x[tok], shared)
    return {"out": nvfp4.bf16_round(out), "out_f64": out, "topk_idx": topk_idx,
            "topk_w": topk_w, "logits": logits, "h": h_all, "y": y_all,
            "a_codes": a_codes, "a_scales": a_scales, "g1": g1, "g2": g2, "tokens": tok}


def reap_saliency(result: dict, num_experts: int):
    """REAP saliency accumulators of one batch ("K-EXAONE-152B-A23B-REAP-80E-BF16"
    model card, "Pruning Setup": saliency = mean(topk_weight * ||f_e(x)||_2)
    over routed tokens, with the real sigmoid-and-bias routing weights and the
    routed_scaling_factor included).  From a ``moe_layer`` result: f_e(x) is
    the expert's down-projection output y (before the routing weight) and
    topk_weight the routing weight w (which carries rsf).  Returns
    (sum [E] fp64 of w * ||y||_2, count [E]); the saliency is sum / count over
    all calibration batches (0 where count is 0)."""
    total = np.zeros(num_experts, np.float64)
    count = np.zeros(num_experts, np.int64)
    idx, w = result["topk_idx"], result["topk_w"]
    row_of = {int(t): n for n, t in enumerate(result["tokens"])}
    for (t, j), y in result["y"].items():
        n = row_of[t]
        e = int(idx[n, j])
        total[e] += float(w[n, j]) * float(np.sqrt(np.sum(np.asarray(y, np.float64) ** 2)))
        count[e] += 1
    return total, count


def reap_keep(saliency: np.ndarray, keep: int) -> np.ndarray:
    """Experts retained by REAP pruning: the ``keep`` highest saliencies (ties
    to the lower index), returned in their original order so that the sliced
    gate.weight / e_score_correction_bias / expert tensors keep their relative
    order ("gate.weight sliced according to retained experts")."""
    s = np.asarray(saliency, np.float64)
    order = sorted(range(s.size), key=lambda e: (-s[e], e))
    return np.array(sorted(order[:keep]), dtype=np.int64)


def dense_moe_layer(x, router_weight, bias, k, rsf, experts_bf16,
                    logit_offset=None, tokens=None):
    """The same layer without any quantisation (fp64 throughout), for the loose
    sanity bound only.  ``experts_bf16(e)`` returns (gate [I,H], up [I,H],
    down [H,I]) as bf16 values."""
    x = np.asarray(x, F32)
    tok = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    logits = router_logits(x[tok], router_weight, logit_offset)
    topk_idx, topk_w = route(logits, bias, k, rsf)
    out = np.zeros((len(tok), x.shape[1]), np.float64)
    for t in range(len(tok)):
        xt = x[tok[t]].astype(np.float64)
        for j in range(k):
            gw, uw, dw = experts_bf16(int(topk_idx[t, j]))
            h = silu(np.asarray(gw, np.float64) @ xt) * (np.asarray(uw, np.float64) @ xt)
            out[t] += float(topk_w[t, j]) * (np.asarray(dw, np.float64) @ h)
    return out
