"""Pins for the oracle's router, permutation and layer (CPU only)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe, nvfp4
from nvfp4_w4a4_quantized_moe_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


# --- exp / sigmoid --------------------------------------------------------------

def _ulp_distance(a, b):
    ia = a.astype(F32).view(np.int32).astype(np.int64)
    ib = b.astype(F32).view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


def test_exp_f32_within_two_ulp_of_exact():
    v = np.linspace(-80, 80, 400_001, dtype=np.float64).astype(F32)
    got = moe.exp_f32(v)
    ref = np.exp(v.astype(np.float64)).astype(F32)     # correctly rounded target
    assert _ulp_distance(got, ref).max() <= 2


def test_exp_f32_special_points():
    assert moe.exp_f32(np.array([0.0], F32))[0] == 1.0
    assert moe.exp_f32(np.array([200.0], F32))[0] == moe.exp_f32(np.array([80.0], F32))[0]


def test_sigmoid_close_to_exact_and_monotone():
    l = np.sort(np.random.default_rng(0).uniform(-30, 30, 200_000).astype(F32))
    s = moe.sigmoid_f32(l)
    ref = (1.0 / (1.0 + np.exp(-l.astype(np.float64)))).astype(F32)
    assert _ulp_distance(s, ref).max() <= 3
    assert np.all(np.diff(s) >= 0)
    assert moe.sigmoid_f32(np.array([0.0], F32))[0] == 0.5


# --- routing --------------------------------------------------------------------

def test_route_hand_example():
    with open(os.path.join(GOLDEN, "routing_hand_example.json")) as f:
        g = json.load(f)
    idx, w = moe.route(np.array(g["logits"], F32), np.array(g["bias"], F32), g["k"], g["rsf"])
    np.testing.assert_array_equal(idx, g["topk_idx"])
    np.testing.assert_allclose(w, g["topk_w"], rtol=g["w_rel_tol"])


def test_route_brute_force_over_subsets():
    rng = np.random.default_rng(1)
    E, k = 7, 3
    for _ in range(200):
        logits = rng.standard_normal((1, E)).astype(F32)
        bias = (rng.standard_normal(E) * 0.3).astype(F32)
        idx, w = moe.route(logits, bias, k, 2.5)
        sig = 1.0 / (1.0 + np.exp(-logits[0].astype(np.float64)))
        c = sig + bias
        best = max(itertools.combinations(range(E), k), key=lambda s: (sum(c[list(s)]), [-i for i in s]))
        assert set(idx[0]) == set(best)
        # output order: biased score descending
        assert np.all(np.diff(c[idx[0]]) <= 0)
        # weights are the renormalised unbiased sigmoids times rsf
        ref = 2.5 * sig[idx[0]] / sig[idx[0]].sum()
        np.testing.assert_allclose(w[0], ref, rtol=1e-6)


def test_route_ties_go_to_lower_index():
    logits = np.zeros((1, 6), F32)
    idx, w = moe.route(logits, np.zeros(6, F32), 4, 1.0)
    np.testing.assert_array_equal(idx[0], [0, 1, 2, 3])
    np.testing.assert_array_equal(w[0], np.full(4, 0.25, F32))


def test_route_without_bias_is_top_k_of_logits():
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((64, 80)).astype(F32)
    idx, w = moe.route(logits, np.zeros(80, F32), 8, 2.5)
    ref = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")[:, :8]
    np.testing.assert_array_equal(idx, ref)
    np.testing.assert_allclose(w.sum(axis=1), 2.5, rtol=2e-6)
    assert np.all(w > 0)


# --- permutation ----------------------------------------------------------------

def test_permutation_properties():
    rng = np.random.default_rng(3)
    T, E, k = 300, 10, 3
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    off, perm, inv = moe.permute(idx, E, tile=128)
    counts = np.bincount(idx.ravel(), minlength=E)
    assert off[0] == 0 and np.all(np.diff(off) == -(-counts // 128) * 128)
    assert np.all(off % 128 == 0)
    # every pair lands on a row of its expert holding its token
    for t in range(T):
        for j in range(k):
            r = inv[t, j]
            assert perm[r] == t and off[idx[t, j]] <= r < off[idx[t, j] + 1]
    assert np.unique(inv).size == T * k
    # stable: inside an expert's segment the tokens ascend, padding at the end
    for e in range(E):
        seg = perm[off[e]:off[e + 1]]
        real = seg[seg >= 0]
        assert real.size == counts[e] and np.all(np.diff(real) > 0)
        assert np.all(seg[counts[e]:] == -1)


# --- expert GEMMs and the layer -------------------------------------------------

def _lossless(rng, n, k, g):
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    v = grid[rng.integers(0, 8, size=(n, k // 16, 16))] * rng.choice([-1, 1], size=(n, k // 16, 16))
    v[:, :, 0] = 6.0
    s = rng.choice(nvfp4.E4M3_VALUES[40:70], size=(n, k // 16))
    s[0, 0] = 448.0
    return (v * s[:, :, None] * g).reshape(n, k).astype(F32)


def test_gemm_on_lossless_operands_is_the_exact_product():
    """Inputs on the NVFP4 grid with power-of-two global scales quantise
    without loss, so the quantised gate/up/down equal exact fp64 products."""
    rng = np.random.default_rng(4)
    M, H, I = 16, 128, 64
    g1 = 2.0 ** -3
    x = _lossless(rng, M, H, g1)
    wg = _lossless(rng, I, H, 2.0 ** -12)
    wu = _lossless(rng, I, H, 2.0 ** -11)
    wd = _lossless(rng, H, I, 2.0 ** -10)
    ac, asc = nvfp4.quantize(x, F32(g1))
    gate_q, up_q, down_q = (nvfp4.quantize_weight(w) for w in (wg, wu, wd))
    gate, up, h = moe.expert_gate_up(ac, asc, F32(g1), gate_q, up_q)
    xd = x.astype(np.float64)
    np.testing.assert_array_equal(gate, xd @ wg.astype(np.float64).T)
    np.testing.assert_array_equal(up, xd @ wu.astype(np.float64).T)
    hd = _lossless(rng, M, I, 2.0 ** -5)
    hc, hs = nvfp4.quantize(hd, F32(2.0 ** -5))
    y = moe.expert_down(hc, hs, F32(2.0 ** -5), down_q)
    np.testing.assert_array_equal(y, hd.astype(np.float64) @ wd.astype(np.float64).T)


def _tiny_layer():
    cfg = workloads.CONFIGS["tiny"]
    x = workloads.hidden_states(cfg).float().numpy()
    wg, bias, off = workloads.router_params(cfg)
    wg = wg.float().numpy()
    bias = bias.numpy()
    bf = {e: tuple(t.float().numpy() for t in workloads.expert_weights(cfg, e)) for e in range(cfg.E)}
    q = {e: tuple(nvfp4.quantize_weight(w) for w in bf[e]) for e in range(cfg.E)}
    return cfg, x, wg, bias, bf, q


def test_layer_close_to_unquantised_layer():
    """Loose sanity bound: NVFP4 W4A4 against the same layer in fp64 without
    quantisation.  Four 4-bit roundings leave roughly 10-20% relative error;
    a transposed operand, a dropped global scale or a lost SiLU gives ~100%."""
    cfg, x, wg, bias, bf, q = _tiny_layer()
    g1 = F32(np.abs(x).max() / F32(2688))
    dense = moe.dense_moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: bf[e])
    # calibrate g2 on the unquantised h of this input
    hmax = 0.0
    L = moe.router_logits(x, wg)
    idx, _ = moe.route(L, bias, cfg.k, cfg.rsf)
    for t in range(cfg.T):
        for e in idx[t]:
            h = moe.silu(bf[e][0].astype(np.float64) @ x[t]) * (bf[e][1].astype(np.float64) @ x[t])
            hmax = max(hmax, np.abs(h).max())
    g2 = F32(F32(hmax) / F32(2688))
    res = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], g1, g2)
    rel = np.linalg.norm(res["out_f64"] - dense) / np.linalg.norm(dense)
    assert 0.02 < rel < 0.35, rel
    # the bf16 output is the rounded fp64 sum
    np.testing.assert_array_equal(res["out"], nvfp4.bf16_round(res["out_f64"]))


def test_layer_token_subset_is_exact():
    cfg, x, wg, bias, bf, q = _tiny_layer()
    g1, g2 = F32(0.01), F32(0.0005)
    full = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], g1, g2)
    sub = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], g1, g2, tokens=[3, 17, 30])
    np.testing.assert_array_equal(sub["out"], full["out"][[3, 17, 30]])


# --- activation global scales per expert and from the batch (reading R16) ---

def _zero_except(q, keep):
    """Expert weights with every expert but ``keep`` replaced by zeros."""
    def ex(e):
        if e == keep:
            return q[e]
        return tuple((np.zeros_like(c), np.zeros_like(s), g) for c, s, g in q[e])
    return ex


def test_per_expert_scales_equal_to_one_value_reproduce_the_tensor_mode():
    cfg, x, wg, bias, bf, q = _tiny_layer()
    g1, g2 = F32(0.0023), F32(0.0004)
    ref = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], g1, g2)
    got = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], np.full(cfg.E, g1, F32),
                        np.full(cfg.E, g2, F32))
    np.testing.assert_array_equal(got["out_f64"], ref["out_f64"])


def test_per_expert_scales_sum_of_single_expert_layers():
    """The per-expert layer equals the sum over experts of the per-tensor layer
    run with that expert's (g1, g2) and every other expert zeroed: a second
    route through the per-tensor code for each expert's share."""
    cfg, x, wg, bias, bf, q = _tiny_layer()
    rng = np.random.default_rng(5)
    g1 = (F32(0.002) * (1 + rng.random(cfg.E))).astype(F32)
    g2 = (F32(0.0003) * (1 + rng.random(cfg.E))).astype(F32)
    got = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], g1, g2)
    acc = np.zeros_like(got["out_f64"])
    for e in range(cfg.E):
        acc += moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, _zero_except(q, e), g1[e], g2[e])["out_f64"]
    np.testing.assert_allclose(got["out_f64"], acc, rtol=1e-12, atol=1e-15)


def test_dynamic_scale_is_invariant_to_power_of_two_rescaling():
    """With g1 taken from the batch, x and 2^j x quantise to the same codes
    and block scales: the global scale moves by exactly 2^j."""
    cfg, x, wg, bias, bf, q = _tiny_layer()
    a = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], "dynamic", F32(0.0004))
    b = moe.moe_layer((x * F32(8.0)).astype(F32), wg, bias, cfg.k, cfg.rsf, lambda e: q[e], "dynamic", F32(0.0004),
                      logits=a["logits"])
    assert b["g1"] == a["g1"] * 8
    np.testing.assert_array_equal(a["a_codes"], b["a_codes"])
    np.testing.assert_array_equal(a["a_scales"], b["a_scales"])
    # the batch amax block lands on the top of the E4M3 range
    assert a["a_scales"].max() == 0x7E


def test_dynamic_expert_scales_bound_the_dynamic_scale():
    cfg, x, wg, bias, bf, q = _tiny_layer()
    res = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], "dynamic_expert", np.full(cfg.E, F32(4e-4)))
    g_all = moe.activation_scales(x, "dynamic", cfg.E)
    g = res["g1"]
    assert g.shape == (cfg.E,) and np.all(g <= g_all)
    t_max = int(np.argmax(np.abs(x).max(axis=1)))
    for e in res["topk_idx"][t_max]:
        assert g[e] == g_all                       # experts of the batch-max token
    idle = np.setdiff1d(np.arange(cfg.E), res["topk_idx"])
    assert np.all(g[idle] == 0)
    # a token subset gives the same rows as the whole batch
    sub = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], "dynamic_expert", np.full(cfg.E, F32(4e-4)),
                        tokens=[1, 9])
    np.testing.assert_array_equal(sub["out"], res["out"][[1, 9]])


# --- REAP saliency ("Pruning Setup" of the BF16 model card) ---

def test_reap_saliency_scales_with_the_down_global_scale():
    """f_e(x) is linear in the down projection's global scale: doubling one
    expert's g_down doubles exactly that expert's saliency and no other."""
    cfg, x, wg, bias, bf, q = _tiny_layer()
    g1, g2 = F32(0.003), F32(0.0005)
    base = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], g1, g2)
    q2 = dict(q)
    dc, ds, dg = q[3][2]
    q2[3] = (q[3][0], q[3][1], (dc, ds, F32(dg * 2)))
    doubled = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q2[e], g1, g2)
    s0, n0 = moe.reap_saliency(base, cfg.E)
    s1, n1 = moe.reap_saliency(doubled, cfg.E)
    np.testing.assert_array_equal(n0, n1)
    assert s1[3] == 2 * s0[3]
    other = np.arange(cfg.E) != 3
    np.testing.assert_array_equal(s1[other], s0[other])


def test_reap_saliency_bounds_the_output_norm():
    """sum_e saliency_sum_e = sum_t sum_j ||w_tj y_tj|| >= sum_t ||out_t|| (the
    triangle inequality on the combine), with the counts summing to T k."""
    cfg, x, wg, bias, bf, q = _tiny_layer()
    res = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], F32(0.003), F32(0.0005))
    s, n = moe.reap_saliency(res, cfg.E)
    assert n.sum() == cfg.T * cfg.k
    assert s.sum() >= np.linalg.norm(res["out_f64"], axis=1).sum() * (1 - 1e-12)
    # a token subset gives the part of the accumulators its slots contribute
    sub = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], F32(0.003), F32(0.0005), tokens=[0, 5])
    ss, ns = moe.reap_saliency(sub, cfg.E)
    assert ns.sum() == 2 * cfg.k and np.all(ss <= s + 1e-15)


def test_reap_keep_takes_the_highest_saliencies_in_expert_order():
    s = np.array([0.5, 0.1, 0.9, 0.5, 0.0, 0.7])
    np.testing.assert_array_equal(moe.reap_keep(s, 3), [0, 2, 5])   # 0.9, 0.7, then 0.5 of the lower index
    # ties go to the lower expert index
    np.testing.assert_array_equal(moe.reap_keep(np.array([1.0, 2.0, 1.0, 1.0]), 2), [0, 1])
    np.testing.assert_array_equal(moe.reap_keep(s, 6), np.arange(6))


# --- the shared BF16 expert (reading R19) ---

def _shared(cfg, seed=3):
    gen = torch.Generator().manual_seed(seed)
    mk = lambda *s: (torch.randn(*s, generator=gen) * 0.02).to(torch.bfloat16).float().numpy()  # noqa: E731
    return mk(cfg.I, cfg.H), mk(cfg.I, cfg.H), mk(cfg.H, cfg.I)


def test_shared_expert_alone_is_torchs_mlp():
    """With every routed expert zeroed, the layer is bf16 of the shared MLP;
    torch's fp64 matmuls and SiLU give the same numbers."""
    cfg, x, wg, bias, bf, q = _tiny_layer()
    sh = _shared(cfg)
    zero = {e: tuple((np.zeros_like(c), np.zeros_like(s), g) for c, s, g in q[e]) for e in range(cfg.E)}
    res = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: zero[e], F32(0.003), F32(0.0005), shared=sh)
    xt = torch.from_numpy(x).double()
    g, u, d = (torch.from_numpy(t).double() for t in sh)
    h = torch.nn.functional.silu(xt @ g.T) * (xt @ u.T)
    ref = (h.to(torch.bfloat16).double() @ d.T).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(res["out"], ref)


def test_shared_expert_adds_to_the_routed_layer():
    cfg, x, wg, bias, bf, q = _tiny_layer()
    sh = _shared(cfg)
    routed = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], F32(0.003), F32(0.0005))
    both = moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], F32(0.003), F32(0.0005), shared=sh)
    np.testing.assert_allclose(both["out_f64"] - moe.shared_expert(x, sh), routed["out_f64"], rtol=0,
                               atol=1e-12 * np.abs(both["out_f64"]).max())
    zeros = tuple(np.zeros_like(t) for t in sh)
    np.testing.assert_array_equal(
        moe.moe_layer(x, wg, bias, cfg.k, cfg.rsf, lambda e: q[e], F32(0.003), F32(0.0005), shared=zeros)["out"],
        routed["out"])
