"""The oracle's readings against the libraries the pages name, on CPU.

The NVFP4 model card ("K-EXAONE-152B-A23B-REAP-80E-NVFP4", "Quantization
Setup") quantises its weights with llmcompressor's NVFP4 scheme, stored in the
compressed-tensors format, and serves the checkpoint with vLLM.  Both
libraries are in this image with plain-PyTorch references:
- compressed-tensors' weight quantisation: global scale 2688/amax, block
  scale amax/6 times it, elements divided by block/global;
- vLLM's activation reference: block scale global * (amax * 1/6), elements
  multiplied by the reciprocal of block/global.
vLLM also provides its block-scale swizzle and dequantiser, its grouped top-k
router and its plain-torch MoE loop.

Exact agreement, pinned here:
- the E2M1 rounding: the libraries' own casts, value by value (ties to the
  even code, saturation at 6, a negative that rounds to zero stays -0);
- the E4M3 scale rounding;
- the global scale, which the libraries store inverted;
- the packed codes and nibble order;
- the tiled scale layout, which is vLLM's swizzled layout;
- a zero scale for an all-zero block in vLLM;
- the router's choices and weights (to a few ulps);
- the layer's composition.

What differs is the order of the fp32 roundings (reading R2).  It shows only
where the exact value sits on a rounding midpoint, and the two results are
then neighbouring codes.  There are also two small convention differences:
- compressed-tensors gives an all-zero block the E4M3 scale eps (0.125), where
  this library gives 0 (reading R7);
- an input of exactly -0.0 becomes +0 in the libraries and -0 here
  (reading R5).
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4

E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
E4M3_VALUES = np.array([nvfp4.e4m3_decode(np.array([c], np.uint8))[0] for c in range(0x7F)], np.float64)
E4M3_MIDPOINTS = (E4M3_VALUES[1:] + E4M3_VALUES[:-1]) / 2


def _near(v, points, rel=1e-5):
    v = np.abs(np.asarray(v, np.float64))[..., None]
    return np.any(np.abs(v - points) <= rel * np.maximum(points, 1e-30), axis=-1)


def _values(codes):
    c = np.stack([codes & 0xF, codes >> 4], -1).reshape(codes.shape[0], -1)
    return nvfp4.e2m1_decode(c).astype(np.float64), c & 0x7


def _magnitude_code(v):
    return np.searchsorted(np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6]), np.abs(v))


def _check_against(x, g, ours_codes, ours_scales, lib_values, lib_scale_codes, zero_scale_code):
    """Exact agreement up to neighbouring codes at rounding midpoints."""
    rows, nblk = ours_scales.shape
    xb = x.astype(np.float64).reshape(rows, nblk, 16)
    amax_b = np.abs(xb).max(-1)
    zero = amax_b == 0
    # all-zero blocks: the libraries' convention, then nothing else to compare
    assert np.all(lib_scale_codes[zero] == zero_scale_code) and np.all(ours_scales[zero] == 0)
    # block scales: equal, or neighbours where the exact value amax_b / (6 g) is a midpoint
    diff = (lib_scale_codes != ours_scales) & ~zero
    assert diff.sum() <= 0.005 * (~zero).sum()
    assert np.all(np.abs(lib_scale_codes[diff].astype(int) - ours_scales[diff].astype(int)) == 1)
    assert np.all(_near(amax_b[diff] / (6.0 * float(g)), E4M3_MIDPOINTS))
    # elements, in blocks whose scales agree
    ours_v, _ = _values(ours_codes)
    same = np.repeat(~diff, 16, axis=1)
    ev = (ours_v != lib_values) & same
    # bf16 inputs put many elements exactly on a midpoint; where the two
    # sequences' effective scales differ by an ulp those land on either side
    assert ev.sum() <= 0.01 * same.sum()
    assert np.all(np.abs(_magnitude_code(ours_v[ev]) - _magnitude_code(lib_values[ev])) == 1)
    s_val = nvfp4.e4m3_decode(ours_scales).astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):        # all-zero blocks have no y
        y = x.astype(np.float64) / (np.repeat(s_val, 16, axis=1) * float(g))
    assert np.all(_near(y[ev], E2M1_MIDPOINTS, rel=1e-4))
    return int(diff.sum()), int(ev.sum())


def _e2m1_probe_values():
    """Every E2M1 midpoint and grid point, their fp32 neighbours, saturation,
    signed zeros and random magnitudes, positive and negative."""
    base = np.concatenate([E2M1_MIDPOINTS, [0.0, 0.5, 1, 1.5, 2, 3, 4, 6, 6.5, 7, 100.0, 1e-30]]).astype(np.float32)
    near = np.concatenate([np.nextafter(base, np.float32(np.inf)), np.nextafter(base, np.float32(0))])
    rnd = np.random.default_rng(0).uniform(0, 7, 4096).astype(np.float32)
    v = np.concatenate([base, near, rnd])
    return np.concatenate([v, -v]).astype(np.float32)


@pytest.mark.parametrize("lib", ["compressed_tensors", "vllm"])
def test_e2m1_rounding_matches_the_libraries(lib, monkeypatch):
    """Round to nearest, ties to the even code, saturation at 6, the sign of
    zero kept: the libraries' E2M1 casts give the oracle's values exactly."""
    if lib == "compressed_tensors":
        qa = pytest.importorskip("compressed_tensors.quantization.quant_args")
        monkeypatch.setattr(torch._dynamo.config, "disable", True)     # eager: the same arithmetic
        cast = qa.FP4_E2M1_DATA.cast_to_fp4
    else:
        cast = pytest.importorskip("vllm.model_executor.layers.quantization.utils.nvfp4_emulation_utils").cast_to_fp4
    y = _e2m1_probe_values()
    got = cast(torch.from_numpy(y.copy()).clamp(-6.0, 6.0)).numpy()
    ours = nvfp4.e2m1_decode(nvfp4.e2m1_encode(y))
    np.testing.assert_array_equal(got, ours)
    # the sign of zero agrees (tiny negatives give -0 on both sides) except for
    # an input of exactly -0.0: the libraries take its sign as 0 and return +0,
    # this library keeps -0 (code 8, reading R5)
    neg_zero = (y == 0) & np.signbit(y)
    assert np.array_equal(np.signbit(got)[~neg_zero], np.signbit(ours)[~neg_zero])
    assert neg_zero.any() and not np.signbit(got[neg_zero]).any() and np.signbit(ours[neg_zero]).all()


def _weights(seed, rows=128, cols=1024):
    gen = torch.Generator().manual_seed(seed)
    w = torch.randn(rows, cols, generator=gen) * 0.02
    w[torch.rand(rows, cols, generator=gen) < 0.01] *= 20          # outliers
    w[seed % 4] = 0.0                                              # an all-zero row
    return w.to(torch.bfloat16)


@pytest.mark.parametrize("seed", range(4))
def test_weight_quantiser_matches_compressed_tensors(seed, monkeypatch):
    ct = pytest.importorskip("compressed_tensors.quantization")
    from compressed_tensors.quantization.lifecycle.forward_helpers import _quantize
    from compressed_tensors.quantization.utils.helpers import calculate_qparams, calculate_range, generate_gparam
    monkeypatch.setattr(torch._dynamo.config, "disable", True)   # its E2M1 cast is torch.compile'd; eager is the same
    w = _weights(seed)
    args = ct.QuantizationArgs(num_bits=4, type="float", strategy="tensor_group", group_size=16, symmetric=True,
                               dynamic=False, scale_dtype=torch.float8_e4m3fn)
    x = w.float()
    gs = generate_gparam(x.min(), x.max())
    xb = x.unflatten(-1, (x.shape[-1] // 16, 16))
    scale, _ = calculate_qparams(xb.amin(-1), xb.amax(-1), args, global_scale=gs)
    q_min, q_max = calculate_range(args, "cpu")
    lib_v = _quantize(xb, scale.unsqueeze(-1), None, q_min, q_max, args, global_scale=gs).flatten(-2)
    lib_s = scale.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    codes, scales, g = nvfp4.quantize_weight(x.numpy())
    # the global scale: reciprocals of each other, to fp32 rounding
    assert abs(float(gs) * float(g) - 1.0) <= 2.0 ** -22
    eps_code = int(torch.tensor([torch.finfo(torch.float8_e4m3fn).eps]).to(torch.float8_e4m3fn).view(torch.uint8))
    _check_against(x.numpy(), g, codes, scales, lib_v.numpy().astype(np.float64), lib_s, eps_code)


@pytest.mark.parametrize("seed", range(4))
def test_activation_quantiser_matches_vllm_reference(seed):
    ref = pytest.importorskip("vllm.model_executor.layers.quantization.utils.nvfp4_emulation_utils")
    gen = torch.Generator().manual_seed(100 + seed)
    x = torch.randn(64, 2048, generator=gen)
    x[torch.rand(64, 2048, generator=gen) < 0.001] *= 20
    x[seed % 3, :48] = 0.0                                          # three all-zero blocks
    x = x.to(torch.bfloat16).float()
    amax = np.float32(x.abs().max())
    g = np.float32(amax / np.float32(2688))                         # calibrated g1 of this library
    gs = torch.tensor([2688.0]) / torch.tensor([float(amax)])       # the same calibration, stored inverted
    lib_v, lib_scale = ref.ref_nvfp4_quant(x, gs, 16)
    lib_s = lib_scale.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    codes, scales = nvfp4.quantize(x.numpy(), g)
    _check_against(x.numpy(), g, codes, scales, lib_v.numpy().astype(np.float64), lib_s, 0)


@pytest.mark.parametrize("rows,nblk", [(256, 24), (200, 8), (128, 4), (300, 16)])
def test_tiled_scale_layout_is_the_swizzled_layout_of_vllm(rows, nblk, monkeypatch):
    """NVFP4_LAYOUT_TILED (the scale layout the tensor-core MMA reads) is
    byte for byte the block-scale layout vLLM prepares for the CUTLASS and
    FlashInfer FP4 kernels (swizzle_blockscale), zero padding rows included.
    The GPU tests check that the library writes the layout of tiled_index."""
    mod = pytest.importorskip("vllm.model_executor.layers.quantization.utils.nvfp4_utils")
    from _util import tiled_index
    monkeypatch.setattr(torch.Tensor, "cuda", lambda self, *a, **k: self)   # its last step moves to the GPU
    sc = np.random.default_rng(rows + nblk).integers(0, 0x7F, size=(rows, nblk), dtype=np.uint8)
    swizzled = mod.swizzle_blockscale(torch.from_numpy(sc).view(torch.float8_e4m3fn))
    swizzled = swizzled.view(torch.uint8).numpy().reshape(-1)
    rows_padded = (rows + 127) // 128 * 128
    ours = np.zeros(rows_padded * nblk, np.uint8)
    ours[tiled_index(rows_padded, nblk * 16)[:rows].reshape(-1)] = sc.reshape(-1)
    np.testing.assert_array_equal(swizzled, ours)


def test_code_packing_is_the_compressed_tensors_packing():
    """Codes and nibble order (readings R5, R6): compressed-tensors' packer,
    given the oracle's quantised values, writes the oracle's bytes: magnitude
    index 0..7, the sign in bit 3, the even-indexed element in the low
    nibble."""
    helpers = pytest.importorskip("compressed_tensors.compressors.nvfp4.helpers")
    codes, _, _ = nvfp4.quantize_weight(_weights(7, rows=64, cols=512).float().numpy())
    values, _ = _values(codes)
    packed = helpers.pack_fp4_to_uint8(torch.from_numpy(values.astype(np.float32)))
    np.testing.assert_array_equal(packed.numpy(), codes)


def test_routing_matches_vllms_grouped_topk_with_one_group():
    """Reading R9 against vLLM's router for this model family (exaone_moe:
    grouped top-k, sigmoid scores, e_score_correction_bias, renormalised,
    routed_scaling_factor), in its CPU form with one expert group, i.e.
    without group-limited routing: the bias only selects, the weights are the
    unbiased sigmoids renormalised over the k chosen, then scaled.  The
    sigmoid and the sum order differ (torch.sigmoid, torch.sum), so the chosen
    sets are compared where the k-th and (k+1)-th biased scores are apart, and
    the weights to a few ulps."""
    cpu_moe = pytest.importorskip("vllm.model_executor.layers.fused_moe.cpu_fused_moe")
    from oracle import moe
    T, E, k, rsf = 512, 80, 8, 2.5
    rng = np.random.default_rng(5)
    logits = rng.normal(0, 1.5, (T, E)).astype(np.float32)
    bias = rng.normal(0, 0.01, E).astype(np.float32)
    w_lib, idx_lib = cpu_moe.grouped_topk(torch.zeros(T, 1), torch.from_numpy(logits), k, True, num_expert_group=1,
                                          topk_group=1, scoring_func="sigmoid", routed_scaling_factor=rsf,
                                          e_score_correction_bias=torch.from_numpy(bias))
    idx, w = moe.route(logits, bias, k, rsf)
    c = np.sort(moe.sigmoid_f32(logits).astype(np.float64) + bias, axis=1)[:, ::-1]
    apart = (c[:, k - 1] - c[:, k]) > 1e-5
    assert apart.mean() > 0.95
    lib_i, lib_w = idx_lib.numpy(), w_lib.numpy()
    for t in np.nonzero(apart)[0]:
        o_l, o_m = np.argsort(lib_i[t]), np.argsort(idx[t])
        np.testing.assert_array_equal(lib_i[t][o_l], idx[t][o_m])
        np.testing.assert_allclose(lib_w[t][o_l], w[t][o_m], rtol=2e-6)
    # our slots come in descending order of the biased score
    sel = np.take_along_axis(moe.sigmoid_f32(logits).astype(np.float64) + bias, idx.astype(np.int64), axis=1)
    assert np.all(np.diff(sel, axis=1) <= 0)


def test_layer_composition_matches_vllms_cpu_moe(monkeypatch):
    """The layer's composition (readings R10, R12) against vLLM's plain-torch
    MoE loop (cpu_fused_moe_torch), both in fp64 and without quantisation:
    gate rows before up rows in the fused gate/up projection, SiLU of the gate
    half times the up half, the down projection, then each expert output
    times its routing weight, summed over the k slots.  The routing itself is
    the oracle's, pinned separately."""
    cm = pytest.importorskip("vllm.model_executor.layers.fused_moe.cpu_fused_moe")
    from vllm.model_executor.layers.activation import SiluAndMul
    from vllm.model_executor.layers.fused_moe.activation import MoEActivation
    from oracle import moe
    # the library's own SiLU-and-mul, called without building a vLLM config
    monkeypatch.setitem(cm._CPU_MOE_ACT_FN, MoEActivation.SILU, SiluAndMul.forward_native)
    rng = np.random.default_rng(3)
    T, H, I, E, k, rsf = 24, 64, 32, 6, 2, 2.5
    x = rng.normal(0, 1, (T, H)).astype(np.float32)
    wg = rng.normal(0, 0.3, (E, H)).astype(np.float32)
    bias = rng.normal(0, 0.01, E).astype(np.float32)
    gate, up, down = rng.normal(0, 0.1, (E, I, H)), rng.normal(0, 0.1, (E, I, H)), rng.normal(0, 0.1, (E, H, I))
    dense = moe.dense_moe_layer(x, wg, bias, k, rsf, lambda e: (gate[e], up[e], down[e]))
    idx, w = moe.route(moe.router_logits(x, wg), bias, k, rsf)

    class Experts:                       # what the vLLM loop reads from its layer
        gate_up_linear = [(lambda t, m=torch.from_numpy(np.concatenate([gate[e], up[e]])): t @ m.T) for e in range(E)]
        down_linear = [(lambda t, m=torch.from_numpy(down[e]): t @ m.T) for e in range(E)]

    layer = Experts()
    key = id(layer)
    monkeypatch.setitem(cm._CPU_MOE_LAYER_CACHE, key, lambda: layer)
    out = torch.zeros(T, H, dtype=torch.float64)
    cm.cpu_fused_moe_torch(key, out, torch.from_numpy(x.astype(np.float64)), torch.from_numpy(w.astype(np.float64)),
                           torch.from_numpy(idx.astype(np.int64)), "silu", global_num_experts=E)
    np.testing.assert_allclose(out.numpy(), dense, rtol=1e-12, atol=1e-12 * np.abs(dense).max())
    # a swapped gate/up order would not agree
    swapped = moe.dense_moe_layer(x, wg, bias, k, rsf, lambda e: (up[e], gate[e], down[e]))
    assert np.abs(out.numpy() - swapped).max() > 1e-3 * np.abs(dense).max()


def test_dequantisation_matches_vllms_dequantiser_on_tiled_scales():
    """vLLM's dequantiser, given the oracle's packed codes, its scales in this
    library's tiled layout and the oracle's g, returns the oracle's
    dequantised values: low nibble first, sign in bit 3, the tiled layout
    undone by vLLM's own un-swizzle, x = E2M1 * E4M3 * g.  The two orders of
    the products (here (v*s)*g, exact in its first step; there v*(s*g)) can
    differ by one ulp, only when v is not a power of two (1.5, 3 or 6)."""
    ref = pytest.importorskip("vllm.model_executor.layers.quantization.utils.nvfp4_emulation_utils")
    from _util import tiled_index
    w = _weights(11, rows=200, cols=512).float().numpy()          # ragged: 200 rows, 2 row tiles
    codes, scales, g = nvfp4.quantize_weight(w)
    rows_padded = 256
    tiled = np.zeros(rows_padded * scales.shape[1], np.uint8)
    tiled[tiled_index(rows_padded, 512)[:200].reshape(-1)] = scales.reshape(-1)
    got = ref.dequantize_to_dtype(torch.from_numpy(codes), torch.from_numpy(tiled), torch.tensor(float(g)),
                                  torch.float32, 16, swizzle=True).numpy()
    ours = nvfp4.dequantize(codes, scales, g)
    assert got.shape == ours.shape
    vals, _ = _values(codes)
    exact = ~np.isin(np.abs(vals), (1.5, 3.0, 6.0))
    np.testing.assert_array_equal(got[exact], ours[exact])
    ulp = np.spacing(np.abs(ours[~exact]).astype(np.float32))
    assert np.all(np.abs(got[~exact] - ours[~exact]) <= ulp)


def test_quantised_layer_matches_vllms_cpu_moe_loop(monkeypatch):
    """moe_layer itself (not the unquantised dense loop) against vLLM's
    plain-torch MoE loop (cpu_fused_moe_torch).  The loop is handed the
    oracle's own quantised expert operations: its gate/up projection
    quantises the rows of x under g1 and runs expert_gate_up; its down
    projection rounds h to fp32 (R11), quantises it under g2 and runs
    expert_down.  The loop then does what the NVFP4 card's per-expert Linears
    and the BF16 card's routing imply: it gathers each expert's tokens, takes
    SiLU of the gate half times the up half, weights each expert's output by
    that slot's routing weight and sums the k slots (R10, R12).  moe_layer's
    fp64 output must equal the loop's to 1e-12.  So a slot paired with the
    wrong weight, a dropped slot or an expert fed another expert's rows fails
    here; the unquantised band of test_oracle_moe could not tell them apart."""
    cm = pytest.importorskip("vllm.model_executor.layers.fused_moe.cpu_fused_moe")
    from vllm.model_executor.layers.activation import SiluAndMul
    from vllm.model_executor.layers.fused_moe.activation import MoEActivation
    from oracle import moe
    monkeypatch.setitem(cm._CPU_MOE_ACT_FN, MoEActivation.SILU, SiluAndMul.forward_native)
    rng = np.random.default_rng(7)
    T, H, I, E, k, rsf = 40, 128, 64, 6, 3, 2.5
    x = torch.from_numpy(rng.normal(0, 1, (T, H)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    wg = rng.normal(0, 0.3, (E, H)).astype(np.float32)
    bias = rng.normal(0, 0.01, E).astype(np.float32)
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).float().numpy()  # noqa: E731
    q = {e: tuple(nvfp4.quantize_weight(bf(rng.normal(0, 0.05, s))) for s in ((I, H), (I, H), (H, I)))
         for e in range(E)}
    g1 = np.float32(np.float32(np.abs(x).max()) / np.float32(2688))
    g2 = np.float32(3e-4)
    ref = moe.moe_layer(x, wg, bias, k, rsf, lambda e: q[e], g1, g2)
    idx, w = ref["topk_idx"], ref["topk_w"]

    def gate_up(e):
        def f(t):
            ac, asc = nvfp4.quantize(t.numpy().astype(np.float32), g1)
            gate_v, up_v, _ = moe.expert_gate_up(ac, asc, g1, q[e][0], q[e][1])
            return torch.from_numpy(np.concatenate([gate_v, up_v], axis=1))
        return f

    def down(e):
        def f(h):
            hc, hs = nvfp4.quantize(h.numpy().astype(np.float32), g2)
            return torch.from_numpy(moe.expert_down(hc, hs, g2, q[e][2]))
        return f

    class Experts:
        gate_up_linear = [gate_up(e) for e in range(E)]
        down_linear = [down(e) for e in range(E)]

    layer = Experts()
    monkeypatch.setitem(cm._CPU_MOE_LAYER_CACHE, id(layer), lambda: layer)
    out = torch.zeros(T, H, dtype=torch.float64)
    cm.cpu_fused_moe_torch(id(layer), out, torch.from_numpy(x.astype(np.float64)),
                           torch.from_numpy(w.astype(np.float64)), torch.from_numpy(idx.astype(np.int64)), "silu",
                           global_num_experts=E)
    got, want = out.numpy(), ref["out_f64"]
    np.testing.assert_allclose(want, got, rtol=1e-12, atol=1e-12 * np.abs(got).max())
    # the same loop with every slot given slot 0's weight is far off
    w0 = np.repeat(w[:, :1], k, axis=1)
    out0 = torch.zeros(T, H, dtype=torch.float64)
    cm.cpu_fused_moe_torch(id(layer), out0, torch.from_numpy(x.astype(np.float64)),
                           torch.from_numpy(w0.astype(np.float64)), torch.from_numpy(idx.astype(np.int64)), "silu",
                           global_num_experts=E)
    assert np.abs(out0.numpy() - want).max() > 1e-3 * np.abs(want).max()
