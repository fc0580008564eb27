"""The layer under the per-expert and batch-derived activation global scales
(moe_nvfp4_forward_scaled) against the oracle (reading R16 of the design
notes: one g1/g2 per expert; g1 = amax/2688 over the batch or over each
expert's tokens, computed on the device).

Compared where both sides route a token identically (the logits differ in
fp32 summation order only): the device-derived g1 values bit for bit, the
quantised x rows bit for bit, h within 1e-3, requantised codes within 0.1%,
the output within 1e-2 relative L2."""
import numpy as np
import pytest
import torch

from _util import capi, host, rel_l2, require_cuda, tiled_rows
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import moe, nvfp4

pytestmark = pytest.mark.gpu
F32 = np.float32

CASES = {
    "tiny": workloads.CONFIGS["tiny"],
    "mid_skewed": workloads.LayerConfig("mid", T=300, H=1024, I=512, E=16, k=4, x_outlier_p=0.001,
                                        logit_offset_std=0.5),
}


def _setup(cfg):
    c = capi()
    x = workloads.hidden_states(cfg, device="cpu")
    wg, bias, off = workloads.router_params(cfg, device="cpu")
    gate, up, down = workloads.stacked_expert_weights(cfg, device="cpu")
    W = c.MoeWeights.quantize(gate.cuda(), up.cuda(), down.cuda(), wg.cuda(), bias.cuda(), cfg.k, cfg.rsf)
    q = {e: tuple(nvfp4.quantize_weight(t[e].float().numpy()) for t in (gate, up, down)) for e in range(cfg.E)}
    return c, x, wg, bias, off, W, q


@pytest.mark.parametrize("mode", ["expert", "dynamic", "dynamic_expert"])
@pytest.mark.parametrize("name", list(CASES))
def test_scaled_forward_matches_oracle(name, mode):
    require_cuda()
    cfg = CASES[name]
    c, x, wg, bias, off, W, q = _setup(cfg)
    xf, wf, bf = x.float().numpy(), wg.float().numpy(), bias.numpy()
    offn = None if off is None else off.numpy()
    per_expert = mode in ("expert", "dynamic_expert")
    rng = np.random.default_rng(11)
    # g1 given per expert: the batch scale times a factor in [0.5, 1.5)
    g_all = moe.activation_scales(xf, "dynamic", cfg.E)
    g1_in = (g_all * (0.5 + rng.random(cfg.E))).astype(F32) if mode == "expert" else mode
    # g2 calibrated on the oracle's own h, per expert or for the tensor
    cal = moe.moe_layer(xf, wf, bf, cfg.k, cfg.rsf, lambda e: q[e], g1_in,
                        np.ones(cfg.E, F32) if per_expert else F32(1.0), logit_offset=offn)
    hmax = np.zeros(cfg.E)
    for (t, j), h in cal["h"].items():
        e = cal["topk_idx"][t, j]
        hmax[e] = max(hmax[e], np.abs(h).max())
    g2 = (hmax.astype(F32) / F32(2688)).astype(F32) if per_expert else F32(F32(hmax.max()) / F32(2688))
    ref = moe.moe_layer(xf, wf, bf, cfg.k, cfg.rsf, lambda e: q[e], g1_in, g2, logit_offset=offn)

    n = cfg.E if per_expert else 1
    act = torch.tensor(np.asarray(g1_in, F32).reshape(-1) if mode == "expert" else np.zeros(n, F32)).cuda()
    hgs = torch.tensor(np.asarray(g2, F32).reshape(-1)).cuda()
    out, dbg = c.moe_nvfp4_forward(W, x.cuda(), act, hgs, logit_offset=None if off is None else off.cuda(),
                                   debug=True, act_scale_mode=mode)
    c.nvfp4_workspace_status(dbg["workspace"])

    gidx = host(dbg["topk_idx"])
    same = np.all(gidx == ref["topk_idx"], axis=1)
    assert same.mean() >= 0.97
    g1_ref = np.asarray(ref["g1"], F32).reshape(-1)
    g1_gpu = host(act).reshape(-1)
    if mode == "dynamic":
        assert g1_gpu[0] == g1_ref[0]
    elif mode == "dynamic_expert":
        # experts whose routed token set is the same on both sides
        for e in range(cfg.E):
            if np.array_equal(np.any(gidx == e, axis=1), np.any(ref["topk_idx"] == e, axis=1)):
                assert g1_gpu[e] == g1_ref[e], e

    inv_g = host(dbg["inv_perm"])
    ac, asc = host(dbg["a_codes"]), host(dbg["a_scales"])
    h_g, hc_g = host(dbg["h"]), host(dbg["h_codes"])
    hs, hr, flips, total = [], [], 0, 0
    for t in np.nonzero(same)[0]:
        for j in range(cfg.k):
            e = int(gidx[t, j])
            r = inv_g[t, j]
            g1e = g1_ref[e] if per_expert else g1_ref[0]
            xc, xs = nvfp4.quantize(xf[t:t + 1], g1e)
            np.testing.assert_array_equal(ac[r], xc[0])
            np.testing.assert_array_equal(tiled_rows(asc, [r], cfg.H)[0], xs[0])
            hs.append(h_g[r])
            hr.append(ref["h"][(t, j)])
            rc, _ = nvfp4.quantize(ref["h"][(t, j)][None, :], np.asarray(g2).reshape(-1)[e if per_expert else 0])
            flips += int(np.count_nonzero(nvfp4.unpack_codes(hc_g[r:r + 1]) != nvfp4.unpack_codes(rc)))
            total += cfg.I
    assert rel_l2(np.array(hs), np.array(hr)) <= 1e-3
    assert flips <= 0.001 * total, f"{flips}/{total} requantised codes differ"
    err = rel_l2(host(out)[same], ref["out"][same])
    assert err <= 1e-2, err


def test_tensor_mode_through_the_scaled_entry_point_is_the_plain_forward():
    require_cuda()
    cfg = CASES["tiny"]
    c, x, wg, bias, off, W, q = _setup(cfg)
    g1, g2 = torch.tensor([0.004]).cuda(), torch.tensor([0.0007]).cuda()
    a = c.moe_nvfp4_forward(W, x.cuda(), g1, g2)
    st = W.struct()
    ws = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8, device="cuda")
    b = torch.empty_like(a)
    import ctypes
    c._check(c.lib.moe_nvfp4_forward_scaled(ctypes.byref(st), c._p(x.cuda()), cfg.T, 0, c._p(g1), c._p(g2), None,
                                            c._p(b), None, c._p(ws), ws.numel(), c._stream()))
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    with pytest.raises(c.Nvfp4Error):
        c._check(c.lib.moe_nvfp4_forward_scaled(ctypes.byref(st), c._p(x.cuda()), cfg.T, 7, c._p(g1), c._p(g2),
                                                None, c._p(b), None, c._p(ws), ws.numel(), c._stream()))
