"""The whole layer (moe_nvfp4_forward) against the oracle.

Routing is computed on both sides from the same bf16 inputs; the logits
differ in fp32 summation order only, so a token whose k-th and (k+1)-th
biased scores are closer than that error may legitimately route differently.
Those tokens are excluded from the value comparisons (and must be rare)."""
import numpy as np
import pytest
import torch

from _util import capi, host, rel_l2, require_cuda, staged_to_canonical, tiled_rows
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import moe, nvfp4

pytestmark = pytest.mark.gpu
F32 = np.float32

CASES = {
    "tiny": workloads.CONFIGS["tiny"],
    "mid_skewed": workloads.LayerConfig("mid", T=300, H=1024, I=512, E=16, k=4, x_outlier_p=0.001,
                                        logit_offset_std=0.5),
    "ragged_small": workloads.LayerConfig("rs", T=3, H=512, I=256, E=6, k=3),
    # k > 8 takes the combine kernel's wide variant
    "wide_k": workloads.LayerConfig("wk", T=40, H=512, I=256, E=12, k=10),
    # a single token
    "one_token": workloads.LayerConfig("ot", T=1, H=512, I=256, E=8, k=2),
    # the largest expert count and top-k the ABI accepts: 9,600 rows run the
    # CTA-pair GEMMs, most experts hold one (odd) m-tile, so most pairs have a
    # second CTA without rows, and k = 16 takes the wide combine
    "max_experts": workloads.LayerConfig("mx", T=600, H=512, I=256, E=256, k=16, logit_offset_std=0.5),
}


def _setup(cfg):
    c = capi()
    x = workloads.hidden_states(cfg, device="cpu")
    wg, bias, off = workloads.router_params(cfg, device="cpu")
    gate, up, down = workloads.stacked_expert_weights(cfg, device="cpu")
    W = c.MoeWeights.quantize(gate.cuda(), up.cuda(), down.cuda(), wg.cuda(), bias.cuda(), cfg.k, cfg.rsf)
    q = {e: tuple(nvfp4.quantize_weight(t[e].float().numpy()) for t in (gate, up, down)) for e in range(cfg.E)}
    return c, x, wg, bias, off, W, q


@pytest.mark.parametrize("name", list(CASES))
def test_forward_matches_oracle(name):
    require_cuda()
    cfg = CASES[name]
    c, x, wg, bias, off, W, q = _setup(cfg)
    xf, wf, bf = x.float().numpy(), wg.float().numpy(), bias.numpy()
    offn = None if off is None else off.numpy()
    g1 = F32(F32(np.abs(xf).max()) / F32(2688))
    # calibrate g2 on the oracle's own h (max over every routed pair)
    cal = moe.moe_layer(xf, wf, bf, cfg.k, cfg.rsf, lambda e: q[e], g1, F32(1.0), logit_offset=offn)
    g2 = F32(F32(max(np.abs(h).max() for h in cal["h"].values())) / F32(2688))
    ref = moe.moe_layer(xf, wf, bf, cfg.k, cfg.rsf, lambda e: q[e], g1, g2, logit_offset=offn)

    out, dbg = c.moe_nvfp4_forward(W, x.cuda(), torch.tensor([g1]).cuda(), torch.tensor([g2]).cuda(),
                                   logit_offset=None if off is None else off.cuda(), debug=True)
    c.nvfp4_workspace_status(dbg["workspace"])

    # routing: same sets wherever the oracle's selection margin is safe
    gidx, gw = host(dbg["topk_idx"]), host(dbg["topk_w"])
    L = ref["logits"].astype(np.float64)
    sig = moe.sigmoid_f32(ref["logits"]).astype(np.float64)
    cb = np.sort(sig + bf[None, :], axis=1)[:, ::-1]
    mag = np.abs(xf.astype(np.float64)) @ np.abs(wf.astype(np.float64)).T
    safe = (cb[:, cfg.k - 1] - cb[:, cfg.k]) > 0.5 * (1e-5 * mag.max(axis=1) + 1e-6) + 1e-6
    # sets must agree where the margin is safe; the order inside a set can
    # differ only between nearly tied scores, so values are compared on
    # tokens whose ordered selection agrees
    same_set = np.all(np.sort(gidx, axis=1) == np.sort(ref["topk_idx"], axis=1), axis=1)
    assert np.all(same_set[safe])
    same = np.all(gidx == ref["topk_idx"], axis=1)
    assert same.mean() >= 0.97
    assert np.all(np.abs(host(dbg["logits"]) - L) <= 1e-5 * mag + 1e-6)
    np.testing.assert_allclose(gw[same], ref["topk_w"][same], rtol=2e-5)

    # permutation consistent with the GPU's own selection
    off_g, perm_g, inv_g = host(dbg["expert_offsets"]), host(dbg["perm"]), host(dbg["inv_perm"])
    ro, rp, ri = moe.permute(ref["topk_idx"], cfg.E)
    if np.all(same):
        np.testing.assert_array_equal(off_g, ro)
        np.testing.assert_array_equal(perm_g[: rp.size], rp)
        np.testing.assert_array_equal(inv_g, ri)

    # quantised x in permuted rows: bit-exact
    ac = host(dbg["a_codes"])
    asc = host(dbg["a_scales"])
    for t in range(cfg.T):
        for j in range(cfg.k):
            r = inv_g[t, j]
            np.testing.assert_array_equal(ac[r], ref["a_codes"][t])
            np.testing.assert_array_equal(tiled_rows(asc, [r], cfg.H)[0], ref["a_scales"][t])

    # h before requantisation, requantised codes, weighted y, and the output
    h_g, hc_g, y_g = host(dbg["h"]), host(dbg["h_codes"]), host(dbg["y"])
    hs, hr, flips, total = [], [], 0, 0
    for t in np.nonzero(same)[0]:
        for j in range(cfg.k):
            r = inv_g[t, j]
            hs.append(h_g[r])
            hr.append(ref["h"][(t, j)])
            rc, _ = nvfp4.quantize(ref["h"][(t, j)][None, :], g2)
            flips += int(np.count_nonzero(nvfp4.unpack_codes(hc_g[r:r + 1]) != nvfp4.unpack_codes(rc)))
            total += cfg.I
    assert rel_l2(np.array(hs), np.array(hr)) <= 1e-3
    assert flips <= 0.001 * total, f"{flips}/{total} requantised codes differ"
    err = rel_l2(host(out)[same], ref["out"][same])
    assert err <= 1e-2, err


def test_staged_and_row_major_codes_give_identical_layers():
    """The staged code layout only moves bytes: the quantiser's staged codes
    read back as its row-major codes, and the layer's output is bit-identical
    with either (gate/up and down both fetch staged tiles)."""
    require_cuda()
    cfg = CASES["mid_skewed"]
    c = capi()
    x = workloads.hidden_states(cfg, device="cpu").cuda()
    wg, bias, off = workloads.router_params(cfg, device="cpu")
    gate, up, down = (t.cuda() for t in workloads.stacked_expert_weights(cfg, device="cpu"))
    Ws = c.MoeWeights.quantize(gate, up, down, wg.cuda(), bias.cuda(), cfg.k, cfg.rsf, codes_layout="staged")
    Wc = c.MoeWeights.quantize(gate, up, down, wg.cuda(), bias.cuda(), cfg.k, cfg.rsf, codes_layout="canonical")
    assert Ws.codes_layout == c.LAYOUT_STAGED and Wc.codes_layout == c.LAYOUT_CANONICAL
    for s, r, (rows, cols) in ((Ws.gate_codes, Wc.gate_codes, (cfg.I, cfg.H)), (Ws.up_codes, Wc.up_codes, (cfg.I, cfg.H)),
                               (Ws.down_codes, Wc.down_codes, (cfg.H, cfg.I))):
        hs, hr = host(s), host(r)
        for e in (0, cfg.E - 1):
            np.testing.assert_array_equal(staged_to_canonical(hs[e], rows, cols), hr[e])
    g1 = torch.tensor([float(x.float().abs().max()) / 2688.0]).cuda()
    g2 = torch.tensor([0.002]).cuda()
    off_d = off.cuda() if off is not None else None
    os_ = c.moe_nvfp4_forward(Ws, x, g1, g2, logit_offset=off_d)
    oc = c.moe_nvfp4_forward(Wc, x, g1, g2, logit_offset=off_d)
    assert torch.equal(os_, oc)


def test_forward_status_word_is_clear_and_repeatable():
    require_cuda()
    cfg = CASES["tiny"]
    c, x, wg, bias, off, W, q = _setup(cfg)
    g = torch.tensor([0.01]).cuda()
    ws = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8, device="cuda")
    o1 = c.moe_nvfp4_forward(W, x.cuda(), g, g, workspace=ws).clone()
    o2 = c.moe_nvfp4_forward(W, x.cuda(), g, g, workspace=ws)
    c.nvfp4_workspace_status(ws)
    assert torch.equal(o1, o2)        # deterministic: no atomics in the value path


@pytest.mark.parametrize("mode", ["tensor", "dynamic"])
def test_each_call_clears_the_status_word(mode):
    """A call starts by clearing the workspace's status word: with the
    tensor-wide scale the router kernel does it (no memset ahead of it), in
    the dynamic mode a memset does.  A stale non-zero word from an earlier
    call must not survive a successful one."""
    require_cuda()
    cfg = CASES["mid_skewed"]
    c, x, wg, bias, off, W, q = _setup(cfg)
    ws = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8, device="cuda")
    g = torch.tensor([0.01]).cuda() if mode == "tensor" else torch.zeros(1).cuda()
    for _ in range(2):
        ws[:4].view(torch.int32).fill_(4)          # NVFP4_ERR_TIMEOUT left behind
        c.moe_nvfp4_forward(W, x.cuda(), g, torch.tensor([0.01]).cuda(), workspace=ws, act_scale_mode=mode,
                            logit_offset=off.cuda() if off is not None else None)
        c.nvfp4_workspace_status(ws)               # raises on a non-zero word


@pytest.mark.parametrize("name", ["tiny", "mid_skewed"])
def test_forward_replays_from_a_cuda_graph(name):
    """The forward queues kernels only (no allocation, no host sync, every
    launch a programmatic dependent), so a serving loop can capture it once
    and replay it: the replayed output is bit-identical to the eager one."""
    require_cuda()
    cfg = CASES[name]
    c, x, wg, bias, off, W, q = _setup(cfg)
    xd = x.cuda()
    off_d = off.cuda() if off is not None else None
    g1 = torch.tensor([float(xd.float().abs().max()) / 2688.0]).cuda()
    g2 = torch.tensor([0.002]).cuda()
    ws = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8, device="cuda")
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    ref = c.moe_nvfp4_forward(W, xd, g1, g2, logit_offset=off_d, workspace=ws).clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        c.moe_nvfp4_forward(W, xd, g1, g2, logit_offset=off_d, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        c.moe_nvfp4_forward(W, xd, g1, g2, logit_offset=off_d, out=out, workspace=ws)
    for _ in range(2):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    c.nvfp4_workspace_status(ws)
