"""The layer with the shared BF16 expert (reading R19: one SiLU-gated MLP of
the routed experts' shape on every token, intermediate rounded to bf16,
added before the output's bf16 rounding) against the oracle.  The shared
expert runs on the same persistent tcgen05 GEMM as the routed experts, with
bf16 operands (kind::f16) instead of block-scaled FP4.  Below half a wave of
tiles (every case here but "long") its K is split over several CTAs whose
fp32 partial sums a second kernel adds in part order."""
import numpy as np
import pytest
import torch

from _util import capi, host, rel_l2, require_cuda
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import moe, nvfp4

pytestmark = pytest.mark.gpu
F32 = np.float32

CASES = {
    "tiny": workloads.CONFIGS["tiny"],
    "mid": workloads.LayerConfig("mid", T=300, H=1024, I=512, E=16, k=4, x_outlier_p=0.001),
    "ragged_small": workloads.LayerConfig("rs", T=3, H=512, I=256, E=6, k=3),
    # enough tokens that the shared GEMMs fill half a wave: no split K
    "long": workloads.LayerConfig("long", T=2560, H=1024, I=512, E=16, k=4),
}


@pytest.mark.parametrize("name", list(CASES))
def test_layer_with_shared_expert_matches_oracle(name):
    require_cuda()
    cfg = CASES[name]
    c = capi()
    x = workloads.hidden_states(cfg, device="cpu")
    wg, bias, off = workloads.router_params(cfg, device="cpu")
    gate, up, down = workloads.stacked_expert_weights(cfg, device="cpu")
    W = c.MoeWeights.quantize(gate.cuda(), up.cuda(), down.cuda(), wg.cuda(), bias.cuda(), cfg.k, cfg.rsf)
    q = {e: tuple(nvfp4.quantize_weight(t[e].float().numpy()) for t in (gate, up, down)) for e in range(cfg.E)}
    sh = workloads.expert_weights(cfg, cfg.E + 7, 0, device="cpu")       # one more expert's worth of bf16 weights
    Ws = W.with_shared(*(t.cuda().contiguous() for t in sh))
    shf = tuple(t.float().numpy() for t in sh)

    xf, wf, bf = x.float().numpy(), wg.float().numpy(), bias.numpy()
    g1 = F32(F32(np.abs(xf).max()) / F32(2688))
    g2 = F32(4e-4)
    ref = moe.moe_layer(xf, wf, bf, cfg.k, cfg.rsf, lambda e: q[e], g1, g2, shared=shf)
    g1t, g2t = torch.tensor([g1]).cuda(), torch.tensor([g2]).cuda()
    out, dbg = c.moe_nvfp4_forward(Ws, x.cuda(), g1t, g2t, debug=True)
    c.nvfp4_workspace_status(dbg["workspace"])
    same = np.all(host(dbg["topk_idx"]) == ref["topk_idx"], axis=1)
    assert same.mean() >= 0.97
    err = rel_l2(host(out)[same], ref["out"][same])
    assert err <= 1e-2, err

    # the shared expert's own contribution: the difference of the layer with
    # and without it, against the oracle's shared MLP
    plain = c.moe_nvfp4_forward(W, x.cuda(), g1t, g2t)
    diff = host(out).astype(np.float64) - host(plain).astype(np.float64)
    ys = moe.shared_expert(xf, shf)
    assert rel_l2(diff, ys) <= 2e-2, rel_l2(diff, ys)
    # deterministic
    assert torch.equal(out, c.moe_nvfp4_forward(Ws, x.cuda(), g1t, g2t))


def test_shared_expert_argument_checks():
    require_cuda()
    cfg = CASES["tiny"]
    c = capi()
    x = workloads.hidden_states(cfg, device="cpu")
    wg, bias, off = workloads.router_params(cfg, device="cpu")
    gate, up, down = workloads.stacked_expert_weights(cfg, device="cpu")
    W = c.MoeWeights.quantize(gate.cuda(), up.cuda(), down.cuda(), wg.cuda(), bias.cuda(), cfg.k, cfg.rsf)
    g = torch.tensor([0.01]).cuda()
    # I_shared not a multiple of 128
    bad = W.with_shared(torch.zeros(64, cfg.H, dtype=torch.bfloat16, device="cuda"),
                        torch.zeros(64, cfg.H, dtype=torch.bfloat16, device="cuda"),
                        torch.zeros(cfg.H, 64, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(c.Nvfp4Error):
        c.moe_nvfp4_forward(bad, x.cuda(), g, g)
