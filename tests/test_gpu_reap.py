"""REAP saliency on the GPU (the down GEMM's epilogue and a per-expert finish
kernel) against the oracle, and the pruned layer ("K-EXAONE-152B-A23B-REAP-
80E-BF16" model card, "Pruning Setup": saliency = mean(topk_weight *
||f_e(x)||_2) over routed tokens; gate.weight and e_score_correction_bias
sliced to the retained experts)."""
import numpy as np
import pytest
import torch

from _util import capi, host, rel_l2, require_cuda
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import moe, nvfp4

pytestmark = pytest.mark.gpu
F32 = np.float32


def _layer(cfg):
    c = capi()
    x = workloads.hidden_states(cfg, device="cpu")
    wg, bias, off = workloads.router_params(cfg, device="cpu")
    gate, up, down = workloads.stacked_expert_weights(cfg, device="cpu")
    W = c.MoeWeights.quantize(gate.cuda(), up.cuda(), down.cuda(), wg.cuda(), bias.cuda(), cfg.k, cfg.rsf)
    q = {e: tuple(nvfp4.quantize_weight(t[e].float().numpy()) for t in (gate, up, down)) for e in range(cfg.E)}
    return c, x, wg, bias, off, W, q


@pytest.mark.parametrize("name,cfg", [
    ("tiny", workloads.CONFIGS["tiny"]),
    ("mid", workloads.LayerConfig("mid", T=300, H=1024, I=512, E=16, k=4, logit_offset_std=0.5)),
    # 2,400 rows: the CTA-pair GEMMs, whose down epilogue both CTAs of a pair
    # run (sums of squares of their own rows)
    ("pair", workloads.LayerConfig("pr", T=600, H=1024, I=256, E=16, k=4, logit_offset_std=0.5)),
])
def test_saliency_and_pruned_layer_match_oracle(name, cfg):
    require_cuda()
    c, x, wg, bias, off, W, q = _layer(cfg)
    xf, wf, bf = x.float().numpy(), wg.float().numpy(), bias.numpy()
    offn = None if off is None else off.numpy()
    g1 = F32(F32(np.abs(xf).max()) / F32(2688))
    g2 = F32(4e-4)
    ref = moe.moe_layer(xf, wf, bf, cfg.k, cfg.rsf, lambda e: q[e], g1, g2, logit_offset=offn)
    s_ref, n_ref = moe.reap_saliency(ref, cfg.E)

    sal = (torch.zeros(cfg.E, dtype=torch.float64, device="cuda"), torch.zeros(cfg.E, dtype=torch.int64, device="cuda"))
    g1t, g2t = torch.tensor([g1]).cuda(), torch.tensor([g2]).cuda()
    offt = None if off is None else off.cuda()
    out, dbg = c.moe_nvfp4_forward(W, x.cuda(), g1t, g2t, logit_offset=offt, debug=True, saliency=sal)
    c.nvfp4_workspace_status(dbg["workspace"])
    # a second batch adds to the accumulators: exactly twice the first
    out2 = c.moe_nvfp4_forward(W, x.cuda(), g1t, g2t, logit_offset=offt, saliency=sal)
    assert torch.equal(out, out2)
    s_gpu, n_gpu = host(sal[0]) / 2, host(sal[1]) // 2

    gidx = host(dbg["topk_idx"])
    if np.array_equal(gidx, ref["topk_idx"]):
        np.testing.assert_array_equal(n_gpu, n_ref)
        np.testing.assert_allclose(s_gpu, s_ref, rtol=2e-3)
    else:   # a near-tie routed differently: compare experts the routing agrees on
        for e in range(cfg.E):
            if np.array_equal(gidx == e, ref["topk_idx"] == e):
                assert n_gpu[e] == n_ref[e]
                assert s_gpu[e] == pytest.approx(s_ref[e], rel=2e-3)

    # prune to 5/8 of the experts (128 -> 80 in the model); the retained set
    # must be the oracle's unless two saliencies at the cut are within 1e-3
    keep_n = cfg.E * 5 // 8
    keep = c.reap_keep(sal[0], sal[1], keep_n)
    mean_ref = np.where(n_ref > 0, s_ref / np.maximum(n_ref, 1), 0.0)
    keep_ref = moe.reap_keep(mean_ref, keep_n)
    srt = np.sort(mean_ref)[::-1]
    if srt[keep_n - 1] - srt[keep_n] > 1e-3 * srt[keep_n - 1]:
        np.testing.assert_array_equal(keep.numpy(), keep_ref)
    kept = keep.numpy()

    # the pruned layer on the GPU against the oracle on the sliced weights
    Wp = c.select_experts(W, keep)
    bp = bf[kept]
    op = None if offn is None else offn[kept]
    refp = moe.moe_layer(xf, wf[kept], bp, cfg.k, cfg.rsf, lambda e: q[int(kept[e])], g1, g2, logit_offset=op)
    outp, dbgp = c.moe_nvfp4_forward(Wp, x.cuda(), g1t, g2t,
                                     logit_offset=None if op is None else torch.from_numpy(op).cuda(), debug=True)
    same = np.all(host(dbgp["topk_idx"]) == refp["topk_idx"], axis=1)
    assert same.mean() >= 0.97
    assert rel_l2(host(outp)[same], refp["out"][same]) <= 1e-2


def test_library_retention_matches_the_oracle_with_ties_and_unrouted_experts():
    """moe_reap_keep against the oracle's reap_keep on accumulators with exact
    ties between means (reached from different sums and counts), experts never
    routed (mean 0) and every keep count from 0 to E."""
    require_cuda()
    c = capi()
    rng = np.random.default_rng(11)
    E = 96
    count = rng.integers(1, 50, E).astype(np.int64)
    total = rng.uniform(0.0, 10.0, E) * count
    count[[3, 17, 40]] = 0
    total[[3, 17, 40]] = 0.0
    # ties: equal means from different (sum, count) pairs, and duplicated pairs
    total[[5, 9, 60]] = [3.0, 6.0, 1.5]
    count[[5, 9, 60]] = [2, 4, 1]
    total[[70, 71]] = total[20], total[20]
    count[[70, 71]] = count[20], count[20]
    mean = np.where(count > 0, total / np.maximum(count, 1), 0.0)
    st = torch.from_numpy(total).cuda()
    ct = torch.from_numpy(count).cuda()
    for keep_n in range(E + 1):
        got = c.reap_keep(st, ct, keep_n).numpy()
        np.testing.assert_array_equal(got, moe.reap_keep(mean, keep_n))
