"""The layer at full size, in the configuration the benchmark times, against
the oracle on sampled tokens.

The GPU runs the whole batch (decode: 16 tokens, prefill: 8192 tokens with
skewed expert loads, outlier: 4096 tokens over 128 experts with outlier
weights).  The oracle evaluates two sampled tokens end to end (its own
routing, x quantisation, the tokens' experts quantised by the oracle itself,
gate/up, requantisation, down, combine) and every token's routing.  Expert
quantisation on the host runs in a spawn process pool.
"""
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

from _util import capi, host, rel_l2, require_cuda, tiled_rows
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import moe, nvfp4

pytestmark = pytest.mark.gpu
F32 = np.float32


def _oracle_experts(gate, up, down, experts):
    from _oracle_pool import quantize_expert
    jobs = [tuple(t[e].float().cpu().numpy() for t in (gate, up, down)) for e in experts]
    with mp.get_context("spawn").Pool(min(len(jobs), max(1, (os.cpu_count() or 2) - 1))) as pool:
        out = pool.map(quantize_expert, jobs)
    return dict(zip(experts, out))


@pytest.mark.parametrize("name", ["decode", "prefill", "outlier"])
def test_full_size_layer_on_sampled_tokens(name):
    require_cuda()
    c = capi()
    cfg = workloads.CONFIGS[name]
    dev = torch.device("cuda")
    x = workloads.hidden_states(cfg, device=dev)
    wg, bias, off = workloads.router_params(cfg, device=dev)
    gate, up, down = workloads.stacked_expert_weights(cfg, device=dev)
    W = c.MoeWeights.quantize(gate, up, down, wg, bias, cfg.k, cfg.rsf)

    xf = x.float().cpu().numpy()
    wf = wg.float().cpu().numpy()
    bf = bias.cpu().numpy()
    offn = None if off is None else off.cpu().numpy()
    tokens = [0, cfg.T // 2 + 1]
    g1 = F32(F32(np.abs(xf).max()) / F32(2688))

    # routing of every token (oracle logits in fp64, selection in fp32)
    L = moe.router_logits(xf, wf, offn)
    idx, wts = moe.route(L, bf, cfg.k, cfg.rsf)
    experts = sorted(set(int(e) for t in tokens for e in idx[t]))
    q = _oracle_experts(gate, up, down, experts)

    # g2 from the oracle's own h of the sampled tokens
    cal = moe.moe_layer(xf, wf, bf, cfg.k, cfg.rsf, lambda e: q[e], g1, F32(1.0), tokens=tokens, logits=L[tokens])
    g2 = F32(F32(max(np.abs(h).max() for h in cal["h"].values())) / F32(2688))
    ref = moe.moe_layer(xf, wf, bf, cfg.k, cfg.rsf, lambda e: q[e], g1, g2, tokens=tokens, logits=L[tokens])

    out, dbg = c.moe_nvfp4_forward(W, x, torch.tensor([g1], device=dev), torch.tensor([g2], device=dev),
                                   logit_offset=off, debug=True)
    c.nvfp4_workspace_status(dbg["workspace"])

    # every token: logits within the fp32 summation bound, safe selections equal
    mag = np.abs(xf.astype(np.float64)) @ np.abs(wf.astype(np.float64)).T
    gl = host(dbg["logits"]).astype(np.float64)
    assert np.all(np.abs(gl - L) <= 1e-5 * mag + 1e-6)
    sig = moe.sigmoid_f32(L).astype(np.float64)
    cb = np.sort(sig + bf[None, :], axis=1)[:, ::-1]
    safe = (cb[:, cfg.k - 1] - cb[:, cfg.k]) > 0.5 * (1e-5 * mag.max(axis=1) + 1e-6) + 1e-6
    gidx = host(dbg["topk_idx"])
    # the selected sets must agree; the order inside a set may differ where two
    # selected scores are closer than the logit error
    same = np.all(np.sort(gidx, axis=1) == np.sort(idx, axis=1), axis=1)
    assert np.all(same[safe]) and (same.mean() > 0.99 or (~same).sum() <= 1)
    # permutation: every (token, slot) lands in its expert's segment, in token order
    off_g, perm_g, inv_g = host(dbg["expert_offsets"]), host(dbg["perm"]), host(dbg["inv_perm"])
    counts = np.bincount(gidx.ravel(), minlength=cfg.E)
    assert np.all(np.diff(off_g) == -(-counts // 128) * 128)
    rows = inv_g.ravel()
    assert np.unique(rows).size == rows.size
    assert np.all(perm_g[inv_g] == np.arange(cfg.T)[:, None])
    assert np.all(off_g[gidx] <= inv_g) and np.all(inv_g < off_g[gidx + 1])

    # the sampled tokens end to end
    a_sc_host = host(dbg["a_scales"])
    for n, t in enumerate(tokens):
        assert same[t], f"token {t} routed differently (margin below the fp32 logit error)"
        slot_of = {int(e): j for j, e in enumerate(ref["topk_idx"][n])}      # oracle slot of each expert
        gw = host(dbg["topk_w"])[t]
        np.testing.assert_allclose(gw, [ref["topk_w"][n][slot_of[int(e)]] for e in gidx[t]], rtol=2e-5)
        a_codes, a_scales = nvfp4.quantize(xf[t:t + 1], g1)
        h_g = host(dbg["h"][torch.as_tensor(inv_g[t], device=dev).long()])
        hc_g = host(dbg["h_codes"][torch.as_tensor(inv_g[t], device=dev).long()])
        flips = 0
        for j in range(cfg.k):
            r = inv_g[t, j]
            np.testing.assert_array_equal(host(dbg["a_codes"][r]), a_codes[0])
            np.testing.assert_array_equal(tiled_rows(a_sc_host, [r], cfg.H)[0], a_scales[0])
            hr = ref["h"][(t, slot_of[int(gidx[t, j])])]
            assert rel_l2(h_g[j], hr) <= 1e-3
            rc, _ = nvfp4.quantize(hr[None, :], g2)
            flips += int(np.count_nonzero(nvfp4.unpack_codes(hc_g[j:j + 1]) != nvfp4.unpack_codes(rc)))
        assert flips <= 0.001 * cfg.k * cfg.I, f"token {t}: {flips} requantised codes differ"
        err = rel_l2(host(out[t]), ref["out"][n])
        assert err <= 1e-2, f"token {t}: output rel L2 {err:.3g}"
    del W, gate, up, down, dbg, out
    torch.cuda.empty_cache()
