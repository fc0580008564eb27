"""Router, top-k and permutation against the oracle."""
import numpy as np
import pytest
import torch

from _util import capi, host, require_cuda
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import moe

pytestmark = pytest.mark.gpu
F32 = np.float32


def _check_selection_and_permutation(c, logits, bias, k, rsf):
    E = bias.size
    res = c.moe_route(None, None, torch.from_numpy(bias).cuda(), k, rsf, logits_in=torch.from_numpy(logits).cuda())
    idx, w = moe.route(logits, bias, k, rsf)
    np.testing.assert_array_equal(host(res["topk_idx"]), idx)
    np.testing.assert_array_equal(host(res["topk_w"]).view(np.uint32), w.view(np.uint32))
    off, perm, inv = moe.permute(idx, E)
    np.testing.assert_array_equal(host(res["expert_offsets"]), off)
    gperm = host(res["perm"])
    np.testing.assert_array_equal(gperm[: perm.size], perm)
    assert np.all(gperm[perm.size:] == -1)
    np.testing.assert_array_equal(host(res["inv_perm"]), inv)
    np.testing.assert_array_equal(host(res["logits"]), logits)
    return res


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (300, 80, 8), (2049, 128, 8), (77, 256, 16), (33, 16, 16),
                                   (5000, 80, 8), (256, 80, 8), (257, 80, 8), (256, 256, 16),
                                   # the large-batch path with one, four and eight experts per lane
                                   (700, 20, 4), (1000, 100, 6), (600, 256, 16)])
def test_selection_and_permutation_from_logits(T, E, k):
    """Batches of up to 256 tokens take the single-block path, larger ones the
    two-kernel path; both must give the oracle's bytes."""
    require_cuda()
    c = capi()
    logits = workloads.random_floats((T, E), 3, f"logits{T}x{E}").numpy()
    bias = workloads.random_floats((E,), 3, f"bias{E}", std=0.01).numpy()
    _check_selection_and_permutation(c, logits, bias, k, 2.5)


def test_selection_ties_go_to_lower_expert():
    require_cuda()
    c = capi()
    # logits on a coarse grid and no bias: many exact ties in sigmoid + bias
    logits = (np.round(workloads.random_floats((512, 64), 4, "tie").numpy() * 2) / 2).astype(F32)
    _check_selection_and_permutation(c, logits, np.zeros(64, F32), 8, 1.0)


def test_skewed_loads_and_empty_experts():
    require_cuda()
    c = capi()
    T, E, k = 1000, 80, 8
    logits = workloads.random_floats((T, E), 5, "skew").numpy()
    logits[:, :20] += 4.0            # experts 0..19 take most tokens
    logits[:, 60:] -= 30.0           # experts 60..79 get none
    res = _check_selection_and_permutation(c, logits.astype(F32), np.zeros(E, F32), k, 2.5)
    off = host(res["expert_offsets"])
    assert np.all(np.diff(off)[60:] == 0)


@pytest.mark.parametrize("name,T,H,E,k,offset_std", [("tiny", 32, 256, 8, 2, 0.0),
                                                     ("mid", 1000, 1024, 80, 8, 0.5),
                                                     ("decode", 16, 6144, 80, 8, 0.0),
                                                     ("prefill", 8192, 6144, 80, 8, 0.5),
                                                     # router split counts 1 and 24 on the large-batch path
                                                     ("one_split", 9600, 512, 80, 8, 0.0),
                                                     ("many_splits", 600, 6144, 80, 8, 0.0),
                                                     # 25 K stages: six splits of five would leave one empty,
                                                     # so the router takes five (one token, then the large path)
                                                     ("odd_stages", 1, 1600, 16, 4, 0.0),
                                                     ("odd_stages_large", 300, 1600, 80, 8, 0.0)])
def test_route_from_hidden_states(name, T, H, E, k, offset_std):
    """Logits match fp64 within the fp32 summation bound; top-k sets match
    wherever the oracle's k-th and (k+1)-th biased scores are apart by more
    than the logit error can move them."""
    require_cuda()
    c = capi()
    cfg = workloads.LayerConfig(name, T=T, H=H, I=128, E=E, k=k, x_outlier_p=0.001, logit_offset_std=offset_std,
                                gen_device="cpu")
    x = workloads.hidden_states(cfg)
    wg, bias, off = workloads.router_params(cfg)
    res = c.moe_route(x.cuda(), wg.cuda(), bias.cuda(), k, 2.5, logit_offset=None if off is None else off.cuda())
    xf, wf = x.float().numpy(), wg.float().numpy()
    L = moe.router_logits(xf, wf, None if off is None else off.numpy())
    mag = np.abs(xf.astype(np.float64)) @ np.abs(wf.astype(np.float64)).T
    err = np.abs(host(res["logits"]).astype(np.float64) - L)
    assert np.all(err <= 1e-5 * mag + 1e-6), float((err / (mag + 1e-30)).max())
    idx, _ = moe.route(L, bias.numpy(), k, 2.5)
    sig = moe.sigmoid_f32(L).astype(np.float64)
    cb = np.sort(sig + bias.numpy()[None, :], axis=1)[:, ::-1]
    margin = cb[:, k - 1] - cb[:, k]
    # d sigma / d logit <= 1/4, so a logit error e moves a score by at most e/4
    safe = margin > 0.5 * (1e-5 * mag.max(axis=1) + 1e-6) + 1e-6
    gidx = host(res["topk_idx"])
    same = np.all(np.sort(gidx, axis=1) == np.sort(idx, axis=1), axis=1)
    assert np.all(same[safe]), np.nonzero(~same & safe)[0][:10]
    assert same.mean() > 0.99
