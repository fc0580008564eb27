"""The device-side give-up path, made to run on the GPU.

Every wait of the library's kernels is bounded: when it runs out, the kernel
sets the status word at the start of the workspace, lets its copies in flight
land, drains its tensor-core work, frees its tensor memory and returns, and
the host reads the word with nvfp4_workspace_status.  Here a test kernel waits
on a barrier that nothing completes, with a 1 ms limit, so the wait gives up
for certain.  The status word must report the timeout (once: reading it
resets it), the copy must have landed, and the context must stay usable: a
layer forward afterwards, on the same workspace, must succeed and give the
bits of a forward on a fresh workspace."""
import numpy as np
import pytest
import torch

from _util import capi, require_cuda
from nvfp4_w4a4_quantized_moe_b200 import workloads

pytestmark = pytest.mark.gpu
LIMIT_NS = 1_000_000          # 1 ms


def _tiny_layer(c):
    cfg = workloads.CONFIGS["tiny"]
    x = workloads.hidden_states(cfg, device="cpu").cuda()
    wg, bias, _ = workloads.router_params(cfg, device="cpu")
    gate, up, down = (t.cuda() for t in workloads.stacked_expert_weights(cfg, device="cpu"))
    W = c.MoeWeights.quantize(gate, up, down, wg.cuda(), bias.cuda(), cfg.k, cfg.rsf)
    g1 = (x.float().abs().amax() / 2688.0).reshape(1)
    g2 = torch.tensor([2e-4], device="cuda")
    return cfg, W, x, g1, g2


def test_a_wait_that_runs_out_sets_the_status_word_and_the_context_stays_usable():
    require_cuda()
    c = capi()
    cfg, W, x, g1, g2 = _tiny_layer(c)
    ws = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8,
                     device="cuda")
    src = workloads.random_bytes((4096,), 9, "timeout_src", device="cpu").cuda()
    elapsed, copied = c.nvfp4_test_wait_timeout(src, LIMIT_NS, ws)
    with pytest.raises(c.Nvfp4Error) as err:
        c.nvfp4_workspace_status(ws)
    assert err.value.status == 4                             # NVFP4_ERR_TIMEOUT
    c.nvfp4_workspace_status(ws)                             # reading it reset it
    el = elapsed.cpu().numpy()
    # the limited wait lasted at least its limit and far less than the
    # library's default 2 s; the second warp left on the abort flag
    assert LIMIT_NS <= el[0] < 500_000_000, el
    assert 0 < el[1] < 1_000_000_000, el
    words = src.cpu().numpy().view(np.uint32)
    assert int(copied.cpu().numpy().view(np.uint32)[0]) == int(np.bitwise_xor.reduce(words))
    # the same workspace serves a forward afterwards, with a clear status word
    out = c.moe_nvfp4_forward(W, x, g1, g2, workspace=ws)
    c.nvfp4_workspace_status(ws)
    ref = c.moe_nvfp4_forward(W, x, g1, g2)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_wait_limit_is_checked_on_the_host():
    require_cuda()
    c = capi()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    src = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    for bad in (0, 2_000_000_000):
        with pytest.raises(c.Nvfp4Error) as err:
            c.nvfp4_test_wait_timeout(src, bad, ws)
        assert err.value.status == 1
    c.nvfp4_workspace_status(ws)                             # nothing was queued
