"""The forward on host buffers (moe_nvfp4_forward_host): x copied in and out
through staging buffers at the end of the workspace, on the library's copy
streams.  Its output must equal the device-buffer forward's bit for bit,
with consecutive calls alternating between two workspaces (so that one
call's copies overlap another's compute) and with calls that reuse one
workspace (so that a call waits for the previous call's copies)."""
import pytest
import torch

from _util import capi, require_cuda
from nvfp4_w4a4_quantized_moe_b200 import workloads

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": workloads.CONFIGS["tiny"],
    "mid": workloads.LayerConfig("mid", T=300, H=1024, I=512, E=16, k=4, x_outlier_p=0.001),
}


@pytest.mark.parametrize("name", list(CASES))
def test_host_forward_equals_device_forward(name):
    require_cuda()
    cfg = CASES[name]
    c = capi()
    dev = torch.device("cuda")
    wg, bias, off = workloads.router_params(cfg, device=dev)
    gate, up, down = workloads.stacked_expert_weights(cfg, device=dev)
    W = c.MoeWeights.quantize(gate, up, down, wg, bias, cfg.k, cfg.rsf)
    xs = [workloads.hidden_states(cfg, seed, device=dev) for seed in range(5)]
    g1 = (xs[0].float().abs().amax() / 2688.0).reshape(1).float()
    g2 = torch.tensor([4e-4], device=dev)
    want = [c.moe_nvfp4_forward(W, x, g1, g2, logit_offset=off).cpu() for x in xs]

    nbytes = c.moe_nvfp4_workspace_size_host(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k)
    wss = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    xh = [x.cpu().pin_memory() for x in xs]
    outs = [torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in xs]
    # calls 0..3 alternate between the two workspaces; call 4 reuses workspace 0
    # right after call 2 and 3 were queued on the two
    for i in range(4):
        c.moe_nvfp4_forward_host(W, xh[i], g1, g2, outs[i], wss[i % 2], logit_offset=off)
    c.moe_nvfp4_forward_host(W, xh[4], g1, g2, outs[4], wss[0], logit_offset=off)
    for ws in wss:
        c.moe_nvfp4_host_join(ws)
    torch.cuda.current_stream().synchronize()
    for i in range(5):
        assert torch.equal(outs[i], want[i]), i
    for ws in wss:
        c.nvfp4_workspace_status(ws)
        c.moe_nvfp4_host_release(ws)
    # a released workspace is usable again (its events are created anew)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
    c.moe_nvfp4_forward_host(W, xh[1], g1, g2, out, wss[1], logit_offset=off)
    c.moe_nvfp4_host_join(wss[1])
    torch.cuda.current_stream().synchronize()
    assert torch.equal(out, want[1])
    c.moe_nvfp4_host_release(wss[1])


def test_host_forward_rejects_device_tensors_and_small_workspaces():
    require_cuda()
    cfg = CASES["tiny"]
    c = capi()
    dev = torch.device("cuda")
    wg, bias, off = workloads.router_params(cfg, device=dev)
    gate, up, down = workloads.stacked_expert_weights(cfg, device=dev)
    W = c.MoeWeights.quantize(gate, up, down, wg, bias, cfg.k, cfg.rsf)
    x = workloads.hidden_states(cfg, 0, device=dev)
    g = torch.tensor([0.01], device=dev)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16)
    ws = torch.empty(c.moe_nvfp4_workspace_size_host(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8,
                     device=dev)
    with pytest.raises(ValueError):
        c.moe_nvfp4_forward_host(W, x, g, g, out, ws)                 # x on the device
    small = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8,
                        device=dev)
    with pytest.raises(c.Nvfp4Error):
        c.moe_nvfp4_forward_host(W, x.cpu(), g, g, out, small)         # no room for the staging buffers
