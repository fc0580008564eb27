"""The weight quantiser's no-allocation entry point.

nvfp4_quantize_weights_noalloc serves callers that cannot allocate device
memory (their device heap belongs to another allocator, or allocation calls
are not allowed where they run): its scratch is an array built into the
library instead of a caller workspace.  It must give exactly the bytes of the
workspace form, on consecutive calls too, since every call reuses the same
array.  Its status word (set when a device-side wait gives up) is read with
nvfp4_quantize_weights_noalloc_status, which must report OK after normal
calls.  This file is collected last so that a run stopping at the first
failure has run every other test already.
"""
import numpy as np
import pytest
import torch

from _util import capi, host, require_cuda
from nvfp4_w4a4_quantized_moe_b200 import workloads

pytestmark = pytest.mark.gpu


def _weights(seed, n, rows, cols):
    w = workloads.random_floats((n, rows, cols), seed, f"noalloc{seed}", std=0.02)
    w[1] = 0.0                                                   # an all-zero matrix
    w[-1] *= 40.0                                                # a different global scale
    return w.to(torch.bfloat16).cuda()


@pytest.mark.parametrize("layout", ["tiled", "canonical", "staged"])
def test_noalloc_matches_workspace_form_on_consecutive_calls(layout):
    require_cuda()
    c = capi()
    # two different problems back to back: the second call must not see the
    # first call's leftovers in the shared scratch array
    for seed, shape in ((1, (6, 256, 512)), (2, (3, 128, 2048))):
        w = _weights(seed, *shape)
        ref = [host(t) for t in c.nvfp4_quantize_weights(w, layout)]
        for _ in range(2):
            got = [host(t) for t in c.nvfp4_quantize_weights_noalloc(w, layout)]
            c.nvfp4_quantize_weights_noalloc_status()        # no wait gave up
            for a, b in zip(got, ref):
                np.testing.assert_array_equal(a.view(np.uint8), b.view(np.uint8))


def test_noalloc_checks_the_output_tensors_it_is_given():
    """Outputs passed in must be CUDA tensors of the right dtype and at least
    the size the call writes; nothing is queued otherwise."""
    require_cuda()
    c = capi()
    w = _weights(3, 2, 128, 256)
    codes, scales, gscale = c.nvfp4_quantize_weights(w, "tiled")
    with pytest.raises(ValueError, match="codes holds"):
        c.nvfp4_quantize_weights_noalloc(w, "tiled", out=(codes[:1], scales, gscale))
    with pytest.raises(ValueError, match="scales holds"):
        c.nvfp4_quantize_weights_noalloc(w, "tiled", out=(codes, scales[:-1], gscale))
    with pytest.raises(ValueError, match="gscale"):
        c.nvfp4_quantize_weights_noalloc(w, "tiled", out=(codes, scales, gscale.double()))
    with pytest.raises(ValueError, match="CUDA tensor"):
        c.nvfp4_quantize_weights_noalloc(w, "tiled", out=(codes.cpu(), scales, gscale))
    got = c.nvfp4_quantize_weights_noalloc(w, "tiled", out=(torch.empty_like(codes), torch.empty_like(scales),
                                                            torch.empty_like(gscale)))
    c.nvfp4_quantize_weights_noalloc_status()
    for a, b in zip(got, (codes, scales, gscale)):
        np.testing.assert_array_equal(host(a).view(np.uint8), host(b).view(np.uint8))


def test_noalloc_rejects_more_matrices_than_its_scratch_holds():
    require_cuda()
    c = capi()
    w = torch.zeros((1025, 128, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(c.Nvfp4Error) as e:
        c.nvfp4_quantize_weights_noalloc(w, "tiled")
    assert e.value.status == 2 and "1024" in str(e.value)
