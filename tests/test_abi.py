"""The C ABI library builds for sm_100a, loads, exports what the headers
declare and rejects bad arguments on the host (CPU only, no kernel launch)."""
import ctypes
import subprocess

import pytest

from _util import ROOT, capi, header_functions


def test_library_exports_every_declared_function():
    c = capi()
    declared = header_functions()
    assert len(declared) >= 18
    out = subprocess.run(["nm", "-D", "--defined-only", c.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [n for n in declared if n not in exported]
    assert not missing, missing
    assert set(c.EXPORTS) == set(declared)
    for n in declared:
        assert hasattr(c.lib, n)


def test_abi_version_and_sizes():
    c = capi()
    assert c.abi_version() == 6
    assert c.moe_route_rows_capacity(8192, 80, 8) == 75776
    assert c.moe_route_rows_capacity(16, 80, 8) % 128 == 0
    assert c.lib.moe_nvfp4_workspace_size(16, 80, 6144, 2048, 8) > 0
    # the host-buffer forward: the forward's workspace, then x and out staging
    r256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    for T in (1, 16, 8192):
        base = c.lib.moe_nvfp4_workspace_size_shared(T, 80, 6144, 2048, 8, 0)
        assert c.moe_nvfp4_workspace_size_host(T, 80, 6144, 2048, 8) == r256(base) + 2 * r256(T * 6144 * 2)
    assert c.moe_nvfp4_workspace_size_host(0, 80, 6144, 2048, 8) == 0
    # zero tokens: the sizes stay defined (no division by the m-tile count)
    assert c.lib.moe_nvfp4_workspace_size(0, 80, 6144, 2048, 8) > 0
    assert c.lib.moe_route_workspace_size(0, 80, 8) > 0
    assert c.lib.nvfp4_quantize_weights_workspace_size(240) >= 256


def test_forward_launch_count_follows_the_shape():
    """The host-only launch count of the forward: router GEMM, routing (one
    kernel up to 256 tokens, else two), quantise-scatter (inside the routing
    kernel when at most 64 KiB of permuted rows), gate/up, down, combine, plus
    the shared expert's three kernels (and a reduction after each of its GEMMs
    when few tokens split their K), and the dynamic modes' amax kernels."""
    c = capi()
    n = c.moe_nvfp4_forward_launches
    assert n(32, 8, 256, 128, 2) == 5          # tiny layer: 32 x 2 rows of 144 bytes
    assert n(16, 80, 6144, 2048, 8) == 6       # decode: 442 KB of rows, a separate quantise kernel
    assert n(256, 80, 6144, 2048, 8) == 6
    assert n(257, 80, 6144, 2048, 8) == 7      # two routing kernels above 256 tokens
    assert n(8192, 80, 6144, 2048, 8) == 7
    # the shared expert at 16 tokens: both GEMMs split K, each adding a reduction
    assert n(16, 80, 6144, 2048, 8, I_shared=2048) == 11
    assert n(8192, 80, 6144, 2048, 8, I_shared=2048) == 10
    # the split K of the shared GEMMs starts below half a wave of tiles: 300
    # tokens are 3 x 4 tiles each (both split), 2560 tokens 20 x 4 (neither)
    assert n(300, 16, 1024, 512, 4, I_shared=512) == 7 + 3 + 2
    assert n(2560, 16, 1024, 512, 4, I_shared=512) == 7 + 3
    assert n(3, 6, 512, 256, 3, I_shared=256) == 5 + 3 + 2
    assert n(32, 8, 256, 128, 2, act_scale_mode="expert") == 6     # per-expert g1: no fused quantisation
    assert n(16, 80, 6144, 2048, 8, act_scale_mode="dynamic") == 7
    assert n(16, 80, 6144, 2048, 8, act_scale_mode="dynamic_expert") == 8
    # the 64 KiB bound of the fused path: 227 rows of 288 bytes fit, 228 do not
    assert n(227, 8, 512, 256, 1) == 5 and n(228, 8, 512, 256, 1) == 6
    with pytest.raises(ValueError):
        n(16, 80, 6000, 2048, 8)                # H % 256 != 0
    assert c.lib.moe_nvfp4_forward_launches(16, 80, 6144, 2048, 8, 0, 7) == -1


def test_router_splits_leave_no_split_empty():
    """The router GEMM's K split (host arithmetic): every split gets K stages,
    at least four where it has company, and the CTAs (one per 128 tokens and
    split) stay within one wave of the 148 SMs."""
    c = capi()
    for T in (1, 16, 100, 128, 129, 257, 300, 1000, 2048, 4096, 8192, 9600, 20000):
        mt = -(-T // 128)
        for H in range(64, 32768 + 1, 64):
            sp, per = c.nvfp4_test_router_splits(T, H)
            kt = H // 64
            assert sp >= 1 and per >= 1
            assert (sp - 1) * per < kt <= sp * per, (T, H, sp, per)    # the last split has stages
            assert sp * mt <= max(148, mt)
            if sp > 1:
                assert per >= 4
    assert c.nvfp4_test_router_splits(16, 6144) == (24, 4)       # decode
    assert c.nvfp4_test_router_splits(8192, 6144) == (2, 48)     # prefill
    assert c.nvfp4_test_router_splits(1, 1600) == (5, 5)         # 25 stages: five splits, not six
    assert c.nvfp4_test_router_splits(129, 19200) == (60, 5)     # 300 stages: 74 splits of 5 would leave 14 empty
    with pytest.raises(ValueError):
        c.nvfp4_test_router_splits(1, 100)


def test_host_side_argument_checks():
    c = capi()
    lib = c.lib
    # NULL pointers: rejected before any CUDA call
    assert lib.nvfp4_quantize_act(None, 4, 64, None, 0, None, None, None) == 1
    assert b"NULL" in lib.nvfp4_last_error()
    fake = ctypes.c_void_p(0x1000)
    # unsupported shapes and layouts
    assert lib.nvfp4_quantize_act(fake, 4, 48, fake, 0, fake, fake, None) == 2
    assert lib.nvfp4_quantize_act(fake, 4, 64, fake, 7, fake, fake, None) == 1
    assert lib.nvfp4_quantize_weights(fake, 1, 100, 64, 1, fake, fake, fake, fake, 1 << 20, None) == 2
    # the staged code layout needs cols % 256 == 0
    assert lib.nvfp4_quantize_weights(fake, 1, 128, 128, 2, fake, fake, fake, fake, 1 << 20, None) == 2
    assert lib.nvfp4_quantize_weights(fake, 1, 128, 64, 3, fake, fake, fake, fake, 1 << 20, None) == 1
    # workspace too small
    assert lib.nvfp4_quantize_weights(fake, 1, 128, 64, 1, fake, fake, fake, fake, 8, None) == 5
    # routing shapes
    assert lib.moe_route(fake, fake, None, fake, None, 4, 64, 8, 9, 1.0, None, fake, fake, fake, fake, fake, fake,
                         1 << 20, None) == 2
    assert lib.moe_route(fake, fake, None, fake, None, 4, 64, 300, 8, 1.0, None, fake, fake, fake, fake, fake, fake,
                         1 << 20, None) == 2
    # layer shapes: H must be a multiple of 256
    W = c.MoeWeightsStruct(8, 192, 128, 2, 2.5, *([fake] * 11))
    assert lib.moe_nvfp4_forward(ctypes.byref(W), fake, 4, fake, fake, None, fake, None, fake, 1 << 30, None) == 2
    W = c.MoeWeightsStruct(8, 256, 128, 2, 2.5, *([fake] * 11))
    assert lib.moe_nvfp4_forward(ctypes.byref(W), fake, 4, fake, fake, None, fake, None, fake, 16, None) == 5
    # codes layout: only row-major or staged, and staged needs I % 256 == 0
    W.codes_layout = 1
    assert lib.moe_nvfp4_forward(ctypes.byref(W), fake, 4, fake, fake, None, fake, None, fake, 1 << 30, None) == 1
    W.codes_layout = 2
    assert lib.moe_nvfp4_forward(ctypes.byref(W), fake, 4, fake, fake, None, fake, None, fake, 1 << 30, None) == 2
    W = c.MoeWeightsStruct(8, 256, 256, 2, 2.5, *([fake] * 11), None, None, None, 0, 2)
    assert lib.moe_nvfp4_forward(ctypes.byref(W), fake, 4, fake, fake, None, fake, None, fake, 16, None) == 5
    # the host-buffer forward: the same shape checks, NULL buffers, its own workspace size
    assert lib.moe_nvfp4_forward_host(ctypes.byref(W), fake, 4, fake, fake, None, fake, fake, 16, None) == 5
    assert lib.moe_nvfp4_forward_host(ctypes.byref(W), None, 4, fake, fake, None, fake, fake, 1 << 30, None) == 1
    W = c.MoeWeightsStruct(8, 192, 128, 2, 2.5, *([fake] * 11))
    assert lib.moe_nvfp4_forward_host(ctypes.byref(W), fake, 4, fake, fake, None, fake, fake, 1 << 30, None) == 2
    assert lib.moe_nvfp4_host_join(None, None) == 1 and lib.moe_nvfp4_host_release(None) == 1


@pytest.mark.parametrize("header", ["nvfp4_moe.h", "nvfp4_moe_testing.h"])
@pytest.mark.parametrize("lang", [("c", "-std=c99"), ("c++", "-std=c++17")])
def test_headers_compile_as_plain_c_and_cpp(header, lang):
    """The boundary is a C ABI: its headers need no CUDA or torch headers and
    compile warning-free as C99 and as C++17."""
    import os
    import shutil
    cc = shutil.which("gcc" if lang[0] == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    r = subprocess.run([cc, "-fsyntax-only", lang[1], "-Wall", "-Wextra", "-Werror", "-x", lang[0],
                        os.path.join(ROOT, "include", header)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
