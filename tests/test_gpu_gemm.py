"""Grouped FP4 GEMMs (gate/up with SiLU*up and requantisation; down with the
weighted epilogue) on identical quantised operands: the same random codes and
scale bytes go to the CUDA kernels and to the oracle."""
import numpy as np
import pytest
import torch

from _util import canonical_to_staged, canonical_to_tiled, capi, host, rel_l2, require_cuda, tiled_to_canonical
from nvfp4_w4a4_quantized_moe_b200 import workloads
from oracle import moe, nvfp4

pytestmark = pytest.mark.gpu
F32 = np.float32
TOL = 1e-3          # rel L2 of GEMM outputs on identical quantised operands


def _codes(shape, seed, name):
    return workloads.random_bytes(shape, seed, name).numpy()


def _scales(shape, seed, name, lo=0x28, hi=0x48):
    # E4M3 codes between 2^-2 and 2^2: products stay far from fp32 limits
    return workloads.random_bytes(shape, seed, name, low=lo, high=hi).numpy()


class Problem:
    def __init__(self, E, H, I, counts, seed=0):
        self.E, self.H, self.I = E, H, I
        self.counts = np.asarray(counts, np.int32)
        padded = -(-self.counts // 128) * 128
        self.offsets = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
        self.rows = int(self.offsets[-1])
        self.cap = self.rows + 128                       # one unused tile at the end
        s = seed
        self.gate = (_codes((E, I, H // 2), s, "gc"), _scales((E, I, H // 16), s, "gs"))
        self.up = (_codes((E, I, H // 2), s, "uc"), _scales((E, I, H // 16), s, "us"))
        self.down = (_codes((E, H, I // 2), s, "dc"), _scales((E, H, I // 16), s, "ds"))
        self.g = {n: (workloads.random_floats((E,), s, "g" + n).abs().numpy() + 0.5).astype(F32)
                  for n in ("gate", "up", "down")}
        self.a_codes = _codes((self.cap, H // 2), s, "ac")
        self.a_scales = _scales((self.cap, H // 16), s, "as")
        self.h_codes = _codes((self.cap, I // 2), s, "hc")
        self.h_scales = _scales((self.cap, I // 16), s, "hs")
        self.row_w = (workloads.random_floats((self.cap,), s, "rw").abs().numpy() + 0.1).astype(F32)
        self.g1 = F32(0.013)
        self.g2 = F32(0.021)

    def weights(self, c, layout="canonical"):
        """The weights on the device; with layout "staged" the codes are
        rearranged into the staged layout (scales are tiled either way)."""
        cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
        tiled = lambda s: cu(canonical_to_tiled(s.reshape(-1, s.shape[-1])))  # noqa: E731

        def codes(a):
            if layout != "staged":
                return cu(a)
            return cu(np.stack([canonical_to_staged(m, m.shape[0], 2 * m.shape[1]) for m in a]))
        return c.MoeWeights(self.E, self.H, self.I, 1, 1.0, torch.zeros((self.E, self.H), dtype=torch.bfloat16).cuda(),
                            torch.zeros(self.E).cuda(), codes(self.gate[0]), tiled(self.gate[1]), cu(self.g["gate"]),
                            codes(self.up[0]), tiled(self.up[1]), cu(self.g["up"]), codes(self.down[0]),
                            tiled(self.down[1]), cu(self.g["down"]),
                            codes_layout=c.LAYOUT_STAGED if layout == "staged" else c.LAYOUT_CANONICAL)

    def segments(self):
        for e in range(self.E):
            yield e, int(self.offsets[e]), int(self.counts[e])


def _oracle_gate_up(P, e, r0, n):
    gq = (P.gate[0][e], P.gate[1][e], P.g["gate"][e])
    uq = (P.up[0][e], P.up[1][e], P.g["up"][e])
    return moe.expert_gate_up(P.a_codes[r0:r0 + n], P.a_scales[r0:r0 + n], P.g1, gq, uq)


PROBLEMS = {
    "one_tile": dict(E=1, H=256, I=128, counts=[128]),
    "ragged": dict(E=3, H=1024, I=256, counts=[5, 0, 300]),
    "tiny_shape": dict(E=8, H=256, I=128, counts=[7, 9, 0, 16, 3, 1, 20, 8]),
    "deep_k": dict(E=2, H=6144, I=256, counts=[130, 64]),
    "wide": dict(E=2, H=512, I=2048, counts=[200, 20]),
}


def _layout_params():
    """(problem, codes layout) pairs: every problem with row-major codes, and
    with staged codes where H and I are multiples of 256."""
    out = []
    for n, p in PROBLEMS.items():
        out.append((n, "canonical"))
        if p["H"] % 256 == 0 and p["I"] % 256 == 0:
            out.append((n, "staged"))
    return out


@pytest.mark.parametrize("name,layout", _layout_params())
def test_gate_up_matches_oracle(name, layout):
    require_cuda()
    c = capi()
    P = Problem(**PROBLEMS[name])
    W = P.weights(c, layout)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    res = c.moe_nvfp4_gate_up(W, cu(P.a_codes), cu(canonical_to_tiled(P.a_scales)), cu(P.offsets), cu(P.counts),
                              cu(np.array([P.g1])), cu(np.array([P.g2])), want_h=True, want_amax=True)
    h = host(res["h"])
    hc = host(res["h_codes"])
    hs = tiled_to_canonical(host(res["h_scales"]), P.cap, P.I)
    flips = total = 0
    amax = 0.0
    for e, r0, n in P.segments():
        if n == 0:
            continue
        _, _, ref_h = _oracle_gate_up(P, e, r0, n)
        err = rel_l2(h[r0:r0 + n], ref_h)
        assert err <= TOL, f"expert {e}: h rel L2 {err:.3g}"
        rc, rs = nvfp4.quantize(ref_h, P.g2)
        flips += int(np.count_nonzero(nvfp4.unpack_codes(hc[r0:r0 + n]) != nvfp4.unpack_codes(rc)))
        total += ref_h.size
        amax = max(amax, float(np.abs(ref_h).max()))
        # padding rows of the segment are zero codes and zero scales
        seg_end = int(P.offsets[e + 1])
        assert not hc[r0 + n:seg_end].any() and not hs[r0 + n:seg_end].any()
    assert flips <= 0.001 * total, f"{flips} of {total} requantised codes differ"
    assert abs(float(host(res["h_amax"])[0]) - amax) <= 1e-3 * amax


def _diagnose_down(P, y, e, r0, n, weighted):
    """Rel errors per 32-row quadrant and 128-column half, and under a few
    alternative readings of the operand layouts, to localise a mismatch."""
    dq = (P.down[0][e], P.down[1][e], P.g["down"][e])
    ref = moe.expert_down(P.h_codes[r0:r0 + n], P.h_scales[r0:r0 + n], P.g2, dq)
    y = y / np.maximum(P.row_w[r0:r0 + n, None], 1e-30) if weighted else y
    out = [f"expert {e} rows {n}: overall {rel_l2(y, ref):.3g}"]
    for q in range(4):
        for hcol in range(P.H // 128):
            rs = slice(32 * q, min(32 * q + 32, n))
            cs = slice(128 * hcol, 128 * hcol + 128)
            if rs.start < n:
                out.append(f"  rows {rs.start}-{rs.stop} cols {cs.start}-{cs.stop}: {rel_l2(y[rs, cs], ref[rs, cs]):.3g}")
    swap = lambda b: ((b & 0xF) << 4) | (b >> 4)  # noqa: E731
    alt = moe.expert_down(swap(P.h_codes[r0:r0 + n]), P.h_scales[r0:r0 + n], P.g2, (swap(dq[0]), dq[1], dq[2]))
    out.append(f"  with both nibble orders swapped: {rel_l2(y, alt):.3g}")
    return "\n".join(out)


@pytest.mark.parametrize("name,layout", _layout_params())
@pytest.mark.parametrize("weighted", [False, True])
def test_down_matches_oracle(name, layout, weighted):
    require_cuda()
    c = capi()
    P = Problem(**PROBLEMS[name])
    W = P.weights(c, layout)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    rw = P.row_w if weighted else np.ones_like(P.row_w)
    res = c.moe_nvfp4_down(W, cu(P.h_codes), cu(canonical_to_tiled(P.h_scales)), cu(P.offsets), cu(P.counts),
                           cu(np.array([P.g2])), cu(rw) if weighted else None, out_dtype=torch.float32)
    y = host(res["y"])
    for e, r0, n in P.segments():
        if n == 0:
            continue
        dq = (P.down[0][e], P.down[1][e], P.g["down"][e])
        ref = moe.expert_down(P.h_codes[r0:r0 + n], P.h_scales[r0:r0 + n], P.g2, dq) * rw[r0:r0 + n, None]
        err = rel_l2(y[r0:r0 + n], ref)
        if err > TOL:
            pytest.fail(_diagnose_down(P, y[r0:r0 + n], e, r0, n, weighted))
        # rows past the count are not written
        assert not y[r0 + n:int(P.offsets[e + 1])].any()


def test_down_bf16_output_rounds_fp32_result():
    require_cuda()
    c = capi()
    P = Problem(**PROBLEMS["ragged"])
    W = P.weights(c)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    args = (W, cu(P.h_codes), cu(canonical_to_tiled(P.h_scales)), cu(P.offsets), cu(P.counts), cu(np.array([P.g2])),
            cu(P.row_w))
    yf = host(c.moe_nvfp4_down(*args, out_dtype=torch.float32)["y"])
    yb = c.moe_nvfp4_down(*args, out_dtype=torch.bfloat16)["y"]
    # internal consistency of the two epilogue outputs (torch does the rounding)
    np.testing.assert_array_equal(host(yb), torch.from_numpy(yf).to(torch.bfloat16).float().numpy())


# More tiles than the GPU has SMs (148): 4 experts of 577-612 rows make 20
# m-tiles, so the gate/up GEMM has 20 x 16 = 320 tiles and the down GEMM
# 20 x 24 = 480.  Every persistent CTA then walks two to four tiles, which
# exercises the stage-phase carry-over between tiles, the reuse of the tensor
# memory accumulator and its hand-back.  Every real row is compared.
MANY_TILES = dict(E=4, H=6144, I=2048, counts=[600, 577, 612, 590])


def _row_rel(got, ref):
    d = np.linalg.norm(ref.astype(np.float64), axis=1)
    return np.linalg.norm(got.astype(np.float64) - ref, axis=1) / np.where(d > 0, d, 1.0)


@pytest.mark.parametrize("layout", ["canonical", "staged"])
def test_gate_up_every_row_over_many_tiles(layout):
    require_cuda()
    c = capi()
    P = Problem(**MANY_TILES, seed=3)
    assert (P.rows // 128) * (P.I // 128) > 2 * 148
    W = P.weights(c, layout)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    res = c.moe_nvfp4_gate_up(W, cu(P.a_codes), cu(canonical_to_tiled(P.a_scales)), cu(P.offsets), cu(P.counts),
                              cu(np.array([P.g1])), cu(np.array([P.g2])), want_h=True)
    h = host(res["h"])
    hc = host(res["h_codes"])
    hs = tiled_to_canonical(host(res["h_scales"]), P.cap, P.I)
    flips = total = 0
    for e, r0, n in P.segments():
        _, _, ref_h = _oracle_gate_up(P, e, r0, n)
        rel = _row_rel(h[r0:r0 + n], ref_h)
        assert rel.max() <= TOL, f"expert {e}: worst row {int(rel.argmax())} rel L2 {rel.max():.3g}"
        rc, rs = nvfp4.quantize(ref_h, P.g2)
        flips += int(np.count_nonzero(nvfp4.unpack_codes(hc[r0:r0 + n]) != nvfp4.unpack_codes(rc)))
        total += ref_h.size
        # scale bytes: differ only where the row's block amax differs from the oracle's by rounding
        assert np.count_nonzero(hs[r0:r0 + n] != rs) <= 0.001 * rs.size
        seg_end = int(P.offsets[e + 1])
        assert not hc[r0 + n:seg_end].any() and not hs[r0 + n:seg_end].any()
    assert flips <= 0.001 * total, f"{flips} of {total} requantised codes differ"


@pytest.mark.parametrize("layout", ["canonical", "staged"])
def test_down_every_row_over_many_tiles(layout):
    require_cuda()
    c = capi()
    P = Problem(**MANY_TILES, seed=4)
    assert (P.rows // 128) * (P.H // 256) > 3 * 148
    W = P.weights(c, layout)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    res = c.moe_nvfp4_down(W, cu(P.h_codes), cu(canonical_to_tiled(P.h_scales)), cu(P.offsets), cu(P.counts),
                           cu(np.array([P.g2])), cu(P.row_w), out_dtype=torch.float32)
    y = host(res["y"])
    for e, r0, n in P.segments():
        dq = (P.down[0][e], P.down[1][e], P.g["down"][e])
        ref = moe.expert_down(P.h_codes[r0:r0 + n], P.h_scales[r0:r0 + n], P.g2, dq) * P.row_w[r0:r0 + n, None]
        rel = _row_rel(y[r0:r0 + n], ref)
        assert rel.max() <= TOL, f"expert {e}: worst row {int(rel.argmax())} rel L2 {rel.max():.3g}"
        assert not y[r0 + n:int(P.offsets[e + 1])].any()
