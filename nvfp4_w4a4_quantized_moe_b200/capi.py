"""ctypes binding of libnvfp4moe.so (argument marshalling only).

Every function here has the name of the C entry point it calls (see
``include/nvfp4_moe.h``) and does nothing but check tensor placement, dtypes
and shapes, allocate outputs and workspace with torch, pass raw device
pointers and torch's current CUDA stream, and turn a non-OK status into an
exception.  All arithmetic of the layer runs in the library's CUDA kernels;
there is no CPU path.  Importing this module loads the library and fails
loudly when it has not been built.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4moe.so")

LAYOUT_CANONICAL = 0
LAYOUT_TILED = 1
LAYOUT_STAGED = 2          # weight codes in K-stage tiles, scales tiled
_LAYOUTS = {"canonical": LAYOUT_CANONICAL, "tiled": LAYOUT_TILED, "staged": LAYOUT_STAGED}

STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED_SHAPE", 3: "CUDA", 4: "TIMEOUT", 5: "WORKSPACE",
                6: "DEVICE"}


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m nvfp4_w4a4_quantized_moe_b200.build` "
                      "(the layer has no other implementation)")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


class MoeWeightsStruct(ctypes.Structure):
    _fields_ = [("E", _i), ("H", _i), ("I", _i), ("k", _i), ("routed_scaling_factor", _f),
                ("router_weight", _vp), ("bias", _vp),
                ("gate_codes", _vp), ("gate_scales", _vp), ("gate_gscale", _vp),
                ("up_codes", _vp), ("up_scales", _vp), ("up_gscale", _vp),
                ("down_codes", _vp), ("down_scales", _vp), ("down_gscale", _vp),
                ("shared_gate", _vp), ("shared_up", _vp), ("shared_down", _vp), ("I_shared", _i),
                ("codes_layout", _i)]


DEBUG_FIELDS = ("logits", "topk_idx", "topk_w", "expert_offsets", "perm", "inv_perm", "a_codes", "a_scales", "h",
                "h_amax", "h_codes", "h_scales", "y")
N_STAGE_EVENTS = 6


class MoeDebugStruct(ctypes.Structure):
    _fields_ = ([(n, _vp) for n in DEBUG_FIELDS] + [("stage_events", _vp * N_STAGE_EVENTS)] +
                [("saliency_sum", _vp), ("saliency_count", _vp), ("shared_event", _vp)])


def _declare(name, restype, *argtypes):
    fn = getattr(lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


_declare("nvfp4_last_error", ctypes.c_char_p)
_declare("nvfp4_abi_version", _i)
_declare("nvfp4_workspace_status", _i, _vp, _vp)
_declare("nvfp4_quantize_weights_workspace_size", _sz, _i)
_declare("nvfp4_quantize_weights", _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp)
_declare("nvfp4_quantize_weights_noalloc", _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp)
_declare("nvfp4_quantize_weights_noalloc_status", _i, _vp)
_declare("nvfp4_quantize_act", _i, _vp, _i, _i, _vp, _i, _vp, _vp, _vp)
_declare("moe_route_rows_capacity", _i, _i, _i, _i)
_declare("moe_route_workspace_size", _sz, _i, _i, _i)
_declare("moe_route", _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
         _vp)
_declare("moe_nvfp4_workspace_size", _sz, _i, _i, _i, _i, _i)
_declare("moe_nvfp4_workspace_size_shared", _sz, _i, _i, _i, _i, _i, _i)
_declare("moe_nvfp4_forward_launches", _i, _i, _i, _i, _i, _i, _i, _i)
_declare("moe_nvfp4_forward", _i, ctypes.POINTER(MoeWeightsStruct), _vp, _i, _vp, _vp, _vp, _vp,
         ctypes.POINTER(MoeDebugStruct), _vp, _sz, _vp)
_declare("moe_nvfp4_forward_scaled", _i, ctypes.POINTER(MoeWeightsStruct), _vp, _i, _i, _vp, _vp, _vp, _vp,
         ctypes.POINTER(MoeDebugStruct), _vp, _sz, _vp)
_declare("moe_nvfp4_workspace_size_host", _sz, _i, _i, _i, _i, _i, _i)
_declare("moe_nvfp4_forward_host", _i, ctypes.POINTER(MoeWeightsStruct), _vp, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp)
_declare("moe_nvfp4_host_join", _i, _vp, _vp)
_declare("moe_nvfp4_host_release", _i, _vp)
_declare("moe_nvfp4_gemm_workspace_size", _sz, _i)
_declare("moe_reap_keep", _i, _vp, _vp, _i, _i, _vp, _vp)
_declare("moe_nvfp4_gate_up", _i, ctypes.POINTER(MoeWeightsStruct), _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
         _vp, _vp, _vp, _sz, _vp)
_declare("moe_nvfp4_down", _i, ctypes.POINTER(MoeWeightsStruct), _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
         _vp, _sz, _vp)

_declare("nvfp4_block_stats_compute", _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp)
_declare("nvfp4_test_e2m1", _i, _vp, _i, _vp, _vp, _vp)
_declare("nvfp4_test_e2m1_sweep", _i, ctypes.c_uint32, ctypes.c_uint64, _vp, _vp, _vp)
_declare("nvfp4_test_e4m3", _i, _vp, _i, _vp, _vp, _vp)
_declare("nvfp4_test_sigmoid", _i, _vp, _i, _vp, _vp)
_declare("nvfp4_test_mma_peak", _i, _i, _i, _i, _i, _vp, _vp, _vp)
_declare("nvfp4_test_wait_timeout", _i, _vp, ctypes.c_uint64, _vp, _sz, _vp, _vp, _vp)
_declare("nvfp4_test_block_scale_div", _i, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp)
_declare("nvfp4_test_router_splits", _i, _i, _i, ctypes.POINTER(ctypes.c_int))

# Every symbol the public headers declare (checked by the CPU test suite).
EXPORTS = ("nvfp4_last_error", "nvfp4_abi_version", "nvfp4_workspace_status",
           "nvfp4_quantize_weights_workspace_size", "nvfp4_quantize_weights", "nvfp4_quantize_weights_noalloc",
           "nvfp4_quantize_weights_noalloc_status", "nvfp4_quantize_act",
           "moe_route_rows_capacity", "moe_route_workspace_size", "moe_route", "moe_nvfp4_workspace_size",
           "moe_nvfp4_forward", "moe_nvfp4_forward_scaled", "moe_nvfp4_workspace_size_shared",
           "moe_nvfp4_forward_launches", "moe_nvfp4_workspace_size_host", "moe_nvfp4_forward_host",
           "moe_nvfp4_host_join", "moe_nvfp4_host_release",
           "moe_nvfp4_gemm_workspace_size", "moe_nvfp4_gate_up",
           "moe_nvfp4_down", "moe_reap_keep",
           "nvfp4_block_stats_compute",
           "nvfp4_test_e2m1", "nvfp4_test_e2m1_sweep", "nvfp4_test_e4m3", "nvfp4_test_sigmoid",
           "nvfp4_test_mma_peak", "nvfp4_test_wait_timeout", "nvfp4_test_block_scale_div",
           "nvfp4_test_router_splits")


def _check(status: int):
    if status != 0:
        raise Nvfp4Error(status, lib.nvfp4_last_error().decode(errors="replace"))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _cuda(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def tiled_scale_bytes(rows: int, cols: int) -> int:
    return (rows + 127) // 128 * 128 * (cols // 16)


def abi_version() -> int:
    return lib.nvfp4_abi_version()


def nvfp4_workspace_status(ws: torch.Tensor):
    """Raises Nvfp4Error(TIMEOUT) if a device-side wait of the call that used
    ``ws`` gave up; synchronises the current stream."""
    _check(lib.nvfp4_workspace_status(_p(ws), _stream()))


def moe_route_rows_capacity(T: int, E: int, k: int) -> int:
    return lib.moe_route_rows_capacity(T, E, k)


# ---------------------------------------------------------------------------
# quantisers
# ---------------------------------------------------------------------------

def _weight_outputs(w: torch.Tensor, lay: int, out):
    """(codes, scales, gscale) for n_mats [rows, cols] matrices: allocated
    with torch, or the caller's ``out``, checked for device, dtype and size."""
    n, rows, cols = w.shape
    need_scales = tiled_scale_bytes(n * rows, cols) if lay != LAYOUT_CANONICAL else n * rows * (cols // 16)
    if out is None:
        codes = torch.empty((n, rows, cols // 2), dtype=torch.uint8, device=w.device)
        scales = (torch.empty(need_scales, dtype=torch.uint8, device=w.device) if lay != LAYOUT_CANONICAL
                  else torch.empty((n, rows, cols // 16), dtype=torch.uint8, device=w.device))
        return codes, scales, torch.empty(n, dtype=torch.float32, device=w.device)
    codes, scales, gscale = out
    _cuda(codes, torch.uint8, "codes")
    _cuda(scales, torch.uint8, "scales")
    _cuda(gscale, torch.float32, "gscale")
    for t, name, need in ((codes, "codes", n * rows * (cols // 2)), (scales, "scales", need_scales),
                          (gscale, "gscale", n)):
        if t.device != w.device:
            raise ValueError(f"{name} must be on {w.device}, got {t.device}")
        if t.numel() < need:
            raise ValueError(f"{name} holds {t.numel()} elements; this call writes {need}")
    return codes, scales, gscale


def nvfp4_quantize_weights(w: torch.Tensor, layout: str = "tiled", workspace: torch.Tensor | None = None,
                           out=None):
    """w [n_mats, rows, cols] bf16 -> (codes [n, rows, cols/2] u8, scales u8, gscale [n] f32).
    ``out`` = (codes, scales, gscale) to write into instead of new tensors."""
    _cuda(w, torch.bfloat16, "w")
    if w.dim() == 2:
        w = w.unsqueeze(0)
    n, rows, cols = w.shape
    lay = _LAYOUTS[layout]
    codes, scales, gscale = _weight_outputs(w, lay, out)
    need = lib.nvfp4_quantize_weights_workspace_size(n)
    ws = workspace if workspace is not None else _workspace(need, w.device)
    _check(lib.nvfp4_quantize_weights(_p(w), n, rows, cols, lay, _p(codes), _p(scales), _p(gscale), _p(ws),
                                      ws.numel(), _stream()))
    return codes, scales, gscale


def nvfp4_quantize_weights_noalloc(w: torch.Tensor, layout: str = "tiled", out=None):
    """The weight quantiser without a workspace (its scratch is built into the
    library).  ``out`` = (codes, scales, gscale) to write into; allocated here
    with torch when None (the library itself allocates nothing)."""
    _cuda(w, torch.bfloat16, "w")
    if w.dim() == 2:
        w = w.unsqueeze(0)
    n, rows, cols = w.shape
    lay = _LAYOUTS[layout]
    codes, scales, gscale = _weight_outputs(w, lay, out)
    _check(lib.nvfp4_quantize_weights_noalloc(_p(w), n, rows, cols, lay, _p(codes), _p(scales), _p(gscale),
                                              _stream()))
    return codes, scales, gscale


def nvfp4_quantize_weights_noalloc_status():
    """Raises Nvfp4Error(TIMEOUT) if a device-side wait of the last
    nvfp4_quantize_weights_noalloc call on this device gave up; synchronises
    the current stream."""
    _check(lib.nvfp4_quantize_weights_noalloc_status(_stream()))


def nvfp4_quantize_act(x: torch.Tensor, gscale: torch.Tensor, layout: str = "canonical"):
    """x [rows, cols] bf16 under gscale (one f32 on the device) -> (codes, scales)."""
    _cuda(x, torch.bfloat16, "x")
    _cuda(gscale, torch.float32, "gscale")
    rows, cols = x.shape
    lay = _LAYOUTS[layout]
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    if lay == LAYOUT_TILED:
        scales = torch.empty(tiled_scale_bytes(rows, cols), dtype=torch.uint8, device=x.device)
    else:
        scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=x.device)
    _check(lib.nvfp4_quantize_act(_p(x), rows, cols, _p(gscale), lay, _p(codes), _p(scales), _stream()))
    return codes, scales


#: Fields of nvfp4_block_stats, in declaration order (9 uint64 counts, 6 fp64 sums).
BLOCK_STATS_FIELDS = ("elements", "outliers", "blocks", "outlier_blocks", "zero_scale_blocks",
                      "subnormal_scale_blocks", "saturated_elements", "neighbours", "clean", "sum_sq", "sse",
                      "sum_sq_neighbours", "sse_neighbours", "sum_sq_clean", "sse_clean")


def nvfp4_block_stats_compute(w: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, gscale: torch.Tensor,
                              layout: str = "tiled", threshold: float = 0.1, stats: torch.Tensor | None = None):
    """Block-scale distortion statistics of n_mats NVFP4 tensors.  Returns the
    device buffer ([n_mats, 15] int64 words: 9 counts, then 6 fp64 sums bit-cast);
    ``block_stats_to_dicts`` turns it into one dict per matrix."""
    _cuda(w, torch.bfloat16, "w")
    if w.dim() == 2:
        w = w.unsqueeze(0)
    n, rows, cols = w.shape
    _cuda(gscale, torch.float32, "gscale")
    if stats is None:
        stats = torch.empty((n, len(BLOCK_STATS_FIELDS)), dtype=torch.int64, device=w.device)
    _check(lib.nvfp4_block_stats_compute(_p(w), _p(codes), _p(scales), _p(gscale), n, rows, cols,
                                         _LAYOUTS[layout], float(threshold), _p(stats), _stream()))
    return stats


def block_stats_to_dicts(stats: torch.Tensor) -> list[dict]:
    h = stats.cpu()
    counts = h[:, :9].tolist()
    sums = h[:, 9:].contiguous().view(torch.float64).tolist()
    return [dict(zip(BLOCK_STATS_FIELDS, c + s)) for c, s in zip(counts, sums)]


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------

def moe_route(x, router_weight, bias, k: int, rsf: float, logit_offset=None, logits_in=None):
    """Router + permutation.  Pass either (x, router_weight) or logits_in."""
    _cuda(bias, torch.float32, "bias")
    E = bias.numel()
    if logits_in is not None:
        _cuda(logits_in, torch.float32, "logits_in")
        T, H = logits_in.shape[0], 64
        dev = logits_in.device
    else:
        _cuda(x, torch.bfloat16, "x")
        _cuda(router_weight, torch.bfloat16, "router_weight")
        T, H = x.shape
        dev = x.device
        if logit_offset is not None:
            _cuda(logit_offset, torch.float32, "logit_offset")
    cap = moe_route_rows_capacity(T, E, k)
    out = {
        "logits": torch.empty((T, E), dtype=torch.float32, device=dev),
        "topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
        "topk_w": torch.empty((T, k), dtype=torch.float32, device=dev),
        "expert_offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "perm": torch.empty(cap, dtype=torch.int32, device=dev),
        "inv_perm": torch.empty((T, k), dtype=torch.int32, device=dev),
    }
    ws = _workspace(lib.moe_route_workspace_size(T, E, k), dev)
    _check(lib.moe_route(_p(x) if logits_in is None else None, _p(router_weight) if logits_in is None else None,
                         _p(logits_in), _p(bias), _p(logit_offset) if logits_in is None else None, T, H, E, k,
                         float(rsf), _p(out["logits"]), _p(out["topk_idx"]), _p(out["topk_w"]),
                         _p(out["expert_offsets"]), _p(out["perm"]), _p(out["inv_perm"]), _p(ws), ws.numel(),
                         _stream()))
    out["workspace"] = ws
    return out


# ---------------------------------------------------------------------------
# the layer
# ---------------------------------------------------------------------------

@dataclass
class MoeWeights:
    """Device tensors of one NVFP4 MoE layer (scales in the tiled layout; codes
    row-major or, with ``codes_layout`` = LAYOUT_STAGED, in K-stage tiles)."""
    E: int
    H: int
    I: int
    k: int
    rsf: float
    router_weight: torch.Tensor      # bf16 [E, H]
    bias: torch.Tensor               # f32 [E]
    gate_codes: torch.Tensor         # u8 [E, I, H/2]
    gate_scales: torch.Tensor
    gate_gscale: torch.Tensor        # f32 [E]
    up_codes: torch.Tensor
    up_scales: torch.Tensor
    up_gscale: torch.Tensor
    down_codes: torch.Tensor         # u8 [E, H, I/2]
    down_scales: torch.Tensor
    down_gscale: torch.Tensor
    # the shared expert, bf16 (None: none): gate, up [I_s, H], down [H, I_s]
    shared_gate: torch.Tensor | None = None
    shared_up: torch.Tensor | None = None
    shared_down: torch.Tensor | None = None
    codes_layout: int = LAYOUT_CANONICAL

    @property
    def I_shared(self) -> int:
        return 0 if self.shared_gate is None else int(self.shared_gate.shape[0])

    def with_shared(self, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor) -> "MoeWeights":
        """This layer plus a shared bf16 expert."""
        for n, t in (("shared gate", gate), ("shared up", up), ("shared down", down)):
            _cuda(t, torch.bfloat16, n)
        return dataclasses.replace(self, shared_gate=gate, shared_up=up, shared_down=down)

    def struct(self) -> MoeWeightsStruct:
        return MoeWeightsStruct(self.E, self.H, self.I, self.k, float(self.rsf), _p(self.router_weight),
                                _p(self.bias), _p(self.gate_codes), _p(self.gate_scales), _p(self.gate_gscale),
                                _p(self.up_codes), _p(self.up_scales), _p(self.up_gscale), _p(self.down_codes),
                                _p(self.down_scales), _p(self.down_gscale), _p(self.shared_gate),
                                _p(self.shared_up), _p(self.shared_down), self.I_shared, int(self.codes_layout))

    @classmethod
    def quantize(cls, gate, up, down, router_weight, bias, k: int, rsf: float,
                 codes_layout: str | None = None) -> "MoeWeights":
        """RTN-quantise bf16 expert weights (gate/up [E, I, H], down [E, H, I])
        with the library's weight quantiser, tiled scales.  The codes are
        staged when H and I are multiples of 256 (``codes_layout`` None), else
        row-major; "staged" or "canonical" forces one."""
        E, I, H = gate.shape
        if codes_layout is None:
            codes_layout = "staged" if H % 256 == 0 and I % 256 == 0 else "canonical"
        lay = "staged" if codes_layout == "staged" else "tiled"
        gc, gs, gg = nvfp4_quantize_weights(gate, lay)
        uc, us, ug = nvfp4_quantize_weights(up, lay)
        dc, ds, dg = nvfp4_quantize_weights(down, lay)
        return cls(E, H, I, k, rsf, _cuda(router_weight, torch.bfloat16, "router_weight"),
                   _cuda(bias, torch.float32, "bias"), gc, gs, gg, uc, us, ug, dc, ds, dg,
                   codes_layout=LAYOUT_STAGED if lay == "staged" else LAYOUT_CANONICAL)


def reap_keep(saliency_sum: torch.Tensor, saliency_count: torch.Tensor, keep: int) -> torch.Tensor:
    """Experts retained by REAP pruning (moe_reap_keep): the ``keep`` highest
    mean saliencies, ties to the lower index, in expert order.  Returns their
    indices as int64 on the host."""
    _cuda(saliency_sum, torch.float64, "saliency sum")
    _cuda(saliency_count, torch.int64, "saliency count")
    E = saliency_sum.numel()
    if saliency_count.numel() != E:
        raise ValueError("saliency sum and count must have one entry per expert")
    idx = torch.empty(max(int(keep), 1), dtype=torch.int32, device=saliency_sum.device)
    _check(lib.moe_reap_keep(_p(saliency_sum), _p(saliency_count), E, int(keep), _p(idx), _stream()))
    return idx[:keep].cpu().long()


def select_experts(W: "MoeWeights", keep: torch.Tensor) -> "MoeWeights":
    """The layer restricted to the experts ``keep`` (in that order), by byte
    slicing only (no arithmetic): gate.weight
    rows and e_score_correction_bias sliced as the pruned checkpoint does, and
    each retained expert's codes, tiled scales and global scales copied over
    (an expert's I or H rows are whole 128-row tiles, so its scales and its
    codes, row-major or staged, are contiguous ranges)."""
    idx = keep.to(W.router_weight.device)
    E2 = int(idx.numel())

    def rows(t, per):
        return t.reshape(W.E, per).index_select(0, idx).reshape(-1).contiguous()

    def codes(t):
        return t.reshape(W.E, -1).index_select(0, idx).reshape(E2, *t.shape[1:]).contiguous()

    return MoeWeights(E2, W.H, W.I, W.k, W.rsf, W.router_weight.index_select(0, idx).contiguous(),
                      W.bias.index_select(0, idx).contiguous(),
                      codes(W.gate_codes), rows(W.gate_scales, W.I * W.H // 16), W.gate_gscale.index_select(0, idx),
                      codes(W.up_codes), rows(W.up_scales, W.I * W.H // 16), W.up_gscale.index_select(0, idx),
                      codes(W.down_codes), rows(W.down_scales, W.H * W.I // 16), W.down_gscale.index_select(0, idx),
                      W.shared_gate, W.shared_up, W.shared_down, W.codes_layout)


def moe_nvfp4_forward_launches(T: int, E: int, H: int, I: int, k: int, I_shared: int = 0,
                               act_scale_mode: str = "tensor") -> int:
    """Kernels one forward call queues for this shape (host arithmetic only)."""
    n = lib.moe_nvfp4_forward_launches(T, E, H, I, k, I_shared, ACT_SCALE_MODES[act_scale_mode])
    if n < 0:
        raise ValueError(f"unsupported forward shape T={T} E={E} H={H} I={I} k={k} I_shared={I_shared}")
    return n


def moe_nvfp4_workspace_size(T: int, E: int, H: int, I: int, k: int, I_shared: int = 0) -> int:
    return lib.moe_nvfp4_workspace_size_shared(T, E, H, I, k, I_shared)


#: Activation global-scale modes of moe_nvfp4_forward_scaled (NVFP4_ACT_SCALE_*).
ACT_SCALE_MODES = {"tensor": 0, "expert": 1, "dynamic": 2, "dynamic_expert": 3}


def moe_nvfp4_forward(W: MoeWeights, x: torch.Tensor, act_gscale: torch.Tensor, h_gscale: torch.Tensor,
                      logit_offset: torch.Tensor | None = None, debug: bool = False,
                      out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      stage_events=None, act_scale_mode: str = "tensor", saliency=None, shared_event=None):
    """out [T, H] bf16; with debug=True also a dict of intermediate results.
    ``act_scale_mode`` is one of ACT_SCALE_MODES: in "tensor" act_gscale and
    h_gscale hold one fp32 each, in "expert" E each; in "dynamic" and
    "dynamic_expert" the library writes g1 into act_gscale ([1] or [E]).
    ``stage_events``: optional list of 6 torch.cuda.Event(enable_timing=True),
    each already recorded once (torch creates the CUDA event lazily), which
    the library records again between the stages of the layer.
    ``saliency``: optional (sum float64 [E], count int64 [E]) REAP saliency
    accumulators on the device that the call adds this batch to.
    ``shared_event``: optional torch.cuda.Event (recorded once already) that
    the library records after the shared expert's GEMMs."""
    mode = ACT_SCALE_MODES[act_scale_mode]
    if saliency is not None:
        _cuda(saliency[0], torch.float64, "saliency sum")
        _cuda(saliency[1], torch.int64, "saliency count")
    _cuda(x, torch.bfloat16, "x")
    _cuda(act_gscale, torch.float32, "act_gscale")
    _cuda(h_gscale, torch.float32, "h_gscale")
    n_scales = W.E if mode & 1 else 1
    if act_gscale.numel() != n_scales or h_gscale.numel() != n_scales:
        raise ValueError(f"act_scale_mode {act_scale_mode!r} needs {n_scales} value(s) in act_gscale and h_gscale")
    T, H = x.shape
    dev = x.device
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else _cuda(out, torch.bfloat16, "out")
    if workspace is None:
        workspace = _workspace(moe_nvfp4_workspace_size(T, W.E, W.H, W.I, W.k, W.I_shared), dev)
    dbg_tensors = None
    dbg_ptr = None
    if debug:
        cap = moe_route_rows_capacity(T, W.E, W.k)
        z = lambda *s, dt=torch.float32: torch.zeros(s, dtype=dt, device=dev)  # noqa: E731
        dbg_tensors = {
            "logits": z(T, W.E), "topk_idx": z(T, W.k, dt=torch.int32), "topk_w": z(T, W.k),
            "expert_offsets": z(W.E + 1, dt=torch.int32), "perm": z(cap, dt=torch.int32),
            "inv_perm": z(T, W.k, dt=torch.int32), "a_codes": z(cap, W.H // 2, dt=torch.uint8),
            "a_scales": z(tiled_scale_bytes(cap, W.H), dt=torch.uint8), "h": z(cap, W.I), "h_amax": z(n_scales),
            "h_codes": z(cap, W.I // 2, dt=torch.uint8), "h_scales": z(tiled_scale_bytes(cap, W.I), dt=torch.uint8),
            "y": z(cap, W.H),
        }
    if debug or stage_events is not None or saliency is not None or shared_event is not None:
        dbg = MoeDebugStruct()
        if saliency is not None:
            dbg.saliency_sum = saliency[0].data_ptr()
            dbg.saliency_count = saliency[1].data_ptr()
        if debug:
            for n in DEBUG_FIELDS:
                setattr(dbg, n, dbg_tensors[n].data_ptr())
        if stage_events is not None:
            for i, ev in enumerate(stage_events):
                if not ev.cuda_event:
                    raise ValueError("stage_events must have been recorded once (so that the CUDA event exists)")
                dbg.stage_events[i] = ev.cuda_event
        if shared_event is not None:
            if not shared_event.cuda_event:
                raise ValueError("shared_event must have been recorded once (so that the CUDA event exists)")
            dbg.shared_event = shared_event.cuda_event
        dbg_ptr = ctypes.pointer(dbg)
    ws_struct = W.struct()
    if mode == 0:
        _check(lib.moe_nvfp4_forward(ctypes.byref(ws_struct), _p(x), T, _p(act_gscale), _p(h_gscale),
                                     _p(logit_offset), _p(out), dbg_ptr, _p(workspace), workspace.numel(), _stream()))
    else:
        _check(lib.moe_nvfp4_forward_scaled(ctypes.byref(ws_struct), _p(x), T, mode, _p(act_gscale), _p(h_gscale),
                                            _p(logit_offset), _p(out), dbg_ptr, _p(workspace), workspace.numel(),
                                            _stream()))
    if debug:
        dbg_tensors["workspace"] = workspace
        return out, dbg_tensors
    return out


def moe_nvfp4_workspace_size_host(T: int, E: int, H: int, I: int, k: int, I_shared: int = 0) -> int:
    return lib.moe_nvfp4_workspace_size_host(T, E, H, I, k, I_shared)


def _host(t, dtype, name):
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor")
    return t


def moe_nvfp4_forward_host(W: MoeWeights, x_host: torch.Tensor, act_gscale: torch.Tensor, h_gscale: torch.Tensor,
                           out_host: torch.Tensor, workspace: torch.Tensor, logit_offset: torch.Tensor | None = None):
    """The forward on host buffers (per-tensor scales): enqueues x in, the
    layer on the current stream and out back, and returns without waiting.
    x_host and out_host are [T, H] bf16 CPU tensors (pinned for the copies to
    overlap); the workspace is a CUDA uint8 tensor of at least
    moe_nvfp4_workspace_size_host bytes.  out_host is complete after
    moe_nvfp4_host_join(workspace) and a synchronize of the current stream."""
    _host(x_host, torch.bfloat16, "x_host")
    _host(out_host, torch.bfloat16, "out_host")
    _cuda(act_gscale, torch.float32, "act_gscale")
    _cuda(h_gscale, torch.float32, "h_gscale")
    _cuda(workspace, torch.uint8, "workspace")
    T, H = x_host.shape
    if tuple(out_host.shape) != (T, H):
        raise ValueError("out_host must have the shape of x_host")
    ws_struct = W.struct()
    _check(lib.moe_nvfp4_forward_host(ctypes.byref(ws_struct), ctypes.c_void_p(x_host.data_ptr()), T,
                                      _p(act_gscale), _p(h_gscale), _p(logit_offset),
                                      ctypes.c_void_p(out_host.data_ptr()), _p(workspace), workspace.numel(),
                                      _stream()))
    return out_host


def moe_nvfp4_host_join(workspace: torch.Tensor):
    """Makes the current stream wait for the last host-buffer call on this
    workspace to have copied its out back."""
    _check(lib.moe_nvfp4_host_join(_p(workspace), _stream()))


def moe_nvfp4_host_release(workspace: torch.Tensor):
    """Waits for the workspace's last host-buffer call and frees the
    library's events for it."""
    _check(lib.moe_nvfp4_host_release(_p(workspace)))


def moe_nvfp4_gate_up(W: MoeWeights, a_codes, a_scales, expert_offsets, expert_counts, act_gscale, h_gscale,
                      want_h: bool = True, want_amax: bool = False):
    """Grouped gate/up GEMM on caller-supplied quantised rows."""
    rows = a_codes.shape[0]
    dev = a_codes.device
    h_codes = torch.empty((rows, W.I // 2), dtype=torch.uint8, device=dev)
    h_scales = torch.empty(tiled_scale_bytes(rows, W.I), dtype=torch.uint8, device=dev)
    h = torch.empty((rows, W.I), dtype=torch.float32, device=dev) if want_h else None
    amax = torch.zeros(1, dtype=torch.float32, device=dev) if want_amax else None
    ws = _workspace(lib.moe_nvfp4_gemm_workspace_size(rows), dev)
    st = W.struct()
    _check(lib.moe_nvfp4_gate_up(ctypes.byref(st), _p(a_codes), _p(a_scales), _p(expert_offsets), _p(expert_counts),
                                 rows, _p(act_gscale), _p(h_gscale), _p(h_codes), _p(h_scales), _p(h), _p(amax),
                                 _p(ws), ws.numel(), _stream()))
    return {"h_codes": h_codes, "h_scales": h_scales, "h": h, "h_amax": amax, "workspace": ws}


def moe_nvfp4_down(W: MoeWeights, h_codes, h_scales, expert_offsets, expert_counts, h_gscale, row_weight=None,
                   out_dtype=torch.float32):
    """Grouped down GEMM on caller-supplied quantised rows; y [rows, H]."""
    rows = h_codes.shape[0]
    dev = h_codes.device
    y = torch.zeros((rows, W.H), dtype=out_dtype, device=dev)
    ws = _workspace(lib.moe_nvfp4_gemm_workspace_size(rows), dev)
    st = W.struct()
    yb = y if out_dtype == torch.bfloat16 else None
    yf = y if out_dtype == torch.float32 else None
    _check(lib.moe_nvfp4_down(ctypes.byref(st), _p(h_codes), _p(h_scales), _p(expert_offsets), _p(expert_counts),
                              rows, _p(h_gscale), _p(row_weight), _p(yb), _p(yf), _p(ws), ws.numel(), _stream()))
    return {"y": y, "workspace": ws}


# ---------------------------------------------------------------------------
# test hooks (include/nvfp4_moe_testing.h)
# ---------------------------------------------------------------------------

def nvfp4_test_e2m1(y: torch.Tensor):
    """(hardware codes, comparison codes) of fp32 values, one code per byte."""
    _cuda(y, torch.float32, "y")
    hw = torch.empty(y.numel(), dtype=torch.uint8, device=y.device)
    sw = torch.empty_like(hw)
    _check(lib.nvfp4_test_e2m1(_p(y), y.numel(), _p(hw), _p(sw), _stream()))
    return hw, sw


def nvfp4_test_e2m1_sweep(first: int, count: int, device="cuda"):
    """(number of disagreeing non-NaN fp32 patterns in [first, first+count), one example or None)."""
    mism = torch.zeros(1, dtype=torch.int64, device=device)
    ex = torch.full((1,), 0xFFFFFFFF, dtype=torch.int64, device=device)
    ex32 = torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib.nvfp4_test_e2m1_sweep(first, count, _p(mism), _p(ex32), _stream()))
    n = int(mism.item())
    return n, (int(ex32.item()) & 0xFFFFFFFF) if n else None


def nvfp4_test_e4m3(s: torch.Tensor):
    _cuda(s, torch.float32, "s")
    codes = torch.empty(s.numel(), dtype=torch.uint8, device=s.device)
    val = torch.empty(s.numel(), dtype=torch.float32, device=s.device)
    _check(lib.nvfp4_test_e4m3(_p(s), s.numel(), _p(codes), _p(val), _stream()))
    return codes, val


def nvfp4_test_router_splits(T: int, H: int):
    """(splits, K stages per split) of the router GEMM for T tokens, hidden H."""
    per = ctypes.c_int(0)
    n = lib.nvfp4_test_router_splits(T, H, ctypes.byref(per))
    if n < 0:
        raise ValueError(f"no router split for T={T} H={H}")
    return n, per.value


def nvfp4_test_sigmoid(l: torch.Tensor):
    _cuda(l, torch.float32, "l")
    out = torch.empty_like(l)
    _check(lib.nvfp4_test_sigmoid(_p(l), l.numel(), _p(out), _stream()))
    return out


def nvfp4_test_mma_peak(iters: int, n: int = 256, with_cp: int = 0, ctas: int | None = None):
    """(FLOP per SM clock per CTA, cycles per CTA) of back-to-back FP4 MMAs."""
    ctas = ctas or torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    cycles = torch.zeros(ctas, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(lib.nvfp4_test_mma_peak(iters, n, int(with_cp), ctas, _p(cycles), _p(status), _stream()))
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise Nvfp4Error(4, "mma peak kernel: the completion wait gave up")
    cyc = cycles.cpu().double()
    flops = iters * 4 * 2.0 * 128 * n * 64
    return flops / cyc, cyc


def nvfp4_test_wait_timeout(src: torch.Tensor, limit_ns: int, workspace: torch.Tensor):
    """Queues the kernel whose bounded wait runs out after limit_ns; returns
    (elapsed_ns int64 [2], copied int32 [1]) device tensors.  The status word
    at the start of ``workspace`` is set when the wait gives up."""
    _cuda(src, torch.uint8, "src")
    if src.numel() < 4096:
        raise ValueError("src must hold at least 4096 bytes")
    elapsed = torch.zeros(2, dtype=torch.int64, device=src.device)
    copied = torch.zeros(1, dtype=torch.int32, device=src.device)
    _check(lib.nvfp4_test_wait_timeout(_p(src), int(limit_ns), _p(workspace), workspace.numel(), _p(elapsed),
                                       _p(copied), _stream()))
    return elapsed, copied


def nvfp4_test_block_scale_div(amax: torch.Tensor, g: torch.Tensor):
    """(q_lib, q_ieee, code_lib, code_ieee) for fp32 amax and g of equal size."""
    _cuda(amax, torch.float32, "amax")
    _cuda(g, torch.float32, "g")
    if amax.numel() != g.numel():
        raise ValueError("amax and g must have the same size")
    n = amax.numel()
    ql, qi = torch.empty_like(amax), torch.empty_like(amax)
    cl = torch.empty(n, dtype=torch.uint8, device=amax.device)
    ci = torch.empty_like(cl)
    _check(lib.nvfp4_test_block_scale_div(_p(amax), _p(g), n, _p(ql), _p(qi), _p(cl), _p(ci), _stream()))
    return ql, qi, cl, ci
