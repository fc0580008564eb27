#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 routed-expert MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
    python bench.py --impl reference ...      # the CPU oracle, timed as it stands

One step = one pass of the layer's hot path over one batch of the workload:
router GEMM, top-k, permutation, FP4 quantisation of x, grouped FP4 GEMM
gate/up with SiLU*up and requantisation, grouped FP4 GEMM down, weighted
combine (one moe_nvfp4_forward call).  The offline RTN weight quantiser runs
once per checkpoint, not per batch; it is timed in the same run over the full
80-expert layer and reported under "quantiser".

Prints one JSON line (rank 0).  Under torchrun every rank runs its own batch
(weak scaling, no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_w4a4_quantized_moe_b200 import workloads  # noqa: E402

METRIC = "MoE-layer tokens/s and TFLOPS (% NVFP4 peak); quantiser GB/s (% HBM) at 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0            # nominal dense ratio (9 vs 2.25 PFLOP/s)


def kernels_per_step(c, cfg) -> int:
    """Kernels one forward launches, as the library counts them: router GEMM,
    routing (one single-block kernel up to 256 tokens, else top-k and three
    permutation kernels), quantise-scatter (folded into the routing kernel
    for small layers), the two GEMMs and the combine."""
    return c.moe_nvfp4_forward_launches(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k)
NVFP4_BYTES_PER_ELEM = 0.5 + 1.0 / 16


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "prefill", "outlier", "tiny", "prefill16"], default="decode")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mma-peak", action="store_true",
                    help="measure the FP4 tensor-core rate with no memory traffic and exit")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS if k in p}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

class Dist:
    """Rank plumbing: one process per GPU under torchrun (NCCL), or CPU ranks
    over gloo for the multi-process tests.  Only a barrier and a max of the
    ranks' times cross ranks; the layer itself has no collective."""

    def __init__(self, backend: str | None = None, timeout_s: float = 300.0):
        """timeout_s bounds every collective: a rank whose peer died or stopped
        answering gets an error instead of waiting for good."""
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cpu"
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if backend == "nccl":
            torch.cuda.set_device(self.local if self.world > 1 else 0)
            self.device = "cuda"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": torch.device("cuda", self.local)} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.barrier()
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(device_index), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 7:
                self.samples.append((time.time(), parts))

    def stop(self, t0, t1):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        sel = [p for t, p in self.samples if t0 - 0.3 <= t <= t1 + 0.3] or [p for _, p in self.samples]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        mhz = [float(p[0]) for p in sel if p[0].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for p in sel for n, v in zip(names, p[3:7]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": float(sel[0][1]) if sel[0][1].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(sel)}


# ---------------------------------------------------------------------------
# traffic of the dominant kernel, from the committed ncu summary
# ---------------------------------------------------------------------------

GEMM_SOURCES = ("gemm.cu", "gemm.cuh", "common.cuh")


def gemm_source_sha() -> str:
    """Hash of the sources the GEMM kernel is compiled from."""
    import hashlib
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        h.update(open(os.path.join(ROOT, "nvfp4_w4a4_quantized_moe_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """dram bytes per launch recorded by ncu for this kernel and workload, or
    None when no record exists or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = gemm_source_sha()
    for line in open(path):
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("kernel") == kernel and f.get("workload") == workload and f.get("source_sha") == sha:
            return float(f["dram_bytes_per_launch"])
    return None


# ---------------------------------------------------------------------------
# oracle on the host cores (the CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

def _oracle_quantize_expert(args):
    from oracle import nvfp4
    return tuple(nvfp4.quantize_weight(w) for w in args)


class OracleSample:
    """The oracle's layer on a bounded sample of the batch: its first token.

    One step is one (token, expert) pair of that token, cycling through its k
    experts: the token's routing and x quantisation, then that expert's
    gate/up, SiLU(gate)*up, requantisation, down and weighted contribution, in
    the order the oracle's layer takes them.  k steps make one token, so the
    rate in tokens/s is pairs/s / k.  The token's experts are quantised by the
    oracle beforehand (untimed, in a spawn pool)."""

    def __init__(self, cfg, seed, x, wg, bias, off):
        from oracle import moe, nvfp4
        self.cfg = cfg
        self.x = x[:1].float().cpu().numpy()
        self.wg = wg.float().cpu().numpy()
        self.bias = bias.cpu().numpy()
        self.off = None if off is None else off.cpu().numpy()
        L = moe.router_logits(self.x, self.wg, self.off)
        idx, _ = moe.route(L, self.bias, cfg.k, cfg.rsf)
        experts = sorted(set(int(e) for e in idx[0]))
        jobs = []
        for e in experts:
            g, u, d = workloads.expert_weights(cfg, e, seed)
            jobs.append(tuple(t.float().cpu().numpy() for t in (g, u, d)))
        import multiprocessing as mp
        with mp.get_context("spawn").Pool(min(len(jobs), os.cpu_count() or 1)) as pool:
            q = pool.map(_oracle_quantize_expert, jobs)
        self.q = dict(zip(experts, q))
        self.g1 = np.float32(np.float32(np.abs(self.x).max()) / np.float32(2688))
        cal = moe.moe_layer(self.x, self.wg, self.bias, cfg.k, cfg.rsf, lambda e: self.q[e], self.g1,
                            np.float32(1.0), logit_offset=self.off)
        self.g2 = np.float32(np.float32(max(np.abs(h).max() for h in cal["h"].values())) / np.float32(2688))
        self.slot = 0
        self.out = np.zeros(self.x.shape, np.float64)
        self._nvfp4 = nvfp4

    def step(self):
        """One (token, expert) pair; returns the token's partial output."""
        from oracle import moe
        nvfp4 = self._nvfp4
        j = self.slot
        self.slot = (j + 1) % self.cfg.k
        logits = moe.router_logits(self.x, self.wg, self.off)
        idx, w = moe.route(logits, self.bias, self.cfg.k, self.cfg.rsf)
        a_codes, a_scales = nvfp4.quantize(self.x, self.g1)
        gate, up, down = self.q[int(idx[0, j])]
        _, _, h = moe.expert_gate_up(a_codes, a_scales, self.g1, gate, up)
        hc, hs = nvfp4.quantize(h, self.g2)
        y = moe.expert_down(hc, hs, self.g2, down)
        if j == 0:
            self.out[:] = 0.0
        self.out[0] += float(w[0, j]) * y[0]
        return self.out

    def tokens_per_step(self):
        return 1.0 / self.cfg.k

    @staticmethod
    def threads():
        try:
            from threadpoolctl import threadpool_info
            return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        except Exception:
            return os.cpu_count() or 1


def sample_desc(cfg):
    return (f"token 0 of the {cfg.name} batch, one (token, expert) pair per step cycling through its {cfg.k} "
            f"experts (routing, x quantisation, the expert's gate/up, SiLU*up, requantisation and down on "
            f"dequantised NVFP4 operands in fp64, weighted add); tokens/s = pairs/s / {cfg.k}; the token's "
            f"experts quantised by the oracle beforehand, untimed")


def run_reference(args, cfg):
    if int(os.environ.get("RANK", "0")) != 0:      # rank 0 alone times the oracle
        return 0
    x = workloads.hidden_states(cfg, args.seed)
    wg, bias, off = workloads.router_params(cfg, args.seed)
    smp = OracleSample(cfg, args.seed, x, wg, bias, off)
    for _ in range(args.warmup):
        smp.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        smp.step()
    dt = (time.perf_counter() - t0) / args.steps
    v = smp.tokens_per_step() / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "tokens_per_step": 1.0 / cfg.k, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E,
                       "k": cfg.k},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": OracleSample.threads(), "kind": "oracle",
                             "sample": sample_desc(cfg)},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, cfg):
    from nvfp4_w4a4_quantized_moe_b200 import capi as c
    dist = Dist()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()

    # inputs (identical on every rank: weak scaling replicates the batch)
    x = workloads.hidden_states(cfg, args.seed, device=dev)
    wg, bias, off = workloads.router_params(cfg, args.seed, device=dev)
    gate, up, down = workloads.stacked_expert_weights(cfg, args.seed, device=dev)
    W = c.MoeWeights.quantize(gate, up, down, wg, bias, cfg.k, cfg.rsf)
    g1 = (x.float().abs().amax() / 2688.0).reshape(1).float()
    # calibration pass: amax of h over the batch, from the gate/up epilogue
    ones = torch.ones(1, device=dev)
    _, dbg = c.moe_nvfp4_forward(W, x, g1, ones, logit_offset=off, debug=True)
    g2 = (dbg["h_amax"] / 2688.0).reshape(1).float()
    topk = dbg["topk_idx"].cpu().numpy()
    del dbg
    P = cfg.T * cfg.k
    hit = len(np.unique(topk))

    ws = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8, device=dev)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)

    def step(evs=None):
        c.moe_nvfp4_forward(W, x, g1, g2, logit_offset=off, out=out, workspace=ws, stage_events=evs)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    c.nvfp4_workspace_status(ws)

    # keep the GPU busy briefly so the clock sampler sees steady state
    sampler = ClockSampler(dev.index) if dist.rank == 0 else None
    t_warm = time.time()
    while time.time() - t_warm < 0.5:
        step()
        torch.cuda.synchronize()

    # the headline: K steps back to back, nothing between the layer's kernels
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    e0.record(stream)
    for i in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    dist.barrier()
    clocks = sampler.stop(t0, t1) if sampler else None
    c.nvfp4_workspace_status(ws)
    ms_total = dist.max(e0.elapsed_time(e1))
    ms_step = ms_total / args.steps

    # the same K steps again with CUDA events recorded by the library between
    # its stages: per-stage device times for the breakdown and the roofline.
    # An event between two kernels stops the second from starting early, so
    # these stages add up to a little more than the headline step.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(c.N_STAGE_EVENTS)] for _ in range(args.steps)]
    for row in evs:                 # torch creates the CUDA events lazily, on first record
        for ev in row:
            ev.record(stream)
    torch.cuda.synchronize()
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize()
    c.nvfp4_workspace_status(ws)
    stage_names = ("route", "quantize_x", "gemm_gate_up", "gemm_down", "combine")
    stage_ms = {n: dist.max(float(np.mean([evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)])))
                for j, n in enumerate(stage_names)}

    # the activation global-scale modes beyond the calibrated per-tensor one
    # (same workload, K steps each, nothing between the kernels)
    mode_ms = {}
    for mode in ("expert", "dynamic", "dynamic_expert"):
        n = cfg.E if mode in ("expert", "dynamic_expert") else 1
        a = g1.repeat(n).contiguous() if mode == "expert" else torch.zeros(n, device=dev)
        h = g2.repeat(n).contiguous()
        run = lambda: c.moe_nvfp4_forward(W, x, a, h, logit_offset=off, out=out, workspace=ws,  # noqa: E731
                                          act_scale_mode=mode)
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record(stream)
        for _ in range(args.steps):
            run()
        m1.record(stream)
        torch.cuda.synchronize()
        mode_ms[mode] = dist.max(m0.elapsed_time(m1)) / args.steps
    c.nvfp4_workspace_status(ws)
    # the same forward accumulating REAP saliency (f3)
    sal = (torch.zeros(cfg.E, dtype=torch.float64, device=dev), torch.zeros(cfg.E, dtype=torch.int64, device=dev))
    for _ in range(3):
        c.moe_nvfp4_forward(W, x, g1, g2, logit_offset=off, out=out, workspace=ws, saliency=sal)
    torch.cuda.synchronize()
    m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    m0.record(stream)
    for _ in range(args.steps):
        c.moe_nvfp4_forward(W, x, g1, g2, logit_offset=off, out=out, workspace=ws, saliency=sal)
    m1.record(stream)
    torch.cuda.synchronize()
    c.nvfp4_workspace_status(ws)
    sal_ms = dist.max(m0.elapsed_time(m1)) / args.steps

    # the layer with its shared BF16 expert (f1): one SiLU-gated MLP of the
    # routed experts' shape (I_shared = I), bf16 N(0, 0.02) weights
    sh = tuple(t.contiguous() for t in workloads.expert_weights(cfg, cfg.E + 7, args.seed, device=dev))
    Ws = W.with_shared(*sh)
    ws_sh = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k, cfg.I), dtype=torch.uint8,
                        device=dev)
    for _ in range(3):
        c.moe_nvfp4_forward(Ws, x, g1, g2, logit_offset=off, out=out, workspace=ws_sh)
    torch.cuda.synchronize()
    m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    m0.record(stream)
    for _ in range(args.steps):
        c.moe_nvfp4_forward(Ws, x, g1, g2, logit_offset=off, out=out, workspace=ws_sh)
    m1.record(stream)
    torch.cuda.synchronize()
    c.nvfp4_workspace_status(ws_sh)
    sh_ms = dist.max(m0.elapsed_time(m1)) / args.steps
    sh_flops = 6.0 * cfg.T * cfg.H * cfg.I
    sh_added = max(sh_ms - ms_step, 1e-6)
    shared_report = {"I_shared": cfg.I, "ms_per_step": sh_ms, "added_ms": sh_added, "flops": sh_flops,
                     "tflops_on_added_time": sh_flops / (sh_added * 1e-3) / 1e12,
                     "frac_of_bf16_peak": sh_flops / (sh_added * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"]}
    del Ws, sh, ws_sh

    # end to end: pinned host x in, host out back, through the same call
    x_h = x.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    x_d = torch.empty_like(x)
    for _ in range(3):
        x_d.copy_(x_h, non_blocking=True)
        c.moe_nvfp4_forward(W, x_d, g1, g2, logit_offset=off, out=out, workspace=ws)
        out_h.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        x_d.copy_(x_h, non_blocking=True)
        c.moe_nvfp4_forward(W, x_d, g1, g2, logit_offset=off, out=out, workspace=ws)
        out_h.copy_(out, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    e2e_ms = dist.max(f0.elapsed_time(f1)) / args.steps

    # offline weight quantiser over the full layer (the quantiser workload)
    qws = torch.empty(c.lib.nvfp4_quantize_weights_workspace_size(cfg.E), dtype=torch.uint8, device=dev)
    qlayout = "staged" if W.codes_layout == c.LAYOUT_STAGED else "tiled"     # what the layer's weights use
    qbytes = 0
    for w in (gate, up, down):
        n = w.numel()
        qbytes += 2 * n + n // 2 + n // 16 + 4 * w.shape[0]
    for _ in range(3):
        for w in (gate, up, down):
            c.nvfp4_quantize_weights(w, qlayout, workspace=qws)
    torch.cuda.synchronize()
    dist.barrier()
    q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    qsteps = max(3, min(args.steps, 20))
    q0.record(stream)
    for _ in range(qsteps):
        for w in (gate, up, down):
            c.nvfp4_quantize_weights(w, qlayout, workspace=qws)
    q1.record(stream)
    torch.cuda.synchronize()
    q_ms = dist.max(q0.elapsed_time(q1)) / qsteps
    q_gbs = qbytes / (q_ms * 1e-3) / 1e9

    # block-scale distortion statistics of the layer's quantised experts
    diag = block_stats_report(c, cfg, (gate, up, down), W, stream, dist, peaks)
    c.nvfp4_workspace_status(qws)

    # roofline of the dominant kernel
    fp4_peak = peaks["bf16_tflops_sustained"] * FP4_OVER_BF16
    gu_flops = 2.0 * P * cfg.H * 2 * cfg.I
    dn_flops = 2.0 * P * cfg.I * cfg.H
    gu_bytes = (hit * 2 * cfg.I * cfg.H + P * cfg.H + P * cfg.I) * NVFP4_BYTES_PER_ELEM
    dn_bytes = (hit * cfg.H * cfg.I + P * cfg.I) * NVFP4_BYTES_PER_ELEM + P * cfg.H * 2
    dom = "gemm_gate_up" if stage_ms["gemm_gate_up"] >= stage_ms["gemm_down"] else "gemm_down"
    flops, nbytes = (gu_flops, gu_bytes) if dom == "gemm_gate_up" else (dn_flops, dn_bytes)
    t_dom = stage_ms[dom] * 1e-3
    compute_bound = flops / (fp4_peak * 1e12) > nbytes / (peaks["hbm_gbs"] * 1e9)
    kname = "grouped_fp4_gemm_kernel<0>" if dom == "gemm_gate_up" else "grouped_fp4_gemm_kernel<1>"
    traffic = recorded_traffic(kname, cfg.name)
    if compute_bound:
        roof = {"bound": "tensor", "achieved": flops / t_dom / 1e12, "peak": fp4_peak, "unit": "TFLOP/s",
                "peak_source": f"{peak_src} bf16 sustained x {FP4_OVER_BF16:g} (nominal FP4/BF16 ratio)"}
    else:
        roof = {"bound": "hbm", "achieved": nbytes / t_dom / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_source": f"{peak_src} copy bandwidth"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof["kernel"] = kname
    roof["algorithmic"] = {"bytes": nbytes, "flops": flops, "experts_hit": hit, "pairs": P}
    gemm_ms = stage_ms["gemm_gate_up"] + stage_ms["gemm_down"]

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        smp = OracleSample(cfg, args.seed, x, wg, bias, off)
        smp.step()
        t = time.perf_counter()
        n = 0
        while n < cfg.k or time.perf_counter() - t < 10.0:
            smp.step()
            n += 1
        dt = (time.perf_counter() - t) / n
        cpu = {"value": smp.tokens_per_step() / dt, "unit": "tokens/s", "cores": OracleSample.threads(), "kind": "oracle",
               "sample": sample_desc(cfg) + f"; {n} pairs timed"}

    tokens = cfg.T * dist.world
    line = {
        "metric": METRIC, "value": weak_scaling_value(cfg.T, dist.world, ms_step), "unit": "tokens/s",
        "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": cfg.name, "tokens_per_gpu": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
                   "rsf": cfg.rsf, "x_outliers": cfg.x_outlier_p, "logit_offset_std": cfg.logit_offset_std,
                   "weight_outliers": cfg.w_outlier_p, "parallelism": f"replicas{dist.world}",
                   "l2": "inputs larger than L2 (expert weights of the layer: "
                         f"{(W.gate_codes.numel() * 3 + W.gate_scales.numel() * 3) / 1e9:.2f} GB)"},
        "gemm": {"ms": gemm_ms, "tflops": (gu_flops + dn_flops) / (gemm_ms * 1e-3) / 1e12,
                 "frac_of_fp4_peak": (gu_flops + dn_flops) / (gemm_ms * 1e-3) / 1e12 / fp4_peak},
        "stages_ms": stage_ms,
        "act_scale_modes_ms_per_step": dict({"tensor": ms_step}, **mode_ms),
        "reap_saliency_ms_per_step": sal_ms,
        "shared_expert": shared_report,
        "roofline": roof,
        "diagnostics": diag,
        "quantiser": {"workload": f"quantiser: {cfg.E} x (gate, up {cfg.I}x{cfg.H}; down {cfg.H}x{cfg.I}) bf16",
                      "ms": q_ms, "gbs": q_gbs, "bytes": qbytes, "bound": "hbm", "peak": peaks["hbm_gbs"],
                      "frac": q_gbs / peaks["hbm_gbs"]},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": out.numel() * 2},
        "gpu_launches": kernels_per_step(c, cfg) * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def block_stats_report(c, cfg, bf16_weights, W, stream, dist, peaks):
    """Block-scale distortion statistics of the quantised experts (gate, up and
    down of every expert): outlier share (|w| > 0.1), relative RMS error over
    all weights, over the neighbours of outliers and over clean blocks, and
    the share of subnormal-scale blocks and clamped elements; plus the time
    and bandwidth of the statistics kernel (2.5625 bytes read per element)."""
    enc = ((W.gate_codes, W.gate_scales, W.gate_gscale), (W.up_codes, W.up_scales, W.up_gscale),
           (W.down_codes, W.down_scales, W.down_gscale))
    layout = "staged" if W.codes_layout == c.LAYOUT_STAGED else "tiled"
    bufs = [torch.empty((w.shape[0], len(c.BLOCK_STATS_FIELDS)), dtype=torch.int64, device=w.device)
            for w in bf16_weights]

    def run():
        for w, (cd, sc, g), b in zip(bf16_weights, enc, bufs):
            c.nvfp4_block_stats_compute(w, cd, sc, g, layout, 0.1, stats=b)

    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(5):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = dist.max(e0.elapsed_time(e1)) / 5
    tot = dict.fromkeys(c.BLOCK_STATS_FIELDS, 0)
    for b in bufs:
        for d in c.block_stats_to_dicts(b):
            for k, v in d.items():
                tot[k] += v
    rel = lambda sse, sq: (sse / sq) ** 0.5 if sq > 0 else 0.0   # noqa: E731
    nbytes = tot["elements"] * 2.5625
    return {
        "tensors": f"{cfg.E} x (gate, up, down)", "outlier_threshold": 0.1,
        "outlier_share": tot["outliers"] / tot["elements"],
        "outlier_block_share": tot["outlier_blocks"] / tot["blocks"],
        "rel_rms_error": rel(tot["sse"], tot["sum_sq"]),
        "rel_rms_error_neighbours": rel(tot["sse_neighbours"], tot["sum_sq_neighbours"]),
        "rel_rms_error_clean": rel(tot["sse_clean"], tot["sum_sq_clean"]),
        "subnormal_scale_block_share": tot["subnormal_scale_blocks"] / tot["blocks"],
        "zero_scale_block_share": tot["zero_scale_blocks"] / tot["blocks"],
        "saturated_share": tot["saturated_elements"] / tot["elements"],
        "kernel": {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9, "bytes": nbytes, "bound": "hbm",
                   "frac": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
    }


def weak_scaling_value(tokens_per_rank: int, world: int, max_ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank's batch, over the slowest rank's time."""
    return tokens_per_rank * world / (max_ms_per_step * 1e-3)


MMA_PEAK_MODES = {
    0: "", 1: "_scale_copies_one_buffer", 5: "_stage_handshake", 6: "_stage_handshake_scale_copies",
    9: "_8_stages", 10: "_8_stages_scale_copies", 13: "_scale_copies_commit", 14: "_commit",
    15: "_scale_copies_fence", 16: "_scale_copies_commit_every_2nd", 17: "_split_issue",
    18: "_split_issue_handshake", 19: "_warp_predicated_scale_copies", 20: "_warp_predicated",
    21: "_warp_branch_scale_copies",
}


def run_mma_peak():
    """FP4 MMA rate per SM clock with operands resident in shared memory."""
    from nvfp4_w4a4_quantized_moe_b200 import capi as c
    res = {}
    for n in (256, 128):
        for mode, name in MMA_PEAK_MODES.items():
            c.nvfp4_test_mma_peak(200, n, mode)                    # warm-up
            fpc, cyc = c.nvfp4_test_mma_peak(20000, n, mode)
            res[f"n{n}{name}"] = {"flop_per_sm_clock": float(fpc.median()), "cycles_median": float(cyc.median())}
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    best = max(v["flop_per_sm_clock"] for v in res.values())
    print(json.dumps({"mma_peak": res, "sms": sms,
                      "pflops_at_1965mhz": best * sms * 1.965e9 / 1e15}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.mma_peak:
        return run_mma_peak()
    cfg = workloads.CONFIGS[args.workload]
    if args.impl == "reference":
        return run_reference(args, cfg)
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device; the layer has no CPU path"}))
        return 1
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
