#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 routed-expert MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill]
    python bench.py --impl reference ...      # the CPU oracle, timed as it stands

One step = one pass of the layer's hot path over one batch of the workload:
router GEMM, top-k, permutation, FP4 quantisation of x, grouped FP4 GEMM
gate/up with SiLU*up and requantisation, grouped FP4 GEMM down, weighted
combine (one moe_nvfp4_forward call).

The headline is the prefill layer (8192 tokens through 80 experts of hidden
6144 and intermediate 2048, top-8, skewed expert loads), the largest
single-GPU configuration; its roofline is the gate/up GEMM's FP4 tensor rate.
The same JSON line carries sub-records for the decode layer (16 tokens,
memory-bound, also timed with the L2 flushed), the unpruned outlier layer
(4096 tokens, 128 experts), the tiny layer, and the offline RTN weight
quantiser over the full 80-expert layer (it runs once per checkpoint, not per
batch; back to back and with the L2 flushed).

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
    routing (one single-block kernel up to 256 tokens, else a top-k and a
    permutation kernel), quantise-scatter (folded into the routing kernel
    for small layers), the two GEMMs and the combine."""
    return c.moe_nvfp4_forward_launches(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k)
NVFP4_BYTES_PER_ELEM = 0.5 + 1.0 / 16


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "prefill", "outlier", "tiny", "prefill16", "quantiser"],
                    default="prefill",
                    help="the headline workload (default: prefill, the largest single-GPU configuration); "
                         "quantiser times the offline weight quantiser alone")
    ap.add_argument("--quantiser-experts", type=int, default=80,
                    help="experts whose gate, up and down matrices the quantiser workload quantises (default 80, "
                         "the full layer; a few make a small case for profiler captures)")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the decode, outlier and tiny sub-records")
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


def _code_only(text: str) -> str:
    """C++ source without its comments and blank lines, so that an edit of a
    comment does not change the hash (the sources hold no comment markers
    inside string literals)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def gemm_source_sha() -> str:
    """Hash of the code (comments stripped) the GEMM kernel is compiled from."""
    import hashlib
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        src = open(os.path.join(ROOT, "nvfp4_w4a4_quantized_moe_b200", "csrc", name), encoding="utf-8").read()
        h.update(_code_only(src).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, algorithmic_bytes: float | None = None):
    """(dram bytes per launch, source) recorded by ncu for this kernel and
    workload, or (None, None) when no record exists or the kernel source
    changed since.  A record taken on a reduced case of the same layer shape
    (its line names the workloads it scales to) gives this workload's traffic
    as its measured-to-algorithmic ratio times this launch's algorithmic
    bytes."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None, None
    sha = gemm_source_sha()
    scaled = None
    for line in open(path):
        if line.startswith("#"):
            continue
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("kernel") != kernel or f.get("source_sha") != sha:
            continue
        if f.get("workload") == workload:
            return float(f["dram_bytes_per_launch"]), f"ncu capture ({workload})"
        if algorithmic_bytes and workload in f.get("scale_to", "").split(","):
            ratio = float(f["dram_bytes_per_launch"]) / float(f["algorithmic_bytes"])
            scaled = (ratio * algorithmic_bytes, f"ncu capture ({f['workload']}) scaled by algorithmic bytes")
    return scaled if scaled else (None, None)


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
                             "sample": sample_desc(cfg), "host": host_cpu()},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

L2_FLUSH_BYTES = 256 << 20          # written between flushed iterations (L2 is 126 MB)
PAIR_MIN_ROWS = 2048                # the library's threshold for the CTA-pair GEMMs (T * k)
MMA_FLOP_PER_SM_CLOCK_NOMINAL = 32768.0


def host_cpu():
    """CPU model and the BLAS library and thread count the oracle runs on."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    blas = None
    try:
        from threadpoolctl import threadpool_info
        libs = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if libs:
            blas = {"library": libs[0].get("internal_api"), "threads": libs[0].get("num_threads")}
    except Exception:
        pass
    return {"cpu_model": model, "logical_cpus": os.cpu_count(), "blas": blas}


def events(n):
    """n CUDA timing events, each recorded once (torch creates the CUDA event
    lazily, and the library records events it is handed)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    return evs


def time_loop(fn, steps, dist, flush=None):
    """Device time per call of fn.  Back to back (flush None): one event pair
    around all the calls.  Flushed: every call between its own event pair,
    with the L2 flushed (a buffer larger than L2 written) before each."""
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    dist.barrier()
    if flush is None:
        e0, e1 = events(2)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
    else:
        pairs = [events(2) for _ in range(steps)]
        for a, b in pairs:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        ms = float(np.mean([a.elapsed_time(b) for a, b in pairs]))
    dist.barrier()
    return dist.max(ms)


class LayerRun:
    """One workload's layer resident on the device: inputs, RTN-quantised
    weights (the library's quantiser), calibrated activation scales (g1 from
    x, g2 from a calibration pass over h) and a workspace."""

    def __init__(self, c, cfg, seed, dev, keep_bf16=False):
        self.c, self.cfg, self.dev = c, cfg, dev
        self.x = workloads.hidden_states(cfg, seed, device=dev)
        self.wg, self.bias, self.off = workloads.router_params(cfg, seed, device=dev)
        gate, up, down = workloads.stacked_expert_weights(cfg, seed, device=dev)
        self.W = c.MoeWeights.quantize(gate, up, down, self.wg, self.bias, cfg.k, cfg.rsf)
        self.bf16 = (gate, up, down) if keep_bf16 else None
        del gate, up, down
        self.g1 = (self.x.float().abs().amax() / 2688.0).reshape(1).float()
        ones = torch.ones(1, device=dev)
        _, dbg = c.moe_nvfp4_forward(self.W, self.x, self.g1, ones, logit_offset=self.off, debug=True)
        self.g2 = (dbg["h_amax"] / 2688.0).reshape(1).float()
        topk = dbg["topk_idx"].cpu().numpy()
        del dbg
        self.hit = int(len(np.unique(topk)))
        self.counts = np.bincount(topk.ravel(), minlength=cfg.E)
        self.ws = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k), dtype=torch.uint8,
                              device=dev)
        self.out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
        torch.cuda.empty_cache()

    def step(self, evs=None):
        self.c.moe_nvfp4_forward(self.W, self.x, self.g1, self.g2, logit_offset=self.off, out=self.out,
                                 workspace=self.ws, stage_events=evs)

    def warm(self, n):
        for _ in range(max(n, 3)):
            self.step()
        torch.cuda.synchronize()
        self.c.nvfp4_workspace_status(self.ws)

    def stages(self, steps, dist):
        """Per-stage device times from events the library records between its
        stages.  An event between two kernels stops the second from starting
        early, so the stages add up to a little more than the step."""
        evs = [events(self.c.N_STAGE_EVENTS) for _ in range(steps)]
        for i in range(steps):
            self.step(evs[i])
        torch.cuda.synchronize()
        self.c.nvfp4_workspace_status(self.ws)
        names = ("route", "quantize_x", "gemm_gate_up", "gemm_down", "combine")
        return {n: dist.max(float(np.mean([evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps)])))
                for j, n in enumerate(names)}

    def e2e(self, steps, dist):
        """Through the library's host-buffer call: every step copies its x in
        from pinned host memory and its out back, inside the timed region.
        Steps alternate between two workspaces, so that one step's copies
        run on the library's copy streams while the other computes."""
        c, cfg = self.c, self.cfg
        x_h = self.x.cpu().pin_memory()
        outs = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory() for _ in range(2)]
        nbytes = c.moe_nvfp4_workspace_size_host(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k)
        wss = [torch.empty(nbytes, dtype=torch.uint8, device=self.dev) for _ in range(2)]

        def run(i):
            c.moe_nvfp4_forward_host(self.W, x_h, self.g1, self.g2, outs[i % 2], wss[i % 2], logit_offset=self.off)

        for i in range(4):
            run(i)
        for ws in wss:
            c.moe_nvfp4_host_join(ws)
        stream = torch.cuda.current_stream()
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = events(2)
        e0.record(stream)
        for i in range(steps):
            run(i)
        for ws in wss:
            c.moe_nvfp4_host_join(ws)
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        ms = dist.max(e0.elapsed_time(e1) / steps)
        for ws in wss:
            c.nvfp4_workspace_status(ws)
            c.moe_nvfp4_host_release(ws)
        del wss
        torch.cuda.empty_cache()
        return {"value": cfg.T * dist.world / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
                "h2d_bytes_per_step": self.x.numel() * 2, "d2h_bytes_per_step": self.out.numel() * 2,
                "path": "moe_nvfp4_forward_host: pinned host x in and out back on the library's copy streams, "
                        "two workspaces alternating so that copies overlap the other step's compute"}

    def work(self):
        """Algorithmic FLOPs and bytes of the two GEMMs for this batch's routing."""
        cfg, P, hit = self.cfg, self.cfg.T * self.cfg.k, self.hit
        return {
            "gemm_gate_up": (2.0 * P * cfg.H * 2 * cfg.I,
                             (hit * 2 * cfg.I * cfg.H + P * cfg.H + P * cfg.I) * NVFP4_BYTES_PER_ELEM),
            "gemm_down": (2.0 * P * cfg.I * cfg.H,
                          (hit * cfg.H * cfg.I + P * cfg.I) * NVFP4_BYTES_PER_ELEM + P * cfg.H * 2),
        }

    def layer_bytes(self):
        """Bytes the whole layer must move: the weights of the experts it hits,
        the router weight, x in and out."""
        cfg = self.cfg
        return (self.hit * 3 * cfg.H * cfg.I * NVFP4_BYTES_PER_ELEM + cfg.E * cfg.H * 2 + 2 * cfg.T * cfg.H * 2)


def gemm_roofline(run, stage_ms, peaks, fp4_peak, fp4_src, kernel_stage):
    """Roofline entry of one GEMM launch: FLOPs against the FP4 peak when its
    intensity is above the ridge, else bytes against HBM."""
    flops, nbytes = run.work()[kernel_stage]
    t = stage_ms[kernel_stage] * 1e-3
    # batches of at least 2048 (token, expert) rows run on CTA pairs
    base = "grouped_fp4_gemm_pair_kernel" if run.cfg.T * run.cfg.k >= PAIR_MIN_ROWS else "grouped_fp4_gemm_kernel"
    kname = base + ("<0>" if kernel_stage == "gemm_gate_up" else "<1>")
    if flops / (fp4_peak * 1e12) > nbytes / (peaks["hbm_gbs"] * 1e9):
        roof = {"bound": "tensor", "achieved": flops / t / 1e12, "peak": fp4_peak, "unit": "TFLOP/s",
                "peak_source": fp4_src}
    else:
        roof = {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_source": "measured copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"], roof["traffic_source"] = recorded_traffic(kname, run.cfg.name, nbytes)
    roof["kernel"] = kname
    roof["ms"] = stage_ms[kernel_stage]
    roof["algorithmic"] = {"bytes": nbytes, "flops": flops, "experts_hit": run.hit, "pairs": run.cfg.T * run.cfg.k}
    return roof


def mma_peak_now(c):
    """FP4 MMA rate per SM clock (operands resident in shared memory), measured
    now; falls back to the nominal 32,768 if the microbenchmark fails."""
    try:
        c.nvfp4_test_mma_peak(200, 256, 0)
        fpc, _ = c.nvfp4_test_mma_peak(5000, 256, 0)
        return float(fpc.median()), "measured"
    except Exception as exc:  # noqa: BLE001
        return MMA_FLOP_PER_SM_CLOCK_NOMINAL, f"nominal ({exc})"


def sub_record(c, cfg, args, dist, peaks, fp4_peak, fp4_src, flush):
    """A workload besides the headline: its own step time, stage breakdown,
    roofline and end-to-end figure."""
    run = LayerRun(c, cfg, args.seed, torch.device("cuda", torch.cuda.current_device()))
    run.warm(args.warmup)
    steps = max(args.steps, 20)
    ms = time_loop(run.step, steps, dist)
    st = run.stages(steps, dist)
    rec = {"workload": cfg.name, "tokens": cfg.T, "E": cfg.E, "k": cfg.k, "steps": steps, "ms_per_step": ms,
           "tokens_per_s": cfg.T * dist.world / (ms * 1e-3), "stages_ms": st}
    if cfg.T * cfg.k <= 256 and cfg.H >= 1024:
        # memory-bound: the L2 is flushed between iterations too, and the whole
        # layer's bytes are set against HBM
        msf = time_loop(run.step, steps, dist, flush=flush)
        rec["ms_per_step_l2_flushed"] = msf
        rec["layer_hbm"] = {"bytes": run.layer_bytes(), "gbs": run.layer_bytes() / (ms * 1e-3) / 1e9,
                            "gbs_l2_flushed": run.layer_bytes() / (msf * 1e-3) / 1e9,
                            "frac": run.layer_bytes() / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                            "frac_l2_flushed": run.layer_bytes() / (msf * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    if cfg.H >= 1024:
        rec["roofline"] = gemm_roofline(run, st, peaks, fp4_peak, fp4_src, "gemm_gate_up")
        rec["roofline_down"] = gemm_roofline(run, st, peaks, fp4_peak, fp4_src, "gemm_down")
        w = run.work()
        gms = st["gemm_gate_up"] + st["gemm_down"]
        rec["gemm"] = {"ms": gms, "tflops": (w["gemm_gate_up"][0] + w["gemm_down"][0]) / (gms * 1e-3) / 1e12}
        rec["gemm"]["frac_of_fp4_peak"] = rec["gemm"]["tflops"] / fp4_peak
    else:
        rec["bound"] = "launch latency (no roofline)"
    rec["e2e"] = run.e2e(steps, dist)
    rec["gpu_launches_per_step"] = kernels_per_step(c, cfg)
    if cfg.T * cfg.k <= 256 and cfg.H >= 1024:
        rec["shared_expert"] = shared_expert_record(c, run, cfg, args, dist, peaks)
    c.nvfp4_workspace_status(run.ws)
    diag = None
    if cfg.name == "outlier":
        gate, up, down = workloads.stacked_expert_weights(cfg, args.seed, device=run.dev)
        diag = block_stats_report(c, cfg, (gate, up, down), run.W, torch.cuda.current_stream(), dist, peaks)
        del gate, up, down
    del run
    torch.cuda.empty_cache()
    return rec, diag


def quantiser_record(c, bf16, dist, peaks, flush, steps, layout):
    """The offline RTN weight quantiser over one full layer (gate, up and down
    of every expert), timed back to back and with the L2 flushed before each
    pass.  Gate and up have the same shape, so they are quantised as one call
    over the experts' gate matrices followed by their up matrices (the fused
    gate/up tensor a serving checkpoint keeps), and down as a second call: two
    calls, each with one ramp and one tail.  Outputs and workspace are
    allocated once, outside the timed region."""
    gate, up, down = bf16
    dev = gate.device
    mats = (torch.cat([gate, up]), down)
    qws = torch.empty(c.lib.nvfp4_quantize_weights_workspace_size(mats[0].shape[0]), dtype=torch.uint8, device=dev)
    outs = [c.nvfp4_quantize_weights(w, layout, workspace=qws) for w in mats]

    def run():
        for w, o in zip(mats, outs):
            c.nvfp4_quantize_weights(w, layout, workspace=qws, out=o)

    qbytes = sum(2 * w.numel() + w.numel() // 2 + w.numel() // 16 + 4 * w.shape[0] for w in mats)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    steps = max(3, min(steps, 20))
    ms = time_loop(run, steps, dist)
    msf = time_loop(run, steps, dist, flush=flush)
    c.nvfp4_workspace_status(qws)
    gbs, gbsf = qbytes / (ms * 1e-3) / 1e9, qbytes / (msf * 1e-3) / 1e9
    n, r, k = gate.shape
    del mats, outs
    return {"workload": f"quantiser: {n} x (gate, up {r}x{k}; down {k}x{r}) bf16 N(0, 0.02)", "layout": layout,
            "calls": "2: gate and up stacked (2 x {} matrices of {}x{}), then down ({} of {}x{})".format(n, r, k, n, k, r),
            "ms": ms, "gbs": gbs, "ms_l2_flushed": msf, "gbs_l2_flushed": gbsf, "bytes": qbytes,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "frac_l2_flushed": gbsf / peaks["hbm_gbs"],
                         "kernel": "quantize_weights_kernel"}}


def shared_expert_record(c, run, cfg, args, dist, peaks):
    """The layer with its shared BF16 expert (f1): one SiLU-gated MLP of the
    routed experts' shape (I_shared = I), bf16 N(0, 0.02) weights.  Its GEMMs
    (with a split-K reduction after each at small batches) are timed between
    the library's events after the routed down GEMM and after the shared
    GEMMs.  Within a step the routed GEMMs stream the expert weights through
    L2 first, so the shared weights are not L2-resident when read."""
    dev = run.dev
    sh = tuple(t.contiguous() for t in workloads.expert_weights(cfg, cfg.E + 7, args.seed, device=dev))
    Ws = run.W.with_shared(*sh)
    ws_sh = torch.empty(c.moe_nvfp4_workspace_size(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k, cfg.I), dtype=torch.uint8,
                        device=dev)
    fn = lambda: c.moe_nvfp4_forward(Ws, run.x, run.g1, run.g2, logit_offset=run.off, out=run.out,  # noqa: E731
                                     workspace=ws_sh)
    for _ in range(3):
        fn()
    steps = max(args.steps, 20)
    sh_step_ms = time_loop(fn, steps, dist)
    sh_evs = [(events(c.N_STAGE_EVENTS), events(1)[0]) for _ in range(steps)]
    for st_evs, sh_ev in sh_evs:
        c.moe_nvfp4_forward(Ws, run.x, run.g1, run.g2, logit_offset=run.off, out=run.out, workspace=ws_sh,
                            stage_events=st_evs, shared_event=sh_ev)
    torch.cuda.synchronize()
    c.nvfp4_workspace_status(ws_sh)
    sh_ms = dist.max(float(np.mean([st[4].elapsed_time(ev) for st, ev in sh_evs])))
    sh_flops = 6.0 * cfg.T * cfg.H * cfg.I
    sh_bytes = 3.0 * cfg.H * cfg.I * 2 + 2.0 * cfg.T * cfg.H * 2 + 2.0 * cfg.T * cfg.I * 2 * 2
    sh_tf = sh_flops / (sh_ms * 1e-3) / 1e12
    sh_gbs = sh_bytes / (sh_ms * 1e-3) / 1e9
    sh_tensor = sh_flops / (peaks["bf16_tflops"] * 1e12) > sh_bytes / (peaks["hbm_gbs"] * 1e9)
    rec = {"I_shared": cfg.I, "ms_per_step": sh_step_ms, "gemms_ms": sh_ms, "flops": sh_flops,
           "bytes": sh_bytes, "tflops": sh_tf, "gbs": sh_gbs,
           "bound": "tensor" if sh_tensor else "hbm",
           "frac": sh_tf / peaks["bf16_tflops"] if sh_tensor else sh_gbs / peaks["hbm_gbs"],
           "peak": peaks["bf16_tflops"] if sh_tensor else peaks["hbm_gbs"],
           "peak_unit": "TFLOP/s (bf16 burst)" if sh_tensor else "GB/s",
           "gpu_launches_per_step": c.moe_nvfp4_forward_launches(cfg.T, cfg.E, cfg.H, cfg.I, cfg.k, cfg.I)}
    del Ws, sh, ws_sh
    torch.cuda.empty_cache()
    return rec


def run_ours(args, cfg):
    from nvfp4_w4a4_quantized_moe_b200 import capi as c
    dist = Dist()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    # FP4 denominator: the measured bf16 burst rate (a kernel timed alone)
    # times the nominal dense FP4/BF16 ratio
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    fp4_src = f"{peak_src} bf16 burst (bf16_tflops) x {FP4_OVER_BF16:g}, the nominal dense FP4/BF16 ratio"
    mma_fpc, mma_src = mma_peak_now(c)

    # ---------------------------------------------------------------- headline
    run = LayerRun(c, cfg, args.seed, dev, keep_bf16=cfg.E == 80 and cfg.H == 6144 and cfg.I == 2048)
    run.warm(args.warmup)
    # keep the GPU busy briefly so the clock sampler sees steady state
    sampler = ClockSampler(dev.index) if dist.rank == 0 else None
    t_warm = time.time()
    while time.time() - t_warm < 0.5:
        run.step()
        torch.cuda.synchronize()
    t0 = time.time()
    ms_step = time_loop(run.step, args.steps, dist)
    t1 = time.time()
    clocks = sampler.stop(t0, t1) if sampler else None
    c.nvfp4_workspace_status(run.ws)
    stage_ms = run.stages(args.steps, dist)

    # the activation global-scale modes beyond the calibrated per-tensor one
    mode_ms = {}
    for mode in ("expert", "dynamic", "dynamic_expert"):
        n = cfg.E if mode in ("expert", "dynamic_expert") else 1
        a = run.g1.repeat(n).contiguous() if mode == "expert" else torch.zeros(n, device=dev)
        h = run.g2.repeat(n).contiguous()
        fn = lambda: c.moe_nvfp4_forward(run.W, run.x, a, h, logit_offset=run.off, out=run.out,  # noqa: E731
                                         workspace=run.ws, act_scale_mode=mode)
        for _ in range(3):
            fn()
        mode_ms[mode] = time_loop(fn, args.steps, dist)
    c.nvfp4_workspace_status(run.ws)
    # the same forward accumulating REAP saliency (f3)
    sal = (torch.zeros(cfg.E, dtype=torch.float64, device=dev), torch.zeros(cfg.E, dtype=torch.int64, device=dev))
    fn = lambda: c.moe_nvfp4_forward(run.W, run.x, run.g1, run.g2, logit_offset=run.off, out=run.out,  # noqa: E731
                                     workspace=run.ws, saliency=sal)
    for _ in range(3):
        fn()
    sal_ms = time_loop(fn, args.steps, dist)
    c.nvfp4_workspace_status(run.ws)
    shared_report = shared_expert_record(c, run, cfg, args, dist, peaks)
    e2e = run.e2e(args.steps, dist)

    # roofline of the dominant kernel (the gate/up GEMM) and of the down GEMM
    roof = gemm_roofline(run, stage_ms, peaks, fp4_peak, fp4_src, "gemm_gate_up")
    roof_down = gemm_roofline(run, stage_ms, peaks, fp4_peak, fp4_src, "gemm_down")
    w = run.work()
    gemm_ms = stage_ms["gemm_gate_up"] + stage_ms["gemm_down"]
    gemm_tf = (w["gemm_gate_up"][0] + w["gemm_down"][0]) / (gemm_ms * 1e-3) / 1e12
    sm_mhz = (clocks or {}).get("sm_mhz")
    mma_at_clock = mma_fpc * sms * sm_mhz * 1e6 / 1e12 if sm_mhz else None
    for r in (roof, roof_down):
        if r["bound"] == "tensor" and mma_at_clock:
            r["mma_microbenchmark_peak_at_sampled_clock"] = {
                "tflops": mma_at_clock, "flop_per_sm_clock": mma_fpc, "source": mma_src, "sm_mhz": sm_mhz,
                "frac": r["achieved"] / mma_at_clock}

    diag = block_stats_report(c, cfg, run.bf16, run.W, stream, dist, peaks) if run.bf16 else None
    quant = None
    if run.bf16 is not None:
        qlayout = "staged" if run.W.codes_layout == c.LAYOUT_STAGED else "tiled"
        quant = quantiser_record(c, run.bf16, dist, peaks, flush, args.steps, qlayout)
    run.bf16 = None
    torch.cuda.empty_cache()

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        smp = OracleSample(cfg, args.seed, run.x, run.wg, run.bias, run.off)
        smp.step()
        t = time.perf_counter()
        n = 0
        while n < cfg.k or time.perf_counter() - t < 10.0:
            smp.step()
            n += 1
        dt = (time.perf_counter() - t) / n
        cpu = {"value": smp.tokens_per_step() / dt, "unit": "tokens/s", "cores": OracleSample.threads(),
               "kind": "oracle", "sample": sample_desc(cfg) + f"; {n} pairs timed", "host": host_cpu()}

    # the other workloads, each its own record
    headline_launches = kernels_per_step(c, cfg) * args.steps
    subs, diag_outlier = {}, None
    if not args.headline_only:
        del run
        torch.cuda.empty_cache()
        for name in ("decode", "outlier", "tiny"):
            if name == cfg.name:
                continue
            rec, d = sub_record(c, workloads.CONFIGS[name], args, dist, peaks, fp4_peak, fp4_src, flush)
            subs[name] = rec
            diag_outlier = d or diag_outlier
        if quant is not None:
            subs["quantiser"] = quant
    elif quant is not None:
        subs["quantiser"] = quant

    line = {
        "metric": METRIC, "value": weak_scaling_value(cfg.T, dist.world, ms_step), "unit": "tokens/s",
        "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": cfg.name, "tokens_per_gpu": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
                   "rsf": cfg.rsf, "x_outliers": cfg.x_outlier_p, "logit_offset_std": cfg.logit_offset_std,
                   "weight_outliers": cfg.w_outlier_p, "parallelism": f"replicas{dist.world}",
                   "l2": "inputs larger than L2 (expert weights of the layer: "
                         f"{(run_weight_bytes(cfg)) / 1e9:.2f} GB; x {cfg.T * cfg.H * 2 / 1e6:.0f} MB); the "
                         "memory-bound sub-records (decode, quantiser) are also timed with L2 flushed"},
        "gemm": {"ms": gemm_ms, "tflops": gemm_tf, "frac_of_fp4_peak": gemm_tf / fp4_peak, "fp4_peak": fp4_peak},
        "stages_ms": stage_ms,
        "roofline": roof,
        "roofline_down": roof_down,
        "act_scale_modes_ms_per_step": dict({"tensor": ms_step}, **mode_ms),
        "reap_saliency_ms_per_step": sal_ms,
        "shared_expert": shared_report,
        "e2e": e2e,
        "gpu_launches": headline_launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "sub_records": subs,
        "diagnostics": {"headline_weights": diag, "outlier_weights": diag_outlier},
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def run_weight_bytes(cfg):
    return cfg.E * 3 * cfg.H * cfg.I * NVFP4_BYTES_PER_ELEM


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
    if args.workload == "quantiser":
        return run_quantiser_only(args)
    return run_ours(args, cfg)


def run_quantiser_only(args):
    """The offline RTN weight quantiser alone, over the gate, up and down
    matrices of --quantiser-experts experts (bf16 N(0, 0.02), hidden 6144,
    intermediate 2048): one JSON line with its GB/s against HBM."""
    from nvfp4_w4a4_quantized_moe_b200 import capi as c
    dist = Dist()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, _ = load_peaks()
    cfg = dataclasses_replace(workloads.CONFIGS["quantiser"], E=args.quantiser_experts)
    bf16 = workloads.stacked_expert_weights(cfg, args.seed, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    rec = quantiser_record(c, bf16, dist, peaks, flush, args.steps, "staged")
    line = {"metric": METRIC, "value": rec["gbs"], "unit": "GB/s", "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": rec["ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
            "config": {"workload": "quantiser", "experts": cfg.E, "H": cfg.H, "I": cfg.I,
                       "l2": "flushed and back-to-back both reported"},
            "quantiser": rec, "roofline": rec["roofline"]}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def dataclasses_replace(cfg, **kw):
    import dataclasses
    return dataclasses.replace(cfg, **kw)


if __name__ == "__main__":
    sys.exit(main())
