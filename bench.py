#!/usr/bin/env python
"""Throughput of the block-causal, frame-wise linear-attention scan on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step is one pass of the whole scan (load Q/K/V, per-frame contractions,
state recurrence, outputs and final state) over one batch of seeded
synthetic input already resident in HBM.  The default workload is the
720p, 60 s frame-wise GDN scan (B=1, H=20, D=128, F=181 latent frames of
22x40 tokens).  Prints one JSON line.

Metric: latent frames per second (B*F per step, all heads), with TFLOP/s
(algorithmic count) and the fraction of the HBM roofline.  Inputs (>3 GB a
step) are far larger than the 126 MB L2, so no L2 flush is needed between
steps.

--impl reference times the CPU oracle on the host cores instead (a bounded
sample of the same workload each step).  N > 1 runs the workload once per
rank on its own data, no collective on the data path (weak scaling); the
reported time is the max over ranks.  Under torchrun the ranks come from
the environment; `--gpus N` without torchrun launches N ranks itself.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

WORKLOADS = {
    # bench name: (synthetic workload, mode)
    "gdn_720p_60s": ("gdn_720p_60s", "gdn"),
    "relu_480p": ("relu_480p", "relu"),
    "stream_gdn": ("gdn_stream", "gdn"),
    "stress_gdn": ("stress_d256", "gdn"),
    "stress_relu": ("stress_d256", "relu"),
    # reversed GDN scan reset every 8 frames, on the 720p 60 s clip
    "gdn_720p_60s_reverse8": ("gdn_720p_60s", "gdn_reverse"),
    # per-token update gate on the 720p 60 s clip
    "gdn_720p_60s_token_beta": ("gdn_720p_60s", "gdn_token_beta"),
    # the same two variants on the stress workload's 256-wide heads
    "stress_gdn_reverse8": ("stress_d256", "gdn_reverse"),
    "stress_gdn_token_beta": ("stress_d256", "gdn_token_beta"),
    # raw q, k with RMSNorm, ReLU and 3D RoPE fused into the scan (22 x 40 grid)
    "gdn_720p_60s_prep": ("gdn_720p_60s_raw", "gdn_prep"),
    "tiny_gdn": ("tiny_fp32", "gdn"),
    "tiny_relu": ("tiny_fp32", "relu"),
}
DEFAULT_WORKLOAD = "gdn_720p_60s"
METRIC = "latent frames/s and TFLOP/s of block-causal GDN/ReLU scan; % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------
# Algorithmic counts (fixed formulas, whatever the kernels do)
# ----------------------------------------------------------------------------
REVERSE_CHUNK = 8      # frames per chunk of the reversed-scan workload
PREP_NORM_EPS = 1e-6   # RMSNorm epsilon of the fused input preparation


def frame_flops(mode: str, S: int, D: int) -> int:
    """ReLU: phi(K)^T V and phi(Q) M (2SD^2 each), z and phi(Q) z (2SD each).
    GDN (either direction): Kh^T Kh, Kh^T V, Q M (2SD^2 each) and G M (2D^3)."""
    if mode == "relu":
        return 4 * S * D * D + 4 * S * D
    return 6 * S * D * D + 2 * D ** 3


def call_bytes(mode: str, B: int, H: int, F: int, S: int, D: int, elem: int,
               state_in: bool) -> int:
    """q, k, v read once and o written once; alpha, beta read once (GDN);
    the state (and z) written once per (b, h) and read once if given (the
    reversed scan has no state in or out)."""
    per_frame = 4 * S * D * elem + (8 if mode != "relu" else 0) + \
        (4 * (S - 1) if mode == "gdn_token_beta" else 0)
    per_bh_prep = 2 * D * 4 if mode == "gdn_prep" else 0     # the two RMSNorm weight rows
    per_bh = D * D * 4 * (2 if state_in else 1) if mode != "gdn_reverse" else 0
    if mode == "relu":
        per_bh += D * 4 * (2 if state_in else 1)
    return B * H * (F * per_frame + per_bh + per_bh_prep)


def step_plan(spec, mode):
    """List of calls one step makes: (frame offset, frames, state_in?)."""
    if spec.chunk_frames:
        C = spec.chunk_frames
        return [(c * C, C, c > 0) for c in range(spec.F // C)]
    return [(0, spec.F, False)]


def step_counts(spec, mode):
    elem = spec.elem_bytes
    byts = sum(call_bytes(mode, spec.B, spec.H, n, spec.S, spec.D, elem, si)
               for _, n, si in step_plan(spec, mode))
    flops = spec.B * spec.H * spec.F * frame_flops(mode, spec.S, spec.D)
    return byts, flops


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Sources the kernels of a path are compiled from (a traffic record names its own).
KERNEL_SOURCES = ("tc_fused.cu", "tc_common.cuh", "tmap.cuh", "common.cuh")


def kernel_source_hash(sources=KERNEL_SOURCES) -> str:
    """Hash of a kernel's sources, so a committed DRAM-traffic figure is used
    only while the kernel it was measured on is unchanged.  Lines of the
    optional event trace are left out: without -DLA_TRACE they compile to
    nothing."""
    h = hashlib.sha256()
    for name in sources:
        p = os.path.join(ROOT, "linear_attention_video_frame_b200", "csrc", name)
        for line in open(p, "rb").read().splitlines(keepends=True):
            if b"LA_TRACE" not in line:
                h.update(line)
    return h.hexdigest()[:16]


def traffic_record(workload: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary, if it was taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(workload)
    except Exception:
        return None
    if not d or d.get("kernel_source_hash") != kernel_source_hash(
            tuple(d.get("sources", KERNEL_SOURCES))):
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------
# Multi-rank host logic (weak scaling: one replica per rank, own data)
# ----------------------------------------------------------------------------
def rank_spec(base, rank: int):
    """Rank r > 0 scans its own batch: the same workload with seed + 1000 r."""
    return base.with_(seed=base.seed + 1000 * rank) if rank else base


def max_over_ranks(value: float, device=None) -> float:
    """The slowest rank's time (the job's time); plumbing only, not on the data path."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------
# Clock sampling during the timed region (NVML; read-only)
# ----------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.001):
        self.samples, self.stamps, self.bits, self.reasons, self.max_mhz = [], [], [], 0, None
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report nothing rather than guess
            self.nv = None
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.reasons |= bits
                self.samples.append(mhz)
                self.bits.append(bits)
                self.stamps.append(time.perf_counter())
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.nv:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self):
        if self._thr:
            self._stop.set()
            self._thr.join()

    def between(self, t0: float, t1: float):
        """SM clock samples taken between host times t0 and t1."""
        return [m for m, t in zip(self.samples, self.stamps) if t0 <= t <= t1]

    def reasons_between(self, t0: float, t1: float):
        """Names of the throttle reasons seen between host times t0 and t1."""
        acc = 0
        for b, t in zip(self.bits, self.stamps):
            if t0 <= t <= t1:
                acc |= b
        return [n for bit, n in self.REASONS.items() if acc & bit and n != "gpu_idle"]

    def summary(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml_unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# The CPU oracle arm (reported baseline, never the product path)
# ----------------------------------------------------------------------------
def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max(int(i.get("num_threads", 1)) for i in info) if info else 1
    except Exception:
        return 1


def time_oracle_sample(spec, mode, budget_s: float, max_heads=None):
    """Run the oracle on whole (b, h) slices of the workload until about
    budget_s of CPU time has passed; return (equivalent frames/s, sample text)."""
    import oracle
    a_all, b_all = synth.gates(spec)
    btok_all = synth.token_gates(spec) if mode == "gdn_token_beta" else None
    pairs = [(b, h) for b in range(spec.B) for h in range(spec.H)]
    done, t_total = 0, 0.0
    for b, h in pairs:
        q, k, v = (synth.slice_values(spec, n, b, h).astype(np.float64)[None, None] for n in "qkv")
        a = a_all[b:b + 1, h:h + 1]
        bt = b_all[b:b + 1, h:h + 1]
        t0 = time.perf_counter()
        if mode == "relu":
            oracle.relu_scan(q, k, v, spec.eps)
        elif mode == "gdn_reverse":
            oracle.gdn_scan_reverse_chunked(q, k, v, a, bt, spec.k_scale, REVERSE_CHUNK)
        elif mode == "gdn_token_beta":
            oracle.gdn_scan_token_beta(q, k, v, a, btok_all[b:b + 1, h:h + 1], spec.k_scale)
        elif mode == "gdn_prep":
            gh, gw = spec.grid
            oracle.gdn_scan_prep(q, k, v, a, bt, spec.k_scale,
                                 synth.norm_weights(spec, "q")[h:h + 1],
                                 synth.norm_weights(spec, "k")[h:h + 1], PREP_NORM_EPS, gh, gw)
        else:
            oracle.gdn_scan(q, k, v, a, bt, spec.k_scale)
        t_total += time.perf_counter() - t0
        done += 1
        if t_total >= budget_s or (max_heads and done >= max_heads):
            break
    frames = spec.B * spec.F * done / (spec.B * spec.H)   # equivalent whole-batch frames
    sample = (f"oracle on {done} of {spec.B * spec.H} (b,h) slices x all {spec.F} frames of "
              f"{spec.name} ({mode}); frames/s scaled by slices/(B*H)")
    return frames / t_total, t_total, sample


def workload_label(spec_name: str, mode: str) -> str:
    """config.workload of a JSON line: the workload's name, plus the variant."""
    return spec_name + {"gdn_reverse": f"_reverse{REVERSE_CHUNK}",
                        "gdn_token_beta": "_token_beta", "gdn_prep": "_prep"}.get(mode, "")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    wname, mode = WORKLOADS[args.workload]
    spec = synth.workload(wname)
    byts, flops = step_counts(spec, mode)
    for _ in range(args.warmup):
        time_oracle_sample(spec, mode, 0.0, max_heads=1)
    vals, ts = [], 0.0
    for _ in range(args.steps):
        v, t, sample = time_oracle_sample(spec, mode, 0.0, max_heads=1)
        vals.append(v)
        ts += t
    value = args.steps / sum(1.0 / v for v in vals)      # frames / total time
    cores = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "latent frames/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * ts / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
        "config": {"workload": workload_label(spec.name, mode), "mode": mode, "B": spec.B,
                   "H": spec.H, "F": spec.F,
                   "S": spec.S, "D": spec.D},
        "cpu_baseline": {"value": value, "unit": "latent frames/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "latent frames/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# Our arm: the CUDA library through its C ABI
# ----------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    import linear_attention_video_frame_b200 as la

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    wname, mode = WORKLOADS[args.workload]
    base = synth.workload(wname)
    if args.frames:
        base = base.with_(F=args.frames, name=f"{base.name}_clip{args.frames}")
    spec = rank_spec(base, rank)   # own data per rank
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    tdt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    dtc = la.LA_BF16 if spec.dtype == "bf16" else la.LA_F32

    # ---- inputs resident in HBM (pinned host copies kept for the e2e leg) ----
    host = {}
    dev_in = {}
    for name in ("q", "k", "v"):
        h = torch.empty((B, H, F, S, D), dtype=tdt, pin_memory=True)
        hv = h.view(torch.int16) if spec.dtype == "bf16" else h

        def put(b, hh, arr, hv=hv):
            hv[b, hh].copy_(torch.from_numpy(arr.view(np.int16) if arr.dtype == np.uint16
                                             else arr))

        synth.for_each_slice(spec, name, put)
        host[name] = h
        dev_in[name] = h.to(dev)
    a, bt = synth.gates(spec)
    host["alpha"] = torch.from_numpy(a).pin_memory()
    host["beta"] = torch.from_numpy(bt).pin_memory()
    dev_in["alpha"] = host["alpha"].to(dev)
    dev_in["beta"] = host["beta"].to(dev)
    o = torch.empty_like(dev_in["q"])
    state = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    z = torch.empty((B, H, D), dtype=torch.float32, device=dev)
    plan = step_plan(spec, mode)
    mode_c = {"gdn": la.LA_MODE_GDN, "relu": la.LA_MODE_RELU,
              "gdn_reverse": la.LA_MODE_GDN_REVERSE,
              "gdn_token_beta": la.LA_MODE_GDN_TOKEN_BETA,
              "gdn_prep": la.LA_MODE_GDN_PREP}[mode]
    prep = None
    if mode == "gdn_prep":
        prep_w = [torch.from_numpy(synth.norm_weights(spec, n)).to(dev) for n in ("q", "k")]
        prep = la.make_prep(prep_w[0], prep_w[1], PREP_NORM_EPS, True, spec.grid)
    if mode == "gdn_token_beta":
        host["beta"] = torch.from_numpy(synth.token_gates(spec)).pin_memory()
        dev_in["beta"] = host["beta"].to(dev)
    ws = la.workspace_for(mode_c,
                          B, H, max(n for _, n, _ in plan), S, D, dev)
    views = []
    for f0, n, si in plan:
        if len(plan) == 1:
            views.append((dev_in["q"], dev_in["k"], dev_in["v"], dev_in["alpha"],
                          dev_in["beta"], o, si))
        else:   # chunked streaming: contiguous per-chunk copies, made once
            sl = slice(f0, f0 + n)
            views.append(tuple(dev_in[x][:, :, sl].contiguous()
                               for x in ("q", "k", "v", "alpha", "beta")) +
                         (torch.empty((B, H, n, S, D), dtype=tdt, device=dev), si))
    stream = torch.cuda.current_stream()

    def one_step():
        for (q, k, v, al, be, oo, si) in views:
            if mode == "gdn_token_beta":
                la.la_scan_gdn_token_beta(q, k, v, al, be, spec.k_scale, o=oo, state_out=state,
                                          workspace=ws, stream=stream)
            elif mode == "gdn_prep":
                la.la_scan_gdn_prep(q, k, v, al, be, spec.k_scale, prep, o=oo, state_out=state,
                                    workspace=ws, stream=stream)
            elif mode == "gdn_reverse":
                la.la_scan_gdn_reverse(q, k, v, al, be, spec.k_scale, REVERSE_CHUNK, o=oo,
                                       workspace=ws, stream=stream)
            elif mode == "gdn":
                la.la_scan_gdn(q, k, v, al, be, spec.k_scale, o=oo,
                               state_in=state if si else None, state_out=state,
                               workspace=ws, stream=stream)
            else:
                la.la_scan_relu(q, k, v, o=oo, state_in=state if si else None,
                                z_in=z if si else None, state_out=state, z_out=z,
                                eps=spec.eps, workspace=ws, stream=stream)

    path, kernels_per_call = la.la_plan(mode_c,
                                        dtc, B, H, plan[0][1], S, D)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- warm-up ----
    for _ in range(max(args.warmup, 0)):
        one_step()
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps ----
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for i in range(K):
        evs[i][0].record(stream)
        one_step()
        evs[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    barrier()
    t_local = t0.elapsed_time(t1) / 1e3
    call_ms = [s.elapsed_time(e) / len(plan) for s, e in evs]
    t_max = max_over_ranks(t_local, dev)

    # ---- optional: sustained back-to-back calls, binned by block, beside the
    # SM clock sampled during each block (does a slowdown track the clock?) ----
    drift = None
    if args.drift_blocks > 0:
        dclk = ClockSampler(local)
        dclk.start()
        drift = []
        for blk in range(args.drift_blocks):
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            h0 = time.perf_counter()
            d0.record(stream)
            for _ in range(args.drift_calls):
                one_step()
            d1.record(stream)
            d1.synchronize()
            h1 = time.perf_counter()
            ms = d0.elapsed_time(d1) / (args.drift_calls * len(plan))
            mhz = dclk.between(h0, h1)
            med = statistics.median(mhz) if mhz else None
            drift.append({"block": blk, "calls": args.drift_calls, "ms_per_call": ms,
                          "sm_mhz_median": med, "sm_mhz_min": min(mhz) if mhz else None,
                          "samples": len(mhz), "ms_x_ghz": ms * med / 1e3 if med else None,
                          "reasons": dclk.reasons_between(h0, h1)})
        dclk.stop()
        barrier()

    byts, flops = step_counts(spec, mode)
    frames_all = B * F * K * world
    value = frames_all / t_max
    ms_per_step = 1e3 * t_max / K
    tflops = flops * K * world / t_max / 1e12

    # ---- e2e: the C-ABI host-buffer call (la_scan_host): H2D of the inputs, the
    # scan and D2H of the output and final state all inside the timed region,
    # pipelined chunk by chunk over the library's copy streams ----
    Ke = max(3, min(K, 10))
    chunk = spec.chunk_frames or 0
    o_host = torch.empty_like(host["q"], pin_memory=True)
    so_host = torch.empty((B, H, D, D), dtype=torch.float32, pin_memory=True)
    zo_host = torch.empty((B, H, D), dtype=torch.float32, pin_memory=True) \
        if mode == "relu" else None
    ins = ("q", "k", "v") if mode == "relu" else ("q", "k", "v", "alpha", "beta")
    if mode == "gdn_reverse":
        so_host = None          # the reversed scan has no state out
    special = mode in ("gdn_reverse", "gdn_token_beta", "gdn_prep")
    h2d = sum(host[x].numel() * host[x].element_size() for x in ins)
    d2h = sum(t.numel() * t.element_size() for t in (o_host, so_host, zo_host) if t is not None)
    e2e_call = "la_scan_host"
    if special:
        # no host-buffer form of these calls: H2D, the call and D2H in order
        # on one stream
        e2e_call = f"H2D + la_scan_{mode} + D2H"
        hws = None

        def e2e_step():
            for x in ins:
                dev_in[x].copy_(host[x], non_blocking=True)
            if mode == "gdn_reverse":
                la.la_scan_gdn_reverse(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["alpha"],
                                       dev_in["beta"], spec.k_scale, REVERSE_CHUNK, o=o,
                                       workspace=ws, stream=stream)
            elif mode == "gdn_prep":
                la.la_scan_gdn_prep(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["alpha"],
                                    dev_in["beta"], spec.k_scale, prep, o=o, state_out=state,
                                    workspace=ws, stream=stream)
                so_host.copy_(state, non_blocking=True)
            else:
                la.la_scan_gdn_token_beta(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["alpha"],
                                          dev_in["beta"], spec.k_scale, o=o, state_out=state,
                                          workspace=ws, stream=stream)
                so_host.copy_(state, non_blocking=True)
            o_host.copy_(o, non_blocking=True)
    else:
        hws = None if args.no_e2e else la.host_workspace_for(mode_c, dtc, B, H, F, S, D, chunk,
                                                             dev)

        def e2e_step():
            la.la_scan_host(mode_c, host["q"], host["k"], host["v"], o=o_host,
                            alpha=host["alpha"] if mode == "gdn" else None,
                            beta=host["beta"] if mode == "gdn" else None,
                            k_scale=spec.k_scale, eps=spec.eps, state_out=so_host, z_out=zo_host,
                            chunk_frames=chunk, workspace=hws, stream=stream)

    e2e_value = None
    if not args.no_e2e:
        e2e_step()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(Ke):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        te = max_over_ranks(e0.elapsed_time(e1) / 1e3, dev)
        e2e_value = B * F * Ke * world / te
    status = la.la_query_device_status(ws)
    if status == la.LA_OK and hws is not None:
        status = la.la_query_device_status(hws)

    # ---- roofline of the dominant kernel ----
    peaks, peak_src = load_peaks()
    kern_s = statistics.mean(call_ms) / 1e3
    per_call_bytes = byts / len(plan)
    achieved = per_call_bytes / kern_s / 1e9
    traffic = traffic_record(args.workload)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": f"{peak_src} (hbm_gbs, STREAM-style copy)",
                "kernel": path, "kernel_ms": kern_s * 1e3,
                "kernel_ms_min": min(call_ms), "kernel_ms_median": statistics.median(call_ms),
                "kernel_ms_max": max(call_ms),
                "alg_bytes_per_launch": per_call_bytes,
                "tensor_tflops_achieved": flops / len(plan) / kern_s / 1e12,
                "tensor_frac_of_bf16_peak": flops / len(plan) / kern_s / 1e12 /
                peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, t, sample = time_oracle_sample(base, mode, args.cpu_budget)
        cpu = {"value": v, "unit": "latent frames/s", "cores": oracle_threads(),
               "kind": "oracle", "sample": sample, "seconds": t}

    line = {
        "metric": METRIC, "value": value, "unit": "latent frames/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if spec.dtype == "bf16" else "f32",
        "data": "synthetic (seeded numpy PCG64, bf16 round-to-nearest-even)",
        "config": {"workload": workload_label(base.name, mode),
                   "mode": mode, "B": B, "H": H, "F": F, "S": S, "D": D,
                   "calls_per_step": len(plan), "global_batch": B * world,
                   "l2": "inputs larger than L2 (no flush)",
                   "parallelism": f"replicas x{world} (no data-path collective)"},
        "tflops": tflops,
        "gpu_launches": kernels_per_call * len(plan) * K,
        "kernel_path": path,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "latent frames/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke, "call": e2e_call,
                "chunk_frames": (la.la_host_chunk_frames(F, chunk) if not special else None),
                "host_memory": "pinned"},
        "clocks": clocks.summary(),
        "device_status": la.la_status_string(status),
    }
    if drift is not None:
        line["drift"] = drift
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def relaunch_ranks(n: int) -> int:
    """Run this same command as n ranks (one process per GPU) under torchrun
    on this node; rank 0 prints the JSON line.  Returns torchrun's status."""
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle work for the cpu_baseline field")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end leg (profiling runs)")
    ap.add_argument("--frames", type=int, default=0,
                    help="profiling only: a shorter clip (this many latent frames) of the workload")
    ap.add_argument("--drift-blocks", type=int, default=0,
                    help="analysis: after the timed steps, run this many blocks of back-to-back "
                         "calls and report each block's ms per call beside the SM clock "
                         "sampled during it")
    ap.add_argument("--drift-calls", type=int, default=50, help="calls per drift block")
    args = ap.parse_args()
    # N ranks, one per GPU: launched here unless torchrun already did
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        return relaunch_ranks(args.gpus)
    if int(world_env or 1) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world_env}", file=sys.stderr)
        return 2
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
