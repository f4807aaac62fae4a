#!/usr/bin/env python
"""Benchmark: forward pass of one MoE layer on B200, tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference] [--no-cpu-baseline]

One step = route -> dispatch -> experts -> combine over one batch of the
workload (default: the 64-expert builder layer, T=4096, H=4096, top-2,
I=1408, bf16, Zipf(1.0)-skewed load), with inputs resident in HBM.  L2 is
flushed before every timed step, outside the timed events: a 256 MiB write,
then a read of the same buffer, so that the timed step does not start by
writing back a cache full of dirty lines.
Each stage is bracketed by CUDA events on the launching stream, so the
per-stage times and the grouped-GEMM roofline come from the same timed
steps.  N > 1 (torchrun, one rank per GPU) runs independent replicas of the
layer, each on its own token batch (weak scaling; the layer has no exchange
step on one GPU's worth of experts), timed as the max over ranks.

Prints ONE JSON line on rank 0.  At N = 1 the line also carries a
``workloads`` object: every full-size workload (the builder layer, the
Qwen1.5-MoE-A2.7B shape at T = 32 and 8192, the Qwen3-30B-A3B shape at
T = 16384, the large-expert decode layer at T = 1, 8, 64) timed the same way,
each with its stage split, its layer roofline and its grouped-GEMM roofline
against the measured and the nominal peaks (``--headline-only`` skips them).
``--impl reference`` times the fp64 CPU oracle instead (a bounded token
sample per step; rank 0 only).

Roofline of the grouped GEMM (``roofline``): its algorithmic bytes are the
weights of the experts that received tokens (plus a shared expert's); its
flops 2*N*3*H*I (+ the shared expert's).  The packed intermediates it also
moves (x_packed, h, y_packed) are reported beside it
(``bytes_incl_packed``, ``frac_incl_packed``), not in ``frac``.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import CONFIGS, make_layer, make_tokens  # noqa: E402

METRIC = "MoE-layer tokens/s on 1xB200; % of HBM or bf16 tensor roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
CPU_SAMPLE_TOKENS = 1024
CPU_MIN_SECONDS = 10.0    # repeat the oracle sample until this much CPU time
CPU_MAX_RUNS = 200
REF_SAMPLE_TOKENS = 256


# ------------------------------------------------------------- helpers ---

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (6.65 TB/s, 1.59 PFLOP/s earlier pool measurement)"


NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}   # B200 nominal HBM3e and dense bf16


def expert_weight_work(cfg, counts):
    """Algorithmic bytes and flops of the grouped-GEMM stage (both passes):
    the weights of every expert with >= 1 row (w13 and w2), plus the shared
    expert's; flops 2*N*3*H*I (+ 2*T*3*H*I_s).  The packed intermediates
    (x_packed, h, y_packed) are not algorithmic and are not counted."""
    es = 2 if cfg.dtype == "bf16" else 4
    active = sum(1 for c in counts if c > 0)
    N = int(sum(counts))
    H, I = cfg.H, cfg.I
    wbytes = active * 3 * H * I * es
    flops = 2 * N * 3 * H * I
    if cfg.shared_I:
        wbytes += 3 * H * cfg.shared_I * es
        flops += 2 * cfg.T * 3 * H * cfg.shared_I
    return wbytes, flops


def expert_stage_work(cfg, counts):
    """The same stage's bytes INCLUDING the materialised intermediates (x_packed
    read, h written and read back, y_packed written -- 2 bytes per element
    (fp16) in bf16 layers, as the layer stores it --, routing weights; with a
    shared expert also its x read, h_s written and read, output written), and
    its flops."""
    es = 2 if cfg.dtype == "bf16" else 4
    N = int(sum(counts))
    H, I = cfg.H, cfg.I
    wbytes, flops = expert_weight_work(cfg, counts)
    abytes = N * H * es + 2 * N * I * es + N * H * es + N * 4
    if cfg.shared_I:
        abytes += cfg.T * H * es + 2 * cfg.T * cfg.shared_I * es + cfg.T * H * es
    return wbytes + abytes, flops


def layer_work(cfg, counts):
    """Algorithmic bytes / flops of the whole layer: activated expert weights,
    router weights, x in, out out (the materialised packed intermediates are
    not counted); flops of the router and the activated experts."""
    es = 2 if cfg.dtype == "bf16" else 4
    active = sum(1 for c in counts if c > 0)
    H, I, E, T = cfg.H, cfg.I, cfg.E, cfg.T
    b = active * 3 * H * I * es + E * H * es + 2 * T * H * es
    f = 2 * T * cfg.k * 3 * H * I + 2 * T * H * E
    if cfg.shared_I:
        b += 3 * H * cfg.shared_I * es + H * es
        f += 2 * T * 3 * H * cfg.shared_I + 2 * T * H
    return b, f


def gemm_roofline(cfg, counts, t_ms, peaks):
    """Roofline of the grouped-GEMM stage over the live stage time t_ms:
    bound "tensor" when its flops per algorithmic byte reach the measured
    ridge, else "hbm"; fractions of the measured peaks and of the nominal
    ones; the intermediates-inclusive byte rate beside it."""
    wb, fl = expert_weight_work(cfg, counts)
    ib, _ = expert_stage_work(cfg, counts)
    t = t_ms / 1e3
    hbm, tf = peaks["hbm_gbs"], peaks["bf16_tflops"]
    if fl / wb >= tf * 1e12 / (hbm * 1e9):
        r = {"bound": "tensor", "achieved": fl / t / 1e12, "peak": tf, "unit": "TFLOP/s"}
        r["frac_nominal"] = r["achieved"] / NOMINAL["bf16_tflops"]
    else:
        r = {"bound": "hbm", "achieved": wb / t / 1e9, "peak": hbm, "unit": "GB/s"}
        r["frac_nominal"] = r["achieved"] / NOMINAL["hbm_gbs"]
    r["frac"] = r["achieved"] / r["peak"]
    r["bytes_alg"] = wb
    r["flops"] = fl
    r["bytes_incl_packed"] = ib
    r["gbs_incl_packed"] = ib / t / 1e9
    r["frac_incl_packed"] = r["gbs_incl_packed"] / hbm
    return r


def layer_roofline(cfg, counts, ms, peaks):
    """t_roof = max(layer bytes / HBM, layer flops / bf16 peak) against the
    measured step time, for the measured and for the nominal peaks."""
    lb, lf = layer_work(cfg, counts)
    out = {"bytes": lb, "flops": lf}
    for tag, pk in (("", peaks), ("_nominal", NOMINAL)):
        tb = lb / (pk["hbm_gbs"] * 1e9)
        tfl = lf / (pk["bf16_tflops"] * 1e12)
        out["bound" + tag] = "hbm" if tb >= tfl else "tensor"
        out["t_roof_ms" + tag] = max(tb, tfl) * 1e3
        out["frac" + tag] = max(tb, tfl) / (ms / 1e3)
    return out


def zipf_slope(counts):
    """Least-squares slope of log(count) against log(rank) over the experts
    that received tokens (rank 1 = the most loaded): the realised skew."""
    import math
    c = sorted((x for x in counts if x > 0), reverse=True)
    if len(c) < 2:
        return None
    xs = [math.log(r) for r in range(1, len(c) + 1)]
    ys = [math.log(v) for v in c]
    mx, my = sum(xs) / len(xs), sum(ys) / len(ys)
    sxx = sum((a - mx) ** 2 for a in xs)
    return sum((a - mx) * (b - my) for a, b in zip(xs, ys)) / sxx


def strip_comments(src: str) -> str:
    """C/C++ source without comments and without whitespace runs (string
    literals in these files hold no comment markers)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash():
    """Hash of the grouped GEMM's code (comments and layout ignored, so that
    a comment edit does not discard counters taken on the same code)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixture_experts_layer_44_b200", "csrc")
    for name in ("experts_tc.cu", "sm100_ptx.cuh", "common.cuh"):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            src = f.read()
        if name == "common.cuh":
            # only its device helpers (namespace moe) reach the kernel; the
            # host launcher declarations after them do not
            src = src[:src.index("namespace moe_host {")]
        h.update(strip_comments(src).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """Per-launch DRAM bytes of the grouped GEMM from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "grouped_gemm_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_sha") != kernel_source_hash():
        return None
    return d.get("per_step_bytes", {}).get(workload)


def max_over_ranks(value: float, device) -> float:
    """The largest ``value`` over all ranks (torch.distributed MAX all-reduce);
    the value itself when no process group is initialised."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(cfg, rank: int) -> dict:
    """One replica's layer: the same seeded weights on every rank, and the
    workload's own tokens on rank 0, a fresh seeded batch on rank r > 0."""
    p = make_layer(cfg, seed=0)
    if rank > 0:
        p["x"] = make_tokens(cfg, seed=rank)
    return p


def parse_clock_samples(text: str) -> dict:
    """Median SM clock, max clock and the throttle reasons seen in
    ``nvidia-smi --query-gpu=...`` CSV rows (the ClockSampler query)."""
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in text.strip().splitlines():
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            smax.append(float(f[2]))
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons), "samples": len(sm)}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while timing."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        props = torch.cuda.get_device_properties(device_index)
        self.bus = None
        try:
            self.bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        except AttributeError:
            pass

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.bus:
            cmd += ["-i", self.bus]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop_raw(self) -> str:
        """Stop sampling; the CSV rows seen ("" without nvidia-smi)."""
        if self.proc is None:
            return ""
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.proc = None
        return out

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        return parse_clock_samples(self.stop_raw())


# ---------------------------------------------------------- CPU oracle ---

def oracle_sample_run(cfg, p, ntok):
    """The fp64 oracle, as it stands, on the first ``ntok`` tokens of the
    workload (full router, dispatch, experts, merge for that sample)."""
    import oracle.moe_oracle as O
    sub = dict(p)
    sub["x"] = p["x"][:ntok]
    t0 = time.perf_counter()
    O.moe_forward(sub, cfg.k, cfg.renormalize)
    return time.perf_counter() - t0


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    p = make_layer(cfg, seed=0)
    ntok = min(REF_SAMPLE_TOKENS, cfg.T)
    for _ in range(args.warmup):
        oracle_sample_run(cfg, p, ntok)
    times = [oracle_sample_run(cfg, p, ntok) for _ in range(args.steps)]
    total = sum(times)
    value = ntok * args.steps / total
    sample = (f"first {ntok} of the workload's {cfg.T} tokens per step (fp64 numpy oracle: "
              f"router, dispatch, experts, merge), {args.steps} steps after {args.warmup} warm-up")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, None),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(cfg, counts):
    c = {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "top_k": cfg.k, "I": cfg.I,
         "renormalize": cfg.renormalize, "zipf_s": cfg.zipf_s, "empty_experts_forced": cfg.empty_tail,
         "shared_I": cfg.shared_I, "seed": 0, "l2": "flushed before every timed step: 256 MiB write, then read back",
         "parallelism": "replicas (one independent layer per GPU)"}
    if counts is not None:
        c["expert_counts"] = [int(x) for x in counts]
    return c


# ------------------------------------------------------------ GPU path ---

FULL_WORKLOADS = ["builder_bf16", "qwen15_t32", "qwen15_t8192", "qwen3_t16384", "decode_t1",
                  "decode_t8", "decode_t64"]


class Layer:
    """One layer instance on the device with its buffers, and its step."""

    def __init__(self, M, cfg, rank, dev, stream):
        self.M, self.cfg, self.stream = M, cfg, stream
        self.p = rank_inputs(cfg, rank)
        self.dp = {k: (v.to(dev) if v is not None else None) for k, v in self.p.items()}
        self.buf = M.MoELayerBuffers(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.torch_dtype,
                                     device=dev, shared_I=cfg.shared_I)

    def step(self, ev=None):
        # Each stage's events are recorded on the stream its kernels run on.
        M, cfg, buf, dp, stream = self.M, self.cfg, self.buf, self.dp, self.stream
        x = dp["x"]
        shared = cfg.shared_I is not None
        if ev:
            ev[0].record(stream)
        gate_done = False
        if buf.route_dispatch:
            # decode batches: router (with a shared expert's gate) and dispatcher are one
            # launch (timed as "route")
            gate_done = M.route_and_dispatch(x, dp, cfg.k, cfg.renormalize, buf, stream)
            if ev:
                ev[1].record(stream)
        elif shared:
            # the shared expert's gate logit comes out of the router's launch
            M.moe_route_gated(x, dp["W_gate"], dp["bias"], dp["w_sg"], cfg.k, cfg.renormalize,
                              buf.logits, buf.ids, buf.w, buf.sg_logit, status=buf.status,
                              stream=stream)
            gate_done = True
            if ev:
                ev[1].record(stream)
            M.moe_dispatch(buf.ids, buf.w, x, cfg.E, buf.counts, buf.offsets, buf.perm,
                           buf.inv_perm, buf.packed_tok, buf.packed_w, buf.x_packed, buf.ws,
                           buf.status, stream=stream)
        else:
            M.moe_route(x, dp["W_gate"], dp["bias"], cfg.k, cfg.renormalize, buf.logits,
                        buf.ids, buf.w, status=buf.status, stream=stream)
            if ev:
                ev[1].record(stream)
            M.moe_dispatch(buf.ids, buf.w, x, cfg.E, buf.counts, buf.offsets, buf.perm,
                           buf.inv_perm, buf.packed_tok, buf.packed_w, buf.x_packed, buf.ws,
                           buf.status, stream=stream)
        if ev:
            ev[2].record(stream)
        if not shared:
            M.moe_experts(buf.x_packed, buf.offsets, buf.packed_w, dp["w13"], dp["w2"], buf.h,
                          buf.y_packed, ws=buf.ws_experts, status=buf.status, stream=stream)
        else:
            if not gate_done:
                M.moe_route(x, dp["w_sg"].view(1, -1), None, 0, False, buf.sg_logit,
                            status=buf.status, stream=stream)
            if buf.fuse_shared:
                M.moe_experts_shared(buf.x_packed, buf.offsets, buf.packed_w, dp["w13"],
                                     dp["w2"], buf.h, buf.y_packed, x, dp["w13s"], dp["w2s"],
                                     buf.sh_h, buf.sh_y, ws=buf.ws_experts, status=buf.status,
                                     stream=stream)
            else:
                M.moe_experts(buf.x_packed, buf.offsets, buf.packed_w, dp["w13"], dp["w2"],
                              buf.h, buf.y_packed, ws=buf.ws_experts, status=buf.status,
                              stream=stream)
                M.moe_experts(x, buf.sh_offsets, None, dp["w13s"].unsqueeze(0),
                              dp["w2s"].unsqueeze(0), buf.sh_h, buf.sh_y, ws=buf.ws_experts,
                              status=buf.status, stream=stream)
        if ev:
            ev[3].record(stream)
        M.moe_combine(buf.y_packed, buf.inv_perm, cfg.T, cfg.k, buf.out,
                      buf.sh_y if shared else None, buf.sg_logit if shared else None,
                      status=buf.status, stream=stream)
        if ev:
            ev[4].record(stream)


def time_layer(layer, steps, warmup, flush, dev, dist=None, clocks=None):
    """Warm up, then time ``steps`` steps (one event pair each, L2 flushed
    before every step, outside the events), then a second pass with an event
    between stages.  Returns (mean ms per step, mean ms per stage, library
    kernels launched in the timed steps, raw clock samples or None)."""
    M, stream = layer.M, layer.stream

    def flush_l2():
        flush.zero_()                 # write > L2 ...
        flush.sum()                   # ... then read it, leaving clean lines only

    for _ in range(warmup):
        flush_l2()
        layer.step()
    torch.cuda.synchronize(dev)
    if int(layer.buf.status.item()) != 0:
        raise SystemExit(f"device status {int(layer.buf.status.item())} after warm-up "
                         f"({layer.cfg.name})")
    # Steps are enqueued in groups behind a short GPU spin (outside every
    # bracket), so the GPU runs each group back to back and no bracket
    # contains time spent waiting for the host.  Events between small kernels
    # cost a few microseconds each, so the step time comes from the first pass.
    GROUP = 8
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.start()
        time.sleep(0.3)
    launches0 = M.moe_launch_count()
    for g0 in range(0, steps, GROUP):
        torch.cuda._sleep(int(20e6))            # ~10 ms of GPU spin while the host enqueues
        for i in range(g0, min(steps, g0 + GROUP)):
            flush_l2()
            step_ev[i][0].record(stream)
            layer.step()
            step_ev[i][1].record(stream)
    launches = M.moe_launch_count() - launches0     # this library's kernels in the timed steps
    torch.cuda.synchronize(dev)
    raw = clocks.stop_raw() if clocks else None
    if dist:
        dist.barrier()
    ms = sum(a.elapsed_time(b) for a, b in step_ev) / steps
    for g0 in range(0, steps, GROUP):
        torch.cuda._sleep(int(20e6))
        for i in range(g0, min(steps, g0 + GROUP)):
            flush_l2()
            layer.step(evs[i])
    torch.cuda.synchronize(dev)
    stage_ms = [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(steps)]
    per_stage = [sum(s[j] for s in stage_ms) / steps for j in range(4)]
    if int(layer.buf.status.item()) != 0:
        raise SystemExit(f"device status {int(layer.buf.status.item())} after timing "
                         f"({layer.cfg.name})")
    return ms, per_stage, launches, raw


def stage_dict(per_stage, fused_route_dispatch=False):
    if fused_route_dispatch:    # one launch routes and dispatches decode batches
        return {"route_dispatch": per_stage[0] + per_stage[1], "experts": per_stage[2],
                "combine": per_stage[3]}
    return {"route": per_stage[0], "dispatch": per_stage[1], "experts": per_stage[2],
            "combine": per_stage[3]}


def route_dispatch_fits(cfg):
    """Mirror of the library's rule for the one-launch router + dispatcher."""
    return 1 <= cfg.T <= 64 and 1 <= cfg.E <= 64 and cfg.H <= 32768 and 1 <= cfg.k <= min(cfg.E, 8)


def workload_summary(cfg, counts, ms, per_stage, launches, steps, peaks):
    """One entry of the line's ``workloads`` object."""
    return {"ms_per_step": ms, "tokens_per_s": cfg.T / (ms / 1e3), "T": cfg.T,
            "stage_ms": stage_dict(per_stage, route_dispatch_fits(cfg)),
            "layer_roofline": layer_roofline(cfg, counts, ms, peaks),
            "gemm_roofline": dict(gemm_roofline(cfg, counts, per_stage[2], peaks),
                                  traffic=ncu_traffic(cfg.name)),
            "active_experts": sum(1 for c in counts if c > 0), "max_expert_rows": max(counts),
            "zipf_slope_realised": zipf_slope(counts) if cfg.zipf_s is not None else None,
            "gpu_launches_per_step": launches / steps}


def run_gpu(args, cfg):
    import mixture_experts_layer_44_b200 as M

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    M.load_library()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, peak_src = load_peaks()

    layer = Layer(M, cfg, rank, dev, stream)
    clocks = ClockSampler(local)
    ms, per_stage, gpu_launches, raw_clocks = time_layer(layer, args.steps, args.warmup, flush,
                                                         dev, dist, clocks)
    counts = layer.buf.counts.cpu().tolist()
    ms_max = max_over_ranks(ms, dev)
    p, dp, buf = layer.p, layer.dp, layer.buf

    # End to end through the C ABI with host buffers (moe_layer_forward_host):
    # every step uploads its own pinned batch and downloads its output, and
    # consecutive steps overlap (upload / layer / download on three streams).
    # No L2 flush here: every workload's expert weights alone exceed L2.
    e2e_layer = M.MoELayer(dp, cfg.T, cfg.k, cfg.renormalize, stream=stream)
    x_hosts = [p["x"].pin_memory(), make_tokens(cfg, seed=1000 + rank).pin_memory()]
    out_hosts = [torch.empty(cfg.T, cfg.H, dtype=cfg.torch_dtype).pin_memory() for _ in range(2)]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, args.steps)
    for i in range(3):
        e2e_layer.forward_host(x_hosts[i % 2], out_hosts[i % 2], stream=stream)
    e2e_layer.join(stream)
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    e_start.record(stream)
    for i in range(e2e_steps):
        e2e_layer.forward_host(x_hosts[i % 2], out_hosts[i % 2], stream=stream)
    e2e_layer.join(stream)
    e_end.record(stream)
    e_end.synchronize()
    e2e_ms = e_start.elapsed_time(e_end) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)
    if e2e_layer.status(stream) != 0:
        raise SystemExit("device status set in the end-to-end steps")
    e2e_layer.close()
    if int(buf.status.item()) != 0:
        raise SystemExit(f"device status {int(buf.status.item())} after timing")
    del layer, dp, buf

    # Every other full-size workload, one at a time, at N = 1 (the same timing).
    workloads = {}
    if cfg.name in FULL_WORKLOADS:
        workloads[cfg.name] = workload_summary(cfg, counts, ms, per_stage, gpu_launches,
                                               args.steps, peaks)
    clock_raw = [raw_clocks] if raw_clocks else []
    if world == 1 and args.all_workloads:
        for name in FULL_WORKLOADS:
            if name == cfg.name:
                continue
            wcfg = CONFIGS[name]
            wl = Layer(M, wcfg, rank, dev, stream)
            wms, wst, wla, wraw = time_layer(wl, args.steps, max(3, min(args.warmup, 5)), flush,
                                             dev, None, clocks)
            if wraw:
                clock_raw.append(wraw)
            workloads[name] = workload_summary(wcfg, wl.buf.counts.cpu().tolist(), wms, wst,
                                               wla, args.steps, peaks)
            del wl
            torch.cuda.empty_cache()

    if rank == 0:
        roof = gemm_roofline(cfg, counts, per_stage[2], peaks)
        roof["traffic"] = ncu_traffic(cfg.name)
        roof["kernel"] = ("grouped_gemm_kernel (tcgen05), both passes of moe_experts: "
                          f"{roof['bytes_alg']/1e9:.3f} GB of activated expert weights and "
                          f"{roof['flops']/1e9:.1f} GFLOP per step")
        roof["peak_source"] = peak_src + ", burst figures (each step lasts under 2 ms)"
        cpu = None
        if not args.no_cpu_baseline:
            ntok = min(CPU_SAMPLE_TOKENS, cfg.T)
            secs, runs = 0.0, 0
            while runs < CPU_MAX_RUNS and (runs == 0 or secs < CPU_MIN_SECONDS):
                secs += oracle_sample_run(cfg, p, ntok)
                runs += 1
            cpu = {"value": ntok * runs / secs, "unit": UNIT, "cores": cpu_cores(),
                   "kind": "oracle",
                   "sample": f"first {ntok} of {cfg.T} tokens, fp64 numpy oracle (router, "
                             f"dispatch, experts, merge), {runs} run(s), {secs:.1f} s"}
        es = 2 if cfg.dtype == "bf16" else 4
        wcfg = workload_config(cfg, counts)
        wcfg["zipf_slope_realised"] = zipf_slope(counts) if cfg.zipf_s is not None else None
        clock_info = parse_clock_samples("\n".join(clock_raw)) if clock_raw else \
            {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        line = {
            "metric": METRIC, "value": cfg.T * world / (ms_max / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) weights)",
            "config": wcfg,
            "roofline": roof,
            "layer_roofline": layer_roofline(cfg, counts, ms, peaks),
            "stage_ms": stage_dict(per_stage, route_dispatch_fits(cfg)),
            "cpu_baseline": cpu,
            "e2e": {"value": cfg.T * world / (e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": cfg.T * cfg.H * es,
                    "d2h_bytes_per_step": cfg.T * cfg.H * es, "ms_per_step": e2e_ms,
                    "api": "moe_layer_forward_host (C ABI): pinned host x in, out back, "
                           "consecutive steps overlapped on three streams"},
            "gpu_launches": gpu_launches,
            "clocks": clock_info,
            "gpu": torch.cuda.get_device_name(dev),
            "workloads": workloads,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="builder_bf16", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", dest="all_workloads", action="store_false",
                    help="skip the other full-size workloads (the line's `workloads` object); "
                         "they are measured by default at N = 1")
    ap.add_argument("--profile-small", action="store_true",
                    help="the workload with E=16 experts and T=1024 tokens (weights 0.55 GB, "
                         "still above L2): the case detailed ncu captures run on")
    ap.add_argument("--profile-shape", type=int, nargs=2, metavar=("E", "T"),
                    help="the workload with at most E experts and T tokens (a mid-size case "
                         "for detailed ncu captures: a few GB on the device)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    cfg = CONFIGS[args.workload]
    if args.profile_small or args.profile_shape:
        import dataclasses
        pe, pt = args.profile_shape or (16, 1024)
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}_e{pe}_t{pt}", E=min(cfg.E, pe),
                                  T=min(cfg.T, pt))
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_gpu(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
