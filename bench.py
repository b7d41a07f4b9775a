"""Benchmark of the MoE layer with zero-computation experts (forward + expert-bias update) on B200.

One step = lc_moe_forward on one batch (router GEMM, softmax + biased top-K + histogram, grouping,
row gather, grouped SwiGLU GEMM, grouped down GEMM, combine) followed by the expert-bias update
(with an all-reduce of the 768 expert counts when several ranks run). Default workload: the
LongCat-Flash-shape prefill batch (T=16384 tokens per GPU, d=6144, 512 FFN experts of width 2048,
256 zero experts, K=12, K_e=8, Zipf(1.1) expert popularity), synthetic data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|decode|small|tiny|...] [--experts bf16|fp8]
    python bench.py --sweep ffn_rows|hist|ffn_subset|control   (one JSON line per case)

Prints one JSON line (rank 0). ``--impl reference`` times the CPU oracle (test infrastructure) on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import pathlib
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "MoE-layer tokens/sec on 1 B200; grouped-GEMM % BF16 TC peak; permute/combine HBM GB/s"
UNIT = "tokens/s"
# the stages of lc_moe_forward, in launch order; kernels per stage
STAGES = ("router_gemm", "topk", "permute", "gather", "gemm1_swiglu", "gemm2_down", "combine")
KERNELS_PER_STAGE = (1, 1, 3, 1, 1, 1, 1)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def workload_config(w, world: int, f8: bool) -> dict:
    """The `config` of both arms' JSON line for workload w on `world` ranks."""
    return {"workload": f"{w.name}: MoE layer with zero-computation experts, T={w.T} tokens per GPU",
            "T": w.T, "d": w.d, "N": w.N, "Z": w.Z, "K": w.K, "K_e": w.K_e, "I": w.I,
            "router": w.router, "mu": w.mu, "parallelism": f"dp{world}",
            "step": "forward + counts all-reduce (N>1) + expert-bias update",
            "experts": ("all expert projections on E4M3 codes with one fp32 scale per weight "
                        "row and per activation row (weights quantised once before timing)")
                       if f8 else "bf16",
            "l2": f"inputs larger than L2 ({w.weight_bytes() / 1e9:.1f} GB expert weights, "
                  f"{w.T * w.d * 2 / 1e6:.0f} MB x per step)"}


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clock sampler --

class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "enforced.power.limit")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for r in csv.reader(io.StringIO(pathlib.Path(self.path).read_text())):
            r = [c.strip() for c in r]
            if len(r) < 10:
                continue
            if self.uuid and self.uuid not in r[1]:
                continue
            rows.append(r)
        os.unlink(self.path)
        return rows

    @staticmethod
    def summarize(rows, window=None):
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        def num(v):
            try:
                return float(v)
            except ValueError:
                return float("nan")
        power = np.array([num(r[4]) for r in rows])
        sm = np.array([num(r[2]) for r in rows])
        loaded = power > 0.5 * np.nanmax(power) if np.isfinite(power).any() else np.ones(len(rows), bool)
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        limits = [num(r[10]) for r in rows if len(r) > 10]
        return {"sm_mhz": float(np.nanmedian(sm[loaded])) if loaded.any() else float(np.nanmedian(sm)),
                "sm_max_mhz": float(np.nanmax([num(r[3]) for r in rows])),
                "power_limit_w": float(np.nanmax(limits)) if limits else None,
                "power_w": float(np.nanmedian(power[loaded])) if loaded.any() else None,
                "reasons": sorted(reasons), "samples": int(len(rows)),
                "samples_under_load": int(loaded.sum())}


# ------------------------------------------------------------------------------- our arm ----

def traffic_record(key: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, if it was taken
    on the current kernel source."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    rec = json.loads(p.read_text()).get(key)
    if not rec:
        return None
    src = ROOT / "mixture_experts_zero_b200" / "csrc" / rec["source"]
    if not src.exists() or hashlib.sha256(src.read_bytes()).hexdigest()[:16] != rec["sha256_16"]:
        return None
    return rec


def gemm_phase_roofline(counts, d: int, I: int, f8: bool, mhz: dict, sm_count: int, hbm_gbs: float,
                        measured_ms: dict) -> dict:
    """Each expert GEMM split by the kind of tile its rows take: rows in 256-row tiles are tensor
    work at the SM clock measured inside the kernel (8192 bf16 / 16384 E4M3 FLOP per SM per
    cycle), the other rows' experts (cold experts, and the leftover rows of hot ones) are weight
    streams at the measured copy bandwidth; the bound runs the two kinds one after the other.
    Both GEMMs take row tiles from 128 rows (a 128..255-row remainder included). counts: rows
    per FFN expert."""
    out = {}
    wb = 1 if f8 else 2
    for name, cold, rem_rows, fl_per_row, w_bytes in (
            ("gemm1_swiglu", 128, 128, 4.0 * d * I, 2 * I * d * wb),
            ("gemm2_down", 128, 128, 2.0 * d * I, d * I * wb)):
        if not mhz.get(name):
            continue
        hot_rows = 0
        stream_bytes = 0
        for n in counts:
            n = int(n)
            if n == 0:
                continue
            if n < cold:
                stream_bytes += w_bytes
                continue
            nfull, rem = divmod(n, 256)
            hot_rows += nfull * 256 + (rem if rem >= rem_rows else 0)
            if 0 < rem < rem_rows:
                stream_bytes += w_bytes
        rate = sm_count * (16384 if f8 else 8192) * mhz[name] * 1e6
        t_hot = fl_per_row * hot_rows / rate
        t_stream = stream_bytes / (hbm_gbs * 1e9)
        out[name] = {"t_bound_ms": round((t_hot + t_stream) * 1e3, 4),
                     "frac": round((t_hot + t_stream) * 1e3 / measured_ms[name], 4),
                     "tensor_ms": round(t_hot * 1e3, 4), "stream_ms": round(t_stream * 1e3, 4),
                     "rows_in_row_tiles": hot_rows, "weight_stream_bytes": stream_bytes}
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    from mixture_experts_zero_b200 import binding as B
    from mixture_experts_zero_b200 import inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    w = inputs.WORKLOADS[args.workload]
    # weights identical on every rank (same seed); each rank draws its own tokens
    data = inputs.make(w, device=dev, grid=False, experts=True)
    if rank > 0:
        g = inputs.generator(w.seed * 1000 + rank, dev)
        data["x"] = inputs.draw_x(w, g, dev)
    x, wr, bias, w13, w2 = data["x"], data["wr"], data["bias"], data["w13"], data["w2"]
    bias = bias.clone()
    T, E, K = w.T, w.E, w.K
    shape = B.Shape(T, w.d, w.N, w.Z, K, w.I)
    f8 = args.experts == "fp8"
    if f8:
        # weights are quantised once, outside the timed region (an offline step for a deployment)
        w13q, w13s = B.lc_moe_quantize_e4m3(w13)
        w2q, w2s = B.lc_moe_quantize_e4m3(w2)
        torch.cuda.synchronize(dev)
    ws = B.new_workspace(shape, B.OP_FORWARD_FP8 if f8 else B.OP_FORWARD, dev)
    out = torch.empty(T, w.d, dtype=torch.bfloat16, device=dev)
    counts = torch.zeros(E, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    T_all = T * world

    def forward(xin, o, events=None):
        if f8:
            B.lc_moe_forward_fp8(xin, wr, bias, w13q, w13s, w2q, w2s, K, out=o, counts=counts, ws=ws,
                                 stream=stream, events=events)
        else:
            B.lc_moe_forward(xin, wr, bias, w13, w2, K, out=o, counts=counts, ws=ws, stream=stream,
                             events=events)

    def step(events=None, xin=x, o=out):
        forward(xin, o, events)
        if world > 1:
            dist.all_reduce(counts)
        B.lc_moe_bias_update(bias, counts, T_all, w.N, w.Z, K, w.K_e, w.mu, reset_counts=True,
                             stream=stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    # ---- device-resident timing
    for _ in range(args.warmup):
        step()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    for row in ev:  # create the events before the timed region
        for e in row:
            e.record(stream)
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    # the grouped GEMMs stamp the global timer and their SM's cycle counter at the start and end
    # of CTA 0 (the last timed step's launches remain): the SM clock inside each GEMM
    probe = torch.zeros(8, dtype=torch.int64, device=dev)
    B.lc_moe_set_clock_probe(probe)
    time.sleep(0.3)
    barrier()
    t_start.record(stream)
    for i in range(args.steps):
        step(events=ev[i])
    t_end.record(stream)
    barrier()
    B.lc_moe_set_clock_probe(None)
    clock_rows = sampler.stop()
    pr = probe.cpu().tolist()
    gemm_mhz = {name: (round((pr[o + 3] - pr[o + 1]) / (pr[o + 2] - pr[o]) * 1e3, 1) if pr[o + 2] > pr[o] else None)
                for name, o in (("gemm1_swiglu", 0), ("gemm2_down", 4))}
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    elapsed_ms = t_start.elapsed_time(t_end)
    stage_ms = np.array([[row[j].elapsed_time(row[j + 1]) for j in range(len(STAGES))] for row in ev])
    if B.lc_moe_read_status(ws, stream=stream, raise_on_error=False):
        raise SystemExit("device status bits set during the benchmark")
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    elapsed_ms = float(t.item())
    ms_per_step = elapsed_ms / args.steps
    value = T * world * args.steps / (elapsed_ms / 1e3)

    # routing statistics of this batch (one more untimed pass, counts not reset)
    counts.zero_()
    forward(x, out)
    c = counts.cpu().numpy().astype(np.int64)
    M = int(c[: w.N].sum())
    touched = int((c[: w.N] > 0).sum())

    # ---- end to end through the public API: every step copies its x from pinned host memory to
    # the device and its output back to pinned host memory. The copies run on a copy stream and
    # overlap the compute of the neighbouring steps (H2D of step i+1 and D2H of step i-1 during
    # step i), with double-buffered device x and out.
    x_host = x.cpu().pin_memory()
    out_host = [torch.empty(T, w.d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    out_dev = [torch.empty_like(out) for _ in range(2)]
    # one stream per copy direction, so that the input and output copies of neighbouring steps
    # also overlap each other (the two directions of the PCIe link)
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    fwd_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        with torch.cuda.stream(h2d):
            h2d.wait_stream(stream)  # earlier work on the buffers has finished
            x_dev[0].copy_(x_host, non_blocking=True)
            h2d_done[0].record(h2d)
        d2h.wait_stream(stream)
        for i in range(n):
            b = i & 1
            if i + 1 < n:
                with torch.cuda.stream(h2d):
                    if i >= 1:
                        h2d.wait_event(fwd_done[b ^ 1])  # step i-1 has finished reading x_dev[b^1]
                    x_dev[b ^ 1].copy_(x_host, non_blocking=True)
                    h2d_done[b ^ 1].record(h2d)
            stream.wait_event(h2d_done[b])
            if i >= 2:
                stream.wait_event(d2h_done[b])  # step i-2's output has left out_dev[b]
            step(xin=x_dev[b], o=out_dev[b])
            fwd_done[b].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(fwd_done[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                d2h_done[b].record(d2h)
        stream.wait_stream(h2d)
        stream.wait_stream(d2h)

    e2e_steps(max(2, args.warmup // 2))
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps_n = max(2, min(args.steps, 40))
    e0.record(stream)
    e2e_steps(e2e_steps_n)
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_ms = float(t.item())
    e2e_value = T * world * e2e_steps_n / (e2e_ms / 1e3)

    # ---- roofline of each stage (algorithmic work only)
    peaks, peak_src = load_peaks()
    d_, I_ = w.d, w.I
    # E4M3 expert weights take 1 byte per element
    wbytes_touched = touched * d_ * I_ * (3 if f8 else 6)
    # tensor peak of each contraction: bf16 measured; E4M3 = 2 x bf16 (nominal dense ratio 4.5/2.25)
    peak16 = peaks["bf16_tflops_sustained"]
    peak_g1 = 2.0 * peak16 if f8 else peak16
    alg = {
        "router_gemm": ("tensor", 2.0 * T * d_ * E),
        "topk": ("hbm", T * E * 4 + T * K * 8 + E * 4),
        "permute": ("hbm", 2 * T * K * 4 + M * 4 + T * K * 4),
        # bf16: x read, M rows written; E4M3: x read, codes written and read, M rows of d bytes
        "gather": ("hbm", T * d_ * 4 + M * d_ if f8 else T * d_ * 2 + M * d_ * 2),
        "gemm1_swiglu": ("tensor", 4.0 * M * d_ * I_),
        "gemm2_down": ("tensor", 2.0 * M * d_ * I_),
        "combine": ("hbm", M * d_ * 2 + 2 * T * d_ * 2 + T * K * 8),
    }
    med = np.median(stage_ms, axis=0)
    mean = np.mean(stage_ms, axis=0)
    # the grouping is one kernel for a batch of at most 256 tokens, three above
    n_kernels = sum(KERNELS_PER_STAGE) - (2 if T <= 256 else 0)
    stages = {}
    for j, name in enumerate(STAGES):
        bound, work = alg[name]
        t_s = mean[j] / 1e3
        if bound == "tensor":
            ach = work / t_s / 1e12
            peak = peak_g1 if name in ("gemm1_swiglu", "gemm2_down") else peaks["bf16_tflops_sustained"]
            unit = "TFLOP/s"
        else:
            ach = work / t_s / 1e9
            peak = peaks["hbm_gbs"]
            unit = "GB/s"
        stages[name] = {"ms": round(float(mean[j]), 4), "ms_median": round(float(med[j]), 4),
                        "share": round(float(mean[j] / mean.sum()), 4), "bound": bound,
                        "achieved": round(ach, 2), "unit": unit, "peak": peak,
                        "frac": round(ach / peak, 4), "algorithmic_work": work}
        if gemm_mhz.get(name):
            # the nominal dense tensor rate at the clock measured inside the kernel: 8192 bf16
            # (16384 E4M3) FLOP per SM per cycle
            rate = sm_count * (16384 if f8 else 8192) * gemm_mhz[name] * 1e6 / 1e12
            stages[name]["sm_mhz_in_kernel"] = gemm_mhz[name]
            stages[name]["frac_of_tensor_rate_at_that_clock"] = round(ach / rate, 4)
    dom = max(STAGES, key=lambda n: stages[n]["ms"])
    ds = stages[dom]
    trec = traffic_record(f"{w.name}/{dom}" + ("@fp8" if f8 else ""))
    roofline = {"bound": ds["bound"], "kernel": dom, "achieved": ds["achieved"], "peak": ds["peak"],
                "unit": ds["unit"], "frac": ds["frac"],
                "peak_source": (f"{peak_src} ("
                                + ("2 x bf16_tflops_sustained, the nominal E4M3/bf16 dense ratio"
                                   if f8 and dom in ("gemm1_swiglu", "gemm2_down") else
                                   "bf16_tflops_sustained" if ds["bound"] == "tensor" else "hbm_gbs")
                                + ", MEASURED_PEAKS.json)") if peak_src == "measured" else "fallback",
                "traffic": (trec["dram_bytes_per_launch"] if trec else None),
                "algorithmic_per_launch": ds["algorithmic_work"]}
    if "sm_mhz_in_kernel" in ds:
        roofline["sm_mhz_in_kernel"] = ds["sm_mhz_in_kernel"]
        roofline["frac_of_tensor_rate_at_that_clock"] = ds["frac_of_tensor_rate_at_that_clock"]
    phase_roofline = gemm_phase_roofline(c[: w.N], d_, I_, f8, gemm_mhz, sm_count, peaks["hbm_gbs"],
                                         {n: stages[n]["ms"] for n in ("gemm1_swiglu", "gemm2_down")})
    # whole-step roofline: max(FLOP / sustained TC peak, touched weights + activations / HBM)
    flops = 2.0 * T * d_ * E + 6.0 * M * d_ * I_
    bytes_ = wbytes_touched + E * d_ * 2 + 2 * T * d_ * 2
    t_tc = 2.0 * T * d_ * E / (peak16 * 1e12) + 6.0 * M * d_ * I_ / (peak_g1 * 1e12)
    t_roof = max(t_tc, bytes_ / (peaks["hbm_gbs"] * 1e9))
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 experts + bf16 router/combine" if f8 else "bf16",
        "data": "synthetic (seeded; random-init weights of the LongCat-Flash MoE-layer shape)",
        "config": workload_config(w, world, f8),
        "roofline": roofline,
        "layer_roofline": {"t_roof_ms": round(t_roof * 1e3, 4), "frac": round(t_roof * 1e3 / ms_per_step, 4),
                           "alg_flop": flops, "alg_bytes": bytes_, "ffn_rows_M": M,
                           "experts_touched": touched,
                           "zero_expert_share": round(float(c[w.N:].sum()) / (T * K), 4),
                           "ffn_per_token": round(M / T, 4),
                           "ffn_experts_by_rows": {
                               f"[{lo},{hi})": int(((c[:w.N] >= lo) & (c[:w.N] < hi)).sum())
                               for lo, hi in ((1, 128), (128, 256), (256, 512), (512, 1024), (1024, T + 1))}},
        "stages": stages,
        "gemm_phase_roofline": phase_roofline,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": int(x.numel() * 2),
                "d2h_bytes_per_step": int(out.numel() * 2), "steps": e2e_steps_n,
                "copies": "pinned host x -> device and out -> pinned host every step, on one copy "
                          "stream per direction, overlapping the neighbouring steps' compute"},
        "gpu_launches": int(args.steps * (n_kernels + 1 + (2 if f8 else 0))),
        "gpu_launches_note": "kernels of this library inside the device-timed region: "
                             f"{n_kernels + (2 if f8 else 0)} per forward "
                             f"{'(incl. the token-row and H-row quantisers) ' if f8 else ''}+ 1 bias update, per step",
        "clocks": dict(ClockSampler.summarize(clock_rows),
                       sm_mhz_in_gemms={k: v for k, v in gemm_mhz.items() if v},
                       sm_mhz_in_gemms_note="SM clock inside each expert GEMM of the last timed step, "
                                            "from the kernels' clock probe (cycles / global-timer ns)"),
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline and not f8:
        result["cpu_baseline"] = cpu_baseline(w, data, route_tokens=args.cpu_route_tokens,
                                              ffn_tokens=args.cpu_ffn_tokens)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ------------------------------------------------------------------- oracle (CPU baseline) ---

def _ffn_pairs(idx, tokens, N):
    """FFN picks (token, rank) of ``tokens`` under routing idx, and their experts."""
    pairs = [(int(t), r) for t in tokens for r in range(idx.shape[1]) if idx[t, r] < N]
    experts = np.array([idx[t, r] for t, r in pairs], np.int64)
    return pairs, experts


def _oracle_ffn(w, x_bits, pairs, experts, expert_weights, chunk: int):
    """Oracle SwiGLU rows of every FFN pick in ``pairs``, one ``oracle.expert_rows`` call per group
    of ``chunk`` distinct experts (every row of those experts in one call, so the oracle's OpenMP
    loop over rows has many rows to spread). ``expert_weights(list)`` returns host copies
    (w13 [n, 2I, d], w2 [n, d, I]) of the listed experts; it runs outside the timed calls.
    Returns (Y [len(pairs), d], seconds inside the oracle, rows per call)."""
    import oracle
    Y = np.empty((len(pairs), w.d), np.uint16)
    uniq = np.unique(experts)
    t_oracle = 0.0
    rows_per_call = []
    for c0 in range(0, uniq.size, chunk):
        group = uniq[c0:c0 + chunk]
        w13c, w2c = expert_weights(group.tolist())
        local = {int(e): i for i, e in enumerate(group)}
        sel = np.nonzero(np.isin(experts, group))[0]
        rows = np.ascontiguousarray(x_bits[[pairs[j][0] for j in sel]])
        row_expert = np.array([local[int(experts[j])] for j in sel], np.int32)
        t0 = time.perf_counter()
        _, y = oracle.expert_rows(rows, row_expert, w13c, w2c, want_h=False)
        t_oracle += time.perf_counter() - t0
        Y[sel] = y
        rows_per_call.append(int(sel.size))
    return Y, t_oracle, rows_per_call


def _oracle_combine(w, x_bits, tokens, idx, gate, pairs, Y):
    import oracle
    pos = {int(t): i for i, t in enumerate(tokens)}
    pr = np.full((len(tokens), w.K), -1, np.int32)
    for j, (t, r) in enumerate(pairs):
        pr[pos[t], r] = j
    xs = np.ascontiguousarray(x_bits[tokens])
    t0 = time.perf_counter()
    oracle.combine(xs, Y, np.ascontiguousarray(idx[tokens]), np.ascontiguousarray(gate[tokens]), pr, w.N)
    return time.perf_counter() - t0


def cpu_baseline(w, data, route_tokens: int | None = None, ffn_tokens: int = 512, chunk: int = 64):
    """The oracle on the host cores, on a bounded sample of the batch, in three timed phases:
    routing (router logits, softmax, biased top-K) of the first ``route_tokens`` tokens (all T by
    default); the SwiGLU experts of every FFN pick of a seeded subset of ``ffn_tokens`` of them,
    batched per group of ``chunk`` experts (the weights of each group copied to the host outside
    the timed calls); and the combine of that subset. tokens/s = 1 / (routing s per token +
    expert and combine s per token), each per-token cost measured on its own sample."""
    import oracle
    from mixture_experts_zero_b200 import inputs
    R = w.T if route_tokens is None else min(route_tokens, w.T)
    x_bits = inputs.bits(data["x"])[:R]
    wr_bits = inputs.bits(data["wr"])
    bias = data["bias"].cpu().numpy()
    t0 = time.perf_counter()
    z = oracle.router_logits(x_bits, wr_bits)
    idx, gate, _, _ = oracle.route(z, bias, w.K)
    t_route = time.perf_counter() - t0
    del z
    rng = np.random.default_rng(123)
    F = min(ffn_tokens, R)
    tokens = np.sort(rng.choice(R, F, replace=False))
    pairs, experts = _ffn_pairs(idx, tokens, w.N)
    w13h = np.empty((chunk, 2 * w.I, w.d), np.uint16)
    w2h = np.empty((chunk, w.d, w.I), np.uint16)

    def weights(group):
        for i, e in enumerate(group):
            w13h[i] = inputs.bits(data["w13"][e])
            w2h[i] = inputs.bits(data["w2"][e])
        return w13h[:len(group)], w2h[:len(group)]

    Y, t_ffn, rows_per_call = _oracle_ffn(w, x_bits, pairs, experts, weights, chunk)
    t_comb = _oracle_combine(w, x_bits, tokens, idx, gate, pairs, Y)
    value = 1.0 / (t_route / R + (t_ffn + t_comb) / F)
    threads = oracle.num_threads()
    return {"value": round(value, 3), "unit": UNIT, "cores": threads,
            "cpu": cpu_model(), "host_cpus": os.cpu_count(), "kind": "oracle",
            "sample": (("full batch: " if (R == w.T and F == w.T) else "subset-measured: ")
                       + f"routing of {R} tokens of the {w.name} batch "
                       f"({t_route:.2f} s), SwiGLU experts of the {len(pairs)} FFN picks of {F} "
                       f"seeded tokens of them ({t_ffn:.2f} s, {len(rows_per_call)} oracle calls "
                       f"of {min(rows_per_call)}-{max(rows_per_call)} rows, every row of up to "
                       f"{chunk} experts per call) and their combine ({t_comb:.3f} s); every "
                       f"phase runs the oracle's OpenMP loops on {threads} threads; the GPU arm's "
                       f"expert weights, copied to the host outside the timed calls"),
            "phases_s": {"route": round(t_route, 3), "experts": round(t_ffn, 3),
                         "combine": round(t_comb, 4)},
            "tokens": {"routed": R, "ffn": F, "ffn_picks": len(pairs)}}


# --------------------------------------------------------------------------- reference arm --

REF_WEIGHT_SETS = 16


def run_reference(args):
    """The oracle (CPU, plain C) as the reference arm, on bounded samples of the same workload:
    each step routes ``--ref-tokens`` fresh tokens and runs every FFN pick of them through the
    SwiGLU experts (one oracle call for all of a step's picks) and the combine. Expert weights
    are drawn on the host: expert e uses weight set e mod 16 of 16 seeded sets (the oracle's cost
    does not depend on the values; the GPU arm's 38.6 GB of weights are not copied)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    import oracle
    from mixture_experts_zero_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    g = inputs.generator(w.seed, "cpu")
    wr_bits = inputs.bits(inputs.draw_router(w, g, "cpu"))
    bias = inputs.draw_bias(w, g, "cpu").numpy()
    std = 1.0 / math.sqrt(w.d)
    P = min(REF_WEIGHT_SETS, w.N)
    ge = inputs.generator(w.seed * 100003, "cpu")
    w13s = inputs.bits((torch.randn(P, 2 * w.I, w.d, generator=ge) * std).to(torch.bfloat16))
    w2s = inputs.bits((torch.randn(P, w.d, w.I, generator=ge) * std).to(torch.bfloat16))

    per_step_tokens = args.ref_tokens
    total = {"route": 0.0, "experts": 0.0, "combine": 0.0}
    picks = 0
    for i in range(args.warmup + args.steps):
        gx = inputs.generator(w.seed * 7919 + i, "cpu")
        xs = torch.randn(per_step_tokens, w.d, generator=gx)
        if w.router == "zipf":
            xs[:, 0] = 1.0
        x_bits = inputs.bits(xs.to(torch.bfloat16))
        t0 = time.perf_counter()
        z = oracle.router_logits(x_bits, wr_bits)
        idx, gate, _, _ = oracle.route(z, bias, w.K)
        t_route = time.perf_counter() - t0
        tokens = np.arange(per_step_tokens)
        pairs, experts = _ffn_pairs(idx, tokens, w.N)
        Y, t_ffn, _ = _oracle_ffn(w, x_bits, pairs, experts % P,
                                  lambda group: (w13s[group], w2s[group]), P)
        t_comb = _oracle_combine(w, x_bits, tokens, idx, gate, pairs, Y)
        if i >= args.warmup:
            total["route"] += t_route
            total["experts"] += t_ffn
            total["combine"] += t_comb
            picks += len(pairs)
    total_s = sum(total.values())
    value = per_step_tokens * args.steps / total_s
    config = workload_config(w, int(os.environ.get("WORLD_SIZE", "1")), False)
    config.update({"T_sampled": per_step_tokens,
                   "sample": f"{per_step_tokens} fresh tokens per step (not the T={w.T} batch)",
                   "expert_weights": f"drawn on the host: expert e uses set e mod {P} of {P} "
                                     "seeded sets, not the GPU arm's weights"})
    threads = oracle.num_threads()
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_s / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": threads,
                         "cpu": cpu_model(), "host_cpus": os.cpu_count(),
                         "kind": "oracle",
                         "sample": (f"{per_step_tokens} fresh tokens per step of the {w.name} "
                                    f"workload: routing, their {picks} FFN picks over the timed "
                                    f"steps (one oracle call per step), combine; the oracle's "
                                    f"OpenMP loops on {threads} threads"),
                         "phases_s": {k: round(v, 3) for k, v in total.items()}},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------------------ kernel sweeps --

FFN_ROWS_CASES = ((16, 512), (32, 512), (64, 512), (96, 512), (128, 512), (160, 512), (192, 512),
                  (256, 512), (320, 256), (384, 256), (512, 256), (768, 128), (1024, 128),
                  (2048, 64), (4096, 32))


def run_sweep(args):
    """Kernel sweeps outside the step, one JSON line per case (one GPU, device-timed, L2 flushed
    with a 256 MB write before every timed call, median of the timed calls).

    ffn_rows: the two grouped expert GEMMs (lc_moe_expert_ffn) at the prefill shape (d=6144,
        I=2048) with c rows for each of n experts, against max(6*M*d*I FLOP / sustained TC peak,
        (3*n*d*I + 2*M*(2d+I)) * 2 bytes / HBM).
    hist: the expert-count histogram over idx[2^24, 12] (805 MB of int32), against HBM.
    control: the bias-control loop at LongCat-Flash shape (run_control).
    ffn_subset: the expert GEMMs on every 8th FFN expert of the prefill workload's routing
        (run_ffn_subset)."""
    import torch
    from mixture_experts_zero_b200 import binding as B

    if args.sweep == "control":
        run_control(args)
        return
    if args.sweep == "ffn_subset":
        run_ffn_subset(args)
        return

    peaks, peak_src = load_peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(256 * 2 ** 20 // 4, device=dev)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ts.sort()
        return ts[len(ts) // 2]

    g = torch.Generator(device=dev).manual_seed(7)
    if args.sweep == "hist":
        T, K, E = 1 << 24, 12, 768
        idx = torch.randint(0, E, (T, K), generator=g, device=dev, dtype=torch.int32)
        counts = torch.zeros(E, dtype=torch.int32, device=dev)
        ms = timed(lambda: B.lc_moe_expert_hist(idx, E, counts=counts), 10)
        gbs = idx.numel() * 4 / ms / 1e6
        print(json.dumps({"sweep": "hist", "T": T, "K": K, "n_bins": E, "ms": round(ms, 4),
                          "achieved_gbs": round(gbs, 1), "peak_gbs": peaks["hbm_gbs"],
                          "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peak_src}), flush=True)
        return
    d, I = 6144, 2048
    n_max = max(n for _, n in FFN_ROWS_CASES)
    w13 = torch.empty(n_max, 2 * I, d, dtype=torch.bfloat16, device=dev)
    w2 = torch.empty(n_max, d, I, dtype=torch.bfloat16, device=dev)
    for e in range(n_max):
        w13[e].normal_(0.0, 0.02, generator=g)
        w2[e].normal_(0.0, 0.02, generator=g)
    tc, hbm = peaks["bf16_tflops_sustained"] * 1e12, peaks["hbm_gbs"] * 1e9
    for c, n in FFN_ROWS_CASES:
        M = c * n
        x = torch.empty(M, d, dtype=torch.bfloat16, device=dev).normal_(generator=g)
        offsets = torch.arange(n + 1, dtype=torch.int32, device=dev) * c
        h = torch.empty(M, I, dtype=torch.bfloat16, device=dev)
        y = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
        ms = timed(lambda: B.lc_moe_expert_ffn(x, offsets, w13[:n], w2[:n], M, 1, h=h, y=y), 8)
        flop = 6 * M * d * I
        bytes_ = (3 * n * d * I + 2 * M * (2 * d + I)) * 2
        roof = max(flop / tc, bytes_ / hbm) * 1e3
        print(json.dumps({"sweep": "ffn_rows", "rows_per_expert": c, "experts": n, "ms": round(ms, 3),
                          "roof_ms": round(roof, 3), "frac": round(roof / ms, 3),
                          "tflops": round(flop / ms / 1e9, 1), "gbs": round(bytes_ / ms / 1e6, 1),
                          "peak_source": peak_src}), flush=True)
        del x, h, y


def run_ffn_subset(args, stride: int = 8):
    """The grouped expert GEMMs (lc_moe_expert_ffn) on a representative eighth of the prefill
    layer's FFN experts: the prefill batch is routed on the device, the 512 FFN experts are ranked
    by their row counts, and every 8th of them (ranks 0, 8, 16, ...) keeps its rows, so the 64
    experts have the full layer's distribution of rows per expert with 1/8 of its weights
    (4.8 GB) and rows. For profiler captures whose traffic scales to the full layer by the number
    of experts (x 8). Prints one JSON line: the experts' row counts, M, and the device time of the
    two GEMMs (median of 8, L2 flushed before each)."""
    import torch
    from mixture_experts_zero_b200 import binding as B
    from mixture_experts_zero_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = inputs.WORKLOADS["prefill"]
    g = inputs.generator(w.seed, dev)
    x = inputs.draw_x(w, g, dev)
    wr = inputs.draw_router(w, g, dev)
    bias = inputs.draw_bias(w, g, dev)
    counts = torch.zeros(w.E, dtype=torch.int32, device=dev)
    idx, _ = B.lc_moe_route(x, wr, bias, w.K, w.N, counts=counts)[:2]
    c = counts[: w.N].cpu().numpy().astype(np.int64)
    order = np.argsort(-c, kind="stable")
    keep = np.sort(order[::stride])
    sizes = c[keep]
    n, M = len(keep), int(sizes.sum())
    # the kept experts' rows: the tokens that picked each of them, grouped by expert
    idx_h = idx.cpu().numpy()
    tokens = np.concatenate([np.nonzero((idx_h == e).any(axis=1))[0] for e in keep])
    xp = x[torch.from_numpy(tokens).to(dev)].contiguous()
    offsets = torch.from_numpy(np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)).to(dev)
    gw = torch.Generator(device=dev).manual_seed(w.seed)
    std = 1.0 / math.sqrt(w.d)
    w13 = torch.empty(n, 2 * w.I, w.d, dtype=torch.bfloat16, device=dev)
    w2 = torch.empty(n, w.d, w.I, dtype=torch.bfloat16, device=dev)
    for e in range(n):
        w13[e].copy_(torch.randn(2 * w.I, w.d, generator=gw, device=dev) * std)
        w2[e].copy_(torch.randn(w.d, w.I, generator=gw, device=dev) * std)
    h = torch.empty(M, w.I, dtype=torch.bfloat16, device=dev)
    y = torch.empty(M, w.d, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 * 2 ** 20 // 4, device=dev)
    ts = []
    for i in range(11):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        B.lc_moe_expert_ffn(xp, offsets, w13, w2, M, 1, h=h, y=y)
        e1.record()
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(e0.elapsed_time(e1))
    ts.sort()
    print(json.dumps({"sweep": "ffn_subset", "stride": stride, "experts": n, "rows_M": M,
                      "rows_per_expert": sizes.tolist(), "ms": round(ts[len(ts) // 2], 3),
                      "weights_gb": round(n * 3 * w.d * w.I * 2 / 1e9, 2)}), flush=True)


def run_control(args):
    """The bias-control loop at LongCat-Flash shape (T = 8192 fresh N(0,1) tokens per step,
    d = 6144, 512 FFN + 256 zero experts, K = 12, K_e = 8, 200 steps): each step routes on the
    device (lc_moe_route: router GEMM, softmax + biased top-K, expert counts) and applies
    b_i += mu (K_e/(K N) - T_i/(K T_all)) (lc_moe_bias_update). One JSON line per (start, mu):
    the mean number of FFN experts per token every 10 steps, the expert-load spread
    max_i T_i / mean_i T_i at the first and last step, and the device time of one control step
    (route + update, CUDA events; drawing the tokens is outside it). Starts: b = 0, and b = +2/E
    on the zero experts (routing pushed toward the zero experts, below K_e FFN experts per token).
    mu = 1e-3 is the workload's; the larger mu show the direction and speed of the control within
    200 steps, since at 1e-3 the pages' convergence needs orders of magnitude more tokens."""
    import torch
    from mixture_experts_zero_b200 import binding as B
    from mixture_experts_zero_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = inputs.WORKLOADS["bias_loop"]
    s = B.Shape(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = B.new_workspace(s, B.OP_ROUTE, dev)
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device=dev)
    gate = torch.empty(w.T, w.K, dtype=torch.float32, device=dev)
    counts = torch.zeros(w.E, dtype=torch.int32, device=dev)
    for start in ("zero", "zero_experts_favoured"):
        for mu in (1e-3, 1e-2, 1e-1):
            g = inputs.generator(w.seed, dev)
            wr = inputs.draw_router(w, g, dev)
            bias = torch.zeros(w.E, dtype=torch.float32, device=dev)
            if start != "zero":
                bias[w.N:] = 2.0 / w.E
            ffn = torch.zeros(w.steps, dtype=torch.int64, device=dev)
            spread = torch.zeros(w.steps, dtype=torch.float64, device=dev)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                   torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(w.steps)]
            counts.zero_()
            for step in range(w.steps):
                x = inputs.draw_x(w, g, dev)
                e0, e1, e2, e3 = ev[step]
                e0.record()
                B.lc_moe_route(x, wr, bias, w.K, w.N, idx=idx, gate=gate, counts=counts, ws=ws)
                e1.record()
                ffn[step] = counts[: w.N].sum()
                spread[step] = counts.max().double() / (w.T * w.K / w.E)
                e2.record()
                B.lc_moe_bias_update(bias, counts, w.T, w.N, w.Z, w.K, w.K_e, mu, reset_counts=True)
                e3.record()
            torch.cuda.synchronize()
            B.lc_moe_read_status(ws)
            ms = sorted(a.elapsed_time(b) + c.elapsed_time(d) for a, b, c, d in ev)
            mean_ffn = (ffn.double() / w.T).cpu().tolist()
            sp = spread.cpu().tolist()
            zero_bias = bias[w.N:].mean().item() - bias[: w.N].mean().item()
            print(json.dumps({
                "sweep": "control", "workload": f"bias_loop: T={w.T} fresh tokens per step, "
                f"d={w.d}, N={w.N}, Z={w.Z}, K={w.K}, K_e={w.K_e}", "steps": w.steps, "mu": mu,
                "start": start, "mean_ffn_per_token_every_10": [round(v, 4) for v in mean_ffn[::10]],
                "mean_ffn_per_token_last": round(mean_ffn[-1], 4),
                "mean_ffn_per_token_last10": round(sum(mean_ffn[-10:]) / 10, 4),
                "load_max_over_mean_first_last": [round(sp[0], 3), round(sp[-1], 3)],
                "zero_minus_ffn_mean_bias": zero_bias,
                "control_step_ms_median": round(ms[len(ms) // 2], 4)}), flush=True)
    if not args.no_cpu_baseline:
        print(json.dumps(control_cpu_baseline(w, dev)), flush=True)


def control_cpu_baseline(w, dev, steps: int = 2):
    """The oracle's control step on the host cores: the first ``steps`` steps of the b = 0,
    mu = 1e-3 loop (same router and tokens as the device run), each timed over router logits in
    double, softmax + biased top-K + counts, and the bias update."""
    import oracle
    from mixture_experts_zero_b200 import inputs
    g = inputs.generator(w.seed, dev)
    wr_bits = inputs.bits(inputs.draw_router(w, g, dev))
    b = np.zeros(w.E, np.float32)
    secs = []
    for _ in range(steps):
        x_bits = inputs.bits(inputs.draw_x(w, g, dev))
        t0 = time.perf_counter()
        z = oracle.router_logits(x_bits, wr_bits)
        _, _, cnt, _ = oracle.route(z, b, w.K)
        b = oracle.bias_update(b, cnt, w.T, w.N, w.Z, w.K, w.K_e, w.mu)
        secs.append(time.perf_counter() - t0)
    step_s = sum(secs) / steps
    return {"sweep": "control", "impl": "cpu_baseline", "kind": "oracle", "cores": oracle.num_threads(),
            "cpu": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"the first {steps} of the {w.steps} control steps (b = 0, mu = {w.mu}): router logits, "
                      f"softmax + biased top-K + counts and the bias update of T = {w.T} tokens each",
            "control_step_ms": round(1e3 * step_s, 3), "tokens_per_s": round(w.T / step_s, 1)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill",
                    choices=["prefill", "decode", "small", "tiny", "prefill_ncu", "route_ncu", "decode_ncu",
                             "cold_ncu"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-route-tokens", type=int, default=None,
                    help="tokens the CPU baseline routes (default: the whole batch)")
    ap.add_argument("--cpu-ffn-tokens", type=int, default=512,
                    help="tokens whose FFN picks the CPU baseline runs through the experts")
    ap.add_argument("--ref-tokens", type=int, default=8, help="tokens per reference-arm step")
    ap.add_argument("--experts", choices=["bf16", "fp8"], default="bf16",
                    help="fp8: E4M3 expert projections (lc_moe_forward_fp8)")
    ap.add_argument("--sweep", choices=["ffn_rows", "hist", "control", "ffn_subset"], default=None,
                    help="run a kernel sweep instead of the step (one GPU)")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
