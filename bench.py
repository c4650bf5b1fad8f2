#!/usr/bin/env python
"""Benchmark of the fused large-vocabulary BCE loss + gradient on B200.

One step = one call of cutbce_forward_backward (loss, dH, dE) over one batch
of synthetic input shaped like the multi-label SASRec head of "Cut Binary
Cross Entropy" (B=64, N=200, D=64, V=876,000 items, Poisson(3) positives per
position drawn Zipf(1.05), 20% trailing padding).  Inputs are resident in HBM
when the timed region starts; L2 is flushed (a 256 MiB write) before every
timed step, outside the step's event pair.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line.  Under torchrun every rank runs its own independent batch
(replicas, weak scaling, no collective on the data path); the step time is the
max over ranks.  --impl reference times the float64 CPU oracle on the host
cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "fused BCE fwd+bwd tokens/s at V=876k,D=64 on 1 B200; % of roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
TILE_SOURCES = ["tile_engine.cuh", "common.cuh", "ptx_sm100.cuh", "elementwise.cuh", "pair_sort.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="sasrec_876k")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the side measurements (metrics, top-8)")
    ap.add_argument("--topk-queries", type=int, default=0,
                    help="with --calls-only: top-8 ranking calls for this many queries instead of the fused step")
    ap.add_argument("--cpu-sample-items", type=int, default=32768)
    ap.add_argument("--calls-only", type=int, default=0,
                    help="run this many untimed fused calls on --workload and exit (a target for ncu)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tile_source_sha():
    h = hashlib.sha256()
    for name in TILE_SOURCES:
        with open(os.path.join(ROOT, "vocabulary_label_bce_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entries = json.load(f)
    for e in entries:
        if e.get("kernel") == kernel and e.get("workload") == workload and e.get("source_sha") == tile_source_sha():
            return e.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """nvidia-smi samples every 50 ms; only those taken inside the timed window are kept."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        """Start sampling (before the warm-up, so that the sampler is running when timing begins)."""
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark_begin(self):
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        self.t1 = datetime.datetime.now()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 10]
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                ts = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f")
                if self.t0 is not None and not (self.t0 <= ts <= self.t1):
                    continue
                sm.append(float(r[2]))
                smax = float(r[3])
                power.append(float(r[4]))
            except ValueError:
                continue
            for name, val in zip(names, r[6:10]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w": statistics.median(power) if power else None}


def sample_problem(p, n_items):
    """The first n_items items (columns) of a drawn problem: ids outside become empty slots."""
    E = p.E[:n_items]
    tg = np.where(p.targets < n_items, p.targets, -1).astype(np.int32)
    return E, tg


def time_oracle_sample(p, n_items):
    from oracle import cutbce_oracle as O
    E, tg = sample_problem(p, n_items)
    t0 = time.perf_counter()
    O.forward_backward(p.H, E, tg, p.mask, reduction=O.MEAN_VALID_POSITIONS)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def workload_config(p, n_valid, world, l2_note):
    return {"workload": p.name, "B": p.B, "N": p.N, "T": p.T, "n_valid": n_valid, "V": p.V, "D": p.D, "K": p.K,
            "tokens": "value counts all B*N positions per step, padding included; valid_tokens_per_s counts "
                      "the n_valid positions that carry work",
            "inputs": f"{p.dtype} H, E; int32 targets; uint8 mask", "seed": 0, "l2": l2_note,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def reduce_max(x: float, world: int, device) -> float:
    """The max of x over all ranks (the step time of a replicated run is its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(tokens_per_rank: int, world: int, step_ms_max: float) -> float:
    """Whole-job throughput: every rank processes its own batch (replicas, weak scaling)."""
    return world * tokens_per_rank / (step_ms_max * 1e-3)


DATASHEET_BF16_TFLOPS = 2250.0   # B200 dense bf16, nominal


def probe_rates():
    """SFU exponential and FMA-pipe rates (operations per clock per SM), measured live
    by the library's own pipe probes on this GPU (median over SMs)."""
    from vocabulary_label_bce_b200 import binding as B
    return {"ex2": B.cutbce_probe_pipe_rate("ex2"), "ffma": B.cutbce_probe_pipe_rate("ffma"),
            "ffma2": B.cutbce_probe_pipe_rate("ffma2")}


def roofline_times(n_valid, V, D, peaks, rates, sms=148):
    """Path roofline: the slower of the tensor-core time of 8*T*V*D FLOP at the
    measured bf16 peak, and the time of T*V transcendental evaluations at the
    SFU rate plus the FMA-pipe rate divided by the 8 FMA-pipe operations of one
    polynomial exponential (rates per clock per SM from the live probes, at the
    maximum SM clock)."""
    f = peaks.get("sm_max_mhz", 1965.0) * 1e6
    flops = 8.0 * n_valid * V * D
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    r_mufu, r_fma = rates["ex2"] * sms * f, rates["ffma"] * sms * f
    t_alu = n_valid * V / (r_mufu + r_fma / 8)
    return flops, t_tensor, t_alu


# ---------------------------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    from vocabulary_label_bce_b200 import workloads as W
    p = W.draw_config(args.workload)
    # size each step's sample from a measured rate so that the whole run takes about two minutes
    probe = 1024
    rate = probe / time_oracle_sample(p, probe)
    n_items = int(rate * 120.0 / max(1, args.steps + args.warmup))
    n_items = max(512, min(p.V, n_items // 512 * 512))
    for _ in range(args.warmup):
        time_oracle_sample(p, n_items)
    ts = [time_oracle_sample(p, n_items) for _ in range(args.steps)]
    step = statistics.mean(ts) * p.V / n_items
    value = p.B * p.N / step
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(p, int(p.mask.sum()), 1, "n/a (CPU)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"float64 numpy oracle on the first {n_items} of {p.V} items, all "
                                   f"{p.T} positions, per step; time scaled by V/{n_items}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from vocabulary_label_bce_b200 import binding as B
    from vocabulary_label_bce_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, dev)

    peaks, peaks_src = load_peaks()
    rates = probe_rates()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    p = W.draw_config(args.workload, seed=0)
    H, E = device_inputs(p, dev)
    tg = torch.from_numpy(p.targets).to(dev)
    m = torch.from_numpy(p.mask).to(dev)
    prob = B.make_problem(H, E, tg, m, "mean")
    ws = torch.empty(B.cutbce_workspace_size(prob), dtype=torch.uint8, device=dev)
    loss = torch.empty((), dtype=torch.float64, device=dev)
    dH = torch.empty((p.T, p.D), dtype=torch.float32, device=dev)
    dE = torch.empty((p.V, p.D), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        B.cutbce_forward_backward(prob, None, loss, dH, dE, ws, stream)

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    status = B.cutbce_read_status(ws, stream)
    if status != 0:
        raise SystemExit(f"device status {B.cutbce_status_string(status)}")
    n_valid, n_pairs = B.cutbce_read_counts(prob, ws, None, stream)

    B.cutbce_profile_read(reset=True)
    B.cutbce_profile_enable(True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    sampler.mark_begin()
    for s, e in ev:
        flush.zero_()
        s.record(stream)
        step()
        e.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    barrier()
    clocks = sampler.stop()
    B.cutbce_profile_enable(False)
    prof = B.cutbce_profile_read(reset=True)
    status = B.cutbce_read_status(ws, stream)
    if status != 0:
        raise SystemExit(f"device status {B.cutbce_status_string(status)}")
    step_ms_local = statistics.mean(s.elapsed_time(e) for s, e in ev)
    step_ms = max_over_ranks(step_ms_local)
    tokens = p.B * p.N
    value = aggregate_value(tokens, world, step_ms)

    # per-kernel durations (events inside the library, same stream)
    avg = {k: (ms / n if n else 0.0) for k, (ms, n) in prof.items()}
    dominant = max(("item_pass", "position_pass"), key=lambda k: avg[k])
    kern_ms = max_over_ranks(avg[dominant])
    flops_path, t_tensor, t_alu = roofline_times(n_valid, p.V, p.D, peaks, rates, sms)
    kernel_flops = 4.0 * n_valid * p.V * p.D
    achieved = kernel_flops / (kern_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    traffic = committed_traffic(dominant, p.name)
    t_roof = max(t_tensor, t_alu)

    # end to end through the host-buffer entry (pinned host memory, copies inside the timed call)
    e2e = None
    if not args.no_e2e:
        Hh, Eh = (t.pin_memory() for t in device_inputs(p, "cpu"))
        th = torch.from_numpy(p.targets).pin_memory()
        mh = torch.from_numpy(p.mask).pin_memory()
        hprob = B.make_problem(Hh, Eh, th, mh, "mean")
        buf = torch.empty(B.cutbce_host_buffer_size(hprob), dtype=torch.uint8, device=dev)
        lh = torch.empty((), dtype=torch.float64).pin_memory()
        dHh = torch.empty((p.T, p.D), dtype=torch.float32).pin_memory()
        dEh = torch.empty((p.V, p.D), dtype=torch.float32).pin_memory()
        for _ in range(2):
            B.cutbce_forward_backward_host(hprob, 1.0, lh, dHh, dEh, buf, stream)
        n_e2e = max(3, min(args.steps, 10))
        barrier()
        ts = []
        for _ in range(n_e2e):
            flush.zero_()
            torch.cuda.synchronize(dev)
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record(stream)
            B.cutbce_forward_backward_host(hprob, 1.0, lh, dHh, dEh, buf, stream)
            e.record(stream)
            e.synchronize()
            ts.append(s.elapsed_time(e))
        barrier()
        e2e_ms = max_over_ranks(statistics.mean(ts))
        bi = Hh.numel() * Hh.element_size() + Eh.numel() * Eh.element_size() + th.numel() * 4 + mh.numel() + 4
        bo = 8 + dHh.numel() * 4 + dEh.numel() * 4
        e2e = {"value": world * tokens / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": bi,
               "d2h_bytes_per_step": bo, "ms_per_step": e2e_ms,
               "entry": "cutbce_forward_backward_host (pinned host H, E, targets, mask in; loss, dH, dE out)"}
        del buf

    extras = measure_extras(B, p, prob, H, E, tg, loss, dH, dE, ws, flush, stream, dev) \
        if (world == 1 and not args.no_extras and p.dtype == "bf16") else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_items = min(p.V, args.cpu_sample_items)
        t = time_oracle_sample(p, n_items)
        cpu_step = t * p.V / n_items
        cpu = {"value": tokens / cpu_step, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"float64 numpy oracle on the first {n_items} of {p.V} items, all {p.T} positions "
                         f"({t:.1f} s), time scaled by V/{n_items}"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if p.dtype == "bf16" else "f32", "data": "synthetic",
            "config": workload_config(p, n_valid, world, "flushed before each timed step (256 MiB write)"),
            "valid_tokens_per_s": world * n_valid / (step_ms * 1e-3),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic, "kernel": dominant,
                         "kernel_ms": kern_ms, "algorithmic_flops_per_launch": kernel_flops,
                         "peak_source": f"{peaks_src} bf16_tflops (burst)",
                         "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peak),
                         "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS},
            "path_roofline": {"flops": flops_path, "t_tensor_ms": t_tensor * 1e3, "t_alu_ms": t_alu * 1e3,
                              "t_roof_ms": t_roof * 1e3, "frac": t_roof * 1e3 / step_ms,
                              "note": "headline fraction of the whole step: t_roof / measured step time; "
                                      "t_alu from the live SFU (ex2) and FMA probe rates",
                              "probe_rates_per_clk_per_sm": rates, "sms": sms},
            "kernels_ms": {k: round(v, 4) for k, v in avg.items()},
            "n_pairs": n_pairs,
            "gpu_launches": args.steps * B.cutbce_kernel_launches(prob, 2),
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "extras": extras,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _time_calls(fn, flush, stream, n=5):
    """Mean CUDA-event time (ms) of n calls on `stream`, L2 flushed before each."""
    import torch
    fn()
    ts = []
    for _ in range(n):
        flush.zero_()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        e.synchronize()
        ts.append(s.elapsed_time(e))
    return statistics.mean(ts)


def measure_extras(B, p, prob, H, E, tg, loss, dH, dE, ws, flush, stream, dev):
    """Side measurements after the timed region (not part of the step): the fused
    step with Cut Metrics on against the plain step, and full-vocabulary top-8
    ranking (one query per sequence: its last valid position; and 8,192 queries)."""
    import torch
    plain = _time_calls(lambda: B.cutbce_forward_backward(prob, None, loss, dH, dE, ws, stream), flush, stream)
    met = torch.empty((p.T, 4), dtype=torch.int32, device=dev)
    opts = B.make_options(metrics=met)
    bits = B.OUT_LOSS | B.OUT_DH | B.OUT_DE | B.OUT_METRICS
    wsm = torch.empty(B.cutbce_workspace_size_ex(prob, opts, bits), dtype=torch.uint8, device=dev)
    with_met = _time_calls(lambda: B.cutbce_forward_backward_ex(prob, opts, None, loss, dH, dE, wsm, stream),
                           flush, stream)
    if B.cutbce_read_status(wsm, stream) != 0:
        raise SystemExit("device status after the metrics call")
    del wsm
    out = {"metrics_overhead": {"step_ms": plain, "step_with_metrics_ms": with_met,
                                "overhead_ms": with_met - plain,
                                "what": "cutbce_forward_backward_ex with per-position TP/FP/FN/TN"}}
    mask = np.asarray(p.mask).reshape(p.B, p.N)
    last = np.array([np.nonzero(mask[b])[0][-1] if mask[b].any() else 0 for b in range(p.B)])
    Hq = H.view(p.B, p.N, p.D)
    rows = {"one_per_sequence": Hq[torch.arange(p.B, device=dev), torch.from_numpy(last).to(dev)].contiguous(),
            "8192_queries": H[torch.from_numpy(np.nonzero(p.mask)[0][:8192]).to(dev)].contiguous()}
    out["topk"] = {}
    for name, Q in rows.items():
        k = 8
        wst = torch.empty(B.cutbce_topk_workspace_size(Q.shape[0], p.V, p.D, k), dtype=torch.uint8, device=dev)
        ms = _time_calls(lambda: B.cutbce_topk(Q, E, k, wst, stream), flush, stream)
        if B.cutbce_read_status(wst, stream) != 0:
            raise SystemExit("device status after the top-k call")
        out["topk"][name] = {"queries": int(Q.shape[0]), "V": p.V, "k": k, "ms": ms,
                             "queries_per_s": Q.shape[0] / (ms * 1e-3),
                             "tflops": 2.0 * Q.shape[0] * p.V * p.D / (ms * 1e-3) / 1e12}
    return out


def device_inputs(p, dev):
    """H and E on the device in the workload's dtype (bf16 bits, or fp32 for the small fp32 check)."""
    import torch
    if p.dtype == "bf16":
        return (torch.from_numpy(p.H_bits.view(np.int16)).view(torch.bfloat16).to(dev),
                torch.from_numpy(p.E_bits.view(np.int16)).view(torch.bfloat16).to(dev))
    return torch.from_numpy(p.H).to(dev), torch.from_numpy(p.E).to(dev)


def run_calls_only(args):
    """N plain fused calls, no timing and no output: the command ncu captures."""
    import torch
    from vocabulary_label_bce_b200 import binding as B
    from vocabulary_label_bce_b200 import workloads as W
    p = W.draw_config(args.workload, seed=0)
    dev = torch.device("cuda", 0)
    H, E = device_inputs(p, dev)
    tg = torch.from_numpy(p.targets).to(dev)
    m = torch.from_numpy(p.mask).to(dev)
    prob = B.make_problem(H, E, tg, m, "mean")
    ws = torch.empty(B.cutbce_workspace_size(prob), dtype=torch.uint8, device=dev)
    loss = torch.empty((), dtype=torch.float64, device=dev)
    dH = torch.empty((p.T, p.D), dtype=torch.float32, device=dev)
    dE = torch.empty((p.V, p.D), dtype=torch.float32, device=dev)
    if args.topk_queries > 0:
        # top-8 ranking of the first topk_queries valid rows of H against the whole vocabulary
        Q = H[torch.from_numpy(np.nonzero(p.mask)[0][:args.topk_queries]).to(dev)].contiguous()
        ws = torch.empty(B.cutbce_topk_workspace_size(Q.shape[0], p.V, p.D, 8), dtype=torch.uint8, device=dev)
        for _ in range(args.calls_only):
            B.cutbce_topk(Q, E, 8, ws)
    else:
        for _ in range(args.calls_only):
            B.cutbce_forward_backward(prob, None, loss, dH, dE, ws)
    torch.cuda.synchronize(dev)
    status = B.cutbce_read_status(ws)
    if status != 0:
        raise SystemExit(f"device status {B.cutbce_status_string(status)}")
    return 0


def main():
    args = parse_args()
    if args.calls_only > 0:
        return run_calls_only(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
