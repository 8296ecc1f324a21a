#!/usr/bin/env python
"""Benchmark exact attention (forward and forward+backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: fa_fwd, then the
three launches of fa_bwd (prep, main, dQ convert).  The default workload is
the long causal context (B=2, H=16, N=8192, d=128), the one the forward +
backward throughput target is stated for.  `value` is algorithmic TFLOP/s of
forward + backward summed over all ranks (4 d flops per kept score entry
forward, 10 d backward); with N > 1 every rank runs its own replica of the
workload (heads are independent, so there is no data-path collective) and
the time is the maximum over ranks.

`--impl reference` times the fp64 CPU oracle on this host instead (rank 0
only), on a bounded sample of the same workload per step.

Prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "attention fwd and fwd+bwd TFLOP/s (bf16) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "long_s8k_d128_causal"
# Decode against a resident KV cache (fa_decode): one new token per sequence
# against a 32K-token history, 8 sequences x 32 heads, d = 128, causal.
# The two-sequence variant (a 1 GiB cache, still far above L2) is the one
# profiled with ncu.
DECODE_WORKLOADS = {"decode_b8_h32_kv32k_d128": dict(B=8, H=32, Nq=1, Nk=32768, d=128, mask="causal"),
                    "decode_b2_h32_kv32k_d128": dict(B=2, H=32, Nq=1, Nk=32768, d=128, mask="causal"),
                    "decode_b8_h32_q16_kv32k_d128": dict(B=8, H=32, Nq=16, Nk=32768, d=128, mask="causal")}
DECODE_METRIC = "decode attention: K/V cache bytes streamed per second (bf16), % of measured HBM bandwidth"

L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def flops(w: workloads.Workload, mask) -> dict:
    E = workloads.kept_entries(w, mask)
    per = w.B * w.H * E * w.d
    return {"fwd": 4 * per, "bwd": 10 * per, "E": E}


def source_sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of that kernel (else None)."""
    f = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(f):
        return None
    rec = json.load(open(f)).get(kernel, {}).get(workload)
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or source_sha(src) != rec["source_sha"]:
        return None
    return rec["dram_bytes_per_launch"]


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons (read only)."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.t0 = self.t1 = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(1.0)
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def result(self):
        if self.proc is None:
            return {"error": "nvidia-smi unavailable"}
        time.sleep(0.3)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:8]))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 - 1 <= r[0] <= self.t1 + 1] or rows
        if not inside:
            return {"error": "no samples"}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in inside for n, v in zip(names, r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


def cpu_sample(w, x, mask, seed_rows=None, heads=1):
    """Time the fp64 oracle (fwd + bwd) on the first `heads` heads of the
    workload, truncated to their first `seed_rows` positions; returns
    (TFLOP/s, seconds, desc, threads)."""
    import oracle  # test infrastructure: only the CPU-baseline legs use it

    n = seed_rows or w.N
    sl = lambda t: t.reshape(w.B * w.H, w.N, w.d)[:heads, :n].contiguous()
    sub = w.with_(B=1, H=heads, N=n)
    m = mask[: sub.nb, : sub.nb].contiguous() if mask is not None else None
    t0 = time.perf_counter()
    oracle.bwd(sl(x["Q"]), sl(x["K"]), sl(x["V"]), sl(x["dO"]), w.mask, m, w.scale)
    dt = time.perf_counter() - t0
    f = flops(sub, m)
    desc = (f"fp64 oracle fwd+bwd (plain definition, all masked entries skipped) on heads 0..{heads - 1} of "
            f"{w.name}, first {n} of {w.N} positions ({f['E']} kept score entries per head)")
    return (f["fwd"] + f["bwd"]) / dt / 1e12, dt, desc, oracle.num_threads()


def cpu_baseline(w, x, mask, target_s=10.0):
    """The oracle on a bounded sample of the workload: one head to gauge the
    rate, then as many whole heads as take about `target_s` seconds."""
    v, dt, desc, cores = cpu_sample(w, x, mask)
    heads = max(1, min(w.B * w.H, int(math.ceil(target_s / max(dt, 1e-6)))))
    if heads > 1:
        v, dt, desc, cores = cpu_sample(w, x, mask, heads=heads)
    return v, dt, desc, cores


def reference_arm(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = workloads.make_inputs(w, args.seed)
    n = min(w.N, 2048)
    for _ in range(args.warmup):
        cpu_sample(w, x, x["mask"], n)
    vals, secs = [], 0.0
    desc = cores = None
    for _ in range(args.steps):
        v, dt, desc, cores = cpu_sample(w, x, x["mask"], n)
        vals.append(v)
        secs += dt
    # the work of one step: one head, the first n positions (and, for a block
    # mask, the part of the tile grid those positions cover)
    sub = w.with_(B=1, H=1, N=n)
    f = flops(sub, x["mask"][: sub.nb, : sub.nb] if x["mask"] is not None else None)
    value = args.steps * (f["fwd"] + f["bwd"]) / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(v: float, dist=None, device=None) -> float:
    """Largest value of `v` over all ranks (the step time that counts)."""
    if dist is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(total_ms: float, steps: int, world: int, flops_per_step: float) -> tuple:
    """(ms per step, whole-job TFLOP/s): every rank runs one replica of the
    workload, so the job does `world` replicas per step in the slowest rank's
    time."""
    ms = total_ms / steps
    return ms, world * flops_per_step / (ms * 1e-3) / 1e12


def head_range(heads: int, world: int, rank: int) -> tuple:
    """Contiguous range [h0, h1) of the flattened B*H heads that `rank` takes
    when one problem is split across `world` ranks by heads.  Heads are
    independent in both passes, so the split needs no collective; ranges
    differ in length by at most one head."""
    if heads < world:
        raise ValueError(f"{heads} heads cannot be split over {world} ranks")
    return rank * heads // world, (rank + 1) * heads // world


def slice_heads(x: dict, w, h0: int, h1: int) -> dict:
    """The rank's part of the problem: heads [h0, h1) of Q, K, V and dO as
    contiguous [1, h1 - h0, N, d] tensors; the block mask is shared by every
    head and is kept whole."""
    out = {}
    for n in ("Q", "K", "V", "dO"):
        t = x[n].reshape(w.B * w.H, w.N, w.d)[h0:h1]
        out[n] = t.reshape(1, h1 - h0, w.N, w.d).contiguous()
    out["mask"] = x["mask"]
    return out


def workload_config(w):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "mask": w.mask, "scale": w.scale}


def trimmed_mean(xs, cut=0.1):
    """Mean of xs without the lowest and highest `cut` fraction."""
    xs = sorted(xs)
    k = int(len(xs) * cut)
    kept = xs[k:len(xs) - k] if len(xs) > 2 * k else xs
    return sum(kept) / len(kept)


def time_other_workloads(fa, dev, stream, peaks, names, reps=100, seed=0):
    """Forward and forward + backward of each named workload on the same GPU,
    in the same run as the headline: the mean of `reps` individually timed
    repetitions (CUDA events on the launching stream) after dropping the
    fastest and slowest tenth.  (Event times of short launches come in steps
    of about 2 us on this part: a median sits on one step, the trimmed mean
    averages across them.)  Workloads whose step
    touches less than twice the L2 are also timed with the L2 flushed before
    every repetition (a 2 x L2 buffer written outside the event pair), and
    that number is the one reported; the warm-L2 figure is kept beside it.
    Achieved HBM GB/s is the algorithmic bytes (forward: read Q, K, V, write
    O and LSE; backward: read Q, K, V, O, dO, LSE and D, write dQ, dK, dV)
    over the time."""
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    out = {}
    for name in names:
        w = workloads.WORKLOADS[name]
        x = workloads.make_inputs(w, seed)
        Q, K, V, dO = (x[n].to(dev) for n in ("Q", "K", "V", "dO"))
        mask = x["mask"].to(dev) if x["mask"] is not None else None
        O = torch.empty_like(Q)
        LSE = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
        ws = torch.empty(fa.bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)

        def fwd():
            fa.fwd(Q, K, V, w.mask, mask, w.scale, O=O, LSE=LSE, stream=stream)

        def fwd_bwd():
            fwd()
            for s in range(3):
                fa.bwd_stage(s, Q, K, V, O, dO, LSE, dQ, dK, dV, ws, w.mask, mask, w.scale, stream=stream)

        touched = sum(t.numel() * t.element_size() for t in (Q, K, V, dO, O, LSE, dQ, dK, dV)) + ws.numel()
        modes = ("flushed", "warm") if touched < 2 * L2_BYTES else ("warm",)
        res = {}
        for kind, run in (("fwd", fwd), ("fwd_bwd", fwd_bwd)):
            for _ in range(5):
                run()
            torch.cuda.synchronize(dev)
            for mode in modes:
                times = []
                for _ in range(reps):
                    if mode == "flushed":
                        flush.fill_(1)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    run()
                    e1.record(stream)
                    times.append((e0, e1))
                torch.cuda.synchronize(dev)
                res.setdefault(kind, {})[mode] = trimmed_mean([a.elapsed_time(b) for a, b in times])
        status = fa.device_status()
        fl = flops(w, x["mask"])
        T = w.B * w.H * w.N * w.d
        rows = w.B * w.H * w.N
        fwd_bytes = 8 * T + 4 * rows
        bwd_bytes = 16 * T + 8 * rows
        rec = {"config": workload_config(w), "l2": "flushed before each repetition" if "flushed" in modes else
               f"no flush: step touches {touched / 2**20:.0f} MiB, more than twice the L2", "reps": reps,
               "device_status": status}
        for kind, fkey, nbytes in (("fwd", ("fwd",), fwd_bytes), ("fwd_bwd", ("fwd", "bwd"), fwd_bytes + bwd_bytes)):
            ms = res[kind][modes[0]]
            tf = sum(fl[k] for k in fkey) / (ms * 1e-3) / 1e12
            rec[kind] = {"ms": ms, "tflops": tf, "frac_of_peak": tf / peaks["bf16_tflops"],
                         "frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
                         "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
                         "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
            if len(modes) == 2:
                rec[kind]["ms_warm_l2"] = res[kind]["warm"]
        out[name] = rec
        del Q, K, V, dO, O, LSE, dQ, dK, dV, ws
    del flush
    return out


def long_run(step, stream, dev, min_seconds=1.0):
    """The headline step repeated back to back for at least `min_seconds`
    (CUDA events around the whole run), with the SM clock sampled: the
    sustained counterpart of the K-step figure, which a short run takes
    before the board reaches its power limit."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    n = max(10, int(math.ceil(min_seconds * 1e3 / max(e0.elapsed_time(e1), 1e-3))))
    clocks = ClockSampler(dev.index)
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    return n, e0.elapsed_time(e1) / n, clocks.result()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=workloads.ORDER + list(DECODE_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sustained-run", action="store_true",
                    help="skip the one-second repeat of the headline step")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the per-workload timing of the other configurations")
    ap.add_argument("--split", default="replicas", choices=["replicas", "heads"],
                    help="with N > 1: one replica of the workload per rank (weak scaling, default), or one "
                         "problem split by heads across the ranks (strong scaling, no collective)")
    ap.add_argument("--vs-standard", action="store_true",
                    help="time the fused forward against standard (materialising) attention instead")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.workload in DECODE_WORKLOADS:
        return decode_main(args, args.workload, DECODE_WORKLOADS[args.workload])
    w = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        return reference_arm(args, w)
    if args.vs_standard:
        return vs_standard_main(args, w)

    import exact_io_aware_65_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- inputs resident in HBM: each rank its own replica of the workload,
    # or (--split heads) its range of the heads of one problem
    split = args.split == "heads" and world > 1
    w_full = w
    if split:
        h0, h1 = head_range(w.B * w.H, world, rank)
        x = slice_heads(workloads.make_inputs(w, args.seed), w, h0, h1)
        w = w.with_(B=1, H=h1 - h0)
    else:
        x = workloads.make_inputs(w, args.seed + rank)
    mask_cpu = x["mask"]
    Q, K, V, dO = (x[n].to(dev) for n in ("Q", "K", "V", "dO"))
    mask = mask_cpu.to(dev) if mask_cpu is not None else None
    O = torch.empty_like(Q)
    LSE = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    ws = torch.empty(fa.bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    names = ("fwd", "bwd_prep", "bwd_main", "bwd_dq_convert")

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        fa.fwd(Q, K, V, w.mask, mask, w.scale, O=O, LSE=LSE, stream=stream)
        if evs is not None:
            evs[1].record(stream)
        for s in range(3):
            fa.bwd_stage(s, Q, K, V, O, dO, LSE, dQ, dK, dV, ws, w.mask, mask, w.scale, stream=stream)
            if evs is not None:
                evs[2 + s].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.device_status() != 0:
        raise SystemExit("device status reports a timed-out wait during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks.mark_end()
    status = fa.device_status()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), dist, dev)
    per_kernel = {n: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, n in enumerate(names)}
    clock_info = clocks.result()

    fl = flops(w, mask_cpu)  # this rank's part
    fl_job = flops(w_full, mask_cpu)
    if split:  # one problem: the whole job is the full problem's work in the slowest rank's time
        ms_step, value = throughput(total_ms, args.steps, 1, fl_job["fwd"] + fl_job["bwd"])
    else:
        ms_step, value = throughput(total_ms, args.steps, world, fl["fwd"] + fl["bwd"])
    peaks, peak_kind = load_peaks()
    fwd_tflops = fl["fwd"] / (per_kernel["fwd"] * 1e-3) / 1e12
    bwd_ms = per_kernel["bwd_prep"] + per_kernel["bwd_main"] + per_kernel["bwd_dq_convert"]
    bwd_tflops = fl["bwd"] / (bwd_ms * 1e-3) / 1e12

    # dominant kernel and its roofline (tensor-bound contraction)
    dom = max(("fwd", "bwd_main"), key=lambda n: per_kernel[n])
    dom_flops = fl["fwd"] if dom == "fwd" else fl["bwd"]
    achieved = dom_flops / (per_kernel[dom] * 1e-3) / 1e12
    dom_src = {"fwd": "exact_io_aware_65_b200/csrc/fa_fwd.cu", "bwd_main": "exact_io_aware_65_b200/csrc/fa_bwd.cu"}
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "peak_source": f"{peak_kind} bf16 dense (burst)",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "traffic": traffic_for(dom, w.name), "source": dom_src[dom]}

    # ---- end to end through the public API with host buffers.  Two device
    # buffer sets; step i uses set i % 2.  Step i+1's inputs go up on their own
    # stream and step i-1's results come down on another while step i
    # computes, the way a training loop with a prefetching loader runs.  Every
    # step still copies all of its inputs in and all of its results out inside
    # the timed region.
    e2e_steps = args.e2e_steps or max(3, min(args.steps, 30))
    hostin = {n: x[n].pin_memory() for n in ("Q", "K", "V", "dO")}
    host_mask = mask_cpu.pin_memory() if mask_cpu is not None else None
    out_names = ("O", "LSE", "dQ", "dK", "dV")
    hostout = {"O": torch.empty_like(O, device="cpu").pin_memory(),
               "LSE": torch.empty_like(LSE, device="cpu").pin_memory(),
               "dQ": torch.empty_like(dQ, device="cpu").pin_memory(),
               "dK": torch.empty_like(dK, device="cpu").pin_memory(),
               "dV": torch.empty_like(dV, device="cpu").pin_memory()}
    sets = []
    for b in range(2):
        ins = {n: torch.empty_like(hostin[n], device=dev) for n in hostin}
        ins["mask"] = torch.empty_like(host_mask, device=dev) if host_mask is not None else None
        outs = {"O": O, "LSE": LSE, "dQ": dQ, "dK": dK, "dV": dV} if b == 0 else \
               {n: torch.empty_like(t) for n, t in (("O", O), ("LSE", LSE), ("dQ", dQ), ("dK", dK), ("dV", dV))}
        sets.append((ins, outs))
    h2d = sum(t.numel() * t.element_size() for t in hostin.values()) + (host_mask.numel() if host_mask is not None else 0)
    d2h = sum(t.numel() * t.element_size() for t in hostout.values())
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps_run(n):
        for i in range(n):
            b = i % 2
            ins, outs = sets[b]
            up.wait_event(computed[b])            # step i-2 has finished reading set b's inputs
            with torch.cuda.stream(up):
                for k in hostin:
                    ins[k].copy_(hostin[k], non_blocking=True)
                if host_mask is not None:
                    ins["mask"].copy_(host_mask, non_blocking=True)
            uploaded[b].record(up)
            stream.wait_event(uploaded[b])
            stream.wait_event(downloaded[b])      # step i-2's results in set b are on the host
            o, lse = fa.fwd(ins["Q"], ins["K"], ins["V"], w.mask, ins["mask"], w.scale, O=outs["O"],
                            LSE=outs["LSE"], stream=stream)
            fa.bwd(ins["Q"], ins["K"], ins["V"], o, ins["dO"], lse, w.mask, ins["mask"], w.scale,
                   dQ=outs["dQ"], dK=outs["dK"], dV=outs["dV"], workspace=ws, stream=stream)
            computed[b].record(stream)
            down.wait_event(computed[b])
            with torch.cuda.stream(down):
                for k in out_names:
                    hostout[k].copy_(outs[k], non_blocking=True)
            downloaded[b].record(down)

    for b in range(2):                            # every event recorded once before the first wait
        for ev in (uploaded[b], computed[b], downloaded[b]):
            ev.record(stream)
    e2e_steps_run(2)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)                                 # the first upload is the first work of the region
    e2e_steps_run(e2e_steps)
    e1.record(down)                               # the last download ends after all other work
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms, e2e_value = throughput(max_over_ranks(e0.elapsed_time(e1), dist, dev), e2e_steps,
                                   1 if split else world,
                                   (fl_job if split else fl)["fwd"] + (fl_job if split else fl)["bwd"])
    status = status or fa.device_status()

    # ---- the same step repeated for at least a second (sustained clocks)
    sustained = None
    if not args.no_sustained_run and world == 1:
        n_long, ms_long, clocks_long = long_run(step, stream, dev)
        sustained = {"steps": n_long, "ms_per_step": ms_long,
                     "tflops": (fl["fwd"] + fl["bwd"]) / (ms_long * 1e-3) / 1e12, "clocks": clocks_long}
        sustained["frac_of_peak"] = sustained["tflops"] / peaks["bf16_tflops"]
        sustained["frac_of_sustained"] = sustained["tflops"] / peaks["bf16_tflops_sustained"]

    # ---- the other configurations, on the same GPU (single-GPU runs only)
    others = None
    if world == 1 and not args.no_other_workloads:
        others = time_other_workloads(fa, dev, stream, peaks, [n for n in workloads.ORDER if n != w.name])
        status = status or max(r["device_status"] for r in others.values())

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, desc, cores = cpu_baseline(w, x, mask_cpu)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc, "seconds": dt}

    in_bytes = sum(t.numel() * t.element_size() for t in (Q, K, V, dO, O, LSE, dQ, dK, dV)) + ws.numel()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded i.i.d. N(0,1) Q, K, V, dO rounded to bf16 (no dataset)",
        "config": dict(workload_config(w_full),
                       parallelism=(f"one problem split by heads over {world} GPUs (contiguous head ranges, "
                                    f"no collective)") if split else f"{world} independent replica(s), one per GPU",
                       l2=f"no flush: step touches {in_bytes / 2**20:.0f} MiB, more than the "
                          f"{L2_BYTES / 2**20:.0f} MiB L2"),
        "fwd": {"ms": per_kernel["fwd"], "tflops": fwd_tflops, "frac_of_peak": fwd_tflops / peaks["bf16_tflops"],
                "frac_of_sustained": fwd_tflops / peaks["bf16_tflops_sustained"]},
        "fwd_bwd": {"ms": ms_step, "tflops": value / world, "frac_of_peak": value / world / peaks["bf16_tflops"],
                    "frac_of_sustained": value / world / peaks["bf16_tflops_sustained"],
                    "per": "GPU (whole-job value / N)"},
        "bwd": {"ms": bwd_ms, "tflops": bwd_tflops},
        "kernels_ms": per_kernel,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "steps": e2e_steps,
                "pipeline": "two buffer sets: step i+1's upload and step i-1's download run on their own "
                            "streams during step i's compute"},
        "gpu_launches": 4 * args.steps,
        "clocks": clock_info,
        "sustained_run": sustained,
        "per_workload": others,
        "device_status": status,
        "peaks": {"bf16_tflops": peaks["bf16_tflops"], "bf16_tflops_sustained": peaks["bf16_tflops_sustained"],
                  "source": peak_kind},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    if status != 0:
        raise SystemExit(f"device status {status}: a bounded wait timed out")


def vs_standard_main(args, w):
    """Forward of the fused kernel against standard attention (S = QK^T and
    P in HBM, cuBLAS products + the library's softmax) on the same workload
    and GPU: the speed and memory ratios the pages quote, measured here."""
    import exact_io_aware_65_b200 as fa

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    x = workloads.make_inputs(w, args.seed, grad=False)
    Q, K, V = (x[n].to(dev) for n in ("Q", "K", "V"))
    mask = x["mask"].to(dev) if x["mask"] is not None else None
    O1, O2 = torch.empty_like(Q), torch.empty_like(Q)
    L1 = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    L2 = torch.empty_like(L1)
    std_ws_bytes = fa.standard_fwd_workspace_size(w.B, w.H, w.N, w.d)
    ws = torch.empty(std_ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    runs = {"fused": lambda: fa.fwd(Q, K, V, w.mask, mask, w.scale, O=O1, LSE=L1, stream=stream),
            "standard": lambda: fa.standard_fwd(Q, K, V, w.mask, mask, w.scale, O=O2, LSE=L2, workspace=ws,
                                                stream=stream)}
    ms = {}
    clocks = ClockSampler(dev.index)
    clocks.mark_start()
    for name, run in runs.items():
        for _ in range(args.warmup):
            run()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            run()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms[name] = e0.elapsed_time(e1) / args.steps
    clocks.mark_end()
    status = fa.device_status()
    max_diff = (O1.float() - O2.float()).abs().max().item()
    fl = flops(w, x["mask"])["fwd"]
    line = {
        "metric": "forward time of standard (materialising) attention / fused forward, same workload and GPU",
        "value": ms["standard"] / ms["fused"], "unit": "x", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w),
        "fused": {"ms": ms["fused"], "tflops": fl / (ms["fused"] * 1e-3) / 1e12,
                  "extra_device_bytes": 0},
        "standard": {"ms": ms["standard"], "tflops_of_kept_work": fl / (ms["standard"] * 1e-3) / 1e12,
                     "extra_device_bytes": std_ws_bytes,
                     "note": "computes the whole N x N grid and masks it; S fp32 and P bf16 through HBM"},
        "max_abs_diff_O": max_diff,
        "clocks": clocks.result(),
        "device_status": status,
    }
    print(json.dumps(line), flush=True)
    if status != 0:
        raise SystemExit(f"device status {status}")


def decode_main(args, name, c):
    """Decode against a KV cache resident in HBM: each step is one fa_decode
    call (split-key partials + merge).  Bound by HBM: every K and V byte is
    read once per step."""
    import exact_io_aware_65_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    B, H, Nq, Nk, d, mask = c["B"], c["H"], c["Nq"], c["Nk"], c["d"], c["mask"]
    scale = float(torch.tensor(d ** -0.5, dtype=torch.float32).item())
    x = workloads.make_cross_inputs(B, H, Nq, Nk, d, mask, seed=args.seed + rank)
    Q, K, V = (x[n].to(dev) for n in ("Q", "K", "V"))
    O = torch.empty_like(Q)
    LSE = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.decode_workspace_size(B, H, Nq, Nk, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.decode(Q, K, V, mask, scale, O=O, LSE=LSE, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.device_status() != 0:
        raise SystemExit("device status reports a timed-out wait during warm-up")
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clocks.mark_end()
    status = fa.device_status()
    total_ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    ms = total_ms / args.steps
    kv_bytes = 2 * B * H * Nk * d * 2                       # K and V, read once
    alg_bytes = kv_bytes + 2 * (Q.numel() * 2) + LSE.numel() * 4  # + Q read, O and LSE written
    peaks, peak_kind = load_peaks()
    value = world * kv_bytes / (ms * 1e-3) / 1e9
    achieved = alg_bytes / (ms * 1e-3) / 1e9
    flop = 4 * B * H * Nq * Nk * d
    roofline = {"bound": "hbm", "kernel": "decode (partial + merge)", "achieved": achieved,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "peak_source": f"{peak_kind} HBM copy bandwidth", "traffic": traffic_for("decode", name),
                "source": "exact_io_aware_65_b200/csrc/fa_decode.cu"}

    # end to end: the cache stays resident (it is a cache); each step brings
    # the new queries in from pinned host memory and the outputs back
    hq = x["Q"].pin_memory()
    ho, hl = torch.empty_like(O, device="cpu").pin_memory(), torch.empty_like(LSE, device="cpu").pin_memory()
    dq = torch.empty_like(Q)

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        fa.decode(dq, K, V, mask, scale, O=O, LSE=LSE, workspace=ws, stream=stream)
        ho.copy_(O, non_blocking=True)
        hl.copy_(LSE, non_blocking=True)

    e2e_steps = args.e2e_steps or max(3, min(args.steps, 30))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev) / e2e_steps
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle  # test infrastructure: only the CPU-baseline leg uses it

        heads = B * H
        t = time.perf_counter()
        oracle.fwd(x["Q"], x["K"], x["V"], mask, None, scale)
        dt = time.perf_counter() - t
        cpu = {"value": kv_bytes / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
               "sample": f"fp64 oracle forward of all {heads} heads ({Nq} query x {Nk} keys each)", "seconds": dt}
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded i.i.d. N(0,1) Q, K, V rounded to bf16 (no dataset)",
        "config": {"workload": name, "B": B, "H": H, "Nq": Nq, "Nk": Nk, "d": d, "mask": mask,
                   "parallelism": f"{world} independent replica(s), one per GPU",
                   "l2": f"no flush: the K/V cache is {kv_bytes / 2**20:.0f} MiB, more than the "
                         f"{L2_BYTES / 2**20:.0f} MiB L2"},
        "tflops": flop / (ms * 1e-3) / 1e12,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": world * kv_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": hq.numel() * 2, "d2h_bytes_per_step": ho.numel() * 2 + hl.numel() * 4,
                "ms_per_step": e2e_ms, "steps": e2e_steps},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks.result(),
        "device_status": status,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    if status != 0:
        raise SystemExit(f"device status {status}: a bounded wait timed out")


if __name__ == "__main__":
    main()
