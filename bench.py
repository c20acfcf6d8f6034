"""Benchmark: effective weight bandwidth of the compressed Llama-3.1-8B MLP.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload (one "step"): one Llama-3.1-8B-shaped MLP layer -- gate and up
[14336, 4096], down [4096, 14336], BF16 N(0, 0.02^2) with 0.05% N(0, 1)
outliers (seeds 1, 2, 3; rank r adds 100 r) -- multiplied by activations X of
M = 1, 4, 16 and 64 rows (12 matmuls, Y = X W^T, fp32 out).  Each
(projection, M) runs the plan picked by libuw's autotuner (full decode +
plain kernel, runtime transcode + fused kernel, or direct palette + fused
kernel; FMA GEMV or tcgen05).  Matmuls are issued M-outer / projection-inner,
so two other matrices (>= 160 MB) stream between two uses of one matrix and
each read comes from HBM, not from the 126 MB L2.

value  = sum over the step's matmuls of 2*N*K (uncompressed BF16 weight bytes)
         / step time  [GB/s], inputs resident in HBM, CUDA events, max over ranks.
e2e    = the same, with X copied from pinned host memory and Y read back to
         pinned host memory inside the timed region, through the C ABI (copies
         on their own streams, ordered by events, overlapping the matmuls).
roofline: the kernel group with the largest share of the step; achieved =
         its algorithmic bytes (compressed planes + X + Y) / its event-timed
         duration, against the measured HBM copy bandwidth.
cpu_baseline: the CPU oracle (decode + float64 matmul) on a bounded sample.

Multi-GPU: every rank owns an independent layer (weak scaling, no collective).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

MS = (1, 4, 16, 64)
PROJ = (("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336))
METRIC = "effective weight GB/s & fused matmul TFLOP/s at M=1..1024 vs HBM/tensor roofline"
WORKLOAD = "llama-3.1-8b MLP layer (gate/up/down), M in {1,4,16,64}, autotuned plans"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def rank_seed(proj_index: int, rank: int) -> int:
    """Seed of projection `proj_index` on `rank`: every rank owns an independent layer."""
    return 1 + proj_index + 100 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest `value` over all ranks (a no-op for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(bytes_per_rank: int, world: int, ms: float) -> float:
    """Whole-job GB/s: the bytes every rank processed over the slowest rank's time."""
    return bytes_per_rank * world / (ms * 1e-3) / 1e9


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (read-only)
    from a background thread every ~1 ms while the timed region runs; with a
    `csv_path` the samples are also written there."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, gpu_index: int, csv_path=None):
        self.gpu = gpu_index
        self.samples = []
        self.error = None
        self.path = csv_path

    def _run(self):
        import pynvml as N
        h = N.nvmlDeviceGetHandleByIndex(self.gpu)
        self.sm_max = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
        masks = [(name, getattr(N, attr)) for name, attr in self.REASONS]
        while not self.stop.is_set():
            sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
            reasons = N.nvmlDeviceGetCurrentClocksEventReasons(h)
            power = N.nvmlDeviceGetPowerUsage(h) / 1000.0
            self.samples.append((time.time(), sm, power, [n for n, m in masks if reasons & m]))
            self.stop.wait(0.001)

    def __enter__(self):
        import threading
        try:
            import pynvml as N
            N.nvmlInit()
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 2.0:
                time.sleep(0.001)
        except Exception as e:   # NVML missing: report it, keep benchmarking
            self.error = repr(e)
            self.thread = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=2)
        if self.thread is not None and self.path:
            try:
                os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
                with open(self.path, "w") as f:
                    f.write("time,sm_mhz,power_w,reasons\n")
                    for t, sm, pw, rs in self.samples:
                        f.write("%.4f,%d,%.1f,%s\n" % (t, sm, pw, "|".join(rs)))
            except OSError:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0,
                    "reasons": ["nvml unavailable: %s" % self.error]}
        reasons = sorted({r for _, _, _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(s[1] for s in self.samples), "sm_max_mhz": self.sm_max,
                "samples": len(self.samples), "power_w_max": max(s[2] for s in self.samples),
                "reasons": reasons, "source": "nvml, 1 ms polling during the timed region"}


# ----------------------------------------------------------------------------- CPU oracle leg

def oracle_sample(budget_s: float = 25.0):
    """Oracle pipeline (bit-by-bit Huffman decode + float64 matmul) for the gate
    projection at M = 1, 4, 16, 64, decoding once per M as the pipeline does.
    Stops after the M whose cumulative time passes budget_s."""
    from oracle import oracle as O
    from decode_gemm_exponent_b200 import synth
    n, k = PROJ[0][1], PROJ[0][2]
    w = synth.weights_bf16(n, k, 0.02, 0.0005, 1.0, seed=1)
    enc = O.encode(w)                      # offline, untimed
    done_bytes, t_total, done = 0, 0.0, []
    for m in MS:
        x = synth.activations_bf16(m, k, seed=1)
        t0 = time.perf_counter()
        wd = O.decode(enc)
        O.gemm(x, wd)
        t_total += time.perf_counter() - t0
        done_bytes += 2 * n * k
        done.append(m)
        if t_total > budget_s:
            break
    return done_bytes / t_total / 1e9, "gate [14336,4096] at M in %s, decode + float64 matmul" % (done,), t_total


def run_reference(args, rank):
    if rank != 0:
        return 0
    from oracle import oracle as O
    from decode_gemm_exponent_b200 import synth
    n, k = PROJ[0][1], PROJ[0][2]
    w = synth.weights_bf16(n, k, 0.02, 0.0005, 1.0, seed=1)
    enc = O.encode(w)
    x = synth.activations_bf16(1, k, seed=1)

    def step():
        wd = O.decode(enc)
        O.gemm(x, wd)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = 2 * n * k / dt / 1e9
    sample = "gate [14336,4096] at M=1 per step: bit-by-bit Huffman decode + float64 matmul"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "reference_sample": sample},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU leg

# DRAM traffic of a kernel group's launch on the 8B gate projection, from one
# ncu capture each (profiles/k_gemv_mma_traffic_8b_gate_m1.md and
# profiles/k_gemm_tc_traffic_8b_gate.md): bytes per launch, the algorithmic
# bytes of that launch, and a SHA-256 over the kernel's sources with comments
# and whitespace removed (source_digest); a figure is reported (scaled to the
# group's mean algorithmic bytes per launch) only while that code is unchanged.
MEASURED_TRAFFIC = {
    "fused/tcgen05_bn64": {
        "bytes": 93612544, "alg_bytes": 94085696,
        "files": ("decode_gemm_exponent_b200/csrc/gemm_tc.cu", "decode_gemm_exponent_b200/csrc/device_common.cuh"),
        "sha256": "278497e4e28f6a45f07770995e5484802aa2dbe40c47ac44886b387b4c4c694c",
    },
    "fused/tcgen05_bn16": {
        "bytes": 93028864, "alg_bytes": 90939968,
        "files": ("decode_gemm_exponent_b200/csrc/gemm_tc.cu", "decode_gemm_exponent_b200/csrc/device_common.cuh"),
        "sha256": "278497e4e28f6a45f07770995e5484802aa2dbe40c47ac44886b387b4c4c694c",
    },
    "fused/mma_gemv_s4_w2": {
        "bytes": 92293888, "alg_bytes": 89956928,
        "files": ("decode_gemm_exponent_b200/csrc/gemv_mma.cu", "decode_gemm_exponent_b200/csrc/device_common.cuh"),
        "sha256": "d7bf659f5a3bcaa34626548b4f4cb8c0f4afbd4ff09d140765941b6a8f6d69f1",
    },
}


def source_digest(texts) -> str:
    """SHA-256 over C/CUDA source texts with comments removed and every run of
    whitespace reduced to one space, so that an edit of a comment leaves it
    unchanged and an edit of the code does not.  String and character
    literals are kept as written."""
    import hashlib
    import re
    tok = re.compile(r'"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'|//[^\n]*|/\*.*?\*/', re.S)
    h = hashlib.sha256()
    for text in texts:
        code = tok.sub(lambda mt: mt.group(0) if mt.group(0)[0] in "\"'" else " ", text)
        h.update(" ".join(code.split()).encode())
        h.update(b"\0")
    return h.hexdigest()


def measured_traffic(group: str, alg_bytes_per_launch: float):
    """ncu DRAM bytes per launch of `group`, scaled by algorithmic bytes, or None."""
    rec = MEASURED_TRAFFIC.get(group)
    if rec is None:
        return None
    texts = []
    for f in rec["files"]:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            texts.append(fh.read())
    if source_digest(texts) != rec["sha256"]:
        return None
    return rec["bytes"] * alg_bytes_per_launch / rec["alg_bytes"]


def compression_stats(infos):
    """Size and exponent statistics of the layer's matrices (weighted by
    their weight counts): compressed size of each form as a fraction of BF16,
    Shannon entropy of the exponent byte, top-16 palette coverage and the
    fraction of 64-weight groups stored raw."""
    w = [i.n * i.k for i in infos]
    tot = sum(w)
    return {
        "compressed_fraction_huffman": round(sum(i.huffman_bytes for i in infos) / (2 * tot), 4),
        "compressed_fraction_palette": round(sum(i.palette_bytes for i in infos) / (2 * tot), 4),
        "exponent_entropy_bits": round(sum(i.entropy_bits * x for i, x in zip(infos, w)) / tot, 4),
        "top16_coverage": round(sum(i.top16_coverage * x for i, x in zip(infos, w)) / tot, 6),
        "raw_group_fraction": round(sum(i.n_raw for i in infos) / sum(i.n_groups for i in infos), 5),
    }


def alg_bytes(mat, m, plan):
    """Algorithmic HBM bytes of the kernels one matmul call launches: what
    each kernel must read of the compressed forms and write."""
    info = mat.info
    n, k = mat.n, mat.k
    nk = n * k
    flags = nk // 64 // 8                                   # raw bitmap (rank bases: as many)
    sm = info.section_bytes[0]                              # sign/mantissa plane
    raw = info.section_bytes[1] + flags                     # raw plane + rank bases
    stream = (info.stream_bits + 7) // 8 + (info.n_chunks + 1) * 4
    xy = m * k * 2 + m * n * 4
    fused_in = sm + raw + flags + nk // 2                   # palette form
    if plan.pipeline == 4:
        return {"fused": fused_in + xy}
    if plan.pipeline == 1:
        return {"decode": stream + flags + raw + sm + 2 * nk, "plain": 2 * nk + xy}
    if plan.pipeline == 2:
        # exponent plane + all-raw bitmap and rank words written, then read with the sm plane
        return {"exp_decode": stream + flags + raw + nk + 2 * flags, "fused": sm + nk + 2 * flags + xy}
    return {"transcode": stream + flags + nk // 2, "fused": fused_in + xy}


def plans_from_json(text, n_mats, uw):
    """Plans from a plan file written by the autotuner (--plan-json)."""
    plans = uw.plans_from_json(text, MS)
    if len(plans) != n_mats:
        raise ValueError("plan file holds %d matrices, the layer has %d" % (len(plans), n_mats))
    return plans


def launches_per_call(plan):
    n = 1 + (1 if plan.pipeline in (1, 2, 3) else 0)
    if plan.kernel == 2 and plan.split_k > 1:
        n += 1
    return n


def kernel_group(plan):
    kern = {1: "fma_gemv", 3: "mma_gemv_s%d_w%d" % (plan.bn, plan.stages)}.get(plan.kernel, "tcgen05_bn%d" % plan.bn)
    pipe = {1: "decode+plain", 2: "exp_decode+fused", 3: "transcode+fused", 4: "fused"}[plan.pipeline]
    return "%s/%s" % (pipe, kern)


def run_gpu(args, rank, world):
    import torch
    import torch.distributed as dist
    from decode_gemm_exponent_b200 import synth, uw

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()

    # ---- inputs (host encode is the offline step, outside any timing)
    mats = []
    for i, (name, n, k) in enumerate(PROJ):
        w = synth.weights_bf16(n, k, 0.02, 0.0005, 1.0, seed=rank_seed(i, rank))
        mats.append(uw.Matrix(uw.encode(w), device=dev))
    xs = {m: {k: torch.from_numpy(synth.activations_bf16(m, k, seed=m).view(np.int16)).to(dev)
              for k in {p[2] for p in PROJ}} for m in MS}

    if args.plans_in:
        with open(args.plans_in) as f:
            plan_json = f.read()
        plans = plans_from_json(plan_json, len(mats), uw)
    else:
        plans, plan_json = uw.autotune(mats, list(MS), reps=10)
    calls = []
    for j, m in enumerate(MS):
        for i, mat in enumerate(mats):
            p = plans[i][j]
            nb = mat.workspace_bytes(m, p)
            ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
            y = torch.empty(m, mat.n, dtype=torch.float32, device=dev)
            calls.append(dict(mat=mat, m=m, plan=p, ws=ws, y=y, x=xs[m][mat.k], name=PROJ[i][0]))
    stream = torch.cuda.current_stream()

    def issue(c):
        c["mat"].matmul(c["x"], c["plan"], y=c["y"], ws=c["ws"])

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        for c in calls:
            issue(c)
    for mat in mats:
        st = mat.device_status()
        if st != 0:
            raise RuntimeError("kernel status %d during warm-up" % st)

    # ---- device-resident timing of whole steps (only a start and an end event)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks_csv = args.clocks_csv.replace("{rank}", str(rank)) if args.clocks_csv else None
    with ClockSampler(local, clocks_csv) as clk:
        t_start.record(stream)
        for s in range(args.steps):
            for c in calls:
                issue(c)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    step_ms = max_over_ranks(t_start.elapsed_time(t_end) / args.steps, world, dev)
    weight_bytes = sum(2 * c["mat"].n * c["mat"].k for c in calls)
    value = aggregate_gbs(weight_bytes, world, step_ms)

    # ---- the same steps again with an event pair around every call, for the
    # per-kernel durations of the roofline (not part of `value`)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
          for _ in range(args.steps)]
    for s in range(args.steps):
        for c, (e0, e1) in zip(calls, ev[s]):
            e0.record(stream)
            issue(c)
            e1.record(stream)
    torch.cuda.synchronize()

    # per-call durations -> kernel groups
    per_call = [statistics.median(ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(args.steps))
                for i in range(len(calls))]
    groups = {}
    for c, ms_ in zip(calls, per_call):
        g = groups.setdefault(kernel_group(c["plan"]), {"ms": 0.0, "bytes": 0, "calls": 0})
        g["ms"] += ms_
        g["bytes"] += sum(alg_bytes(c["mat"], c["m"], c["plan"]).values())
        g["calls"] += 1
    dom_name, dom = max(groups.items(), key=lambda kv: kv[1]["ms"])
    achieved = dom["bytes"] / (dom["ms"] * 1e-3) / 1e9
    peak = float(peaks["hbm_gbs"])

    # ---- end-to-end through the C ABI with pinned host buffers.  As a
    # serving loop would, the copies run on their own streams ordered by
    # events: a step's inputs go up on one copy stream into one of two device
    # input sets (so they can be sent while the previous step still reads the
    # other set), every result comes down on another copy stream as soon as
    # its matmul ends, and the step's matmuls wait only for their inputs.
    hx = {(c["m"], c["mat"].k): c["x"].cpu().pin_memory() for c in calls}
    hy = [torch.empty_like(c["y"], device="cpu").pin_memory() for c in calls]
    h2d = sum(t.numel() * 2 for t in hx.values())
    d2h = sum(t.numel() * 4 for t in hy)
    xsets = [{key: xs[key[0]][key[1]] for key in hx}, {key: xs[key[0]][key[1]].clone() for key in hx}]
    copy_in, copy_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    x_ready = [ev() for _ in range(args.steps)]
    x_free = [ev() for _ in range(args.steps)]
    y_ready = [[ev() for _ in calls] for _ in range(args.steps)]
    y_free = [[ev() for _ in calls] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for s in range(args.steps):
        xset = xsets[s & 1]
        copy_in.wait_event(e0 if s < 2 else x_free[s - 2])     # matmuls of step s-2 read this set
        with torch.cuda.stream(copy_in):
            for key, t in hx.items():
                xset[key].copy_(t, non_blocking=True)
        x_ready[s].record(copy_in)
        stream.wait_event(x_ready[s])
        for i, (c, h) in enumerate(zip(calls, hy)):
            if s > 0:
                stream.wait_event(y_free[s - 1][i])              # last step's result is on the host
            c["mat"].matmul(xset[(c["m"], c["mat"].k)], c["plan"], y=c["y"], ws=c["ws"])
            y_ready[s][i].record(stream)
            copy_out.wait_event(y_ready[s][i])
            with torch.cuda.stream(copy_out):
                h.copy_(c["y"], non_blocking=True)
            y_free[s][i].record(copy_out)
        x_free[s].record(stream)
    stream.wait_stream(copy_out)                                # every result is on the host
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    for mat in mats:
        st = mat.device_status()
        if st != 0:
            raise RuntimeError("kernel status %d after timing" % st)

    if rank != 0:
        return 0
    clocks = clk.summary()
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, sample, secs = oracle_sample()
        cpu = {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
               "seconds": round(secs, 2)}
    infos = [m.info for m in mats]
    out = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": WORKLOAD,
            "l2": "no flush: each matrix is re-read after >= 160 MB of other matrices (inputs larger than L2)",
            **compression_stats(infos),
            "plans": {"%s@M=%d" % (c["name"], c["m"]): kernel_group(c["plan"]) +
                      ("/split%d" % c["plan"].split_k if c["plan"].kernel == 2 else "") for c in calls},
            "per_call_us": {"%s@M=%d" % (c["name"], c["m"]): round(1e3 * t, 2) for c, t in zip(calls, per_call)},
        },
        "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak,
                     "traffic": measured_traffic(dom_name, dom["bytes"] / dom["calls"]),
                     "peak_source": peaks["_source"] + " hbm_gbs"},
        "cpu_baseline": cpu,
        "e2e": {"value": aggregate_gbs(weight_bytes, world, e2e_ms), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": sum(launches_per_call(c["plan"]) for c in calls) * args.steps,   # the timed region
        "clocks": clocks,
    }
    if args.plan_json:
        with open(args.plan_json, "w") as f:
            f.write(plan_json)
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="uw", choices=["uw", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-csv", default=None,
                    help="also write the clock samples of the timed region to this CSV ({rank} = rank)")
    ap.add_argument("--plan-json", default=None, help="write the autotuner's plan file here")
    ap.add_argument("--plans-in", default=None, help="use this plan file instead of autotuning")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_gpu(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
