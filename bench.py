"""Benchmark: effective weight bandwidth and fused-matmul throughput of the
compressed Llama MLP projections on one B200 (or N, one independent layer
per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --case kernel|stack|moe|sweep70b [options]

Default case (one "step"): one Llama-3.1-8B-shaped MLP layer -- gate and up
[14336, 4096], down [4096, 14336], BF16 N(0, 0.02^2) with 0.05% N(0, 1)
outliers (seeds 1, 2, 3; rank r adds 100 r) -- multiplied by activations X of
M = 1, 4, 16 and 64 rows (12 matmuls, Y = X W^T, fp32 out).  Each
(projection, M) runs the plan picked by libuw's autotuner.  Matmuls are
issued M-outer / projection-inner, so two other matrices (>= 160 MB) stream
between two uses of one matrix and each read comes from HBM, not from the
126 MB L2.

value  = sum over the step's matmuls of 2*N*K (uncompressed BF16 weight bytes)
         / step time  [GB/s], inputs resident in HBM, CUDA events, max over ranks.
e2e    = the same, with X copied from pinned host memory and Y read back to
         pinned host memory inside the timed region, through the C ABI (copies
         on their own streams, ordered by events; inputs and results double-
         buffered, so a step's copies overlap the neighbouring steps' matmuls).
plain_bf16: the same 12 calls with the same plans on uncompressed BF16 weights.
large_m: the same layer at M = 256, 512 and 1024 (fused TFLOP/s against the
         dense BF16 tensor peak, next to decode + GEMM and uncompressed BF16).
roofline: the kernel group with the largest share of the step; achieved =
         its algorithmic bytes (compressed planes + X + Y) / its event-timed
         duration, against the measured HBM copy bandwidth.
cpu_baseline: the CPU oracle (bit-by-bit decode + float64 matmul) on a row
         sample of the same 12 calls, on every host core and on one.

Other cases (one JSON line per measurement, nothing timed by the driver):
  kernel   one kernel on one synthetic matrix, for timing or ncu capture
  stack    32-layer 8B MLP stack with cross-layer overlap (decodes on a side
           stream) and the decode/compute SM split tuner
  moe      routed experts of a mixture-of-experts projection, batched vs one
           call per expert
  sweep70b Llama-70B MLP projections over outlier fraction x sigma x M

Multi-GPU: every rank owns an independent layer (weak scaling, no collective).
"""
from __future__ import annotations

import argparse
import json
import multiprocessing as mp
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

MS = (1, 4, 16, 64)
MS_LARGE = (256, 512, 1024)
PROJ = (("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336))
METRIC = "effective weight GB/s & fused matmul TFLOP/s at M=1..1024 vs HBM/tensor roofline"
WORKLOAD = "llama-3.1-8b MLP layer (gate/up/down), M in {1,4,16,64}, autotuned plans"
L2_NOTE = "no flush: each matrix is re-read after >= 160 MB of other matrices (inputs larger than L2)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ORACLE_ROW_FRACTION = 16      # the oracle sample keeps 1/16 of each matrix's rows
ORACLE_PART_ROWS = 128        # ... in parts of 128 rows, one pool task each


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


def workload_config():
    """The `config` object of both arms: what defines the workload, nothing else."""
    return {"workload": WORKLOAD, "l2": L2_NOTE}


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
#
# The oracle runs the step's 12 calls (decode of the matrix + float64 matmul,
# as pipeline 1 does per call) on a row sample of each matrix: the first
# 1/ORACLE_ROW_FRACTION of its rows, encoded on its own by the oracle (same
# recipe and seeds, so the same weight statistics).  Each call's sample is
# cut into parts of ORACLE_PART_ROWS rows, each encoded on its own, so that a
# step is many equal-sized tasks and a spawn process pool on every host core
# stays busy; a step's wall time covers all 12 calls.

_ORACLE = {}


def oracle_sample_rows(n: int) -> int:
    return max(64, n // ORACLE_ROW_FRACTION)


def oracle_parts(n: int) -> int:
    return max(1, oracle_sample_rows(n) // ORACLE_PART_ROWS)


def _oracle_init(rank: int):
    from oracle import oracle as O
    from decode_gemm_exponent_b200 import synth
    for i, (_, n, k) in enumerate(PROJ):
        w = synth.weights_bf16(n, k, 0.02, 0.0005, 1.0, seed=rank_seed(i, rank))[:oracle_sample_rows(n)]
        rows = w.shape[0] // oracle_parts(n)
        for p in range(oracle_parts(n)):              # offline, untimed
            _ORACLE[("w", i, p)] = O.encode(w[p * rows:(p + 1) * rows])
    for m in MS:
        for k in {p[2] for p in PROJ}:
            _ORACLE[("x", m, k)] = synth.activations_bf16(m, k, seed=m)


def _oracle_call(task):
    from oracle import oracle as O
    i, m, p = task
    enc = _ORACLE[("w", i, p)]
    t0 = time.perf_counter()
    wd = O.decode(enc)
    O.gemm(_ORACLE[("x", m, enc.k)], wd)
    return time.perf_counter() - t0


def oracle_tasks():
    # the largest calls first, so that the pool ends on short tasks
    tasks = [(i, m, p) for m in MS for i, (_, n, _) in enumerate(PROJ) for p in range(oracle_parts(n))]
    return sorted(tasks, key=lambda t: -t[1] * PROJ[t[0]][2])


def oracle_step_bytes() -> int:
    return sum(2 * oracle_sample_rows(n) * k for m in MS for (_, n, k) in PROJ)


def oracle_sample_text(workers: int) -> str:
    rows = ", ".join("%s %d of %d rows" % (nm, oracle_sample_rows(n), n) for nm, n, _ in PROJ)
    return ("the step's 12 calls (M in %s x gate/up/down), each bit-by-bit Huffman decode + float64 matmul, "
            "on a row sample (%s) in parts of %d rows, %d worker process%s"
            % (list(MS), rows, ORACLE_PART_ROWS, workers, "" if workers == 1 else "es"))


class OracleRunner:
    """The oracle's step on `workers` processes (1: in this process)."""

    def __init__(self, workers: int, rank: int = 0):
        self.workers = workers
        self.pool = None
        if workers > 1:
            self.pool = mp.get_context("spawn").Pool(workers, initializer=_oracle_init, initargs=(rank,))
        else:
            _oracle_init(rank)

    def step(self) -> float:
        t0 = time.perf_counter()
        if self.pool is not None:
            self.pool.map(_oracle_call, oracle_tasks(), chunksize=1)
        else:
            for t in oracle_tasks():
                _oracle_call(t)
        return time.perf_counter() - t0

    def close(self):
        if self.pool is not None:
            self.pool.close()
            self.pool.join()


def oracle_throughput(workers: int, budget_s: float, min_steps: int = 1):
    """GB/s of the oracle's sampled steps run for about budget_s (after one warm-up step)."""
    r = OracleRunner(workers)
    try:
        r.step()
        total, steps = 0.0, 0
        while steps < min_steps or total < budget_s:
            total += r.step()
            steps += 1
    finally:
        r.close()
    return oracle_step_bytes() * steps / total / 1e9, steps, total


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, rank):
    """The oracle as the reference arm: the same workload and config, each
    step a row sample of the step's 12 calls, on every host core."""
    if rank != 0:
        return 0
    workers = min(host_cores(), len(oracle_tasks()))
    r = OracleRunner(workers)
    try:
        for _ in range(args.warmup):
            r.step()
        total = sum(r.step() for _ in range(args.steps))
    finally:
        r.close()
    dt = total / args.steps
    value = oracle_step_bytes() / dt / 1e9
    sample = oracle_sample_text(workers)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": workers, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU leg

# DRAM traffic of a kernel group's launch on the 8B gate projection, from one
# ncu capture each (profiles/): bytes per launch, the algorithmic bytes of
# that launch, and a SHA-256 over the kernel's sources with comments and
# whitespace removed (source_digest); a figure is reported (scaled to the
# group's mean algorithmic bytes per launch) only while that code is unchanged.
MEASURED_TRAFFIC = {
    "fused/mma_gemv_s4_w2": {
        "bytes": 93354496, "alg_bytes": 90053056,
        "files": ("decode_gemm_exponent_b200/csrc/gemv_mma.cu", "decode_gemm_exponent_b200/csrc/device_common.cuh"),
        "sha256": "0c3c9bfe77a48482f36535771ae0dc6284161f7274b914ece782a64ad89656b7",
    },
    "fused/tcgen05_bn16": {
        "bytes": 93274368, "alg_bytes": 91036096,
        "files": ("decode_gemm_exponent_b200/csrc/gemm_tc.cu", "decode_gemm_exponent_b200/csrc/device_common.cuh"),
        "sha256": "350c214b73223a30fc576bab087a9219cf0d14ad5914cde7ab5cc3e4c2ed3fb3",
    },
    "fused/tcgen05_bn64": {
        "bytes": 93622784, "alg_bytes": 94181824,
        "files": ("decode_gemm_exponent_b200/csrc/gemm_tc.cu", "decode_gemm_exponent_b200/csrc/device_common.cuh"),
        "sha256": "350c214b73223a30fc576bab087a9219cf0d14ad5914cde7ab5cc3e4c2ed3fb3",
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
    if plan.pipeline == 5:
        # the Huffman form (stream, chunk offsets, bitmap, raw plane, sign/mantissa) read by one kernel
        return {"fused": stream + flags + raw + sm + xy}
    if plan.pipeline == 1:
        return {"decode": stream + flags + raw + sm + 2 * nk, "plain": 2 * nk + xy}
    if plan.pipeline == 2:
        # exponent plane + all-raw bitmap and rank words written, then read with the sm plane
        return {"exp_decode": stream + flags + raw + nk + 2 * flags, "fused": sm + nk + 2 * flags + xy}
    return {"transcode": stream + flags + nk // 2, "fused": fused_in + xy}


def plans_from_json(text, n_mats, uw, ms=MS):
    """Plans from a plan file written by the autotuner (--plan-json)."""
    plans = uw.plans_from_json(text, ms)
    if len(plans) != n_mats:
        raise ValueError("plan file holds %d matrices, the layer has %d" % (len(plans), n_mats))
    return plans


def launches_per_call(plan):
    n = 1 + (1 if plan.pipeline in (1, 2, 3) else 0)
    if plan.kernel == 2 and plan.split_k > 1:
        n += 1
    return n


def kernel_name(plan):
    return {1: "fma_gemv", 3: "mma_gemv_s%d_w%d" % (plan.bn, plan.stages),
            4: "tc_sk_bn%d" % plan.bn, 5: "mma_sk_w%d_s%d" % (plan.bn, plan.stages)}.get(
                plan.kernel, "tcgen05_bn%d" % plan.bn)


def kernel_group(plan):
    pipe = {1: "decode+plain", 2: "exp_decode+fused", 3: "transcode+fused", 4: "fused",
            5: "huffman_fused"}[plan.pipeline]
    return "%s/%s" % (pipe, kernel_name(plan))


def plan_label(plan):
    return kernel_group(plan) + ("/split%d" % plan.split_k if plan.kernel == 2 else "")


def same_plan(uw, p, pipeline=None):
    return uw.make_plan(p.pipeline if pipeline is None else pipeline, p.kernel, p.bn, p.split_k, p.stages)


def time_steps(torch, stream, steps, issue_all):
    """Mean ms per step of `steps` back-to-back runs of issue_all(), CUDA events."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        issue_all()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_gpu(args, rank, world):
    import torch
    import torch.distributed as dist
    from decode_gemm_exponent_b200 import synth, uw

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()

    # ---- inputs (host encode is the offline step, outside any timing)
    mats, plain_w = [], []
    for i, (name, n, k) in enumerate(PROJ):
        w = synth.weights_bf16(n, k, 0.02, 0.0005, 1.0, seed=rank_seed(i, rank))
        mats.append(uw.Matrix(uw.encode(w), device=dev))
        plain_w.append(torch.from_numpy(w.view(np.int16)).to(dev))
    all_ms = MS + MS_LARGE
    xs = {m: {k: torch.from_numpy(synth.activations_bf16(m, k, seed=m).view(np.int16)).to(dev)
              for k in {p[2] for p in PROJ}} for m in all_ms}

    if args.plans_in:
        with open(args.plans_in) as f:
            plan_json = f.read()
        plans = plans_from_json(plan_json, len(mats), uw, all_ms)
    else:
        plans, plan_json = uw.autotune(mats, list(all_ms), reps=10)

    def make_calls(ms_list):
        calls = []
        for m in ms_list:
            j = all_ms.index(m)
            for i, mat in enumerate(mats):
                p = plans[i][j]
                ws = torch.zeros(max(mat.workspace_bytes(m, p), 256), dtype=torch.uint8, device=dev)
                # the BF16 twin gets a workspace of its own: a stream-K plan keeps its tile
                # counters where a preprocessing pipeline's output would lie in a shared one
                ws_plain = torch.zeros(max(mat.workspace_bytes(m, same_plan(uw, p, 4)), 256), dtype=torch.uint8,
                                       device=dev)
                y = torch.empty(m, mat.n, dtype=torch.float32, device=dev)
                calls.append(dict(mat=mat, m=m, plan=p, ws=ws, ws_plain=ws_plain, y=y, x=xs[m][mat.k],
                                  name=PROJ[i][0],
                                  w=plain_w[i]))
        return calls

    calls = make_calls(MS)
    stream = torch.cuda.current_stream()

    def issue(c):
        c["mat"].matmul(c["x"], c["plan"], y=c["y"], ws=c["ws"])

    def issue_plain(c):
        uw.matmul_bf16(c["x"], c["w"], c["plan"], y=c["y"], ws=c["ws_plain"])

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
    barrier()
    clocks_csv = args.clocks_csv.replace("{rank}", str(rank)) if args.clocks_csv else None
    with ClockSampler(local, clocks_csv) as clk:
        step_ms = time_steps(torch, stream, args.steps, lambda: [issue(c) for c in calls])
    barrier()
    step_ms = max_over_ranks(step_ms, world, dev)
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

    # ---- uncompressed BF16 twin: the same 12 calls, same kernels, plain weights
    for _ in range(2):
        for c in calls:
            issue_plain(c)
    plain_ms = max_over_ranks(time_steps(torch, stream, args.steps, lambda: [issue_plain(c) for c in calls]),
                              world, dev)

    # ---- large M: fused, decode + GEMM (pipeline 1, same kernel), plain BF16
    large = {}
    lcalls = make_calls(MS_LARGE)
    t_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    lsteps = max(3, args.steps // 4)
    for m in MS_LARGE:
        cs = [c for c in lcalls if c["m"] == m]
        dec = []
        for c in cs:
            p1 = same_plan(uw, c["plan"], 1)
            dec.append(dict(c, plan=p1, ws=torch.zeros(max(c["mat"].workspace_bytes(m, p1), 256),
                                                        dtype=torch.uint8, device=dev)))
        for c in cs + dec:
            issue(c)
        for c in cs:
            issue_plain(c)
        flops = sum(2.0 * m * c["mat"].n * c["mat"].k for c in cs)
        t_f = max_over_ranks(time_steps(torch, stream, lsteps, lambda: [issue(c) for c in cs]), world, dev)
        t_d = max_over_ranks(time_steps(torch, stream, lsteps, lambda: [issue(c) for c in dec]), world, dev)
        t_p = max_over_ranks(time_steps(torch, stream, lsteps, lambda: [issue_plain(c) for c in cs]), world, dev)
        tf = flops * world / (t_f * 1e-3) / 1e12
        large["M=%d" % m] = {
            "fused_tflops": round(tf, 1), "fused_tensor_frac": round(tf / world / t_peak, 4),
            "fused_us": round(1e3 * t_f, 1),
            "decode_gemm_tflops": round(flops * world / (t_d * 1e-3) / 1e12, 1),
            "plain_bf16_tflops": round(flops * world / (t_p * 1e-3) / 1e12, 1),
            "plans": {c["name"]: plan_label(c["plan"]) for c in cs},
        }
    for mat in mats:
        st = mat.device_status()
        if st != 0:
            raise RuntimeError("kernel status %d after the large-M runs" % st)
    del lcalls

    # ---- end-to-end through the C ABI with pinned host buffers.  As a
    # serving loop would, the copies run on their own streams ordered by
    # events, and inputs and results are double-buffered: a step's inputs go
    # up on one copy stream into one of two device input sets (while the
    # previous step still reads the other), its 12 matmuls run back to back
    # into one of two result sets (so the early start of each matmul is not
    # broken by event operations between them), and the step's results come
    # down on another copy stream while the next step computes.  A step's
    # inputs are one pinned host buffer (every (M, K) activation block back to
    # back) and go up in one copy; its 12 results are views of one device
    # buffer and come down in one copy: few large copies, not 20 small ones.
    xkeys = sorted({(c["m"], c["mat"].k) for c in calls})
    x_off = np.cumsum([0] + [m * k for m, k in xkeys])
    y_off = np.cumsum([0] + [c["m"] * c["mat"].n for c in calls])
    hx = torch.empty(int(x_off[-1]), dtype=torch.int16).pin_memory()
    for i, (m, k) in enumerate(xkeys):
        hx[int(x_off[i]):int(x_off[i + 1])].copy_(xs[m][k].reshape(-1).cpu())
    hy = torch.empty(int(y_off[-1]), dtype=torch.float32).pin_memory()
    h2d, d2h = hx.numel() * 2, hy.numel() * 4
    dx = [torch.empty_like(hx, device=dev) for _ in range(2)]
    dy = [torch.empty_like(hy, device=dev) for _ in range(2)]
    xsets = [{key: dx[b][int(x_off[i]):int(x_off[i + 1])].view(key[0], key[1]) for i, key in enumerate(xkeys)}
             for b in range(2)]
    ysets = [[dy[b][int(y_off[i]):int(y_off[i + 1])].view(c["m"], c["mat"].n) for i, c in enumerate(calls)]
             for b in range(2)]
    copy_in, copy_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    mk = lambda: torch.cuda.Event()
    x_ready = [mk() for _ in range(args.steps)]
    x_free = [mk() for _ in range(args.steps)]
    y_ready = [mk() for _ in range(args.steps)]
    y_free = [mk() for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for s in range(args.steps):
        xset, yset = xsets[s & 1], ysets[s & 1]
        copy_in.wait_event(e0 if s < 2 else x_free[s - 2])     # matmuls of step s-2 read this set
        with torch.cuda.stream(copy_in):
            dx[s & 1].copy_(hx, non_blocking=True)
        x_ready[s].record(copy_in)
        stream.wait_event(x_ready[s])
        if s >= 2:
            stream.wait_event(y_free[s - 2])                    # step s-2's results (this set) are on the host
        for c, y in zip(calls, yset):
            c["mat"].matmul(xset[(c["m"], c["mat"].k)], c["plan"], y=y, ws=c["ws"])
        x_free[s].record(stream)
        y_ready[s].record(stream)
        copy_out.wait_event(y_ready[s])
        with torch.cuda.stream(copy_out):
            hy.copy_(dy[s & 1], non_blocking=True)
        y_free[s].record(copy_out)
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
        cores = host_cores()
        v1, st1, s1 = oracle_throughput(1, args.cpu_seconds / 2)
        vn, stn, sn = oracle_throughput(min(cores, len(oracle_tasks())), args.cpu_seconds / 2, min_steps=3)
        workers = min(cores, len(oracle_tasks()))
        cpu = {"value": vn, "unit": "GB/s", "cores": workers, "kind": "oracle",
               "sample": oracle_sample_text(workers) + "; %d steps in %.1f s" % (stn, sn),
               "host_cores": cores,
               "single_core": {"value": v1, "unit": "GB/s", "cores": 1,
                               "sample": oracle_sample_text(1) + "; %d steps in %.1f s" % (st1, s1)}}
    infos = [m.info for m in mats]
    out = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(),
        "details": {
            **compression_stats(infos),
            "plans": {"%s@M=%d" % (c["name"], c["m"]): plan_label(c["plan"]) for c in calls},
            "per_call_us": {"%s@M=%d" % (c["name"], c["m"]): round(1e3 * t, 2) for c, t in zip(calls, per_call)},
        },
        "plain_bf16": {"value": aggregate_gbs(weight_bytes, world, plain_ms), "unit": "GB/s",
                       "ms_per_step": plain_ms,
                       "what": "the same 12 calls with the same kernels and plans on uncompressed BF16 weights"},
        "large_m": {"peak_tflops": t_peak, "peak_source": peaks["_source"] + " bf16_tflops", **large},
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


# ----------------------------------------------------------------------------- other cases

def case_kernel(argv):
    """One libuw kernel on one synthetic matrix, for timing or profiler capture:
    one warm-up launch, then --reps timed launches (CUDA events) -- back to
    back after one more untimed launch, or (--flush) each on its own after a
    512 MB read; prints the per-launch time and the algorithmic bytes / FLOPs
    per launch.  Under ncu, `-s 1 -c 1` captures the second launch."""
    ap = argparse.ArgumentParser(prog="bench.py --case kernel")
    ap.add_argument("--kernel", required=True,
                    choices=["decode", "exp_decode", "transcode", "fma", "tc", "mma", "sk", "mma_sk",
                             "plain_fma", "plain_tc", "plain_mma", "plain_sk", "plain_mma_sk"])
    ap.add_argument("--n", type=int, default=28672)
    ap.add_argument("--k", type=int, default=8192)
    ap.add_argument("--m", type=int, default=1)
    ap.add_argument("--bn", type=int, default=0,
                    help="TC token tile, FMA rows per warp, MMA K slices or MMA_SK warps per SM")
    ap.add_argument("--split", type=int, default=1)
    ap.add_argument("--stages", type=int, default=0)
    ap.add_argument("--pipeline", type=int, default=4, help="fused kernels: 4 (palette plane) or 3 / 2")
    ap.add_argument("--sigma", type=float, default=0.015)
    ap.add_argument("--frac", type=float, default=0.0005)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--flush", action="store_true",
                    help="read 512 MB before each timed call (weights come from HBM, not L2; "
                         "a read leaves no dirty lines to write back) and time every call on its own")
    a = ap.parse_args(argv)
    import torch
    from decode_gemm_exponent_b200 import synth, uw

    w = synth.weights_bf16(a.n, a.k, a.sigma, a.frac, 1.0, a.seed)
    mat = uw.Matrix(uw.encode(w))
    info = mat.info
    x = torch.from_numpy(synth.activations_bf16(a.m, a.k, a.seed).view(np.int16)).cuda()
    y = torch.empty(a.m, a.n, dtype=torch.float32, device="cuda")
    nk = a.n * a.k
    # bytes each kernel reads of the compressed forms: the raw bitmap (nk/512)
    # and its rank bases (nk/512); the Huffman stream and chunk offsets; the
    # raw plane; the sign/mantissa plane (the transcode needs only the stream
    # and the bitmap, the exponent decode no sign/mantissa bytes)
    flags = nk // 64 // 8
    stream = (info.stream_bits + 7) // 8 + (info.n_chunks + 1) * 4
    raw = info.section_bytes[uw.SEC_RAWEXP] + flags
    sm = info.section_bytes[uw.SEC_SM]
    common = sm + raw + flags
    huff_in = common + stream
    xy = a.m * a.k * 2 + a.m * a.n * 4
    flops = 2.0 * a.m * nk
    kind = a.kernel.replace("plain_", "")
    if kind == "fma":
        plan = uw.make_plan(a.pipeline, uw.KERNEL_FMA, a.bn or 1, 1)
    elif kind == "mma":
        plan = uw.make_plan(a.pipeline, uw.KERNEL_MMA, a.bn or 2, 1, a.stages)
    elif kind == "sk":
        plan = uw.make_plan(a.pipeline, uw.KERNEL_TC_SK, a.bn or 16, 1, a.stages)
    elif kind == "mma_sk":
        plan = uw.make_plan(a.pipeline, uw.KERNEL_MMA_SK, a.bn or 8, 1, a.stages)
    else:
        plan = uw.make_plan(a.pipeline, uw.KERNEL_TC, a.bn or 16, a.split, a.stages)
    preprocessing = a.kernel in ("decode", "exp_decode", "transcode")
    ws_bytes = 0 if preprocessing else uw.workspace_size(a.m, a.n, a.k, plan)
    ws = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    if a.kernel == "decode":
        out = torch.empty(a.n, a.k, dtype=torch.int16, device="cuda")
        run = lambda: mat.decode(out)
        alg = huff_in + 2 * nk
    elif a.kernel == "exp_decode":
        out = torch.empty(a.n, a.k, dtype=torch.uint8, device="cuda")
        run = lambda: mat.decode_exponents(out)
        alg = stream + flags + raw + nk
    elif a.kernel == "transcode":
        out = torch.empty(nk // 2, dtype=torch.uint8, device="cuda")
        run = lambda: mat.transcode(out)
        alg = stream + flags + nk // 2
    elif not a.kernel.startswith("plain_"):
        run = lambda: mat.matmul(x, plan, y=y, ws=ws)
        alg = sum(alg_bytes(mat, a.m, plan).values())
    else:
        wd = torch.from_numpy(w.view(np.int16)).cuda()
        run = lambda: uw.matmul_bf16(x, wd, plan, y=y, ws=ws)
        alg = 2 * nk + xy
    run()
    torch.cuda.synchronize()
    assert mat.device_status() == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.flush:
        scrub = torch.zeros(128 << 20, dtype=torch.int32, device="cuda")   # 512 MB: also covers the host launch time
        total = 0.0
        for _ in range(a.reps):
            scrub.sum()
            e0.record()
            run()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        us = 1e3 * total / a.reps
    else:
        # one untimed launch first, so that the GPU is busy while the host
        # issues the start event and the timed launches: the host's issue
        # time of the first timed launch does not count as GPU time
        run()
        e0.record()
        for _ in range(a.reps):
            run()
        e1.record()
        torch.cuda.synchronize()
        us = 1e3 * e0.elapsed_time(e1) / a.reps
    print(json.dumps({"kernel": a.kernel, "n": a.n, "k": a.k, "m": a.m, "bn": plan.bn, "pipeline": plan.pipeline,
                      "split": plan.split_k, "us": us, "alg_bytes": int(alg),
                      "gbs": alg / us / 1e3, "tflops": None if preprocessing else flops / us / 1e6,
                      "l2": "flushed before each call" if a.flush else
                      ("not flushed; the kernel's %.0f MB exceed the 126 MB L2" % (alg / 1e6) if alg > 126e6 else
                       "not flushed: %.0f MB can stay in the 126 MB L2 between calls" % (alg / 1e6))}))
    return 0


def _encode_job(job):
    """Host encode of one synthetic matrix in a spawn worker (before any CUDA call)."""
    n, k, sigma, frac, seed = job
    from decode_gemm_exponent_b200 import synth, uw
    return uw.encode(synth.weights_bf16(n, k, sigma, frac, 1.0, seed=seed))


def _encode_all(jobs, workers):
    with mp.get_context("spawn").Pool(max(1, min(workers, len(jobs)))) as pool:
        return pool.map(_encode_job, jobs, chunksize=1)


def case_stack(argv):
    """Cross-layer overlap on a stack of Llama-3.1-8B-shaped MLP layers
    (Unweight page §八): uw_stack_run with the decodes on a side stream
    against the same stack on one stream, and the decode/compute SM split
    chosen by uw_stack_tune_split.  Layers: gate and up [14336, 4096], down
    [4096, 14336], N(0, 0.02^2) with 0.05% N(0, 1) outliers, seed
    100 * layer + projection.  Plan sets per M: "autotuned" (the autotuner's
    per-(projection, M) plans on layer 0, used for every layer) and
    "alternating" (even layers full decode + plain kernel, odd layers the
    fused palette kernel, each with the autotuned kernel choice)."""
    ap = argparse.ArgumentParser(prog="bench.py --case stack")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--ms", type=int, nargs="+", default=[1, 64, 1024])
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--workers", type=int, default=min(32, host_cores()))
    ap.add_argument("--splits", type=int, nargs="+", default=[0, 16, 32],
                    help="preprocessing SM counts tried by the split tuner (0 = no split)")
    a = ap.parse_args(argv)
    jobs = [(n, k, 0.02, 0.0005, 100 * layer + i) for layer in range(a.layers) for i, (_, n, k) in enumerate(PROJ)]
    blobs = _encode_all(jobs, a.workers)

    import torch
    from decode_gemm_exponent_b200 import synth, uw
    mats = [uw.Matrix(b) for b in blobs]
    del blobs
    ms = sorted(set(a.ms))
    xs = {(m, k): torch.from_numpy(synth.activations_bf16(m, k, seed=m).view(np.int16)).cuda()
          for m in ms for k in {s[2] for s in PROJ}}
    plans, _ = uw.autotune(mats[:3], ms, reps=5)
    side = torch.cuda.Stream()
    main_s = torch.cuda.current_stream()
    weight_bytes = sum(2 * mat.n * mat.k for mat in mats)

    def timed(stack, side_stream):
        for _ in range(a.warmup):
            stack.run(side_stream=side_stream)
        return 1e3 * time_steps(torch, main_s, a.reps, lambda: stack.run(side_stream=side_stream))

    for j, m in enumerate(ms):
        for kind in ("autotuned", "alternating"):
            steps = []
            for idx, mat in enumerate(mats):
                layer, proj = divmod(idx, 3)
                plan = same_plan(uw, plans[proj][j])
                if kind == "alternating":
                    plan.pipeline = uw.PIPE_DECODE_GEMM if layer % 2 == 0 else uw.PIPE_DIRECT_PALETTE
                y = torch.empty(m, mat.n, dtype=torch.float32, device="cuda")
                steps.append((mat, xs[(m, mat.k)], y, plan))
            stack = uw.Stack(steps)
            us_overlap = timed(stack, side)
            us_serial = timed(stack, None)
            if any(mat.device_status() != 0 for mat in mats[:3]):
                raise RuntimeError("kernel status during the stack run")
            best_split, split_us = stack.tune_split(a.splits, reps=a.reps)
            if any(mat.device_status() != 0 for mat in mats[:3]):
                raise RuntimeError("kernel status during the split tuning")
            n_prep = sum(1 for s in steps if s[3].pipeline != uw.PIPE_DIRECT_PALETTE)
            print(json.dumps({
                "workload": "llama-3.1-8b MLP stack", "layers": a.layers, "m": m, "plans": kind,
                "steps": len(steps), "preprocessed_steps": n_prep,
                "us_overlap": round(us_overlap, 1), "us_one_stream": round(us_serial, 1),
                "speedup": round(us_serial / us_overlap, 4),
                "weight_gbs_overlap": round(weight_bytes / us_overlap / 1e3, 1),
                "weight_gbs_one_stream": round(weight_bytes / us_serial / 1e3, 1),
                "tflops_overlap": round(2.0 * m * weight_bytes / 2 / us_overlap / 1e6, 1),
                "split_best_prep_sms": best_split,
                "split_us": {str(c): round(u, 1) for c, u in zip(a.splits, split_us)},
                "plan_per_projection": [plan_label(plans[p][j]) for p in range(3)],
            }), flush=True)
            del stack, steps
    return 0


def case_moe(argv):
    """The routed experts of one mixture-of-experts projection, all in one
    batched call (uw_fused_matmul_batched) against one uw_fused_matmul call
    per expert.  Experts: N(0, 0.02^2) with 0.05% N(0, 1) outliers, expert e
    seeded e + 1, palette form.  Routing: each of T tokens picks `topk`
    distinct experts uniformly at random (seed T).  Each timed call follows a
    512 MB read (weights stream from HBM) and is timed on its own, both
    issued from Python and replayed from a CUDA graph."""
    ap = argparse.ArgumentParser(prog="bench.py --case moe")
    ap.add_argument("--experts", type=int, default=128)
    ap.add_argument("--n", type=int, default=768)
    ap.add_argument("--k", type=int, default=2048)
    ap.add_argument("--topk", type=int, default=8)
    ap.add_argument("--tokens", type=int, nargs="+", default=[1, 4, 16])
    ap.add_argument("--slices", type=int, default=4)
    ap.add_argument("--reps", type=int, default=10)
    a = ap.parse_args(argv)
    import torch
    from decode_gemm_exponent_b200 import synth, uw

    mats = [uw.Matrix(uw.encode(synth.weights_bf16(a.n, a.k, 0.02, 0.0005, 1.0, seed=e + 1)))
            for e in range(a.experts)]
    plan = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, a.slices, 1, 0)
    scrub = torch.zeros(128 << 20, dtype=torch.int32, device="cuda")   # 512 MB, read before each call
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(a.reps):
            scrub.sum()
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        return 1e3 * total / a.reps

    for t in a.tokens:
        rng = np.random.default_rng(t)
        counts = np.zeros(a.experts, np.int64)
        for _ in range(t):
            counts[rng.choice(a.experts, a.topk, replace=False)] += 1
        items = []
        for e in np.nonzero(counts)[0]:
            m = int(counts[e])
            x = torch.from_numpy(synth.activations_bf16(m, a.k, seed=int(e)).view(np.int16)).cuda()
            items.append((mats[e], x, torch.empty(m, a.n, dtype=torch.float32, device="cuda")))
        ys_single = [torch.empty_like(y) for _, _, y in items]
        run_batched = lambda: uw.fused_matmul_batched(items, plan)
        run_loop = lambda: [mat.matmul(x, plan, y=ys) for (mat, x, _), ys in zip(items, ys_single)]
        us_batched = timed(run_batched)
        us_loop = timed(run_loop)
        graphs = []
        for fn in (run_batched, run_loop):
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                fn()                                   # warm-up outside the capture
            torch.cuda.current_stream().wait_stream(side)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            graphs.append(g)
        us_batched_g = timed(graphs[0].replay)
        us_loop_g = timed(graphs[1].replay)
        same = all(torch.equal(y.view(torch.int32), ys.view(torch.int32)) for (_, _, y), ys in zip(items, ys_single))
        if any(mat.device_status() != 0 for mat, _, _ in items):
            raise RuntimeError("kernel status")
        wbytes = 2 * a.n * a.k * len(items)
        print(json.dumps({"workload": "MoE projection, %d experts of [%d, %d], top-%d" % (a.experts, a.n, a.k, a.topk),
                          "tokens": t, "routed_experts": len(items), "max_m": int(counts.max()),
                          "us_batched": round(us_batched, 1), "launches_batched": (len(items) + 31) // 32,
                          "us_per_expert_calls": round(us_loop, 1), "launches_per_expert_calls": len(items),
                          "speedup": round(us_loop / us_batched, 3),
                          "us_batched_graph": round(us_batched_g, 1), "us_per_expert_calls_graph": round(us_loop_g, 1),
                          "speedup_graph": round(us_loop_g / us_batched_g, 3),
                          "weight_gbs_batched": round(wbytes / us_batched / 1e3, 1),
                          "weight_gbs_per_expert_calls": round(wbytes / us_loop / 1e3, 1),
                          "weight_gbs_batched_graph": round(wbytes / us_batched_g / 1e3, 1),
                          "bit_identical": bool(same), "l2": "512 MB read before each timed call"}), flush=True)
    return 0


def case_sweep70b(argv):
    """Llama-70B MLP projections (gate and up [28672, 8192], down [8192, 28672])
    over the outlier (element) fraction and the per-matrix sigma, at several
    M: compressed sizes, the measured raw-group rate, and the fused matmul
    against the same kernel on uncompressed BF16 weights (bit-identical
    outputs checked).  Every timed call follows a 512 MB read."""
    ap = argparse.ArgumentParser(prog="bench.py --case sweep70b")
    ap.add_argument("--fracs", type=float, nargs="+", default=[0.0, 0.001, 0.01, 0.05])
    ap.add_argument("--sigmas", type=float, nargs="+", default=[0.005, 0.01, 0.015, 0.02, 0.05])
    ap.add_argument("--ms", type=int, nargs="+", default=[1, 256, 1024])
    ap.add_argument("--grid", choices=["full", "axes"], default="axes",
                    help="axes: the outlier sweep at sigma 0.015 and the sigma sweep at 0.1%% outliers")
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--workers", type=int, default=min(32, host_cores()))
    a = ap.parse_args(argv)
    shapes = (("gate", 28672, 8192), ("up", 28672, 8192), ("down", 8192, 28672))
    if a.grid == "full":
        combos = [(f, s) for f in a.fracs for s in a.sigmas]
    else:
        combos = [(f, 0.015) for f in a.fracs] + [(0.001, s) for s in a.sigmas if s != 0.015]
    jobs = [(n, k, s, f, 7000 + 10 * ci + pi) for ci, (f, s) in enumerate(combos) for pi, (_, n, k) in enumerate(shapes)]
    blobs = _encode_all(jobs, a.workers)
    import torch
    from decode_gemm_exponent_b200 import synth, uw
    scrub = torch.zeros(128 << 20, dtype=torch.int32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(a.reps):
            scrub.sum()
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        return 1e3 * total / a.reps

    for (job, blob) in zip(jobs, blobs):
        n, k, sigma, frac, seed = job
        name = shapes[(seed - 7000) % 10][0]   # gate and up share a shape: the seed tells them apart
        mat = uw.Matrix(blob)
        info = mat.info
        w = synth.weights_bf16(n, k, sigma, frac, 1.0, seed=seed)
        wd = torch.from_numpy(w.view(np.int16)).cuda()
        del w
        for m in a.ms:
            x = torch.from_numpy(synth.activations_bf16(m, k, seed=m).view(np.int16)).cuda()
            plans, _ = uw.autotune([mat], [m], reps=3)
            p = same_plan(uw, plans[0][0])
            ws = torch.zeros(max(mat.workspace_bytes(m, p), 256), dtype=torch.uint8, device="cuda")
            yf = torch.empty(m, n, dtype=torch.float32, device="cuda")
            yp = torch.empty_like(yf)
            us_f = timed(lambda: mat.matmul(x, p, y=yf, ws=ws))
            pp = same_plan(uw, p, 4)
            ws_plain = torch.zeros(max(mat.workspace_bytes(m, pp), 256), dtype=torch.uint8, device="cuda")
            us_p = timed(lambda: uw.matmul_bf16(x, wd, pp, y=yp, ws=ws_plain))
            same = torch.equal(yf.view(torch.int32), yp.view(torch.int32))
            if mat.device_status() != 0:
                raise RuntimeError("kernel status")
            print(json.dumps({
                "workload": "llama-70b MLP %s [%d, %d]" % (name, n, k), "sigma": sigma, "outlier_frac": frac,
                "raw_group_rate": round(info.n_raw / info.n_groups, 5),
                "huffman_fraction": round(info.huffman_bytes / (2 * n * k), 4),
                "palette_fraction": round(info.palette_bytes / (2 * n * k), 4),
                "entropy_bits": round(info.entropy_bits, 4), "m": m, "plan": plan_label(p),
                "fused_us": round(us_f, 1), "plain_bf16_us": round(us_p, 1),
                "fused_weight_gbs": round(2 * n * k / us_f / 1e3, 1),
                "fused_tflops": round(2.0 * m * n * k / us_f / 1e6, 1),
                "fused_over_plain": round(us_f / us_p, 3), "bit_identical_to_plain": bool(same),
                "l2": "512 MB read before each timed call"}), flush=True)
        del mat, wd
        torch.cuda.empty_cache()
    return 0


# ----------------------------------------------------------------------------- main

def main():
    if "--case" in sys.argv:
        i = sys.argv.index("--case")
        case = sys.argv[i + 1] if i + 1 < len(sys.argv) else ""
        rest = sys.argv[1:i] + sys.argv[i + 2:]
        cases = {"kernel": case_kernel, "stack": case_stack, "moe": case_moe, "sweep70b": case_sweep70b}
        if case != "step":
            if case not in cases:
                sys.exit("unknown --case %r (step, %s)" % (case, ", ".join(cases)))
            return cases[case](rest)
        sys.argv = [sys.argv[0]] + rest
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="uw", choices=["uw", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=24.0,
                    help="host time for the CPU baseline (split between one core and all cores)")
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
