"""Cross-layer overlap on a stack of Llama-3.1-8B-shaped MLP layers
(Unweight page §八): time uw_stack_run with the decodes on a side stream
against the same stack on one stream.

    python -m decode_gemm_exponent_b200.stack_case [--layers 32] [--ms 1 64 1024]

Layers: gate and up [14336, 4096], down [4096, 14336], BF16 N(0, 0.02^2)
with 0.05% N(0, 1) outliers, seed 3*layer + projection + 1.  Activations per
(M, K) from the usual activation generator.  Two plan sets per M:
  * autotuned: the per-(projection, M) plans the autotuner picks on layer 0,
    used for every layer;
  * alternating: even layers full decode + plain kernel (pipeline 1), odd
    layers the fused palette kernel (pipeline 4), the arrangement the page
    describes (a Huffman layer decoded while a palette layer computes); the
    kernel choice (FMA or tcgen05, token tile, split) is the autotuned one.
Each line reports the stack's time with and without the side stream and the
effective weight bandwidth (uncompressed BF16 bytes / time), and the
decode/compute SM split chosen by uw_stack_tune_split among --splits
(preprocessing SMs in a green-context partition of their own; 0 = the side
stream shares all SMs) with each candidate's time.  The host encode runs in a
spawn process pool before any CUDA call.
"""
from __future__ import annotations

import argparse
import json
import multiprocessing as mp
import os
import sys

import numpy as np

SHAPES = (("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336))


def _encode_one(args):
    layer, i, n, k = args
    from decode_gemm_exponent_b200 import synth, uw
    w = synth.weights_bf16(n, k, 0.02, 0.0005, 1.0, seed=3 * layer + i + 1)
    return uw.encode(w)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--ms", type=int, nargs="+", default=[1, 64, 1024])
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--workers", type=int, default=min(16, os.cpu_count() or 1))
    ap.add_argument("--splits", type=int, nargs="+", default=[0, 16, 32, 48],
                    help="preprocessing SM counts tried by the split tuner (0 = no split)")
    a = ap.parse_args(argv)

    jobs = [(layer, i, n, k) for layer in range(a.layers) for i, (_, n, k) in enumerate(SHAPES)]
    with mp.get_context("spawn").Pool(a.workers) as pool:
        blobs = pool.map(_encode_one, jobs, chunksize=1)

    import torch
    from decode_gemm_exponent_b200 import synth, uw
    mats = [uw.Matrix(b) for b in blobs]
    del blobs
    ms = sorted(set(a.ms))
    xs = {(m, k): torch.from_numpy(synth.activations_bf16(m, k, seed=m).view(np.int16)).cuda()
          for m in ms for k in {s[2] for s in SHAPES}}
    plans, _ = uw.autotune(mats[:3], ms, reps=5)
    side = torch.cuda.Stream()
    main_s = torch.cuda.current_stream()
    weight_bytes = sum(2 * mat.n * mat.k for mat in mats)

    def timed(stack, side_stream):
        for _ in range(a.warmup):
            stack.run(side_stream=side_stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(main_s)
        for _ in range(a.reps):
            stack.run(side_stream=side_stream)
        e1.record(main_s)
        torch.cuda.synchronize()
        return 1e3 * e0.elapsed_time(e1) / a.reps

    for j, m in enumerate(ms):
        for kind in ("autotuned", "alternating"):
            steps = []
            for idx, mat in enumerate(mats):
                layer, proj = divmod(idx, 3)
                p = plans[proj][j]
                plan = uw.make_plan(p.pipeline, p.kernel, p.bn, p.split_k, p.stages)
                if kind == "alternating":
                    plan.pipeline = uw.PIPE_DECODE_GEMM if layer % 2 == 0 else uw.PIPE_DIRECT_PALETTE
                y = torch.empty(m, mat.n, dtype=torch.float32, device="cuda")
                steps.append((mat, xs[(m, mat.k)], y, plan))
            stack = uw.Stack(steps)
            us_overlap = timed(stack, side)
            us_serial = timed(stack, None)
            for mat in mats[:3]:
                if mat.device_status() != 0:
                    raise RuntimeError("kernel status during the stack run")
            best_split, split_us = stack.tune_split(a.splits, reps=a.reps)
            for mat in mats[:3]:
                if mat.device_status() != 0:
                    raise RuntimeError("kernel status during the split tuning")
            n_prep = sum(1 for s in steps if s[3].pipeline != uw.PIPE_DIRECT_PALETTE)
            print(json.dumps({
                "workload": "llama-3.1-8b MLP stack", "layers": a.layers, "m": m, "plans": kind,
                "steps": len(steps), "preprocessed_steps": n_prep,
                "us_overlap": round(us_overlap, 1), "us_one_stream": round(us_serial, 1),
                "speedup": round(us_serial / us_overlap, 4),
                "weight_gbs_overlap": round(weight_bytes / us_overlap / 1e3, 1),
                "weight_gbs_one_stream": round(weight_bytes / us_serial / 1e3, 1),
                "split_best_prep_sms": best_split,
                "split_us": {str(c): round(u, 1) for c, u in zip(a.splits, split_us)},
                "plan_per_projection": [str(plans[p][j].as_dict()) for p in range(3)],
            }), flush=True)
        del stack, steps
    return 0


if __name__ == "__main__":
    sys.exit(main())
