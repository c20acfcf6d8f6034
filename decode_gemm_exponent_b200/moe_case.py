"""The routed experts of one mixture-of-experts projection, all in one batched
call (uw_fused_matmul_batched) against one uw_fused_matmul call per expert.

    python -m decode_gemm_exponent_b200.moe_case [--experts 128] [--n 768] [--k 2048]
           [--topk 8] [--tokens 1 4 16] [--reps 10]

Experts: BF16 N(0, 0.02^2) with 0.05% N(0, 1) outliers, expert e seeded
e + 1, encoded in palette form.  Routing: each of T tokens picks `topk`
distinct experts uniformly at random (seed T); an expert's m is the number of
tokens routed to it, and experts with no token are skipped.  Each timed call
(the batched one, or the per-expert loop) is preceded by a 512 MB read so that
the weights stream from HBM, and is timed on its own with CUDA events, both as
issued from Python and replayed from a CUDA graph (no host launch cost); the
line reports the mean microseconds, the number of launches and the effective
weight bandwidth (uncompressed BF16 bytes of the routed experts / time).
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import synth, uw


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--experts", type=int, default=128)
    ap.add_argument("--n", type=int, default=768)
    ap.add_argument("--k", type=int, default=2048)
    ap.add_argument("--topk", type=int, default=8)
    ap.add_argument("--tokens", type=int, nargs="+", default=[1, 4, 16])
    ap.add_argument("--slices", type=int, default=4)
    ap.add_argument("--reps", type=int, default=10)
    a = ap.parse_args(argv)

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
        for mat, _, _ in items:
            if mat.device_status() != 0:
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


if __name__ == "__main__":
    main()
