"""Run one libuw kernel on a synthetic matrix, for timing or profiler capture.

    python -m decode_gemm_exponent_b200.profile_case --kernel fma --n 28672 --k 8192 --m 1

kernels: decode, exp_decode, transcode (Huffman stream -> BF16 / exponent
bytes / 4-bit palette),
fma, tc (fused palette matmul, CUDA-core GEMV or tcgen05), plain_fma,
plain_tc (the same kernels on BF16 weights).  One warm-up launch is followed
by --reps timed launches (CUDA events); the per-launch time and the
algorithmic bytes / FLOPs per launch are printed as one JSON line.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import synth, uw


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", required=True,
                    choices=["decode", "exp_decode", "transcode", "fma", "tc", "mma", "plain_fma", "plain_tc", "plain_mma"])
    ap.add_argument("--n", type=int, default=28672)
    ap.add_argument("--k", type=int, default=8192)
    ap.add_argument("--m", type=int, default=1)
    ap.add_argument("--bn", type=int, default=0, help="TC token tile, FMA rows per warp or MMA K slices")
    ap.add_argument("--split", type=int, default=1)
    ap.add_argument("--stages", type=int, default=0)
    ap.add_argument("--sigma", type=float, default=0.015)
    ap.add_argument("--frac", type=float, default=0.0005)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--flush", action="store_true",
                    help="read 512 MB before each timed call (weights come from HBM, not L2; "
                         "a read leaves no dirty lines to write back) and time every call on its own")
    a = ap.parse_args(argv)

    w = synth.weights_bf16(a.n, a.k, a.sigma, a.frac, 1.0, a.seed)
    blob = uw.encode(w)
    mat = uw.Matrix(blob)
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
    if a.kernel in ("fma", "plain_fma"):
        plan = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_FMA, a.bn or 1, 1)
    elif a.kernel in ("mma", "plain_mma"):
        plan = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, a.bn or 2, 1, a.stages)
    else:
        plan = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, a.bn or 16, a.split, a.stages)
    preprocessing = a.kernel in ("decode", "exp_decode", "transcode")
    ws_bytes = 0 if preprocessing else uw.workspace_size(a.m, a.n, a.k, plan)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    wd = None
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
    elif a.kernel in ("fma", "tc", "mma"):
        run = lambda: mat.matmul(x, plan, y=y, ws=ws)
        alg = common + nk // 2 + xy
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
        for r in range(a.reps):
            scrub.sum()
            e0.record()
            run()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        us = 1e3 * total / a.reps
    else:
        e0.record()
        for _ in range(a.reps):
            run()
        e1.record()
        torch.cuda.synchronize()
        us = 1e3 * e0.elapsed_time(e1) / a.reps
    print(json.dumps({"kernel": a.kernel, "n": a.n, "k": a.k, "m": a.m, "bn": plan.bn,
                      "split": plan.split_k, "us": us, "alg_bytes": int(alg),
                      "gbs": alg / us / 1e3, "tflops": None if preprocessing else flops / us / 1e6,
                      "l2": "flushed before each call" if a.flush else
                      "not flushed (a matrix under 126 MB stays in L2 between calls)"}))


if __name__ == "__main__":
    main()
