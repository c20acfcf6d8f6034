"""Host-side logic of bench.py that needs no GPU: the measured-traffic
lookup, the source digest that keys it, and the plan-file round trip."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_measured_traffic_lookup():
    # unknown kernel group: no figure
    assert bench.measured_traffic("fused/no_such_kernel", 1e6) is None
    for group, rec in bench.MEASURED_TRAFFIC.items():
        got = bench.measured_traffic(group, 2 * rec["alg_bytes"])
        # either the sources still match the capture (scaled figure) or they
        # changed since (None); never a figure for different sources
        assert got is None or abs(got - 2 * rec["bytes"]) < 1e-6 * rec["bytes"]
    saved = dict(bench.MEASURED_TRAFFIC)
    try:
        # a record keyed on the current source of a committed kernel file
        f = "decode_gemm_exponent_b200/csrc/gemm_sk.cu"
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            digest = bench.source_digest([fh.read()])
        rec = {"bytes": 1000, "alg_bytes": 800, "files": (f,), "sha256": digest}
        bench.MEASURED_TRAFFIC["fused/test_kernel"] = rec
        assert abs(bench.measured_traffic("fused/test_kernel", 1600) - 2000) < 1e-9
        bench.MEASURED_TRAFFIC["fused/test_kernel"] = dict(rec, sha256="0" * 64)   # pretend the kernel changed
        assert bench.measured_traffic("fused/test_kernel", 800) is None
    finally:
        bench.MEASURED_TRAFFIC.clear()
        bench.MEASURED_TRAFFIC.update(saved)


def test_source_digest_ignores_comments_only():
    src = 'int f(int a) {  // add one\n  return a + 1; /* "x" */\n}\nconst char* s = "// kept";\n'
    d = bench.source_digest([src])
    assert bench.source_digest([src.replace("add one", "increment")]) == d
    assert bench.source_digest([src.replace("  return", "\n\n    return")]) == d
    assert bench.source_digest([src.replace("a + 1", "a + 2")]) != d
    assert bench.source_digest([src.replace('"// kept"', '"// gone"')]) != d   # literal, not a comment
    assert bench.source_digest([src, ""]) != d                                  # file boundaries count


def test_alg_bytes_per_pipeline():
    """Each kernel is charged for what it must read and write: the decode
    kernels never read the sign/mantissa plane unless they write BF16."""
    from types import SimpleNamespace as NS
    from decode_gemm_exponent_b200 import uw
    n, k, m = 256, 1024, 4
    nk = n * k
    sec = [nk, 4096, 0, 0, 0, 0, 0, nk // 2]            # sm, raw plane, ...
    mat = NS(n=n, k=k, info=NS(section_bytes=sec, stream_bits=8 * 70000, n_chunks=nk // 256))
    stream = 70000 + (nk // 256 + 1) * 4
    flags = nk // 512
    xy = m * k * 2 + m * n * 4
    plan = lambda p: uw.make_plan(p, uw.KERNEL_MMA, 4)
    assert bench.alg_bytes(mat, m, plan(4)) == {"fused": nk + 4096 + 2 * flags + nk // 2 + xy}
    assert bench.alg_bytes(mat, m, plan(1)) == {"decode": stream + nk + 4096 + 2 * flags + 2 * nk,
                                                 "plain": 2 * nk + xy}
    assert bench.alg_bytes(mat, m, plan(2)) == {"exp_decode": stream + 4096 + 4 * flags + nk,
                                                 "fused": 2 * nk + 2 * flags + xy}
    assert bench.alg_bytes(mat, m, plan(3)) == {"transcode": stream + flags + nk // 2,
                                                 "fused": nk + 4096 + 2 * flags + nk // 2 + xy}


def test_compression_stats_on_real_blobs():
    """The bench line's size and exponent statistics come from the blob
    headers; checked against the oracle's own histogram on two small
    matrices of different sizes (weights-weighted means)."""
    import numpy as np
    from decode_gemm_exponent_b200 import synth, uw
    from oracle import oracle as O
    ws = [synth.weights_bf16(128, 512, 0.02, 0.001, 1.0, seed=1), synth.weights_bf16(64, 256, 0.05, 0.01, 1.0, seed=2)]
    infos = [uw.blob_info(uw.encode(w)) for w in ws]
    st = bench.compression_stats(infos)
    n_w = [w.size for w in ws]
    ent, cov, raw, groups = 0.0, 0.0, 0, 0
    for w in ws:
        e = ((w >> 7) & 0xFF).astype(np.int64)
        p = np.bincount(e.ravel(), minlength=256) / e.size
        nz = p[p > 0]
        ent += float(-(nz * np.log2(nz)).sum()) * w.size
        cov += float(np.sort(p)[::-1][:16].sum()) * w.size
        ref = O.encode(w)
        raw += ref.n_raw
        groups += ref.raw.size
    assert abs(st["exponent_entropy_bits"] - ent / sum(n_w)) < 1e-3
    assert abs(st["top16_coverage"] - cov / sum(n_w)) < 1e-5
    assert abs(st["raw_group_fraction"] - raw / groups) < 1e-5
    # (on matrices this small the Huffman form's fixed 16 KB decode table outweighs its saving)
    assert 0 < st["compressed_fraction_huffman"] < 1 and 0 < st["compressed_fraction_palette"] < 1


def test_plans_from_json_round_trip():
    from decode_gemm_exponent_b200 import uw
    doc = {"plans": []}
    kinds = [("fma", 1, 1, 0), ("tc", 64, 4, 0), ("mma", 4, 1, 2), ("tc_sk", 16, 1, 3)]
    pipes = [("decode_gemm", uw.PIPE_DECODE_GEMM), ("decode_exp_fused", uw.PIPE_DECODE_EXP_FUSED),
             ("transcode_fused", uw.PIPE_TRANSCODE_FUSED), ("direct_palette", uw.PIPE_DIRECT_PALETTE)]
    for i in range(3):
        for j, m in enumerate(bench.MS):
            kern, bn, split, stages = kinds[(i + j) % 4]
            doc["plans"].append({"matrix": i, "m": m, "best": {"pipeline": pipes[(i + 2 * j) % 4][0], "kernel": kern,
                                                                "bn": bn, "split_k": split, "stages": stages}})
    plans = bench.plans_from_json(json.dumps(doc), 3, uw)
    for i in range(3):
        for j in range(len(bench.MS)):
            kern, bn, split, stages = kinds[(i + j) % 4]
            p = plans[i][j]
            assert p.kernel == {"fma": 1, "tc": 2, "mma": 3, "tc_sk": 4}[kern] and p.bn == bn and p.split_k == split
            assert p.stages == stages and p.pipeline == pipes[(i + 2 * j) % 4][1]
            # every plan has a kernel group and a launch count; pipelines 1-3 add a preprocessing launch
            assert bench.kernel_group(p).split("/")[0]
            assert bench.launches_per_call(p) >= (2 if p.pipeline != uw.PIPE_DIRECT_PALETTE else 1)


def test_plan_file_reader_rejects_incomplete_or_unknown_plans():
    import pytest
    from decode_gemm_exponent_b200 import uw
    best = {"pipeline": "direct_palette", "kernel": "mma", "bn": 4, "split_k": 1, "stages": 2, "us": 1.0}
    doc = {"plans": [{"matrix": 0, "n": 64, "k": 64, "m": 1, "best": best, "candidates": [best]},
                     {"matrix": 1, "n": 64, "k": 64, "m": 1, "best": best, "candidates": [best]}]}
    plans = uw.plans_from_json(json.dumps(doc), [1])
    assert len(plans) == 2 and plans[1][0].kernel == uw.KERNEL_MMA and plans[1][0].stages == 2
    with pytest.raises(ValueError):                       # no plan for m = 4
        uw.plans_from_json(json.dumps(doc), [1, 4])
    bad = json.loads(json.dumps(doc))
    bad["plans"][1]["best"]["kernel"] = "wgmma"
    with pytest.raises(ValueError):
        uw.plans_from_json(json.dumps(bad), [1])
    with pytest.raises(ValueError):                       # the bench's layer has three matrices
        bench.plans_from_json(json.dumps(doc), 3, uw)


def test_oracle_sample_is_the_step_on_a_row_sample():
    """The reference arm and the CPU baseline run the step's 12 calls on the
    first 1/16 of each matrix's rows; both arms print the same config."""
    tasks = bench.oracle_tasks()
    rows = [bench.oracle_sample_rows(n) for _, n, _ in bench.PROJ]
    assert rows == [896, 896, 256]
    # every call's sample in 128-row parts: 7, 7 and 2 parts per M
    assert [bench.oracle_parts(n) for _, n, _ in bench.PROJ] == [7, 7, 2]
    assert sorted(tasks) == sorted((i, m, p) for m in bench.MS for i in range(len(bench.PROJ))
                                   for p in range(bench.oracle_parts(bench.PROJ[i][1])))
    assert all(r % bench.ORACLE_PART_ROWS == 0 for r in rows)
    assert bench.oracle_step_bytes() == sum(2 * r * k for r, (_, _, k) in zip(rows, bench.PROJ)) * len(bench.MS)
    assert bench.workload_config() == {"workload": bench.WORKLOAD, "l2": bench.L2_NOTE}
    assert "12 calls" in bench.oracle_sample_text(4) and "4 worker processes" in bench.oracle_sample_text(4)


def test_kernel_names_of_every_plan_kind():
    from decode_gemm_exponent_b200 import uw
    assert bench.kernel_group(uw.make_plan(4, uw.KERNEL_TC_SK, 64, 1)) == "fused/tc_sk_bn64"
    assert bench.kernel_group(uw.make_plan(4, uw.KERNEL_MMA_SK, 8, 1, 6)) == "fused/mma_sk_w8_s6"
    assert bench.launches_per_call(uw.make_plan(4, uw.KERNEL_MMA_SK, 8, 1, 6)) == 1
    assert bench.plan_label(uw.make_plan(1, uw.KERNEL_TC, 64, 4)) == "decode+plain/tcgen05_bn64/split4"
    assert bench.launches_per_call(uw.make_plan(4, uw.KERNEL_TC_SK, 16, 1)) == 1
    assert bench.launches_per_call(uw.make_plan(3, uw.KERNEL_TC_SK, 16, 1)) == 2
    assert bench.launches_per_call(uw.make_plan(4, uw.KERNEL_TC, 16, 4)) == 2
