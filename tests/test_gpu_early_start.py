"""Early start (programmatic dependent launch) of direct-palette matmuls on the
blob's own planes: a call may be scheduled while the previous libuw kernel on
the stream drains, reading only the blob's compressed planes before it waits.
These cases chain calls with no synchronisation in between, where a wrong
ordering would show up as different bits:

* back-to-back calls that write the same Y and the same workspace (split-K
  partials), each checked against the same call run alone;
* a call whose X is produced on the stream right before it by another kernel
  (a torch copy of fresh values), after a libuw call that reads the old X;
* a preprocessing pipeline (transcode, then the fused kernel on the workspace
  plane) right after a direct-palette call that reuses the same workspace.
"""
import numpy as np
import pytest
import torch

from decode_gemm_exponent_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def uw():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_gemm_exponent_b200 import uw as U
    assert (U.KERNEL_TC, U.KERNEL_MMA) == (KERNEL_TC, KERNEL_MMA)
    return U


def dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def bits(t):
    return t.cpu().numpy().view(np.uint32)


KERNEL_TC, KERNEL_MMA = 2, 3   # uw.KERNEL_TC, uw.KERNEL_MMA
PLANS = [
    ("mma", dict(kernel=KERNEL_MMA, bn=4, split_k=1, stages=2)),
    ("tc_split4", dict(kernel=KERNEL_TC, bn=16, split_k=4, stages=0)),
    ("tc_bn64", dict(kernel=KERNEL_TC, bn=64, split_k=1, stages=0)),
]


@pytest.mark.parametrize("name,kw", PLANS)
def test_back_to_back_calls_share_y_and_workspace(uw, name, kw):
    n, k, m = 512, 2048, 16 if kw["kernel"] == KERNEL_TC else 4
    mats = [uw.Matrix(uw.encode(synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=s))) for s in (31, 32, 33)]
    xs = [dev16(synth.activations_bf16(m, k, seed=s)) for s in (41, 42, 43)]
    plan = uw.make_plan(**{**kw, "pipeline": uw.PIPE_DIRECT_PALETTE})
    ws = uw.new_workspace(max(mat.workspace_bytes(m, plan) for mat in mats) + 256, "cuda")
    alone = []
    for mat, x in zip(mats, xs):
        alone.append(bits(mat.matmul(x, plan, ws=ws)))
        torch.cuda.synchronize()
    y = torch.empty(m, n, dtype=torch.float32, device="cuda")
    outs = []
    for rep in range(3):
        for mat, x in zip(mats, xs):
            mat.matmul(x, plan, y=y, ws=ws)      # same Y, same workspace, no synchronisation
        outs.append(bits(y))
    assert all(mat.device_status() == 0 for mat in mats)
    for o in outs:
        assert np.array_equal(o, alone[-1])
    # each call's result taken right after it, still without synchronising the calls themselves
    ys = [torch.empty(m, n, dtype=torch.float32, device="cuda") for _ in mats]
    for mat, x, yy in zip(mats, xs, ys):
        mat.matmul(x, plan, y=yy, ws=ws)
    for yy, ref in zip(ys, alone):
        assert np.array_equal(bits(yy), ref)


@pytest.mark.parametrize("name,kw", PLANS)
def test_x_written_by_a_kernel_right_before_the_call(uw, name, kw):
    n, k, m = 512, 2048, 16 if kw["kernel"] == KERNEL_TC else 4
    mat = uw.Matrix(uw.encode(synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=51)))
    x_old, x_new = dev16(synth.activations_bf16(m, k, seed=52)), dev16(synth.activations_bf16(m, k, seed=53))
    plan = uw.make_plan(**{**kw, "pipeline": uw.PIPE_DIRECT_PALETTE})
    ws = uw.new_workspace(mat.workspace_bytes(m, plan) + 256, "cuda")
    ref_new = bits(mat.matmul(x_new, plan, ws=ws))
    torch.cuda.synchronize()
    x = x_old.clone()
    y1 = torch.empty(m, n, dtype=torch.float32, device="cuda")
    y2 = torch.empty_like(y1)
    for _ in range(3):
        x.copy_(x_old)
        mat.matmul(x, plan, y=y1, ws=ws)   # reads the old X
        x.copy_(x_new)                     # a kernel writes X on the stream
        mat.matmul(x, plan, y=y2, ws=ws)   # must read the new X
        assert np.array_equal(bits(y2), ref_new)
    assert mat.device_status() == 0


def test_preprocessing_pipeline_after_a_direct_call_on_the_same_workspace(uw):
    n, k, m = 512, 2048, 16
    w = synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=61)
    mat = uw.Matrix(uw.encode(w))
    x = dev16(synth.activations_bf16(m, k, seed=62))
    direct = uw.make_plan(pipeline=uw.PIPE_DIRECT_PALETTE, kernel=KERNEL_TC, bn=16, split_k=4, stages=0)
    transcode = uw.make_plan(pipeline=uw.PIPE_TRANSCODE_FUSED, kernel=KERNEL_TC, bn=16, split_k=4, stages=0)
    plain = uw.make_plan(pipeline=uw.PIPE_DIRECT_PALETTE, kernel=KERNEL_TC, bn=16, split_k=4, stages=0)
    ref = bits(uw.matmul_bf16(x, dev16(w), plain))
    ws = uw.new_workspace(max(mat.workspace_bytes(m, direct), mat.workspace_bytes(m, transcode)) + 256, "cuda")
    y = torch.empty(m, n, dtype=torch.float32, device="cuda")
    for _ in range(3):
        mat.matmul(x, direct, y=y, ws=ws)
        mat.matmul(x, transcode, y=y, ws=ws)   # transcodes into the workspace the direct call used
        mat.matmul(x, direct, y=y, ws=ws)
    assert np.array_equal(bits(y), ref)
    assert mat.device_status() == 0
