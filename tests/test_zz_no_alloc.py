"""uw_fused_matmul_noalloc: the matmul for callers that cannot allocate.

Some callers cannot hand the library device memory when they call in (an
engine that gives its plug-ins no allocator and forbids cudaMalloc after
start-up).  This entry point keeps its split-K scratch in a fixed array in the
library's own device memory.  The test calls it through the C ABI twice in a
row and checks each result against uw_fused_matmul with a caller workspace;
it also checks that a plan needing more scratch than the array holds is
refused.  It lives in its own file that pytest collects last.
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
    return U


def test_noalloc_matches_workspace_path_twice(uw):
    n, k, m = 512, 1024, 16
    w = synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=31)
    mat = uw.Matrix(uw.encode(w))
    plan = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 16, 4)
    assert uw.workspace_size(m, n, k, plan) > 0          # the split-K path uses scratch
    for seed in (41, 42):                                # two calls in a row
        x = torch.from_numpy(synth.activations_bf16(m, k, seed=seed).view(np.int16)).cuda()
        y_ref = mat.matmul(x, plan).cpu().numpy()
        y = uw.fused_matmul_noalloc(mat, x, plan).cpu().numpy()
        assert mat.device_status() == 0
        # same kernel, same split, same reduction order: identical bits
        np.testing.assert_allclose(y, y_ref, rtol=0, atol=0)


def test_noalloc_rejects_oversized_scratch(uw):
    n, k, m = 4096, 4096, 256
    mat = uw.Matrix(uw.encode(synth.weights_bf16(n, k, 0.02, 0.0, 1.0, seed=32)))
    plan = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 256, 8)
    assert uw.workspace_size(m, n, k, plan) > 16 << 20
    x = torch.zeros(m, k, dtype=torch.int16, device="cuda")
    with pytest.raises(uw.UwError) as e:
        uw.fused_matmul_noalloc(mat, x, plan)
    assert e.value.status == 7                           # UW_ERR_WORKSPACE
    with pytest.raises(uw.UwError):
        uw.fused_matmul_noalloc(mat, x, uw.make_plan(uw.PIPE_DECODE_GEMM, uw.KERNEL_TC, 256, 1))


def test_noalloc_alternating_plans_and_sizes(uw):
    """Calls of different sizes and kernels in a row share the one array: a
    large split-K call, then smaller ones that overwrite less of it, and
    stream-K calls (tcgen05 and warp-MMA) whose tile counters sit apart from
    the partial sums.  Each result equals uw_fused_matmul with a fresh
    zero-filled workspace."""
    n, k = 512, 1024
    mat = uw.Matrix(uw.encode(synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=33)))
    calls = [(64, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 64, 8)),
             (16, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 16, 2)),
             (16, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC_SK, 16, 1)),
             (64, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 64, 8)),
             (100, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC_SK, 64, 1)),
             (3, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 16, 3)),
             (16, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC_SK, 16, 1)),
             (1, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA_SK, 8, 1, 0)),
             (64, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 64, 8)),
             (16, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA_SK, 8, 1, 2)),
             (5, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA_SK, 16, 1, 2))]
    for i, (m, plan) in enumerate(calls):
        x = torch.from_numpy(synth.activations_bf16(m, k, seed=50 + i).view(np.int16)).cuda()
        y_ref = mat.matmul(x, plan).cpu().numpy()
        y = uw.fused_matmul_noalloc(mat, x, plan).cpu().numpy()
        assert mat.device_status() == 0
        assert np.array_equal(y.view(np.uint32), y_ref.view(np.uint32)), "call %d" % i
