"""Layer stacks with cross-layer overlap (uw_stack_run, Unweight page §八).

Each step of a stack must give exactly what uw_fused_matmul gives for the
same matrix, input and plan, whichever stream the preprocessing ran on, and
the fused results must lie within the oracle's bound.  Steps mix all four
pipelines and both kernels, and more preprocessing steps than slots, so that
slots are reused while earlier matmuls may still read them.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from decode_gemm_exponent_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module")
def uw():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_gemm_exponent_b200 import uw as U
    return U


def make_stack(uw, layers=3, m_list=(1, 64)):
    """`layers` MLP-shaped layers (gate/up [384, 256], down [256, 384]) with
    independent seeds; per step a plan cycling over pipelines and kernels."""
    shapes = (("gate", 384, 256), ("up", 384, 256), ("down", 256, 384))
    mats, ws = [], []
    for layer in range(layers):
        for i, (_, n, k) in enumerate(shapes):
            w = synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=100 * layer + i)
            ws.append(w)
            mats.append(uw.Matrix(uw.encode(w)))
    pipes = (uw.PIPE_DECODE_GEMM, uw.PIPE_TRANSCODE_FUSED, uw.PIPE_DIRECT_PALETTE, uw.PIPE_DECODE_EXP_FUSED,
             uw.PIPE_DECODE_GEMM)
    steps = []
    for j, m in enumerate(m_list):
        for i, mat in enumerate(mats):
            pipe = pipes[(i + j) % len(pipes)]
            if m <= 4:
                plan = uw.make_plan(pipe, uw.KERNEL_FMA, 1 + (i % 2), 1)
            else:
                plan = uw.make_plan(pipe, uw.KERNEL_TC, 64, 1 + (i % 3))
            x = torch.from_numpy(synth.activations_bf16(m, mat.k, seed=7 * i + m).view(np.int16)).cuda()
            y = torch.full((m, mat.n), float("nan"), dtype=torch.float32, device="cuda")
            steps.append((mat, x, y, plan))
    return mats, ws, steps


def reference_outputs(uw, steps):
    outs = []
    for mat, x, _, plan in steps:
        outs.append(mat.matmul(x, plan).cpu().numpy())
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("overlap", [True, False])
def test_stack_matches_single_calls(uw, overlap):
    mats, ws, steps = make_stack(uw)
    want = reference_outputs(uw, steps)
    stack = uw.Stack(steps)
    side = torch.cuda.Stream() if overlap else None
    for rep in range(2):                      # the second run reuses the slots and events
        for _, _, y, _ in steps:
            y.fill_(float("nan"))
        stack.run(side_stream=side)
        torch.cuda.synchronize()
        for s, (st, w_ref) in enumerate(zip(steps, want)):
            got = st[2].cpu().numpy()
            assert np.array_equal(got.view(np.uint32), w_ref.view(np.uint32)), "step %d rep %d" % (s, rep)
    for mat in mats:
        assert mat.device_status() == 0


def test_stack_within_oracle_bound(uw):
    mats, ws, steps = make_stack(uw, layers=1, m_list=(4,))
    uw.Stack(steps).run(side_stream=torch.cuda.Stream())
    torch.cuda.synchronize()
    for (mat, x, y, _), w in zip(steps, ws):
        xh = x.cpu().numpy().view(np.uint16)
        y_ref, a_ref = O.gemm(xh, w)
        err = np.abs(y.cpu().numpy().astype(np.float64) - y_ref)
        assert (err <= TOL * a_ref + 1e-30).all()


def test_stack_slot_reuse_on_one_matrix(uw):
    """Five decode steps on one matrix use the two slots three times over;
    the side stream must not overwrite a slot before its matmul has read it."""
    w = synth.weights_bf16(256, 512, 0.02, 0.002, 1.0, seed=42)
    mat = uw.Matrix(uw.encode(w))
    plan = uw.make_plan(uw.PIPE_DECODE_GEMM, uw.KERNEL_FMA, 1, 1)
    xs = [torch.from_numpy(synth.activations_bf16(1, 512, seed=s).view(np.int16)).cuda() for s in range(5)]
    ys = [torch.empty(1, 256, dtype=torch.float32, device="cuda") for _ in xs]
    stack = uw.Stack([(mat, x, y, plan) for x, y in zip(xs, ys)])
    stack.run(side_stream=torch.cuda.Stream())
    torch.cuda.synchronize()
    for x, y in zip(xs, ys):
        assert np.array_equal(y.cpu().numpy(), mat.matmul(x, plan).cpu().numpy())
    assert mat.device_status() == 0


# ---------------------------------------------------------------- decode/compute SM split

def test_sm_split_partitions(uw):
    total = torch.cuda.get_device_properties(0).multi_processor_count
    with uw.SmSplit(20) as sp:
        assert sp.prep_sms >= 20 and sp.prep_sms % 8 == 0       # whole 8-SM granules
        assert 0 < sp.compute_sms and sp.prep_sms + sp.compute_sms <= total
    for bad in (0, total):
        with pytest.raises(uw.UwError):
            uw.SmSplit(bad)


def test_stack_on_split_streams_matches_single_calls(uw):
    """The matmuls on the compute partition's stream, the decodes and
    transcodes on the preprocessing partition's: every step bit-identical to
    the single call."""
    mats, ws, steps = make_stack(uw)
    want = reference_outputs(uw, steps)
    stack = uw.Stack(steps)
    with uw.SmSplit(24) as sp:
        for rep in range(2):
            for _, _, y, _ in steps:
                y.fill_(float("nan"))
            torch.cuda.synchronize()
            stack.run(stream=sp.compute_stream, side_stream=sp.prep_stream)
            sp.compute_stream.synchronize()
            for s, (st, w_ref) in enumerate(zip(steps, want)):
                got = st[2].cpu().numpy()
                assert np.array_equal(got.view(np.uint32), w_ref.view(np.uint32)), "step %d rep %d" % (s, rep)
    for mat in mats:
        assert mat.device_status() == 0


def test_tune_split_picks_a_candidate(uw):
    mats, ws, steps = make_stack(uw, layers=2, m_list=(1,))
    want = reference_outputs(uw, steps)
    stack = uw.Stack(steps)
    cands = [0, 16, 32]
    best, us = stack.tune_split(cands, reps=2)
    assert best in cands and len(us) == 3 and all(u > 0 for u in us)
    assert us[cands.index(best)] == min(us)
    for (_, _, y, _), w_ref in zip(steps, want):          # the last timed run's outputs
        assert np.array_equal(y.cpu().numpy().view(np.uint32), w_ref.view(np.uint32))
    for mat in mats:
        assert mat.device_status() == 0
