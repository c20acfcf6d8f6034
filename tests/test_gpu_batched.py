"""Many fused matmuls in one launch (uw_fused_matmul_batched), the shape of a
mixture-of-experts layer: every item must equal the single-matrix call bit for
bit and lie within the oracle's bound.  Items mix n, k, token counts
(including experts with no tokens) and palettes, and there are more items than
one launch takes, so the items are split over several launches."""
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


def make_items(uw, shapes, n_items, seed0):
    ms = [0, 1, 2, 3, 5, 8, 9, 16]
    items, ws, xs = [], [], []
    for i in range(n_items):
        n, k = shapes[i % len(shapes)]
        m = ms[i % len(ms)]
        w = synth.weights_bf16(n, k, 0.01 + 0.002 * (i % 5), 0.002, 1.0, seed=seed0 + i)
        x = synth.activations_bf16(m, k, seed=seed0 + i) if m else np.zeros((0, k), np.uint16)
        mat = uw.Matrix(uw.encode(w))
        xd = torch.from_numpy(x.view(np.int16)).cuda()
        yd = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        items.append((mat, xd, yd))
        ws.append(w)
        xs.append(x)
    return items, ws, xs


@pytest.mark.parametrize("slices,width", [(1, 0), (4, 0), (4, 1), (8, 2)])
def test_batched_equals_single_calls(uw, slices, width):
    # every k a multiple of 128: width 0 takes 32 weights per lane, as the single call does
    items, ws, xs = make_items(uw, [(256, 1024), (128, 1536), (512, 512), (64, 2048)], 40, 300 + slices)
    plan = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, slices, 1, width)
    uw.fused_matmul_batched(items, plan)
    for i, (mat, xd, yd) in enumerate(items):
        if xd.shape[0] == 0:
            continue
        want = mat.matmul(xd, plan).cpu().numpy()
        got = yd.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), "item %d" % i
        assert mat.device_status() == 0
    for i in (1, 7, 15):      # m = 1, 16, 16
        y_ref, a_ref = O.gemm(xs[i], ws[i])
        err = np.abs(items[i][2].cpu().numpy().astype(np.float64) - y_ref)
        assert (err <= TOL * a_ref + 1e-30).all()


def test_batched_mixed_k_uses_one_step_width(uw):
    # k = 1600 is not a multiple of 128: with width 0 the whole launch takes 16
    # weights per lane, the same as the single call with width 1
    items, ws, xs = make_items(uw, [(128, 1600), (256, 1024), (64, 704)], 12, 900)
    uw.fused_matmul_batched(items, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, 3, 1, 0))
    single = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, 3, 1, 1)
    for i, (mat, xd, yd) in enumerate(items):
        if xd.shape[0]:
            want = mat.matmul(xd, single).cpu().numpy()
            assert np.array_equal(yd.cpu().numpy().view(np.uint32), want.view(np.uint32)), "item %d" % i
