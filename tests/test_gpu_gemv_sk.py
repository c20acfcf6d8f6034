"""GPU parity of the persistent stream-K warp-MMA kernel (UW_KERNEL_MMA_SK).

The fused kernel (W rebuilt from its compressed planes, which each lane
copies into a shared-memory ring) must be bit-identical to the same kernel on
plain BF16 weights through every pipeline, and every output must lie within
|y - y_oracle| <= 1e-4 * sum|x w| of the float64 oracle.  The shapes make the
schedule cut tiles between warps in every way it can: one unit per warp
(every tile in 8 or 112 pieces), runs of one to a few units that start and end
inside tiles, whole tiles inside a run, and the last CTA's spare warps; the
weights include raw-heavy matrices (5% outliers) and bitmap words that
straddle rows.  The tile counters must be left at zero by every call.
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


def dev16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def check_bound(y_gpu, y_ref, a_ref):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bad = err > TOL * a_ref + 1e-30
    assert not bad.any(), "max err/bound %.3g at %s" % (
        float((err / np.maximum(TOL * a_ref, 1e-30)).max()), np.argwhere(bad)[:5].tolist())


def plan(uw, pipe, warps, stages):
    return uw.make_plan(pipeline=pipe, kernel=uw.KERNEL_MMA_SK, bn=warps, split_k=1, stages=stages)


def sk_case(uw, n, k, m, warps, stages=0, seed=0, frac=0.002, pipelines=(1, 2, 3, 4), oracle=True):
    """Plain BF16 twin vs every pipeline bit for bit, and the oracle bound."""
    w = synth.weights_bf16(n, k, 0.02, frac, 1.0, seed=seed)
    x = synth.activations_bf16(m, k, seed=seed)
    mat = uw.Matrix(uw.encode(w))
    xd, wd = dev16(x), dev16(w)
    p = plan(uw, 4, warps, stages)
    ws = uw.new_workspace(uw.workspace_size(m, n, k, p), xd.device)
    y_plain = uw.matmul_bf16(xd, wd, p, ws=ws).cpu().numpy()
    for pipe in pipelines:
        y = mat.matmul(xd, plan(uw, pipe, warps, stages)).cpu().numpy()
        assert np.array_equal(y.view(np.uint32), y_plain.view(np.uint32)), "pipeline %d differs" % pipe
    assert mat.device_status() == 0
    # every call that completes leaves the tile counters at zero
    tiles = n // 16
    assert int(ws[: tiles * 4].view(torch.int32).abs().sum()) == 0
    if oracle:
        y_ref, a_ref = O.gemm(x, w)
        check_bound(y_plain, y_ref, a_ref)
    return y_plain


@pytest.mark.parametrize("m", [1, 2, 5, 8, 9, 13, 16])
def test_gemv_sk_parity(uw, m):
    # 256 tiles x 8 chunks = 2048 units over 1184 warps: runs of 1-2 units
    # that start and end inside tiles
    sk_case(uw, 4096, 1024, m, 8, 0, seed=m)


@pytest.mark.parametrize("warps,stages", [(1, 2), (4, 8), (8, 4), (12, 3), (16, 2), (16, 0)])
def test_gemv_sk_warps_and_stages(uw, warps, stages):
    # 128 tiles x 32 chunks: runs from 1 to 28 units, whole tiles inside runs
    sk_case(uw, 2048, 4096, 4, warps, stages, seed=20 + warps)


def test_gemv_sk_one_unit_per_warp(uw):
    # 1024^2: 512 units, fewer than the warps: one unit each, 8 pieces per tile
    sk_case(uw, 1024, 1024, 1, 16, 2, seed=31)
    # a long K on few rows: 16 tiles x 112 chunks = 1792 units, one per warp,
    # so every tile is summed from 112 pieces
    sk_case(uw, 256, 14336, 9, 12, 2, seed=32, frac=0.001)
    # fewer units than one CTA's warps: a single CTA with spare warps
    sk_case(uw, 64, 128, 3, 16, 2, seed=33)


def test_gemv_sk_raw_heavy_and_straddling_bitmap_words(uw):
    # k = 1408 = 22 groups per row: raw-bitmap words straddle rows; 5% outlier
    # elements make most groups raw
    sk_case(uw, 320, 1408, 3, 8, 4, seed=41, frac=0.05)
    sk_case(uw, 192, 1408, 16, 8, 2, seed=42, frac=0.05)
    sk_case(uw, 448, 2432, 7, 12, 2, seed=43, frac=0.002)


def test_gemv_sk_ring_depth_does_not_change_bits(uw):
    """The schedule depends on the warps per CTA only, so ring depths give
    the same bits."""
    ys = [sk_case(uw, 1024, 2048, 6, 8, s, seed=50, pipelines=(4,), oracle=(s == 2)) for s in (2, 3, 4, 0)]
    assert all(np.array_equal(ys[0].view(np.uint32), y.view(np.uint32)) for y in ys[1:])


def test_gemv_sk_workspace_reuse_across_shapes(uw):
    """One zero-filled workspace serves calls of different shapes, token
    counts and warps in any order (every completed call leaves the counters
    zero), shared with the tcgen05 stream-K kernel."""
    cases = [(4096, 1024, 1, 8, 5, uw.KERNEL_MMA_SK), (256, 14336, 16, 8, 2, uw.KERNEL_MMA_SK),
             (384, 1024, 64, 64, 0, uw.KERNEL_TC_SK), (1024, 1024, 9, 12, 2, uw.KERNEL_MMA_SK)]
    mats, xs, plans, fresh = [], [], [], []
    for i, (n, k, m, bn, stages, kern) in enumerate(cases):
        w = synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=60 + i)
        mats.append(uw.Matrix(uw.encode(w)))
        xs.append(dev16(synth.activations_bf16(m, k, seed=60 + i)))
        plans.append(uw.make_plan(pipeline=4, kernel=kern, bn=bn, split_k=1, stages=stages))
        fresh.append(mats[-1].matmul(xs[-1], plans[-1]).cpu().numpy())
    size = max(mat.workspace_bytes(x.shape[0], p) for mat, x, p in zip(mats, xs, plans))
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    for order in ([0, 1, 2, 3], [3, 2, 1, 0], [1, 1, 0, 0, 3, 2]):
        for i in order:
            y = mats[i].matmul(xs[i], plans[i], ws=ws).cpu().numpy()
            assert np.array_equal(y.view(np.uint32), fresh[i].view(np.uint32))
    assert all(mat.device_status() == 0 for mat in mats)


def test_gemv_sk_unsynchronised_chain(uw):
    """Direct-palette calls issued back to back with no synchronisation,
    sharing one Y and one workspace (each starts early and reads only the
    blob's planes before the previous kernel ends): every result equals the
    same call run alone."""
    n, k = 2048, 4096
    mats = [uw.Matrix(uw.encode(synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=70 + i))) for i in range(3)]
    xs = [dev16(synth.activations_bf16(m, k, seed=70 + m)) for m in (1, 8, 16)]
    plans = [plan(uw, 4, 8, 0), plan(uw, 4, 11, 0), plan(uw, 4, 6, 0)]
    alone = [[mats[i].matmul(xs[j], plans[(i + j) % 3]).cpu().numpy() for j in range(3)] for i in range(3)]
    size = max(mats[0].workspace_bytes(16, p) for p in plans)
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    y = torch.empty(16, n, dtype=torch.float32, device="cuda")
    outs = []
    for i in range(3):
        for j in range(3):
            m = xs[j].shape[0]
            mats[i].matmul(xs[j], plans[(i + j) % 3], y=y[:m], ws=ws)
            outs.append(y[:m].clone())   # on the same stream: ordered after the call
    torch.cuda.synchronize()
    for i in range(3):
        for j in range(3):
            got = outs[3 * i + j].cpu().numpy()
            assert np.array_equal(got.view(np.uint32), alone[i][j].view(np.uint32)), (i, j)
    assert all(mat.device_status() == 0 for mat in mats)


def test_gemv_sk_in_a_stack_with_split_k_steps(uw):
    """A stack mixing split-K tcgen05 steps (whose partial sums share the
    stack's scratch) with stream-K warp-MMA steps: every step equals its
    single call bit for bit."""
    n, k = 1024, 2048
    mats = [uw.Matrix(uw.encode(synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=80 + i))) for i in range(3)]
    x = dev16(synth.activations_bf16(16, k, seed=80))
    plans = [uw.make_plan(pipeline=4, kernel=uw.KERNEL_TC, bn=16, split_k=8), plan(uw, 4, 8, 2),
             plan(uw, 1, 10, 2), uw.make_plan(pipeline=4, kernel=uw.KERNEL_TC, bn=16, split_k=4),
             plan(uw, 3, 6, 3)]
    steps = []
    for i, p in enumerate(plans):
        steps.append((mats[i % 3], x, torch.empty(16, n, dtype=torch.float32, device="cuda"), p))
    st = uw.Stack(steps)
    side = torch.cuda.Stream()
    for _ in range(2):
        st.run(side_stream=side)
        torch.cuda.synchronize()
        for (mat, _, y, p) in steps:
            ref = mat.matmul(x, p).cpu().numpy()
            assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert all(mat.device_status() == 0 for mat in mats)


@pytest.mark.slow
@pytest.mark.parametrize("m,warps,stages", [(1, 8, 5), (4, 16, 2), (16, 8, 2)])
@pytest.mark.parametrize("proj", [(14336, 4096), (4096, 14336)])
def test_gemv_sk_full_size_8b_sampled(uw, m, warps, stages, proj):
    """Llama-3.1-8B gate and down shapes at the bench's batch sizes: fused
    (palette and exponent-plane pipelines) == plain bit for bit over the whole
    output, and 512 sampled outputs within the oracle bound."""
    n, k = proj
    w = synth.weights_bf16(n, k, 0.02, 0.0005, 1.0, seed=1)
    x = synth.activations_bf16(m, k, seed=1)
    mat = uw.Matrix(uw.encode(w))
    xd, wd = dev16(x), dev16(w)
    yp = uw.matmul_bf16(xd, wd, plan(uw, 4, warps, stages)).cpu().numpy()
    for pipe in (4, 2):
        yf = mat.matmul(xd, plan(uw, pipe, warps, stages)).cpu().numpy()
        assert np.array_equal(yf.view(np.uint32), yp.view(np.uint32)), "pipeline %d" % pipe
    assert mat.device_status() == 0
    rng = np.random.default_rng(0)
    ri = rng.integers(0, m, 512)
    rj = rng.integers(0, n, 512)
    ri[:2], rj[:2] = [0, m - 1], [0, n - 1]
    y_ref, a_ref = O.gemm_sampled(x, w, ri, rj)
    check_bound(yp[ri, rj], y_ref, a_ref)
