"""GPU parity of the persistent stream-K tcgen05 kernel (UW_KERNEL_TC_SK).

The fused kernel (W rebuilt from its compressed planes in shared memory) must
be bit-identical to the same kernel on plain BF16 weights, through every
pipeline, and every output must lie within |y - y_oracle| <= 1e-4 * sum|x w|
of the float64 oracle.  The shapes are chosen so that tiles are cut between
CTAs in every way the schedule allows: two pieces, dozens of pieces (a long K
over few row blocks), one unit per CTA (tiny problems), a ragged last row
block, K steps whose raw-bitmap words straddle rows, and raw-heavy weights.
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


def sk_case(uw, n, k, m, bn, seed=0, frac=0.002, pipelines=(1, 2, 3, 4, 5), stages=0, oracle=True, w=None):
    """Plain BF16 twin vs every pipeline (pipeline 5, the in-kernel Huffman
    decode, where the shape allows it) bit for bit, and the oracle bound."""
    if w is None:
        w = synth.weights_bf16(n, k, 0.02, frac, 1.0, seed=seed)
    x = synth.activations_bf16(m, k, seed=seed)
    mat = uw.Matrix(uw.encode(w))
    xd, wd = dev16(x), dev16(w)
    kw = dict(kernel=uw.KERNEL_TC_SK, bn=bn, split_k=1, stages=stages)
    y_plain = uw.matmul_bf16(xd, wd, uw.make_plan(pipeline=4, **kw)).cpu().numpy()
    for pipe in pipelines:
        if pipe == uw.PIPE_HUFFMAN_FUSED and (bn > 32 or k % 256):
            continue
        y = mat.matmul(xd, uw.make_plan(pipeline=pipe, **kw)).cpu().numpy()
        assert np.array_equal(y.view(np.uint32), y_plain.view(np.uint32)), "pipeline %d differs" % pipe
    assert mat.device_status() == 0
    if oracle:
        y_ref, a_ref = O.gemm(x, w)
        check_bound(y_plain, y_ref, a_ref)
    return y_plain


@pytest.mark.parametrize("bn,m", [(16, 1), (16, 16), (32, 20), (64, 64), (64, 100), (128, 128),
                                  (128, 300), (256, 256), (256, 513)])
def test_sk_parity(uw, bn, m):
    # 3 row blocks x 16 K-steps x ceil(m / bn) token blocks: every tile in pieces
    sk_case(uw, 384, 1024, m, bn, seed=bn + m)


def test_sk_ragged_rows_and_unaligned_bitmap_words(uw):
    # n = 320: the last row block has 64 rows; k = 704 = 11 groups per row, so
    # raw-bitmap words straddle rows; 5% outliers make most groups raw
    sk_case(uw, 320, 704, 40, 64, seed=3, frac=0.05)
    sk_case(uw, 320, 704, 3, 16, seed=4, frac=0.05)
    sk_case(uw, 192, 1344, 17, 32, seed=5, frac=0.002)
    # k = 1280 (5 chunks per row) for the in-kernel Huffman decode: ragged rows, raw-heavy
    sk_case(uw, 320, 1280, 24, 32, seed=13, frac=0.05)
    sk_case(uw, 192, 1280, 5, 16, seed=14, frac=0.002)


def test_sk_huffman_chunks_larger_than_a_stream_slot(uw):
    """Exponents uniform over 16 values: every code is 4 bits, a chunk takes
    1024 bits, and a super-step's 128 chunks (18 KB with their granules) do
    not all fit the 12 KB stream slot, so some decoders read the stream from
    global memory.  Results still equal the plain kernel bit for bit."""
    rng = np.random.default_rng(21)
    n, k = 256, 2048
    e = rng.integers(110, 126, n * k).astype(np.uint16)
    sm = rng.integers(0, 256, n * k).astype(np.uint16)
    w = (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16).reshape(n, k)
    sk_case(uw, n, k, 16, 16, seed=22, pipelines=(4, 5), w=w)
    sk_case(uw, n, k, 100, 32, seed=23, pipelines=(5,), w=w)


def test_sk_huffman_corrupt_stream_is_reported(uw):
    w = synth.weights_bf16(256, 1024, 0.02, 0.001, 1.0, seed=24)
    blob = uw.encode(w)
    mat = uw.Matrix(blob)
    off = mat.info.section_offset[uw.SEC_STREAM] + 256
    mat.dev[off:off + 16] ^= 0x5A                      # the device copy only
    xd = dev16(synth.activations_bf16(8, 1024, seed=24))
    p = uw.make_plan(pipeline=uw.PIPE_HUFFMAN_FUSED, kernel=uw.KERNEL_TC_SK, bn=16, split_k=1)
    mat.matmul(xd, p)
    assert mat.device_status() == 3                   # UW_ERR_CORRUPT
    clean = uw.Matrix(blob)                           # the context is still usable
    y = clean.matmul(xd, p).cpu().numpy()
    assert clean.device_status() == 0
    y_ref, a_ref = O.gemm(synth.activations_bf16(8, 1024, seed=24), w)
    check_bound(y, y_ref, a_ref)


def test_sk_huffman_plan_checks(uw):
    w = synth.weights_bf16(128, 704, 0.02, 0.0, 1.0, seed=25)
    mat = uw.Matrix(uw.encode(w))
    xd = dev16(synth.activations_bf16(4, 704, seed=25))
    for kw in (dict(kernel=uw.KERNEL_TC_SK, bn=16),       # k = 704 is not a multiple of 256
               dict(kernel=uw.KERNEL_TC, bn=16)):          # only the stream-K kernel decodes in place
        with pytest.raises(uw.UwError) as e:
            mat.matmul(xd, uw.make_plan(pipeline=uw.PIPE_HUFFMAN_FUSED, split_k=1, **kw))
        assert e.value.status == 1
    w1 = synth.weights_bf16(128, 1024, 0.02, 0.0, 1.0, seed=27)
    mat1 = uw.Matrix(uw.encode(w1))
    for kw in (dict(kernel=uw.KERNEL_TC_SK, bn=64),):      # the Huffman kernel's token tiles stop at 32
        with pytest.raises(uw.UwError) as e:
            mat1.matmul(dev16(synth.activations_bf16(4, 1024, seed=27)),
                        uw.make_plan(pipeline=uw.PIPE_HUFFMAN_FUSED, split_k=1, **kw))
        assert e.value.status == 1
    w2 = synth.weights_bf16(128, 1024, 0.02, 0.0, 1.0, seed=26)
    mat2 = uw.Matrix(uw.encode(w2, flags=uw.EMIT_PALETTE))  # no Huffman stream in the blob
    with pytest.raises(uw.UwError):
        mat2.matmul(dev16(synth.activations_bf16(4, 1024, seed=26)),
                    uw.make_plan(pipeline=uw.PIPE_HUFFMAN_FUSED, kernel=uw.KERNEL_TC_SK, bn=16, split_k=1))


def test_sk_many_pieces_per_tile(uw):
    # 2 row blocks x 224 K-steps on all SMs: each tile is cut into ~75 pieces
    sk_case(uw, 256, 14336, 16, 16, seed=6, frac=0.001)


def test_sk_tiny_problems(uw):
    # fewer units than SMs: one K-step per CTA; a single 64-row tile
    sk_case(uw, 64, 64, 1, 16, seed=7, pipelines=(1, 4))
    sk_case(uw, 64, 128, 300, 256, seed=8, pipelines=(4,))
    sk_case(uw, 128, 64, 17, 32, seed=9, pipelines=(4,))


def test_sk_stage_depth_does_not_change_bits(uw):
    ys = [sk_case(uw, 256, 768, 32, 32, seed=11, pipelines=(4,), stages=s, oracle=False) for s in (2, 3, 0)]
    assert all(np.array_equal(ys[0].view(np.uint32), y.view(np.uint32)) for y in ys[1:])


def test_sk_workspace_reuse_across_shapes(uw):
    """Every completed call leaves the tile counters zero: one workspace
    serves calls of different shapes and token tiles in any order."""
    cases = [(384, 1024, 100, 64), (256, 14336, 16, 16), (384, 1024, 300, 128), (256, 14336, 1, 16)]
    mats, xs, plans, fresh = [], [], [], []
    for i, (n, k, m, bn) in enumerate(cases):
        w = synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=40 + i)
        mats.append(uw.Matrix(uw.encode(w)))
        xs.append(dev16(synth.activations_bf16(m, k, seed=40 + i)))
        plans.append(uw.make_plan(pipeline=4, kernel=uw.KERNEL_TC_SK, bn=bn, split_k=1))
        fresh.append(mats[-1].matmul(xs[-1], plans[-1]).cpu().numpy())
    size = max(mat.workspace_bytes(x.shape[0], p) for mat, x, p in zip(mats, xs, plans))
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    for order in ([0, 1, 2, 3], [3, 2, 1, 0], [1, 1, 0, 0]):
        for i in order:
            y = mats[i].matmul(xs[i], plans[i], ws=ws).cpu().numpy()
            assert np.array_equal(y.view(np.uint32), fresh[i].view(np.uint32))
    # counters are back at zero
    assert all(mat.device_status() == 0 for mat in mats)


def test_sk_bounded_wait_times_out_and_context_survives(uw):
    w = synth.weights_bf16(256, 512, 0.02, 0.001, 1.0, seed=12)
    x = synth.activations_bf16(16, 512, seed=12)
    mat = uw.Matrix(uw.encode(w))
    xd = dev16(x)
    bad = uw.make_plan(pipeline=4, kernel=uw.KERNEL_TC_SK, bn=16, split_k=1,
                       debug_flags=uw.DEBUG_NEVER_ARRIVE, timeout_ns=2_000_000)
    mat.matmul(xd, bad)
    assert mat.device_status() == 6        # UW_ERR_TIMEOUT
    ok = uw.make_plan(pipeline=4, kernel=uw.KERNEL_TC_SK, bn=16, split_k=1)
    y = mat.matmul(xd, ok).cpu().numpy()   # a fresh (zeroed) workspace
    assert mat.device_status() == 0
    y_ref, a_ref = O.gemm(x, w)
    check_bound(y, y_ref, a_ref)


def test_sk_stack_shares_scratch_with_split_k_steps(uw):
    """A stack whose split-K (TC) steps and stream-K steps share the partial
    scratch: the stream-K counters live apart, so every step equals its
    single call bit for bit."""
    n, k = 384, 1024
    mats = [uw.Matrix(uw.encode(synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=60 + i))) for i in range(3)]
    x = dev16(synth.activations_bf16(64, k, seed=60))
    plans = [uw.make_plan(pipeline=4, kernel=uw.KERNEL_TC, bn=64, split_k=4),
             uw.make_plan(pipeline=3, kernel=uw.KERNEL_TC_SK, bn=64, split_k=1),
             uw.make_plan(pipeline=4, kernel=uw.KERNEL_TC, bn=32, split_k=8),
             uw.make_plan(pipeline=1, kernel=uw.KERNEL_TC_SK, bn=32, split_k=1)]
    steps, ys = [], []
    for i, p in enumerate(plans):
        y = torch.empty(64, n, dtype=torch.float32, device="cuda")
        steps.append((mats[i % 3], x, y, p))
        ys.append(y)
    st = uw.Stack(steps)
    side = torch.cuda.Stream()
    for _ in range(2):
        st.run(side_stream=side)
        torch.cuda.synchronize()
        for (mat, _, y, p) in steps:
            ref = mat.matmul(x, p).cpu().numpy()
            assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert all(m.device_status() == 0 for m in mats)


@pytest.mark.slow
@pytest.mark.parametrize("m,bn", [(1, 16), (4, 16), (16, 16), (64, 64), (256, 256), (1024, 256)])
@pytest.mark.parametrize("proj", [(14336, 4096), (4096, 14336)])
def test_sk_full_size_8b_sampled(uw, m, bn, proj):
    """Llama-3.1-8B gate and down shapes at the bench's batch sizes: fused
    (palette, exponent-plane and in-kernel Huffman pipelines) == plain bit for
    bit over the whole output, and 512 sampled outputs within the oracle bound."""
    n, k = proj
    w = synth.weights_bf16(n, k, 0.02, 0.0005, 1.0, seed=1)
    x = synth.activations_bf16(m, k, seed=1)
    mat = uw.Matrix(uw.encode(w))
    xd, wd = dev16(x), dev16(w)
    kw = dict(kernel=uw.KERNEL_TC_SK, bn=bn, split_k=1)
    yp = uw.matmul_bf16(xd, wd, uw.make_plan(pipeline=4, **kw)).cpu().numpy()
    for pipe in ((4, 2, 5) if bn <= 32 else (4, 2)):
        yf = mat.matmul(xd, uw.make_plan(pipeline=pipe, **kw)).cpu().numpy()
        assert np.array_equal(yf.view(np.uint32), yp.view(np.uint32)), "pipeline %d" % pipe
    assert mat.device_status() == 0
    rng = np.random.default_rng(0)
    ri = rng.integers(0, m, 512)
    rj = rng.integers(0, n, 512)
    ri[:2], rj[:2] = [0, m - 1], [0, n - 1]
    y_ref, a_ref = O.gemm_sampled(x, w, ri, rj)
    check_bound(yp[ri, rj], y_ref, a_ref)
