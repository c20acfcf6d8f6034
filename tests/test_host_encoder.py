"""Host side of libuw on CPU: exports, encoder vs oracle, blob checks, plans.

No GPU is needed: these tests load libuw.so, call only host entry points (and
device entry points with invalid arguments, which must fail before touching
the GPU) and compare the production encoder with the CPU oracle section by
section.
"""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import oracle as O
from decode_gemm_exponent_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def uw():
    from decode_gemm_exponent_b200 import build
    build.build()
    from decode_gemm_exponent_b200 import uw as U
    return U


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "uw.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(uw_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(uw):
    declared = _declared_functions()
    assert len(declared) >= 16
    lib = ctypes.CDLL(uw.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(uw.EXPORTS) == declared
    assert "sm_100a" in uw.version()


# ------------------------------------------------------------------ encoder parity

def _cases():
    rng = np.random.default_rng(0)
    e = np.tile(np.arange(60, 124, dtype=np.uint16), 8)
    all_raw = ((e << 7) | rng.integers(0, 128, e.size).astype(np.uint16)).reshape(4, 128)
    one_exp = ((np.uint16(121) << 7) | (rng.integers(0, 256, 64 * 128).astype(np.uint16) & 0x807F))
    return {
        "small_cfg": synth.weights_bf16(128, 1024, 0.02, 0.001, 2.0, seed=0),
        "ragged_chunk": synth.weights_bf16(64, 192, 0.02, 0.01, 1.0, seed=2),
        "all_patterns": np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(1024, 64),
        "all_raw": np.tile(all_raw, (16, 1)),
        "one_exponent": one_exp.astype(np.uint16).reshape(64, 128),
        "heavy_outliers": synth.weights_bf16(64, 512, 0.015, 0.05, 1.0, seed=5),
        "wide_sigma": synth.weights_bf16(64, 256, 0.05, 0.0, 1.0, seed=6),
        # a mixture-of-experts expert's gate shape, as the batched matmul runs it
        "moe_expert_768x2048": synth.weights_bf16(768, 2048, 0.02, 0.0005, 1.0, seed=1),
    }


def _bits(words: np.ndarray, count: int) -> np.ndarray:
    """u32 word array -> 0/1 flags (LSB of word 0 first)."""
    return ((words[:, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(np.uint8).ravel()[:count]


@pytest.mark.parametrize("case", list(_cases().keys()))
def test_encoder_matches_oracle(uw, case):
    w = _cases()[case]
    if w.shape[0] % 64:
        pytest.skip("rows must be a multiple of 64")
    blob = uw.encode(w)
    info = uw.blob_info(blob, verify_payload=True)
    ref = O.encode(w)
    n, k = w.shape
    assert (info.n, info.k) == (n, k)
    assert list(info.palette)[:info.palette_size] == list(ref.palette)
    assert list(info.code_len) == list(ref.code_len)
    assert info.n_raw == ref.n_raw and info.stream_bits == ref.stream_bits
    assert np.array_equal(uw.section(blob, uw.SEC_SM, info), ref.sm)
    assert np.array_equal(uw.section(blob, uw.SEC_RAWEXP, info), ref.rawexp)
    flags = uw.section(blob, uw.SEC_FLAGS, info).view("<u4")
    assert np.array_equal(_bits(flags, n * k // 64), ref.raw)
    base = uw.section(blob, uw.SEC_RAWBASE, info).view("<u4")
    nw = (n * k // 64 + 31) // 32
    pc = np.array([bin(int(x)).count("1") for x in flags[:nw]], np.int64)
    assert np.array_equal(base[:nw].astype(np.int64), np.concatenate([[0], np.cumsum(pc)[:-1]]))
    stream = uw.section(blob, uw.SEC_STREAM, info).view("<u4")
    nwords = len(ref.stream)
    assert np.array_equal(stream[:nwords], ref.stream) and not stream[nwords:].any()
    off = uw.section(blob, uw.SEC_CHUNKOFF, info).view("<u4")
    assert np.array_equal(off[:len(ref.chunk_off)], ref.chunk_off)
    assert np.array_equal(uw.section(blob, uw.SEC_PAL, info), ref.pal_plane)
    # statistics reported in the header
    h = O.histogram(w)
    assert info.entropy_bits == pytest.approx(O.entropy_bits(h), abs=1e-9)
    assert info.top16_coverage == pytest.approx(float(h[ref.palette].sum()) / w.size, abs=1e-12)


def test_encoder_is_deterministic_and_sizes(uw):
    w = synth.weights_bf16(256, 1024, 0.02, 0.0005, 1.0, seed=3)
    a, b = uw.encode(w), uw.encode(w)
    assert a == b
    info = uw.blob_info(a)
    # Huffman form is smaller than BF16, the palette form in between
    assert info.huffman_bytes < info.palette_bytes < w.nbytes
    only_h = uw.blob_info(uw.encode(w, uw.EMIT_HUFFMAN))
    only_p = uw.blob_info(uw.encode(w, uw.EMIT_PALETTE))
    assert only_h.section_bytes[uw.SEC_PAL] == 0 and only_p.section_bytes[uw.SEC_STREAM] == 0
    for s in range(uw.NUM_SECTIONS):
        assert info.section_offset[s] % 256 == 0


def test_decode_table_reproduces_oracle_symbols(uw):
    """Decode the production stream on the CPU with the production 12-bit
    multi-symbol table and compare the symbols with the oracle's palette
    indices (catches table bugs before any kernel runs)."""
    w = synth.weights_bf16(64, 512, 0.02, 0.002, 1.0, seed=8)
    blob = uw.encode(w)
    info = uw.blob_info(blob)
    lut = uw.section(blob, uw.SEC_DLUT, info).view("<u4")
    stream = uw.section(blob, uw.SEC_STREAM, info).view("<u4")
    ref = O.encode(w)
    want = []
    e = ((w.ravel() >> 7) & 0xFF)
    raw_el = np.repeat(ref.raw.astype(bool), 64)
    want = np.searchsorted(ref.palette, e[~raw_el])
    got = []
    p = 0
    total = len(want)
    while len(got) < total:
        wi = p >> 5
        win = ((int(stream[wi]) << 32 | int(stream[wi + 1])) >> (64 - 12 - (p & 31))) & 0xFFF
        ent = int(lut[win])
        symbits, invalid, nb = (ent >> 20) & 31, (ent >> 25) & 1, ent >> 28
        cnt = symbits // 4
        assert cnt > 0 and symbits % 4 == 0 and not invalid and (ent >> 26) & 3 == 0
        assert ent & 0xFFFFF < 1 << symbits
        if cnt <= total - len(got):
            got += [(ent >> (4 * j)) & 15 for j in range(cnt)]
            p += nb
        else:
            s0 = ent & 15
            got.append(s0)
            p += int(info.code_len[s0])
    assert p == info.stream_bits
    assert np.array_equal(np.array(got), want)


def test_decode_table_one_symbol_code(uw):
    """With one palette symbol the code is the single bit 0: a window that
    starts with z zero bits holds min(z, 5) codes in as many bits; windows
    that start with 1 match no code, are marked invalid and skip the whole
    12-bit window."""
    rng = np.random.default_rng(5)
    w = (0x3C80 | rng.integers(0, 1 << 7, (64, 256)) | (rng.integers(0, 2, (64, 256)) << 15)).astype(np.uint16)
    blob = uw.encode(w)
    info = uw.blob_info(blob)
    assert info.palette_size == 1 and info.code_len[0] == 1
    lut = uw.section(blob, uw.SEC_DLUT, info).view("<u4").astype(np.int64)
    for v in range(2048):
        cnt = min(5, 12 - v.bit_length())
        assert lut[v] == (cnt << 28) | (4 * cnt << 20), v
    assert np.all(lut[2048:] == (12 << 28) | (1 << 25))
    assert info.stream_bits == 64 * 256


# ------------------------------------------------------------------ fault injection (host)

def test_blob_corruption_is_rejected(uw):
    w = synth.weights_bf16(64, 256, 0.02, 0.001, 1.0, seed=4)
    blob = bytearray(uw.encode(w))
    uw.blob_info(bytes(blob), verify_payload=True)

    def status(b, verify=True):
        try:
            uw.blob_info(bytes(b), verify_payload=verify)
            return 0
        except uw.UwError as e:
            return e.status

    CORRUPT = 3
    assert status(blob[:-256]) == CORRUPT                       # truncated
    assert status(blob[:100]) == CORRUPT                        # shorter than a header
    bad = bytearray(blob); bad[0] ^= 0xFF
    assert status(bad) == CORRUPT                               # magic
    bad = bytearray(blob); bad[4] = 7
    assert status(bad) == CORRUPT                               # version (and header CRC)
    bad = bytearray(blob); bad[40] ^= 1
    assert status(bad) == CORRUPT                               # any header byte (CRC)
    bad = bytearray(blob); bad[len(bad) - 300] ^= 0x10
    assert status(bad, verify=True) == CORRUPT                  # payload CRC
    assert status(bad, verify=False) == 0                       # header-only check passes


def test_invalid_arguments(uw):
    lib = uw.lib()
    out = ctypes.c_void_p()
    w = np.zeros((64, 64), np.uint16)
    assert lib.uw_encode(None, 64, 64, 0, ctypes.byref(out)) == 1
    assert lib.uw_encode(w.ctypes.data, 0, 64, 0, ctypes.byref(out)) == 1
    w2 = np.zeros((64, 96), np.uint16)
    assert lib.uw_encode(w2.ctypes.data, 64, 96, 0, ctypes.byref(out)) == 2
    w3 = np.zeros((63, 64), np.uint16)
    assert lib.uw_encode(w3.ctypes.data, 63, 64, 0, ctypes.byref(out)) == 2
    assert lib.uw_encode(w.ctypes.data, 64, 64, 8, ctypes.byref(out)) == 1
    # device entry points reject bad arguments before any CUDA call
    dm = uw.DMat()
    assert lib.uw_decode_to_bf16(None, None, None) == 1
    assert lib.uw_decode_to_bf16(ctypes.byref(dm), None, None) == 1
    assert lib.uw_decode_exponents(None, None, None) == 1
    assert lib.uw_decode_exponents(ctypes.byref(dm), None, None) == 1
    p = uw.make_plan()
    assert lib.uw_fused_matmul(None, 1, ctypes.byref(dm), None, None, ctypes.byref(p), None, 0, None) == 1
    assert lib.uw_matmul_bf16(None, 1, None, 64, 64, None, ctypes.byref(p), None, 0, None, None) == 1
    # a misaligned device blob is refused by bind
    blob = np.frombuffer(uw.encode(w), np.uint8)
    assert lib.uw_matrix_bind(blob.ctypes.data, blob.size, ctypes.c_void_p(0x1001), None, 0,
                              ctypes.byref(dm)) == 1


def test_plans_and_workspace(uw):
    p = uw.plan_default(1, 14336, 4096)
    assert p.kernel == uw.KERNEL_MMA and p.split_k == 1 and p.bn == 4
    p = uw.plan_default(8, 4096, 14336)
    assert p.kernel == uw.KERNEL_MMA
    p = uw.plan_default(9, 4096, 14336)
    assert p.kernel == uw.KERNEL_TC
    p = uw.plan_default(1024, 14336, 4096)
    assert p.kernel == uw.KERNEL_TC and p.bn == 256
    p = uw.plan_default(64, 4096, 14336)
    assert p.kernel == uw.KERNEL_TC and p.bn == 64 and p.split_k >= 1
    n, k = 4096, 1024
    assert uw.workspace_size(1, n, k, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_FMA, 1)) == 0
    assert uw.workspace_size(1, n, k, uw.make_plan(uw.PIPE_DECODE_GEMM, uw.KERNEL_FMA, 1)) == n * k * 2
    assert uw.workspace_size(1, n, k, uw.make_plan(uw.PIPE_TRANSCODE_FUSED, uw.KERNEL_FMA, 1)) == n * k // 2
    # pipeline 2: exponent plane + all-raw bitmap + rank bases (one word per 32 groups each)
    assert uw.workspace_size(1, n, k, uw.make_plan(uw.PIPE_DECODE_EXP_FUSED, uw.KERNEL_MMA, 4)) == \
        n * k + 2 * (n * k // 64 // 32) * 4
    assert uw.workspace_size(64, n, k, uw.make_plan(uw.PIPE_DECODE_EXP_FUSED, uw.KERNEL_TC, 64, 2)) == \
        n * k + 2 * (n * k // 64 // 32) * 4 + 2 * 64 * n * 4
    assert uw.workspace_size(16, n, k, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 16, 4)) == 4 * 16 * n * 4
    for bad in (uw.make_plan(kernel=9), uw.make_plan(bn=48), uw.make_plan(pipeline=0), uw.make_plan(pipeline=5),
                uw.make_plan(kernel=uw.KERNEL_FMA, bn=1, split_k=2), uw.make_plan(split_k=0)):
        with pytest.raises(uw.UwError):
            uw.workspace_size(4, n, k, bad)
    with pytest.raises(uw.UwError):
        uw.workspace_size(16, n, k, uw.make_plan(kernel=uw.KERNEL_FMA, bn=1))   # FMA needs m <= 8
    for slices in (1, 2, 4, 8):
        assert uw.workspace_size(16, n, k, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, slices)) == 0
    for bad_m, bad in ((17, uw.make_plan(kernel=uw.KERNEL_MMA, bn=1)),     # MMA needs m <= 16
                       (4, uw.make_plan(kernel=uw.KERNEL_MMA, bn=0)),
                       (4, uw.make_plan(kernel=uw.KERNEL_MMA, bn=9)),
                       (4, uw.make_plan(kernel=uw.KERNEL_MMA, bn=2, split_k=2)),
                       (4, uw.make_plan(kernel=uw.KERNEL_MMA, bn=2, stages=3))):
        with pytest.raises(uw.UwError):
            uw.workspace_size(bad_m, n, k, bad)
    with pytest.raises(uw.UwError):   # 128-weight steps need K a multiple of 128
        uw.workspace_size(4, n, 1600, uw.make_plan(kernel=uw.KERNEL_MMA, bn=2, stages=2))


def test_binding_constants_match_the_header(uw):
    """Every enum value and flag the binding passes across the ABI equals the
    one include/uw.h declares (the binding restates them by hand)."""
    with open(os.path.join(ROOT, "include", "uw.h"), encoding="utf-8") as f:
        text = re.sub(r"/\*.*?\*/", " ", f.read(), flags=re.S)
    decl = {name: int(val) for name, val in re.findall(r"\b(UW_[A-Z0-9_]+)\s*=\s*(\d+)", text)}
    decl.update({name: int(val) for name, val in re.findall(r"#define\s+(UW_[A-Z0-9_]+)\s+(\d+)u?\b", text)})
    pairs = {"UW_OK": uw.UW_OK, "UW_EMIT_HUFFMAN": uw.EMIT_HUFFMAN, "UW_EMIT_PALETTE": uw.EMIT_PALETTE}
    for name in ("INVALID_ARG", "UNSUPPORTED_SHAPE", "CORRUPT", "CUDA", "NOMEM", "TIMEOUT", "WORKSPACE"):
        pairs["UW_ERR_" + name] = getattr(uw, "ERR_" + name)
    for name in ("SM", "RAWEXP", "FLAGS", "RAWBASE", "STREAM", "CHUNKOFF", "DLUT", "PAL"):
        pairs["UW_SEC_" + name] = getattr(uw, "SEC_" + name)
    for name in ("DECODE_GEMM", "DECODE_EXP_FUSED", "TRANSCODE_FUSED", "DIRECT_PALETTE", "HUFFMAN_FUSED"):
        pairs["UW_PIPE_" + name] = getattr(uw, "PIPE_" + name)
    for name in ("FMA", "TC", "MMA", "TC_SK", "MMA_SK"):
        pairs["UW_KERNEL_" + name] = getattr(uw, "KERNEL_" + name)
    for name, value in pairs.items():
        assert decl.get(name) == value, (name, decl.get(name), value)
    # and every kernel the header declares has a name in the binding's plan files
    assert sorted(uw.KERNEL_NAMES) == sorted(v for n, v in decl.items() if n.startswith("UW_KERNEL_"))


def test_stream_k_gemv_plans_and_workspace(uw):
    """UW_KERNEL_MMA_SK: tile counters (one u32 per 16-row tile, 256-byte
    rounded) then two fragment sets (32 lanes x 4 floats per 8-token tile) per
    warp of the grid; with no GPU the library sizes the grid for 148 SMs.  A
    ring slot and its barrier take 5128 + 256 m bytes, and a CTA's slots must
    fit 227 KB less 128 bytes of alignment slack."""
    def up(x):
        return (x + 255) // 256 * 256

    def fits(warps, stages, m):
        return warps * stages * (5128 + 256 * m) <= 227 * 1024 - 128

    n, k = 14336, 4096
    tiles, units = n // 16, n // 16 * (k // 128)
    for m, nt in ((1, 1), (4, 1), (8, 1), (9, 2), (16, 2)):
        for warps, stages in ((8, 5), (16, 2), (12, 3), (11, 2), (8, 2), (1, 2), (16, 0), (12, 0), (4, 8)):
            p = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA_SK, warps, 1, stages)
            ok = fits(warps, stages, m) if stages else fits(warps, 2, m)
            if ok:
                w = min(148 * warps, units)
                assert uw.workspace_size(m, n, k, p) == up(tiles * 4) + up(2 * w * nt * 32 * 4 * 4), (m, warps, stages)
            else:
                with pytest.raises(uw.UwError):
                    uw.workspace_size(m, n, k, p)
    # a small matrix: at most one warp per unit
    p = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA_SK, 16, 1, 2)
    assert uw.workspace_size(1, 1024, 1024, p) == up(64 * 4) + up(2 * 512 * 32 * 4 * 4)
    # the preprocessing output comes first
    assert uw.workspace_size(1, 1024, 1024, uw.make_plan(uw.PIPE_DECODE_GEMM, uw.KERNEL_MMA_SK, 16, 1, 2)) == \
        1024 * 1024 * 2 + up(64 * 4) + up(2 * 512 * 32 * 4 * 4)
    for bad_m, bad_k, bad in ((17, k, uw.make_plan(kernel=uw.KERNEL_MMA_SK, bn=8)),        # m <= 16
                              (4, 1600, uw.make_plan(kernel=uw.KERNEL_MMA_SK, bn=8)),      # k % 128
                              (4, k, uw.make_plan(kernel=uw.KERNEL_MMA_SK, bn=0)),
                              (4, k, uw.make_plan(kernel=uw.KERNEL_MMA_SK, bn=17)),
                              (4, k, uw.make_plan(kernel=uw.KERNEL_MMA_SK, bn=8, split_k=2)),
                              (4, k, uw.make_plan(kernel=uw.KERNEL_MMA_SK, bn=8, stages=1)),
                              (4, k, uw.make_plan(kernel=uw.KERNEL_MMA_SK, bn=8, stages=9)),
                              (4, k, uw.make_plan(pipeline=5, kernel=uw.KERNEL_MMA_SK, bn=8))):
        with pytest.raises(uw.UwError):
            uw.workspace_size(bad_m, n, bad_k, bad)


def test_stack_workspace_and_argument_checks(uw):
    """uw_stack_workspace_size / uw_stack_run host logic.  The matrix is bound
    to a device address that is never dereferenced (binding reads only the
    host copy), and every uw_stack_run call here fails its argument checks,
    which come before any launch."""
    w = synth.weights_bf16(128, 256, 0.02, 0.002, 1.0, seed=3)
    host = np.frombuffer(uw.encode(w), np.uint8)
    fake = 1 << 40
    dm = uw.DMat()
    uw.check(uw.lib().uw_matrix_bind(host.ctypes.data, host.size, fake, fake, 0, ctypes.byref(dm)),
             "uw_matrix_bind")
    n, k = 128, 256
    plans = [uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 64, 4),
             uw.make_plan(uw.PIPE_TRANSCODE_FUSED, uw.KERNEL_FMA, 1, 1),
             uw.make_plan(uw.PIPE_DECODE_GEMM, uw.KERNEL_TC, 16, 2)]
    ms = [64, 1, 16]
    steps = (uw.StackStep * 3)()
    for i, (p, m) in enumerate(zip(plans, ms)):
        steps[i] = uw.StackStep(ctypes.pointer(dm), fake, m, fake, p, None)
    size = ctypes.c_size_t()
    assert uw.lib().uw_stack_workspace_size(steps, 3, ctypes.byref(size)) == 0
    slot = max(2 * n * k, n * k // 2)                      # decode buffer is the larger
    partial = max(4 * 64 * n * 4, 2 * 16 * n * 4)         # split-K scratch, reused by every step
    assert size.value == 2 * slot + partial
    run = uw.lib().uw_stack_run
    assert run(steps, 3, None, 0, None, None) == uw.ERR_WORKSPACE
    assert run(steps, 3, fake + 1, size.value, None, None) == uw.ERR_WORKSPACE   # misaligned
    assert run(steps, 3, fake, size.value - 1, None, None) == uw.ERR_WORKSPACE
    assert run(steps, 0, fake, size.value, None, None) == uw.ERR_INVALID_ARG
    bad = (uw.StackStep * 3)(*steps)
    bad[1].x_dev = None
    assert run(bad, 3, fake, size.value, None, None) == uw.ERR_INVALID_ARG
    # a pipeline-2 step: its slot holds the exponent plane and two small index
    # arrays (16 words each here, each padded to 256 bytes)
    one = (uw.StackStep * 1)(uw.StackStep(ctypes.pointer(dm), fake, 4, fake,
                                          uw.make_plan(uw.PIPE_DECODE_EXP_FUSED, uw.KERNEL_MMA, 2), None))
    assert uw.lib().uw_stack_workspace_size(one, 1, ctypes.byref(size)) == 0
    assert size.value == 2 * (n * k + 2 * 256)
    one[0].y_dev = None
    assert run(one, 1, fake, size.value, None, None) == uw.ERR_INVALID_ARG
    bad = (uw.StackStep * 3)(*steps)
    bad[2].plan.bn = 24                                   # not a tcgen05 token tile
    assert uw.lib().uw_stack_workspace_size(bad, 3, ctypes.byref(size)) == uw.ERR_INVALID_ARG


def test_sm_split_argument_checks(uw):
    """uw_sm_split_* and uw_stack_tune_split reject bad arguments before any
    CUDA call; with no driver (this host) a valid split request fails with
    UW_ERR_CUDA instead of crashing."""
    lib = uw.lib()
    h = ctypes.c_void_p()
    assert lib.uw_sm_split_create(0, 0, ctypes.byref(h)) == uw.ERR_INVALID_ARG
    assert lib.uw_sm_split_create(-1, 16, ctypes.byref(h)) == uw.ERR_INVALID_ARG
    assert lib.uw_sm_split_create(0, 16, None) == uw.ERR_INVALID_ARG
    st = lib.uw_sm_split_create(0, 16, ctypes.byref(h))
    assert st in (uw.UW_OK, uw.ERR_CUDA)
    if st == uw.UW_OK:                     # a machine with a GPU
        lib.uw_sm_split_destroy(h)
    assert lib.uw_sm_split_get(None, None, None, None, None) == uw.ERR_INVALID_ARG
    lib.uw_sm_split_destroy(None)
    # the tuner: argument and workspace checks on a bound-but-never-read matrix
    w = synth.weights_bf16(128, 256, 0.02, 0.002, 1.0, seed=3)
    host = np.frombuffer(uw.encode(w), np.uint8)
    fake = 1 << 40
    dm = uw.DMat()
    uw.check(lib.uw_matrix_bind(host.ctypes.data, host.size, fake, fake, 0, ctypes.byref(dm)), "uw_matrix_bind")
    steps = (uw.StackStep * 1)(uw.StackStep(ctypes.pointer(dm), fake, 4, fake,
                                            uw.make_plan(uw.PIPE_DECODE_GEMM, uw.KERNEL_MMA, 2), None))
    size = ctypes.c_size_t()
    assert lib.uw_stack_workspace_size(steps, 1, ctypes.byref(size)) == 0
    cand = (ctypes.c_int * 2)(0, 16)
    best = ctypes.c_int()
    tune = lib.uw_stack_tune_split
    assert tune(None, 1, fake, size.value, 0, cand, 2, 1, ctypes.byref(best), None, None) == uw.ERR_INVALID_ARG
    assert tune(steps, 1, fake, size.value, 0, cand, 0, 1, ctypes.byref(best), None, None) == uw.ERR_INVALID_ARG
    assert tune(steps, 1, fake, size.value, 0, cand, 2, 1, None, None, None) == uw.ERR_INVALID_ARG
    assert tune(steps, 1, fake, size.value, -1, cand, 2, 1, ctypes.byref(best), None, None) == uw.ERR_INVALID_ARG
    neg = (ctypes.c_int * 2)(0, -8)
    assert tune(steps, 1, fake, size.value, 0, neg, 2, 1, ctypes.byref(best), None, None) == uw.ERR_INVALID_ARG
    assert tune(steps, 1, fake, size.value - 1, 0, cand, 2, 1, ctypes.byref(best), None, None) == uw.ERR_WORKSPACE
    assert tune(steps, 1, fake + 16, size.value, 0, cand, 2, 1, ctypes.byref(best), None, None) == uw.ERR_WORKSPACE


def test_batched_matmul_argument_checks(uw):
    """uw_fused_matmul_batched checks every item before launching anything
    (the matrices are bound to device addresses that are never read)."""
    lib = uw.lib()
    fake = 1 << 40
    dms = []
    for n, k in ((128, 256), (64, 192)):
        w = synth.weights_bf16(n, k, 0.02, 0.002, 1.0, seed=n + k)
        host = np.frombuffer(uw.encode(w, uw.EMIT_HUFFMAN | uw.EMIT_PALETTE), np.uint8)
        dm = uw.DMat()
        uw.check(lib.uw_matrix_bind(host.ctypes.data, host.size, fake, fake, 0, ctypes.byref(dm)), "uw_matrix_bind")
        dms.append(dm)

    def items(*spec):
        arr = (uw.BatchItem * len(spec))()
        for i, (j, m, x, y) in enumerate(spec):
            arr[i] = uw.BatchItem(ctypes.pointer(dms[j]), x, m, y)
        return arr

    ok = uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, 2, 1, 0)
    run = lambda arr, plan: lib.uw_fused_matmul_batched(arr, len(arr), ctypes.byref(plan), None)
    good = items((0, 4, fake, fake), (1, 1, fake, fake))
    assert lib.uw_fused_matmul_batched(good, 0, ctypes.byref(ok), None) == uw.ERR_INVALID_ARG
    assert lib.uw_fused_matmul_batched(None, 2, ctypes.byref(ok), None) == uw.ERR_INVALID_ARG
    assert run(good, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_TC, 16, 1)) == uw.ERR_INVALID_ARG
    assert run(good, uw.make_plan(uw.PIPE_DECODE_GEMM, uw.KERNEL_MMA, 2, 1)) == uw.ERR_INVALID_ARG
    assert run(good, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, 9, 1)) == uw.ERR_INVALID_ARG
    # 32 weights per lane need every k to be a multiple of 128 (k = 192 is not)
    assert run(good, uw.make_plan(uw.PIPE_DIRECT_PALETTE, uw.KERNEL_MMA, 2, 1, 2)) == uw.ERR_INVALID_ARG
    assert run(items((0, 17, fake, fake)), ok) == uw.ERR_INVALID_ARG
    assert run(items((0, -1, fake, fake)), ok) == uw.ERR_INVALID_ARG
    assert run(items((0, 4, fake + 8, fake)), ok) == uw.ERR_INVALID_ARG      # misaligned x
    assert run(items((0, 4, fake, None)), ok) == uw.ERR_INVALID_ARG          # no y
    assert run(items((0, 4, fake, fake), (1, 2, None, fake)), ok) == uw.ERR_INVALID_ARG
    # experts that nobody routed to are skipped: a batch of them launches nothing and succeeds
    # (this host has no GPU, so any launch would fail)
    assert run(items((0, 0, None, None), (1, 0, None, None)), ok) == uw.UW_OK


def test_header_is_plain_c(tmp_path):
    """include/uw.h is a C interface: it compiles as pedantic C99 and every
    declared entry point links against the library."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use_uw.c"
    src.write_text('#include "uw.h"\n'
                   'int main(void) {\n'
                   '    uw_batch_item it = {0}; uw_stack_step st = {0}; uw_plan p = {0}; uw_sm_split *s = 0;\n'
                   '    (void)it; (void)st; (void)p; (void)s;\n'
                   '    return uw_status_str(UW_OK)[0] == 0;\n'
                   '}\n')
    cuda_inc = "/usr/local/cuda/include"
    lib_dir = os.path.join(root, "decode_gemm_exponent_b200")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(root, "include"), "-I", cuda_inc, str(src),
                        "-L", lib_dir, "-l:libuw.so", "-o", str(tmp_path / "use_uw")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
