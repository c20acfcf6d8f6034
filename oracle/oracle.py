"""CPU oracle for lossless BF16 exponent compression (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product package never does; the
oracle and the product share no code.

The arithmetic lives in ``uw_oracle.c`` (plain C, double accumulation); this
module compiles it with gcc and wraps it with ctypes, taking and returning
numpy arrays.  Every function states the passage of the Unweight page
("Unweight：Cloudflare 如何在不损失精度的情况下把大模型压缩 22%") that it
follows; the readings where the page is silent are listed at the top of
``uw_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "uw_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CHUNK_GROUPS = 4      # reading R5: one stored offset per 4 groups
LMAX = 12             # reading R4: code-length limit


def build(force: bool = False) -> str:
    """Compile uw_oracle.c into liboracle.so next to it (gcc, -O2, no fp contraction)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC),
                                              os.path.getmtime(os.path.join(_HERE, "uw_oracle.h"))):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
                               "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.uwo_exponent.restype = ctypes.c_uint8
        lib.uwo_exponent.argtypes = [ctypes.c_uint16]
        lib.uwo_sign_mantissa.restype = ctypes.c_uint8
        lib.uwo_sign_mantissa.argtypes = [ctypes.c_uint16]
        lib.uwo_join.restype = ctypes.c_uint16
        lib.uwo_join.argtypes = [ctypes.c_uint8, ctypes.c_uint8]
        lib.uwo_histogram.argtypes = [P, I64, P]
        lib.uwo_entropy_bits.restype = ctypes.c_double
        lib.uwo_entropy_bits.argtypes = [P]
        lib.uwo_palette.restype = ctypes.c_int
        lib.uwo_palette.argtypes = [P, P]
        lib.uwo_raw_groups.argtypes = [P, I64, I64, P, ctypes.c_int, P]
        lib.uwo_code_lengths.restype = ctypes.c_int
        lib.uwo_code_lengths.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
        lib.uwo_canonical_codes.argtypes = [P, ctypes.c_int, P]
        lib.uwo_pal_get.restype = ctypes.c_int
        lib.uwo_pal_get.argtypes = [P, I64]
        lib.uwo_encode.restype = ctypes.c_int
        lib.uwo_encode.argtypes = [P, I64, I64, P, P, P, P, P, P, P, P, I64, P, P, P]
        lib.uwo_decode.restype = ctypes.c_int
        lib.uwo_decode.argtypes = [I64, I64, P, ctypes.c_int, P, P, P, P, P,
                                   ctypes.c_uint64, P, P]
        lib.uwo_transcode.restype = ctypes.c_int
        lib.uwo_transcode.argtypes = [I64, I64, ctypes.c_int, P, P, P, ctypes.c_uint64, P, P]
        lib.uwo_gemm.argtypes = [P, P, I64, I64, I64, P, P]
        lib.uwo_gemm_sampled.argtypes = [P, P, I64, P, P, I64, P, P]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(w) -> np.ndarray:
    w = np.ascontiguousarray(w)
    if w.dtype != np.uint16:
        w = w.view(np.uint16) if w.dtype.itemsize == 2 else w.astype(np.uint16)
    return np.ascontiguousarray(w)


# --------------------------------------------------------------------------
# field split (Unweight page §三: 1 sign, 8 exponent, 7 mantissa bits)

def exponent(w: int) -> int:
    return int(_load().uwo_exponent(int(w)))


def sign_mantissa(w: int) -> int:
    return int(_load().uwo_sign_mantissa(int(w)))


def join(e: int, sm: int) -> int:
    return int(_load().uwo_join(int(e), int(sm)))


# --------------------------------------------------------------------------
# statistics and palette (Unweight page §三, §四)

def histogram(w) -> np.ndarray:
    w = _u16(w).ravel()
    h = np.zeros(256, np.uint64)
    _load().uwo_histogram(_p(w), w.size, _p(h))
    return h


def entropy_bits(hist) -> float:
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    return float(_load().uwo_entropy_bits(_p(h)))


def palette(hist) -> np.ndarray:
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    pal = np.zeros(16, np.uint8)
    size = _load().uwo_palette(_p(h), _p(pal))
    return pal[:size].copy()


def raw_groups(w, palette_values) -> np.ndarray:
    w = _u16(w)
    n, k = w.shape
    pal = np.zeros(16, np.uint8)
    pal[:len(palette_values)] = palette_values
    raw = np.zeros(n * k // 64, np.uint8)
    _load().uwo_raw_groups(_p(w), n, k, _p(pal), len(palette_values), _p(raw))
    return raw


# --------------------------------------------------------------------------
# Huffman code (Unweight page §四), reading R4

def code_lengths(freq, lmax: int = LMAX) -> np.ndarray:
    f = np.ascontiguousarray(freq, dtype=np.uint64)
    lens = np.zeros(len(f), np.uint8)
    rc = _load().uwo_code_lengths(_p(f), len(f), lmax, _p(lens))
    if rc != 0:
        raise ValueError("uwo_code_lengths failed: %d" % rc)
    return lens


def canonical_codes(lens) -> np.ndarray:
    l8 = np.ascontiguousarray(lens, dtype=np.uint8)
    codes = np.zeros(len(l8), np.uint32)
    _load().uwo_canonical_codes(_p(l8), len(l8), _p(codes))
    return codes


# --------------------------------------------------------------------------
# encoder / decoder / transcoder

@dataclass
class Encoded:
    n: int
    k: int
    palette: np.ndarray       # uint8[psize], ascending
    code_len: np.ndarray      # uint8[16]
    sm: np.ndarray            # uint8[n*k]
    raw: np.ndarray           # uint8[n*k/64], 0/1 per group
    rawexp: np.ndarray        # uint8[n_raw*64]
    stream: np.ndarray        # uint32[ceil(bits/32)]
    stream_bits: int
    chunk_off: np.ndarray     # uint32[n_chunks+1]
    pal_plane: np.ndarray     # uint8[n*k/2]

    @property
    def n_raw(self) -> int:
        return int(self.raw.sum())


def encode(w) -> Encoded:
    """Unweight page §三-§四 and §六: split, palette, raw rows, Huffman stream,
    plus the pre-transcoded 4-bit palette plane."""
    w = _u16(w)
    n, k = w.shape
    count = n * k
    groups = count // 64
    chunks = (groups + CHUNK_GROUPS - 1) // CHUNK_GROUPS
    pal = np.zeros(16, np.uint8)
    psize = ctypes.c_int(0)
    code_len = np.zeros(16, np.uint8)
    sm = np.zeros(count, np.uint8)
    raw = np.zeros(groups, np.uint8)
    rawexp = np.zeros(count, np.uint8)
    n_raw = ctypes.c_int64(0)
    cap = (count * LMAX) // 32 + 2
    stream = np.zeros(cap, np.uint32)
    bits = ctypes.c_uint64(0)
    off = np.zeros(chunks + 1, np.uint32)
    pal_plane = np.zeros(count // 2, np.uint8)
    rc = _load().uwo_encode(_p(w), n, k, _p(pal), ctypes.byref(psize), _p(code_len),
                            _p(sm), _p(raw), _p(rawexp), ctypes.byref(n_raw),
                            _p(stream), cap, ctypes.byref(bits), _p(off), _p(pal_plane))
    if rc != 0:
        raise ValueError("uwo_encode failed: %d" % rc)
    nb = int(bits.value)
    return Encoded(n, k, pal[:psize.value].copy(), code_len, sm, raw,
                   rawexp[:n_raw.value * 64].copy(), stream[:(nb + 31) // 32].copy(), nb,
                   off, pal_plane)


def _stream_padded(enc: Encoded) -> np.ndarray:
    s = np.zeros(len(enc.stream) + 2, np.uint32)
    s[:len(enc.stream)] = enc.stream
    return s


def decode(enc: Encoded) -> np.ndarray:
    """Full decode back to BF16 bits (Unweight page §六, first pipeline)."""
    pal = np.zeros(16, np.uint8)
    pal[:len(enc.palette)] = enc.palette
    out = np.zeros(enc.n * enc.k, np.uint16)
    rawexp = enc.rawexp if enc.rawexp.size else np.zeros(64, np.uint8)
    rc = _load().uwo_decode(enc.n, enc.k, _p(pal), len(enc.palette), _p(enc.code_len),
                            _p(enc.sm), _p(enc.raw), _p(rawexp), _p(_stream_padded(enc)),
                            enc.stream_bits, _p(enc.chunk_off), _p(out))
    if rc != 0:
        raise ValueError("uwo_decode: corrupt input (%d)" % rc)
    return out.reshape(enc.n, enc.k)


def transcode(enc: Encoded) -> np.ndarray:
    """Huffman stream -> 4-bit palette plane (Unweight page §六, third pipeline)."""
    out = np.zeros(enc.n * enc.k // 2, np.uint8)
    rc = _load().uwo_transcode(enc.n, enc.k, len(enc.palette), _p(enc.code_len), _p(enc.raw),
                               _p(_stream_padded(enc)), enc.stream_bits, _p(enc.chunk_off),
                               _p(out))
    if rc != 0:
        raise ValueError("uwo_transcode: corrupt input (%d)" % rc)
    return out


def pal_get(plane, elem: int) -> int:
    p = np.ascontiguousarray(plane, dtype=np.uint8)
    return int(_load().uwo_pal_get(_p(p), int(elem)))


# --------------------------------------------------------------------------
# matmul (Unweight page §七), double accumulation

def gemm(x, w):
    """Y = X W^T and A = |X| |W|^T elementwise-abs sums, both float64 [m, n]."""
    x = _u16(x)
    w = _u16(w)
    m, k = x.shape
    n, k2 = w.shape
    assert k == k2
    y = np.zeros((m, n), np.float64)
    a = np.zeros((m, n), np.float64)
    _load().uwo_gemm(_p(x), _p(w), m, n, k, _p(y), _p(a))
    return y, a


def gemm_sampled(x, w, rows_i, rows_j):
    """Y[i_c, j_c] and A[i_c, j_c] for the listed (token row, weight row) pairs."""
    x = _u16(x)
    w = _u16(w)
    k = x.shape[1]
    assert w.shape[1] == k
    ri = np.ascontiguousarray(rows_i, dtype=np.int64)
    rj = np.ascontiguousarray(rows_j, dtype=np.int64)
    y = np.zeros(len(ri), np.float64)
    a = np.zeros(len(ri), np.float64)
    _load().uwo_gemm_sampled(_p(x), _p(w), k, _p(ri), _p(rj), len(ri), _p(y), _p(a))
    return y, a
