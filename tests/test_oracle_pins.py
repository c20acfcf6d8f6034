"""Pins for the CPU oracle: checks it against facts fixed outside itself.

Each test ties an oracle function to something independent of it: IEEE/BF16
semantics, hand-worked golden examples (tests/golden/), closed forms, brute
force over tiny alphabets, a textbook Huffman, a dynamic program for
length-limited codes, numpy/scipy library routines, and the exponent
statistics the Unweight page reports (section 三: top-16 exponents cover
more than 99% of weights, about 2.6 bits of entropy).
"""
import heapq
import itertools
import json
import math
import os
import struct

import numpy as np
import pytest

from oracle import oracle as O
from decode_gemm_exponent_b200 import synth


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _words_le(plane_bytes: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(plane_bytes).view("<u4")


# ---------------------------------------------------------------- BF16 fields

def test_bf16_golden_fields(golden_dir):
    g = _golden(golden_dir, "bf16_fields.json")
    for row in g["rows"]:
        b = int(row["bits"], 16)
        assert O.exponent(b) == row["exponent"]
        assert O.sign_mantissa(b) == int(row["sm"], 16)
        assert O.join(row["exponent"], int(row["sm"], 16)) == b
        # the bits denote the stated value (float32 = bf16 bits << 16)
        v = struct.unpack("<f", struct.pack("<I", b << 16))[0]
        want = float(row["value"])
        if math.isnan(want):
            assert math.isnan(v)
        else:
            assert v == want and math.copysign(1, v) == math.copysign(1, want)


def test_split_join_exhaustive_against_ieee_semantics():
    """All 65,536 patterns: join(split(w)) == w, and the split fields agree with
    the number the pattern denotes (frexp-based exponent, sign bit)."""
    for b in range(65536):
        e = O.exponent(b)
        sm = O.sign_mantissa(b)
        assert O.join(e, sm) == b
        v = struct.unpack("<f", struct.pack("<I", b << 16))[0]
        sign = 1 if math.copysign(1.0, v) < 0 else 0
        assert (sm >> 7) == sign
        if math.isinf(v) or math.isnan(v):
            assert e == 255
        elif v == 0.0:
            assert e == 0 and (sm & 0x7F) == 0
        else:
            mant, ex = math.frexp(abs(v))          # abs(v) = mant * 2**ex, mant in [0.5, 1)
            if e == 0:                              # subnormal: 0.m * 2**-126
                assert abs(v) == (sm & 0x7F) * 2.0 ** -133
            else:
                assert e == ex - 1 + 127
                assert abs(v) == (1 + (sm & 0x7F) / 128.0) * 2.0 ** (e - 127)


# ---------------------------------------------------------------- palette / raw

def _palette_by_sort(hist):
    nz = np.nonzero(hist)[0]
    order = np.lexsort((nz, -hist[nz].astype(np.int64)))   # count desc, exponent asc
    return np.sort(nz[order][:16]).astype(np.uint8)


@pytest.mark.parametrize("seed", range(20))
def test_palette_is_top16_by_sort(seed):
    rng = np.random.default_rng(seed)
    hist = np.zeros(256, np.uint64)
    ndistinct = int(rng.integers(1, 40))
    idx = rng.choice(256, ndistinct, replace=False)
    # small count range so ties are common
    hist[idx] = rng.integers(1, 6, ndistinct).astype(np.uint64)
    assert np.array_equal(O.palette(hist), _palette_by_sort(hist))


def test_raw_groups_bruteforce():
    w = synth.weights_bf16(16, 256, 0.02, 0.01, 1.0, seed=3)
    hist = O.histogram(w)
    pal = O.palette(hist)
    raw = O.raw_groups(w, pal)
    e = ((w >> 7) & 0xFF).reshape(-1, 64)
    want = (~np.isin(e, pal)).any(axis=1).astype(np.uint8)
    assert raw.sum() > 0 and raw.sum() < raw.size
    assert np.array_equal(raw, want)


def test_histogram_vs_bincount():
    w = synth.weights_bf16(64, 128, 0.02, 0.01, 1.0, seed=4)
    assert np.array_equal(O.histogram(w), np.bincount(((w >> 7) & 0xFF).ravel(),
                                                      minlength=256).astype(np.uint64))


# ---------------------------------------------------------------- code lengths

def _cost(freq, lens):
    return int(sum(int(f) * int(l) for f, l in zip(freq, lens)))


def _brute_force_min_cost(freq, lmax):
    used = [f for f in freq if f > 0]
    n = len(used)
    if n <= 1:
        return sum(used)  # one symbol: one bit each
    best = None
    grid = np.array(list(itertools.product(range(1, lmax + 1), repeat=n)), dtype=np.int64)
    kraft = (2.0 ** (-grid)).sum(axis=1)
    ok = grid[kraft <= 1.0 + 1e-12]
    costs = ok @ np.array(used, dtype=np.int64)
    best = int(costs.min())
    return best


@pytest.mark.parametrize("seed", range(40))
def test_code_lengths_brute_force_optimal(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 8))
    lmax = int(rng.integers(max(2, math.ceil(math.log2(n))), 7)) if n <= 6 else 6
    kind = seed % 3
    if kind == 0:
        freq = rng.integers(0, 20, n)
    elif kind == 1:
        freq = (2 ** rng.integers(0, 12, n))           # skewed, forces the limit
    else:
        freq = np.full(n, int(rng.integers(1, 5)))     # all ties
    freq = freq.astype(np.uint64)
    if (freq > 0).sum() == 0:
        freq[0] = 1
    lens = O.code_lengths(freq, lmax)
    used = freq > 0
    assert np.all(lens[~used] == 0)
    assert np.all(lens[used] >= 1) and lens.max() <= lmax
    if used.sum() >= 2:
        kraft = sum(2.0 ** -int(l) for l in lens[used])
        assert kraft == 1.0                          # optimal codes are complete
    assert _cost(freq, lens) == _brute_force_min_cost(list(freq), lmax)


def _textbook_huffman_lengths(freq):
    """Huffman's algorithm with a heap (depth of each leaf)."""
    items = [(int(f), i, (i,)) for i, f in enumerate(freq) if f > 0]
    if len(items) == 1:
        return {items[0][1]: 1}
    depth = {i: 0 for _, i, _ in items}
    heapq.heapify(items)
    uid = len(freq)
    while len(items) > 1:
        f1, _, s1 = heapq.heappop(items)
        f2, _, s2 = heapq.heappop(items)
        for s in s1 + s2:
            depth[s] += 1
        heapq.heappush(items, (f1 + f2, uid, s1 + s2))
        uid += 1
    return depth


@pytest.mark.parametrize("seed", range(30))
def test_code_lengths_match_textbook_huffman_cost(seed):
    rng = np.random.default_rng(200 + seed)
    freq = rng.integers(0, 1000, 16).astype(np.uint64)
    freq[rng.integers(0, 16)] += 1
    d = _textbook_huffman_lengths(freq)
    if max(d.values()) > 12:
        pytest.skip("unconstrained Huffman exceeds the limit for this draw")
    lens = O.code_lengths(freq, 12)
    assert _cost(freq, lens) == sum(int(freq[s]) * l for s, l in d.items())


def _dp_length_limited_cost(freq, lmax):
    """Optimal cost under a length limit by dynamic programming over
    non-decreasing lengths for symbols sorted by decreasing frequency (an
    optimal code can always be taken monotone); Kraft in units of 2^-lmax."""
    f = sorted((int(x) for x in freq if x > 0), reverse=True)
    n = len(f)
    full = 1 << lmax
    from functools import lru_cache

    @lru_cache(maxsize=None)
    def best(i, minlen, used):
        if i == n:
            return 0 if used <= full else None
        res = None
        for l in range(minlen, lmax + 1):
            u = used + (full >> l)
            # remaining symbols need at least (n-i-1) * 2^-lmax more
            if u + (n - i - 1) > full:
                continue
            r = best(i + 1, l, u)
            if r is not None:
                c = r + f[i] * l
                if res is None or c < res:
                    res = c
        return res
    return best(0, 1, 0)


@pytest.mark.parametrize("case", ["fibonacci", "geometric", "gaussian_exponents"])
def test_code_lengths_limited_vs_dp(case):
    if case == "fibonacci":
        a, b, freq = 1, 1, []
        for _ in range(16):
            freq.append(a)
            a, b = b, a + b
    elif case == "geometric":
        freq = [2 ** i for i in range(16)]
    else:
        w = synth.weights_bf16(256, 1024, 0.02, 0.0, 1.0, seed=9)
        h = O.histogram(w)
        pal = O.palette(h)
        freq = [int(h[e]) for e in pal]
    freq = np.array(freq, dtype=np.uint64)
    lens = O.code_lengths(freq, 12)
    assert lens.max() <= 12
    assert _cost(freq, lens) == _dp_length_limited_cost(freq, 12)


def test_canonical_codes_prefix_free_and_ordered():
    rng = np.random.default_rng(7)
    for _ in range(50):
        freq = rng.integers(0, 500, 16).astype(np.uint64)
        freq[0] += 1
        lens = O.code_lengths(freq, 12)
        codes = O.canonical_codes(lens)
        words = [format(int(c), "0%db" % int(l)) for c, l in zip(codes, lens) if l > 0]
        for a, b in itertools.permutations(words, 2):
            assert not b.startswith(a)
        # canonical: sorted by (length, symbol) the codes are increasing
        order = sorted((int(l), s) for s, l in enumerate(lens) if l > 0)
        vals = [int(codes[s]) << (12 - l) for l, s in order]
        assert vals == sorted(vals) and len(set(vals)) == len(vals)


# ---------------------------------------------------------------- golden encodes

def _weights_from_dyadic():
    e = [120] * 32 + [121] * 16 + [119] * 8 + [122] * 4 + [118] * 2 + [123] + [117]
    return (np.array(e, dtype=np.uint16) << 7).reshape(1, 64)


def _weights_from_uniform16():
    w = np.zeros((1, 128), np.uint16)
    for t in range(64):
        e0 = 100 + (7 * t) % 16
        e1 = 100 + (t % 16) if t < 63 else 130
        sm = ((t & 1) << 7) | (t & 63)
        w[0, t] = ((sm >> 7) << 15) | (e0 << 7) | (sm & 0x7F)
        w[0, 64 + t] = ((sm >> 7) << 15) | (e1 << 7) | (sm & 0x7F)
    return w


def test_golden_dyadic_group(golden_dir):
    g = _golden(golden_dir, "dyadic_group.json")
    w = _weights_from_dyadic()
    enc = O.encode(w)
    assert list(enc.palette) == g["palette"]
    assert list(enc.code_len) == g["code_len"]
    codes = O.canonical_codes(enc.code_len)
    for s, want in g["codes_msb_first"].items():
        s = int(s)
        assert format(int(codes[s]), "0%db" % int(enc.code_len[s])) == want
    assert enc.stream_bits == g["stream_bits"]
    assert [int(x) for x in enc.stream] == [int(x, 16) for x in g["stream_words"]]
    assert list(enc.chunk_off) == g["chunk_off"]
    assert list(enc.raw) == g["raw_groups"]
    assert [int(x) for x in _words_le(enc.pal_plane)] == [int(x, 16) for x in g["pal_plane_words"]]
    assert O.entropy_bits(O.histogram(w)) == pytest.approx(g["entropy_bits"], abs=1e-12)
    assert np.array_equal(O.decode(enc), w)
    assert np.array_equal(O.transcode(enc), enc.pal_plane)


def test_golden_uniform16_with_raw_group(golden_dir):
    g = _golden(golden_dir, "uniform16_raw.json")
    w = _weights_from_uniform16()
    enc = O.encode(w)
    assert list(enc.palette) == g["palette"]
    assert list(enc.code_len) == g["code_len"]
    assert enc.stream_bits == g["stream_bits"]
    assert [int(x) for x in enc.stream] == [int(x, 16) for x in g["stream_words"]]
    assert list(enc.chunk_off) == g["chunk_off"]
    assert list(enc.raw) == g["raw_groups"] and enc.n_raw == g["n_raw"]
    assert list(enc.rawexp[-4:]) == g["raw_plane_last4"]
    words = _words_le(enc.pal_plane)
    assert int(words[0]) == int(g["pal_plane_word0"], 16)
    assert [int(x) for x in words[8:16]] == [int(x, 16) for x in g["pal_plane_group1_words"]]
    assert np.array_equal(enc.sm, np.array([((t & 1) << 7) | (t & 63) for t in range(64)] * 2,
                                           np.uint8))
    assert np.array_equal(O.decode(enc), w)
    assert np.array_equal(O.transcode(enc), enc.pal_plane)


# ---------------------------------------------------------------- stream structure

def _symbols(w, pal):
    e = ((w >> 7) & 0xFF).ravel()
    return np.searchsorted(pal, e)      # palette index of each element (valid where in palette)


@pytest.mark.parametrize("shape,frac", [((8, 1024), 0.002), ((13, 320), 0.0), ((3, 192), 0.05)])
def test_stream_lengths_and_chunk_offsets(shape, frac):
    w = synth.weights_bf16(*shape, 0.02, frac, 1.0, seed=11)
    enc = O.encode(w)
    sym = _symbols(w, enc.palette)
    raw_el = np.repeat(enc.raw.astype(bool), 64)
    lens = enc.code_len.astype(np.int64)[np.where(raw_el, 0, sym)]
    lens[raw_el] = 0
    assert enc.stream_bits == int(lens.sum())
    per_chunk = np.add.reduceat(lens, np.arange(0, lens.size, 256))
    assert np.array_equal(np.diff(enc.chunk_off.astype(np.int64)), per_chunk)
    # the histogram over non-raw groups is what the lengths were built from
    freq = np.bincount(sym[~raw_el], minlength=16)
    assert np.array_equal(enc.code_len, O.code_lengths(freq.astype(np.uint64), 12))


def test_pal_plane_indices_match_palette_positions():
    w = synth.weights_bf16(32, 512, 0.02, 0.002, 1.0, seed=12)
    enc = O.encode(w)
    sym = _symbols(w, enc.palette)
    raw_el = np.repeat(enc.raw.astype(bool), 64)
    for el in range(0, w.size, 37):
        want = 0 if raw_el[el] else int(sym[el])
        assert O.pal_get(enc.pal_plane, el) == want
    assert np.array_equal(O.transcode(enc), enc.pal_plane)


# ---------------------------------------------------------------- round trips

def _all_patterns():
    return np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(1024, 64)


@pytest.mark.parametrize("case", ["all_patterns", "small_cfg", "all_raw", "no_raw",
                                  "one_exponent", "two_exponents", "ragged_chunk",
                                  "specials"])
def test_round_trip(case):
    rng = np.random.default_rng(5)
    if case == "all_patterns":
        w = _all_patterns()
    elif case == "small_cfg":
        w = synth.weights_bf16(128, 1024, 0.02, 0.001, 2.0, seed=0)
    elif case == "all_raw":
        # 64 distinct exponents inside every group -> every group holds one outside the top 16
        e = np.tile(np.arange(60, 124, dtype=np.uint16), 8)
        w = ((e << 7) | rng.integers(0, 128, e.size).astype(np.uint16)).reshape(4, 128)
    elif case == "no_raw":
        w = synth.weights_bf16(16, 256, 0.02, 0.0, 1.0, seed=1) & np.uint16(0xFFFF)
        w = np.where(((w >> 7) & 0xFF) < 110, np.uint16(110 << 7), w).astype(np.uint16)
    elif case == "one_exponent":
        w = ((np.uint16(121) << 7) | rng.integers(0, 256, 8 * 128).astype(np.uint16) & 0x807F)
        w = w.astype(np.uint16).reshape(8, 128)
    elif case == "two_exponents":
        e = rng.choice(np.array([120, 125], np.uint16), 4 * 64, p=[0.9, 0.1])
        w = (e << 7).astype(np.uint16).reshape(4, 64)
    elif case == "ragged_chunk":
        w = synth.weights_bf16(7, 192, 0.02, 0.01, 1.0, seed=2)   # 21 groups: last chunk has 1
    else:
        sp = np.array([0x0000, 0x8000, 0x0001, 0x807F, 0x7F80, 0xFF80, 0x7FC0, 0xFFFF],
                      np.uint16)
        w = np.tile(sp, 16).reshape(2, 64)
    enc = O.encode(w)
    assert np.array_equal(O.decode(enc), w)
    assert np.array_equal(O.transcode(enc), enc.pal_plane)
    if case == "all_raw":
        assert enc.raw.all() and enc.stream_bits == 0
    if case in ("no_raw", "one_exponent", "two_exponents"):
        assert not enc.raw.any()
    if case == "one_exponent":
        assert enc.stream_bits == w.size and int(enc.code_len.max()) == 1


def test_corruption_is_detected():
    w = synth.weights_bf16(16, 512, 0.02, 0.001, 1.0, seed=6)
    enc = O.encode(w)
    bad = O.Encoded(**{**enc.__dict__, "chunk_off": enc.chunk_off.copy()})
    bad.chunk_off[5] += 1
    with pytest.raises(ValueError):
        O.decode(bad)
    bad2 = O.Encoded(**{**enc.__dict__, "stream_bits": enc.stream_bits - 1})
    with pytest.raises(ValueError):
        O.decode(bad2)
    # a flipped stream bit either breaks a code or changes chunk boundaries
    flips = 0
    for bit in range(3, 400, 17):
        s = enc.stream.copy()
        s[bit // 32] ^= np.uint32(1 << (31 - bit % 32))
        b = O.Encoded(**{**enc.__dict__, "stream": s})
        try:
            out = O.decode(b)
            flips += int(not np.array_equal(out, w))
        except ValueError:
            flips += 1
    assert flips > 0


# ---------------------------------------------------------------- statistics (page §三)

def test_exponent_statistics_match_page():
    w = synth.small_matrix(seed=0)
    h = O.histogram(w)
    H = O.entropy_bits(h)
    from scipy.stats import entropy
    assert H == pytest.approx(entropy(h.astype(np.float64), base=2), rel=1e-12)
    pal = O.palette(h)
    coverage = float(h[pal].sum()) / w.size
    # the page: top-16 exponents cover > 99% of a layer; ~2.6 bits of entropy
    assert coverage > 0.99
    assert 2.3 < H < 2.9


# ---------------------------------------------------------------- matmul

@pytest.mark.parametrize("m,n,k", [(1, 5, 64), (3, 7, 128), (5, 2, 320)])
def test_gemm_vs_numpy(m, n, k):
    x = synth.activations_bf16(m, k, seed=1)
    w = synth.weights_bf16(n, k, 0.02, 0.01, 1.0, seed=2)
    y, a = O.gemm(x, w)
    xf = synth.bf16_bits_to_float(x).astype(np.float64)
    wf = synth.bf16_bits_to_float(w).astype(np.float64)
    np.testing.assert_allclose(y, xf @ wf.T, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(a, np.abs(xf) @ np.abs(wf).T, rtol=1e-12)
    ri = np.array([0, m - 1, m // 2]); rj = np.array([n - 1, 0, n // 2])
    ys, as_ = O.gemm_sampled(x, w, ri, rj)
    assert np.array_equal(ys, y[ri, rj]) and np.array_equal(as_, a[ri, rj])
