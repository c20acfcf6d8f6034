// decode.cu -- Huffman exponent decoding on sm_100a (Unweight page §六:
// pipeline 1 rebuilds full BF16 weights in HBM; pipeline 2 writes only the
// exponent bytes; pipeline 3 transcodes the Huffman stream to 4-bit palette
// indices at run time).
//
// One CTA of 256 threads owns a tile of 256 chunks (1024 groups, 65536
// weights); three CTAs fit on an SM.
//   1. One thread TMA-bulk-copies the 16 KB decode table and the tile's slice
//      of the bitstream into shared memory (a slice larger than the buffer is
//      read from global memory instead).  Meanwhile every thread loads its
//      chunk's bounds and, for BF16 output, the first sign/mantissa vectors
//      it will write, so that their latency hides under the decode.
//   2. Every thread decodes one chunk (4 groups).  Per step it reads the two
//      stream words under its bit position, funnel-shifts the next 32 bits to
//      the top, and makes two table lookups from them (each consumes at most
//      12 bits); a lookup yields up to 5 whole codes and the two shift
//      amounts.  Symbols (palette indices) are appended 4 bits at a time to a
//      word queue that is flushed to shared memory, 8 symbols per word; the
//      chunk's non-raw groups are stored back to back.  A chunk must end
//      exactly where the next one starts and must not touch a window with no
//      valid code, otherwise the corrupt bit is raised.
//   3. The tile is written with coalesced 16-byte accesses: palette words in
//      the stored 4-bit layout (transcode), exponent bytes (exponent decode),
//      or BF16 = palette exponent (or raw-plane exponent) joined with the
//      sign/mantissa byte (decode).
#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kThreads = 256;
constexpr int kTileChunks = kThreads;
constexpr int kTileGroups = kTileChunks * kChunkGroups;   // 1024
constexpr int kSegWords = 6 * 1024;                       // 24 KB staged bitstream (3 bits/weight)
constexpr int kFlagWords = kTileGroups / 32;              // 32
constexpr int kChunkWords = kChunkGroups * kGroup / 8;    // 32 symbol words per chunk
constexpr int kPrefetch = 8;                              // sm vectors in flight per thread
constexpr uint64_t kTimeoutNs = 2000000000ull;

// what the write phase produces
constexpr int kOutBf16 = 0;   // BF16 weights [n*k]
constexpr int kOutPal = 1;    // 4-bit palette plane [n*k/2]
constexpr int kOutExp = 2;    // exponent bytes [n*k]

struct DecodeArgs {
    const uint32_t *stream;
    const uint32_t *chunk_off;
    const uint32_t *dlut;
    const uint32_t *flagbits;
    const uint32_t *rawbase;
    const uint8_t *rawexp;
    const uint8_t *sm;
    uint64_t stream_words;
    uint64_t stream_bits;
    uint64_t code_len;          // code length of palette index s in bits 4s..4s+3
    int64_t n_groups, n_chunks;
    Palette16 pal;              // rotr8 of the palette exponents (BF16 rebuild)
    Palette16 pal_nat;          // the palette exponents themselves
    uint16_t *out_bf16;
    uint32_t *out_pal;
    uint8_t *out_exp;
    uint32_t *out_flags;        // exponent decode: all-raw bitmap (may be null)
    uint32_t *out_rank;         // exponent decode: its rank bases (with out_flags)
    uint32_t *status;
};

struct __align__(16) DecodeSmem {
    uint32_t lut[kLutEntries];
    uint32_t seg[kSegWords];
    uint32_t sym[kTileChunks * kChunkWords];   // per chunk: its non-raw groups' symbols, 8 per word,
                                               // word k of chunk c at c*32 + (k + sym_rot(c)) % 32
    uint32_t flags[kFlagWords];
    uint64_t bar;
    uint32_t seg_word0;
    int use_global;
};

// Rotation of a chunk's symbol words in shared memory: neighbouring threads
// flush word k of their chunks at about the same time, and the rotation puts
// those stores in different banks (2-way at most) while keeping word pairs
// 8-byte aligned.
__device__ __forceinline__ uint32_t sym_rot(uint32_t c) { return (2u * c) & 31u; }

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v));
}

struct SmemWords {            // bitstream words staged in shared memory
    uint32_t base;
    __device__ __forceinline__ uint32_t operator()(uint32_t i) const { return lds32(base + 4u * i); }
};
struct GlobalWords {          // bitstream words read from global memory
    const uint32_t *p;
    __device__ __forceinline__ uint32_t operator()(uint32_t i) const { return __ldg(p + i); }
};

// The 32 stream bits starting at bit p, first bit in the MSB.
template <class Src>
__device__ __forceinline__ uint32_t window32(const Src &src, uint32_t p) {
    const uint32_t wi = p >> 5;
    return __funnelshift_l(src(wi + 1), src(wi), p);
}

__device__ __forceinline__ uint32_t lut_at(uint32_t lut_base, uint32_t top) {
    return lds32(lut_base + ((top >> (32 - kLutBits)) << 2));
}

// Queue of decoded symbols, 4 bits each, oldest lowest; full words go to the
// chunk's 128-byte block in shared memory (at `base`), word k at byte offset
// `off` = 4 * ((k + rot) mod 32).  Holds fewer than 32 bits between appends.
struct SymQueue {
    uint32_t lo = 0, na = 0, base, off;
    // append the `nbits` (<= 20) low bits of `s` (higher bits zero)
    __device__ __forceinline__ void push(uint32_t s, uint32_t nbits) {
        lo |= s << na;
        const uint32_t carry = __funnelshift_l(s, 0u, na);
        na += nbits;
        if (na >= 32) {
            sts32(base + off, lo);
            off = (off + 4u) & 127u;
            lo = carry;
            na -= 32;
        }
    }
    __device__ __forceinline__ void finish() {
        if (na) sts32(base + off, lo);
    }
};

// Decode the `rem4 / 4` symbols of one chunk that starts at bit `p` of `src`
// and must end at bit `end`, storing them in the 128-byte block at shared
// address `blk` rotated by `rot` words.  Returns
// true when the chunk decodes cleanly and ends exactly at `end`.  Every read
// stays within the words under bits [p, end + 32), because no step starts
// past `end`.
template <class Src>
__device__ __forceinline__ bool decode_chunk(const Src src, uint32_t p, uint32_t end, uint32_t rem4,
                                             uint32_t lut_base, uint32_t blk, uint32_t rot, uint64_t code_len) {
    SymQueue q;
    q.base = blk;
    q.off = 4u * rot;
    uint32_t err = 0;
    // two whole table entries per window while at least 10 symbols remain
    while (rem4 >= 40 && p <= end) {
        const uint32_t top = window32(src, p);
        const uint32_t e1 = lut_at(lut_base, top);
        const uint32_t b1 = lut_bits(e1);
        const uint32_t e2 = lut_at(lut_base, top << b1);
        p += b1 + lut_bits(e2);
        err |= e1 | e2;
        const uint32_t n1 = lut_symbits(e1), n2 = lut_symbits(e2);
        q.push(e1 & 0xFFFFFu, n1);
        q.push(e2 & 0xFFFFFu, n2);
        rem4 -= n1 + n2;
    }
    // then whole entries while at least 5 remain
    while (rem4 >= 20 && p <= end) {
        const uint32_t e = lut_at(lut_base, window32(src, p));
        p += lut_bits(e);
        err |= e;
        const uint32_t n = lut_symbits(e);
        q.push(e & 0xFFFFFu, n);
        rem4 -= n;
    }
    // the last <= 4 symbols one code at a time
    while (rem4 > 0 && p <= end) {
        const uint32_t e = lut_at(lut_base, window32(src, p));
        const uint32_t s = e & 15u;
        p += uint32_t(code_len >> (4 * s)) & 15u;
        err |= e;
        q.push(s, 4);
        rem4 -= 4;
    }
    q.finish();
    return rem4 == 0 && p == end && !(err & kLutInvalid);
}

template <int OUT>
__global__ void __launch_bounds__(kThreads, 3) k_huff_decode(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int64_t c_begin = int64_t(blockIdx.x) * kTileChunks;
    const int64_t c_end = min(a.n_chunks, c_begin + kTileChunks);
    const int64_t g_begin = c_begin * kChunkGroups;
    const int64_t g_end = min(a.n_groups, c_end * kChunkGroups);
    const uint32_t b_begin = a.chunk_off[c_begin], b_end = a.chunk_off[c_end];

    if (tid < kFlagWords) {
        const int64_t wi = g_begin / 32 + tid;
        S.flags[tid] = (wi * 32 < g_end) ? a.flagbits[wi] : 0u;
        if (OUT == kOutExp && a.out_flags && wi * 32 < g_end) {
            const int64_t left = g_end - wi * 32;
            a.out_flags[wi] = left >= 32 ? ~0u : (1u << left) - 1u;
            a.out_rank[wi] = uint32_t(wi * 32);
        }
    }
    if (tid == 0) {
        const bool bad = b_end < b_begin || uint64_t(b_end) > a.stream_bits;
        const uint64_t w0 = (b_begin >> 5) & ~3u;
        const uint64_t w1 = (((uint64_t(b_end) + 31u) >> 5) + 2u + 3u) & ~uint64_t(3);
        const bool use_global = bad || w1 - w0 > uint64_t(kSegWords) || w1 > a.stream_words;
        S.seg_word0 = use_global ? 0u : uint32_t(w0);
        S.use_global = use_global;
        if (bad) flag_error(a.status, UW_DEVERR_CORRUPT);
        mbar_init(&S.bar, 1);
        fence_mbar_init();
        const uint32_t seg_bytes = use_global ? 0u : uint32_t(w1 - w0) * 4u;
        mbar_arrive_expect_tx(&S.bar, uint32_t(kLutEntries * 4) + seg_bytes);
        bulk_g2s(S.lut, a.dlut, kLutEntries * 4, &S.bar);
        if (seg_bytes) bulk_g2s(S.seg, a.stream + w0, seg_bytes, &S.bar);
    }

    // chunk bounds and the first sign/mantissa vectors, loaded while the copies fly
    const int64_t c = c_begin + tid;
    const bool has_chunk = c < c_end;
    const uint32_t start = has_chunk ? a.chunk_off[c] : 0u;
    const uint32_t end = has_chunk ? a.chunk_off[c + 1] : 0u;
    uint4 smv[kPrefetch];
    if (OUT == kOutBf16) {
#pragma unroll
        for (int u = 0; u < kPrefetch; u++) {
            const int i = u * kThreads + tid;   // same item numbering as the write phase
            const int64_t g = g_begin + (i >> 2);
            smv[u] = g < g_end ? __ldcs(reinterpret_cast<const uint4 *>(a.sm + g * kGroup + (i & 3) * 16))
                               : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    __syncthreads();
    const bool landed = mbar_wait(&S.bar, 0, kTimeoutNs);
    if (__syncthreads_or(!landed)) {
        if (tid == 0) {
            flag_error(a.status, UW_DEVERR_TIMEOUT);
            mbar_wait(&S.bar, 0, kTimeoutNs);   // let any copy in flight land before exit
        }
        return;
    }

    // ---- 2. one chunk per thread
    if (has_chunk) {
        const int lg0 = tid * kChunkGroups;
        const int64_t left = a.n_groups - (g_begin + lg0);
        const int ng = left < kChunkGroups ? int(left) : kChunkGroups;
        const uint32_t raw4 = (S.flags[lg0 >> 5] >> (lg0 & 31)) & 0xFu;
        const uint32_t nn = uint32_t(ng) - __popc(raw4 & ((1u << ng) - 1u));
        const uint32_t base = S.seg_word0 * 32u;
        bool bad = start < base || end < start || end > b_end || uint64_t(end) > a.stream_bits;
        if (!bad && nn > 0) {
            const uint32_t lut_base = smem_addr(S.lut);
            const uint32_t blk = smem_addr(S.sym) + 4u * uint32_t(tid * kChunkWords);
            const uint32_t rot = sym_rot(uint32_t(tid));
            bad = S.use_global
                      ? !decode_chunk(GlobalWords{a.stream}, start, end, nn * 256u, lut_base, blk, rot, a.code_len)
                      : !decode_chunk(SmemWords{smem_addr(S.seg)}, start - base, end - base, nn * 256u,
                                      lut_base, blk, rot, a.code_len);
        } else if (!bad) {
            bad = start != end;
        }
        if (bad) flag_error(a.status, UW_DEVERR_CORRUPT);
    }
    __syncthreads();

    // ---- 3. write the tile
    // In both layouts below a thread's items are 64 (or 128) groups apart, so
    // the group's position inside its flag word and chunk, and its chunk's
    // rotation, are the same for all of a thread's items.  Group lg's symbols
    // follow the chunk's non-raw groups below it.
    if (OUT == kOutPal) {
        // item = half a group (32 weights, 4 palette words): group it*128 + tid/2
        constexpr int kItems = kTileGroups * 2 / kThreads;
        const int half = tid & 1, lg0 = tid >> 1;
        const uint32_t bit = uint32_t(lg0 & 31), in_chunk = uint32_t(lg0 & 3);
        const uint32_t below = ((1u << bit) - 1u) & ~((1u << (bit & 28u)) - 1u);
        const uint32_t sym0 = smem_addr(S.sym) + 4u * uint32_t((lg0 >> 2) * kChunkWords);
        const uint32_t rot = sym_rot(uint32_t(lg0 >> 2)) + uint32_t(half) * 4u;
        uint4 *out4 = reinterpret_cast<uint4 *>(a.out_pal) + (g_begin + lg0) * 2 + half;
#pragma unroll 4
        for (int it = 0; it < kItems; it++) {
            const int lg = it * (kThreads / 2) + lg0;
            if (g_begin + lg >= g_end) break;
            const uint32_t fw = S.flags[lg >> 5];
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (!((fw >> bit) & 1u)) {
                const uint32_t k = (in_chunk - __popc(fw & below)) * 8u + rot;
                const uint32_t sa = sym0 + uint32_t(it) * (kThreads / 8) * kChunkWords * 4u;
                const uint2 n0 = lds64(sa + 4u * (k & 31u)), n1 = lds64(sa + 4u * ((k + 2u) & 31u));
                v = make_uint4(natural_to_pal(n0.x), natural_to_pal(n0.y), natural_to_pal(n1.x),
                               natural_to_pal(n1.y));
            }
            __stcs(out4 + int64_t(it) * kThreads, v);
        }
    } else if (OUT == kOutExp) {
        // item = a quarter group (16 exponent bytes): group it * 64 + tid/4,
        // numbered as in the BF16 layout below
        constexpr int kItems = kTileGroups * 4 / kThreads;
        constexpr int kGroupsPerStep = kThreads / 4;
        const int q = tid & 3, lg0 = tid >> 2;
        const uint32_t bit = uint32_t(lg0 & 31), in_chunk = uint32_t(lg0 & 3);
        const uint32_t below = ((1u << bit) - 1u) & ~((1u << (bit & 28u)) - 1u);
        const uint32_t sym0 = smem_addr(S.sym) + 4u * uint32_t((lg0 >> 2) * kChunkWords);
        const uint32_t rot = sym_rot(uint32_t(lg0 >> 2)) + uint32_t(q) * 2u;
        const int64_t e0 = (g_begin + lg0) * kGroup + q * 16;   // first byte of the first item
        const int64_t live = g_end - g_begin - lg0;             // items it with it * 64 < live exist
#pragma unroll 4
        for (int it = 0; it < kItems; it++) {
            if (it * kGroupsPerStep >= live) break;
            const int lg = it * kGroupsPerStep + lg0;
            const uint32_t fw = S.flags[lg >> 5];
            uint4 v;
            if ((fw >> bit) & 1u) {
                const int64_t g = g_begin + lg;
                const uint32_t rank = a.rawbase[g >> 5] + __popc(fw & ((1u << bit) - 1u));
                v = __ldcs(reinterpret_cast<const uint4 *>(a.rawexp + uint64_t(rank) * kGroup + q * 16));
            } else {
                const uint32_t k = ((in_chunk - __popc(fw & below)) * 8u + rot) & 31u;
                const uint2 nw = lds64(sym0 + uint32_t(it) * (kGroupsPerStep / 4) * kChunkWords * 4u + 4u * k);
                nat_rot(nw.x, a.pal_nat, v.x, v.y);
                nat_rot(nw.y, a.pal_nat, v.z, v.w);
            }
            __stcs(reinterpret_cast<uint4 *>(a.out_exp + e0 + int64_t(it) * kGroupsPerStep * kGroup), v);
        }
    } else {
        // item = a quarter group (16 weights): group (it0 + u) * 64 + tid/4.
        // The sign/mantissa vector of the item kPrefetch items ahead is
        // requested as soon as an item is written, so kPrefetch loads per
        // thread are always in flight.
        constexpr int kItems = kTileGroups * 4 / kThreads;
        constexpr int kGroupsPerStep = kThreads / 4;
        static_assert(kItems % kPrefetch == 0, "whole batches");
        const int q = tid & 3, lg0 = tid >> 2;
        const uint32_t bit = uint32_t(lg0 & 31), in_chunk = uint32_t(lg0 & 3);
        const uint32_t below = ((1u << bit) - 1u) & ~((1u << (bit & 28u)) - 1u);
        const uint32_t sym0 = smem_addr(S.sym) + 4u * uint32_t((lg0 >> 2) * kChunkWords);
        const uint32_t rot = sym_rot(uint32_t(lg0 >> 2)) + uint32_t(q) * 2u;
        const int64_t e0 = (g_begin + lg0) * kGroup + q * 16;   // first weight of the first item
        const int64_t live = g_end - g_begin - lg0;             // items u with u * 64 < live exist
#pragma unroll 1
        for (int it0 = 0; it0 < kItems; it0 += kPrefetch) {
#pragma unroll
            for (int u = 0; u < kPrefetch; u++) {
                const int it = it0 + u;
                const int lg = it * kGroupsPerStep + lg0;
                if (it * kGroupsPerStep < live) {
                    const uint32_t fw = S.flags[lg >> 5];
                    uint32_t r0, r1, r2, r3;
                    if ((fw >> bit) & 1u) {
                        const int64_t g = g_begin + lg;
                        const uint32_t rank = a.rawbase[g >> 5] + __popc(fw & ((1u << bit) - 1u));
                        const uint4 e = __ldcs(reinterpret_cast<const uint4 *>(a.rawexp + uint64_t(rank) * kGroup + q * 16));
                        r0 = rot4(e.x), r1 = rot4(e.y), r2 = rot4(e.z), r3 = rot4(e.w);
                    } else {
                        const uint32_t k = ((in_chunk - __popc(fw & below)) * 8u + rot) & 31u;
                        const uint2 nw = lds64(sym0 + uint32_t(it) * (kGroupsPerStep / 4) * kChunkWords * 4u + 4u * k);
                        nat_rot(nw.x, a.pal, r0, r1);
                        nat_rot(nw.y, a.pal, r2, r3);
                    }
                    uint4 *o = reinterpret_cast<uint4 *>(a.out_bf16 + e0 + int64_t(it) * kGroupsPerStep * kGroup);
                    __stcs(o, join8(r0, r1, smv[u].x, smv[u].y));
                    __stcs(o + 1, join8(r2, r3, smv[u].z, smv[u].w));
                }
                const int it2 = it + kPrefetch;
                if (it2 < kItems && it2 * kGroupsPerStep < live)
                    smv[u] = __ldcs(reinterpret_cast<const uint4 *>(a.sm + e0 + int64_t(it2) * kGroupsPerStep * kGroup));
            }
        }
    }
}

}  // namespace

namespace {

// The palette exponents as bytes, 4 per word (the lookup table of the
// exponent decode; the BF16 decode uses their rotr8 form, make_palette16).
Palette16 make_palette16_natural(const uint8_t palette[16]) {
    auto word = [&](int i) {
        return uint32_t(palette[i]) | uint32_t(palette[i + 1]) << 8 | uint32_t(palette[i + 2]) << 16 |
               uint32_t(palette[i + 3]) << 24;
    };
    return Palette16{word(0), word(4), word(8), word(12)};
}

DecodeArgs decode_args(const uw_dmat &w) {
    DecodeArgs a{};
    a.stream = w.stream;
    a.stream_words = w.stream_words;
    a.stream_bits = w.stream_bits;
    a.chunk_off = w.chunk_off;
    a.dlut = w.dlut;
    a.flagbits = w.flagbits;
    a.rawbase = w.rawbase;
    a.rawexp = w.rawexp;
    a.sm = w.sm;
    a.code_len = 0;
    for (int i = 0; i < 16; i++) a.code_len |= uint64_t(w.code_len[i] & 15u) << (4 * i);
    a.n_groups = w.n_groups;
    a.n_chunks = w.n_chunks;
    a.pal = make_palette16(w.palette);
    a.pal_nat = make_palette16_natural(w.palette);
    a.status = w.dev_status;
    return a;
}

template <int OUT>
cudaError_t launch_mode(const DecodeArgs &a, cudaStream_t stream) {
    const unsigned grid = unsigned((a.n_chunks + kTileChunks - 1) / kTileChunks);
    const size_t smem = sizeof(DecodeSmem);
    static thread_local int ready_dev = -1;   // shared-memory opt-in done on this device
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (ready_dev != dev) {
        err = cudaFuncSetAttribute(k_huff_decode<OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (err != cudaSuccess) return err;
        ready_dev = dev;
    }
    k_huff_decode<OUT><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_huff_decode(const uw_dmat &w, uint16_t *out_bf16, uint8_t *out_pal,
                               cudaStream_t stream) {
    DecodeArgs a = decode_args(w);
    a.out_bf16 = out_bf16;
    a.out_pal = reinterpret_cast<uint32_t *>(out_pal);
    return out_pal ? launch_mode<kOutPal>(a, stream) : launch_mode<kOutBf16>(a, stream);
}

cudaError_t launch_exp_decode(const uw_dmat &w, uint8_t *out_exp, uint32_t *all_raw_flags,
                              uint32_t *all_raw_rank, cudaStream_t stream) {
    DecodeArgs a = decode_args(w);
    a.out_exp = out_exp;
    a.out_flags = all_raw_rank ? all_raw_flags : nullptr;
    a.out_rank = all_raw_rank;
    return launch_mode<kOutExp>(a, stream);
}

}  // namespace uw
