// decode.cu -- Huffman exponent decoding on sm_100a (Unweight page §六:
// pipeline 1 rebuilds full BF16 weights in HBM; pipeline 3 transcodes the
// Huffman stream to 4-bit palette indices at run time).
//
// One CTA owns a tile of 128 chunks (512 groups, 32768 weights).
//   1. One thread TMA-bulk-copies the 16 KB decode table and the tile's slice
//      of the bitstream into shared memory (a slice larger than the buffer is
//      read from global memory instead).
//   2. Every thread decodes one chunk (4 groups).  The next 12 stream bits
//      (kept in a 64-bit register window, refilled one word at a time) index
//      the table, which yields up to 5 whole codes per lookup; the symbols
//      (palette indices) are packed 8 per word into shared memory in natural
//      order.  Raw groups are skipped.  A chunk must end exactly where the
//      next one starts, otherwise the corrupt bit is raised.
//   3. The tile is written with coalesced 16-byte accesses: palette words in
//      the stored 4-bit layout (transcode), or BF16 = palette exponent (or
//      raw-plane exponent) joined with the sign/mantissa byte (decode).
#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kThreads = 128;
constexpr int kTileChunks = kThreads;
constexpr int kTileGroups = kTileChunks * kChunkGroups;   // 512
constexpr int kSegWords = 3 * 1024;                       // 12 KB staged bitstream
constexpr int kFlagWords = kTileGroups / 32;              // 16
constexpr int kSymStride = 34;        // words per thread's chunk in sym[]: 32 + 2 pad (bank spread)
constexpr uint64_t kTimeoutNs = 2000000000ull;

struct DecodeArgs {
    const uint32_t *stream;
    uint64_t stream_words;
    uint64_t stream_bits;
    const uint32_t *chunk_off;
    const uint32_t *dlut;
    const uint32_t *flagbits;
    const uint32_t *rawbase;
    const uint8_t *rawexp;
    const uint8_t *sm;
    int64_t n_groups, n_chunks;
    Palette16 pal;
    uint16_t *out_bf16;
    uint32_t *out_pal;
    uint32_t *status;
};

struct __align__(16) DecodeSmem {
    uint32_t lut[kLutEntries];
    uint32_t seg[kSegWords];
    uint32_t sym[kThreads * kSymStride];   // symbols of the tile's non-raw groups, 8 per word
    uint32_t flags[kFlagWords];
    uint64_t bar;
    uint32_t seg_word0;
    int use_global;
};

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

struct SmemWords {            // bitstream words staged in shared memory
    uint32_t base;
    __device__ __forceinline__ uint32_t operator()(uint32_t i) const { return lds32(base + 4u * i); }
};
struct GlobalWords {          // bitstream words read from global memory
    const uint32_t *p;
    __device__ __forceinline__ uint32_t operator()(uint32_t i) const { return __ldg(p + i); }
};

// word w of local group g lives at sym[(g / 4) * kSymStride + (g % 4) * 8 + w]
__device__ __forceinline__ uint32_t sym_index(uint32_t g, uint32_t w) {
    return (g >> 2) * kSymStride + (g & 3u) * 8 + w;
}

__device__ __forceinline__ void put_symbols(uint32_t sym_base, uint32_t group0, uint32_t dest,
                                            uint32_t flushed, uint32_t word) {
    const uint32_t g = group0 + ((dest >> (2 * (flushed >> 3))) & 3u);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(sym_base + 4u * sym_index(g, flushed & 7u)), "r"(word));
}

// Decode `nsym` symbols of one chunk starting at bit `p` of `src` (words
// 0..last are readable) into sym[] (shared address `sym_base`, one word per 8
// symbols).  `dest` packs the local indices (2 bits each) of the chunk's
// non-raw groups in order.  Returns the bit position after the last symbol,
// or 0xFFFFFFFF on a window that holds no valid code.
template <class Src>
__device__ __forceinline__ uint32_t decode_chunk(const Src src, uint32_t last, uint32_t p, uint32_t nsym,
                                                 uint32_t dest, uint32_t group0, uint32_t lut_base,
                                                 uint32_t sym_base) {
    const uint32_t wi = p >> 5;
    uint64_t buf = (uint64_t(src(min(wi, last))) << 32) | src(min(wi + 1, last));
    buf <<= (p & 31u);
    uint32_t nb = 64u - (p & 31u);       // valid bits in buf, left-aligned
    uint32_t next = wi + 2;
    uint32_t used = 0;                   // bits consumed
    uint64_t acc = 0;                    // pending symbols, 4 bits each, oldest lowest
    uint32_t na = 0, flushed = 0;
    // whole table entries while at least 5 symbols remain (an entry holds <= 5)
    while (nsym >= 5) {
        const uint32_t e = lds32(lut_base + 4u * uint32_t(buf >> (64 - kLutBits)));
        const uint32_t cnt = (e >> 20) & 7u;
        if (cnt == 0) return 0xFFFFFFFFu;
        const uint32_t bits = (e >> 23) & 15u;
        buf <<= bits;
        nb -= bits;
        used += bits;
        if (nb < 32) {
            buf |= uint64_t(src(min(next, last))) << (32 - nb);
            next++;
            nb += 32;
        }
        acc |= uint64_t(e & 0xFFFFFu) << (4 * na);
        na += cnt;
        nsym -= cnt;
        if (na >= 8) {
            put_symbols(sym_base, group0, dest, flushed, uint32_t(acc));
            acc >>= 32;
            na -= 8;
            flushed++;
        }
    }
    // the last <= 4 symbols one code at a time
    while (nsym > 0) {
        const uint32_t e = lds32(lut_base + 4u * uint32_t(buf >> (64 - kLutBits)));
        if (((e >> 20) & 7u) == 0) return 0xFFFFFFFFu;
        const uint32_t bits = e >> 27;
        buf <<= bits;
        nb -= bits;
        used += bits;
        if (nb < 32) {
            buf |= uint64_t(src(min(next, last))) << (32 - nb);
            next++;
            nb += 32;
        }
        acc |= uint64_t(e & 0xFu) << (4 * na);
        na++;
        nsym--;
        if (na >= 8) {
            put_symbols(sym_base, group0, dest, flushed, uint32_t(acc));
            acc >>= 32;
            na -= 8;
            flushed++;
        }
    }
    return p + used;
}

template <bool TO_PAL>
__global__ void __launch_bounds__(kThreads) k_huff_decode(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int64_t c_begin = int64_t(blockIdx.x) * kTileChunks;
    const int64_t c_end = min(a.n_chunks, c_begin + kTileChunks);
    const int64_t g_begin = c_begin * kChunkGroups;
    const int64_t g_end = min(a.n_groups, c_end * kChunkGroups);

    if (tid < kFlagWords) {
        const int64_t wi = g_begin / 32 + tid;
        S.flags[tid] = (wi * 32 < g_end) ? a.flagbits[wi] : 0u;
    }
    if (tid == 0) {
        const uint32_t b0 = a.chunk_off[c_begin], b1 = a.chunk_off[c_end];
        const bool bad = b1 < b0 || uint64_t(b1) > a.stream_bits;
        const uint64_t w0 = (b0 >> 5) & ~3u;
        const uint64_t w1 = (((uint64_t(b1) + 31u) >> 5) + 2u + 3u) & ~uint64_t(3);
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
    const int64_t c = c_begin + tid;
    if (c < c_end) {
        const int lg0 = tid * kChunkGroups;
        const int64_t left = a.n_groups - (g_begin + lg0);
        const int ng = left < kChunkGroups ? int(left) : kChunkGroups;
        const uint32_t fl = (S.flags[lg0 >> 5] >> (lg0 & 31)) & 0xFu;
        uint32_t dest = 0, nn = 0;
#pragma unroll
        for (int j = 0; j < kChunkGroups; j++)
            if (j < ng && !((fl >> j) & 1u)) {
                dest |= uint32_t(j) << (2 * nn);
                nn++;
            }
        const uint32_t start = a.chunk_off[c], end = a.chunk_off[c + 1];
        const uint32_t base = S.seg_word0 * 32u;
        bool bad = start < base || end < start;
        if (!bad && nn > 0) {
            const uint32_t lut_base = smem_addr(S.lut), sym_base = smem_addr(S.sym);
            uint32_t pend;
            if (S.use_global)
                pend = decode_chunk(GlobalWords{a.stream}, uint32_t(a.stream_words - 1), start - base,
                                    nn * 64u, dest, uint32_t(lg0), lut_base, sym_base);
            else
                pend = decode_chunk(SmemWords{smem_addr(S.seg)}, uint32_t(kSegWords - 1), start - base,
                                    nn * 64u, dest, uint32_t(lg0), lut_base, sym_base);
            bad = pend != end - base;
        } else if (!bad) {
            bad = start != end;
        }
        if (bad) flag_error(a.status, UW_DEVERR_CORRUPT);
    }
    __syncthreads();

    // ---- 3. write the tile
    if (TO_PAL) {
        uint4 *out4 = reinterpret_cast<uint4 *>(a.out_pal);
#pragma unroll 4
        for (int i = tid; i < kTileGroups * 2; i += kThreads) {
            const int lg = i >> 1;
            const int64_t g = g_begin + lg;
            if (g >= g_end) continue;
            const bool raw = (S.flags[lg >> 5] >> (lg & 31)) & 1u;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (!raw) {
                const uint32_t j = sym_index(uint32_t(lg), uint32_t(i & 1) * 4);
                const uint2 n0 = *reinterpret_cast<const uint2 *>(&S.sym[j]);
                const uint2 n1 = *reinterpret_cast<const uint2 *>(&S.sym[j + 2]);
                v = make_uint4(natural_to_pal(n0.x), natural_to_pal(n0.y), natural_to_pal(n1.x),
                               natural_to_pal(n1.y));
            }
            out4[g * 2 + (i & 1)] = v;
        }
    } else {
        constexpr int kItems = kTileGroups * 4 / kThreads;   // 16 weights per item
        constexpr int kU = 4;
#pragma unroll 1
        for (int it0 = 0; it0 < kItems; it0 += kU) {
            uint4 smv[kU], rv[kU];
            bool live[kU];
#pragma unroll
            for (int u = 0; u < kU; u++) {
                const int i = (it0 + u) * kThreads + tid;
                const int lg = i >> 2, q = i & 3;
                const int64_t g = g_begin + lg;
                live[u] = g < g_end;
                if (!live[u]) continue;
                const int64_t e0 = g * kGroup + q * 16;
                smv[u] = __ldcs(reinterpret_cast<const uint4 *>(a.sm + e0));
                const uint32_t fw = S.flags[lg >> 5];
                if ((fw >> (lg & 31)) & 1u) {
                    const uint32_t rank = a.rawbase[g >> 5] + __popc(fw & ((1u << (lg & 31)) - 1u));
                    const uint4 e = __ldcs(reinterpret_cast<const uint4 *>(a.rawexp + uint64_t(rank) * kGroup + q * 16));
                    rv[u] = make_uint4(rot4(e.x), rot4(e.y), rot4(e.z), rot4(e.w));
                } else {
                    const uint2 nw = *reinterpret_cast<const uint2 *>(&S.sym[sym_index(uint32_t(lg), uint32_t(q) * 2)]);
                    nat_rot(nw.x, a.pal, rv[u].x, rv[u].y);
                    nat_rot(nw.y, a.pal, rv[u].z, rv[u].w);
                }
            }
#pragma unroll
            for (int u = 0; u < kU; u++) {
                if (!live[u]) continue;
                const int i = (it0 + u) * kThreads + tid;
                const int64_t e0 = (g_begin + (i >> 2)) * kGroup + (i & 3) * 16;
                uint4 *o = reinterpret_cast<uint4 *>(a.out_bf16 + e0);
                o[0] = join8(rv[u].x, rv[u].y, smv[u].x, smv[u].y);
                o[1] = join8(rv[u].z, rv[u].w, smv[u].z, smv[u].w);
            }
        }
    }
}

}  // namespace

cudaError_t launch_huff_decode(const uw_dmat &w, uint16_t *out_bf16, uint8_t *out_pal,
                               cudaStream_t stream) {
    DecodeArgs a;
    a.stream = w.stream;
    a.stream_words = w.stream_words;
    a.stream_bits = w.stream_bits;
    a.chunk_off = w.chunk_off;
    a.dlut = w.dlut;
    a.flagbits = w.flagbits;
    a.rawbase = w.rawbase;
    a.rawexp = w.rawexp;
    a.sm = w.sm;
    a.n_groups = w.n_groups;
    a.n_chunks = w.n_chunks;
    a.pal = make_palette16(w.palette);
    a.out_bf16 = out_bf16;
    a.out_pal = reinterpret_cast<uint32_t *>(out_pal);
    a.status = w.dev_status;
    const unsigned grid = unsigned((w.n_chunks + kTileChunks - 1) / kTileChunks);
    const size_t smem = sizeof(DecodeSmem);
    static thread_local int ready_dev[2] = {-1, -1};   // shared-memory opt-in done on device
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    const int which = out_pal ? 1 : 0;
    if (ready_dev[which] != dev) {
        err = out_pal ? cudaFuncSetAttribute(k_huff_decode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem))
                      : cudaFuncSetAttribute(k_huff_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (err != cudaSuccess) return err;
        ready_dev[which] = dev;
    }
    if (out_pal) k_huff_decode<true><<<grid, kThreads, smem, stream>>>(a);
    else k_huff_decode<false><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace uw
