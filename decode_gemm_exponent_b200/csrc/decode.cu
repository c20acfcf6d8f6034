// decode.cu -- Huffman exponent decoding on sm_100a (Unweight page §六:
// pipeline 1 rebuilds full BF16 weights in HBM; pipeline 3 transcodes the
// Huffman stream to 4-bit palette indices at run time).
//
// One CTA owns a tile of 128 chunks (512 groups, 32768 weights).
//   1. One thread TMA-bulk-copies the 16 KB decode table and the tile's slice
//      of the bitstream into shared memory (a slice too large for the buffer
//      is read from global memory instead).
//   2. Every thread decodes one chunk (4 groups): a 12-bit window indexes the
//      table, which yields up to 5 symbols per lookup; symbols are packed 8 at
//      a time into 4-bit-palette words in shared memory.  Raw groups are
//      skipped.  The chunk must end exactly where the next chunk starts,
//      otherwise the corrupt bit is raised.
//   3. The tile is written out with coalesced 16-byte accesses: palette words
//      (transcode), or BF16 = palette exponent (or raw-plane exponent) joined
//      with the sign/mantissa byte (decode).
#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kThreads = 128;
constexpr int kTileChunks = kThreads;
constexpr int kTileGroups = kTileChunks * kChunkGroups;   // 512
constexpr int kSegWords = 5 * 1024;                       // 20 KB staged bitstream
constexpr int kFlagWords = kTileGroups / 32;              // 16
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
    uint32_t sym[kTileGroups * 8];     // palette words of the tile's non-raw groups
    uint32_t flags[kFlagWords];
    uint64_t bar;
    uint32_t seg_word0;
    int use_global;
};

// Decode `nsym` symbols of one chunk starting at bit `p` of `src` (words
// src[0..max_word+1] are readable) into palette words in sym[].  `dest` packs
// the local indices (2 bits each) of the non-raw groups, in order.  Returns
// the bit position after the last symbol, or 0xFFFFFFFF on an invalid code.
__device__ __forceinline__ uint32_t decode_chunk(const uint32_t *__restrict__ src, uint32_t max_word,
                                                 uint32_t p, uint32_t nsym, uint32_t dest,
                                                 uint32_t group0, const uint32_t *lut,
                                                 uint32_t *sym) {
    uint64_t acc = 0;      // pending symbols, 4 bits each, oldest lowest
    uint32_t na = 0;       // number of pending symbols
    uint32_t flushed = 0;  // palette words written
    while (nsym > 0) {
        const uint32_t wi = min(p >> 5, max_word);
        const uint32_t win = __funnelshift_l(src[wi + 1], src[wi], p & 31u) >> (32 - kLutBits);
        const uint32_t e = lut[win];
        const uint32_t cnt = (e >> 20) & 7u;
        if (cnt == 0) return 0xFFFFFFFFu;
        const bool whole = cnt <= nsym;
        const uint32_t take = whole ? cnt : 1u;
        const uint32_t bits = whole ? ((e >> 23) & 15u) : (e >> 27);
        const uint32_t syms = whole ? (e & 0xFFFFFu) : (e & 0xFu);
        acc |= uint64_t(syms) << (4 * na);
        na += take;
        nsym -= take;
        p += bits;
        if (na >= 8) {
            const uint32_t g = group0 + ((dest >> (2 * (flushed >> 3))) & 3u);
            sym[g * 8 + (flushed & 7u)] = natural_to_pal(uint32_t(acc));
            acc >>= 32;
            na -= 8;
            flushed++;
        }
    }
    return p;
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
        const int64_t g0 = g_begin + lg0;
        const int64_t left = a.n_groups - g0;
        const int ng = left < kChunkGroups ? int(left) : kChunkGroups;
        const uint32_t fl = (S.flags[lg0 >> 5] >> (lg0 & 31)) & 0xFu;
        uint32_t dest = 0, nn = 0;
        for (int j = 0; j < kChunkGroups; j++)
            if (j < ng && !((fl >> j) & 1u)) {
                dest |= uint32_t(j) << (2 * nn);
                nn++;
            }
        const uint32_t start = a.chunk_off[c], end = a.chunk_off[c + 1];
        const uint32_t base = S.seg_word0 * 32u;
        const uint32_t *src = S.use_global ? a.stream : S.seg;
        const uint32_t max_word = S.use_global ? uint32_t(a.stream_words - 2) : uint32_t(kSegWords - 2);
        bool bad = start < base || end < start;
        if (!bad && nn > 0) {
            const uint32_t pend = decode_chunk(src, max_word, start - base, nn * 64u, dest,
                                               uint32_t(lg0), S.lut, S.sym);
            bad = pend != end - base;
        } else if (!bad) {
            bad = start != end;
        }
        if (bad) flag_error(a.status, UW_DEVERR_CORRUPT);
    }
    __syncthreads();

    // ---- 3. write the tile
    if (TO_PAL) {
        const uint4 *sym4 = reinterpret_cast<const uint4 *>(S.sym);
        uint4 *out4 = reinterpret_cast<uint4 *>(a.out_pal);
#pragma unroll 4
        for (int i = tid; i < kTileGroups * 2; i += kThreads) {
            const int lg = i >> 1;
            const int64_t g = g_begin + lg;
            if (g >= g_end) continue;
            const bool raw = (S.flags[lg >> 5] >> (lg & 31)) & 1u;
            out4[g * 2 + (i & 1)] = raw ? make_uint4(0u, 0u, 0u, 0u) : sym4[i];
        }
    } else {
        constexpr int kItems = kTileGroups * 4 / kThreads;   // 16 weights per item
        constexpr int kU = 4;
#pragma unroll 1
        for (int it0 = 0; it0 < kItems; it0 += kU) {
            uint4 smv[kU], ev[kU];
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
                    ev[u] = __ldcs(reinterpret_cast<const uint4 *>(a.rawexp + uint64_t(rank) * kGroup + q * 16));
                } else {
                    const uint2 pw = *reinterpret_cast<const uint2 *>(&S.sym[lg * 8 + q * 2]);
                    pal_exponents(pw.x, a.pal, ev[u].x, ev[u].y);
                    pal_exponents(pw.y, a.pal, ev[u].z, ev[u].w);
                }
            }
#pragma unroll
            for (int u = 0; u < kU; u++) {
                if (!live[u]) continue;
                const int i = (it0 + u) * kThreads + tid;
                const int64_t e0 = (g_begin + (i >> 2)) * kGroup + (i & 3) * 16;
                uint4 *o = reinterpret_cast<uint4 *>(a.out_bf16 + e0);
                o[0] = join8(ev[u].x, ev[u].y, smv[u].x, smv[u].y);
                o[1] = join8(ev[u].z, ev[u].w, smv[u].z, smv[u].w);
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
    auto pack = [&](int i) {
        return uint32_t(w.palette[i]) | uint32_t(w.palette[i + 1]) << 8 |
               uint32_t(w.palette[i + 2]) << 16 | uint32_t(w.palette[i + 3]) << 24;
    };
    a.pal = Palette16{pack(0), pack(4), pack(8), pack(12)};
    a.out_bf16 = out_bf16;
    a.out_pal = reinterpret_cast<uint32_t *>(out_pal);
    a.status = w.dev_status;
    const unsigned grid = unsigned((w.n_chunks + kTileChunks - 1) / kTileChunks);
    const size_t smem = sizeof(DecodeSmem);
    cudaError_t err;
    if (out_pal) {
        err = cudaFuncSetAttribute(k_huff_decode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   int(smem));
        if (err != cudaSuccess) return err;
        k_huff_decode<true><<<grid, kThreads, smem, stream>>>(a);
    } else {
        err = cudaFuncSetAttribute(k_huff_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   int(smem));
        if (err != cudaSuccess) return err;
        k_huff_decode<false><<<grid, kThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace uw
