// uw_format.h -- serialized blob layout (version 2) and helpers shared by the
// host encoder and the C-ABI.  Little-endian throughout.
//
// A blob is a 512-byte header followed by the sections listed in uw.h
// (UW_SEC_*), each starting on a 256-byte boundary so that TMA and 128-bit
// vector loads can address them directly once the blob is copied to a
// 256-byte-aligned device buffer.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/uw.h"

namespace uw {

constexpr uint32_t kMagic = 0x31425755u;     // "UWB1"
constexpr uint32_t kVersion = 2;
constexpr int kChunkGroups = 4;              // groups (of 64 weights) per stream chunk
constexpr int kGroup = 64;                   // weights per group ("row of 64 weights")
constexpr int kMaxCodeLen = 12;              // code-length limit == decode window bits
constexpr int kLutBits = 12;
constexpr int kLutEntries = 1 << kLutBits;
constexpr int kLutMaxSyms = 5;               // symbols packed in one table entry
constexpr uint64_t kSectionAlign = 256;
constexpr uint64_t kStreamPadWords = 8;      // zero words after the last stream word

struct Header {
    uint32_t magic;
    uint32_t version;
    uint32_t header_bytes;
    uint32_t flags;
    int64_t n, k;
    int64_t n_groups, n_raw, n_chunks;
    uint64_t stream_bits;
    uint64_t stream_words;                   // padded
    int32_t palette_size;
    uint32_t max_code_len;
    uint32_t chunk_groups;
    uint32_t lut_bits;
    uint8_t palette[16];
    uint8_t code_len[16];
    double entropy_bits;
    double top16_coverage;
    uint64_t sec_off[UW_NUM_SECTIONS];
    uint64_t sec_bytes[UW_NUM_SECTIONS];
    uint64_t total_bytes;
    uint32_t payload_crc;                    // CRC-32 of bytes [header_bytes, total_bytes)
    uint32_t header_crc;                     // CRC-32 of the header with this field zero
};
constexpr uint32_t kHeaderBytes = 512;
static_assert(sizeof(Header) <= kHeaderBytes, "header too large");

// Decode-table entry (UW_SEC_DLUT), indexed by the next 12 stream bits:
//   bits  0..19  up to 5 decoded symbols (palette indices), 4 bits each, first lowest
//   bits 20..24  4 x the number of whole codes in the window, i.e. the number
//                of symbol bits in 0..19 (0 = no code matches the window)
//   bit  25      set when no code matches the window (corrupt stream or an
//                incomplete one-symbol code)
//   bits 28..31  total stream bits those codes use (12 when none matches, so a
//                decoder that keeps going over a corrupt window still advances)
// The symbol-bit count and the stream-bit count are the two shift amounts a
// decoder needs per lookup, so both are stored ready to use.
#ifdef __CUDACC__
#define UW_HOST_DEVICE __host__ __device__
#else
#define UW_HOST_DEVICE
#endif
constexpr uint32_t kLutInvalid = 1u << 25;
UW_HOST_DEVICE constexpr uint32_t lut_symbits(uint32_t e) { return (e >> 20) & 31u; }
UW_HOST_DEVICE constexpr uint32_t lut_nsym(uint32_t e) { return lut_symbits(e) >> 2; }
UW_HOST_DEVICE constexpr uint32_t lut_bits(uint32_t e) { return e >> 28; }
constexpr uint32_t lut_entry(uint32_t syms, uint32_t nsym, uint32_t bits) {
    return nsym ? syms | (4u * nsym) << 20 | bits << 28 : kLutInvalid | uint32_t(kLutBits) << 28;
}

uint32_t crc32(const void *data, size_t bytes, uint32_t crc = 0);
uint32_t header_crc(const Header &h);

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

}  // namespace uw
