// encode.cpp -- host encoder and blob parsing for libuw.
//
// Implements the offline half of the Unweight page (§三 field split and
// exponent statistics, §四 exponent-only Huffman coding with raw rows for rare
// exponents, §六 the pre-transcoded 4-bit palette form).  The choices the page
// leaves open are fixed as follows, so that every encoding is unique:
//   * group = 64 consecutive weights of one row of W[n,k] (the page's "row of
//     64 weights");
//   * palette = the 16 most frequent exponents (count > 0), ties towards the
//     smaller exponent, stored ascending, index = position;
//   * a group is raw iff it holds an exponent outside the palette; raw groups
//     are coded by neither form, so the Huffman alphabet is the palette index;
//   * code lengths: minimum-redundancy code limited to 12 bits by
//     package-merge (coins ordered by (count, index), coins before packages
//     of equal weight), canonical codewords in (length, index) order, a lone
//     symbol gets the 1-bit code 0;
//   * stream: u32 words, MSB first, chunks of 4 groups with stored start bits.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "uw_format.h"

struct uw_blob {
    std::vector<uint8_t> bytes;
};

namespace uw {

// ---------------------------------------------------------------- CRC-32
namespace {
struct CrcTable {
    uint32_t t[256];
    CrcTable() {
        for (uint32_t i = 0; i < 256; i++) {
            uint32_t c = i;
            for (int j = 0; j < 8; j++) c = (c & 1u) ? (0xEDB88320u ^ (c >> 1)) : (c >> 1);
            t[i] = c;
        }
    }
};
const CrcTable &crc_table() {
    static CrcTable table;
    return table;
}
}  // namespace

uint32_t crc32(const void *data, size_t bytes, uint32_t crc) {
    const uint32_t *t = crc_table().t;
    const uint8_t *p = static_cast<const uint8_t *>(data);
    crc = ~crc;
    for (size_t i = 0; i < bytes; i++) crc = t[(crc ^ p[i]) & 0xFFu] ^ (crc >> 8);
    return ~crc;
}

uint32_t header_crc(const Header &h) {
    Header c = h;
    c.header_crc = 0;
    return crc32(&c, sizeof(Header));
}

// ---------------------------------------------------------------- code lengths
namespace {

struct PMItem {
    uint64_t weight;
    uint8_t mult[16];   // occurrences of each symbol inside the item
};

// Package-merge for a length limit of `lmax` over the symbols with freq > 0.
void package_merge(const uint64_t freq[16], int lmax, uint8_t len[16]) {
    std::memset(len, 0, 16);
    std::vector<PMItem> coins;
    for (int s = 0; s < 16; s++) {
        if (!freq[s]) continue;
        PMItem it{};
        it.weight = freq[s];
        it.mult[s] = 1;
        coins.push_back(it);
    }
    const size_t n = coins.size();
    if (n == 0) return;
    if (n == 1) {
        for (int s = 0; s < 16; s++)
            if (freq[s]) len[s] = 1;
        return;
    }
    auto lighter = [](const PMItem &a, const PMItem &b) { return a.weight < b.weight; };
    std::stable_sort(coins.begin(), coins.end(), lighter);   // ties keep symbol order

    std::vector<PMItem> row = coins, packages, merged;
    for (int level = 1; level < lmax; level++) {
        packages.clear();
        for (size_t i = 0; i + 1 < row.size(); i += 2) {
            PMItem p{};
            p.weight = row[i].weight + row[i + 1].weight;
            for (int s = 0; s < 16; s++) p.mult[s] = uint8_t(row[i].mult[s] + row[i + 1].mult[s]);
            packages.push_back(p);
        }
        merged.resize(coins.size() + packages.size());
        // std::merge takes from the first range on ties: coins before packages
        std::merge(coins.begin(), coins.end(), packages.begin(), packages.end(), merged.begin(),
                   lighter);
        row.swap(merged);
    }
    for (size_t i = 0; i < 2 * n - 2; i++)
        for (int s = 0; s < 16; s++) len[s] = uint8_t(len[s] + row[i].mult[s]);
}

void canonical_codes(const uint8_t len[16], uint32_t code[16]) {
    uint32_t c = 0;
    int prev = 0;
    bool first = true;
    for (int l = 1; l <= kMaxCodeLen; l++)
        for (int s = 0; s < 16; s++) {
            if (len[s] != l) continue;
            c = first ? 0u : (c + 1u) << (l - prev);
            first = false;
            prev = l;
            code[s] = c;
        }
}

void build_dlut(const uint8_t len[16], const uint32_t code[16], uint32_t *lut) {
    // single-code table first: every 12-bit window -> (symbol, length) of its first code
    std::vector<uint8_t> sym1(kLutEntries, 0), len1(kLutEntries, 0);
    for (int s = 0; s < 16; s++) {
        int l = len[s];
        if (!l) continue;
        uint32_t lo = code[s] << (kLutBits - l), hi = (code[s] + 1u) << (kLutBits - l);
        for (uint32_t v = lo; v < hi; v++) {
            sym1[v] = uint8_t(s);
            len1[v] = uint8_t(l);
        }
    }
    for (uint32_t v = 0; v < uint32_t(kLutEntries); v++) {
        uint32_t syms = 0, cnt = 0, pos = 0;
        while (cnt < uint32_t(kLutMaxSyms)) {
            uint32_t rest = (v << pos) & uint32_t(kLutEntries - 1);
            uint32_t l = len1[rest];
            if (!l || pos + l > uint32_t(kLutBits)) break;
            syms |= uint32_t(sym1[rest]) << (4 * cnt);
            cnt++;
            pos += l;
        }
        lut[v] = lut_entry(syms, cnt, pos);
    }
}

// 4-bit palette word for 8 consecutive weights (layout described in uw.h).
inline uint32_t pal_word(const uint8_t idx[8]) {
    uint32_t w = 0;
    for (int j = 0; j < 8; j++) {
        uint32_t v = idx[j];
        w |= (v & 7u) << (4 * j);
        w |= ((v >> 3) & 1u) << (j < 4 ? 8 * j + 7 : 8 * (j - 4) + 3);
    }
    return w;
}

// MSB-first bit packer into u32 words.
struct BitWriter {
    uint32_t *out;
    uint64_t pos = 0;      // bits written
    uint64_t acc = 0;      // pending bits, left-aligned in the low `nacc` bits
    int nacc = 0;
    explicit BitWriter(uint32_t *o) : out(o) {}
    inline void put(uint32_t code, int len) {
        acc = (acc << len) | code;
        nacc += len;
        pos += uint64_t(len);
        if (nacc >= 32) {
            nacc -= 32;
            out[(pos - uint64_t(nacc)) / 32 - 1] = uint32_t(acc >> nacc);
        }
    }
    void flush() {
        if (nacc > 0) out[(pos + 31) / 32 - 1] = uint32_t(acc << (32 - nacc));
        nacc = 0;
    }
};

}  // namespace
}  // namespace uw

using namespace uw;

extern "C" uw_status uw_encode(const uint16_t *w, int64_t n, int64_t k, uint32_t flags,
                               uw_blob **out) {
    if (!w || !out) return UW_ERR_INVALID_ARG;
    *out = nullptr;
    if (n <= 0 || k <= 0) return UW_ERR_INVALID_ARG;
    if (n % 64 || k % 64) return UW_ERR_UNSUPPORTED_SHAPE;
    if (flags == 0) flags = UW_EMIT_HUFFMAN | UW_EMIT_PALETTE;
    if (flags & ~(UW_EMIT_HUFFMAN | UW_EMIT_PALETTE)) return UW_ERR_INVALID_ARG;
    const bool emit_huff = flags & UW_EMIT_HUFFMAN, emit_pal = flags & UW_EMIT_PALETTE;

    try {
        const uint64_t count = uint64_t(n) * uint64_t(k);
        const uint64_t groups = count / kGroup;
        const uint64_t chunks = (groups + kChunkGroups - 1) / kChunkGroups;

        // histogram of exponents
        uint64_t hist[256] = {0};
        for (uint64_t i = 0; i < count; i++) hist[(w[i] >> 7) & 0xFF]++;

        // palette: top 16 by (count desc, exponent asc), stored ascending
        int order[256];
        for (int e = 0; e < 256; e++) order[e] = e;
        std::stable_sort(order, order + 256, [&](int a, int b) { return hist[a] > hist[b]; });
        uint8_t palette[16] = {0};
        int psize = 0;
        for (int i = 0; i < 256 && psize < 16; i++)
            if (hist[order[i]]) palette[psize++] = uint8_t(order[i]);
        std::sort(palette, palette + psize);
        int inv[256];
        for (int e = 0; e < 256; e++) inv[e] = -1;
        for (int i = 0; i < psize; i++) inv[palette[i]] = i;

        double entropy = 0.0, covered = 0.0;
        for (int e = 0; e < 256; e++) {
            if (!hist[e]) continue;
            double p = double(hist[e]) / double(count);
            entropy -= p * std::log2(p);
            if (inv[e] >= 0) covered += double(hist[e]);
        }

        // raw groups and symbol frequencies
        const uint64_t flag_words = (groups + 31) / 32;
        std::vector<uint32_t> flagbits(flag_words, 0);
        uint64_t freq[16] = {0};
        uint64_t n_raw = 0;
        for (uint64_t g = 0; g < groups; g++) {
            const uint16_t *p = w + g * kGroup;
            bool raw = false;
            for (int t = 0; t < kGroup; t++) raw |= inv[(p[t] >> 7) & 0xFF] < 0;
            if (raw) {
                flagbits[g / 32] |= 1u << (g % 32);
                n_raw++;
            } else {
                for (int t = 0; t < kGroup; t++) freq[inv[(p[t] >> 7) & 0xFF]]++;
            }
        }
        uint8_t code_len[16];
        package_merge(freq, kMaxCodeLen, code_len);
        uint32_t code[16] = {0};
        canonical_codes(code_len, code);

        uint64_t stream_bits = 0;
        for (int s = 0; s < 16; s++) stream_bits += freq[s] * code_len[s];
        if (emit_huff && stream_bits > 0xFFFFFFFFull) return UW_ERR_UNSUPPORTED_SHAPE;
        const uint64_t stream_words =
            emit_huff ? align_up((stream_bits + 31) / 32 + kStreamPadWords, 4) : 0;

        // section layout
        Header h{};
        h.magic = kMagic;
        h.version = kVersion;
        h.header_bytes = kHeaderBytes;
        h.flags = flags;
        h.n = n;
        h.k = k;
        h.n_groups = int64_t(groups);
        h.n_raw = int64_t(n_raw);
        h.n_chunks = int64_t(chunks);
        h.stream_bits = emit_huff ? stream_bits : 0;
        h.stream_words = stream_words;
        h.palette_size = psize;
        h.max_code_len = kMaxCodeLen;
        h.chunk_groups = kChunkGroups;
        h.lut_bits = kLutBits;
        std::memcpy(h.palette, palette, 16);
        std::memcpy(h.code_len, code_len, 16);
        h.entropy_bits = entropy;
        h.top16_coverage = covered / double(count);
        const uint64_t sec_bytes[UW_NUM_SECTIONS] = {
            count,                                            // SM
            n_raw * kGroup,                                   // RAWEXP
            align_up(flag_words, 4) * 4,                      // FLAGS
            align_up(flag_words, 4) * 4,                      // RAWBASE
            stream_words * 4,                                 // STREAM
            emit_huff ? align_up(chunks + 1, 4) * 4 : 0,      // CHUNKOFF
            emit_huff ? uint64_t(kLutEntries) * 4 : 0,        // DLUT
            emit_pal ? count / 2 : 0,                         // PAL
        };
        uint64_t off = kHeaderBytes;
        for (int s = 0; s < UW_NUM_SECTIONS; s++) {
            off = align_up(off, kSectionAlign);
            h.sec_off[s] = off;
            h.sec_bytes[s] = sec_bytes[s];
            off += sec_bytes[s];
        }
        h.total_bytes = align_up(off, kSectionAlign);

        uw_blob *blob = new uw_blob;
        blob->bytes.assign(h.total_bytes, 0);
        uint8_t *base = blob->bytes.data();

        // SM plane
        uint8_t *sm = base + h.sec_off[UW_SEC_SM];
        for (uint64_t i = 0; i < count; i++)
            sm[i] = uint8_t(((w[i] >> 8) & 0x80u) | (w[i] & 0x7Fu));

        // raw exponents, flag words, prefix counts
        uint8_t *rawexp = base + h.sec_off[UW_SEC_RAWEXP];
        uint64_t r = 0;
        for (uint64_t g = 0; g < groups; g++) {
            if (!((flagbits[g / 32] >> (g % 32)) & 1u)) continue;
            const uint16_t *p = w + g * kGroup;
            for (int t = 0; t < kGroup; t++) rawexp[r * kGroup + t] = uint8_t((p[t] >> 7) & 0xFF);
            r++;
        }
        uint32_t *fw = reinterpret_cast<uint32_t *>(base + h.sec_off[UW_SEC_FLAGS]);
        uint32_t *rb = reinterpret_cast<uint32_t *>(base + h.sec_off[UW_SEC_RAWBASE]);
        uint32_t running = 0;
        for (uint64_t i = 0; i < flag_words; i++) {
            fw[i] = flagbits[i];
            rb[i] = running;
            running += uint32_t(__builtin_popcount(flagbits[i]));
        }

        // Huffman stream with per-chunk start bits, and the decode table
        if (emit_huff) {
            uint32_t *stream = reinterpret_cast<uint32_t *>(base + h.sec_off[UW_SEC_STREAM]);
            uint32_t *coff = reinterpret_cast<uint32_t *>(base + h.sec_off[UW_SEC_CHUNKOFF]);
            BitWriter bw(stream);
            for (uint64_t c = 0; c < chunks; c++) {
                coff[c] = uint32_t(bw.pos);
                const uint64_t gend = std::min<uint64_t>(groups, (c + 1) * kChunkGroups);
                for (uint64_t g = c * kChunkGroups; g < gend; g++) {
                    if ((flagbits[g / 32] >> (g % 32)) & 1u) continue;
                    const uint16_t *p = w + g * kGroup;
                    for (int t = 0; t < kGroup; t++) {
                        int s = inv[(p[t] >> 7) & 0xFF];
                        bw.put(code[s], code_len[s]);
                    }
                }
            }
            bw.flush();
            coff[chunks] = uint32_t(bw.pos);
            build_dlut(code_len, code,
                       reinterpret_cast<uint32_t *>(base + h.sec_off[UW_SEC_DLUT]));
        }

        // 4-bit palette plane; raw groups stay zero
        if (emit_pal) {
            uint32_t *pal = reinterpret_cast<uint32_t *>(base + h.sec_off[UW_SEC_PAL]);
            for (uint64_t g = 0; g < groups; g++) {
                if ((flagbits[g / 32] >> (g % 32)) & 1u) continue;
                const uint16_t *p = w + g * kGroup;
                for (int q = 0; q < kGroup / 8; q++) {
                    uint8_t idx[8];
                    for (int j = 0; j < 8; j++) idx[j] = uint8_t(inv[(p[8 * q + j] >> 7) & 0xFF]);
                    pal[g * 8 + q] = pal_word(idx);
                }
            }
        }

        h.payload_crc = crc32(base + kHeaderBytes, h.total_bytes - kHeaderBytes);
        h.header_crc = header_crc(h);
        std::memcpy(base, &h, sizeof(Header));
        *out = blob;
        return UW_OK;
    } catch (const std::bad_alloc &) {
        return UW_ERR_NOMEM;
    }
}

extern "C" const void *uw_blob_data(const uw_blob *blob, size_t *bytes) {
    if (!blob) {
        if (bytes) *bytes = 0;
        return nullptr;
    }
    if (bytes) *bytes = blob->bytes.size();
    return blob->bytes.data();
}

extern "C" void uw_blob_free(uw_blob *blob) { delete blob; }

namespace uw {
// Parse and check a host copy of a blob; fills `h`.
uw_status parse_header(const void *host_blob, size_t bytes, int verify_payload, Header &h) {
    if (!host_blob) return UW_ERR_INVALID_ARG;
    if (bytes < kHeaderBytes) return UW_ERR_CORRUPT;
    std::memcpy(&h, host_blob, sizeof(Header));
    if (h.magic != kMagic || h.version != kVersion || h.header_bytes != kHeaderBytes)
        return UW_ERR_CORRUPT;
    if (header_crc(h) != h.header_crc) return UW_ERR_CORRUPT;
    if (h.total_bytes != bytes) return UW_ERR_CORRUPT;
    if (h.n <= 0 || h.k <= 0 || h.n % 64 || h.k % 64) return UW_ERR_CORRUPT;
    const uint64_t count = uint64_t(h.n) * uint64_t(h.k);
    if (uint64_t(h.n_groups) != count / kGroup ||
        uint64_t(h.n_chunks) != (count / kGroup + kChunkGroups - 1) / kChunkGroups)
        return UW_ERR_CORRUPT;
    if (h.palette_size < 1 || h.palette_size > 16 || h.n_raw < 0 || h.n_raw > h.n_groups)
        return UW_ERR_CORRUPT;
    if (h.chunk_groups != uint32_t(kChunkGroups) || h.lut_bits != uint32_t(kLutBits) ||
        h.max_code_len != uint32_t(kMaxCodeLen))
        return UW_ERR_CORRUPT;
    for (int s = 0; s < UW_NUM_SECTIONS; s++) {
        if (h.sec_off[s] % kSectionAlign || h.sec_off[s] < kHeaderBytes) return UW_ERR_CORRUPT;
        if (h.sec_off[s] + h.sec_bytes[s] > h.total_bytes || h.sec_off[s] + h.sec_bytes[s] < h.sec_off[s])
            return UW_ERR_CORRUPT;
    }
    const uint64_t flag_words = (uint64_t(h.n_groups) + 31) / 32;
    if (h.sec_bytes[UW_SEC_SM] != count || h.sec_bytes[UW_SEC_RAWEXP] != uint64_t(h.n_raw) * kGroup ||
        h.sec_bytes[UW_SEC_FLAGS] < flag_words * 4 || h.sec_bytes[UW_SEC_RAWBASE] < flag_words * 4)
        return UW_ERR_CORRUPT;
    if (h.flags & UW_EMIT_HUFFMAN) {
        if (h.sec_bytes[UW_SEC_STREAM] != h.stream_words * 4 ||
            h.stream_words < (h.stream_bits + 31) / 32 + kStreamPadWords ||
            h.sec_bytes[UW_SEC_CHUNKOFF] < (uint64_t(h.n_chunks) + 1) * 4 ||
            h.sec_bytes[UW_SEC_DLUT] != uint64_t(kLutEntries) * 4)
            return UW_ERR_CORRUPT;
        for (int s = 0; s < 16; s++)
            if (h.code_len[s] > kMaxCodeLen) return UW_ERR_CORRUPT;
    }
    if ((h.flags & UW_EMIT_PALETTE) && h.sec_bytes[UW_SEC_PAL] != count / 2) return UW_ERR_CORRUPT;
    if (verify_payload &&
        crc32(static_cast<const uint8_t *>(host_blob) + kHeaderBytes, bytes - kHeaderBytes) !=
            h.payload_crc)
        return UW_ERR_CORRUPT;
    return UW_OK;
}
}  // namespace uw

extern "C" uw_status uw_blob_info_get(const void *host_blob, size_t bytes, int verify_payload,
                                      uw_blob_info *info) {
    if (!info) return UW_ERR_INVALID_ARG;
    Header h;
    uw_status st = parse_header(host_blob, bytes, verify_payload, h);
    if (st != UW_OK) return st;
    std::memset(info, 0, sizeof(*info));
    info->n = h.n;
    info->k = h.k;
    info->flags = h.flags;
    info->palette_size = h.palette_size;
    std::memcpy(info->palette, h.palette, 16);
    std::memcpy(info->code_len, h.code_len, 16);
    info->n_groups = h.n_groups;
    info->n_raw = h.n_raw;
    info->n_chunks = h.n_chunks;
    info->stream_bits = h.stream_bits;
    info->entropy_bits = h.entropy_bits;
    info->top16_coverage = h.top16_coverage;
    info->total_bytes = h.total_bytes;
    const uint64_t common = kHeaderBytes + h.sec_bytes[UW_SEC_SM] + h.sec_bytes[UW_SEC_RAWEXP] +
                            h.sec_bytes[UW_SEC_FLAGS] + h.sec_bytes[UW_SEC_RAWBASE];
    info->huffman_bytes = (h.flags & UW_EMIT_HUFFMAN)
                              ? common + h.sec_bytes[UW_SEC_STREAM] + h.sec_bytes[UW_SEC_CHUNKOFF] +
                                    h.sec_bytes[UW_SEC_DLUT]
                              : 0;
    info->palette_bytes = (h.flags & UW_EMIT_PALETTE) ? common + h.sec_bytes[UW_SEC_PAL] : 0;
    for (int s = 0; s < UW_NUM_SECTIONS; s++) {
        info->section_offset[s] = h.sec_off[s];
        info->section_bytes[s] = h.sec_bytes[s];
    }
    return UW_OK;
}
