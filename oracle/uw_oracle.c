/*
 * uw_oracle.c -- plain, slow, obviously-correct CPU oracle for lossless BF16
 * exponent compression and the matmul that consumes it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this file.  The product library never
 * links, calls or includes it, and it shares no code, header, table or
 * constant generator with the product.
 *
 * Source of the method ("UW-page" below): the web page
 *   "Unweight：Cloudflare 如何在不损失精度的情况下把大模型压缩 22%"
 * (a Chinese rendering of Cloudflare's Unweight article).  Sections are its
 * numbered headings: 三 (BF16 layout, exponent statistics), 四 (compression
 * strategy: Huffman on the exponent only, MLP only, rare-exponent rows stored
 * raw), 六 (the four execution pipelines, incl. the 4-bit palette), 七
 * (reconstructive matmul).
 *
 * Readings where the page is silent (each is also listed in the design notes):
 *   R1  a "row of 64 weights" is 64 consecutive weights along K inside one row
 *       of W[N,K] (a "group"); K must be a multiple of 64.
 *   R2  palette = the 16 most frequent exponent values of the matrix (count>0),
 *       ties broken towards the smaller exponent; stored ascending; palette
 *       index = position in that ascending list.
 *   R3  one raw-group set serves both formats: Huffman codes only exponents of
 *       non-raw groups, so its alphabet is the <=16 palette indices.
 *   R4  "Huffman" = a minimum-redundancy prefix code, length-limited to 12 bits
 *       with the package-merge algorithm (coins sorted by (count, symbol);
 *       on equal weight a coin precedes a package); canonical codewords
 *       assigned in (length, symbol) order; a single-symbol alphabet gets one
 *       1-bit code "0".
 *   R5  bitstream: codes concatenated in element order, chunk after chunk; the
 *       stream is a little-endian array of u32 words, stream bit b is bit
 *       (31 - b%32) of word b/32.  A chunk is 4 consecutive groups; the start
 *       bit of every chunk is stored (plus a final entry = total bits).
 *   R6  raw groups: all 64 exponent bytes go, in group order, to a raw plane.
 *       The sign/mantissa byte of every weight (raw or not) is kept in one
 *       dense plane: sm = (w >> 8 & 0x80) | (w & 0x7F).
 *   R7  4-bit palette plane: one little-endian u32 word per 8 consecutive
 *       elements (row-major flattening).  For element j (0..7) of the word with
 *       palette index v: bits 4j..4j+2 hold v & 7; bit 3 of v is stored at bit
 *       8j+7 when j < 4 and at bit 8(j-4)+3 when j >= 4.  Raw groups hold 0.
 *
 * Floating point: the matmul accumulates in IEEE double; bf16 -> double is
 * exact.  Build with -O2 -ffp-contract=off (no fast-math).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#include "uw_oracle.h"

/* ------------------------------------------------------------------------ */
/* BF16 field split and rebuild.  UW-page §三: a BF16 number is 1 sign bit,
 * 8 exponent bits and 7 mantissa bits, in that order from the top.         */

uint8_t uwo_exponent(uint16_t w) { return (uint8_t)((w >> 7) & 0xFF); }

uint8_t uwo_sign_mantissa(uint16_t w)
{
    uint8_t sign = (uint8_t)((w >> 15) & 1);
    uint8_t mant = (uint8_t)(w & 0x7F);
    return (uint8_t)((sign << 7) | mant);
}

uint16_t uwo_join(uint8_t exponent, uint8_t sm)
{
    uint16_t sign = (uint16_t)((sm >> 7) & 1);
    uint16_t mant = (uint16_t)(sm & 0x7F);
    return (uint16_t)((sign << 15) | ((uint16_t)exponent << 7) | mant);
}

/* ------------------------------------------------------------------------ */
/* Exponent histogram and its Shannon entropy (UW-page §三: the exponent
 * distribution is highly skewed, ~2.6 bits of information).                */

void uwo_histogram(const uint16_t *w, int64_t count, uint64_t hist[256])
{
    for (int i = 0; i < 256; i++) hist[i] = 0;
    for (int64_t i = 0; i < count; i++) hist[uwo_exponent(w[i])]++;
}

double uwo_entropy_bits(const uint64_t hist[256])
{
    double total = 0.0;
    for (int i = 0; i < 256; i++) total += (double)hist[i];
    if (total == 0.0) return 0.0;
    double h = 0.0;
    for (int i = 0; i < 256; i++) {
        if (hist[i] == 0) continue;
        double p = (double)hist[i] / total;
        h -= p * log2(p);
    }
    return h;
}

/* ------------------------------------------------------------------------ */
/* Palette: UW-page §四 / §六 -- the 16 most common exponents; reading R2.
 * Selection is done the slow way: 16 passes, each taking the not-yet-chosen
 * exponent with the largest count (smallest exponent on a tie).             */

int uwo_palette(const uint64_t hist[256], uint8_t palette[16])
{
    int chosen[256];
    for (int i = 0; i < 256; i++) chosen[i] = 0;
    int size = 0;
    for (int round = 0; round < 16; round++) {
        int best = -1;
        for (int e = 0; e < 256; e++) {
            if (chosen[e] || hist[e] == 0) continue;
            if (best < 0 || hist[e] > hist[best]) best = e;   /* '>' keeps smaller e on ties */
        }
        if (best < 0) break;
        chosen[best] = 1;
        size++;
    }
    int j = 0;
    for (int e = 0; e < 256; e++)
        if (chosen[e]) palette[j++] = (uint8_t)e;       /* ascending order */
    for (; j < 16; j++) palette[j] = 0;
    return size;
}

/* index of exponent e in the palette, or -1 when e is not in it */
static int palette_index(const uint8_t *palette, int psize, uint8_t e)
{
    for (int i = 0; i < psize; i++)
        if (palette[i] == e) return i;
    return -1;
}

/* ------------------------------------------------------------------------ */
/* Raw groups: UW-page §四 -- if any of a row's 64 weights has an exponent
 * outside the top-16 palette, that whole row is stored raw (reading R1).    */

void uwo_raw_groups(const uint16_t *w, int64_t n, int64_t k,
                    const uint8_t *palette, int psize, uint8_t *raw)
{
    int64_t groups_per_row = k / 64;
    for (int64_t r = 0; r < n; r++) {
        for (int64_t g = 0; g < groups_per_row; g++) {
            int is_raw = 0;
            for (int64_t t = 0; t < 64; t++) {
                uint8_t e = uwo_exponent(w[r * k + g * 64 + t]);
                if (palette_index(palette, psize, e) < 0) is_raw = 1;
            }
            raw[r * groups_per_row + g] = (uint8_t)is_raw;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Code lengths: UW-page §四 -- classic Huffman on the exponent byte (short
 * codes for common values, long codes for rare ones).  Reading R4: the
 * minimum-redundancy code under a 12-bit limit, by package-merge.           */

typedef struct {
    uint64_t weight;
    int is_package;
    uint16_t count[16];   /* how many times each symbol occurs inside this item */
} pm_item;

int uwo_code_lengths(const uint64_t *freq, int nsym, int lmax, uint8_t *len)
{
    if (nsym < 0 || nsym > 16 || lmax < 1 || lmax > 16) return -1;
    for (int s = 0; s < nsym; s++) len[s] = 0;

    int used[16], nused = 0;
    for (int s = 0; s < nsym; s++)
        if (freq[s] > 0) used[nused++] = s;
    if (nused == 0) return 0;
    if (nused == 1) { len[used[0]] = 1; return 0; }
    if (nused > (1 << lmax)) return -1;

    /* coins sorted by (weight, symbol): simple insertion sort */
    pm_item coins[16];
    for (int i = 0; i < nused; i++) {
        memset(&coins[i], 0, sizeof(pm_item));
        coins[i].weight = freq[used[i]];
        coins[i].count[used[i]] = 1;
    }
    /* stable insertion sort on weight; 'used' is ascending, so equal weights
       keep ascending symbol order */
    for (int i = 1; i < nused; i++) {
        pm_item key = coins[i];
        int j = i - 1;
        while (j >= 0 && coins[j].weight > key.weight) {
            coins[j + 1] = coins[j];
            j--;
        }
        coins[j + 1] = key;
    }

    /* list at the finest denomination 2^-lmax is the coins themselves */
    /* a list never holds more than 2*16 items (16 coins + <=16 packages) */
    pm_item buf_a[34], buf_b[34], pkgs[17];
    pm_item *list = buf_a, *next = buf_b;
    int nlist = nused;
    for (int i = 0; i < nused; i++) list[i] = coins[i];

    for (int level = 1; level < lmax; level++) {
        /* package adjacent pairs */
        int npk = nlist / 2;
        for (int p = 0; p < npk; p++) {
            memset(&pkgs[p], 0, sizeof(pm_item));
            pkgs[p].weight = list[2 * p].weight + list[2 * p + 1].weight;
            pkgs[p].is_package = 1;
            for (int s = 0; s < 16; s++)
                pkgs[p].count[s] = (uint16_t)(list[2 * p].count[s] + list[2 * p + 1].count[s]);
        }
        /* merge coins and packages by weight; a coin goes first on a tie */
        int ic = 0, ip = 0, nn = 0;
        while (ic < nused || ip < npk) {
            if (ip >= npk || (ic < nused && coins[ic].weight <= pkgs[ip].weight))
                next[nn++] = coins[ic++];
            else
                next[nn++] = pkgs[ip++];
        }
        pm_item *t = list; list = next; next = t;
        nlist = nn;
    }

    /* the first 2n-2 items at denomination 1/2 form the optimal solution */
    int take = 2 * nused - 2;
    for (int i = 0; i < take && i < nlist; i++)
        for (int s = 0; s < 16 && s < nsym; s++)
            len[s] = (uint8_t)(len[s] + list[i].count[s]);
    return 0;
}

/* Canonical codewords (reading R4): symbols in (length, symbol) order get
 * consecutive code values, shifted left whenever the length grows.         */
void uwo_canonical_codes(const uint8_t *len, int nsym, uint32_t *code)
{
    for (int s = 0; s < nsym; s++) code[s] = 0;
    uint32_t next_code = 0;
    int prev_len = 0, first = 1;
    for (int l = 1; l <= 32; l++) {
        for (int s = 0; s < nsym; s++) {
            if (len[s] != l) continue;
            if (first) { next_code = 0; first = 0; }
            else next_code = (next_code + 1) << (l - prev_len);
            code[s] = next_code;
            prev_len = l;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Bit writer / reader for reading R5 (u32 words, MSB of each word first).  */

static void put_bit(uint32_t *stream, uint64_t pos, int bit)
{
    if (bit) stream[pos / 32] |= (uint32_t)1u << (31 - (pos % 32));
}

static int get_bit(const uint32_t *stream, uint64_t pos)
{
    return (int)((stream[pos / 32] >> (31 - (pos % 32))) & 1u);
}

/* Reading R7: position of the 4 index bits of element j of an 8-element word */
static void pal_put(uint8_t *plane, int64_t elem, int index)
{
    int64_t word = elem / 8;
    int j = (int)(elem % 8);
    uint32_t v = (uint32_t)plane[4 * word] | ((uint32_t)plane[4 * word + 1] << 8) |
                 ((uint32_t)plane[4 * word + 2] << 16) | ((uint32_t)plane[4 * word + 3] << 24);
    uint32_t low3 = (uint32_t)(index & 7);
    uint32_t bit3 = (uint32_t)((index >> 3) & 1);
    int hi_pos = (j < 4) ? (8 * j + 7) : (8 * (j - 4) + 3);
    v &= ~((uint32_t)7u << (4 * j));
    v |= low3 << (4 * j);
    v &= ~((uint32_t)1u << hi_pos);
    v |= bit3 << hi_pos;
    plane[4 * word] = (uint8_t)(v & 0xFF);
    plane[4 * word + 1] = (uint8_t)((v >> 8) & 0xFF);
    plane[4 * word + 2] = (uint8_t)((v >> 16) & 0xFF);
    plane[4 * word + 3] = (uint8_t)((v >> 24) & 0xFF);
}

int uwo_pal_get(const uint8_t *plane, int64_t elem)
{
    int64_t word = elem / 8;
    int j = (int)(elem % 8);
    uint32_t v = (uint32_t)plane[4 * word] | ((uint32_t)plane[4 * word + 1] << 8) |
                 ((uint32_t)plane[4 * word + 2] << 16) | ((uint32_t)plane[4 * word + 3] << 24);
    int hi_pos = (j < 4) ? (8 * j + 7) : (8 * (j - 4) + 3);
    return (int)(((v >> (4 * j)) & 7u) | (((v >> hi_pos) & 1u) << 3));
}

/* ------------------------------------------------------------------------ */
/* Encoder: UW-page §三-§四 (split, histogram, palette, raw rows, Huffman on
 * the exponent only) and §六 (the pre-transcoded 4-bit palette form).       */

int uwo_encode(const uint16_t *w, int64_t n, int64_t k,
               uint8_t *palette, int *psize, uint8_t *code_len,
               uint8_t *sm, uint8_t *raw, uint8_t *rawexp, int64_t *n_raw,
               uint32_t *stream, int64_t stream_cap_words, uint64_t *stream_bits,
               uint32_t *chunk_off, uint8_t *pal_plane)
{
    if (n <= 0 || k <= 0 || k % 64 != 0) return -1;
    int64_t count = n * k;
    int64_t groups = count / 64;
    int64_t chunks = (groups + 3) / 4;

    uint64_t hist[256];
    uwo_histogram(w, count, hist);
    *psize = uwo_palette(hist, palette);

    uwo_raw_groups(w, n, k, palette, *psize, raw);

    /* sign/mantissa plane for every weight */
    for (int64_t i = 0; i < count; i++) sm[i] = uwo_sign_mantissa(w[i]);

    /* raw plane: exponents of raw groups in group order */
    int64_t nr = 0;
    for (int64_t g = 0; g < groups; g++) {
        if (!raw[g]) continue;
        for (int t = 0; t < 64; t++) rawexp[nr * 64 + t] = uwo_exponent(w[g * 64 + t]);
        nr++;
    }
    *n_raw = nr;

    /* symbol frequencies over non-raw groups */
    uint64_t freq[16];
    for (int s = 0; s < 16; s++) freq[s] = 0;
    for (int64_t g = 0; g < groups; g++) {
        if (raw[g]) continue;
        for (int t = 0; t < 64; t++)
            freq[palette_index(palette, *psize, uwo_exponent(w[g * 64 + t]))]++;
    }
    if (uwo_code_lengths(freq, 16, 12, code_len) != 0) return -2;
    uint32_t code[16];
    uwo_canonical_codes(code_len, 16, code);

    /* bitstream, chunk by chunk */
    for (int64_t i = 0; i < stream_cap_words; i++) stream[i] = 0;
    uint64_t pos = 0;
    for (int64_t c = 0; c < chunks; c++) {
        chunk_off[c] = (uint32_t)pos;
        for (int64_t g = 4 * c; g < 4 * c + 4 && g < groups; g++) {
            if (raw[g]) continue;
            for (int t = 0; t < 64; t++) {
                int s = palette_index(palette, *psize, uwo_exponent(w[g * 64 + t]));
                int l = code_len[s];
                for (int b = l - 1; b >= 0; b--) {
                    if ((int64_t)(pos / 32) >= stream_cap_words) return -3;
                    put_bit(stream, pos, (int)((code[s] >> b) & 1u));
                    pos++;
                }
            }
        }
    }
    if (pos > 0xFFFFFFFFull) return -4;
    chunk_off[chunks] = (uint32_t)pos;
    *stream_bits = pos;

    /* 4-bit palette plane (reading R7), raw groups left at index 0 */
    for (int64_t i = 0; i < count / 2; i++) pal_plane[i] = 0;
    for (int64_t g = 0; g < groups; g++) {
        if (raw[g]) continue;
        for (int t = 0; t < 64; t++) {
            int64_t e = g * 64 + t;
            pal_put(pal_plane, e, palette_index(palette, *psize, uwo_exponent(w[e])));
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Huffman decoding, one bit at a time (deliberately no lookup table): read
 * bits, and after each bit look for a symbol whose (length, code) matches.
 * Returns the symbol and advances *pos, or -1 if no code of <= 16 bits
 * matches or the stream is exhausted.                                        */
static int decode_symbol(const uint32_t *stream, uint64_t stream_bits, uint64_t *pos,
                         const uint8_t *code_len, const uint32_t *code)
{
    uint32_t value = 0;
    for (int l = 1; l <= 16; l++) {
        if (*pos >= stream_bits) return -1;
        value = (value << 1) | (uint32_t)get_bit(stream, *pos);
        (*pos)++;
        for (int s = 0; s < 16; s++)
            if (code_len[s] == l && code[s] == value) return s;
    }
    return -1;
}

/* Walk the whole stream in element order; every chunk must start exactly at
 * its stored offset and the last must end at stream_bits.  Each decoded
 * symbol is handed to 'emit'.                                                */
typedef void (*emit_fn)(void *ctx, int64_t elem, int symbol);

static int walk_stream(int64_t n, int64_t k, const uint8_t *code_len,
                       const uint8_t *raw, const uint32_t *stream, uint64_t stream_bits,
                       const uint32_t *chunk_off, emit_fn emit, void *ctx)
{
    int64_t groups = n * k / 64;
    int64_t chunks = (groups + 3) / 4;
    uint32_t code[16];
    uwo_canonical_codes(code_len, 16, code);
    uint64_t pos = 0;
    for (int64_t c = 0; c < chunks; c++) {
        if ((uint64_t)chunk_off[c] != pos) return -2;
        for (int64_t g = 4 * c; g < 4 * c + 4 && g < groups; g++) {
            if (raw[g]) continue;
            for (int t = 0; t < 64; t++) {
                int s = decode_symbol(stream, stream_bits, &pos, code_len, code);
                if (s < 0) return -1;
                emit(ctx, g * 64 + t, s);
            }
        }
    }
    if ((uint64_t)chunk_off[chunks] != pos || pos != stream_bits) return -3;
    return 0;
}

typedef struct {
    const uint8_t *palette;
    int psize;
    const uint8_t *sm;
    uint16_t *out;
    int bad;
} decode_ctx;

static void emit_bf16(void *vctx, int64_t elem, int symbol)
{
    decode_ctx *ctx = (decode_ctx *)vctx;
    if (symbol >= ctx->psize) { ctx->bad = 1; return; }
    ctx->out[elem] = uwo_join(ctx->palette[symbol], ctx->sm[elem]);
}

/* Full decode to BF16 (UW-page §六, first pipeline).  Raw groups come back
 * from the raw plane; all others from the Huffman stream.                    */
int uwo_decode(int64_t n, int64_t k, const uint8_t *palette, int psize,
               const uint8_t *code_len, const uint8_t *sm, const uint8_t *raw,
               const uint8_t *rawexp, const uint32_t *stream, uint64_t stream_bits,
               const uint32_t *chunk_off, uint16_t *w_out)
{
    if (n <= 0 || k <= 0 || k % 64 != 0) return -10;
    int64_t groups = n * k / 64;
    int64_t nr = 0;
    for (int64_t g = 0; g < groups; g++) {
        if (!raw[g]) continue;
        for (int t = 0; t < 64; t++)
            w_out[g * 64 + t] = uwo_join(rawexp[nr * 64 + t], sm[g * 64 + t]);
        nr++;
    }
    decode_ctx ctx = { palette, psize, sm, w_out, 0 };
    int rc = walk_stream(n, k, code_len, raw, stream, stream_bits, chunk_off, emit_bf16, &ctx);
    if (rc != 0) return rc;
    return ctx.bad ? -4 : 0;
}

typedef struct { uint8_t *plane; int psize; int bad; } transcode_ctx;

static void emit_pal(void *vctx, int64_t elem, int symbol)
{
    transcode_ctx *ctx = (transcode_ctx *)vctx;
    if (symbol >= ctx->psize) { ctx->bad = 1; return; }
    pal_put(ctx->plane, elem, symbol);
}

/* Runtime palette transcode (UW-page §六, third pipeline): the Huffman
 * alphabet is the palette index, so transcoding is decoding the symbols and
 * writing them as 4-bit indices (reading R7); raw groups stay 0.            */
int uwo_transcode(int64_t n, int64_t k, int psize, const uint8_t *code_len,
                  const uint8_t *raw, const uint32_t *stream, uint64_t stream_bits,
                  const uint32_t *chunk_off, uint8_t *pal_plane)
{
    if (n <= 0 || k <= 0 || k % 64 != 0) return -10;
    for (int64_t i = 0; i < n * k / 2; i++) pal_plane[i] = 0;
    transcode_ctx ctx = { pal_plane, psize, 0 };
    int rc = walk_stream(n, k, code_len, raw, stream, stream_bits, chunk_off, emit_pal, &ctx);
    if (rc != 0) return rc;
    return ctx.bad ? -4 : 0;
}

/* ------------------------------------------------------------------------ */
/* Matmul Y = X * W^T (UW-page §七: the rebuilt weights feed the matmul),
 * accumulated in double, with A = sum |x*w| for the error bound.            */

static double bf16_to_double(uint16_t b)
{
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

void uwo_gemm(const uint16_t *x, const uint16_t *w, int64_t m, int64_t n, int64_t k,
              double *y, double *a)
{
    for (int64_t i = 0; i < m; i++) {
        for (int64_t j = 0; j < n; j++) {
            double s = 0.0, t = 0.0;
            for (int64_t q = 0; q < k; q++) {
                double p = bf16_to_double(x[i * k + q]) * bf16_to_double(w[j * k + q]);
                s += p;
                t += fabs(p);
            }
            y[i * n + j] = s;
            a[i * n + j] = t;
        }
    }
}

/* Same, for a list of (row i of X, row j of W) pairs. */
void uwo_gemm_sampled(const uint16_t *x, const uint16_t *w, int64_t k,
                      const int64_t *rows_i, const int64_t *rows_j, int64_t count,
                      double *y, double *a)
{
    for (int64_t c = 0; c < count; c++) {
        double s = 0.0, t = 0.0;
        for (int64_t q = 0; q < k; q++) {
            double p = bf16_to_double(x[rows_i[c] * k + q]) * bf16_to_double(w[rows_j[c] * k + q]);
            s += p;
            t += fabs(p);
        }
        y[c] = s;
        a[c] = t;
    }
}
