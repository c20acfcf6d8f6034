/*
 * uw_oracle.h -- declarations of the CPU oracle (test infrastructure only).
 * This header belongs to the oracle alone; the product library neither
 * includes it nor shares any definition with it.  The method and the readings
 * it follows are described at the top of uw_oracle.c.
 */
#ifndef UW_ORACLE_H
#define UW_ORACLE_H
#include <stdint.h>

uint8_t uwo_exponent(uint16_t w);
uint8_t uwo_sign_mantissa(uint16_t w);
uint16_t uwo_join(uint8_t exponent, uint8_t sm);

void uwo_histogram(const uint16_t *w, int64_t count, uint64_t hist[256]);
double uwo_entropy_bits(const uint64_t hist[256]);
int uwo_palette(const uint64_t hist[256], uint8_t palette[16]);
void uwo_raw_groups(const uint16_t *w, int64_t n, int64_t k,
                    const uint8_t *palette, int psize, uint8_t *raw);

int uwo_code_lengths(const uint64_t *freq, int nsym, int lmax, uint8_t *len);
void uwo_canonical_codes(const uint8_t *len, int nsym, uint32_t *code);
int uwo_pal_get(const uint8_t *plane, int64_t elem);

int uwo_encode(const uint16_t *w, int64_t n, int64_t k,
               uint8_t *palette, int *psize, uint8_t *code_len,
               uint8_t *sm, uint8_t *raw, uint8_t *rawexp, int64_t *n_raw,
               uint32_t *stream, int64_t stream_cap_words, uint64_t *stream_bits,
               uint32_t *chunk_off, uint8_t *pal_plane);
int uwo_decode(int64_t n, int64_t k, const uint8_t *palette, int psize,
               const uint8_t *code_len, const uint8_t *sm, const uint8_t *raw,
               const uint8_t *rawexp, const uint32_t *stream, uint64_t stream_bits,
               const uint32_t *chunk_off, uint16_t *w_out);
int uwo_transcode(int64_t n, int64_t k, int psize, const uint8_t *code_len,
                  const uint8_t *raw, const uint32_t *stream, uint64_t stream_bits,
                  const uint32_t *chunk_off, uint8_t *pal_plane);

void uwo_gemm(const uint16_t *x, const uint16_t *w, int64_t m, int64_t n, int64_t k,
              double *y, double *a);
void uwo_gemm_sampled(const uint16_t *x, const uint16_t *w, int64_t k,
                      const int64_t *rows_i, const int64_t *rows_j, int64_t count,
                      double *y, double *a);
#endif
