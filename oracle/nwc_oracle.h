/*
 * nwc_oracle.h — the test oracle for lossless BF16 weight compression.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product library
 * (libnwc) shares no source with it and never calls it.
 *
 * Plain, single-threaded C++: obvious loops, no blocking, no lookup tables for
 * decoding, FP64 accumulation for the matrix-vector product.  Each function
 * names the page passage it follows:
 *
 *   [DT]  "Efficient ML #1 — Deep Learning Data Types", §3 "Special values"
 *         and §4 "Half the size: FP16 and BF16" (BF16 = 1 sign, 8 exponent
 *         bits with bias 127, 7 fraction bits; worked example 2.5).
 *   [UW]  "Unweight: how we compressed an LLM 22% without sacrificing
 *         quality", section "Compressing BF16 Weights" (Huffman coding of the
 *         exponent byte; sign and mantissa stored unchanged).
 *   [NWC] "NWC — Neural Weight Compression" (neural-weight-compression 0.9.0),
 *         section "How it works": "Byte planes" (split into a raw byte and an
 *         entropy-coded byte), "Prefix code instead of rANS" (12-bit peek),
 *         "Fused kernel" (blocks of 8 rows x 512 columns, one bit stream per
 *         lane, padding for any shape).
 *
 * The formats these functions write and read ("NWB1", the variant "NWR1" of
 * [NWC]'s ranked unary code and the variant "NWE1" of [UW]'s verbatim runs)
 * are stated field by field at the top of nwc_oracle.cpp.  Status codes:
 * 0 = OK, negative = error (see ORC_E_*).
 */
#ifndef NWC_ORACLE_H
#define NWC_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_OK 0
#define ORC_E_ARG (-1)      /* invalid argument                                */
#define ORC_E_SPACE (-2)    /* output buffer too small                         */
#define ORC_E_CORRUPT (-3)  /* blob does not follow the format                 */
#define ORC_E_LMAX (-4)     /* more distinct symbols than 2^lmax codes allow   */

/* [DT] §4: a BF16 word is sign(1) | exponent(8) | fraction(7).
 * s = exponent byte (bits 14..7); r = sign bit << 7 | fraction (bits 6..0). */
void orc_plane_split(uint16_t w, uint8_t* s, uint8_t* r);
uint16_t orc_plane_join(uint8_t s, uint8_t r);

/* Histogram of exponent bytes over the rows x cols real weights. */
int orc_histogram(const uint16_t* w, int64_t rows, int64_t cols, uint64_t cnt[256]);

/* Optimal prefix-code lengths limited to lmax bits (package-merge).  Symbols
 * with cnt == 0 get length 0.  A lone symbol gets length 1. */
int orc_code_lengths(const uint64_t cnt[256], int lmax, uint8_t len[256]);

/* Canonical codes from lengths (codes of equal length are consecutive in
 * symbol order; shorter codes are numerically smaller when left-aligned). */
int orc_canonical_codes(const uint8_t len[256], uint32_t code[256]);

/* Exact blob size for W under the given tile geometry and length limit. */
int orc_blob_size(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                  int tile_cols, int lmax, int64_t* size);

/* Encode W (rows x cols BF16 bit patterns, row-major) into blob[0..cap). */
int orc_encode(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
               int tile_cols, int lmax, uint8_t* blob, int64_t cap, int64_t* size);

/* The same with `streams` (1, 2 or 4) bit streams per lane and tile (format
 * statement, "Streams per lane"); streams = 1 gives the bytes above. */
int orc_blob_size_streams(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                          int tile_cols, int lmax, int streams, int64_t* size);
int orc_encode_streams(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                       int tile_cols, int lmax, int streams, uint8_t* blob, int64_t cap,
                       int64_t* size);

/* Read rows/cols from a blob header (validates the header). */
int orc_blob_info(const uint8_t* blob, int64_t size, int64_t* rows, int64_t* cols);

/* Decode a whole blob into w_out (rows x cols, row-major). */
int orc_decode(const uint8_t* blob, int64_t size, uint16_t* w_out, int64_t cap_elems);

/* Decode only the tiles in [tile_begin, tile_end) (storage order) into
 * w_out (a full rows x cols buffer; other entries are left untouched). */
int orc_decode_tiles(const uint8_t* blob, int64_t size, int64_t tile_begin,
                     int64_t tile_end, uint16_t* w_out, int64_t cap_elems);

/* y[b][n] = sum_k double(W[n][k]) * double(x[b][k]) for n in [row_begin,
 * row_end); x is BF16 [batch x cols]; y is FP64 [batch x rows]. */
int orc_gemv(const uint16_t* w, int64_t rows, int64_t cols, const uint16_t* x,
             int batch, int64_t row_begin, int64_t row_end, double* y);

/* Variant "NWR1" (stated at the top of nwc_oracle.cpp): [NWC] "Prefix code
 * instead of rANS", format v9 — exponent bits 14..8 ranked by frequency in a
 * unary code with the sign as a raw bit and an escape, bits 7..0 raw.  ranks
 * in 1..7.  orc_rank_table gives the ranked values (rank order) and their
 * number. */
int orc_rank_table(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                   int tile_cols, int ranks, uint8_t table[7], int* n);
int orc_rank_blob_size(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                       int tile_cols, int ranks, int64_t* size);
int orc_rank_encode(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                    int tile_cols, int ranks, uint8_t* blob, int64_t cap, int64_t* size);
int orc_rank_decode(const uint8_t* blob, int64_t size, uint16_t* w_out, int64_t cap_elems);

/* Variant "NWE1" (stated at the top of nwc_oracle.cpp): [UW] "Compressing BF16
 * Weights" — the `keep` most common exponent bytes are coded (limit lmax); a
 * run of 64 weights of a row that holds any other exponent keeps its exponent
 * bytes verbatim. */
int orc_escape_blob_size(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                         int tile_cols, int lmax, int keep, int64_t* size);
int orc_escape_encode(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                      int tile_cols, int lmax, int keep, uint8_t* blob, int64_t cap,
                      int64_t* size);
int orc_escape_decode(const uint8_t* blob, int64_t size, uint16_t* w_out, int64_t cap_elems);

#ifdef __cplusplus
}
#endif
#endif
