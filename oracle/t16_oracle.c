/*
 * CPU oracle for the T16 trellis decode -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the CPU-baseline leg of the benchmark
 * load this library.  The product path (the CUDA library) never links, includes or
 * calls it, and it shares no code, header or table with that path.
 *
 * What it computes (source: "DeepSeek-V4.1-Flash-1017 · dsx T16" model card,
 * section "How T16 works", items 1 and 2; the bitshift trellis named in its intro):
 *
 *   - A 16x16 tile of weights is coded by a tail-biting bit stream of n = 256*K bits
 *     (K = 2, 3 or 4 bits per weight), stored as 8*K little-endian 32-bit words.
 *     Stream bit j is bit (j mod 32) of word floor(j / 32).           [reading]
 *   - The weight at tile position p (0..255) takes the 16-bit window whose bit i
 *     is stream bit (p*K + i) mod n: consecutive windows shift by K bits.  [reading]
 *   - T16 codebook (item 1): P = (window * 0x3A2F) mod 2^16, t = low byte of P plus
 *     high byte of P, both unsigned, so t lies in 0..510; the centred code is
 *     c = t - 255.                                          [centring: reading]
 *   - Position p sits at row p mod 16 and column floor(p / 16) of its tile:
 *     column-major positions (item 2).  Rows are output channels.      [row=out: reading]
 *   - Tiles of an R x C matrix are stored in row-major tile order: tile (i, j),
 *     covering rows 16i..16i+15 and columns 16j..16j+15, starts at word
 *     (i*(C/16) + j) * 8*K.                                              [reading]
 *
 * Every function here is scalar and reads one bit at a time, so that a reader can
 * check it against the statements above by eye.  Nothing is blocked or vectorised.
 */
#include <stdint.h>
#include <stddef.h>

#define T16_MULTIPLIER 0x3A2Fu

/* Stream bit j of a word array (LSB-first inside each little-endian word). */
static int stream_bit(const uint32_t *words, int64_t j)
{
    return (int)((words[j / 32] >> (j % 32)) & 1u);
}

/* The 16-bit window of position p in a tail-biting stream of n_bits bits. */
uint32_t oracle_window(const uint32_t *words, int64_t n_bits, int K, int64_t p)
{
    uint32_t w = 0;
    for (int i = 0; i < 16; ++i) {
        int64_t j = (p * K + i) % n_bits;
        w |= (uint32_t)stream_bit(words, j) << i;
    }
    return w;
}

/* T16 codebook value t in 0..510 of one 16-bit window. */
int oracle_t16(uint32_t window)
{
    uint32_t product = (window * T16_MULTIPLIER) % 65536u;
    uint32_t low_byte = product % 256u;
    uint32_t high_byte = product / 256u;
    return (int)(low_byte + high_byte);
}

/* Centred code c = t - 255 of one window. */
int oracle_code(uint32_t window)
{
    return oracle_t16(window) - 255;
}

/*
 * Decode a general tail-biting stream of n weights at K bits each (n*K bits, packed
 * into ceil(n*K/32) words) into n centred codes in position order.  A 16x16 tile is
 * the case n = 256.
 */
void oracle_decode_stream(const uint32_t *words, int64_t n, int K, int32_t *codes)
{
    int64_t n_bits = n * K;
    for (int64_t p = 0; p < n; ++p)
        codes[p] = oracle_code(oracle_window(words, n_bits, K, p));
}

/*
 * Decode one 16x16 tile (8*K words) into codes[16][16], row-major in the output
 * (codes[r*16 + q] is row r, column q).
 */
void oracle_decode_tile(const uint32_t *tile_words, int K, int32_t *codes)
{
    int64_t n_bits = 256 * (int64_t)K;
    for (int p = 0; p < 256; ++p) {
        int r = p % 16;   /* column-major: position runs down a column first */
        int q = p / 16;
        codes[r * 16 + q] = oracle_code(oracle_window(tile_words, n_bits, K, p));
    }
}

/*
 * Decode selected rows of a rows x cols matrix (both multiples of 16) into
 * out[n_sel][cols], one output row per entry of row_ids.
 */
int oracle_decode_rows(const uint32_t *bits, int K, int64_t rows, int64_t cols,
                       const int64_t *row_ids, int64_t n_sel, int32_t *out)
{
    if (K < 2 || K > 4 || rows % 16 || cols % 16) return 1;
    int64_t tiles_per_row = cols / 16;
    int64_t words_per_tile = 8 * (int64_t)K;
    int64_t n_bits = 256 * (int64_t)K;
    for (int64_t s = 0; s < n_sel; ++s) {
        int64_t row = row_ids[s];
        if (row < 0 || row >= rows) return 2;
        int64_t i = row / 16, r = row % 16;
        for (int64_t j = 0; j < tiles_per_row; ++j) {
            const uint32_t *tile = bits + (i * tiles_per_row + j) * words_per_tile;
            for (int q = 0; q < 16; ++q) {
                int64_t p = 16 * q + r;
                out[s * cols + j * 16 + q] = oracle_code(oracle_window(tile, n_bits, K, p));
            }
        }
    }
    return 0;
}

/* Decode a whole rows x cols matrix into out[rows][cols]. */
int oracle_decode_matrix(const uint32_t *bits, int K, int64_t rows, int64_t cols, int32_t *out)
{
    if (K < 2 || K > 4 || rows % 16 || cols % 16) return 1;
    int64_t tiles_per_row = cols / 16;
    int64_t words_per_tile = 8 * (int64_t)K;
    int32_t tile_codes[256];
    for (int64_t i = 0; i < rows / 16; ++i)
        for (int64_t j = 0; j < tiles_per_row; ++j) {
            oracle_decode_tile(bits + (i * tiles_per_row + j) * words_per_tile, K, tile_codes);
            for (int r = 0; r < 16; ++r)
                for (int q = 0; q < 16; ++q)
                    out[(i * 16 + r) * cols + j * 16 + q] = tile_codes[r * 16 + q];
        }
    return 0;
}
