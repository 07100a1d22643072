/*
 * Oracle: per-weight loops of the two lossless BF16 codecs, written as
 * plainly as possible (one bit at a time). TEST INFRASTRUCTURE ONLY: only
 * the tests, the smoke check and the benchmark's CPU-baseline leg load this
 * file. It shares no code with the CUDA library; the two meet only through
 * the blob format.
 *
 * Sources (page title, then section):
 *  - "Koniec z kompromisami! DFloat11 ratuje dokładność modeli AI, czyli
 *    kompresja, na którą czekałem" (gadzety360.pl), section "Przełom:
 *    DFloat11 – bezstratna kompresja z wydajnością GPU": a BF16 weight is
 *    1 sign bit, 8 exponent bits and 7 mantissa bits; only the exponent is
 *    Huffman coded, sign and mantissa stay unchanged, and the decoded model is
 *    bit-for-bit identical to the original.
 *  - "Codebook Lossless Compression: когда 25% памяти значат больше, чем
 *    кажется" (ai-manual.ru), section "Как работает эта магия?": a dictionary
 *    of values plus a list of indices, with the original values substituted
 *    back at inference and no approximation; and "無損 LLM 壓縮減少 10-25% RAM"
 *    (setupai.cc), key points: bit-packed codebook indices into the unique
 *    weights.
 *
 * Bit orders (the pages leave them open; chosen reading):
 *  - Huffman stream: bit j is bit (31 - j % 32) of little-endian u32 word j / 32
 *    (MSB first inside each word).
 *  - Codebook indices: bit j of index i is stream bit i*k + j, and stream bit
 *    b is bit (b % 32) of u32 word b / 32 (LSB first).
 */
#include <stdint.h>
#include <string.h>

/* ---- BF16 split / merge (DFloat11 page, "Przełom: DFloat11": sign | exponent | mantissa) ---- */

void orc_split(const uint16_t *w, uint64_t n, uint8_t *e, uint8_t *s)
{
    for (uint64_t i = 0; i < n; i++) {
        unsigned sign = (w[i] >> 15) & 1u;
        unsigned exponent = (w[i] >> 7) & 0xFFu;
        unsigned mantissa = w[i] & 0x7Fu;
        e[i] = (uint8_t)exponent;
        s[i] = (uint8_t)((sign << 7) | mantissa);
    }
}

void orc_merge(const uint8_t *e, const uint8_t *s, uint64_t n, uint16_t *w)
{
    for (uint64_t i = 0; i < n; i++) {
        unsigned sign = (s[i] >> 7) & 1u;
        unsigned mantissa = s[i] & 0x7Fu;
        w[i] = (uint16_t)((sign << 15) | ((unsigned)e[i] << 7) | mantissa);
    }
}

void orc_histogram(const uint8_t *e, uint64_t n, uint64_t *counts)
{
    memset(counts, 0, 256 * sizeof(uint64_t));
    for (uint64_t i = 0; i < n; i++)
        counts[e[i]]++;
}

/* ---- Huffman bitstream (DFloat11 page, "Przełom: DFloat11": entropy coding of the exponent) ---- */

static void put_bit_msb(uint32_t *words, uint64_t j, unsigned bit)
{
    if (bit)
        words[j >> 5] |= 1u << (31 - (j & 31));
}

static unsigned get_bit_msb(const uint32_t *words, uint64_t j)
{
    return (words[j >> 5] >> (31 - (j & 31))) & 1u;
}

/* Appends the code of every exponent, most significant code bit first.
 * `words` must be zeroed and hold at least ceil(total_bits / 32) words.
 * Returns the number of bits written. */
uint64_t orc_df11_emit(const uint8_t *e, uint64_t n, const uint8_t *len,
                       const uint32_t *code, uint32_t *words)
{
    uint64_t pos = 0;
    for (uint64_t i = 0; i < n; i++) {
        unsigned l = len[e[i]];
        uint32_t c = code[e[i]];
        for (int b = (int)l - 1; b >= 0; b--)
            put_bit_msb(words, pos++, (c >> b) & 1u);
    }
    return pos;
}

/* Canonical Huffman decode, one bit at a time: after reading l bits the
 * accumulated value v is a codeword of length l iff
 * first[l] <= v < first[l] + cnt[l]; its symbol is sorted_syms[base[l] + v - first[l]].
 * Decodes `count` codes starting at stream bit `start_bit`, writes the symbol
 * of code i to sym_out[i] and its length to len_out[i] (either may be NULL).
 * Returns 0, -1 if the stream ends (total_bits) inside a code, or -2 if no
 * codeword of length <= max_len matches. *end_bit receives the bit after the
 * last code. */
int orc_df11_decode_syms(const uint32_t *words, uint64_t total_bits, uint64_t start_bit,
                         uint64_t count, const uint32_t *first, const uint32_t *cnt,
                         const uint32_t *base, const uint8_t *sorted_syms, int max_len,
                         uint8_t *sym_out, uint8_t *len_out, uint64_t *end_bit)
{
    uint64_t pos = start_bit;
    for (uint64_t i = 0; i < count; i++) {
        uint32_t v = 0;
        int found = 0;
        for (int l = 1; l <= max_len; l++) {
            if (pos >= total_bits) {
                *end_bit = pos;
                return -1;
            }
            v = (v << 1) | get_bit_msb(words, pos++);
            if (cnt[l] != 0 && v >= first[l] && v - first[l] < cnt[l]) {
                if (sym_out)
                    sym_out[i] = sorted_syms[base[l] + (v - first[l])];
                if (len_out)
                    len_out[i] = (uint8_t)l;
                found = 1;
                break;
            }
        }
        if (!found) {
            *end_bit = pos;
            return -2;
        }
    }
    *end_bit = pos;
    return 0;
}

/* ---- Codebook: fixed-width indices into the table of unique values ---- */

/* idx[i] occupies stream bits [i*k, i*k + k), least significant bit first.
 * `words` must be zeroed. */
void orc_pack_lsb(const uint32_t *idx, uint64_t n, uint32_t k, uint32_t *words)
{
    for (uint64_t i = 0; i < n; i++) {
        for (uint32_t j = 0; j < k; j++) {
            uint64_t b = i * (uint64_t)k + j;
            if ((idx[i] >> j) & 1u)
                words[b >> 5] |= 1u << (b & 31);
        }
    }
}

/* out[i] = table[index i0 + i] for i in [0, count). Returns 0, or -1 if an
 * index is >= U. */
int orc_cb_decode(const uint32_t *words, uint64_t i0, uint64_t count, uint32_t k,
                  const uint16_t *table, uint32_t U, uint16_t *out)
{
    for (uint64_t i = 0; i < count; i++) {
        uint32_t v = 0;
        for (uint32_t j = 0; j < k; j++) {
            uint64_t b = (i0 + i) * (uint64_t)k + j;
            v |= ((words[b >> 5] >> (b & 31)) & 1u) << j;
        }
        if (v >= U)
            return -1;
        out[i] = table[v];
    }
    return 0;
}
