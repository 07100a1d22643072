// Internal declarations shared by the host encoder (lwc_host.cpp), the
// device decoders (lwc_df11.cu, lwc_codebook.cu) and the device encoder
// (lwc_encode.cu). Not part of the C ABI.
#pragma once

#include <cstdint>
#include <cstddef>
#include <vector>

#include "lwc.h"

namespace lwc {

// Blob container constants (header layout: see the field comments of lwc_desc).
constexpr uint32_t kMagic = 0x3143574Cu;
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 256;
constexpr uint32_t kSectionAlign = 256;
constexpr uint32_t kFlagSingleExponent = 1u;
constexpr uint32_t kFlagChunkCounts = 2u;   // DFloat11: u8 code count per chunk at off_counts
constexpr uint32_t kFormatMaxLen = 32;      // longest Huffman code the format allows
constexpr uint32_t kMaxTables = 256;        // lookup tables the decoders stage in shared memory

// DFloat11 encoder defaults. Blocks of 32 chunks are decoded one per warp
// (no CTA-wide barrier per block); a 36-byte chunk is an odd number of words,
// so the 32 lanes of a warp read their chunks from different banks.
constexpr uint32_t kDefaultChunkBytes = 36;
constexpr uint32_t kDefaultThreadsPerBlock = 32;
constexpr uint32_t kDefaultMaxLen = 32;
constexpr uint32_t kDefaultChunkCounts = 1;

// Record a message for lwc_last_error() and return `s`.
lwc_status fail(lwc_status s, const char *fmt, ...);
void clear_error();

// Consistency checks of a descriptor (sections inside the blob, sizes
// derived from n and the codec parameters). Return LWC_OK or an error that
// has already been recorded with fail().
lwc_status check_df11_desc(const lwc_desc *d);
lwc_status check_codebook_desc(const lwc_desc *d);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
constexpr uint64_t round_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

// Section placement inside a blob: each section at the next multiple of kSectionAlign.
struct BlobLayout {
    uint64_t pos = kHeaderBytes;
    uint64_t place(uint64_t bytes) {
        const uint64_t off = round_up(pos, kSectionAlign);
        pos = off + bytes;
        return off;
    }
    uint64_t total() const { return round_up(pos, 16); }
};

// Everything a DFloat11 blob holds besides the per-weight sections, derived
// from the exponent histogram: the descriptor (all fields but
// max_block_count), code lengths, canonical codewords and lookup tables.
struct Df11Plan {
    lwc_desc d;
    uint32_t len[256];
    uint32_t code[256];
    std::vector<uint16_t> tables;
    bool single;   // one exponent value (or n = 0): no stream
};
lwc_status check_df11_params(uint32_t chunk_bytes, uint32_t threads_per_block, uint32_t max_len);
// lo_bytes: size of the raw low-mantissa section placed after the
// sign|mantissa bytes (FP32 and FP16 elements; 0 for BF16). chunk_counts:
// store the per-chunk code counts when the code bounds every count below 256.
lwc_status plan_dfloat11(const uint64_t counts[256], uint64_t n, uint32_t chunk_bytes, uint32_t threads_per_block,
                         uint32_t max_len, bool chunk_counts, Df11Plan &plan, uint64_t lo_bytes = 0);

// Size of the raw low-mantissa section for n elements of type elem.
uint64_t lo_section_bytes(uint32_t elem, uint64_t n);

// Codebook blob plan from the set of present 16-bit patterns (seen[v] != 0).
struct CbPlan {
    lwc_desc d;
    std::vector<uint16_t> table;   // ascending distinct patterns
    std::vector<uint16_t> rank;    // pattern -> index
};
void plan_codebook(const std::vector<uint8_t> &seen, uint64_t n, CbPlan &plan);

// Codebook descriptor (U, k and the section layout) for U distinct patterns.
void codebook_layout(uint32_t U, uint64_t n, lwc_desc &d);

// Writes the 256-byte blob header for `d`.
void write_header(uint8_t *header, const lwc_desc &d);

}  // namespace lwc
