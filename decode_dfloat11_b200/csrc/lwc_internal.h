// Internal declarations shared by the host encoder (lwc_host.cpp) and the
// device decoders (lwc_df11.cu, lwc_codebook.cu). Not part of the C ABI.
#pragma once

#include <cstdint>
#include <cstddef>

#include "lwc.h"

namespace lwc {

// Blob container constants (header layout: see the field comments of lwc_desc).
constexpr uint32_t kMagic = 0x3143574Cu;
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 256;
constexpr uint32_t kSectionAlign = 256;
constexpr uint32_t kFlagSingleExponent = 1u;
constexpr uint32_t kFormatMaxLen = 32;      // longest Huffman code the format allows
constexpr uint32_t kMaxTables = 256;        // lookup tables this build stages in shared memory

// Record a message for lwc_last_error() and return `s`.
lwc_status fail(lwc_status s, const char *fmt, ...);
void clear_error();

// Consistency checks of a descriptor (sections inside the blob, sizes
// derived from n and the codec parameters). Return LWC_OK or an error that
// has already been recorded with fail().
lwc_status check_df11_desc(const lwc_desc *d);
lwc_status check_codebook_desc(const lwc_desc *d);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace lwc
