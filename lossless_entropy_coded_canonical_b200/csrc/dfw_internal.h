// dfw_internal.h -- declarations shared by the host and device halves of libdfw.
#pragma once

#include <cstdint>
#include <vector>

#include "../../include/dfw.h"

namespace dfw {

// LUT entry (32 bits).  Pointer entries: LUT_PTR | child table index.  Leaf
// entries: symbol in bits 0..7, total code length in bits 8..13; in table 0
// also the number of whole codewords inside the 8 key bits (bits 14..17) and
// the bits they use (bits 18..21); a pointer entry in table 0 has count 0.
constexpr uint32_t LUT_PTR = 0x80000000u;
constexpr uint32_t LUT_CHILD_MASK = 0x3FFFu;  // keeps bits 14..21 of pointers zero
constexpr int LUT_LEN_SHIFT = 8;
constexpr int LUT_CNT_SHIFT = 14;
constexpr int LUT_CBITS_SHIFT = 18;

// Bits of the device status word.
constexpr uint32_t ST_COUNT = 1u;   // a tile decoded a different number of codes than out_start says
constexpr uint32_t ST_LUT = 2u;     // a LUT pointer left the table or a code ran past four levels
constexpr uint32_t ST_RANGE = 4u;   // out_start out of order or beyond n, or tile too large

dfw_status code_lengths(const uint64_t hist[256], int cap, uint8_t len[256]);
void canonical_codes(const uint8_t len[256], uint32_t code[256]);
bool kraft_complete(const uint8_t len[256], int cap);
uint64_t stream_bytes_for(uint64_t total_bits);
dfw_status build_lut(const dfw_table *table, std::vector<uint32_t> &lut);
bool plan_shape_supported(uint32_t W, uint32_t T);
dfw_status validate_table(const dfw_table *t);

}  // namespace dfw
