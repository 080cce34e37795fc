// dfw_internal.h -- declarations shared by the host and device halves of libdfw.
#pragma once

#include <cstdint>
#include <vector>

#include "../../include/dfw.h"

#include <nvtx3/nvToolsExt.h>

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

// Fast table: 2^K entries of two u32 words.  Word 0: the symbols of up to
// four whole codewords inside the K key bits (first in the low byte, absent
// ones zero).  Word 1: byte 0 = bits those codewords use, byte 1 = 8 * their
// count, bits 16..27 = end mask (bit j-1 set when one of them ends at key
// offset j), bit 31 = escape (first codeword longer than K bits; its bits
// byte is 255 so any bounds test sends it to the slow path).
constexpr int FAST_BITS_DEFAULT = 10;        // windowed plan
constexpr int FAST_BITS_DEFAULT_LANES = 12;  // known-start plan
constexpr int FAST_BITS_MIN = 8;
constexpr int FAST_BITS_MAX = 12;
constexpr int FAST_MAX_SYMS = 4;
constexpr int FAST_C8_SHIFT = 8;
constexpr int FAST_ENDS_SHIFT = 16;
constexpr uint32_t FAST_ESC = 0x80000000u;
constexpr uint32_t FAST_ESC_WORD = FAST_ESC | 255u;

// Known-start chunks: codewords per chunk, chunks per group (one warp).
constexpr uint32_t LANE_SYMS = 64;
constexpr uint32_t GROUP_CHUNKS = 32;

// Tensors one fused decode + matrix-vector launch can serve (a transformer
// block has seven).
constexpr uint32_t GEMV_MAX_TENSORS = DFW_GEMV_MAX_TENSORS;

// Bits of the device status word.
constexpr uint32_t ST_COUNT = 1u;   // a tile decoded a different number of codes than out_start says
constexpr uint32_t ST_LUT = 2u;     // a LUT pointer left the table or a code ran past four levels
constexpr uint32_t ST_RANGE = 4u;   // out_start out of order or beyond n, or tile too large
constexpr uint32_t ST_TIMEOUT = 8u; // a wait for a bulk copy gave up (the kernel returned early)
constexpr uint32_t ST_CHECK = 16u;  // checks build only: an index or range left its buffer (access skipped)

// Sites of the checks build's range checks (the first failing one is kept).
enum CheckSite : uint32_t {
    CK_NONE = 0,
    CK_LANES_STREAM_COPY = 1,   // a group's stream span or chunk bits beyond their buffers or slot
    CK_LANES_MANT_COPY = 2,     // a group's raw bytes beyond their buffer
    CK_LANES_READ_END = 3,      // a lane's stream reads ran past its warp's shared area
    CK_LANES_SLOT_END = 4,      // a lane's exponent slots ran past their rows
    CK_LANES_STORE = 5,         // an output store beyond n
    CK_LANES_TABLE_COPY = 6,    // a fast table larger than its shared area
    CK_FILL_READ = 7,           // a one-exponent fill read past the raw bytes
    CK_TILES_COPY = 8,          // a tile's copies beyond their buffers or slots
    CK_TILES_WINDOW = 9,        // a window's words or slots beyond their shared areas
    CK_TILES_STORE = 10,        // a tile's output beyond n
    CK_RANS_COPY = 11,          // a rANS block's copy beyond its buffer or slot
    CK_RANS_READ = 12,          // a rANS reload beyond its block
    CK_RANS_STORE = 13,         // a rANS output beyond n
    CK_ENC_SPLIT = 14,          // encoder pass 1 beyond its buffers
    CK_ENC_PACK_BUF = 15,       // encoder packing beyond its shared word buffer
    CK_ENC_PACK_STREAM = 16,    // encoder packing beyond the stream
    CK_CLOSED_READ = 17,        // a closed-form decode read past the stream
};

// A named range on profiler timelines (NVTX) for the duration of a call;
// costs a function-pointer check when no tool is attached.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

dfw_status code_lengths(const uint64_t hist[256], int cap, uint8_t len[256]);
void canonical_codes(const uint8_t len[256], uint32_t code[256]);
bool kraft_complete(const uint8_t len[256], int cap);
uint64_t stream_bytes_for(uint64_t total_bits);
dfw_status build_lut(const dfw_table *table, std::vector<uint32_t> &lut);
dfw_status build_fast(const std::vector<uint32_t> &lut, int fast_bits, std::vector<uint32_t> &fast);
bool plan_shape_supported(uint32_t W, uint32_t T);
dfw_status validate_table(const dfw_table *t);
uint32_t group_span_bytes(uint64_t start_bit, uint64_t end_bit);

}  // namespace dfw
