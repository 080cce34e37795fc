// dfw_rans.cpp -- host encoder of the rANS variant of the exponent coder.
//
// Source: the ~1.5:1 page's abstract (an ANS coder feeding the compute
// engine) and the LazyWeights write-up (Huffman against rANS for weight
// streams).  The pages fix no format; this library's (include/dfw.h, "rANS
// VARIANT"): 32-bit states in [2^16, 2^32) renormalised 16 bits at a time,
// frequencies quantised to 2^12, 32 states interleaved per block of 16384
// exponents, blocks coded independently (so threads encode them in
// parallel and a GPU warp decodes one).
#include <algorithm>
#include <cstring>
#include <thread>
#include <vector>

#include "dfw_internal.h"

namespace dfw {
namespace {

constexpr uint32_t RANS_LOW = 1u << 16;  // states live in [RANS_LOW, RANS_LOW << 16)

// Frequencies summing to 2^scale_bits: floor(count * M / n), at least 1 for
// a present exponent; a positive remainder goes to the most frequent
// exponent, a negative one is taken one unit at a time from the exponent
// with the largest frequency above 1 (smallest exponent on ties, both ways).
bool quantise(const uint64_t hist[256], uint64_t n, uint32_t scale_bits, uint16_t freq[256]) {
    const uint64_t M = 1ull << scale_bits;
    std::memset(freq, 0, 256 * sizeof(uint16_t));
    if (n == 0) return true;
    int64_t total = 0;
    int top = -1;
    for (int s = 0; s < 256; ++s) {
        if (!hist[s]) continue;
        const uint64_t q = (uint64_t)(((unsigned __int128)hist[s] * M) / n);
        freq[s] = (uint16_t)std::max<uint64_t>(q, 1);
        total += freq[s];
        if (top < 0 || hist[s] > hist[top]) top = s;
    }
    int64_t diff = (int64_t)M - total;
    if (diff > 0) freq[top] = (uint16_t)(freq[top] + diff);
    while (diff < 0) {
        int pick = -1;
        for (int s = 0; s < 256; ++s)
            if (freq[s] > 1 && (pick < 0 || freq[s] > freq[pick])) pick = s;
        if (pick < 0) return false;
        --freq[pick];
        ++diff;
    }
    return true;
}

// One block: exponents e[0..cnt) into out (lanes states, then words in the
// order a decoder takes them, then zero padding to 16 bytes).  Returns the
// bytes written.  The encoder runs backwards so the decoder runs forwards.
uint64_t encode_block(const uint8_t *e, uint64_t cnt, const uint16_t freq[256], const uint32_t cum[256],
                      uint32_t scale_bits, uint8_t *out, std::vector<uint16_t> &spill) {
    uint32_t state[DFW_RANS_LANES];
    for (uint32_t j = 0; j < DFW_RANS_LANES; ++j) state[j] = RANS_LOW;
    spill.clear();
    const uint64_t bound_unit = (uint64_t)(RANS_LOW >> scale_bits) << 16;
    for (uint64_t i = cnt; i-- > 0;) {
        uint32_t &x = state[i % DFW_RANS_LANES];
        const uint32_t s = e[i], f = freq[s];
        if ((uint64_t)x >= bound_unit * f) {  // make room: emit the low half
            spill.push_back((uint16_t)x);
            x >>= 16;
        }
        x = ((x / f) << scale_bits) + (x % f) + cum[s];
    }
    uint8_t *p = out;
    for (uint32_t j = 0; j < DFW_RANS_LANES; ++j, p += 4) std::memcpy(p, &state[j], 4);  // little-endian host
    for (size_t w = spill.size(); w-- > 0; p += 2) std::memcpy(p, &spill[w], 2);
    const uint64_t used = (uint64_t)(p - out), padded = (used + 15) & ~15ull;
    std::memset(p, 0, padded - used);
    return padded;
}

}  // namespace
}  // namespace dfw

using namespace dfw;

extern "C" uint64_t dfw_rans_stream_bound(uint64_t n) {
    const uint64_t blocks = (n + DFW_RANS_BLOCK - 1) / DFW_RANS_BLOCK;
    return 2 * n + blocks * (4ull * DFW_RANS_LANES + 16);
}

extern "C" dfw_status dfw_rans_encode(const uint16_t *const *tensors, const uint64_t *sizes, int k,
                                      uint8_t *stream, uint64_t stream_capacity, uint8_t *mant,
                                      uint64_t mant_capacity, uint64_t *block_start, dfw_rans_table *table,
                                      int n_threads) {
    dfw::NvtxRange nvtx_range("dfw_rans_encode");
    if (!table || k < 0 || (k && (!tensors || !sizes))) return DFW_EINVAL;
    uint64_t n = 0;
    for (int t = 0; t < k; ++t) {
        if (sizes[t] && !tensors[t]) return DFW_EINVAL;
        n += sizes[t];
    }
    std::memset(table, 0, sizeof(*table));
    table->version = DFW_FORMAT_VERSION;
    table->n = n;
    table->scale_bits = DFW_RANS_SCALE_BITS;
    table->lanes = DFW_RANS_LANES;
    table->block_syms = DFW_RANS_BLOCK;
    table->n_blocks = (n + DFW_RANS_BLOCK - 1) / DFW_RANS_BLOCK;
    if (mant_capacity < dfw_mant_bytes(n) || (n && (!mant || !stream || !block_start))) return DFW_ENOMEM;

    // split: exponents (kept for coding) and raw bytes; histogram
    std::vector<uint8_t> e(n);
    uint64_t hist[256] = {0};
    {
        uint64_t i = 0;
        for (int t = 0; t < k; ++t)
            for (uint64_t j = 0; j < sizes[t]; ++j, ++i) {
                const uint32_t u = tensors[t][j];
                e[i] = (uint8_t)((u >> 7) & 0xFFu);
                mant[i] = (uint8_t)(((u >> 8) & 0x80u) | (u & 0x7Fu));
                ++hist[e[i]];
            }
        std::memset(mant + n, 0, dfw_mant_bytes(n) - n);
    }
    if (!quantise(hist, n, DFW_RANS_SCALE_BITS, table->freq)) return DFW_EINVAL;
    uint32_t cum[256], c = 0;
    for (int s = 0; s < 256; ++s) {
        cum[s] = c;
        c += table->freq[s];
    }
    if (n == 0) return DFW_OK;

    // blocks in parallel into per-thread staging, then concatenated
    const uint64_t nb = table->n_blocks;
    const unsigned hw = std::max(1u, std::thread::hardware_concurrency());
    const unsigned nt = (unsigned)std::min<uint64_t>(nb, n_threads > 0 ? (unsigned)n_threads : hw);
    std::vector<uint64_t> bytes(nb);
    std::vector<std::vector<uint8_t>> part(nt);
    auto work = [&](unsigned t) {
        const uint64_t b0 = nb * t / nt, b1 = nb * (t + 1) / nt;
        std::vector<uint16_t> spill;
        std::vector<uint8_t> &buf = part[t];
        buf.resize((b1 - b0) * (2ull * DFW_RANS_BLOCK + 4ull * DFW_RANS_LANES + 16));
        uint64_t pos = 0;
        for (uint64_t b = b0; b < b1; ++b) {
            const uint64_t i0 = b * DFW_RANS_BLOCK, cnt = std::min<uint64_t>(DFW_RANS_BLOCK, n - i0);
            bytes[b] = encode_block(e.data() + i0, cnt, table->freq, cum, DFW_RANS_SCALE_BITS, buf.data() + pos, spill);
            pos += bytes[b];
        }
        buf.resize(pos);
    };
    std::vector<std::thread> pool;
    for (unsigned t = 1; t < nt; ++t) pool.emplace_back(work, t);
    work(0);
    for (auto &th : pool) th.join();

    uint64_t pos = 0;
    uint32_t mx = 0;
    for (uint64_t b = 0; b < nb; ++b) {
        block_start[b] = pos;
        pos += bytes[b];
        mx = std::max<uint32_t>(mx, (uint32_t)bytes[b]);
    }
    block_start[nb] = pos;
    table->stream_bytes = pos;
    table->max_block_bytes = mx;
    if (stream_capacity < pos) return DFW_ENOMEM;
    uint64_t off = 0;
    for (unsigned t = 0; t < nt; ++t) {
        std::memcpy(stream + off, part[t].data(), part[t].size());
        off += part[t].size();
    }
    return DFW_OK;
}
