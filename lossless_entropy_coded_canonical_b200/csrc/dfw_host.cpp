// dfw_host.cpp -- host half of libdfw: encoder, planner, LUT builder, errors.
//
// Sources: DFloat11 abstract ("70% Size, 100% Accuracy: Lossless LLM
// Compression for Efficient GPU Inference via Dynamic-Length Float") for
// frequency-based codes of bf16 exponents, compact SRAM lookup tables and
// lightweight auxiliary position arrays; the LazyWeights write-up and the
// Huff-LLM abstract for Huffman as the code.  The exact format is the one
// documented in include/dfw.h.
#include "dfw_internal.h"

#include <algorithm>
#include <cstring>
#include <thread>
#include <vector>

namespace dfw {

// ---------------------------------------------------------------- lengths
//
// Package-merge (Larmore & Hirschberg 1990) in its counting form: each level
// keeps only whether every merged item is a leaf or a package, and the final
// selection of the 2k-2 cheapest items is pushed down level by level
// (selecting q packages at one level selects the first 2q items of the level
// below).  Leaves are ordered by (count, symbol); on equal weight a leaf is
// merged ahead of a package.
dfw_status code_lengths(const uint64_t hist[256], int cap, uint8_t len[256]) {
    std::memset(len, 0, 256);
    if (cap < 1 || cap > DFW_MAX_CAP) return DFW_EINVAL;
    std::vector<int> sym;
    for (int s = 0; s < 256; ++s)
        if (hist[s]) sym.push_back(s);
    const int k = (int)sym.size();
    if (k <= 1) return DFW_OK;
    if (cap < 9 && (1 << cap) < k) return DFW_ECAP;
    std::stable_sort(sym.begin(), sym.end(), [&](int a, int b) { return hist[a] < hist[b]; });
    std::vector<uint64_t> leafw(k);
    for (int i = 0; i < k; ++i) leafw[i] = hist[sym[i]];

    // levels[d][pos] = true if item pos of merged list d is a package
    std::vector<std::vector<uint8_t>> is_pkg(cap);
    std::vector<uint64_t> prev(leafw), cur;
    is_pkg[0].assign(k, 0);
    for (int d = 1; d < cap; ++d) {
        const size_t np = prev.size() / 2;
        cur.clear();
        is_pkg[d].clear();
        size_t i = 0, j = 0;
        while (i < (size_t)k || j < np) {
            const uint64_t pw = j < np ? prev[2 * j] + prev[2 * j + 1] : 0;
            if (j >= np || (i < (size_t)k && leafw[i] <= pw)) {
                cur.push_back(leafw[i++]);
                is_pkg[d].push_back(0);
            } else {
                cur.push_back(pw);
                is_pkg[d].push_back(1);
                ++j;
            }
        }
        prev.swap(cur);
    }
    size_t take = 2 * (size_t)k - 2;
    for (int d = cap - 1; d >= 0; --d) {
        size_t leaf_i = 0, pk = 0;
        for (size_t p = 0; p < take; ++p) {
            if (is_pkg[d][p]) {
                ++pk;
            } else {
                len[sym[leaf_i]]++;
                ++leaf_i;
            }
        }
        take = 2 * pk;
    }
    return DFW_OK;
}

// Canonical codewords: walk symbols in (length, symbol) order; each next
// codeword is the previous plus one, shifted left by the length increase.
void canonical_codes(const uint8_t len[256], uint32_t code[256]) {
    std::vector<std::pair<int, int>> order;
    for (int s = 0; s < 256; ++s) {
        code[s] = 0;
        if (len[s]) order.push_back({len[s], s});
    }
    std::sort(order.begin(), order.end());
    uint64_t c = 0;
    int prev_len = 0;
    for (size_t i = 0; i < order.size(); ++i) {
        const int l = order[i].first;
        if (i == 0) {
            c = 0;
        } else {
            c = (c + 1) << (l - prev_len);
        }
        code[order[i].second] = (uint32_t)c;
        prev_len = l;
    }
}

bool kraft_complete(const uint8_t len[256], int cap) {
    uint64_t sum = 0;
    int k = 0;
    for (int s = 0; s < 256; ++s) {
        if (!len[s]) continue;
        if (len[s] > cap || len[s] > DFW_MAX_CAP) return false;
        sum += 1ull << (32 - len[s]);
        ++k;
    }
    return k >= 2 && sum == (1ull << 32);
}

uint64_t stream_bytes_for(uint64_t total_bits) {
    const uint64_t raw = (total_bits + 7) >> 3;
    return ((raw + 63) & ~63ull) + DFW_STREAM_PAD;
}

// ---------------------------------------------------------------- encoder

namespace {

struct Segments {
    const uint16_t *const *ptr;
    const uint64_t *size;
    int k;
    std::vector<uint64_t> off;  // prefix sums, k + 1
    // Calls f(p, count) for the input words of global range [i0, i1).
    template <class F>
    void for_range(uint64_t i0, uint64_t i1, F &&f) const {
        int s = int(std::upper_bound(off.begin(), off.end(), i0) - off.begin()) - 1;
        while (i0 < i1 && s < k) {
            const uint64_t lo = i0 - off[s];
            const uint64_t hi = std::min(i1, off[s + 1]) - off[s];
            if (hi > lo) f(ptr[s] + lo, hi - lo);
            i0 = off[s] + hi;
            ++s;
        }
    }
};

int resolve_threads(int n_threads, uint64_t n) {
    int t = n_threads > 0 ? n_threads : (int)std::thread::hardware_concurrency();
    if (t < 1) t = 1;
    const uint64_t max_by_size = n / (1u << 16) + 1;  // at least 64Ki weights per thread
    if ((uint64_t)t > max_by_size) t = (int)max_by_size;
    return t;
}

template <class F>
void parallel_for(int nt, F &&f) {
    if (nt == 1) {
        f(0);
        return;
    }
    std::vector<std::thread> th;
    th.reserve(nt);
    for (int t = 0; t < nt; ++t) th.emplace_back([&, t] { f(t); });
    for (auto &x : th) x.join();
}

struct ChunkOut {
    uint64_t hist[256];
    uint64_t bit0, bits;
    uint8_t head, tail;
    bool has_tail;
};

dfw_status encode_segments(Segments &seg, int cap, uint8_t *stream, uint64_t stream_capacity,
                           uint8_t *mant, uint64_t mant_capacity, dfw_table *table, int n_threads) {
    if (!table || cap < 1 || cap > DFW_MAX_CAP) return DFW_EINVAL;
    const uint64_t n = seg.off[seg.k];
    if (n && (!mant || !stream)) return DFW_EINVAL;
    std::memset(table, 0, sizeof(*table));
    table->version = DFW_FORMAT_VERSION;
    table->cap = (uint32_t)cap;
    table->n = n;
    if (mant_capacity < dfw_mant_bytes(n)) {
        table->stream_bytes = stream_bytes_for(0);
        return DFW_ENOMEM;
    }
    const int nt = resolve_threads(n_threads, n);
    std::vector<ChunkOut> ch(nt);
    std::vector<uint64_t> lo(nt + 1);
    for (int t = 0; t <= nt; ++t) lo[t] = n * (uint64_t)t / (uint64_t)nt;

    // pass 1: split off the raw bytes and count exponents per chunk
    parallel_for(nt, [&](int t) {
        uint64_t h[256] = {0};
        uint64_t i = lo[t];
        seg.for_range(lo[t], lo[t + 1], [&](const uint16_t *p, uint64_t c) {
            uint8_t *m = mant + i;
            for (uint64_t j = 0; j < c; ++j) {
                const uint32_t u = p[j];
                h[(u >> 7) & 0xFF]++;
                m[j] = (uint8_t)(((u >> 8) & 0x80) | (u & 0x7F));
            }
            i += c;
        });
        std::memcpy(ch[t].hist, h, sizeof(h));
    });
    if (mant) std::memset(mant + n, 0, dfw_mant_bytes(n) - n);

    uint64_t hist[256] = {0};
    for (int t = 0; t < nt; ++t)
        for (int s = 0; s < 256; ++s) hist[s] += ch[t].hist[s];
    int k = 0, only = 0;
    for (int s = 0; s < 256; ++s)
        if (hist[s]) {
            ++k;
            only = s;
        }
    table->n_symbols = (uint32_t)k;
    table->single_symbol = k == 1 ? (uint32_t)only : 0u;
    dfw_status st = code_lengths(hist, cap, table->len);
    if (st != DFW_OK) return st;
    uint32_t code[256];
    canonical_codes(table->len, code);

    uint64_t total = 0;
    for (int t = 0; t < nt; ++t) {
        uint64_t b = 0;
        for (int s = 0; s < 256; ++s) b += ch[t].hist[s] * table->len[s];
        ch[t].bit0 = total;
        ch[t].bits = b;
        total += b;
    }
    table->total_bits = total;
    table->stream_bytes = stream_bytes_for(total);
    if (stream_capacity < table->stream_bytes) return DFW_ENOMEM;
    if (!stream) return DFW_EINVAL;

    // pass 2: pack each chunk at its bit offset; the byte shared by two
    // chunks is assembled afterwards from the two halves
    const uint8_t *len = table->len;
    parallel_for(nt, [&](int t) {
        ChunkOut &c = ch[t];
        c.head = c.tail = 0;
        c.has_tail = false;
        if (c.bits == 0) return;
        uint8_t *p = stream + (c.bit0 >> 3);
        const int r = (int)(c.bit0 & 7);
        bool head_pending = r != 0;
        uint64_t acc = 0;
        int nacc = r;
        seg.for_range(lo[t], lo[t + 1], [&](const uint16_t *src, uint64_t cnt) {
            for (uint64_t j = 0; j < cnt; ++j) {
                const uint32_t e = (src[j] >> 7) & 0xFF;
                acc = (acc << len[e]) | code[e];
                nacc += len[e];
                while (nacc >= 8) {
                    const uint8_t byte = (uint8_t)(acc >> (nacc - 8));
                    nacc -= 8;
                    if (head_pending) {
                        c.head = byte;
                        head_pending = false;
                        ++p;
                    } else {
                        *p++ = byte;
                    }
                }
            }
        });
        if (nacc > 0) {
            c.tail = (uint8_t)(acc << (8 - nacc));
            c.has_tail = true;
        }
    });
    // A chunk starting mid-byte shares that byte with the previous chunk's
    // tail (chunks hold >= 32Ki weights, so each spans many bytes).
    for (int t = 1; t < nt; ++t)
        if (ch[t].bits && (ch[t].bit0 & 7)) stream[ch[t].bit0 >> 3] = (uint8_t)(ch[t - 1].tail | ch[t].head);
    if (ch[nt - 1].has_tail) stream[(ch[nt - 1].bit0 + ch[nt - 1].bits) >> 3] = ch[nt - 1].tail;
    const uint64_t used = (total + 7) >> 3;
    std::memset(stream + used, 0, table->stream_bytes - used);
    return DFW_OK;
}

}  // namespace

// ---------------------------------------------------------------- LUT image

dfw_status build_lut(const dfw_table *table, std::vector<uint32_t> &lut) {
    lut.assign(256, 0);
    if (table->total_bits == 0) return DFW_OK;
    if (!kraft_complete(table->len, (int)table->cap)) return DFW_EINVAL;
    uint32_t code[256];
    canonical_codes(table->len, code);
    for (int s = 0; s < 256; ++s) {
        const int l = table->len[s];
        if (!l) continue;
        const uint32_t left = code[s] << (32 - l);  // codeword left-aligned in 32 bits
        size_t tab = 0;
        for (int level = 0; level < 4; ++level) {
            const int rem = l - 8 * level;  // code bits from this level's key on
            const uint32_t key = (left >> (24 - 8 * level)) & 0xFF;
            if (rem <= 8) {
                const uint32_t span = 1u << (8 - rem);
                const uint32_t leaf = (uint32_t)s | ((uint32_t)l << LUT_LEN_SHIFT);
                for (uint32_t j = 0; j < span; ++j) lut[tab * 256 + key + j] = leaf;
                break;
            }
            uint32_t &e = lut[tab * 256 + key];
            if (!(e & LUT_PTR)) {
                const size_t child = lut.size() / 256;
                if (child > LUT_CHILD_MASK) return DFW_EINVAL;
                e = LUT_PTR | (uint32_t)child;
                lut.resize(lut.size() + 256, 0);
            }
            tab = lut[tab * 256 + key] & LUT_CHILD_MASK;
        }
    }
    // level 0: how many whole codewords fit in the 8 key bits, and their bits
    for (uint32_t key = 0; key < 256; ++key) {
        int pos = 0, cnt = 0;
        while (pos < 8) {
            const uint32_t e = lut[(key << pos) & 0xFF];
            if (e & LUT_PTR) break;
            const int l = (int)((e >> LUT_LEN_SHIFT) & 63);
            if (l > 8 - pos) break;
            pos += l;
            ++cnt;
        }
        if (!(lut[key] & LUT_PTR))
            lut[key] |= ((uint32_t)cnt << LUT_CNT_SHIFT) | ((uint32_t)pos << LUT_CBITS_SHIFT);
    }
    return DFW_OK;
}

// One codeword from the hierarchy: x holds the next 32 bits, left-aligned.
// Returns false if the tables do not resolve it within four levels.
static bool hier_decode(const std::vector<uint32_t> &lut, uint32_t x, int &sym, int &len) {
    size_t tab = 0;
    for (int level = 0; level < 4; ++level) {
        const uint32_t e = lut[tab * 256 + ((x >> (24 - 8 * level)) & 0xFF)];
        if (!(e & LUT_PTR)) {
            sym = (int)(e & 0xFF);
            len = (int)((e >> LUT_LEN_SHIFT) & 63);
            return len > 0;
        }
        tab = e & LUT_CHILD_MASK;
        if (tab * 256 >= lut.size()) return false;
    }
    return false;
}

// Fast table: for every K-bit key, the whole codewords (at most four) that
// start at the key's first bit and end within its K bits.  Symbols are stored
// rotated right by one bit, the order in which the bf16 pattern's two bytes
// use the exponent's bits, so the device joins them with masks alone.
dfw_status build_fast(const std::vector<uint32_t> &lut, int fast_bits, std::vector<uint32_t> &fast) {
    if (fast_bits < FAST_BITS_MIN || fast_bits > FAST_BITS_MAX) return DFW_EINVAL;
    const uint32_t entries = 1u << fast_bits;
    fast.assign(2 * (size_t)entries, 0);
    for (uint32_t key = 0; key < entries; ++key) {
        const uint32_t x = key << (32 - fast_bits);
        int pos = 0, cnt = 0;
        uint32_t syms = 0, ends = 0;
        while (cnt < FAST_MAX_SYMS) {
            int sym = 0, len = 0;
            if (!hier_decode(lut, x << pos, sym, len)) break;
            if (pos + len > fast_bits) break;
            syms |= (((uint32_t)sym >> 1) | (((uint32_t)sym & 1u) << 7)) << (8 * cnt);  // rotated right by one
            pos += len;
            ends |= 1u << (pos - 1);
            ++cnt;
            if (pos == 32) break;
        }
        if (cnt == 0) {
            fast[2 * key] = 0;
            fast[2 * key + 1] = FAST_ESC_WORD;
        } else {
            fast[2 * key] = syms;
            fast[2 * key + 1] = (uint32_t)pos | ((uint32_t)(8 * cnt) << FAST_C8_SHIFT) | (ends << FAST_ENDS_SHIFT);
        }
    }
    return DFW_OK;
}

// W * T <= 4096 keeps a tile's worst case (one codeword per stream bit) within
// shared memory: about 174 KB with a 12-bit fast table.
bool plan_shape_supported(uint32_t W, uint32_t T) {
    return (W == 8 || W == 16) && (T == 128 || T == 256 || T == 512) && W * T <= 4096;
}

}  // namespace dfw

// ================================================================ C ABI

using namespace dfw;

extern "C" uint64_t dfw_stream_bound(uint64_t n) { return stream_bytes_for(32ull * n); }

extern "C" uint64_t dfw_mant_bytes(uint64_t n) { return (n + 15) & ~15ull; }

extern "C" dfw_status dfw_encode(const uint16_t *bf16, uint64_t n, int cap, uint8_t *stream,
                                 uint64_t stream_capacity, uint8_t *mant, uint64_t mant_capacity,
                                 dfw_table *table, int n_threads) {
    dfw::NvtxRange nvtx_range("dfw_encode");
    if (n && !bf16) return DFW_EINVAL;
    Segments seg{&bf16, &n, 1, {0, n}};
    return encode_segments(seg, cap, stream, stream_capacity, mant, mant_capacity, table, n_threads);
}

extern "C" dfw_status dfw_encode_multi(const uint16_t *const *tensors, const uint64_t *sizes, int k,
                                       int cap, uint8_t *stream, uint64_t stream_capacity,
                                       uint8_t *mant, uint64_t mant_capacity, dfw_table *table,
                                       uint64_t *tensor_offsets, int n_threads) {
    dfw::NvtxRange nvtx_range("dfw_encode_multi");
    if (k < 1 || !tensors || !sizes || !tensor_offsets) return DFW_EINVAL;
    Segments seg{tensors, sizes, k, std::vector<uint64_t>(k + 1, 0)};
    for (int i = 0; i < k; ++i) {
        if (sizes[i] && !tensors[i]) return DFW_EINVAL;
        seg.off[i + 1] = seg.off[i] + sizes[i];
    }
    for (int i = 0; i <= k; ++i) tensor_offsets[i] = seg.off[i];
    return encode_segments(seg, cap, stream, stream_capacity, mant, mant_capacity, table, n_threads);
}

dfw_status dfw::validate_table(const dfw_table *t) {
    if (!t || t->version != DFW_FORMAT_VERSION || t->cap < 1 || t->cap > DFW_MAX_CAP) return DFW_EINVAL;
    if (t->stream_bytes != stream_bytes_for(t->total_bits)) return DFW_EINVAL;
    if (t->n == 0) return t->total_bits == 0 ? DFW_OK : DFW_EINVAL;
    if (t->total_bits == 0) {  // one symbol: no lengths, exponent in single_symbol
        for (int s = 0; s < 256; ++s)
            if (t->len[s]) return DFW_EINVAL;
        return (t->n_symbols == 1 && t->single_symbol < 256) ? DFW_OK : DFW_EINVAL;
    }
    if (!kraft_complete(t->len, (int)t->cap)) return DFW_EINVAL;
    int mn = 64, mx = 0;
    for (int s = 0; s < 256; ++s)
        if (t->len[s]) {
            mn = std::min(mn, (int)t->len[s]);
            mx = std::max(mx, (int)t->len[s]);
        }
    if (t->total_bits < t->n * (uint64_t)mn || t->total_bits > t->n * (uint64_t)mx) return DFW_ECORRUPT;
    return DFW_OK;
}

extern "C" dfw_status dfw_plan_query(const dfw_table *table, uint32_t window_bytes,
                                     uint32_t tile_windows, dfw_plan_info *info) {
    if (!info || !plan_shape_supported(window_bytes, tile_windows)) return DFW_EINVAL;
    dfw_status st = validate_table(table);
    if (st != DFW_OK) return st;
    const uint32_t fb = info->fast_bits ? info->fast_bits : (uint32_t)FAST_BITS_DEFAULT;
    if (fb < (uint32_t)FAST_BITS_MIN || fb > (uint32_t)FAST_BITS_MAX) return DFW_EINVAL;
    std::memset(info, 0, sizeof(*info));
    info->fast_bits = fb;
    info->window_bytes = window_bytes;
    info->tile_windows = tile_windows;
    const uint64_t wbits = 8ull * window_bytes;
    info->n_windows = (table->total_bits + wbits - 1) / wbits;
    info->n_tiles = (info->n_windows + tile_windows - 1) / tile_windows;
    std::vector<uint32_t> lut;
    st = build_lut(table, lut);
    if (st != DFW_OK) return st;
    info->lut_tables = (uint32_t)(lut.size() / 256);
    info->lut_words = (2u << fb) + (uint32_t)lut.size();
    return DFW_OK;
}

extern "C" dfw_status dfw_plan(const uint8_t *stream, const dfw_table *table, uint8_t *gap,
                               uint64_t *out_start, uint32_t *lut, dfw_plan_info *info) {
    dfw::NvtxRange nvtx_range("dfw_plan");
    if (!info || !out_start || !lut) return DFW_EINVAL;
    dfw_plan_info q;
    q.fast_bits = info->fast_bits;
    dfw_status st = dfw_plan_query(table, info->window_bytes, info->tile_windows, &q);
    if (st != DFW_OK) return st;
    if (q.n_windows != info->n_windows || q.n_tiles != info->n_tiles || q.lut_words != info->lut_words)
        return DFW_EINVAL;
    if (q.n_windows && (!gap || !stream)) return DFW_EINVAL;
    std::vector<uint32_t> img, fast;
    build_lut(table, img);
    st = build_fast(img, (int)q.fast_bits, fast);
    if (st != DFW_OK) return st;
    std::memcpy(lut, fast.data(), fast.size() * sizeof(uint32_t));
    std::memcpy(lut + fast.size(), img.data(), img.size() * sizeof(uint32_t));
    const uint64_t n = table->n, tb = table->total_bits;
    const uint64_t wbits = 8ull * q.window_bytes, tbits = wbits * q.tile_windows;
    if (tb == 0) {
        out_start[0] = n;
        info->max_tile_symbols = 0;
        return DFW_OK;
    }
    // length of the codeword at a left-aligned 32-bit window: a 12-bit table
    // for short codes, then the canonical limits for longer ones
    uint32_t code[256];
    canonical_codes(table->len, code);
    uint64_t limit[34] = {0};
    {
        uint64_t cnt[34] = {0};
        for (int s = 0; s < 256; ++s)
            if (table->len[s]) cnt[table->len[s]]++;
        uint64_t first = 0;
        for (int l = 1; l <= 32; ++l) {
            first = (first + cnt[l - 1]) << 1;
            limit[l] = first + cnt[l];
        }
    }
    std::vector<uint8_t> len12(4096, 0);
    for (uint32_t x = 0; x < 4096; ++x) {
        for (int l = 1; l <= 12; ++l)
            if ((x >> (12 - l)) < limit[l]) {
                len12[x] = (uint8_t)l;
                break;
            }
    }
    uint64_t pos = 0, count = 0, t_next = 0, b_next = 0;
    const uint64_t nwin = q.n_windows, ntiles = q.n_tiles;
    while (pos < tb) {
        while (t_next < nwin && t_next * wbits <= pos) {
            const uint64_t g = pos - t_next * wbits;
            if (g >= 32) return DFW_ECORRUPT;
            gap[t_next++] = (uint8_t)g;
        }
        while (b_next < ntiles && b_next * tbits <= pos) out_start[b_next++] = count;
        // 40 bits from pos, big-endian (the stream carries >= 16 guard bytes)
        const uint8_t *p = stream + (pos >> 3);
        uint64_t v = 0;
        for (int i = 0; i < 5; ++i) v = (v << 8) | p[i];
        const uint32_t x = (uint32_t)(v >> (8 - (pos & 7)));
        int l = len12[x >> 20];
        if (!l) {
            for (l = 13; l <= 32; ++l)
                if ((uint64_t)(x >> (32 - l)) < limit[l]) break;
            if (l > 32) return DFW_ECORRUPT;
        }
        pos += (uint64_t)l;
        if (++count > n) return DFW_ECORRUPT;
    }
    if (pos != tb || count != n) return DFW_ECORRUPT;
    while (t_next < nwin) {
        const uint64_t g = tb - t_next * wbits;
        if (g >= 32) return DFW_ECORRUPT;
        gap[t_next++] = (uint8_t)g;
    }
    std::memset(gap + nwin, 0, (size_t)(q.n_tiles * q.tile_windows - nwin));  // pad to whole tiles
    while (b_next < ntiles) out_start[b_next++] = n;
    out_start[ntiles] = n;
    uint64_t mx = 0;
    for (uint64_t b = 0; b < ntiles; ++b) mx = std::max(mx, out_start[b + 1] - out_start[b]);
    info->max_tile_symbols = mx;
    return DFW_OK;
}

// Stream bytes a group reads: from the 16-byte boundary at or below its first
// bit to 8 guard bytes past its last bit, rounded up to 16.
uint32_t dfw::group_span_bytes(uint64_t start_bit, uint64_t end_bit) {
    const uint64_t b0 = (start_bit >> 3) & ~15ull;
    const uint64_t b1 = (((end_bit + 7) >> 3) + 8 + 15) & ~15ull;
    return (uint32_t)(b1 - b0);
}

namespace {
// Codeword lengths at successive stream positions, from the canonical limits
// (a 12-bit table for short codes).
struct LengthWalker {
    uint64_t limit[34] = {0};
    std::vector<uint8_t> len12;
    explicit LengthWalker(const uint8_t len[256]) : len12(4096, 0) {
        uint64_t cnt[34] = {0};
        for (int s = 0; s < 256; ++s)
            if (len[s]) cnt[len[s]]++;
        uint64_t first = 0;
        for (int l = 1; l <= 32; ++l) {
            first = (first + cnt[l - 1]) << 1;
            limit[l] = first + cnt[l];
        }
        for (uint32_t x = 0; x < 4096; ++x)
            for (int l = 1; l <= 12; ++l)
                if ((x >> (12 - l)) < limit[l]) {
                    len12[x] = (uint8_t)l;
                    break;
                }
    }
    // Length of the codeword at bit pos (the stream has >= 16 guard bytes), 0 if none.
    int at(const uint8_t *stream, uint64_t pos) const {
        const uint8_t *p = stream + (pos >> 3);
        uint64_t v = 0;
        for (int i = 0; i < 5; ++i) v = (v << 8) | p[i];
        const uint32_t x = (uint32_t)(v >> (8 - (pos & 7)));
        int l = len12[x >> 20];
        if (!l) {
            for (l = 13; l <= 32; ++l)
                if ((uint64_t)(x >> (32 - l)) < limit[l]) break;
            if (l > 32) return 0;
        }
        return l;
    }
};
}  // namespace

extern "C" dfw_status dfw_plan_lanes_query(const dfw_table *table, dfw_lanes_info *info) {
    if (!info) return DFW_EINVAL;
    dfw_status st = validate_table(table);
    if (st != DFW_OK) return st;
    const uint32_t fb = info->fast_bits ? info->fast_bits : (uint32_t)FAST_BITS_DEFAULT_LANES;
    if (fb < (uint32_t)FAST_BITS_MIN || fb > (uint32_t)FAST_BITS_MAX) return DFW_EINVAL;
    std::memset(info, 0, sizeof(*info));
    info->fast_bits = fb;
    info->chunk_symbols = LANE_SYMS;
    info->group_chunks = GROUP_CHUNKS;
    info->n_chunks = (table->n + LANE_SYMS - 1) / LANE_SYMS;
    info->n_groups = (info->n_chunks + GROUP_CHUNKS - 1) / GROUP_CHUNKS;
    std::vector<uint32_t> lut;
    st = build_lut(table, lut);
    if (st != DFW_OK) return st;
    info->lut_tables = (uint32_t)(lut.size() / 256);
    info->lut_words = (2u << fb) + (uint32_t)lut.size();
    return DFW_OK;
}

extern "C" dfw_status dfw_plan_lanes(const uint8_t *stream, const dfw_table *table, uint16_t *chunk_bits,
                                     uint64_t *group_start, uint32_t *lut, dfw_lanes_info *info) {
    dfw::NvtxRange nvtx_range("dfw_plan_lanes");
    if (!info || !group_start || !lut) return DFW_EINVAL;
    dfw_lanes_info q;
    q.fast_bits = info->fast_bits;
    dfw_status st = dfw_plan_lanes_query(table, &q);
    if (st != DFW_OK) return st;
    if (q.n_groups != info->n_groups || q.lut_words != info->lut_words) return DFW_EINVAL;
    if (q.n_groups && !chunk_bits) return DFW_EINVAL;
    std::vector<uint32_t> img, fast;
    build_lut(table, img);
    st = build_fast(img, (int)q.fast_bits, fast);
    if (st != DFW_OK) return st;
    std::memcpy(lut, fast.data(), fast.size() * sizeof(uint32_t));
    std::memcpy(lut + fast.size(), img.data(), img.size() * sizeof(uint32_t));
    const uint64_t n = table->n, tb = table->total_bits;
    std::memset(chunk_bits, 0, (size_t)(q.n_groups * GROUP_CHUNKS) * sizeof(uint16_t));
    if (tb == 0) {  // one symbol: no bits anywhere
        for (uint64_t g = 0; g <= q.n_groups; ++g) group_start[g] = 0;
        info->max_group_bytes = 16;
        return DFW_OK;
    }
    if (!stream) return DFW_EINVAL;
    LengthWalker walk(table->len);
    uint64_t pos = 0, cstart = 0;
    for (uint64_t i = 0; i < n; ++i) {
        if (i % LANE_SYMS == 0) {
            cstart = pos;
            if (i % ((uint64_t)LANE_SYMS * GROUP_CHUNKS) == 0) group_start[i / ((uint64_t)LANE_SYMS * GROUP_CHUNKS)] = pos;
        }
        if (pos >= tb) return DFW_ECORRUPT;
        const int l = walk.at(stream, pos);
        if (!l) return DFW_ECORRUPT;
        pos += (uint64_t)l;
        if ((i + 1) % LANE_SYMS == 0 || i + 1 == n) chunk_bits[i / LANE_SYMS] = (uint16_t)(pos - cstart);
    }
    if (pos != tb) return DFW_ECORRUPT;
    group_start[q.n_groups] = tb;
    uint32_t mx = 16;
    for (uint64_t g = 0; g < q.n_groups; ++g) mx = std::max(mx, group_span_bytes(group_start[g], group_start[g + 1]));
    info->max_group_bytes = mx;
    return DFW_OK;
}

extern "C" const char *dfw_strerror(dfw_status s) {
    switch (s) {
        case DFW_OK: return "ok";
        case DFW_EINVAL: return "invalid argument";
        case DFW_ECAP: return "length cap too small for the number of distinct exponents";
        case DFW_ENOMEM: return "buffer too small or out of host memory";
        case DFW_ECORRUPT: return "stream, aux arrays or table are inconsistent";
        case DFW_EALIGN: return "device pointer not 16-byte aligned";
        case DFW_ECUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

extern "C" dfw_status dfw_lanes_lut(const dfw_table *table, const dfw_lanes_info *info, uint32_t *lut) {
    if (!info || !lut) return DFW_EINVAL;
    dfw_lanes_info q;
    std::memset(&q, 0, sizeof(q));
    q.fast_bits = info->fast_bits;
    dfw_status st = dfw_plan_lanes_query(table, &q);
    if (st != DFW_OK) return st;
    if (q.lut_words != info->lut_words || q.fast_bits != info->fast_bits) return DFW_EINVAL;
    std::vector<uint32_t> img, fast;
    st = build_lut(table, img);
    if (st != DFW_OK) return st;
    st = build_fast(img, (int)q.fast_bits, fast);
    if (st != DFW_OK) return st;
    std::memcpy(lut, fast.data(), fast.size() * sizeof(uint32_t));
    std::memcpy(lut + fast.size(), img.data(), img.size() * sizeof(uint32_t));
    return DFW_OK;
}

// ------------------------------------------------------------ container
//
// The encoded artefact as one byte buffer (layout in include/dfw.h): a fixed
// header of little-endian fields, the tensor offsets, the stream, the raw
// bytes and, optionally, the known-start plan; every section starts on a
// 16-byte boundary; an FNV-1a 64-bit hash of all earlier bytes closes it.

namespace {

constexpr uint64_t CONT_HEADER = 312;  // magic .. code lengths
constexpr char CONT_MAGIC[8] = {'D', 'F', 'W', 'B', 'F', '1', '6', '\0'};

uint64_t up16(uint64_t x) { return (x + 15) & ~15ull; }

struct ContLayout {
    uint64_t offsets_at, stream_at, mant_at, chunk_bits_at, group_start_at, hash_at, total;
};

// Section offsets; false if a size overflows.
bool cont_layout(uint64_t n, uint64_t stream_bytes, uint64_t k, bool plan, ContLayout &L) {
    if (k == 0 || k > (1ull << 32) || n > (1ull << 56) || stream_bytes > (1ull << 56)) return false;
    const uint64_t n_chunks = (n + LANE_SYMS - 1) / LANE_SYMS;
    const uint64_t n_groups = (n_chunks + GROUP_CHUNKS - 1) / GROUP_CHUNKS;
    L.offsets_at = up16(CONT_HEADER);
    L.stream_at = up16(L.offsets_at + 8 * (k + 1));
    L.mant_at = up16(L.stream_at + stream_bytes);
    uint64_t end = L.mant_at + ((n + 15) & ~15ull);
    L.chunk_bits_at = L.group_start_at = 0;
    if (plan) {
        L.chunk_bits_at = up16(end);
        L.group_start_at = up16(L.chunk_bits_at + 2 * (uint64_t)GROUP_CHUNKS * n_groups);
        end = L.group_start_at + 8 * (n_groups + 1);
    }
    L.hash_at = up16(end);
    L.total = L.hash_at + 8;
    return true;
}

uint64_t fnv1a64(const uint8_t *p, uint64_t bytes) {
    uint64_t h = 0xcbf29ce484222325ull;
    for (uint64_t i = 0; i < bytes; ++i) {
        h ^= p[i];
        h *= 0x100000001b3ull;
    }
    return h;
}

void put32(uint8_t *p, uint32_t v) {
    for (int i = 0; i < 4; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
void put64(uint8_t *p, uint64_t v) {
    for (int i = 0; i < 8; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
uint32_t get32(const uint8_t *p) {
    uint32_t v = 0;
    for (int i = 0; i < 4; ++i) v |= (uint32_t)p[i] << (8 * i);
    return v;
}
uint64_t get64(const uint8_t *p) {
    uint64_t v = 0;
    for (int i = 0; i < 8; ++i) v |= (uint64_t)p[i] << (8 * i);
    return v;
}

}  // namespace

extern "C" uint64_t dfw_container_bytes(const dfw_table *table, int k, int with_plan) {
    if (!table || k < 1) return 0;
    ContLayout L;
    if (!cont_layout(table->n, table->stream_bytes, (uint64_t)k, with_plan != 0, L)) return 0;
    return L.total;
}

extern "C" dfw_status dfw_container_write(const dfw_table *table, int k, const uint64_t *tensor_offsets,
                                          const uint8_t *stream, const uint8_t *mant, const uint16_t *chunk_bits,
                                          const uint64_t *group_start, uint8_t *out, uint64_t out_bytes) {
    dfw::NvtxRange nvtx_range("dfw_container_write");
    dfw_status st = validate_table(table);
    if (st != DFW_OK) return st;
    if (k < 1 || !out || (table->stream_bytes && !stream) || (table->n && !mant)) return DFW_EINVAL;
    if ((chunk_bits == nullptr) != (group_start == nullptr)) return DFW_EINVAL;
    const bool plan = chunk_bits != nullptr;
    ContLayout L;
    if (!cont_layout(table->n, table->stream_bytes, (uint64_t)k, plan, L)) return DFW_EINVAL;
    if (out_bytes < L.total) return DFW_ENOMEM;
    if (tensor_offsets) {
        if (tensor_offsets[0] != 0 || tensor_offsets[k] != table->n) return DFW_EINVAL;
        for (int i = 0; i < k; ++i)
            if (tensor_offsets[i + 1] < tensor_offsets[i]) return DFW_EINVAL;
    } else if (k != 1) {
        return DFW_EINVAL;
    }
    std::memset(out, 0, L.total);
    std::memcpy(out, CONT_MAGIC, 8);
    put32(out + 8, DFW_FORMAT_VERSION);
    put32(out + 12, plan ? 1u : 0u);
    put32(out + 16, table->cap);
    put32(out + 20, table->n_symbols);
    put32(out + 24, table->single_symbol);
    put32(out + 28, (uint32_t)k);
    put64(out + 32, table->n);
    put64(out + 40, table->total_bits);
    put64(out + 48, table->stream_bytes);
    std::memcpy(out + 56, table->len, 256);
    for (int i = 0; i <= k; ++i)
        put64(out + L.offsets_at + 8 * i, tensor_offsets ? tensor_offsets[i] : (i ? table->n : 0));
    if (table->stream_bytes) std::memcpy(out + L.stream_at, stream, table->stream_bytes);
    if (table->n) std::memcpy(out + L.mant_at, mant, (table->n + 15) & ~15ull);
    if (plan) {
        const uint64_t n_groups = ((table->n + LANE_SYMS - 1) / LANE_SYMS + GROUP_CHUNKS - 1) / GROUP_CHUNKS;
        for (uint64_t i = 0; i < (uint64_t)GROUP_CHUNKS * n_groups; ++i) {
            out[L.chunk_bits_at + 2 * i] = (uint8_t)chunk_bits[i];
            out[L.chunk_bits_at + 2 * i + 1] = (uint8_t)(chunk_bits[i] >> 8);
        }
        for (uint64_t g = 0; g <= n_groups; ++g) put64(out + L.group_start_at + 8 * g, group_start[g]);
    }
    put64(out + L.hash_at, fnv1a64(out, L.hash_at));
    return DFW_OK;
}

extern "C" dfw_status dfw_container_read(const uint8_t *buf, uint64_t bytes, dfw_table *table,
                                         dfw_container_view *view) {
    dfw::NvtxRange nvtx_range("dfw_container_read");
    if (!buf || !table || !view) return DFW_EINVAL;
    if (bytes < CONT_HEADER + 8 || std::memcmp(buf, CONT_MAGIC, 8) != 0) return DFW_ECORRUPT;
    if (get32(buf + 8) != DFW_FORMAT_VERSION) return DFW_EINVAL;
    const uint32_t flags = get32(buf + 12);
    if (flags & ~1u) return DFW_ECORRUPT;
    const uint64_t k = get32(buf + 28), n = get64(buf + 32), stream_bytes = get64(buf + 48);
    ContLayout L;
    if (!cont_layout(n, stream_bytes, k, flags & 1u, L) || L.total != bytes) return DFW_ECORRUPT;
    if (get64(buf + L.hash_at) != fnv1a64(buf, L.hash_at)) return DFW_ECORRUPT;
    dfw_table t;
    std::memset(&t, 0, sizeof(t));
    t.version = DFW_FORMAT_VERSION;
    t.cap = get32(buf + 16);
    t.n_symbols = get32(buf + 20);
    t.single_symbol = get32(buf + 24);
    t.n = n;
    t.total_bits = get64(buf + 40);
    t.stream_bytes = stream_bytes;
    std::memcpy(t.len, buf + 56, 256);
    if (validate_table(&t) != DFW_OK) return DFW_ECORRUPT;
    if (get64(buf + L.offsets_at) != 0 || get64(buf + L.offsets_at + 8 * k) != n) return DFW_ECORRUPT;
    for (uint64_t i = 0; i < k; ++i)
        if (get64(buf + L.offsets_at + 8 * (i + 1)) < get64(buf + L.offsets_at + 8 * i)) return DFW_ECORRUPT;
    if (flags & 1u) {  // the plan must agree with itself and with the table
        const uint64_t n_groups = ((n + LANE_SYMS - 1) / LANE_SYMS + GROUP_CHUNKS - 1) / GROUP_CHUNKS;
        if (get64(buf + L.group_start_at) != 0 || get64(buf + L.group_start_at + 8 * n_groups) != t.total_bits)
            return DFW_ECORRUPT;
        for (uint64_t g = 0; g < n_groups; ++g) {
            uint64_t s = 0;
            for (uint32_t c = 0; c < GROUP_CHUNKS; ++c) {
                const uint64_t at = L.chunk_bits_at + 2 * ((uint64_t)GROUP_CHUNKS * g + c);
                s += (uint64_t)buf[at] | ((uint64_t)buf[at + 1] << 8);
            }
            if (get64(buf + L.group_start_at + 8 * (g + 1)) - get64(buf + L.group_start_at + 8 * g) != s)
                return DFW_ECORRUPT;
        }
    }
    *table = t;
    view->k = (int)k;
    view->has_plan = (int)(flags & 1u);
    view->offsets_at = L.offsets_at;
    view->stream_at = L.stream_at;
    view->mant_at = L.mant_at;
    view->chunk_bits_at = L.chunk_bits_at;
    view->group_start_at = L.group_start_at;
    return DFW_OK;
}
