// dfw_encode.cu -- the encoder on the GPU.  Same output as the host encoder
// (dfw_encode), byte for byte, plus the known-start plan's aux arrays, made
// in the passes that need them anyway.
//
// Source: DFloat11 abstract (frequency-based variable-length codes for the
// bf16 exponents; bit-exact), the LazyWeights write-up (Huffman; lanes that
// start at known bits).  The passes:
//   1  split + histogram   each thread reads 8 bf16 (16 bytes), writes their 8
//                          raw bytes, and counts their exponents in its
//                          warp's shared histogram (4 copies, lanes spread
//                          over them to thin out same-bin atomics)
//   -  code (host)         package-merge lengths and canonical codes from the
//                          histogram, exactly as the host encoder does
//   2  chunk bits          one warp per group of 32 chunks x 64 codewords:
//                          coalesced loads (lane l holds 8 consecutive
//                          weights), code lengths from a shared table, a
//                          3-step shuffle sum per chunk -> chunk_bits[]; the
//                          group total goes to group_start[g]
//   3  group starts        CTAs over contiguous ranges of groups: one
//                          kernel sums each range, a second adds the earlier
//                          ranges' sums and turns the group totals into
//                          exclusive prefix sums in place (group_start[]);
//                          the last range writes the total bit count; all
//                          record the largest group span
//   4  pack                one warp per group: each lane joins its 8
//                          codewords into one 64-bit value (almost always
//                          enough; longer runs take a general path) and ORs
//                          it at its bit offset (warp prefix sum) into the
//                          warp's shared word buffer (neighbours share a
//                          word, so the ORs are atomic); the warp then writes
//                          the group's words, big-endian, with plain stores
//                          inside and atomic ORs on the two words it may
//                          share with the neighbouring groups (a small kernel
//                          zeroes those words and the padding first)
// Nothing waits on another CTA; every loop is bounded by n.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "dfw_internal.h"

namespace dfw {
namespace {

// The checks build (DFW_CHECKS): the encoder kernels' own record of the first
// range check that failed (this file's kernels have no status word); in the
// ordinary build enc_check is the constant true.
__device__ unsigned int g_enc_check_site;
#ifdef DFW_CHECKS
__device__ __noinline__ void enc_check_failed(uint32_t site) { atomicCAS(&g_enc_check_site, 0u, site); }
__device__ __forceinline__ bool enc_check(bool ok, uint32_t site) {
    if (!ok) enc_check_failed(site);
    return ok;
}
#else
__device__ __forceinline__ constexpr bool enc_check(bool, uint32_t) { return true; }
#endif

constexpr int SPLIT_NT = 256;     // threads per CTA of pass 1
constexpr int HIST_COPIES = 4;    // histogram copies per warp
constexpr int GROUP_NT = 512;     // threads per CTA of passes 2 and 4
constexpr int SCAN_NT = 256;      // threads per CTA of pass 3
constexpr uint32_t GROUP_W = LANE_SYMS * GROUP_CHUNKS;  // weights per group (2048)

// Layout of the caller's scratch buffer.
constexpr uint32_t SCAN_CTAS = 1024;  // most CTAs of the group-start passes
struct EncScratch {
    unsigned long long hist[256];
    unsigned long long total_bits;
    unsigned int max_span;  // largest group span in bytes (as the lanes plan counts it)
    unsigned int max_group_bits;
    unsigned long long range_total[SCAN_CTAS];  // pass 3a: bits of each CTA's range of groups
};

struct LenTable {
    uint8_t len[256];
};
struct CodeTable {
    unsigned long long lc[256];  // (length << 32) | canonical code
};

__device__ __forceinline__ uint32_t span_bytes_dev(uint64_t start_bit, uint64_t end_bit) {
    const uint64_t b0 = (start_bit >> 3) & ~15ull;
    const uint64_t b1 = (((end_bit + 7) >> 3) + 8 + 15) & ~15ull;
    return (uint32_t)(b1 - b0);
}

__device__ __forceinline__ uint32_t bswap32_dev(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// ------------------------------------------------------------ pass 1

// Raw bytes of four bf16 patterns held in two words: (hi byte & 0x80) |
// (lo byte & 0x7F) per pattern.  Exponents: (hi byte << 1) | (lo byte >> 7).
__device__ __forceinline__ void split4(uint32_t x0, uint32_t x1, uint32_t &m4, uint32_t &e4) {
    const uint32_t lo = __byte_perm(x0, x1, 0x6420), hi = __byte_perm(x0, x1, 0x7531);
    m4 = (hi & 0x80808080u) | (lo & 0x7F7F7F7Fu);
    e4 = ((hi << 1) & 0xFEFEFEFEu) | ((lo >> 7) & 0x01010101u);
}

__global__ void __launch_bounds__(SPLIT_NT) enc_split_hist(const uint16_t *__restrict__ in, uint64_t n,
                                                            uint8_t *__restrict__ mant, uint64_t mant_bytes,
                                                            unsigned long long *__restrict__ hist) {
    __shared__ uint32_t h[SPLIT_NT / 32][256 * HIST_COPIES];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < (SPLIT_NT / 32) * 256 * HIST_COPIES; i += SPLIT_NT) (&h[0][0])[i] = 0u;
    __syncthreads();
    uint32_t *hw = h[warp] + (lane & (HIST_COPIES - 1));
    const uint64_t n8 = n >> 3;
    const uint64_t stride = (uint64_t)gridDim.x * SPLIT_NT;
    // one 16-byte item: raw bytes out, exponents into the histogram
    auto item = [&](uint64_t i, const uint4 v) {
        uint32_t m0, e0, m1, e1;
        split4(v.x, v.y, m0, e0);
        split4(v.z, v.w, m1, e1);
        if (enc_check(8u * i + 8u <= mant_bytes, CK_ENC_SPLIT))
            __stcs(reinterpret_cast<uint2 *>(mant) + i, make_uint2(m0, m1));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            atomicAdd(hw + HIST_COPIES * ((e0 >> (8 * k)) & 0xFFu), 1u);
            atomicAdd(hw + HIST_COPIES * ((e1 >> (8 * k)) & 0xFFu), 1u);
        }
    };
    uint64_t i = (uint64_t)blockIdx.x * SPLIT_NT + tid;
    // four loads in flight per thread before any is used (the pass is bound
    // by memory latency, not by its arithmetic)
    for (; i + 3 * stride < n8; i += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldcs(reinterpret_cast<const uint4 *>(in) + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) item(i + u * stride, v[u]);
    }
    for (; i < n8; i += stride) item(i, __ldcs(reinterpret_cast<const uint4 *>(in) + i));
    if (blockIdx.x == 0) {  // the < 8 trailing weights and the zero padding of the raw bytes
        for (uint64_t j = (n8 << 3) + tid; j < mant_bytes; j += SPLIT_NT) {
            uint8_t m = 0;
            if (j < n) {
                const uint32_t u = in[j];
                m = (uint8_t)(((u >> 8) & 0x80u) | (u & 0x7Fu));
                atomicAdd(hw + HIST_COPIES * ((u >> 7) & 0xFFu), 1u);
            }
            mant[j] = m;
        }
    }
    __syncthreads();
    for (int b = tid; b < 256; b += SPLIT_NT) {
        unsigned long long s = 0;
        for (int w = 0; w < SPLIT_NT / 32; ++w)
            for (int c = 0; c < HIST_COPIES; ++c) s += h[w][HIST_COPIES * b + c];
        if (s) atomicAdd(hist + b, s);
    }
}

// ------------------------------------------------------------ pass 2

constexpr unsigned FULL = 0xFFFFFFFFu;

// Exponents of the 8 bf16 patterns in v, as two words of 4 bytes.
__device__ __forceinline__ void exps8(const uint4 v, uint32_t &e0, uint32_t &e1) {
    uint32_t m;
    split4(v.x, v.y, m, e0);
    split4(v.z, v.w, m, e1);
}

// The 8 weights of lane `lane` in step j of a group: weights 8 (32 j + lane)
// .. + 7 of the group, i.e. of chunk 4 j + lane / 8.  Fills the exponents
// (0 past n) and returns how many of the 8 exist.
__device__ __forceinline__ uint32_t load8(const uint16_t *__restrict__ in, uint64_t n, uint64_t e0, uint32_t &x0,
                                          uint32_t &x1) {
    if (e0 + 8 <= n) {
        exps8(__ldcs(reinterpret_cast<const uint4 *>(in + e0)), x0, x1);
        return 8u;
    }
    x0 = x1 = 0u;
    uint32_t c = 0;
    for (uint64_t k = e0; k < n; ++k, ++c) {  // the tensor's last, partial step
        const uint32_t e = (in[k] >> 7) & 0xFFu;
        if (c < 4) x0 |= e << (8 * c);
        else x1 |= e << (8 * (c - 4));
    }
    return c;
}

__global__ void __launch_bounds__(GROUP_NT) enc_chunk_bits(const uint16_t *__restrict__ in, uint64_t n,
                                                            const LenTable lt, uint16_t *__restrict__ chunk_bits,
                                                            uint64_t *__restrict__ group_start, uint32_t n_groups) {
    __shared__ uint32_t s_len[256];
    for (int i = threadIdx.x; i < 256; i += GROUP_NT) s_len[i] = lt.len[i];
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t wstride = gridDim.x * (GROUP_NT / 32);
    for (uint32_t g = blockIdx.x * (GROUP_NT / 32) + (threadIdx.x >> 5); g < n_groups; g += wstride) {
        const uint64_t base = (uint64_t)g * GROUP_W;
        const bool whole = base + GROUP_W <= n;
        uint4 raw[8];  // all eight loads in flight before any is used
        if (whole) {
#pragma unroll
            for (uint32_t j = 0; j < 8; ++j)
                raw[j] = __ldcs(reinterpret_cast<const uint4 *>(in + base + 8u * (32u * j + lane)));
        }
        uint32_t mine = 0;
#pragma unroll
        for (uint32_t j = 0; j < 8; ++j) {
            uint32_t b = 0;
            if (whole) {  // every group but the tensor's last: eight exponents, no checks
                uint32_t x0, x1;
                exps8(raw[j], x0, x1);
#pragma unroll
                for (uint32_t k = 0; k < 4; ++k)
                    b += s_len[__byte_perm(x0, 0u, 0x4440u + k)] + s_len[__byte_perm(x1, 0u, 0x4440u + k)];
            } else {
                uint32_t x0, x1;
                const uint32_t cnt = load8(in, n, base + 8u * (32u * j + lane), x0, x1);
                for (uint32_t k = 0; k < 4; ++k) b += k < cnt ? s_len[(x0 >> (8 * k)) & 0xFFu] : 0u;
                for (uint32_t k = 4; k < 8; ++k) b += k < cnt ? s_len[(x1 >> (8 * (k - 4))) & 0xFFu] : 0u;
            }
            // lanes 8q .. 8q + 7 hold chunk 4 j + q: sum them
            b += __shfl_xor_sync(FULL, b, 1);
            b += __shfl_xor_sync(FULL, b, 2);
            b += __shfl_xor_sync(FULL, b, 4);
            const uint32_t from = __shfl_sync(FULL, b, 8u * (lane & 3u));
            if ((lane >> 2) == j) mine = from;  // lane l keeps chunk l
        }
        chunk_bits[(uint64_t)g * GROUP_CHUNKS + lane] = (uint16_t)mine;
        uint32_t tot = mine;
        for (int d = 16; d > 0; d >>= 1) tot += __shfl_xor_sync(FULL, tot, d);
        if (lane == 0) group_start[g] = tot;  // the group's total until pass 3
    }
}

// ------------------------------------------------------------ pass 3

// Block-wide inclusive scan of one value per thread (SCAN_NT threads);
// returns the inclusive prefix and sets `total` for every thread.
__device__ __forceinline__ unsigned long long block_scan(unsigned long long x, unsigned long long &total,
                                                         unsigned long long *s_warp) {
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    unsigned long long incl = x;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const unsigned long long y = __shfl_up_sync(FULL, incl, d);
        if (lane >= (uint32_t)d) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    unsigned long long before = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < SCAN_NT / 32; ++w) {
        const unsigned long long v = s_warp[w];
        if (w < (int)warp) before += v;
        total += v;
    }
    __syncthreads();  // s_warp may be reused
    return before + incl;
}

// Pass 3a: CTA b sums the group totals of its range [b R, (b + 1) R).
__global__ void __launch_bounds__(SCAN_NT) enc_range_totals(const uint64_t *__restrict__ gs, uint32_t n_groups,
                                                            uint32_t range, EncScratch *__restrict__ res) {
    __shared__ unsigned long long s_warp[SCAN_NT / 32];
    const uint32_t lo = blockIdx.x * range, hi = min(n_groups, lo + range);
    unsigned long long s = 0;
    uint32_t mb = 0;
    for (uint32_t i = lo + threadIdx.x; i < hi; i += SCAN_NT) {
        const uint64_t v = gs[i];
        s += v;
        mb = max(mb, (uint32_t)v);
    }
    unsigned long long total;
    block_scan(s, total, s_warp);
    if (threadIdx.x == 0) res->range_total[blockIdx.x] = total;
    for (int d = 16; d > 0; d >>= 1) mb = max(mb, __shfl_xor_sync(FULL, mb, d));
    if ((threadIdx.x & 31u) == 0) atomicMax(&res->max_group_bits, mb);
}

// Pass 3b: CTA b adds the totals of the ranges before its own, then turns
// its range's group totals into exclusive prefix sums in place, a tile of
// SCAN_NT at a time.  The last CTA writes group_start[n_groups] and the total.
__global__ void __launch_bounds__(SCAN_NT) enc_range_scan(uint64_t *__restrict__ gs, uint32_t n_groups,
                                                          uint32_t range, EncScratch *__restrict__ res) {
    __shared__ unsigned long long s_warp[SCAN_NT / 32];
    unsigned long long part = 0, carry;
    for (uint32_t b = threadIdx.x; b < blockIdx.x; b += SCAN_NT) part += res->range_total[b];
    block_scan(part, carry, s_warp);  // carry = bits of every earlier range
    const uint32_t lo = blockIdx.x * range, hi = min(n_groups, lo + range);
    uint32_t ms = 16;
    for (uint32_t base = lo; base < hi; base += SCAN_NT) {
        const uint32_t i = base + threadIdx.x;
        const uint64_t v = i < hi ? gs[i] : 0ull;
        unsigned long long tile;
        const unsigned long long incl = block_scan(v, tile, s_warp);
        if (i < hi) {
            const unsigned long long start = carry + incl - v;
            gs[i] = start;
            ms = max(ms, span_bytes_dev(start, start + v));
        }
        carry += tile;
    }
    if (blockIdx.x + 1 == gridDim.x && threadIdx.x == 0) {
        gs[n_groups] = carry;
        res->total_bits = carry;
    }
    for (int d = 16; d > 0; d >>= 1) ms = max(ms, __shfl_xor_sync(FULL, ms, d));
    if ((threadIdx.x & 31u) == 0) atomicMax(&res->max_span, ms);
}

// ------------------------------------------------------------ pass 4

// Before packing: zeroes the words that packing ORs into (the first and the
// last word of every group; a neighbouring group may share them) and the
// padding words after the last codeword.  Packing writes every other word
// whole, so the rest of the stream needs no clearing.
__global__ void __launch_bounds__(SCAN_NT) enc_zero_edges(const uint64_t *__restrict__ group_start, uint32_t n_groups,
                                                          uint64_t total_bits, uint32_t *__restrict__ stream_words,
                                                          uint64_t n_words) {
    const uint64_t stride = (uint64_t)gridDim.x * SCAN_NT, t0 = (uint64_t)blockIdx.x * SCAN_NT + threadIdx.x;
    for (uint64_t g = t0; g < n_groups; g += stride) {
        const uint64_t a = group_start[g], b = group_start[g + 1];
        if (b > a && ((b - 1) >> 5) < n_words) {
            stream_words[a >> 5] = 0u;
            stream_words[(b - 1) >> 5] = 0u;
        }
    }
    for (uint64_t w = ((total_bits + 31) >> 5) + t0; w < n_words; w += stride) stream_words[w] = 0u;
}

__global__ void __launch_bounds__(GROUP_NT) enc_pack(const uint16_t *__restrict__ in, uint64_t n, const CodeTable ct,
                                                      const uint64_t *__restrict__ group_start, uint32_t n_groups,
                                                      uint32_t *__restrict__ stream_words, uint64_t n_words,
                                                      uint32_t buf_words) {
    extern __shared__ __align__(16) uint32_t s_dyn[];
    unsigned long long *s_lc = reinterpret_cast<unsigned long long *>(s_dyn);
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    uint32_t *buf = s_dyn + 512 + warp * buf_words;
    for (int i = threadIdx.x; i < 256; i += GROUP_NT) s_lc[i] = ct.lc[i];
    for (uint32_t i = lane; i < buf_words; i += 32) buf[i] = 0u;
    __syncthreads();
    const uint32_t wstride = gridDim.x * (GROUP_NT / 32);
    for (uint32_t g = blockIdx.x * (GROUP_NT / 32) + warp; g < n_groups; g += wstride) {
        const uint64_t gs0 = group_start[g], gs1 = group_start[g + 1];
        if (gs1 <= gs0) continue;  // warp-uniform
        const uint64_t base = (uint64_t)g * GROUP_W;
        const uint32_t sh0 = (uint32_t)(gs0 & 31u);
        uint32_t carry = sh0;
        const bool whole = base + GROUP_W <= n;
        for (uint32_t j = 0; j < 8; ++j) {
            uint32_t x0, x1;
            unsigned long long lc[8];
            uint32_t b = 0;
            if (whole) {  // every group but the tensor's last: eight weights, no checks
                exps8(__ldcs(reinterpret_cast<const uint4 *>(in + base + 8u * (32u * j + lane))), x0, x1);
#pragma unroll
                for (uint32_t k = 0; k < 8; ++k) {
                    lc[k] = s_lc[__byte_perm(k < 4 ? x0 : x1, 0u, 0x4440u + (k & 3u))];
                    b += (uint32_t)(lc[k] >> 32);
                }
            } else {
                const uint32_t cnt = load8(in, n, base + 8u * (32u * j + lane), x0, x1);
#pragma unroll
                for (uint32_t k = 0; k < 8; ++k) {
                    const uint32_t e = ((k < 4 ? x0 : x1) >> (8 * (k & 3))) & 0xFFu;
                    lc[k] = k < cnt ? s_lc[e] : 0ull;
                    b += (uint32_t)(lc[k] >> 32);
                }
            }
            uint32_t incl = b;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t y = __shfl_up_sync(FULL, incl, d);
                if (lane >= (uint32_t)d) incl += y;
            }
            const uint32_t off = carry + incl - b;  // bit offset in the warp's buffer
            carry += __shfl_sync(FULL, incl, 31);
            if (b && b <= 64u) {
                // almost every step: the 8 codewords fit 64 bits and are
                // placed with at most 3 ORs (one long codeword among short
                // ones no longer sends the lane down the general path)
                unsigned long long v = 0;
#pragma unroll
                for (uint32_t k = 0; k < 8; ++k) v = (v << (uint32_t)(lc[k] >> 32)) | (uint32_t)lc[k];
                const uint32_t sh = off & 31u, wi = off >> 5;
                const unsigned long long a = v << (64u - b);  // first bit at bit 63
                if (!enc_check(wi + ((sh + b + 31u) >> 5) <= buf_words, CK_ENC_PACK_BUF)) continue;
                atomicOr(buf + wi, (uint32_t)(a >> (32u + sh)));
                if (sh + b > 32u) atomicOr(buf + wi + 1, (uint32_t)(a >> sh));
                if (sh + b > 64u) atomicOr(buf + wi + 2, (uint32_t)(a << (32u - sh)));
            } else if (b) {
                unsigned long long acc = 0;
                uint32_t nacc = off & 31u, wi = off >> 5;
#pragma unroll
                for (uint32_t k = 0; k < 8; ++k) {
                    const uint32_t L = (uint32_t)(lc[k] >> 32);
                    if (!L) continue;
                    acc = (acc << L) | (uint32_t)lc[k];
                    nacc += L;
                    if (nacc >= 32u) {
                        if (enc_check(wi < buf_words, CK_ENC_PACK_BUF)) atomicOr(buf + wi, (uint32_t)(acc >> (nacc - 32u)));
                        ++wi;
                        nacc -= 32u;
                    }
                }
                if (nacc && enc_check(wi < buf_words, CK_ENC_PACK_BUF)) atomicOr(buf + wi, (uint32_t)(acc << (32u - nacc)));
            }
        }
        __syncwarp();
        uint32_t nw = (uint32_t)((sh0 + (gs1 - gs0) + 31u) >> 5);
        if (!enc_check(nw <= buf_words && (gs0 >> 5) + nw <= n_words, CK_ENC_PACK_STREAM)) nw = 0;
        uint32_t *dst = stream_words + (gs0 >> 5);
        for (uint32_t i = lane; i < nw; i += 32) {
            const uint32_t v = bswap32_dev(buf[i]);
            buf[i] = 0u;
            if (i == 0 || i + 1 == nw) atomicOr(dst + i, v);  // may be shared with a neighbouring group
            else dst[i] = v;
        }
        __syncwarp();
    }
}

}  // namespace
}  // namespace dfw

// ------------------------------------------------------------ host side

namespace dfw {
// Reads and clears the encoder kernels' check word (0 if none failed or the
// read fails).
uint32_t take_encoder_check_site() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_enc_check_site, sizeof(v)) != cudaSuccess) return 0u;
    if (cudaMemcpyToSymbol(g_enc_check_site, &zero, sizeof(zero)) != cudaSuccess) return 0u;
    return v;
}
}  // namespace dfw

namespace {

using namespace dfw;

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return sms;
}

bool misaligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace

extern "C" uint64_t dfw_encode_device_scratch_bytes(uint64_t n) {
    (void)n;
    return (sizeof(EncScratch) + 255) & ~(uint64_t)255;
}

namespace {

// One scope of the first call, in stages: prepare (host checks, no GPU work),
// pass 1 (histogram, read back into h_hist), code + passes 2 and 3 (totals
// read back into h_res), finish (host checks, table and info).  Between the
// stages the caller waits for the read-backs; dfw_encode_device_multi lets
// the GPU run the next scope's pass 1 meanwhile.
struct EncJob {
    const uint16_t *d_bf16;
    uint64_t n;
    int cap;
    uint8_t *d_mant;
    uint16_t *d_chunk_bits;
    uint64_t *d_group_start;
    EncScratch *sc;
    dfw_table *table;
    dfw_lanes_info *info;
    uint32_t fb;
    uint64_t n_groups;
    unsigned long long *h_hist;  // 256 counts (host)
    unsigned long long *h_res;   // total_bits, (max_group_bits << 32) | max_span (host)
};

dfw_status enc_prepare(EncJob &j, void *d_scratch, uint64_t scratch_bytes) {
    if (!j.table || !j.info || j.cap < 1 || j.cap > DFW_MAX_CAP) return DFW_EINVAL;
    j.fb = j.info->fast_bits;
    std::memset(j.table, 0, sizeof(*j.table));
    j.table->version = DFW_FORMAT_VERSION;
    j.table->cap = (uint32_t)j.cap;
    j.table->n = j.n;
    j.table->stream_bytes = stream_bytes_for(0);
    const uint64_t n_chunks = (j.n + LANE_SYMS - 1) / LANE_SYMS;
    j.n_groups = (n_chunks + GROUP_CHUNKS - 1) / GROUP_CHUNKS;
    if (n_chunks >= (1ull << 32)) return DFW_EINVAL;
    if (j.n == 0) return DFW_OK;
    if (!j.d_bf16 || !j.d_mant || !j.d_chunk_bits || !j.d_group_start || !d_scratch) return DFW_EINVAL;
    if (misaligned(j.d_bf16) || misaligned(j.d_mant) || misaligned(j.d_chunk_bits) || misaligned(j.d_group_start) ||
        misaligned(d_scratch))
        return DFW_EALIGN;
    if (scratch_bytes < sizeof(EncScratch)) return DFW_ENOMEM;
    j.sc = static_cast<EncScratch *>(d_scratch);
    return DFW_OK;
}

// An empty tensor: its plan (no groups) and group_start[0] = 0.
dfw_status enc_empty(EncJob &j, cudaStream_t s) {
    dfw_lanes_info q;
    std::memset(&q, 0, sizeof(q));
    q.fast_bits = j.fb;
    const dfw_status st = dfw_plan_lanes_query(j.table, &q);
    if (st != DFW_OK) return st;
    q.max_group_bytes = 16;
    *j.info = q;
    if (j.d_group_start && cudaMemsetAsync(j.d_group_start, 0, sizeof(uint64_t), s) != cudaSuccess)
        return DFW_ECUDA;
    return DFW_OK;
}

// pass 1: raw bytes and the exponent histogram, copied to h_hist
dfw_status enc_pass1(EncJob &j, int sms, cudaStream_t s) {
    if (cudaMemsetAsync(j.sc, 0, sizeof(EncScratch), s) != cudaSuccess) return DFW_ECUDA;
    const uint64_t want = ((j.n >> 3) + SPLIT_NT - 1) / SPLIT_NT, cap_blocks = (uint64_t)sms * 8;
    const unsigned blocks = (unsigned)std::max<uint64_t>(1, std::min(want, cap_blocks));
    enc_split_hist<<<blocks, SPLIT_NT, 0, s>>>(j.d_bf16, j.n, j.d_mant, dfw_mant_bytes(j.n), j.sc->hist);
    if (cudaGetLastError() != cudaSuccess) return DFW_ECUDA;
    if (cudaMemcpyAsync(j.h_hist, j.sc->hist, 256 * sizeof(unsigned long long), cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return DFW_ECUDA;
    return DFW_OK;
}

// the code, on the host, exactly as the host encoder builds it; then passes
// 2 and 3 (chunk bits, group totals -> group starts), totals copied to h_res
dfw_status enc_pass23(EncJob &j, int sms, cudaStream_t s) {
    uint64_t hist[256], sum = 0;
    int k = 0, only = 0;
    for (int b = 0; b < 256; ++b) {
        hist[b] = j.h_hist[b];
        sum += hist[b];
        if (hist[b]) {
            ++k;
            only = b;
        }
    }
    if (sum != j.n) return DFW_ECUDA;  // the histogram pass did not complete
    j.table->n_symbols = (uint32_t)k;
    j.table->single_symbol = k == 1 ? (uint32_t)only : 0u;
    const dfw_status st = code_lengths(hist, j.cap, j.table->len);
    if (st != DFW_OK) return st;
    LenTable lt;
    std::memcpy(lt.len, j.table->len, 256);
    const uint64_t want = (j.n_groups + GROUP_NT / 32 - 1) / (GROUP_NT / 32), cap_blocks = (uint64_t)sms * 4;
    enc_chunk_bits<<<(unsigned)std::min(want, cap_blocks), GROUP_NT, 0, s>>>(j.d_bf16, j.n, lt, j.d_chunk_bits,
                                                                             j.d_group_start, (uint32_t)j.n_groups);
    if (cudaGetLastError() != cudaSuccess) return DFW_ECUDA;
    // pass 3: ranges of whole tiles, at most SCAN_CTAS of them
    uint64_t range = (j.n_groups + SCAN_CTAS - 1) / SCAN_CTAS;
    range = (range + SCAN_NT - 1) / SCAN_NT * SCAN_NT;
    const unsigned ctas = (unsigned)((j.n_groups + range - 1) / range);
    enc_range_totals<<<ctas, SCAN_NT, 0, s>>>(j.d_group_start, (uint32_t)j.n_groups, (uint32_t)range, j.sc);
    if (cudaGetLastError() != cudaSuccess) return DFW_ECUDA;
    enc_range_scan<<<ctas, SCAN_NT, 0, s>>>(j.d_group_start, (uint32_t)j.n_groups, (uint32_t)range, j.sc);
    if (cudaGetLastError() != cudaSuccess) return DFW_ECUDA;
    if (cudaMemcpyAsync(j.h_res, &j.sc->total_bits, 2 * sizeof(unsigned long long), cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return DFW_ECUDA;
    return DFW_OK;
}

dfw_status enc_finish(EncJob &j) {
    uint64_t expect = 0;
    for (int b = 0; b < 256; ++b) expect += (uint64_t)j.h_hist[b] * j.table->len[b];
    if (j.h_res[0] != expect) return DFW_ECUDA;  // the counting passes disagree with the histogram
    j.table->total_bits = j.h_res[0];
    j.table->stream_bytes = stream_bytes_for(j.h_res[0]);
    dfw_lanes_info q;
    std::memset(&q, 0, sizeof(q));
    q.fast_bits = j.fb;
    const dfw_status st = dfw_plan_lanes_query(j.table, &q);
    if (st != DFW_OK) return st;
    q.max_group_bytes = std::max<uint32_t>(16u, (uint32_t)(j.h_res[1] & 0xFFFFFFFFull));
    *j.info = q;
    return DFW_OK;
}

}  // namespace

extern "C" dfw_status dfw_encode_device(const uint16_t *d_bf16, uint64_t n, int cap, uint8_t *d_mant,
                                        uint16_t *d_chunk_bits, uint64_t *d_group_start, void *d_scratch,
                                        uint64_t scratch_bytes, dfw_table *table, dfw_lanes_info *info,
                                        void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_encode_device");
    unsigned long long h_hist[256], h_res[2];
    EncJob j{d_bf16, n, cap, d_mant, d_chunk_bits, d_group_start, nullptr, table, info, 0, 0, h_hist, h_res};
    dfw_status st = enc_prepare(j, d_scratch, scratch_bytes);
    if (st != DFW_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    if (n == 0) return enc_empty(j, s);
    const int sms = device_sms();
    if (sms <= 0) return DFW_ECUDA;
    if ((st = enc_pass1(j, sms, s)) != DFW_OK) return st;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DFW_ECUDA;
    if ((st = enc_pass23(j, sms, s)) != DFW_OK) return st;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DFW_ECUDA;
    return enc_finish(j);
}

extern "C" uint64_t dfw_encode_device_multi_staging_bytes(uint32_t k) {
    return (uint64_t)k * 258u * sizeof(unsigned long long);
}

extern "C" dfw_status dfw_encode_device_multi(uint32_t k, const dfw_encode_scope *scopes, int cap, void *d_scratch,
                                              uint64_t scratch_bytes, void *h_staging, uint64_t staging_bytes,
                                              dfw_table *tables, dfw_lanes_info *infos, void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_encode_device_multi");
    if (k == 0) return DFW_OK;
    if (!scopes || !tables || !infos || !h_staging) return DFW_EINVAL;
    if ((reinterpret_cast<uintptr_t>(h_staging) & 7u) != 0) return DFW_EALIGN;
    if (staging_bytes < dfw_encode_device_multi_staging_bytes(k)) return DFW_ENOMEM;
    const uint64_t per = dfw_encode_device_scratch_bytes(0);
    if (scratch_bytes / per < k) return DFW_ENOMEM;
    // every scope checked before anything is launched
    std::vector<EncJob> jobs(k);
    unsigned long long *stage = static_cast<unsigned long long *>(h_staging);
    for (uint32_t i = 0; i < k; ++i) {
        const dfw_encode_scope &c = scopes[i];
        jobs[i] = EncJob{c.d_bf16, c.n, cap, c.d_mant, c.d_chunk_bits, c.d_group_start, nullptr, tables + i,
                         infos + i, 0, 0, stage + 258u * i, stage + 258u * i + 256u};
        void *sc_i = d_scratch ? static_cast<unsigned char *>(d_scratch) + per * i : nullptr;
        const dfw_status st = enc_prepare(jobs[i], sc_i, per);
        if (st != DFW_OK) return st;
    }
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    const int sms = device_sms();
    if (sms <= 0) return DFW_ECUDA;
    cudaEvent_t ev[2] = {nullptr, nullptr};
    if (cudaEventCreateWithFlags(&ev[0], cudaEventDisableTiming) != cudaSuccess) return DFW_ECUDA;
    if (cudaEventCreateWithFlags(&ev[1], cudaEventDisableTiming) != cudaSuccess) {
        cudaEventDestroy(ev[0]);
        return DFW_ECUDA;
    }
    // Stream order: pass 1 of scope i + 1 is queued before the host waits
    // for scope i's histogram, so the GPU has it to run while the host
    // builds scope i's code and queues its passes 2 and 3.
    auto start = [&](uint32_t i) -> dfw_status {
        if (jobs[i].n == 0) return enc_empty(jobs[i], s);
        const dfw_status st = enc_pass1(jobs[i], sms, s);
        if (st != DFW_OK) return st;
        return cudaEventRecord(ev[i & 1u], s) == cudaSuccess ? DFW_OK : DFW_ECUDA;
    };
    dfw_status st = start(0);
    for (uint32_t i = 0; i < k && st == DFW_OK; ++i) {
        if (i + 1 < k && (st = start(i + 1)) != DFW_OK) break;
        if (jobs[i].n == 0) continue;
        if (cudaEventSynchronize(ev[i & 1u]) != cudaSuccess) {
            st = DFW_ECUDA;
            break;
        }
        st = enc_pass23(jobs[i], sms, s);
    }
    // all queued work ends before the call returns, on success or not
    if (cudaStreamSynchronize(s) != cudaSuccess && st == DFW_OK) st = DFW_ECUDA;
    cudaEventDestroy(ev[0]);
    cudaEventDestroy(ev[1]);
    for (uint32_t i = 0; i < k && st == DFW_OK; ++i)
        if (jobs[i].n) st = enc_finish(jobs[i]);
    return st;
}

extern "C" dfw_status dfw_pack_device(const uint16_t *d_bf16, const dfw_table *table, const dfw_lanes_info *info,
                                      const uint64_t *d_group_start, uint8_t *d_stream, uint64_t stream_capacity,
                                      void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_pack_device");
    dfw_status st = validate_table(table);
    if (st != DFW_OK) return st;
    if (!info || !d_stream) return DFW_EINVAL;
    if (stream_capacity < table->stream_bytes) return DFW_ENOMEM;
    const uint64_t n = table->n;
    const uint64_t n_chunks = (n + LANE_SYMS - 1) / LANE_SYMS;
    const uint64_t n_groups = (n_chunks + GROUP_CHUNKS - 1) / GROUP_CHUNKS;
    if (info->n_groups != n_groups || info->max_group_bytes < 16 || info->max_group_bytes > 64u * 1024u)
        return DFW_EINVAL;
    if (misaligned(d_stream) || (n && (misaligned(d_bf16) || misaligned(d_group_start)))) return DFW_EALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    if (table->total_bits == 0)  // zero or one distinct exponent: no bits, the stream is its padding
        return cudaMemsetAsync(d_stream, 0, table->stream_bytes, s) == cudaSuccess ? DFW_OK : DFW_ECUDA;
    if (!d_bf16 || !d_group_start) return DFW_EINVAL;
    const int sms = device_sms();
    if (sms <= 0) return DFW_ECUDA;
    {
        const uint64_t want = (n_groups + SCAN_NT - 1) / SCAN_NT, cap_blocks = (uint64_t)sms * 8;
        enc_zero_edges<<<(unsigned)std::max<uint64_t>(1, std::min(want, cap_blocks)), SCAN_NT, 0, s>>>(
            d_group_start, (uint32_t)n_groups, table->total_bits, reinterpret_cast<uint32_t *>(d_stream),
            table->stream_bytes / 4);
        if (cudaGetLastError() != cudaSuccess) return DFW_ECUDA;
    }
    uint32_t code[256];
    canonical_codes(table->len, code);
    CodeTable ct;
    for (int b = 0; b < 256; ++b) ct.lc[b] = ((unsigned long long)table->len[b] << 32) | code[b];
    const uint32_t buf_words = info->max_group_bytes / 4 + 2;
    const size_t smem = 2048 + (size_t)(GROUP_NT / 32) * buf_words * 4;
    if (smem > 227u * 1024u) return DFW_EINVAL;
    if (cudaFuncSetAttribute(enc_pack, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
        return DFW_ECUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, enc_pack, GROUP_NT, smem) != cudaSuccess) return DFW_ECUDA;
    const uint64_t want = (n_groups + GROUP_NT / 32 - 1) / (GROUP_NT / 32);
    const uint64_t cap_blocks = (uint64_t)sms * (uint64_t)std::max(1, per_sm);
    enc_pack<<<(unsigned)std::min(want, cap_blocks), GROUP_NT, smem, s>>>(
        d_bf16, n, ct, d_group_start, (uint32_t)n_groups, reinterpret_cast<uint32_t *>(d_stream),
        table->stream_bytes / 4, buf_words);
    return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
}

// ------------------------------------------------------------ no-allocation variant
//
// For callers that cannot allocate device memory where they encode: the
// scratch of the first call lives in an array compiled into the library
// instead of a caller buffer.  One array per device that loads the library,
// held until the process exits; every call shares it (dfw_encode_device
// clears it first), so calls whose GPU work overlaps race on it.

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DFW_NOALLOC_SCRATCH_BYTES];

constexpr int NOALLOC_MAX_DEVICES = 64;
void *g_noalloc_ptr[NOALLOC_MAX_DEVICES] = {nullptr};
std::mutex g_noalloc_mu;

// The array's device address on the current device; looked up (and cached)
// on the first call there.  The cache is never invalidated: a context
// destroyed and re-created in the same process (cudaDeviceReset) would leave
// a stale address, which is why such a reset is documented as unsupported.
dfw_status noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES) return DFW_ECUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DFW_ECUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return DFW_OK;
}

}  // namespace

extern "C" dfw_status dfw_encode_device_noalloc(const uint16_t *d_bf16, uint64_t n, int cap, uint8_t *d_mant,
                                                uint16_t *d_chunk_bits, uint64_t *d_group_start, dfw_table *table,
                                                dfw_lanes_info *info, void *cuda_stream) {
    if (dfw_encode_device_scratch_bytes(n) > DFW_NOALLOC_SCRATCH_BYTES) return DFW_ENOMEM;
    void *scratch = nullptr;
    const dfw_status st = noalloc_scratch(&scratch);
    if (st != DFW_OK) return st;
    return dfw_encode_device(d_bf16, n, cap, d_mant, d_chunk_bits, d_group_start, scratch,
                             DFW_NOALLOC_SCRATCH_BYTES, table, info, cuda_stream);
}
