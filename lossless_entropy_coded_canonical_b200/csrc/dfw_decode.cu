// dfw_decode.cu -- device half of libdfw: the sm_100a decode kernels.
//
// Source: DFloat11 abstract ("70% Size, 100% Accuracy: Lossless LLM
// Compression for Efficient GPU Inference via Dynamic-Length Float"): compact
// LUTs in GPU SRAM, a two-phase kernel that coordinates thread read/write
// positions through lightweight auxiliary arrays, block-level decompression,
// bit-exact output.  This kernel is written for B200 from that description.
//
// Persistent CTAs (grid = SMs x resident CTAs) load the fast table into
// shared memory once, then loop over tiles of T windows of W stream bytes
// (one window per thread).  Tiles are double-buffered: while tile i is
// decoded, one thread has already started TMA bulk copies (cp.async.bulk,
// completion on an mbarrier, no multicast) of the next tile's stream bytes,
// gap bytes and raw-byte range into the other buffer.  Per tile:
//   phase 1  each thread decodes the codewords that start in its window; one
//            fast-table lookup yields up to four whole codewords; symbols go
//            through a 64-bit register accumulator into the thread's own
//            word slots (interleaved by thread: conflict-free stores)
//   scan     warp shuffle scan of the counts; one CTA barrier publishes the
//            warp totals, and every warp scans those itself (no second
//            barrier); the tile total must equal out_start[b+1] - out_start[b]
//   phase 2  each thread joins its symbols with their raw bytes (both read a
//            word at a time, funnel-shifted to the output's alignment) into
//            bf16 in a shared staging buffer in output order
//   store    each warp bulk-stores its output range from the staging buffer
//            with one TMA store (cp.async.bulk shared -> global); the <= 7
//            weights at either unaligned end are stored one by one.  Before
//            the next tile writes the staging buffer, each warp waits until
//            its store has read it (bulk wait_group.read), then the CTA
//            barrier orders all warps.
//
// Bounds: every lookup advances at least one bit and a walk stops at its
// window end, so loops end whatever the data; tables are validated once per
// CTA; waits on bulk copies give up after a time limit (status bit, early
// return); a tile whose counts or ranges disagree writes nothing and sets a
// bit of the device status word.  Nothing waits on another CTA.
#include <cuda_runtime.h>

#include "dfw_internal.h"

namespace dfw {
__device__ unsigned int g_status;      // device status word (sticky error bits)
__device__ unsigned int g_check_site;  // checks build: the first range check that failed (0: none)
}

#include "dfw_device.cuh"
#include "dfw_lanes.cuh"
#include "dfw_rans.cuh"

namespace dfw {
namespace {

// Phase 1 for one window held as NSEG big-endian words plus a guard word:
// decodes the codewords starting in [p, wend) and appends their symbols to
// the thread's word slots wp[0], wp[NT], ...  Returns the codeword count.
// A final lookup that crosses wend appends all its symbols but counts only
// the codewords that start before wend (the extra bytes are never read).
template <int NSEG, int NT>
__device__ __forceinline__ uint32_t decode_window(const uint32_t (&wd)[NSEG + 1], int p, const int wend,
                                                  const uint2 *__restrict__ s_fast, const uint32_t kshift,
                                                  const uint32_t *__restrict__ g_hier, uint32_t n_tables,
                                                  uint32_t *__restrict__ wp, uint32_t &err) {
    uint32_t *const wp0 = wp;
    uint32_t lo = 0u, hi = 0u, sh = 0u, extra = 0u;
#pragma unroll
    for (int seg = 0; seg < NSEG; ++seg) {
        const uint32_t a = wd[seg], b = wd[seg + 1];
        const int seg_end = min(32 * (seg + 1), wend);
        while (p < seg_end) {
            const uint32_t x = __funnelshift_l(b, a, (uint32_t)p);  // stream bits [p, p + 32)
            const uint2 e = s_fast[x >> kshift];
            uint32_t syms = e.x, c8 = __byte_perm(e.y, 0u, 0x4441);
            int pn = p + (int)(e.y & 255u);
            if (pn > wend) {
                if (e.y & FAST_ESC) {
                    const uint32_t f = resolve_escape(x, g_hier, n_tables);
                    if (f & ESC_BAD) err |= ST_LUT;
                    syms = rot_sym(f);
                    c8 = 8u;
                    pn = p + (int)((f >> LUT_LEN_SHIFT) & 63u);
                } else {
                    // codeword 0 starts at p < wend; codeword k+1 starts where k
                    // ends, so it counts if that end offset is below wend - p
                    const uint32_t ends = (e.y >> FAST_ENDS_SHIFT) & 0xFFFu;
                    const uint32_t r = (uint32_t)(wend - p);
                    const uint32_t t8 = min(c8, 8u + 8u * (uint32_t)__popc(ends & ((1u << (r - 1u)) - 1u)));
                    extra = c8 - t8;
                }
            }
            lo |= syms << sh;
            hi |= __funnelshift_l(syms, 0u, sh);
            sh += c8;
            const bool full = sh >= 32u;
            if (full) *wp = lo;
            wp += full ? NT : 0;
            lo = full ? hi : lo;
            hi = full ? 0u : hi;
            sh &= 31u;
            p = pn;
        }
    }
    if (sh) *wp = lo;
    const uint32_t words = (uint32_t)(wp - wp0) / NT;  // full words flushed
    return (32u * words + sh - extra) >> 3;
}

struct Params {
    const uint8_t *stream;
    const uint8_t *mant;
    const uint32_t *lut;
    const uint8_t *gap;
    const uint64_t *out_start;
    uint16_t *out;
    uint64_t total_bits, stream_bytes, n_windows, n_tiles, n;
    uint32_t fast_bits, n_tables;
    uint32_t ebuf_bytes;  // staging entries (>= max tile symbols + 16); 2 bytes each
    uint32_t mbuf_bytes;  // raw-byte buffer per slot (>= max tile symbols + 32)
};

// Shared memory: fast table | scan slots | 2 mbarriers | word slots |
// bf16 staging | 2 x (stream bytes | gap bytes | raw bytes).
template <int W, int NT>
struct Layout {
    static constexpr uint32_t PRIV_WORDS = 2 * W + 1;  // 8W + 4 bytes: a window's worst case
    static constexpr uint32_t SBUF = NT * W + 16;      // a tile's stream bytes + guard
    uint32_t fast, scan, mbar, priv, ebuf, slot0, slot_bytes, total;
    __host__ __device__ Layout(uint32_t fast_bits, uint32_t ebuf_bytes, uint32_t mbuf_bytes) {
        fast = 0;
        scan = 8u << fast_bits;
        mbar = scan + 64 * 4;
        priv = mbar + 16;
        ebuf = priv + 4 * PRIV_WORDS * NT;
        slot0 = ebuf + 2 * ebuf_bytes;  // staging: 2 bytes per tile-buffer entry
        slot_bytes = SBUF + NT + mbuf_bytes;
        total = slot0 + 2 * slot_bytes;
    }
};

template <int W, int NT>
__global__ void __launch_bounds__(NT) decode_tiles(const Params prm) {
    constexpr int NSEG = W / 4;
    constexpr int NWARP = NT / 32;
    using L = Layout<W, NT>;
    static_assert(NWARP <= 32, "block scan assumes at most 32 warps");
    extern __shared__ __align__(16) uint8_t smem[];
    const L lay(prm.fast_bits, prm.ebuf_bytes, prm.mbuf_bytes);
    const uint32_t n_fast = 1u << prm.fast_bits;
    uint2 *s_fast = reinterpret_cast<uint2 *>(smem + lay.fast);
    uint32_t *s_scan = reinterpret_cast<uint32_t *>(smem + lay.scan);
    uint32_t *s_priv = reinterpret_cast<uint32_t *>(smem + lay.priv);
    uint8_t *ebuf = smem + lay.ebuf;
    const uint32_t bar0 = smem_u32(smem + lay.mbar);
    const uint32_t *g_hier = prm.lut + 2u * n_fast;
    const uint32_t kshift = 32u - prm.fast_bits;
    const uint64_t tile_bytes = (uint64_t)NT * W;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // Starts the copies of tile t's bytes into slot s (thread 0 only). A tile
    // whose out_start range is out of bounds copies no raw bytes; the consumer
    // rejects it by the same test.
    auto issue = [&](uint64_t t, uint32_t s, uint64_t os, uint64_t oe) {
        uint8_t *slot = smem + lay.slot0 + s * lay.slot_bytes;
        const uint64_t sb0 = t * tile_bytes;
        const uint32_t sbytes = (uint32_t)min((uint64_t)L::SBUF, prm.stream_bytes - sb0);
        const bool ok = oe >= os && oe <= prm.n && oe - os + 32 <= prm.mbuf_bytes;
        const uint64_t m0 = os & ~15ull, m1 = (oe + 15) & ~15ull;
        uint32_t mbytes = ok ? (uint32_t)(m1 - m0) : 0u;
        const bool cp_ok = check(t < prm.n_tiles && sb0 < prm.stream_bytes && sbytes <= L::SBUF, CK_TILES_COPY);
        if (!check(mbytes <= prm.mbuf_bytes && (mbytes == 0u || m1 <= ((prm.n + 15) & ~15ull)), CK_TILES_COPY))
            mbytes = 0u;
        fence_proxy_async();
        mbar_expect_tx(bar0 + 8 * s, (cp_ok ? sbytes + NT : 0u) + mbytes);
        if (cp_ok) {
            bulk_load(smem_u32(slot), prm.stream + sb0, sbytes, bar0 + 8 * s);
            bulk_load(smem_u32(slot + L::SBUF), prm.gap + t * NT, NT, bar0 + 8 * s);
        }
        if (mbytes) bulk_load(smem_u32(slot + L::SBUF + NT), prm.mant + m0, mbytes, bar0 + 8 * s);
    };

    if (tid == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        fence_mbar_init();
    }
    // fast table into shared memory, each entry checked once per CTA
    bool bad = false;
    for (uint32_t i = tid; i < n_fast; i += NT) {
        const uint2 e = __ldg(reinterpret_cast<const uint2 *>(prm.lut) + i);
        if (e.y & FAST_ESC) {
            bad |= e.y != FAST_ESC_WORD || e.x != 0u;
        } else {
            const uint32_t cb = e.y & 255u, c8 = (e.y >> FAST_C8_SHIFT) & 255u,
                           ends = (e.y >> FAST_ENDS_SHIFT) & 0xFFFu;
            bad |= c8 == 0u || (c8 & 7u) || c8 > 8u * FAST_MAX_SYMS || cb == 0u || cb > prm.fast_bits ||
                   8u * cb < c8 || (uint32_t)__popc(ends) * 8u != c8 || (ends >> (cb - 1u)) != 1u ||
                   (e.y & 0x70000000u) || (c8 < 32u && (e.x >> c8) != 0u);
        }
        s_fast[i] = e;
    }
    uint64_t tile = blockIdx.x;
    uint64_t os = 0, oe = 0;
    if (tile < prm.n_tiles) {
        os = __ldg(prm.out_start + tile);
        oe = __ldg(prm.out_start + tile + 1);
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0) atomicOr(&g_status, ST_LUT);
        return;
    }
    if (tid == 0 && tile < prm.n_tiles) issue(tile, 0, os, oe);

    for (uint32_t k = 0; tile < prm.n_tiles; ++k) {
        const uint32_t s = k & 1u;
        const uint8_t *slot = smem + lay.slot0 + s * lay.slot_bytes;
        const uint64_t next = tile + gridDim.x;
        uint64_t nos = 0, noe = 0;
        if (next < prm.n_tiles) {  // next tile's output range, needed after the first barrier
            nos = __ldg(prm.out_start + next);
            noe = __ldg(prm.out_start + next + 1);
        }
        const bool waited = mbar_wait_bounded(bar0 + 8 * s, (k >> 1) & 1u);
        if (lane == 0) bulk_wait_read();  // this warp's last store has read the staging buffer
        const bool valid = oe >= os && oe <= prm.n && oe - os + 32 <= prm.mbuf_bytes &&
                           oe - os + 16 <= prm.ebuf_bytes;  // uniform across the CTA

        // phase 1: decode this thread's window into its word slots
        const uint64_t w = tile * NT + tid;
        uint32_t cnt = 0, err = 0;
        if (valid && waited && w < prm.n_windows) {
            uint32_t wd[NSEG + 1];
            const uint8_t *src = slot + tid * W;
            if constexpr (W == 8) {
                const uint2 v = *reinterpret_cast<const uint2 *>(src);
                wd[0] = bswap32(v.x);
                wd[1] = bswap32(v.y);
            } else {
                const uint4 v = *reinterpret_cast<const uint4 *>(src);
                wd[0] = bswap32(v.x);
                wd[1] = bswap32(v.y);
                wd[2] = bswap32(v.z);
                wd[3] = bswap32(v.w);
            }
            wd[NSEG] = bswap32(*reinterpret_cast<const uint32_t *>(src + W));
            const int p = slot[L::SBUF + tid];
            const uint64_t rem = prm.total_bits - w * (8ull * W);
            const int wend = rem < 8ull * W ? (int)rem : 8 * W;
            cnt = decode_window<NSEG, NT>(wd, p, wend, s_fast, kshift, g_hier, prm.n_tables, s_priv + tid, err);
            if (!check(cnt <= 4u * L::PRIV_WORDS, CK_TILES_WINDOW)) cnt = 0;
            if (err) atomicOr(&g_status, err);
        }

        // scan: warp shuffles; the warp totals go through shared memory
        uint32_t *scan = s_scan + (s ? 32 : 0);
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        if (lane == 31) scan[warp] = incl;
        if (!__syncthreads_and(waited)) {  // a bulk copy never completed: give up
            if (tid == 0) {
                atomicOr(&g_status, ST_TIMEOUT);
                mbar_wait_bounded(bar0 + 8 * s, (k >> 1) & 1u);  // let an in-flight copy land first
            }
            if (lane == 0) bulk_wait_all();
            return;
        }
        // every thread is past the previous tile: its slot can take the next one
        if (tid == 0 && next < prm.n_tiles) issue(next, s ^ 1u, nos, noe);
        // each warp scans the warp totals itself
        uint32_t v = lane < NWARP ? scan[lane] : 0u;
#pragma unroll
        for (int d = 1; d < NWARP; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, v, d);
            if (lane >= d) v += y;
        }
        const uint32_t total = __shfl_sync(0xFFFFFFFFu, v, NWARP - 1);
        const uint32_t wbase = warp ? __shfl_sync(0xFFFFFFFFu, v, (warp - 1) & 31) : 0u;
        const uint32_t wcount = __shfl_sync(0xFFFFFFFFu, incl, 31);
        const uint32_t excl = wbase + incl - cnt;
        const uint32_t count = (uint32_t)(oe - os);
        if (!valid || total != count) {  // the same decision in every warp
            if (tid == 0) atomicOr(&g_status, valid ? ST_COUNT : ST_RANGE);
        } else {
            // phase 2: join into the staging buffer; st[i] holds weight (os & ~15) + i
            uint16_t *st = reinterpret_cast<uint16_t *>(ebuf);
            const uint8_t *mb = slot + L::SBUF + NT;
            const uint32_t b16 = (uint32_t)(os & 15u);
            if (cnt && check(b16 + excl + cnt <= prm.ebuf_bytes && b16 + excl + cnt <= prm.mbuf_bytes, CK_TILES_WINDOW)) {
                const uint32_t d = b16 + excl;
                const uint32_t *src = s_priv + tid;
                const uint32_t h = min((4u - (d & 3u)) & 3u, cnt);
                uint32_t cur = src[0];
                for (uint32_t i = 0; i < h; ++i) st[d + i] = join1((cur >> (8u * i)) & 0xFFu, mb[d + i]);
                const uint32_t nbody = (cnt - h) >> 2;
                const uint32_t s8 = 8u * h;
                const uint32_t q0 = d + h;  // multiple of 4
                for (uint32_t j = 0; j < nbody; ++j) {
                    const uint32_t nxt = src[(j + 1) * NT];
                    const uint32_t E = __funnelshift_r(cur, nxt, s8);
                    const uint32_t M = *reinterpret_cast<const uint32_t *>(mb + q0 + 4u * j);
                    uint2 r;
                    join4(E, M, r.x, r.y);
                    *reinterpret_cast<uint2 *>(st + q0 + 4u * j) = r;
                    cur = nxt;
                }
                const uint32_t rem = cnt - h - 4u * nbody;  // 0..3 weights left
                if (rem) {
                    const uint32_t t = __funnelshift_r(cur, src[(nbody + 1) * NT], s8);
                    const uint32_t i0 = q0 + 4u * nbody;
                    for (uint32_t i = 0; i < rem; ++i) st[i0 + i] = join1((t >> (8u * i)) & 0xFFu, mb[i0 + i]);
                }
            }
            fence_proxy_async();  // these writes before the warp's bulk store reads them
            __syncwarp();

            // store: the warp's range [lo_i, hi_i) of local indices; ot[i] is weight (os & ~15) + i
            uint16_t *ot = prm.out + (os & ~15ull);
            const uint32_t lo_i = b16 + wbase;
            uint32_t hi_i = lo_i + wcount;
            if (!check((os & ~15ull) + hi_i <= prm.n, CK_TILES_STORE)) hi_i = lo_i;
            const uint32_t A = (lo_i + 7u) & ~7u, B = hi_i & ~7u;  // 16-byte aligned interior
            if (lane == 0 && B > A) bulk_store(ot + A, smem_u32(st + A), 2u * (B - A));
            if (lane < 8) {
                const uint32_t i = lo_i + lane;
                if (i < min(A, hi_i)) ot[i] = st[i];
            } else if (lane < 16) {
                const uint32_t i = max(B, A) + (lane - 8);
                if (i < hi_i) ot[i] = st[i];
            }
        }
        os = nos;
        oe = noe;
        tile = next;
    }
    if (lane == 0) bulk_wait_all();
}

typedef void (*decode_fn)(const Params);

struct Variant {
    uint32_t W, T;
    decode_fn fn;
    int smem_set[16];  // dynamic shared memory opted in, per device
};

Variant g_variants[] = {
    {8, 128, decode_tiles<8, 128>, {0}},   {8, 256, decode_tiles<8, 256>, {0}},
    {8, 512, decode_tiles<8, 512>, {0}},   {16, 128, decode_tiles<16, 128>, {0}},
    {16, 256, decode_tiles<16, 256>, {0}},
};

int g_sms[16];

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int W, int NT>
uint32_t smem_bytes(uint32_t fb, uint32_t ebuf, uint32_t mbuf) {
    return Layout<W, NT>(fb, ebuf, mbuf).total;
}

uint32_t variant_smem(const Variant &v, uint32_t fb, uint32_t ebuf, uint32_t mbuf) {
    switch (v.W * 1000 + v.T) {
        case 8128: return smem_bytes<8, 128>(fb, ebuf, mbuf);
        case 8256: return smem_bytes<8, 256>(fb, ebuf, mbuf);
        case 8512: return smem_bytes<8, 512>(fb, ebuf, mbuf);
        case 16128: return smem_bytes<16, 128>(fb, ebuf, mbuf);
        default: return smem_bytes<16, 256>(fb, ebuf, mbuf);
    }
}

}  // namespace

dfw_status launch_decode(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                         const uint8_t *d_gap, const uint64_t *d_out_start, const dfw_table *table,
                         const dfw_plan_info *info, uint16_t *d_out, cudaStream_t s) {
    dfw_status st = validate_table(table);
    if (st != DFW_OK) return st;
    if (!info || !plan_shape_supported(info->window_bytes, info->tile_windows)) return DFW_EINVAL;
    const uint64_t n = table->n;
    const uint64_t wbits = 8ull * info->window_bytes;
    if (info->n_windows != (table->total_bits + wbits - 1) / wbits ||
        info->n_tiles != (info->n_windows + info->tile_windows - 1) / info->tile_windows)
        return DFW_EINVAL;
    if (n == 0) return DFW_OK;
    if (!d_mant || !d_out) return DFW_EINVAL;
    if (!aligned16(d_mant) || !aligned16(d_out)) return DFW_EALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return DFW_ECUDA;
    if (!g_sms[dev] && cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DFW_ECUDA;
    if (table->total_bits == 0) {
        const uint64_t want = ((n >> 3) + 256) / 256;
        const uint64_t cap = (uint64_t)g_sms[dev] * 8;
        fill_single<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(d_mant, table->single_symbol, n, d_out);
        return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
    }
    if (!d_stream || !d_lut || !d_gap || !d_out_start) return DFW_EINVAL;
    if (!aligned16(d_stream) || !aligned16(d_lut) || !aligned16(d_out_start) || !aligned16(d_gap))
        return DFW_EALIGN;
    const uint32_t fb = info->fast_bits;
    if (fb < (uint32_t)FAST_BITS_MIN || fb > (uint32_t)FAST_BITS_MAX || info->lut_tables < 1 ||
        info->lut_words != (2u << fb) + 256u * info->lut_tables)
        return DFW_EINVAL;
    if (info->max_tile_symbols > 8ull * info->window_bytes * info->tile_windows) return DFW_EINVAL;
    if (table->stream_bytes & 15u) return DFW_EINVAL;
    Variant *v = nullptr;
    for (auto &x : g_variants)
        if (x.W == info->window_bytes && x.T == info->tile_windows) v = &x;
    if (!v) return DFW_EINVAL;
    Params prm;
    prm.stream = d_stream;
    prm.mant = d_mant;
    prm.lut = d_lut;
    prm.gap = d_gap;
    prm.out_start = d_out_start;
    prm.out = d_out;
    prm.total_bits = table->total_bits;
    prm.stream_bytes = table->stream_bytes;
    prm.n_windows = info->n_windows;
    prm.n_tiles = info->n_tiles;
    prm.n = n;
    prm.fast_bits = fb;
    prm.n_tables = info->lut_tables;
    prm.ebuf_bytes = (uint32_t)((info->max_tile_symbols + 16 + 15) & ~15ull);
    prm.mbuf_bytes = (uint32_t)((info->max_tile_symbols + 32 + 15) & ~15ull);
    const uint32_t smem = variant_smem(*v, fb, prm.ebuf_bytes, prm.mbuf_bytes);
    if (!v->smem_set[dev]) {
        if (cudaFuncSetAttribute(v->fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
            return DFW_ECUDA;
        v->smem_set[dev] = 1;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v->fn, (int)v->T, smem) != cudaSuccess)
        return DFW_ECUDA;
    if (per_sm < 1) return DFW_EINVAL;
    const uint64_t slots = (uint64_t)per_sm * g_sms[dev];
    const unsigned grid = (unsigned)(info->n_tiles < slots ? info->n_tiles : slots);
    v->fn<<<grid, v->T, smem, s>>>(prm);
    return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
}

}  // namespace dfw

using namespace dfw;

extern "C" dfw_status dfw_decode(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                                 const uint8_t *d_gap, const uint64_t *d_out_start, const dfw_table *table,
                                 const dfw_plan_info *info, uint16_t *d_out, void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_decode");
    return launch_decode(d_stream, d_mant, d_lut, d_gap, d_out_start, table, info, d_out,
                         static_cast<cudaStream_t>(cuda_stream));
}

extern "C" dfw_status dfw_decode_block(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                                       const uint8_t *d_gap, const uint64_t *d_out_start,
                                       const dfw_table *table, const dfw_plan_info *info,
                                       const uint64_t *tensor_offsets, int k, uint16_t *d_scratch,
                                       uint64_t scratch_elems, void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_decode_block");
    if (!table || !tensor_offsets || k < 1) return DFW_EINVAL;
    if (tensor_offsets[0] != 0 || tensor_offsets[k] != table->n) return DFW_EINVAL;
    for (int i = 0; i < k; ++i)
        if (tensor_offsets[i + 1] < tensor_offsets[i]) return DFW_EINVAL;
    if (scratch_elems < table->n) return DFW_ENOMEM;
    return launch_decode(d_stream, d_mant, d_lut, d_gap, d_out_start, table, info, d_scratch,
                         static_cast<cudaStream_t>(cuda_stream));
}

extern "C" dfw_status dfw_decode_lanes(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                                       const uint16_t *d_chunk_bits, const uint64_t *d_group_start,
                                       const dfw_table *table, const dfw_lanes_info *info, uint16_t *d_out,
                                       void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_decode_lanes");
    dfw_status st = validate_table(table);
    if (st != DFW_OK) return st;
    if (!info) return DFW_EINVAL;
    const uint64_t n = table->n;
    if (n == 0) return DFW_OK;
    if (!d_mant || !d_out) return DFW_EINVAL;
    if ((reinterpret_cast<uintptr_t>(d_mant) | reinterpret_cast<uintptr_t>(d_out)) & 15u) return DFW_EALIGN;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DFW_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    if (table->total_bits == 0) {
        const uint64_t want = ((n >> 3) + 256) / 256, cap = (uint64_t)sms * 8;
        fill_single<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(d_mant, table->single_symbol, n, d_out);
        return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
    }
    return launch_decode_lanes(d_stream, d_mant, d_lut, d_chunk_bits, d_group_start, table, info, d_out, s, sms);
}

extern "C" dfw_status dfw_decode_lanes_seq(int k, const dfw_lanes_scope *scopes, uint16_t *d_out, void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_decode_lanes_seq");
    if (k < 0 || (k > 0 && (!scopes || !d_out))) return DFW_EINVAL;
    if (k == 0) return DFW_OK;
    if (reinterpret_cast<uintptr_t>(d_out) & 15u) return DFW_EALIGN;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DFW_ECUDA;
    return launch_decode_lanes_seq(k, scopes, d_out, static_cast<cudaStream_t>(cuda_stream), sms, nullptr, false);
}

extern "C" dfw_status dfw_decode_lanes_seq_launches(int k, const dfw_lanes_scope *scopes, int *launches) {
    if (k < 0 || !launches || (k > 0 && !scopes)) return DFW_EINVAL;
    *launches = 0;
    if (k == 0) return DFW_OK;
    return launch_decode_lanes_seq(k, scopes, nullptr, nullptr, 0, launches, true);
}

extern "C" dfw_status dfw_decode_gemv_lanes(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                                            const uint16_t *d_chunk_bits, const uint64_t *d_group_start,
                                            const dfw_table *table, const dfw_lanes_info *info, int k,
                                            const uint64_t *tensor_offsets, const uint32_t *cols,
                                            const uint16_t *const *d_x, float *const *d_y, float *d_partial,
                                            uint64_t partial_elems, void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_decode_gemv_lanes");
    dfw_status st = validate_table(table);
    if (st != DFW_OK) return st;
    if (!info || table->n == 0) return DFW_EINVAL;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DFW_ECUDA;
    return launch_gemv_lanes(d_stream, d_mant, d_lut, d_chunk_bits, d_group_start, table, info, k, tensor_offsets,
                             cols, d_x, d_y, d_partial, partial_elems, static_cast<cudaStream_t>(cuda_stream), sms);
}

extern "C" dfw_status dfw_rans_decode(const uint8_t *d_stream, const uint8_t *d_mant, const uint64_t *d_block_start,
                                      const dfw_rans_table *table, uint16_t *d_out, void *cuda_stream) {
    dfw::NvtxRange nvtx_range("dfw_rans_decode");
    if (!table || table->version != DFW_FORMAT_VERSION || table->scale_bits != DFW_RANS_SCALE_BITS ||
        table->lanes != DFW_RANS_LANES || table->block_syms != DFW_RANS_BLOCK ||
        table->n_blocks != (table->n + DFW_RANS_BLOCK - 1) / DFW_RANS_BLOCK)
        return DFW_EINVAL;
    if (table->n == 0) return DFW_OK;
    if (!d_stream || !d_mant || !d_block_start || !d_out) return DFW_EINVAL;
    if ((reinterpret_cast<uintptr_t>(d_stream) | reinterpret_cast<uintptr_t>(d_block_start)) & 15u) return DFW_EALIGN;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DFW_ECUDA;
    return launch_rans_decode(d_stream, d_mant, d_block_start, table, d_out, static_cast<cudaStream_t>(cuda_stream),
                              sms);
}

extern "C" dfw_status dfw_status_bits(void *cuda_stream, uint32_t *bits) {
    if (bits) *bits = 0u;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess) return DFW_ECUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return DFW_ECUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return DFW_ECUDA;
    if (bits) *bits = v;
    return v ? DFW_ECORRUPT : DFW_OK;
}

extern "C" dfw_status dfw_check(void *cuda_stream) { return dfw_status_bits(cuda_stream, nullptr); }

namespace dfw {
uint32_t take_encoder_check_site();  // dfw_encode.cu: the encoder kernels' own word (0 on failure to read)
}

extern "C" dfw_status dfw_checks_report(uint32_t *enabled, uint32_t *site) {
    if (!enabled || !site) return DFW_EINVAL;
#ifdef DFW_CHECKS
    *enabled = 1u;
#else
    *enabled = 0u;
#endif
    *site = 0u;
    if (cudaDeviceSynchronize() != cudaSuccess) return DFW_ECUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_check_site, sizeof(v)) != cudaSuccess) return DFW_ECUDA;
    if (cudaMemcpyToSymbol(g_check_site, &zero, sizeof(zero)) != cudaSuccess) return DFW_ECUDA;
    const uint32_t e = take_encoder_check_site();
    *site = v ? v : e;
    return DFW_OK;
}

namespace dfw {
namespace {

// One warp waits, with the bounded wait of the decode kernels, on an
// mbarrier whose transaction no copy will ever complete (16 bytes expected,
// none issued): the wait gives up at its time limit and the kernel reports
// ST_TIMEOUT, as a decode whose bulk copy never landed does.
__global__ void selftest_wait_timeout() {
    __shared__ __align__(8) unsigned long long bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_mbar_init();
        mbar_expect_tx(b, 16u);
    }
    __syncwarp();
    const bool ok = mbar_wait(b, 0u);
    if (!__all_sync(0xFFFFFFFFu, ok) && threadIdx.x == 0) atomicOr(&g_status, ST_TIMEOUT);
}

}  // namespace
}  // namespace dfw

extern "C" dfw_status dfw_selftest_wait_timeout(void *cuda_stream) {
    dfw::selftest_wait_timeout<<<1, 32, 0, static_cast<cudaStream_t>(cuda_stream)>>>();
    return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
}
