// dfw_decode.cu -- device half of libdfw: the sm_100a decode kernels.
//
// Source: DFloat11 abstract ("70% Size, 100% Accuracy: Lossless LLM
// Compression for Efficient GPU Inference via Dynamic-Length Float"): compact
// LUTs in GPU SRAM, a two-phase kernel that coordinates thread read/write
// positions through lightweight auxiliary arrays, block-level decompression,
// bit-exact output.  This kernel is written for B200 from that description:
//
//   one CTA per tile of T windows of W stream bytes (one window per thread)
//   phase 0  LUT table 0 -> shared memory (validated once per CTA);
//            each thread loads its W (+4 guard) stream bytes and its gap
//   phase 1  each thread walks the codewords that start in its window and
//            counts them; whole codewords inside the next 8 bits are counted
//            in one table lookup
//   scan     warp shuffle scan + block scan of the counts; the tile's total
//            must equal out_start[b+1] - out_start[b]
//   phase 2  each thread walks its window again and writes the exponent
//            symbols into a shared-memory buffer at its scanned offset
//   phase 3  all threads turn (exponent, raw byte) pairs into bf16, 8 weights
//            per thread per step: 64-bit shared and global loads, 128-bit
//            coalesced global stores; ragged tile edges go element by element
//
// Bounds: every walk advances at least one bit per step and stops at its
// window end (8W bits), so no loop depends on the data for termination; the
// LUT is checked before use; tiles whose counts or ranges are inconsistent
// write nothing and set a bit of the device status word.
#include <cuda_runtime.h>

#include "dfw_internal.h"

namespace dfw {

__device__ unsigned int g_status;

namespace {

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// Walks subtables (global memory, read-only path) for a codeword longer than
// 8 bits.  x holds the 32 stream bits starting at the codeword.
__device__ __noinline__ uint32_t resolve_long(uint32_t x, uint32_t e, const uint32_t *__restrict__ g_lut,
                                              uint32_t n_tables, uint32_t &err) {
#pragma unroll 1
    for (int level = 1; level < 4; ++level) {
        const uint32_t child = e & LUT_CHILD_MASK;
        if (child >= n_tables) break;
        e = __ldg(g_lut + child * 256u + ((x >> (24 - 8 * level)) & 0xFFu));
        if (!(e & LUT_PTR)) {
            const uint32_t l = (e >> LUT_LEN_SHIFT) & 63u;
            if (l > 8u * level && l <= 8u * level + 8u) return e;
            break;
        }
    }
    err |= ST_LUT;
    return 1u << LUT_LEN_SHIFT;  // length 1 keeps the walk finite
}

// Walks the codewords starting in [p, wend) of a window held as NSEG
// big-endian words plus one guard word.  Counts them (EMIT = false) or also
// writes their symbols to ebuf[o...] (EMIT = true), never past ebuf[lim].
template <bool EMIT, int NSEG>
__device__ __forceinline__ uint32_t walk(const uint32_t (&wd)[NSEG + 1], int p, const int wend,
                                         const uint32_t *__restrict__ s_lut,
                                         const uint32_t *__restrict__ g_lut, uint32_t n_tables,
                                         uint8_t *__restrict__ ebuf, uint32_t o, uint32_t lim,
                                         uint32_t &err) {
    uint32_t cnt = 0;
#pragma unroll
    for (int seg = 0; seg < NSEG; ++seg) {
        const uint32_t hi = wd[seg], lo = wd[seg + 1];
        const int seg_end = min(32 * (seg + 1), wend);
        while (p < seg_end) {
            const uint32_t x = __funnelshift_l(lo, hi, (uint32_t)p);  // bits [p, p + 32)
            uint32_t e = s_lut[x >> 24];
            if (!EMIT) {
                const uint32_t c = (e >> LUT_CNT_SHIFT) & 15u;
                if (c != 0u && p + 8 <= wend) {  // all c codewords start before wend
                    cnt += c;
                    p += (int)((e >> LUT_CBITS_SHIFT) & 15u);
                    continue;
                }
            }
            if (e & LUT_PTR) e = resolve_long(x, e, g_lut, n_tables, err);
            if (EMIT) ebuf[min(o + cnt, lim)] = (uint8_t)e;  // clamp only matters for a corrupt LUT
            ++cnt;
            p += (int)((e >> LUT_LEN_SHIFT) & 63u);
        }
    }
    return cnt;
}

// Four (exponent, raw byte) pairs -> four bf16 patterns in two words.
__device__ __forceinline__ void join4(uint32_t E, uint32_t M, uint32_t &w0, uint32_t &w1) {
    const uint32_t hi = (M & 0x80808080u) | ((E >> 1) & 0x7F7F7F7Fu);  // sign | exp[7:1]
    const uint32_t lo = ((E << 7) & 0x80808080u) | (M & 0x7F7F7F7Fu);  // exp[0] | mant
    w0 = __byte_perm(lo, hi, 0x5140);
    w1 = __byte_perm(lo, hi, 0x7362);
}

__device__ __forceinline__ uint16_t join1(uint32_t e, uint32_t m) {
    return (uint16_t)(((m & 0x80u) << 8) | (e << 7) | (m & 0x7Fu));
}

constexpr int SMEM_HEAD = 1024 + 128;  // LUT table 0 + per-warp scan slots

template <int W, int NT>
__global__ void __launch_bounds__(NT) decode_tiles(
    const uint8_t *__restrict__ stream, const uint8_t *__restrict__ mant,
    const uint32_t *__restrict__ g_lut, uint32_t n_tables, const uint8_t *__restrict__ gap,
    const uint64_t *__restrict__ out_start, uint64_t total_bits, uint64_t n_windows, uint64_t n,
    uint32_t ebuf_syms, uint16_t *__restrict__ out) {
    constexpr int NSEG = W / 4;
    constexpr int NWARP = NT / 32;
    static_assert(NWARP <= 32, "block scan assumes at most 32 warps");
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *s_lut = reinterpret_cast<uint32_t *>(smem);
    uint32_t *s_warp = s_lut + 256;
    uint8_t *ebuf = smem + SMEM_HEAD;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint64_t tile = blockIdx.x;
    const uint64_t os = out_start[tile], oe = out_start[tile + 1];

    // phase 0: table 0 into shared memory, checked entry by entry
    bool lut_bad = false;
    for (int i = tid; i < 256; i += NT) {
        const uint32_t e = __ldg(g_lut + i);
        if (!(e & LUT_PTR)) {
            const uint32_t l = (e >> LUT_LEN_SHIFT) & 63u, c = (e >> LUT_CNT_SHIFT) & 15u,
                           cb = (e >> LUT_CBITS_SHIFT) & 15u;
            lut_bad |= l == 0u || l > 8u || c == 0u || cb == 0u || cb > 8u;
        }
        s_lut[i] = e;
    }
    const uint64_t w = tile * NT + tid;
    uint32_t wd[NSEG + 1];
    int p = 0, wend = 0;
    if (w < n_windows) {
        const uint8_t *src = stream + w * W;
        if constexpr (W == 8) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src));
            wd[0] = bswap32(v.x);
            wd[1] = bswap32(v.y);
        } else {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src));
            wd[0] = bswap32(v.x);
            wd[1] = bswap32(v.y);
            wd[2] = bswap32(v.z);
            wd[3] = bswap32(v.w);
        }
        wd[NSEG] = bswap32(__ldg(reinterpret_cast<const uint32_t *>(src + W)));
        p = __ldg(gap + w);
        const uint64_t rem = total_bits - w * (8ull * W);
        wend = rem < 8ull * W ? (int)rem : 8 * W;
    } else {
#pragma unroll
        for (int i = 0; i <= NSEG; ++i) wd[i] = 0u;
    }
    if (__syncthreads_or(lut_bad)) {
        if (tid == 0) atomicOr(&g_status, ST_LUT);
        return;
    }
    if (oe < os || oe > n || oe - os > ebuf_syms) {
        if (tid == 0) atomicOr(&g_status, ST_RANGE);
        return;
    }

    // phase 1: count the codewords that start in this thread's window
    uint32_t err = 0;
    const uint32_t cnt = walk<false, NSEG>(wd, p, wend, s_lut, g_lut, n_tables, nullptr, 0, 0, err);

    // scan: warp shuffles, then one warp scans the warp totals
    uint32_t incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t v = lane < NWARP ? s_warp[lane] : 0u;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, v, d);
            if (lane >= d) v += y;
        }
        if (lane < NWARP) s_warp[lane] = v;
    }
    __syncthreads();
    const uint32_t total = s_warp[NWARP - 1];
    const uint32_t excl = (warp ? s_warp[warp - 1] : 0u) + incl - cnt;
    if (total != (uint32_t)(oe - os)) {
        if (tid == 0) atomicOr(&g_status, ST_COUNT);
        return;
    }

    // phase 2: symbols into the tile buffer; ebuf[j - (os & ~15)] holds weight j
    const uint32_t cnt2 = walk<true, NSEG>(wd, p, wend, s_lut, g_lut, n_tables, ebuf,
                                           (uint32_t)(os & 15u) + excl, ebuf_syms + 15u, err);
    if (err) atomicOr(&g_status, err);
    // both walks must agree (they can only differ if the LUT's counts contradict its lengths)
    if (__syncthreads_or(cnt2 != cnt)) {
        if (tid == 0) atomicOr(&g_status, ST_COUNT);
        return;
    }

    // phase 3: bf16 assembly, 8 weights per thread per step
    const uint64_t base = os & ~15ull;
    const uint64_t c0 = os >> 3, c1 = (oe + 7) >> 3;
    for (uint64_t c = c0 + tid; c < c1; c += NT) {
        const uint64_t j0 = c << 3;
        if (j0 >= os && j0 + 8 <= oe) {
            const uint2 m = __ldcs(reinterpret_cast<const uint2 *>(mant + j0));
            const uint2 e = *reinterpret_cast<const uint2 *>(ebuf + (j0 - base));
            uint4 r;
            join4(e.x, m.x, r.x, r.y);
            join4(e.y, m.y, r.z, r.w);
            __stcs(reinterpret_cast<uint4 *>(out + j0), r);
        } else {
            const uint64_t lo = j0 > os ? j0 : os, hi = j0 + 8 < oe ? j0 + 8 : oe;
            for (uint64_t j = lo; j < hi; ++j) out[j] = join1(ebuf[j - base], mant[j]);
        }
    }
}

// One distinct exponent: every weight is (sym, raw byte).
__global__ void fill_single(const uint8_t *__restrict__ mant, uint32_t sym, uint64_t n,
                           uint16_t *__restrict__ out) {
    const uint32_t E = sym * 0x01010101u;
    const uint64_t nfull = n >> 3;
    for (uint64_t c = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; c < nfull;
         c += (uint64_t)gridDim.x * blockDim.x) {
        const uint2 m = __ldcs(reinterpret_cast<const uint2 *>(mant + (c << 3)));
        uint4 r;
        join4(E, m.x, r.x, r.y);
        join4(E, m.y, r.z, r.w);
        __stcs(reinterpret_cast<uint4 *>(out + (c << 3)), r);
    }
    if (blockIdx.x == 0 && threadIdx.x < (n & 7)) {
        const uint64_t j = (nfull << 3) + threadIdx.x;
        out[j] = join1(sym, mant[j]);
    }
}

typedef void (*decode_fn)(const uint8_t *, const uint8_t *, const uint32_t *, uint32_t, const uint8_t *,
                          const uint64_t *, uint64_t, uint64_t, uint64_t, uint32_t, uint16_t *);

struct Variant {
    uint32_t W, T;
    decode_fn fn;
    int smem_set[16];  // dynamic shared memory opted in per device
};

Variant g_variants[] = {
    {8, 128, decode_tiles<8, 128>, {0}},   {8, 256, decode_tiles<8, 256>, {0}},
    {8, 512, decode_tiles<8, 512>, {0}},   {16, 128, decode_tiles<16, 128>, {0}},
    {16, 256, decode_tiles<16, 256>, {0}}, {16, 512, decode_tiles<16, 512>, {0}},
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
    if (table->total_bits == 0) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const uint64_t chunks = (n >> 3) + 1;
        const uint64_t want = (chunks + 255) / 256;
        const unsigned grid = (unsigned)(want < (uint64_t)sms * 8 ? want : (uint64_t)sms * 8);
        fill_single<<<grid, 256, 0, s>>>(d_mant, table->single_symbol, n, d_out);
        return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
    }
    if (!d_stream || !d_lut || !d_gap || !d_out_start) return DFW_EINVAL;
    if (!aligned16(d_stream) || !aligned16(d_lut) || !aligned16(d_out_start)) return DFW_EALIGN;
    if (info->lut_tables < 1 || info->lut_words != 256u * info->lut_tables) return DFW_EINVAL;
    if (info->max_tile_symbols > 8ull * info->window_bytes * info->tile_windows) return DFW_EINVAL;
    if (info->n_tiles > 0x7FFFFFFFull) return DFW_EINVAL;
    Variant *v = nullptr;
    for (auto &x : g_variants)
        if (x.W == info->window_bytes && x.T == info->tile_windows) v = &x;
    if (!v) return DFW_EINVAL;
    const uint32_t ebuf_bytes = (uint32_t)((info->max_tile_symbols + 16 + 15) & ~15ull);
    const size_t smem = SMEM_HEAD + ebuf_bytes;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DFW_ECUDA;
    if (smem > 48 * 1024 && dev < 16 && !v->smem_set[dev]) {
        if (cudaFuncSetAttribute(v->fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
            return DFW_ECUDA;
        v->smem_set[dev] = 1;
    }
    v->fn<<<(unsigned)info->n_tiles, v->T, smem, s>>>(d_stream, d_mant, d_lut, info->lut_tables, d_gap,
                                                      d_out_start, table->total_bits, info->n_windows, n,
                                                      ebuf_bytes - 16, d_out);
    return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
}

}  // namespace dfw

using namespace dfw;

extern "C" dfw_status dfw_decode(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                                 const uint8_t *d_gap, const uint64_t *d_out_start, const dfw_table *table,
                                 const dfw_plan_info *info, uint16_t *d_out, void *cuda_stream) {
    return launch_decode(d_stream, d_mant, d_lut, d_gap, d_out_start, table, info, d_out,
                         static_cast<cudaStream_t>(cuda_stream));
}

extern "C" dfw_status dfw_decode_block(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                                       const uint8_t *d_gap, const uint64_t *d_out_start,
                                       const dfw_table *table, const dfw_plan_info *info,
                                       const uint64_t *tensor_offsets, int k, uint16_t *d_scratch,
                                       uint64_t scratch_elems, void *cuda_stream) {
    if (!table || !tensor_offsets || k < 1) return DFW_EINVAL;
    if (tensor_offsets[0] != 0 || tensor_offsets[k] != table->n) return DFW_EINVAL;
    for (int i = 0; i < k; ++i)
        if (tensor_offsets[i + 1] < tensor_offsets[i]) return DFW_EINVAL;
    if (scratch_elems < table->n) return DFW_ENOMEM;
    return launch_decode(d_stream, d_mant, d_lut, d_gap, d_out_start, table, info, d_scratch,
                         static_cast<cudaStream_t>(cuda_stream));
}

extern "C" dfw_status dfw_check(void *cuda_stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess) return DFW_ECUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return DFW_ECUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return DFW_ECUDA;
    return v ? DFW_ECORRUPT : DFW_OK;
}
