// dfw_rans.cuh -- GPU decoder of the rANS variant (included by dfw_decode.cu).
//
// Persistent warps, one rANS block (16384 exponents, 32 interleaved states)
// at a time.  Per CTA the decode table for the 2^12 slots is built once in
// shared memory: entry = exponent | (f - 1) << 8 | (slot - c) << 20, so a
// step costs one shared load and one multiply-add per state.  Per warp, lane
// 0 stages blocks into two shared slots with 1-D TMA bulk copies (mbarrier
// completion, started one block ahead).  A step: each lane decodes the
// exponent of its state, the warp ballots which states fell below 2^16, each
// of those takes the word at (next word + its rank among them), and the
// lane joins its exponent with the raw byte into bf16 (one 2-byte store per
// lane: 64 contiguous bytes per warp).  Raw bytes arrive 4 per lane in
// coalesced 128-byte rows, three rows (12 steps) ahead of use, and reach
// the lane that needs them by shuffle.  A block must end with every state at
// 2^16 and every word used; otherwise the status word records it.
//
// Slots per warp (nslot): two let the next block's copy run during this
// block's decode; one halves the shared memory per warp, so twice as many
// warps fit on an SM, and the copy of the next block is then issued after
// this block's last read and waited for at the top of the next one.  The
// launcher takes whichever keeps more warps resident (the decode is bound by
// the latency of each state's chain of dependent steps, so more warps win).
#pragma once

#include <type_traits>

#include "dfw_device.cuh"

namespace dfw {
namespace {

constexpr uint32_t RANS_SLOTS = 1u << DFW_RANS_SCALE_BITS;
constexpr uint32_t RANS_HEAD = 4u * DFW_RANS_LANES;  // state bytes at the start of a block
constexpr uint32_t RANS_TABLE_BYTES = 4u * RANS_SLOTS + 1040u;  // decode table + 257 cumulative starts, 16-aligned

struct RansParams {
    const uint8_t *stream;
    const uint8_t *mant;
    const uint64_t *block_start;
    uint16_t *out;
    uint64_t n, stream_bytes, mant_bytes;
    uint32_t n_blocks, slot_bytes, nslot;
    uint16_t freq[256];
};

template <int NT>
__global__ void __launch_bounds__(NT) rans_decode_kernel(const RansParams prm) {
    constexpr int NWARP = NT / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *s_tab = reinterpret_cast<uint32_t *>(smem);
    uint32_t *s_cum = s_tab + RANS_SLOTS;  // 257 cumulative starts
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // decode table: exponent s owns slots [c_s, c_s + f_s)
    if (tid == 0) {
        uint32_t c = 0;
        for (int s = 0; s < 256; ++s) {
            s_cum[s] = c;
            c += prm.freq[s];
        }
        s_cum[256] = c;
    }
    __syncthreads();
    bool bad = s_cum[256] != RANS_SLOTS;
    for (int s = tid; s < 256 && !bad; s += NT) {
        const uint32_t f = prm.freq[s], c = s_cum[s];
        for (uint32_t k = 0; k < f; ++k) s_tab[c + k] = (uint32_t)s | ((f - 1u) << 8) | (k << 20);
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0) atomicOr(&g_status, ST_LUT);
        return;
    }

    uint8_t *wbase = smem + RANS_TABLE_BYTES + warp * (16u + prm.nslot * prm.slot_bytes);
    const uint32_t bar0 = smem_u32(wbase);
    uint8_t *slots = wbase + 16;
    const uint32_t gstride = gridDim.x * NWARP;
    uint32_t b = blockIdx.x * NWARP + warp;
    if (b >= prm.n_blocks) return;
    if (lane == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8u, 1);
        fence_mbar_init();
    }
    __syncwarp();

    // lane 0: block bb into slot s (its bytes, capped to the slot)
    auto issue = [&](uint32_t bb, uint32_t s) {
        const uint64_t b0 = __ldg(prm.block_start + bb), b1 = __ldg(prm.block_start + bb + 1);
        uint32_t bytes = 0;
        if (b1 > b0 && b1 <= prm.stream_bytes && !(b0 & 15u)) bytes = (uint32_t)min(b1 - b0, (uint64_t)prm.slot_bytes);
        bytes &= ~15u;
        if (!check(bb < prm.n_blocks && bytes <= prm.slot_bytes && (bytes == 0u || b0 + bytes <= prm.stream_bytes),
                   CK_RANS_COPY))
            bytes = 0u;
        fence_proxy_async();
        mbar_expect_tx(bar0 + 8u * s, bytes);
        if (bytes) bulk_load(smem_u32(slots + s * prm.slot_bytes), prm.stream + b0, bytes, bar0 + 8u * s);
    };
    if (lane == 0) issue(b, 0);

    const uint32_t lt_mask = (1u << lane) - 1u;
    const bool two = prm.nslot == 2u;
    for (uint32_t it = 0;; ++it) {
        const uint32_t s = two ? (it & 1u) : 0u;
        const uint32_t bn = b + gstride;
        __syncwarp();  // every lane is done with the other slot
        if (two && bn < prm.n_blocks && lane == 0) issue(bn, s ^ 1u);
        const uint32_t parity = two ? (it >> 1) & 1u : it & 1u;
        bool ok = mbar_wait(bar0 + 8u * s, parity);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
            if (lane == 0) {  // report, then give the copies in flight one more bounded wait each
                atomicOr(&g_status, ST_TIMEOUT);
                mbar_wait_bounded(bar0 + 8u * s, parity);
                if (two && bn < prm.n_blocks) mbar_wait_bounded(bar0 + 8u * (s ^ 1u), ((it + 1) >> 1) & 1u);
            }
            return;
        }
        const uint64_t b0 = __ldg(prm.block_start + b), b1 = __ldg(prm.block_start + b + 1);
        const uint64_t i0 = (uint64_t)b * DFW_RANS_BLOCK;
        const uint32_t cnt = (uint32_t)min((uint64_t)DFW_RANS_BLOCK, prm.n - i0);
        const bool fits = b1 > b0 && b1 - b0 >= RANS_HEAD && b1 - b0 <= prm.slot_bytes && b1 <= prm.stream_bytes &&
                          !(b0 & 15u) && !((b1 - b0) & 15u);
        if (!fits) {
            if (lane == 0) atomicOr(&g_status, ST_RANGE);
        } else {
            const uint32_t sl = smem_u32(slots + s * prm.slot_bytes);
            const uint32_t words = (uint32_t)(b1 - b0 - RANS_HEAD) / 2u;  // includes the zero padding
            uint32_t x = lds32(sl + 4u * lane);
            uint32_t ptr = 0;
            // raw bytes: lane l loads the 4 bytes at 128 q + 4 l of the block
            // (coalesced), three quads ahead; step 4 q + t takes its byte from
            // lane 8 t + l / 4 by shuffle
            const uint8_t *mrow = prm.mant + i0;
            const uint32_t mlim = (uint32_t)min((uint64_t)DFW_RANS_BLOCK, prm.mant_bytes - i0);
            auto mload = [&](uint32_t q) -> uint32_t {
                const uint32_t o = 128u * q + 4u * lane;
                return o + 4u <= mlim ? __ldg(reinterpret_cast<const uint32_t *>(mrow + o)) : 0u;
            };
            uint32_t m1 = mload(0), m2 = mload(1), m3 = mload(2);
            uint16_t *op = prm.out + i0 + lane;
            const uint32_t quads = (cnt + 127u) / 128u;
            const uint32_t tab = smem_u32(s_tab), wbase = sl + RANS_HEAD;
            // the quads of the block; WHOLE (every block but possibly the
            // scope's last) drops the per-step checks against cnt
            auto quads_of = [&](auto whole_c) {
                constexpr bool WHOLE = decltype(whole_c)::value;
                for (uint32_t q = 0; q < quads; ++q) {
                    const uint32_t mc = m1;
                    m1 = m2;
                    m2 = m3;
                    m3 = mload(q + 3u);
#pragma unroll
                    for (uint32_t t = 0; t < 4; ++t) {
                        const bool live = WHOLE || 128u * q + 32u * t + lane < cnt;
                        const uint32_t e = lds32(tab + 4u * (x & (RANS_SLOTS - 1u)));
                        const uint32_t xd = (((e >> 8) & 0xFFFu) + 1u) * (x >> DFW_RANS_SCALE_BITS) + (e >> 20);
                        x = live ? xd : x;
                        const bool need = live && x < 65536u;
                        const uint32_t mask = __ballot_sync(0xFFFFFFFFu, need);
                        const uint32_t w = ptr + __popc(mask & lt_mask);
                        // a reload past the block's words is skipped (a corrupt
                        // block; the checks after the block then fail)
                        const uint32_t v = lds16_if(need && w < words, wbase + 2u * w);
                        x = need ? (x << 16) | v : x;
                        ptr += __popc(mask);
                        const uint32_t mb = __byte_perm(__shfl_sync(0xFFFFFFFFu, mc, 8u * t + (lane >> 2)), 0u,
                                                        0x4440u | (lane & 3u));
                        // bf16 = sign << 15 | exponent << 7 | mantissa: the
                        // raw byte doubled into both halves keeps its sign at
                        // bit 15 and its mantissa at bits 6..0; the table
                        // entry's low byte is the exponent
                        if (live && check(i0 + 128u * q + 32u * t + lane < prm.n, CK_RANS_STORE))
                            op[32u * t] = (uint16_t)(((mb * 0x101u) & 0x807Fu) | ((e << 7) & 0x7F80u));
                    }
                    op += 128;
                }
            };
            if (cnt == DFW_RANS_BLOCK) quads_of(std::integral_constant<bool, true>{});
            else quads_of(std::integral_constant<bool, false>{});
            // integrity: every state back at 2^16, every word used and none
            // past the block's end (a skipped reload leaves ptr beyond it)
            const bool good = __all_sync(0xFFFFFFFFu, x == 65536u) &&
                              ((RANS_HEAD + 2ull * ptr + 15ull) & ~15ull) == b1 - b0;
            if (!good && lane == 0) atomicOr(&g_status, ST_COUNT);
        }
        if (bn >= prm.n_blocks) break;
        if (!two) {
            __syncwarp();  // every lane is done with the slot
            if (lane == 0) issue(bn, 0u);
        }
        b = bn;
    }
}

struct RansVariant {
    int nt;
    void (*fn)(const RansParams);
    int smem_set[16];
};
RansVariant g_rans[] = {
    {512, rans_decode_kernel<512>, {0}},
    {256, rans_decode_kernel<256>, {0}},
    {128, rans_decode_kernel<128>, {0}},
    {64, rans_decode_kernel<64>, {0}},
};

}  // namespace

dfw_status launch_rans_decode(const uint8_t *d_stream, const uint8_t *d_mant, const uint64_t *d_block_start,
                              const dfw_rans_table *t, uint16_t *d_out, cudaStream_t s, int sms) {
    if (t->max_block_bytes < RANS_HEAD || t->max_block_bytes > 2u * DFW_RANS_BLOCK + RANS_HEAD + 16u ||
        (t->max_block_bytes & 15u) || t->n_blocks >= (1ull << 32))
        return DFW_EINVAL;
    RansParams prm;
    prm.stream = d_stream;
    prm.mant = d_mant;
    prm.block_start = d_block_start;
    prm.out = d_out;
    prm.n = t->n;
    prm.stream_bytes = t->stream_bytes;
    prm.mant_bytes = (t->n + 15) & ~15ull;
    prm.n_blocks = (uint32_t)t->n_blocks;
    prm.slot_bytes = t->max_block_bytes;
    std::memcpy(prm.freq, t->freq, sizeof(prm.freq));
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return DFW_ECUDA;
    // the CTA size and slots per warp that keep the most warps resident per
    // SM (blocks of incompressible data need 16.5 KB slots); on a tie, two
    // slots (the next block's copy overlaps this block's decode)
    RansVariant *best = nullptr;
    uint32_t best_smem = 0, best_nslot = 0;
    int best_warps = 0, best_per_sm = 0;
    for (uint32_t nslot = 2; nslot >= 1; --nslot) {
        for (RansVariant &v : g_rans) {
            const uint32_t smem = RANS_TABLE_BYTES + (uint32_t)(v.nt / 32) * (16u + nslot * prm.slot_bytes);
            if (smem > 227u * 1024u) continue;
            if (!v.smem_set[dev]) {
                if (cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
                    return DFW_ECUDA;
                v.smem_set[dev] = 1;
            }
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v.fn, v.nt, smem) != cudaSuccess)
                return DFW_ECUDA;
            if (per_sm * (v.nt / 32) > best_warps) {
                best = &v;
                best_smem = smem;
                best_nslot = nslot;
                best_warps = per_sm * (v.nt / 32);
                best_per_sm = per_sm;
            }
        }
    }
    if (!best) return DFW_EINVAL;
    prm.nslot = best_nslot;
    const uint64_t wpc = (uint64_t)best->nt / 32;
    const uint64_t warps = (uint64_t)best_per_sm * sms * wpc;
    const uint64_t want = t->n_blocks < warps ? t->n_blocks : warps;
    best->fn<<<(unsigned)((want + wpc - 1) / wpc), best->nt, best_smem, s>>>(prm);
    return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
}


}  // namespace dfw
