// dfw_lanes.cuh -- the known-start decode kernel (included by dfw_decode.cu).
//
// Same stream and tables as the windowed kernel; the plan differs: codewords
// are cut into chunks of 64, chunk_bits[c] says how many stream bits chunk c
// uses and group_start[g] where group g (32 chunks) begins (the LazyWeights
// write-up's interleaved lanes with known starts, body and Verified Facts).
// One warp decodes one group at a time, persistently.  All bulk copies are
// issued by lane 0, one per buffer (copy instructions take warp-uniform
// operands, so per-lane copies would be serialised lane by lane):
//   - the group's chunk_bits and stream span arrive in one of the warp's two
//     stream slots (started one group ahead), its 2048 raw bytes in the
//     warp's raw-byte buffer (started as soon as the previous group's join
//     has read that buffer);
//   - each lane finds its chunk's first bit with a warp prefix sum of
//     chunk_bits and decodes its 64 codewords with the fast table (up to
//     four codewords per lookup) into its own word slots, one row per word
//     index, the 32 lanes side by side;
//   - the warp then joins exponents and raw bytes into bf16 with the lanes
//     reassigned: in store j lane l joins piece l & 3 (16 weights) of chunk
//     8 j + l / 4 and writes it with one 256-bit store, so each store
//     instruction covers 1 KB of contiguous output (two 128-bit stores per
//     lane when the output is only 16-byte aligned); no staging buffer is
//     needed, which leaves shared memory for up to 32 warps per SM.
// No count phase, no block scan, no CTA barrier after the table load, and no
// realignment: every chunk's output is 64-weight aligned.
//
// Bounds: a lane makes at most 64 lookups per chunk (each yields >= 1
// codeword; an escape resolves one codeword of at most 32 bits), so its
// stream reads end within 2048 bits and a few words of its start: a corrupt
// stream can read past its slot but not past the warp's own shared-memory
// area; a group whose chunk_bits do not add up to its group_start span, or
// whose lanes do not end exactly where chunk_bits says, writes nothing and
// sets a status bit; waits on bulk copies are bounded.
#pragma once

#include <cstring>

#include "dfw_device.cuh"

namespace dfw {
namespace {

constexpr uint32_t EXP_WORDS = 17;        // a chunk's 64 exponent bytes + up to 3 more from the last lookup
// Word k of the exponent slots of chunk c (0..31 within its group) lives at
// EXP_STRIDE * k + 4 c: one row per word index, 34 words wide, so the word is
// in bank (2 k + c) mod 32.  A lane appending to its own chunk moves down
// one row per word; the join reads words 4 i .. 4 i + 3 of eight chunks in
// four pieces i at once, which the two-bank step per row spreads over all 32
// banks.
constexpr uint32_t EXP_STRIDE = 136;
// The slots' area, rounded up to 16 bytes so every warp's area (and the bulk
// copies and 128-bit loads into it) stays 16-byte aligned.
constexpr uint32_t EXP_BYTES = (EXP_WORDS * EXP_STRIDE + 15u) & ~15u;
constexpr uint32_t GROUP_SYMS = LANE_SYMS * GROUP_CHUNKS;  // 2048 weights per warp group

struct LanesParams {
    const uint8_t *stream;
    const uint8_t *mant;
    const uint32_t *lut;
    const uint16_t *chunk_bits;
    const uint64_t *group_start;
    uint16_t *out;
    uint64_t stream_bytes, mant_bytes;
    uint32_t n_chunks, n_groups;  // both below 2^32 (checked on the host)
    uint32_t last_t;              // codewords in the last chunk (1..64)
    uint32_t fast_bits, n_tables, sbuf_bytes;
    uint32_t out32;  // out is 32-byte aligned: one 256-bit store per 16 weights
    // Launched as a programmatic dependent of the previous decode into the
    // same output: may start while that launch drains, but waits for it to
    // complete before its first store.
    uint32_t wait_prior;
};

// Programmatic dependent launch: let the next launch on the stream start as
// SMs free up / wait until the launch before this one has completed and its
// writes are visible.
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bytes a group's stream copy takes: from the 16-byte boundary at or below
// its first bit s0 to 8 guard bytes past its last byte, rounded up to 16.
// r0 = s0 mod 128 (the first bit's offset from that boundary) and d = the
// group's bits (below 2^17), so 32-bit arithmetic suffices.
__device__ __forceinline__ uint32_t span_bytes(uint32_t r0, uint32_t d) {
    return (((r0 + d + 7u) >> 3) + 8u + 15u) & ~15u;
}

// In shared memory the lanes kernel keeps a fast entry's second word as in
// the LUT image (byte 0 bits used, byte 1 eight times the count, bits 16..27
// the end mask) except for escapes, which become LANES_ESC_WORD: no bits, no
// symbols, and the top bit, which the loop's byte permute spreads over bytes
// 1 and 2 so an escape subtracts LANES_ESC_DEC from the count and leaves the
// loop through its ordinary end test.
constexpr uint32_t LANES_ESC_WORD = 0x80000000u;
constexpr int LANES_ESC_DEC = 0x00FFFF00;

// Decodes `left8 / 8` codewords starting at bit r of the stream words held in
// shared memory at sw (32-bit shared address) and appends their symbols to
// this lane's word slots ep, ep + EXP_STRIDE, ... (slots of the 32 lanes
// interleave).  fast is the shared address of the fast table.  Returns the
// stream bit position (relative to sw) after codeword left8 / 8.
//
// The inner loop is straight-line code that runs until the chunk's count is
// reached: the last lookup may decode up to three codewords of the next
// chunk, whose symbols land in slack slots that are never read, and the exact
// end is worked out once afterwards from that lookup's end mask.  So a lane
// that finishes early has nothing left to do but wait for the others.  The
// loop keeps the word after the current pair in a register, moves it in
// (predicated) when the position crosses a word and only then loads the next
// one; it always stores the accumulator's low word and moves to the next slot
// when the word is full.  Only an escape (a codeword longer than the fast
// key) leaves it early.
__device__ __forceinline__ uint32_t decode_chunk(uint32_t sw, uint32_t r, int left8, uint32_t fast,
                                                 uint32_t kshift, const uint32_t *__restrict__ g_hier,
                                                 uint32_t n_tables, uint32_t ep, uint32_t &err, uint32_t &rd_end,
                                                 uint32_t &wr_end) {
    // p is the bit position (from sw); a and b hold the two stream words the
    // window [p, p + 32) lies in (the funnel shift takes p mod 32), c the
    // word after them (not yet byte-swapped), wa the address of the word
    // after c and qn the position where the window's first word ends.  Reads
    // past the slot (only a corrupt stream causes them) stay inside this
    // warp's shared area, and the caller's end check rejects it.
    uint32_t wa = sw + 4u * (r >> 5);
    uint32_t a = bswap32(lds32(wa));
    uint32_t b = bswap32(lds32(wa + 4u));
    uint32_t c = lds32(wa + 8u);
    wa += 12u;
    uint32_t p = r, qn = (r & ~31u) + 32u;
    uint32_t lo = 0u, m = 1u;  // m = 2^(bits of lo in use)
    const uint32_t kmul = 1u << (32u - kshift);  // x >> kshift == mulhi(x, 2^(32 - kshift))
    uint32_t x, ey;
    for (;;) {
        // Symbols are appended by multiplication with m = 2^sh (lo += syms *
        // m, spill = mulhi(syms, m)); m advances by a rotation by 8 * count,
        // which wraps exactly when the word fills.  An escape entry appends
        // nothing and leaves bits and m alone, but its rotation by zero reads
        // as a full word, so the slot pointer moves on once: undone below.
        asm volatile(
            "{\n\t"
            ".reg .pred pa, pf, pc;\n\t"
            ".reg .b32 t0, mn, sp, ex, ad, cb, c8;\n"
            // two lookups per pass, m and mn trading roles, so the rotated
            // multiplier needs no copy
            "LANES_LOOP:\n\t"
            // lookup (m -> mn)
            "shf.l.wrap.b32 %0, %4, %3, %6;\n\t"  // x = stream bits [p, p + 32)
            "mul.hi.u32 t0, %0, %13;\n\t"         // fast-table key
            "mad.lo.u32 ad, t0, 8, %12;\n\t"
            "ld.shared.v2.u32 {ex, %1}, [ad];\n\t"
            "and.b32 cb, %1, 255;\n\t"
            "prmt.b32 c8, %1, 0, 0x4BB1;\n\t"     // 8 * count, or LANES_ESC_DEC
            "mad.lo.u32 %6, cb, 1, %6;\n\t"       // p += bits used (multiply-add pipe)
            "setp.ge.u32 pa, %6, %11;\n\t"          // crossed into b
            "@pa mov.b32 %3, %4;\n\t"                // a = b
            "@pa prmt.b32 %4, %5, 0, 0x0123;\n\t"    // b = c, byte-swapped
            "@pa ld.shared.u32 %5, [%7];\n\t"
            "@pa add.u32 %7, %7, 4;\n\t"
            "@pa add.u32 %11, %11, 32;\n\t"         // next word boundary
            "mad.lo.u32 %8, ex, %9, %8;\n\t"        // lo += syms * m
            "mul.hi.u32 sp, ex, %9;\n\t"            // the part past the word
            "st.shared.u32 [%2], %8;\n\t"
            "shf.l.wrap.b32 mn, %9, %9, c8;\n\t"   // m rotated by 8 * count
            "setp.le.u32 pf, mn, %9;\n\t"          // wrapped: the word is full
            "@pf add.u32 %2, %2, 136;\n\t"           // next word slot of this lane (EXP_STRIDE)
            "@pf mov.b32 %8, sp;\n\t"
            "mad.lo.s32 %10, c8, -1, %10;\n\t"       // left8 -= 8 * count (multiply-add pipe)
            "setp.gt.s32 pc, %10, 0;\n\t"
            "@!pc bra LANES_EXIT_A;\n\t"
            // lookup (mn -> m)
            "shf.l.wrap.b32 %0, %4, %3, %6;\n\t"  // x = stream bits [p, p + 32)
            "mul.hi.u32 t0, %0, %13;\n\t"         // fast-table key
            "mad.lo.u32 ad, t0, 8, %12;\n\t"
            "ld.shared.v2.u32 {ex, %1}, [ad];\n\t"
            "and.b32 cb, %1, 255;\n\t"
            "prmt.b32 c8, %1, 0, 0x4BB1;\n\t"     // 8 * count, or LANES_ESC_DEC
            "mad.lo.u32 %6, cb, 1, %6;\n\t"       // p += bits used (multiply-add pipe)
            "setp.ge.u32 pa, %6, %11;\n\t"          // crossed into b
            "@pa mov.b32 %3, %4;\n\t"                // a = b
            "@pa prmt.b32 %4, %5, 0, 0x0123;\n\t"    // b = c, byte-swapped
            "@pa ld.shared.u32 %5, [%7];\n\t"
            "@pa add.u32 %7, %7, 4;\n\t"
            "@pa add.u32 %11, %11, 32;\n\t"         // next word boundary
            "mad.lo.u32 %8, ex, mn, %8;\n\t"        // lo += syms * m
            "mul.hi.u32 sp, ex, mn;\n\t"            // the part past the word
            "st.shared.u32 [%2], %8;\n\t"
            "shf.l.wrap.b32 %9, mn, mn, c8;\n\t"   // m rotated by 8 * count
            "setp.le.u32 pf, %9, mn;\n\t"          // wrapped: the word is full
            "@pf add.u32 %2, %2, 136;\n\t"           // next word slot of this lane (EXP_STRIDE)
            "@pf mov.b32 %8, sp;\n\t"
            "mad.lo.s32 %10, c8, -1, %10;\n\t"       // left8 -= 8 * count (multiply-add pipe)
            "setp.gt.s32 pc, %10, 0;\n\t"
            "@pc bra LANES_LOOP;\n\t"
            "bra LANES_DONE;\n"
            "LANES_EXIT_A:\n\t"
            "mov.b32 %9, mn;\n"
            "LANES_DONE:\n\t"
            "}"
            : "=r"(x), "=r"(ey), "+r"(ep), "+r"(a), "+r"(b), "+r"(c), "+r"(p), "+r"(wa), "+r"(lo), "+r"(m),
              "+r"(left8), "+r"(qn)
            : "r"(fast), "r"(kmul)
            : "memory");
        if (left8 > -LANES_ESC_DEC / 2) break;  // the chunk's count is reached
        // an escape: take back the slot step and resolve the codeword in the
        // byte-keyed hierarchy
        left8 += LANES_ESC_DEC;
        ep -= EXP_STRIDE;
        lo = lds32(ep);
        const uint32_t f = resolve_escape(x, g_hier, n_tables);
        if (f & ESC_BAD) err |= ST_LUT;
        p += (f >> LUT_LEN_SHIFT) & 63u;  // <= 32: at most one word to shift in
        if (p >= qn) {
            a = b;
            b = bswap32(c);
            c = lds32(wa);
            wa += 4u;
            qn += 32u;
        }
        const uint32_t syms = rot_sym(f);
        const uint32_t spill = __umulhi(syms, m);
        lo += syms * m;
        const uint32_t mn = __funnelshift_l(m, m, 8u);
        if (mn <= m) {
            sts32(ep, lo);
            ep += EXP_STRIDE;
            lo = spill;
        }
        m = mn;
        left8 -= 8;
        ey = 0u;
        if (left8 <= 0) break;
    }
    if (m != 1u) sts32(ep, lo);
    rd_end = wa;  // one past the last stream word read
    wr_end = ep;  // the last slot word written
    uint32_t end = p;
    if (left8 < 0) {
        // the last lookup (a fast entry) ran -left8 / 8 codewords past the
        // chunk: its end is that of codeword number keep of the lookup
        uint32_t ends = (ey >> FAST_ENDS_SHIFT) & 0xFFFu;
        const uint32_t c8 = (ey >> FAST_C8_SHIFT) & 255u;
        const uint32_t keep = (c8 - (uint32_t)(-left8)) >> 3;  // >= 1
#pragma unroll
        for (uint32_t i = 1; i < FAST_MAX_SYMS; ++i)  // keep <= FAST_MAX_SYMS: predicated, no branch
            if (i < keep) ends &= ends - 1u;
        end = end - (ey & 255u) + (uint32_t)__ffs(ends);
    }
    return end;
}

// What a warp does with its decoded group: the 32 chunks' rotated exponents
// sit in the word slots at exps0 (word k of chunk c at exps0 + EXP_STRIDE * k
// + 4 c), their 2048 raw bytes at mbuf (chunk c at mbuf + 64 c); g is the
// group.  A chunk holds 64 weights except the scope's last one (last_t).

// Weights of chunk c of the scope (64 except the last chunk; 0 past it).
__device__ __forceinline__ uint32_t chunk_weights(const LanesParams &prm, uint32_t c) {
    return c + 1u < prm.n_chunks ? LANE_SYMS : (c + 1u == prm.n_chunks ? prm.last_t : 0u);
}

// Sixteen weights: raw bytes at m (16 bytes), rotated exponents in four
// words at e, e + EXP_STRIDE, ... -> sixteen bf16 patterns.
__device__ __forceinline__ void join16(uint32_t m_addr, uint32_t e_addr, uint4 &r0, uint4 &r1) {
    const uint4 m = lds128(m_addr);
    const uint32_t e0 = lds32(e_addr), e1 = lds32(e_addr + EXP_STRIDE), e2 = lds32(e_addr + 2u * EXP_STRIDE),
                   e3 = lds32(e_addr + 3u * EXP_STRIDE);
    join4(e0, m.x, r0.x, r0.y);
    join4(e1, m.y, r0.z, r0.w);
    join4(e2, m.z, r1.x, r1.y);
    join4(e3, m.w, r1.z, r1.w);
}

// Decode: join into bf16 and store.  Store j of the warp writes bytes
// [1024 j, 1024 j + 1024) of the group's output, lane l the 32 bytes of piece
// l & 3 (16 weights) of chunk 8 j + l / 4, so each store instruction writes
// eight whole 128-byte lines; the raw bytes it reads are one contiguous 512
// bytes and its exponent words fall in 32 different banks.
// Lane l writes weights 512 j + 16 l .. + 15 of group g (j = 0..3) in every
// path below; the multi-scope kernel relies on that (a group's bytes are
// written by the same lane whichever scope it belongs to).
__device__ __forceinline__ void store_group(uint16_t *out, uint32_t out32, uint32_t n_chunks, uint32_t last_t,
                                            uint32_t lane, uint32_t g, uint32_t mbuf, uint32_t exps0) {
    const uint32_t i = lane & 3u, cl = lane >> 2;
    const uint32_t mrow = mbuf + 16u * lane;                             // + 512 j
    const uint32_t erow = exps0 + 4u * cl + 4u * EXP_STRIDE * i;         // + 32 j, + EXP_STRIDE per word
    uint16_t *dst = out + (size_t)g * GROUP_SYMS + 16u * lane;         // + 512 j
    const uint32_t c0 = g * GROUP_CHUNKS;
    const bool whole = c0 + GROUP_CHUNKS < n_chunks || (c0 + GROUP_CHUNKS == n_chunks && last_t == LANE_SYMS);
    if (!check(c0 < n_chunks, CK_LANES_STORE)) return;
    if (whole && out32) {  // every group but the scope's last: no checks
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 r0, r1;
            join16(mrow + 512u * j, erow + 32u * j, r0, r1);
            stg256_cs(dst + 512u * j, r0, r1);  // a whole sector per lane, 1 KB per warp
        }
        return;
    }
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
        uint4 r0, r1;
        join16(mrow + 512u * j, erow + 32u * j, r0, r1);
        const uint32_t c = c0 + 8u * j + cl;
        const uint32_t t = whole ? LANE_SYMS : (c + 1u < n_chunks ? LANE_SYMS : (c + 1u == n_chunks ? last_t : 0u));
        if (16u * i + 16u <= t) {
            if (out32) {
                stg256_cs(dst + 512u * j, r0, r1);
            } else {
                __stcs(reinterpret_cast<uint4 *>(dst + 512u * j), r0);
                __stcs(reinterpret_cast<uint4 *>(dst + 512u * j + 8u), r1);
            }
        } else {  // the last, partial chunk of the scope: one weight at a time
            const uint32_t cw = 8u * j + cl;
            for (uint32_t w = 16u * i; w < t; ++w) {
                const uint32_t e = (lds32(exps0 + EXP_STRIDE * (w >> 2) + 4u * cw) >> (8u * (w & 3u))) & 0xFFu;
                const uint32_t mb = (lds32(mbuf + 64u * cw + (w & ~3u)) >> (8u * (w & 3u))) & 0xFFu;
                if (check(c0 + cw + 1u < n_chunks || (c0 + cw + 1u == n_chunks && w < last_t), CK_LANES_STORE))
                    out[(size_t)(c0 + cw) * LANE_SYMS + w] = join1(e, mb);
            }
        }
    }
}

struct StoreEpi {
    struct Params {};
    __device__ static __forceinline__ void apply(const LanesParams &prm, const Params &, uint32_t lane, uint32_t g,
                                                 uint32_t mbuf, uint32_t exps0) {
        store_group(prm.out, prm.out32, prm.n_chunks, prm.last_t, lane, g, mbuf, exps0);
    }
};

// Decode fused with y = W x: the chunk's 64 weights never leave the SM.
// Every tensor is whole chunks (its columns a multiple of 64), so a chunk is
// 64 consecutive columns of one row; lane l takes chunk l of the group and
// writes that row segment's dot product with x to partial[c] (fp32, products
// exact, one rounding per fused multiply-add, four interleaved sums added in
// a fixed order).
struct DotEpi {
    struct Params {
        uint32_t k;                              // tensors in the scope
        uint32_t cols[GEMV_MAX_TENSORS];         // columns (a multiple of 64)
        uint64_t off[GEMV_MAX_TENSORS + 1];      // first weight of each tensor
        const uint16_t *x[GEMV_MAX_TENSORS];     // bf16 input of each tensor, 32-byte aligned
        float *partial;                          // one fp32 per chunk
    };
    __device__ static __forceinline__ void apply(const LanesParams &prm, const Params &ep, uint32_t lane, uint32_t g,
                                                 uint32_t mbuf, uint32_t exps0) {
        const uint32_t c = g * GROUP_CHUNKS + lane;
        if (chunk_weights(prm, c) == 0u) return;
        const uint32_t mrow = mbuf + 64u * lane, exps = exps0 + 4u * lane;
        const uint64_t w0 = (uint64_t)c * LANE_SYMS;
        uint32_t ti = 0;
#pragma unroll
        for (uint32_t i = 1; i < GEMV_MAX_TENSORS; ++i)
            if (i < ep.k && w0 >= ep.off[i]) ti = i;
        const uint32_t col0 = (uint32_t)(w0 - ep.off[ti]) % ep.cols[ti];
        const uint16_t *xp = ep.x[ti] + col0;
        float acc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // piece q of the row segment, in the order (j + lane / 2) mod 4,
            // which spreads the lanes' 16-byte raw-byte reads over the banks
            const uint32_t q = (uint32_t)(j + (lane >> 1)) & 3u;
            uint4 r0, r1, x0, x1;
            ldg256_nc(xp + 16u * q, x0, x1);
            join16(mrow + 16u * q, exps + 4u * EXP_STRIDE * q, r0, r1);
            float a = 0.f;
            a = fma2_bf16(r0.x, x0.x, a);
            a = fma2_bf16(r0.y, x0.y, a);
            a = fma2_bf16(r0.z, x0.z, a);
            a = fma2_bf16(r0.w, x0.w, a);
            a = fma2_bf16(r1.x, x1.x, a);
            a = fma2_bf16(r1.y, x1.y, a);
            a = fma2_bf16(r1.z, x1.z, a);
            a = fma2_bf16(r1.w, x1.w, a);
            acc[j] = a;
        }
        ep.partial[c] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
};

// Per-warp shared memory: 3 mbarriers (stream slot 0, 1, raw bytes; warp 0
// keeps the fast table's in the fourth word) | 2 x (chunk_bits | stream span)
// | raw bytes (2048) | exponent word slots (EXP_WORDS rows of EXP_STRIDE
// bytes).
__host__ __device__ constexpr uint32_t warp_smem_bytes(uint32_t sbuf_bytes) {
    return 32u + 2u * (64u + sbuf_bytes) + GROUP_SYMS + EXP_BYTES;
}
static_assert(warp_smem_bytes(16u) % 16u == 0u, "per-warp shared areas must stay 16-byte aligned");

// Checks this thread's share of the fast table in shared memory (every
// entry of 2^fast_bits) and gives escapes the loop's escape word; true if an
// entry is malformed.
template <int NT>
__device__ __forceinline__ bool check_fast_table(uint2 *s_fast, uint32_t n_fast, uint32_t fast_bits, int tid) {
    bool bad = false;
    for (uint32_t i = tid; i < n_fast; i += NT) {
        uint2 e = s_fast[i];
        if (e.y & FAST_ESC) {
            bad |= e.y != FAST_ESC_WORD || e.x != 0u;
            s_fast[i].y = LANES_ESC_WORD;
        } else {
            const uint32_t cb = e.y & 255u, c8 = (e.y >> FAST_C8_SHIFT) & 255u,
                           ends = (e.y >> FAST_ENDS_SHIFT) & 0xFFFu;
            bad |= c8 == 0u || (c8 & 7u) || c8 > 8u * FAST_MAX_SYMS || cb == 0u || cb > fast_bits ||
                   8u * cb < c8 || (uint32_t)__popc(ends) * 8u != c8 || (ends >> (cb - 1u)) != 1u ||
                   (e.y & 0x70000000u) || (c8 < 32u && (e.x >> c8) != 0u);
        }
    }
    return bad;
}

template <int NT, class Epi>
__global__ void __launch_bounds__(NT) decode_lanes(const LanesParams prm, const typename Epi::Params ep) {
    constexpr int NWARP = NT / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t n_fast = 1u << prm.fast_bits;
    uint2 *s_fast = reinterpret_cast<uint2 *>(smem);
    const uint32_t wbytes = warp_smem_bytes(prm.sbuf_bytes);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint8_t *wbase = smem + (8u << prm.fast_bits) + warp * wbytes;
    const uint32_t bar_s0 = smem_u32(wbase), bar_m = bar_s0 + 16u;
    uint8_t *wslots = wbase + 32;
    const uint32_t slot_bytes = 64u + prm.sbuf_bytes;
    uint8_t *mbuf = wslots + 2u * slot_bytes;
    const uint32_t exps0 = smem_u32(mbuf + GROUP_SYMS), exps = exps0 + 4u * lane;  // word k at exps + EXP_STRIDE k
    const uint32_t *g_hier = prm.lut + 2u * n_fast;
    const uint32_t kshift = 32u - prm.fast_bits;
    // the next decode in a sequence may take SMs as this one's CTAs finish
    griddep_launch_dependents();

    // Warp slots are numbered warp-major across the CTAs, so when the groups
    // do not divide evenly the extra ones spread over all SMs rather than
    // piling onto the first CTAs.
    const uint32_t gstride = gridDim.x * NWARP;
    uint32_t g = (uint32_t)warp * gridDim.x + blockIdx.x;
    const bool active = g < prm.n_groups;
    uint32_t g1 = g + gstride;
    // this warp's first two group starts: their latency overlaps the table load
    uint64_t gs0 = 0, gs1 = 0, ns0 = 0, ns1 = 0;
    if (active) {
        gs0 = __ldg(prm.group_start + g);
        gs1 = __ldg(prm.group_start + g + 1);
        if (g1 < prm.n_groups) {
            ns0 = __ldg(prm.group_start + g1);
            ns1 = __ldg(prm.group_start + g1 + 1);
        }
    }

    // The fast table arrives in one bulk copy (tracked by the spare mbarrier
    // word of warp 0's area); the group copies go out only after it is in,
    // since issued earlier they slow it down and every warp waits for it.
    const uint32_t bar_t = smem_u32(smem + (8u << prm.fast_bits)) + 24u;
    if (lane == 0) {
        mbar_init(bar_s0, 1);
        mbar_init(bar_s0 + 8u, 1);
        mbar_init(bar_m, 1);
        if (tid == 0) mbar_init(bar_t, 1);
        fence_mbar_init();
        if (tid == 0) {
            mbar_expect_tx(bar_t, 8u << prm.fast_bits);
            bulk_load(smem_u32(s_fast), prm.lut, 8u << prm.fast_bits, bar_t);
        }
    }
    __syncthreads();  // the barriers are initialised
    bool tok = mbar_wait(bar_t, 0u);
    if (!__syncthreads_and(tok)) {  // the table copy never completed: give up
        if (tid == 0) {
            atomicOr(&g_status, ST_TIMEOUT);
            mbar_wait_bounded(bar_t, 0u);
        }
        return;
    }
    // check every entry; escapes get the loop's escape word
    const bool bad = check_fast_table<NT>(s_fast, n_fast, prm.fast_bits, tid);
    if (__syncthreads_or(bad)) {
        if (tid == 0) atomicOr(&g_status, ST_LUT);
        return;
    }
    if (!active) return;  // no CTA barrier follows

    // lane 0: chunk_bits and stream span of group gg into slot s
    auto issue_stream = [&](uint32_t gg, uint32_t s, uint64_t s0, uint64_t s1) {
        uint8_t *slot = wslots + s * slot_bytes;
        const uint32_t bar = bar_s0 + 8u * s;
        const uint64_t sb0 = (s0 >> 3) & ~15ull;
        uint32_t sbytes = 0;
        if (sb0 < prm.stream_bytes) {
            // a start past its end (a corrupt plan) copies a full slot; the
            // group is rejected before it is decoded
            const uint64_t d = s1 - s0;
            sbytes = min(span_bytes((uint32_t)s0 & 127u, d < (1u << 17) ? (uint32_t)d : (1u << 17)), prm.sbuf_bytes);
            sbytes = (uint32_t)min((uint64_t)sbytes, prm.stream_bytes - sb0);
        }
        const bool cb_ok = check(gg < prm.n_groups, CK_LANES_STREAM_COPY);
        const bool st_ok = check(sbytes <= prm.sbuf_bytes && (sbytes == 0u || sb0 + sbytes <= prm.stream_bytes),
                                 CK_LANES_STREAM_COPY);
        fence_proxy_async();
        mbar_expect_tx(bar, (cb_ok ? 64u : 0u) + (st_ok ? sbytes : 0u));
        if (cb_ok) bulk_load(smem_u32(slot), prm.chunk_bits + (size_t)gg * GROUP_CHUNKS, 64u, bar);
        if (st_ok && sbytes) bulk_load(smem_u32(slot + 64), prm.stream + sb0, sbytes, bar);
    };
    // lane 0: the group's raw bytes into the warp buffer
    auto issue_mant = [&](uint32_t gg) {
        const uint64_t m0 = (uint64_t)gg * GROUP_SYMS;
        const uint32_t bytes = (uint32_t)min((uint64_t)GROUP_SYMS, prm.mant_bytes - m0);
        const bool ok = check(m0 < prm.mant_bytes && m0 + bytes <= prm.mant_bytes, CK_LANES_MANT_COPY);
        fence_proxy_async();
        mbar_expect_tx(bar_m, ok ? bytes : 0u);
        if (ok) bulk_load(smem_u32(mbuf), prm.mant + m0, bytes, bar_m);
    };

    if (lane == 0) {
        issue_stream(g, 0, gs0, gs1);
        issue_mant(g);
    }

    for (uint32_t k = 0;; ++k) {
        const uint32_t s = k & 1u;
        const uint8_t *slot = wslots + s * slot_bytes;
        const bool has_next = g1 < prm.n_groups;
        const uint32_t g2 = g1 + gstride;
        __syncwarp();  // every lane is done with the other slot
        if (has_next && lane == 0) issue_stream(g1, s ^ 1u, ns0, ns1);

        bool ok = mbar_wait(bar_s0 + 8u * s, (k >> 1) & 1u);
        const uint32_t cbits = reinterpret_cast<const uint16_t *>(slot)[lane];
        uint32_t incl = cbits;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        const uint32_t excl = incl - cbits, gbits = __shfl_sync(0xFFFFFFFFu, incl, 31);
        const uint32_t c = g * GROUP_CHUNKS + lane;
        const uint32_t t = c + 1u < prm.n_chunks ? LANE_SYMS : (c + 1u == prm.n_chunks ? prm.last_t : 0u);
        const uint32_t r0 = (uint32_t)gs0 & 127u;  // first bit, from the copy's 16-byte boundary
        const uint32_t span = span_bytes(r0, gbits);  // gbits < 2^21; a valid group has <= 32 * 2048
        const bool valid = __all_sync(0xFFFFFFFFu, gs1 - gs0 == gbits && cbits <= 32u * LANE_SYMS &&
                                                       span <= prm.sbuf_bytes &&
                                                       ((gs0 >> 3) & ~15ull) + span <= prm.stream_bytes &&
                                                       (t != 0u || cbits == 0u));
        uint32_t err = 0;
        if (ok && valid && t) {
            const uint32_t r = r0 + excl;
            uint32_t rd_end, wr_end;
            const uint32_t end = decode_chunk(smem_u32(slot + 64), r, (int)(8u * t), smem_u32(s_fast), kshift,
                                              g_hier, prm.n_tables, exps, err, rd_end, wr_end);
            if (end != r + cbits) err |= ST_COUNT;
            check(rd_end <= smem_u32(wbase) + wbytes, CK_LANES_READ_END);
            check(wr_end < exps + EXP_STRIDE * EXP_WORDS, CK_LANES_SLOT_END);
        }
        // starts two groups ahead, for the copy issued next round: loaded
        // after the decode loop, so they hold no registers during it, and
        // before the join, which hides their latency
        uint64_t ms0 = 0, ms1 = 0;
        if (g2 < prm.n_groups) {
            ms0 = __ldg(prm.group_start + g2);
            ms1 = __ldg(prm.group_start + g2 + 1);
        }
        ok = mbar_wait(bar_m, k & 1u) && ok;
        if (!__all_sync(0xFFFFFFFFu, ok)) {  // a bulk copy never completed: give up
            if (lane == 0) {  // report, then give each copy in flight one more bounded wait
                atomicOr(&g_status, ST_TIMEOUT);
                mbar_wait_bounded(bar_s0 + 8u * s, (k >> 1) & 1u);
                mbar_wait_bounded(bar_m, k & 1u);
                if (has_next) mbar_wait_bounded(bar_s0 + 8u * (s ^ 1u), ((k + 1) >> 1) & 1u);
            }
            return;
        }
        const bool good = valid && !__any_sync(0xFFFFFFFFu, err != 0u);
        // the previous decode of a sequence owns the output until it ends:
        // wait once, before this warp's first store
        if (k == 0 && prm.wait_prior) griddep_wait();
        if (!valid) {
            if (lane == 0) atomicOr(&g_status, ST_RANGE);
        } else if (!good) {
            if (err) atomicOr(&g_status, err);
        } else {
            __syncwarp();  // the epilogue reads other lanes' exponent slots
            Epi::apply(prm, ep, lane, g, smem_u32(mbuf), exps0);
        }
        if (!has_next) break;
        __syncwarp();  // all lanes have read the raw bytes
        if (lane == 0) issue_mant(g1);
        g = g1;
        g1 = g2;
        gs0 = ns0;
        gs1 = ns1;
        ns0 = ms0;
        ns1 = ms1;
    }
}

// ------------------------------------------------------------ closed forms
//
// Two shapes of the canonical code decode without a table walk: two symbols
// with 1-bit codes (the stream is a bitmap, code 0 being the smaller symbol)
// and all 256 symbols with 8-bit codes (ordered by symbol, code s is symbol
// s: stream byte i is exponent i).  With every codeword L bits long, weight
// w's code starts at bit L w, so the 16 weights from a multiple of 16 have
// their codes in 2 L whole bytes; no plan is needed to find them.
constexpr uint32_t CLOSED_NONE = 0, CLOSED_BITMAP = 1, CLOSED_IDENTITY = 8;

// Which closed form a (validated) table has; for a bitmap, syms gets the
// symbols of codes 0 (bits 0..7) and 1 (bits 8..15).
inline uint32_t closed_form(const dfw_table *t, uint32_t &syms) {
    syms = 0;
    if (t->total_bits == 0 || (t->n_symbols != 2u && t->n_symbols != 256u)) return CLOSED_NONE;
    uint32_t k = 0, len = 0, s[2] = {0, 0};
    for (uint32_t e = 0; e < 256u; ++e) {
        if (!t->len[e]) continue;
        if (len && t->len[e] != len) return CLOSED_NONE;
        len = t->len[e];
        if (k < 2u) s[k] = e;
        ++k;
    }
    if (k == 2u && len == 1u) {
        syms = s[0] | (s[1] << 8);
        return CLOSED_BITMAP;
    }
    return k == 256u && len == 8u ? CLOSED_IDENTITY : CLOSED_NONE;
}

// Exponent bytes of four weights, each rotated as the joins take them.
__device__ __forceinline__ uint32_t rot4(uint32_t x) { return ((x >> 1) & 0x7F7F7F7Fu) | ((x << 7) & 0x80808080u); }

// The rotated exponents of the 16 weights from w (a multiple of 16 below the
// scope's n), four to a word: R[q] holds weights w + 4 q .. w + 4 q + 3.
// The stream holds at least ceil(L n / 8) + 16 bytes, so both reads stay in it.
__device__ __forceinline__ void closed_exps(uint32_t mode, const uint8_t *stream, uint32_t syms, uint64_t w,
                                            uint32_t (&R)[4]) {
    if (mode == CLOSED_IDENTITY) {
        const uint4 x = __ldcs(reinterpret_cast<const uint4 *>(stream + w));
        R[0] = rot4(x.x);
        R[1] = rot4(x.y);
        R[2] = rot4(x.z);
        R[3] = rot4(x.w);
        return;
    }
    // bitmap: bytes w / 8 and w / 8 + 1, weight w + j at bit 7 - j of the
    // first (MSB first); reversed, weight w + j is bit 24 + j, w + 8 + j bit 16 + j
    const uint32_t v = __brev((uint32_t)__ldcs(reinterpret_cast<const unsigned short *>(stream + (w >> 3))));
    const uint32_t e0 = rot_sym(syms & 0xFFu) * 0x01010101u, d = (rot_sym(syms >> 8) * 0x01010101u) ^ e0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t nib = (v >> (q < 2 ? 24 + 4 * q : 8 + 4 * q)) & 0xFu;  // weights w + 4 q .. + 3, bit j = w + 4 q + j
        const uint32_t mask = ((nib * 0x00204081u) & 0x01010101u) * 0xFFu;  // bit j -> byte j all ones
        R[q] = e0 ^ (d & mask);
    }
}

// A scope in a closed form, one thread per 16 weights (raw bytes, codes and
// output all whole 16- or 32-byte pieces).
__global__ void __launch_bounds__(256) decode_closed(const uint8_t *__restrict__ stream,
                                                     const uint8_t *__restrict__ mant, uint32_t mode, uint32_t syms,
                                                     uint64_t n, uint64_t stream_bytes, uint16_t *__restrict__ out,
                                                     uint32_t out32) {
    const uint64_t pieces = (n + 15u) >> 4;
    for (uint64_t p = (uint64_t)blockIdx.x * 256u + threadIdx.x; p < pieces; p += (uint64_t)gridDim.x * 256u) {
        const uint64_t w = p << 4;
        if (!check((mode == CLOSED_IDENTITY ? w + 16u : (w >> 3) + 2u) <= stream_bytes, CK_CLOSED_READ)) break;
        uint32_t R[4];
        closed_exps(mode, stream, syms, w, R);
        const uint4 m = __ldcs(reinterpret_cast<const uint4 *>(mant + w));  // raw bytes: a multiple of 16
        uint4 r0, r1;
        join4(R[0], m.x, r0.x, r0.y);
        join4(R[1], m.y, r0.z, r0.w);
        join4(R[2], m.z, r1.x, r1.y);
        join4(R[3], m.w, r1.z, r1.w);
        if (w + 16u <= n) {
            if (out32) {
                stg256_cs(out + w, r0, r1);
            } else {
                __stcs(reinterpret_cast<uint4 *>(out + w), r0);
                __stcs(reinterpret_cast<uint4 *>(out + w + 8u), r1);
            }
        } else {  // the scope's last weights, one at a time
            for (uint32_t q = 0; w + q < n; ++q) {
                const uint32_t mq = q < 4u ? m.x : q < 8u ? m.y : q < 12u ? m.z : m.w;
                const uint32_t rq = q < 4u ? R[0] : q < 8u ? R[1] : q < 12u ? R[2] : R[3];
                out[w + q] = join1(rq >> (8u * (q & 3u)), (mq >> (8u * (q & 3u))) & 0xFFu);
            }
        }
    }
}

// ------------------------------------------------------------ many scopes, one launch
//
// A sequence of code-table scopes (a model's blocks) decoded by one
// persistent launch into one output buffer.  Warp slot w (numbered
// warp-major across CTAs, as in decode_lanes) takes groups w, w + S, w + 2S,
// ... (S = resident warps) of every scope in turn, and within a group lane l
// always writes the same weights (store_group), so any output byte is written
// by one thread in every scope: the scopes' writes land in order by program
// order alone, and the buffer ends as k separate decodes in order would leave
// it, with no barrier between scopes across the grid.  Per scope each CTA
// loads that scope's fast table after a CTA barrier (every warp is done with
// the previous one); a warp's copies for its next group, which may belong to
// a later scope, are issued one group ahead as in decode_lanes, so they are
// in flight across the table switch.  One-exponent scopes are filled from
// their raw bytes with the same lane-to-weight layout.  Control flow over the
// scopes is uniform across the CTA: a warp whose copy wait gave up stops
// decoding but still takes every CTA barrier.

struct SeqScope {
    const uint8_t *stream;
    const uint8_t *mant;
    const uint32_t *lut;
    const uint16_t *chunk_bits;
    const uint64_t *group_start;
    uint64_t stream_bytes, mant_bytes;
    uint32_t n_chunks, n_groups;  // n_groups == 0: an empty scope
    uint32_t last_t;              // codewords in the last chunk (1..64)
    uint32_t fast_bits;           // 0: no table (one distinct exponent, or a closed form)
    uint32_t n_tables;            // hierarchy tables; the exponent of a one-exponent scope; a bitmap's symbols
    uint32_t closed;              // with fast_bits 0: CLOSED_BITMAP or CLOSED_IDENTITY (the stream is read)
};

constexpr uint32_t SEQ_MAX_SCOPES = DFW_SEQ_MAX_SCOPES;

struct SeqParams {
    uint16_t *out;
    uint32_t k;               // scopes in this launch
    uint32_t out32;           // out is 32-byte aligned
    uint32_t wait_prior;      // a programmatic dependent of an earlier decode into out
    uint32_t sbuf_bytes;      // stream slot bytes (the largest group span of the launch's scopes)
    uint32_t fast_bytes;      // shared bytes of the fast table (the largest of the launch's scopes)
    uint32_t reserved;
    SeqScope sc[SEQ_MAX_SCOPES];
};
static_assert(sizeof(SeqParams) <= 4096, "kernel parameters stay within the classic 4 KB limit");

// A scope without a table (one exponent, or a closed form): the warp's
// groups built from their raw bytes and, for a closed form, their codes.
__device__ __forceinline__ void fill_groups(const SeqScope &S, uint16_t *out, uint32_t out32, uint32_t slot0,
                                            uint32_t gstride, uint32_t lane) {
    const uint32_t C = rot_sym(S.n_tables) * 0x01010101u;
    const uint64_t n = (uint64_t)(S.n_chunks - 1u) * LANE_SYMS + S.last_t;
    for (uint32_t g = slot0; g < S.n_groups; g += gstride) {
        const uint64_t w0 = (uint64_t)g * GROUP_SYMS + 16u * lane;  // + 512 j
        for (int j = 0; j < 4; ++j) {
            const uint64_t w = w0 + 512u * j;
            if (w >= n) break;
            if (!check(w + 16u <= S.mant_bytes, CK_FILL_READ)) break;
            const uint4 m = __ldcs(reinterpret_cast<const uint4 *>(S.mant + w));  // w + 16 <= mant_bytes
            uint32_t R[4] = {C, C, C, C};
            if (S.closed) {
                if (!check((S.closed == CLOSED_IDENTITY ? w + 16u : (w >> 3) + 2u) <= S.stream_bytes, CK_CLOSED_READ))
                    break;
                closed_exps(S.closed, S.stream, S.n_tables, w, R);
            }
            uint4 r0, r1;
            join4(R[0], m.x, r0.x, r0.y);
            join4(R[1], m.y, r0.z, r0.w);
            join4(R[2], m.z, r1.x, r1.y);
            join4(R[3], m.w, r1.z, r1.w);
            if (w + 16u <= n) {
                if (out32) {
                    stg256_cs(out + w, r0, r1);
                } else {
                    __stcs(reinterpret_cast<uint4 *>(out + w), r0);
                    __stcs(reinterpret_cast<uint4 *>(out + w + 8u), r1);
                }
            } else {  // the scope's last weights, one at a time
                for (uint32_t q = 0; w + q < n; ++q) {
                    const uint32_t mq = q < 4u ? m.x : q < 8u ? m.y : q < 12u ? m.z : m.w;
                    const uint32_t rq = q < 4u ? R[0] : q < 8u ? R[1] : q < 12u ? R[2] : R[3];
                    out[w + q] = join1(rq >> (8u * (q & 3u)), (mq >> (8u * (q & 3u))) & 0xFFu);
                }
            }
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(NT, 1) decode_lanes_multi(const SeqParams P) {
    constexpr int NWARP = NT / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    uint2 *s_fast = reinterpret_cast<uint2 *>(smem);
    const uint32_t wbytes = warp_smem_bytes(P.sbuf_bytes);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint8_t *wbase = smem + P.fast_bytes + warp * wbytes;
    const uint32_t bar_s0 = smem_u32(wbase), bar_m = bar_s0 + 16u;
    uint8_t *wslots = wbase + 32;
    const uint32_t slot_bytes = 64u + P.sbuf_bytes;
    uint8_t *mbuf = wslots + 2u * slot_bytes;
    const uint32_t exps0 = smem_u32(mbuf + GROUP_SYMS), exps = exps0 + 4u * lane;
    const uint32_t bar_t = smem_u32(smem + P.fast_bytes) + 24u;  // spare word of warp 0's barriers
    griddep_launch_dependents();

    const uint32_t gstride = gridDim.x * NWARP;
    // this warp's slot, recomputed where needed (off the per-group path)
    auto slot_of = [&]() -> uint32_t { return (threadIdx.x >> 5) * gridDim.x + blockIdx.x; };
    // this warp's decode work is the sequence of (scope, group) pairs with a
    // stream: groups slot0, slot0 + gstride, ... of each such scope in turn
    auto first_from = [&](uint32_t j) -> uint32_t {
        const uint32_t slot0 = slot_of();
        while (j < P.k && (P.sc[j].fast_bits == 0u || slot0 >= P.sc[j].n_groups)) ++j;
        return j;
    };
    auto advance = [&](uint32_t &j, uint32_t &g) {
        g += gstride;
        if (g >= P.sc[j].n_groups) {
            j = first_from(j + 1u);
            g = slot_of();
        }
    };
    uint32_t jc = first_from(0), gc = slot_of();  // the group this warp decodes next (number kc)
    uint32_t jn = jc, gn = gc;                 // the one after it (kc + 1)
    if (jn < P.k) advance(jn, gn);
    // Group starts reach the lanes through shared memory: the 8 bytes at the
    // end of each exponent-slot row (bytes 128..135 of the 136) are never used
    // by the slots, so rows 0..3 hold the starts of group kc in pair kc & 1.
    // Lane 0 loads group kc + 2's starts after a decode loop, keeps them in
    // registers until the top of the next iteration (no decode loop in
    // between), then stores them and issues that group's stream copy.
    auto stash = [&](uint32_t pair, uint32_t which) { return exps0 + EXP_STRIDE * (2u * pair + which) + 128u; };
    auto lds64 = [](uint32_t a) {
        uint64_t v;
        asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(a) : "memory");
        return v;
    };
    auto sts64 = [](uint32_t a, uint64_t v) { asm volatile("st.shared.u64 [%0], %1;" ::"r"(a), "l"(v) : "memory"); };

    // The first scope with a table: its copy goes out right after the
    // barriers are set up (every warp waits for it; each warp's first group
    // copies follow once it is in, as in decode_lanes).
    uint32_t j0 = 0;
    while (j0 < P.k && (P.sc[j0].fast_bits == 0u || P.sc[j0].n_groups == 0u)) ++j0;
    if (lane == 0) {
        mbar_init(bar_s0, 1);
        mbar_init(bar_s0 + 8u, 1);
        mbar_init(bar_m, 1);
        if (tid == 0) mbar_init(bar_t, 1);
        fence_mbar_init();
        if (tid == 0 && j0 < P.k) {
            mbar_expect_tx(bar_t, 8u << P.sc[j0].fast_bits);
            bulk_load(smem_u32(s_fast), P.sc[j0].lut, 8u << P.sc[j0].fast_bits, bar_t);
        }
    }
    __syncthreads();  // the barriers are initialised

    // lane 0: chunk_bits and stream span of group gg of scope jj into slot s
    auto issue_stream = [&](uint32_t jj, uint32_t gg, uint32_t s, uint64_t s0, uint64_t s1) {
        const SeqScope &S = P.sc[jj];
        uint8_t *slot = wslots + s * slot_bytes;
        const uint32_t bar = bar_s0 + 8u * s;
        const uint64_t sb0 = (s0 >> 3) & ~15ull;
        uint32_t sbytes = 0;
        if (sb0 < S.stream_bytes) {
            const uint64_t d = s1 - s0;
            sbytes = min(span_bytes((uint32_t)s0 & 127u, d < (1u << 17) ? (uint32_t)d : (1u << 17)), P.sbuf_bytes);
            sbytes = (uint32_t)min((uint64_t)sbytes, S.stream_bytes - sb0);
        }
        const bool cb_ok = check(gg < S.n_groups, CK_LANES_STREAM_COPY);
        const bool st_ok = check(sbytes <= P.sbuf_bytes && (sbytes == 0u || sb0 + sbytes <= S.stream_bytes),
                                 CK_LANES_STREAM_COPY);
        fence_proxy_async();
        mbar_expect_tx(bar, (cb_ok ? 64u : 0u) + (st_ok ? sbytes : 0u));
        if (cb_ok) bulk_load(smem_u32(slot), S.chunk_bits + (size_t)gg * GROUP_CHUNKS, 64u, bar);
        if (st_ok && sbytes) bulk_load(smem_u32(slot + 64), S.stream + sb0, sbytes, bar);
    };
    // lane 0: the raw bytes of group gg of scope jj into the warp buffer
    auto issue_mant = [&](uint32_t jj, uint32_t gg) {
        const SeqScope &S = P.sc[jj];
        const uint64_t m0 = (uint64_t)gg * GROUP_SYMS;
        const uint32_t bytes = (uint32_t)min((uint64_t)GROUP_SYMS, S.mant_bytes - m0);
        const bool ok = check(m0 < S.mant_bytes && m0 + bytes <= S.mant_bytes, CK_LANES_MANT_COPY);
        fence_proxy_async();
        mbar_expect_tx(bar_m, ok ? bytes : 0u);
        if (ok) bulk_load(smem_u32(mbuf), S.mant + m0, bytes, bar_m);
    };
    uint64_t ms0 = 0, ms1 = 0;  // lane 0: the starts of group kc + 1, waiting to be stored and issued
    uint64_t a0 = 0, a1 = 0;    // lane 0: the first group's starts (its copies go out after the first table)
    if (lane == 0 && jc < P.k) {
        a0 = __ldg(P.sc[jc].group_start + gc);
        a1 = __ldg(P.sc[jc].group_start + gc + 1);
        if (jn < P.k) {
            ms0 = __ldg(P.sc[jn].group_start + gn);
            ms1 = __ldg(P.sc[jn].group_start + gn + 1);
        }
    }

    uint32_t kc = 0;        // groups this warp has taken (slot, phase and stash bookkeeping)
    uint32_t tphase = 0;    // phase of the table barrier
    // a launch chained after another decode into out holds its first store
    // (and everything after it) until that launch has completed
    if (P.wait_prior) griddep_wait();
    for (uint32_t j = 0; j < P.k; ++j) {  // uniform across the CTA
        const uint32_t fb = P.sc[j].fast_bits;
        if (P.sc[j].n_groups == 0u) continue;
        if (fb == 0u) {  // one distinct exponent: no table, no stream
            const uint32_t slot0 = slot_of();
            if (slot0 < P.sc[j].n_groups && jc <= P.k) fill_groups(P.sc[j], P.out, P.out32, slot0, gstride, lane);
            continue;
        }
        // scope j's fast table replaces the previous one once every warp is
        // done with it (the first one is already on its way)
        if (j != j0) {
            __syncthreads();
            if (tid == 0) {
                const bool ok = check((8u << fb) <= P.fast_bytes, CK_LANES_TABLE_COPY);
                fence_proxy_async();
                mbar_expect_tx(bar_t, ok ? 8u << fb : 0u);
                if (ok) bulk_load(smem_u32(s_fast), P.sc[j].lut, 8u << fb, bar_t);
            }
        }
        if (tid == 0) {
            for (uint32_t jj = j + 1u; jj < P.k; ++jj)  // the next table, into L2 meanwhile
                if (P.sc[jj].fast_bits && P.sc[jj].n_groups) {
                    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(P.sc[jj].lut),
                                 "r"(8u << P.sc[jj].fast_bits)
                                 : "memory");
                    break;
                }
        }
        const bool tok = mbar_wait(bar_t, tphase);
        tphase ^= 1u;
        if (!__syncthreads_and(tok)) {  // the table copy never completed: give up, after the copies in flight
            if (tid == 0) {
                atomicOr(&g_status, ST_TIMEOUT);
                mbar_wait_bounded(bar_t, tphase ^ 1u);
            }
            if (lane == 0 && jc < P.k && kc > 0u) {  // (a warp's first copies go out after the first table)
                mbar_wait_bounded(bar_s0 + 8u * (kc & 1u), (kc >> 1) & 1u);
                mbar_wait_bounded(bar_m, kc & 1u);
            }
            return;
        }
        const bool table_ok = !__syncthreads_or(check_fast_table<NT>(s_fast, 1u << fb, fb, tid));
        if (!table_ok && tid == 0) atomicOr(&g_status, ST_LUT);
        // Scope j's fields, read once here: j is the same across the CTA, so
        // these stay uniform values for the group loop below instead of
        // indexed parameter loads on every group.  The next group is in
        // scope j too except at a warp's last group of the scope.
        const uint8_t *const j_stream = P.sc[j].stream;
        const uint8_t *const j_mant = P.sc[j].mant;
        const uint32_t *const j_lut = P.sc[j].lut;
        const uint16_t *const j_chunk_bits = P.sc[j].chunk_bits;
        const uint64_t *const j_group_start = P.sc[j].group_start;
        const uint64_t j_stream_bytes = P.sc[j].stream_bytes, j_mant_bytes = P.sc[j].mant_bytes;
        const uint32_t j_n_chunks = P.sc[j].n_chunks, j_n_groups = P.sc[j].n_groups, j_last_t = P.sc[j].last_t;
        const uint32_t j_n_tables = P.sc[j].n_tables;
        // lane 0: copies of group gg (scope jj) into slot s; starts s0, s1
        auto issue_next_stream = [&](uint32_t jj, uint32_t gg, uint32_t s, uint64_t s0, uint64_t s1) {
            if (jj != j) {
                issue_stream(jj, gg, s, s0, s1);
                return;
            }
            uint8_t *slot = wslots + s * slot_bytes;
            const uint32_t bar = bar_s0 + 8u * s;
            const uint64_t sb0 = (s0 >> 3) & ~15ull;
            uint32_t sbytes = 0;
            if (sb0 < j_stream_bytes) {
                const uint64_t d = s1 - s0;
                sbytes = min(span_bytes((uint32_t)s0 & 127u, d < (1u << 17) ? (uint32_t)d : (1u << 17)),
                             P.sbuf_bytes);
                sbytes = (uint32_t)min((uint64_t)sbytes, j_stream_bytes - sb0);
            }
            const bool cb_ok = check(gg < j_n_groups, CK_LANES_STREAM_COPY);
            const bool st_ok = check(sbytes <= P.sbuf_bytes && (sbytes == 0u || sb0 + sbytes <= j_stream_bytes),
                                     CK_LANES_STREAM_COPY);
            fence_proxy_async();
            mbar_expect_tx(bar, (cb_ok ? 64u : 0u) + (st_ok ? sbytes : 0u));
            if (cb_ok) bulk_load(smem_u32(slot), j_chunk_bits + (size_t)gg * GROUP_CHUNKS, 64u, bar);
            if (st_ok && sbytes) bulk_load(smem_u32(slot + 64), j_stream + sb0, sbytes, bar);
        };
        auto issue_next_mant = [&](uint32_t jj, uint32_t gg) {
            if (jj != j) {
                issue_mant(jj, gg);
                return;
            }
            const uint64_t m0 = (uint64_t)gg * GROUP_SYMS;
            const uint32_t bytes = (uint32_t)min((uint64_t)GROUP_SYMS, j_mant_bytes - m0);
            const bool ok = check(m0 < j_mant_bytes && m0 + bytes <= j_mant_bytes, CK_LANES_MANT_COPY);
            fence_proxy_async();
            mbar_expect_tx(bar_m, ok ? bytes : 0u);
            if (ok) bulk_load(smem_u32(mbuf), j_mant + m0, bytes, bar_m);
        };

        if (kc == 0u && jc == j && lane == 0) {  // the warp's first group: its starts and copies
            sts64(stash(0, 0), a0);
            sts64(stash(0, 1), a1);
            issue_next_stream(jc, gc, 0, a0, a1);
            issue_next_mant(jc, gc);
        }
        while (jc == j) {  // this warp's groups of scope j
            const uint32_t s = kc & 1u;
            const uint8_t *slot = wslots + s * slot_bytes;
            const bool has_next = jn < P.k;
            __syncwarp();  // every lane is done with the other slot and with stash pair s ^ 1
            if (has_next && lane == 0) {
                sts64(stash(s ^ 1u, 0), ms0);
                sts64(stash(s ^ 1u, 1), ms1);
                issue_next_stream(jn, gn, s ^ 1u, ms0, ms1);
            }

            bool ok = mbar_wait(bar_s0 + 8u * s, (kc >> 1) & 1u);
            const uint64_t gs0 = lds64(stash(s, 0)), gs1 = lds64(stash(s, 1));
            const uint32_t cbits = reinterpret_cast<const uint16_t *>(slot)[lane];
            uint32_t incl = cbits;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
                if (lane >= d) incl += y;
            }
            const uint32_t excl = incl - cbits, gbits = __shfl_sync(0xFFFFFFFFu, incl, 31);
            const uint32_t c = gc * GROUP_CHUNKS + lane;
            const uint32_t t = c + 1u < j_n_chunks ? LANE_SYMS : (c + 1u == j_n_chunks ? j_last_t : 0u);
            const uint32_t r0 = (uint32_t)gs0 & 127u;
            const uint32_t span = span_bytes(r0, gbits);
            const bool valid = __all_sync(0xFFFFFFFFu, gs1 - gs0 == gbits && cbits <= 32u * LANE_SYMS &&
                                                           span <= P.sbuf_bytes &&
                                                           ((gs0 >> 3) & ~15ull) + span <= j_stream_bytes &&
                                                           (t != 0u || cbits == 0u));
            uint32_t err = 0;
            if (ok && valid && table_ok && t) {
                const uint32_t r = r0 + excl;
                uint32_t rd_end, wr_end;
                const uint32_t end = decode_chunk(smem_u32(slot + 64), r, (int)(8u * t), smem_u32(s_fast), 32u - fb,
                                                  j_lut + (2u << fb), j_n_tables, exps, err, rd_end, wr_end);
                if (end != r + cbits) err |= ST_COUNT;
                check(rd_end <= smem_u32(wbase) + wbytes, CK_LANES_READ_END);
                check(wr_end < exps + EXP_STRIDE * EXP_WORDS, CK_LANES_SLOT_END);
            }
            // move on: the current group is kept only as gcur (for the store);
            // (jc, gc) becomes the next group, (jn, gn) the one after it, whose
            // starts lane 0 loads now
            const uint32_t gcur = gc;
            jc = jn;
            gc = gn;
            if (has_next) {
                gn += gstride;
                if (gn >= (jn == j ? j_n_groups : P.sc[jn].n_groups)) {
                    jn = first_from(jn + 1u);
                    gn = slot_of();
                }
                if (jn < P.k && lane == 0) {
                    const uint64_t *gsp = (jn == j ? j_group_start : P.sc[jn].group_start) + gn;
                    ms0 = __ldg(gsp);
                    ms1 = __ldg(gsp + 1);
                }
            }
            ok = mbar_wait(bar_m, kc & 1u) && ok;
            if (!__all_sync(0xFFFFFFFFu, ok)) {  // a copy never completed: this warp stops decoding
                if (lane == 0) {
                    atomicOr(&g_status, ST_TIMEOUT);
                    mbar_wait_bounded(bar_s0 + 8u * s, (kc >> 1) & 1u);
                    mbar_wait_bounded(bar_m, kc & 1u);
                    if (has_next) mbar_wait_bounded(bar_s0 + 8u * (s ^ 1u), ((kc + 1) >> 1) & 1u);
                }
                jc = P.k + 1u;  // past every scope: no more groups, no fills; the CTA barriers still come
                break;
            }
            const bool good = valid && table_ok && !__any_sync(0xFFFFFFFFu, err != 0u);
            if (!valid) {
                if (lane == 0) atomicOr(&g_status, ST_RANGE);
            } else if (good) {
                __syncwarp();  // the join reads other lanes' exponent slots
                store_group(P.out, P.out32, j_n_chunks, j_last_t, lane, gcur, smem_u32(mbuf), exps0);
            } else if (err) {
                atomicOr(&g_status, err);
            }
            __syncwarp();  // all lanes have read the raw bytes
            if (has_next && lane == 0) issue_next_mant(jc, gc);
            ++kc;
        }
    }
}

template <int NT>
uint32_t lanes_multi_smem(uint32_t fast_bytes, uint32_t sbuf_bytes) {
    return fast_bytes + (NT / 32) * warp_smem_bytes(sbuf_bytes);
}

struct MultiVariant {
    int nt;
    void (*fn)(const SeqParams);
    uint32_t (*smem)(uint32_t, uint32_t);
    int smem_set[16];
};
static MultiVariant g_multi[5] = {
    {1024, decode_lanes_multi<1024>, lanes_multi_smem<1024>, {0}},
    {768, decode_lanes_multi<768>, lanes_multi_smem<768>, {0}},
    {512, decode_lanes_multi<512>, lanes_multi_smem<512>, {0}},
    {256, decode_lanes_multi<256>, lanes_multi_smem<256>, {0}},
    {128, decode_lanes_multi<128>, lanes_multi_smem<128>, {0}},
};

// The largest CTA whose shared memory fits (fast table + per-warp areas);
// -1 if none does.
int multi_variant(uint32_t fast_bytes, uint32_t sbuf_bytes) {
    for (int i = 0; i < 5; ++i)
        if (g_multi[i].smem(fast_bytes, sbuf_bytes) <= 227u * 1024u) return i;
    return -1;
}

template <int NT>
uint32_t lanes_smem(uint32_t fast_bits, uint32_t sbuf_bytes) {
    return (8u << fast_bits) + (NT / 32) * warp_smem_bytes(sbuf_bytes);
}

// One table of CTA shapes per epilogue, largest CTA first: a larger CTA
// shares one copy of the fast table among more warps; data with long codes
// needs bigger stream slots and falls back to a smaller CTA.
template <class Epi>
struct LanesVariants {
    typedef void (*fn_t)(const LanesParams, const typename Epi::Params);
    struct V {
        int nt;
        fn_t fn;
        uint32_t (*smem)(uint32_t, uint32_t);
        int smem_set[16];  // dynamic shared memory opted in, per device
    };
    static V v[5];
};
template <class Epi>
typename LanesVariants<Epi>::V LanesVariants<Epi>::v[5] = {
    {1024, decode_lanes<1024, Epi>, lanes_smem<1024>, {0}},
    {768, decode_lanes<768, Epi>, lanes_smem<768>, {0}},
    {512, decode_lanes<512, Epi>, lanes_smem<512>, {0}},
    {256, decode_lanes<256, Epi>, lanes_smem<256>, {0}},
    {128, decode_lanes<128, Epi>, lanes_smem<128>, {0}},
};

// pdl: launch as a programmatic dependent of the previous kernel on the
// stream (prm.wait_prior must then be set).
template <class Epi>
dfw_status launch_lanes(const LanesParams &prm, const typename Epi::Params &ep, uint64_t n_groups, cudaStream_t s,
                        int sms, bool pdl = false) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return DFW_ECUDA;
    for (auto &v : LanesVariants<Epi>::v) {
        const uint32_t smem = v.smem(prm.fast_bits, prm.sbuf_bytes);
        if (smem > 227u * 1024u) continue;
        if (!v.smem_set[dev]) {
            if (cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
                return DFW_ECUDA;
            v.smem_set[dev] = 1;
        }
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v.fn, v.nt, smem) != cudaSuccess) return DFW_ECUDA;
        if (per_sm < 1) continue;
        const uint64_t wpc = (uint64_t)v.nt / 32;
        const uint64_t warps = (uint64_t)per_sm * sms * wpc;
        const uint64_t want = n_groups < warps ? n_groups : warps;
        const unsigned grid = (unsigned)((want + wpc - 1) / wpc);
        if (!pdl) {
            v.fn<<<grid, v.nt, smem, s>>>(prm, ep);
            return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3((unsigned)v.nt);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, v.fn, prm, ep) == cudaSuccess ? DFW_OK : DFW_ECUDA;
    }
    return DFW_EINVAL;  // even the smallest CTA does not fit
}

// A scope in a closed form: decode_closed over its 16-weight pieces.
dfw_status launch_closed(const LanesParams &prm, uint32_t mode, uint32_t syms, uint64_t n, cudaStream_t s, int sms) {
    const uint64_t want = (((n + 15u) >> 4) + 255u) / 256u, cap = (uint64_t)sms * 8u;
    decode_closed<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(prm.stream, prm.mant, mode, syms, n,
                                                                        prm.stream_bytes, prm.out, prm.out32);
    return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
}

// Checks a known-start plan against its table and fills the kernel
// parameters (out left null).
dfw_status lanes_params(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                        const uint16_t *d_chunk_bits, const uint64_t *d_group_start, const dfw_table *table,
                        const dfw_lanes_info *info, LanesParams &prm) {
    const uint64_t n = table->n;
    if (info->chunk_symbols != LANE_SYMS || info->group_chunks != GROUP_CHUNKS ||
        info->n_chunks != (n + LANE_SYMS - 1) / LANE_SYMS ||
        info->n_groups != (info->n_chunks + GROUP_CHUNKS - 1) / GROUP_CHUNKS || info->n_chunks >= (1ull << 32))
        return DFW_EINVAL;
    const uint32_t fb = info->fast_bits;
    if (fb < (uint32_t)FAST_BITS_MIN || fb > (uint32_t)FAST_BITS_MAX || info->lut_tables < 1 ||
        info->lut_words != (2u << fb) + 256u * info->lut_tables)
        return DFW_EINVAL;
    if (!d_stream || !d_lut || !d_chunk_bits || !d_group_start) return DFW_EINVAL;
    if ((reinterpret_cast<uintptr_t>(d_stream) | reinterpret_cast<uintptr_t>(d_lut) |
         reinterpret_cast<uintptr_t>(d_chunk_bits) | reinterpret_cast<uintptr_t>(d_group_start)) & 15u)
        return DFW_EALIGN;
    if (info->max_group_bytes < 16 || (info->max_group_bytes & 15u) || info->max_group_bytes > 64u * 1024u)
        return DFW_EINVAL;
    prm.stream = d_stream;
    prm.mant = d_mant;
    prm.lut = d_lut;
    prm.chunk_bits = d_chunk_bits;
    prm.group_start = d_group_start;
    prm.out = nullptr;
    prm.n_chunks = (uint32_t)info->n_chunks;
    prm.n_groups = (uint32_t)info->n_groups;
    prm.last_t = (uint32_t)(n - LANE_SYMS * (info->n_chunks - 1));
    prm.stream_bytes = table->stream_bytes;
    prm.mant_bytes = (n + 15) & ~15ull;
    prm.fast_bits = fb;
    prm.n_tables = info->lut_tables;
    prm.sbuf_bytes = info->max_group_bytes;
    prm.out32 = 0u;
    prm.wait_prior = 0u;
    return DFW_OK;
}

// y = W x, one warp per output row: the row's chunk partials summed lane by
// lane, then a fixed xor tree (the same order on every run).
struct RowsParams {
    uint32_t k;
    uint32_t per_row[GEMV_MAX_TENSORS];     // chunks per row (columns / 64)
    uint64_t chunk0[GEMV_MAX_TENSORS];      // first chunk of each tensor
    uint64_t row0[GEMV_MAX_TENSORS + 1];    // rows before each tensor
    float *y[GEMV_MAX_TENSORS];
    const float *partial;
};

__global__ void __launch_bounds__(256) gemv_rows(const RowsParams rp) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint64_t total = rp.row0[rp.k];
    const uint64_t wstride = (uint64_t)gridDim.x * 8u;
    for (uint64_t R = (uint64_t)blockIdx.x * 8u + (threadIdx.x >> 5); R < total; R += wstride) {
        uint32_t ti = 0;
#pragma unroll
        for (uint32_t i = 1; i < GEMV_MAX_TENSORS; ++i)
            if (i < rp.k && R >= rp.row0[i]) ti = i;
        const uint64_t r = R - rp.row0[ti];
        const uint32_t per = rp.per_row[ti];
        const float *p = rp.partial + rp.chunk0[ti] + r * per;
        float sum = 0.f;
        for (uint32_t j = lane; j < per; j += 32) sum += p[j];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, d);
        if (lane == 0) rp.y[ti][r] = sum;
    }
}

// Partials for a one-exponent scope (no stream): every weight is (sym, raw byte).
__global__ void __launch_bounds__(256) gemv_single_partials(const uint8_t *__restrict__ mant, uint32_t sym,
                                                            uint32_t n_chunks, const DotEpi::Params ep) {
    const uint32_t R = rot_sym(sym) * 0x01010101u;
    for (uint32_t c = blockIdx.x * 256u + threadIdx.x; c < n_chunks; c += gridDim.x * 256u) {
        const uint64_t w0 = (uint64_t)c * LANE_SYMS;
        uint32_t ti = 0;
#pragma unroll
        for (uint32_t i = 1; i < GEMV_MAX_TENSORS; ++i)
            if (i < ep.k && w0 >= ep.off[i]) ti = i;
        const uint32_t col0 = (uint32_t)(w0 - ep.off[ti]) % ep.cols[ti];
        const uint16_t *xp = ep.x[ti] + col0;
        float acc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 m = __ldg(reinterpret_cast<const uint4 *>(mant + w0) + q);
            uint4 r0, r1, x0, x1;
            ldg256_nc(xp + 16u * q, x0, x1);
            join4(R, m.x, r0.x, r0.y);
            join4(R, m.y, r0.z, r0.w);
            join4(R, m.z, r1.x, r1.y);
            join4(R, m.w, r1.z, r1.w);
            float a = 0.f;
            a = fma2_bf16(r0.x, x0.x, a);
            a = fma2_bf16(r0.y, x0.y, a);
            a = fma2_bf16(r0.z, x0.z, a);
            a = fma2_bf16(r0.w, x0.w, a);
            a = fma2_bf16(r1.x, x1.x, a);
            a = fma2_bf16(r1.y, x1.y, a);
            a = fma2_bf16(r1.z, x1.z, a);
            a = fma2_bf16(r1.w, x1.w, a);
            acc[q] = a;
        }
        ep.partial[c] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
}

}  // namespace

dfw_status launch_decode_lanes(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                               const uint16_t *d_chunk_bits, const uint64_t *d_group_start, const dfw_table *table,
                               const dfw_lanes_info *info, uint16_t *d_out, cudaStream_t s, int sms) {
    LanesParams prm;
    const dfw_status st = lanes_params(d_stream, d_mant, d_lut, d_chunk_bits, d_group_start, table, info, prm);
    if (st != DFW_OK) return st;
    prm.out = d_out;
    prm.out32 = (reinterpret_cast<uintptr_t>(d_out) & 31u) == 0u;
    uint32_t syms = 0;
    if (const uint32_t mode = closed_form(table, syms)) return launch_closed(prm, mode, syms, table->n, s, sms);
    return launch_lanes<StoreEpi>(prm, StoreEpi::Params{}, info->n_groups, s, sms);
}

// launches: if not null, receives the number of launches; dry: count them,
// launch nothing (no GPU call is made).
dfw_status launch_decode_lanes_seq(int k, const dfw_lanes_scope *scopes, uint16_t *d_out, cudaStream_t s, int sms,
                                   int *launches, bool dry) {
    // every scope is checked before the first launch
    for (int i = 0; i < k; ++i) {
        const dfw_lanes_scope &sc = scopes[i];
        dfw_status st = validate_table(sc.table);
        if (st != DFW_OK) return st;
        if (!sc.info || !sc.d_mant) return DFW_EINVAL;
        if (reinterpret_cast<uintptr_t>(sc.d_mant) & 15u) return DFW_EALIGN;
        if (sc.table->n == 0 || sc.table->total_bits == 0) continue;
        LanesParams prm;
        st = lanes_params(sc.d_stream, sc.d_mant, sc.d_lut, sc.d_chunk_bits, sc.d_group_start, sc.table, sc.info, prm);
        if (st != DFW_OK) return st;
    }
    int dev = 0;
    if (!dry && (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16)) return DFW_ECUDA;
    if (launches) *launches = 0;
    // One launch per run of consecutive scopes (at most SEQ_MAX_SCOPES) that
    // the same CTA shape serves: a scope whose table or group spans would
    // need a smaller CTA than the run so far starts a new run.
    SeqParams P;
    std::memset(&P, 0, sizeof(P));
    uint32_t groups_max = 0, fast_bytes = 0, sbuf = 16;
    int run_var = -1;
    bool prior = false;  // a launch into d_out is already on the stream from this call
    int solo = -1;  // the scope index of a run's only scope
    auto flush = [&]() -> dfw_status {
        if (P.k == 0) return DFW_OK;
        if (launches) ++*launches;
        if (dry) {
            std::memset(&P, 0, sizeof(P));
            groups_max = 0;
            fast_bytes = 0;
            sbuf = 16;
            run_var = -1;
            return DFW_OK;
        }
        if (P.k == 1 && (P.sc[0].fast_bits != 0u || P.sc[0].closed)) {
            // a run of one scope with a table or in a closed form: the
            // one-scope kernels, which have no scope bookkeeping (same output;
            // after a prior launch the table kernel is its programmatic
            // dependent and holds its stores, the closed-form kernel simply
            // follows it on the stream)
            const dfw_lanes_scope &sc = scopes[solo];
            LanesParams prm;
            lanes_params(sc.d_stream, sc.d_mant, sc.d_lut, sc.d_chunk_bits, sc.d_group_start, sc.table, sc.info, prm);
            prm.out = d_out;
            prm.out32 = (reinterpret_cast<uintptr_t>(d_out) & 31u) == 0u;
            prm.wait_prior = prior ? 1u : 0u;
            const dfw_status st = P.sc[0].closed
                                      ? launch_closed(prm, P.sc[0].closed, P.sc[0].n_tables, sc.table->n, s, sms)
                                      : launch_lanes<StoreEpi>(prm, StoreEpi::Params{}, sc.info->n_groups, s, sms, prior);
            if (st != DFW_OK) return st;
            prior = true;
            std::memset(&P, 0, sizeof(P));
            groups_max = 0;
            fast_bytes = 0;
            sbuf = 16;
            run_var = -1;
            return DFW_OK;
        }
        const int vi = run_var < 0 ? 0 : run_var;
        MultiVariant &v = g_multi[vi];
        const uint32_t smem = v.smem(fast_bytes, sbuf);
        if (!v.smem_set[dev]) {
            if (cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
                return DFW_ECUDA;
            v.smem_set[dev] = 1;
        }
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v.fn, v.nt, smem) != cudaSuccess) return DFW_ECUDA;
        if (per_sm < 1) return DFW_EINVAL;
        const uint64_t wpc = (uint64_t)v.nt / 32, warps = (uint64_t)per_sm * sms * wpc;
        const uint64_t want = groups_max < warps ? groups_max : warps;
        P.out = d_out;
        P.out32 = (reinterpret_cast<uintptr_t>(d_out) & 31u) == 0u;
        P.wait_prior = prior ? 1u : 0u;
        P.sbuf_bytes = sbuf;
        P.fast_bytes = fast_bytes;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((want + wpc - 1) / wpc));
        cfg.blockDim = dim3((unsigned)v.nt);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = prior ? 1 : 0;
        if (cudaLaunchKernelEx(&cfg, v.fn, P) != cudaSuccess) return DFW_ECUDA;
        prior = true;
        std::memset(&P, 0, sizeof(P));
        groups_max = 0;
        fast_bytes = 0;
        sbuf = 16;
        run_var = -1;
        return DFW_OK;
    };
    for (int i = 0; i < k; ++i) {
        const dfw_lanes_scope &sc = scopes[i];
        const uint64_t n = sc.table->n;
        if (n == 0) continue;
        SeqScope q;
        std::memset(&q, 0, sizeof(q));
        const uint64_t n_chunks = (n + LANE_SYMS - 1) / LANE_SYMS;
        const uint64_t n_groups = (n_chunks + GROUP_CHUNKS - 1) / GROUP_CHUNKS;
        if (n_chunks >= (1ull << 32)) return DFW_EINVAL;
        q.mant = sc.d_mant;
        q.mant_bytes = (n + 15) & ~15ull;
        q.n_chunks = (uint32_t)n_chunks;
        q.n_groups = (uint32_t)n_groups;
        q.last_t = (uint32_t)(n - LANE_SYMS * (n_chunks - 1));
        uint32_t fb_bytes = 0, sb = 16, syms = 0;
        if (sc.table->total_bits == 0) {  // one distinct exponent: a fill
            q.fast_bits = 0;
            q.n_tables = sc.table->single_symbol;
        } else if (const uint32_t mode = closed_form(sc.table, syms)) {  // codes read in place: no table
            q.stream = sc.d_stream;
            q.stream_bytes = sc.table->stream_bytes;
            q.fast_bits = 0;
            q.n_tables = syms;
            q.closed = mode;
        } else {
            LanesParams prm;
            lanes_params(sc.d_stream, sc.d_mant, sc.d_lut, sc.d_chunk_bits, sc.d_group_start, sc.table, sc.info, prm);
            q.stream = prm.stream;
            q.lut = prm.lut;
            q.chunk_bits = prm.chunk_bits;
            q.group_start = prm.group_start;
            q.stream_bytes = prm.stream_bytes;
            q.fast_bits = prm.fast_bits;
            q.n_tables = prm.n_tables;
            fb_bytes = 8u << prm.fast_bits;
            sb = prm.sbuf_bytes;
        }
        const uint32_t nf = fast_bytes > fb_bytes ? fast_bytes : fb_bytes, ns = sbuf > sb ? sbuf : sb;
        const bool fill = q.fast_bits == 0u;  // needs no table or slot: joins any run
        const int alone = fill && P.k > 0 ? run_var : multi_variant(fb_bytes, sb), joined = multi_variant(nf, ns);
        if (alone < 0) return DFW_EINVAL;  // even the smallest CTA does not fit
        if (P.k > 0 && (P.k == SEQ_MAX_SCOPES || joined != run_var || alone != run_var)) {
            const dfw_status st = flush();
            if (st != DFW_OK) return st;
        }
        if (P.k == 0) {
            run_var = alone;
            fast_bytes = fb_bytes;
            sbuf = sb;
        } else {
            fast_bytes = nf;
            sbuf = ns;
        }
        if (P.k == 0) solo = i;
        P.sc[P.k++] = q;
        if (q.n_groups > groups_max) groups_max = q.n_groups;
    }
    return flush();
}

dfw_status launch_gemv_lanes(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                             const uint16_t *d_chunk_bits, const uint64_t *d_group_start, const dfw_table *table,
                             const dfw_lanes_info *info, int k, const uint64_t *tensor_offsets, const uint32_t *cols,
                             const uint16_t *const *d_x, float *const *d_y, float *d_partial, uint64_t partial_elems,
                             cudaStream_t s, int sms) {
    const uint64_t n = table->n;
    if (k < 1 || k > (int)GEMV_MAX_TENSORS || !tensor_offsets || !cols || !d_x || !d_y || !d_partial)
        return DFW_EINVAL;
    if (tensor_offsets[0] != 0 || tensor_offsets[k] != n) return DFW_EINVAL;
    const uint64_t n_chunks = n / LANE_SYMS;
    if (partial_elems < n_chunks) return DFW_ENOMEM;
    DotEpi::Params ep;
    RowsParams rp;
    std::memset(&ep, 0, sizeof(ep));
    std::memset(&rp, 0, sizeof(rp));
    ep.k = rp.k = (uint32_t)k;
    ep.partial = d_partial;
    rp.partial = d_partial;
    for (int i = 0; i < k; ++i) {
        const uint64_t size = tensor_offsets[i + 1] - tensor_offsets[i];
        if (tensor_offsets[i + 1] <= tensor_offsets[i] || cols[i] == 0 || cols[i] % LANE_SYMS || size % cols[i] ||
            size >= (1ull << 32) || !d_x[i] || !d_y[i])
            return DFW_EINVAL;
        if ((reinterpret_cast<uintptr_t>(d_x[i]) & 31u) || (reinterpret_cast<uintptr_t>(d_y[i]) & 3u))
            return DFW_EALIGN;
        ep.cols[i] = cols[i];
        ep.off[i] = tensor_offsets[i];
        ep.x[i] = d_x[i];
        rp.per_row[i] = cols[i] / LANE_SYMS;
        rp.chunk0[i] = tensor_offsets[i] / LANE_SYMS;
        rp.row0[i + 1] = rp.row0[i] + size / cols[i];
        rp.y[i] = d_y[i];
    }
    ep.off[k] = n;
    if (!d_mant || (reinterpret_cast<uintptr_t>(d_mant) & 15u) || (reinterpret_cast<uintptr_t>(d_partial) & 15u))
        return d_mant ? DFW_EALIGN : DFW_EINVAL;
    if (table->total_bits == 0) {  // one distinct exponent: no stream, no plan needed
        const uint64_t want = (n_chunks + 255) / 256, cap = (uint64_t)sms * 8;
        gemv_single_partials<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(d_mant, table->single_symbol,
                                                                                 (uint32_t)n_chunks, ep);
        if (cudaGetLastError() != cudaSuccess) return DFW_ECUDA;
    } else {
        LanesParams prm;
        const dfw_status st = lanes_params(d_stream, d_mant, d_lut, d_chunk_bits, d_group_start, table, info, prm);
        if (st != DFW_OK) return st;
        const dfw_status st2 = launch_lanes<DotEpi>(prm, ep, info->n_groups, s, sms);
        if (st2 != DFW_OK) return st2;
    }
    const uint64_t rows = rp.row0[k];
    const uint64_t want = (rows + 7) / 8, cap = (uint64_t)sms * 16;
    gemv_rows<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(rp);
    return cudaGetLastError() == cudaSuccess ? DFW_OK : DFW_ECUDA;
}

}  // namespace dfw
