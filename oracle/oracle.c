/*
 * oracle.c -- plain, slow, CPU oracle for entropy-coded bf16 weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this file's library.  The
 * product (libdfw and its Python binding) never links, imports or calls it,
 * and it shares no code, header, table or constant with the product.
 *
 * What the method computes (sources):
 *   - "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
 *     Inference via Dynamic-Length Float" (DFloat11), abstract: bf16 weights
 *     have low-entropy exponents; entropy coding gives each value a
 *     frequency-based variable-length code; decoding is bit-for-bit exact;
 *     the GPU decoder coordinates thread read/write positions with small
 *     auxiliary arrays.
 *   - "From a Lossless (~1.5:1) Compression Algorithm for Llama2 7B Weights
 *     ...", abstract: lossless ~1.5:1 on Llama2-7B bf16 weights.
 *   - The LazyWeights write-up (bedrocknews.com, arXiv 2611.17108v1) and the
 *     Huff-LLM abstract: the entropy code is Huffman.
 * The pages leave the exact format open; the readings taken here are:
 *   R1 exponent = bits 14..7 of the bf16 pattern, raw byte = sign<<7 | mant7;
 *   R2 code lengths = optimal length-limited prefix code (package-merge,
 *      Larmore & Hirschberg 1990) with cap `cap` (<= 32), leaves ordered by
 *      (count, symbol), and on equal weight a leaf is merged before a package;
 *   R3 one distinct exponent -> length 0, empty bitstream;
 *   R4 canonical codewords in (length, symbol) order (RFC 1951 sec. 3.2.2);
 *   R5 codewords written MSB-first, first bit into bit 7 of byte 0; the byte
 *      stream is zero-padded to a multiple of 64 bytes plus 16 guard bytes;
 *   R6 aux: for a window of W bytes starting at bit 8*W*t, gap[t] is the
 *      distance from the window start to the first code start at or after
 *      it (or to total_bits when no code starts there); for a tile of T
 *      windows, out_start[b] counts the code starts before bit 8*W*T*b, and
 *      out_start[n_tiles] = n.
 *   R7 known-start chunks (the per-chunk bit offsets of a second decode
 *      plan): chunk_bits[c] = bits of codewords Mc .. M(c+1)-1, and
 *      group_start[g] = first bit of codeword MGg.
 * Parity: every function here is pinned by tests in tests/test_oracle_*.py
 * (round trip, Kraft equality, entropy bounds, brute-force optimality,
 * closed forms, independent recounts).  The tie rule of R2 is this
 * library's reading, pinned only by a hand-worked tie case.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_EINVAL 1
#define OR_ECAP 2
#define OR_ENOMEM 3
#define OR_ECORRUPT 4

/* ---- R1: split each bf16 pattern into exponent and sign+mantissa bytes. */
void oracle_split(const uint16_t *u, uint64_t n, uint8_t *e, uint8_t *m)
{
    for (uint64_t i = 0; i < n; i++) {
        uint16_t x = u[i];
        e[i] = (uint8_t)((x >> 7) & 0xFFu);
        m[i] = (uint8_t)(((x >> 8) & 0x80u) | (x & 0x7Fu));
    }
}

/* Inverse of the split: sign from bit 7 of m, exponent e, mantissa m&0x7F. */
uint16_t oracle_join(uint8_t e, uint8_t m)
{
    return (uint16_t)(((uint32_t)(m & 0x80u) << 8) | ((uint32_t)e << 7) | (m & 0x7Fu));
}

/* ---- frequency count that drives the code ("based on frequency"). */
void oracle_histogram(const uint8_t *e, uint64_t n, uint64_t hist[256])
{
    for (int s = 0; s < 256; s++)
        hist[s] = 0;
    for (uint64_t i = 0; i < n; i++)
        hist[e[i]]++;
}

/* ---- R2: package-merge.  Each list item carries how often every symbol
 * occurs inside it, so a symbol's code length is read off directly as the
 * number of times it occurs among the selected items. */
typedef struct {
    uint64_t weight;
    int leaf;
    uint16_t mult[256];
} pm_item;

int oracle_code_lengths(const uint64_t hist[256], int cap, uint8_t len[256])
{
    memset(len, 0, 256);
    if (cap < 1 || cap > 32)
        return OR_EINVAL;
    int k = 0;
    for (int s = 0; s < 256; s++)
        if (hist[s] > 0)
            k++;
    if (k <= 1)
        return OR_OK; /* R3: zero or one symbol needs no bits */
    if (cap < 9 && (1 << cap) < k)
        return OR_ECAP; /* no prefix code of k words fits in cap bits */

    pm_item *leaves = (pm_item *)calloc((size_t)k, sizeof(pm_item));
    pm_item *cur = (pm_item *)calloc((size_t)(2 * k), sizeof(pm_item));
    pm_item *nxt = (pm_item *)calloc((size_t)(2 * k), sizeof(pm_item));
    pm_item *pkg = (pm_item *)calloc((size_t)k, sizeof(pm_item));
    if (!leaves || !cur || !nxt || !pkg) {
        free(leaves); free(cur); free(nxt); free(pkg);
        return OR_ENOMEM;
    }
    /* leaves in symbol order, then a stable insertion sort by count, which
     * gives (count, symbol) order */
    int nl = 0;
    for (int s = 0; s < 256; s++) {
        if (hist[s] == 0)
            continue;
        leaves[nl].weight = hist[s];
        leaves[nl].leaf = 1;
        leaves[nl].mult[s] = 1;
        nl++;
    }
    for (int i = 1; i < k; i++) {
        pm_item tmp = leaves[i];
        int j = i - 1;
        while (j >= 0 && leaves[j].weight > tmp.weight) {
            leaves[j + 1] = leaves[j];
            j--;
        }
        leaves[j + 1] = tmp;
    }

    int ncur = k;
    memcpy(cur, leaves, (size_t)k * sizeof(pm_item));
    for (int iter = 1; iter <= cap - 1; iter++) {
        /* package adjacent pairs; an unpaired last item is dropped */
        int np = ncur / 2;
        for (int i = 0; i < np; i++) {
            pkg[i].weight = cur[2 * i].weight + cur[2 * i + 1].weight;
            pkg[i].leaf = 0;
            for (int s = 0; s < 256; s++)
                pkg[i].mult[s] = (uint16_t)(cur[2 * i].mult[s] + cur[2 * i + 1].mult[s]);
        }
        /* merge packages with the leaves; a leaf goes first on equal weight */
        int i = 0, j = 0, o = 0;
        while (i < k || j < np) {
            if (j >= np || (i < k && leaves[i].weight <= pkg[j].weight))
                nxt[o++] = leaves[i++];
            else
                nxt[o++] = pkg[j++];
        }
        pm_item *t = cur;
        cur = nxt;
        nxt = t;
        ncur = o;
    }
    /* the 2k-2 cheapest items of the final list */
    for (int i = 0; i < 2 * k - 2; i++)
        for (int s = 0; s < 256; s++)
            len[s] = (uint8_t)(len[s] + cur[i].mult[s]);

    free(leaves); free(cur); free(nxt); free(pkg);
    return OR_OK;
}

/* ---- R4: canonical codewords, RFC 1951 sec. 3.2.2. */
void oracle_canonical_codes(const uint8_t len[256], uint32_t code[256])
{
    uint64_t bl_count[34];
    uint64_t next_code[34];
    for (int b = 0; b < 34; b++)
        bl_count[b] = next_code[b] = 0;
    for (int s = 0; s < 256; s++)
        if (len[s] > 0)
            bl_count[len[s]]++;
    uint64_t c = 0;
    for (int bits = 1; bits <= 32; bits++) {
        c = (c + bl_count[bits - 1]) << 1;
        next_code[bits] = c;
    }
    for (int s = 0; s < 256; s++) {
        code[s] = 0;
        if (len[s] > 0)
            code[s] = (uint32_t)next_code[len[s]]++;
    }
}

/* ---- R5: padded stream length for a given number of coded bits. */
uint64_t oracle_stream_bytes(uint64_t total_bits)
{
    uint64_t raw = (total_bits + 7) / 8;
    return (raw + 63) / 64 * 64 + 16;
}

/* ---- R5: MSB-first packing, one bit at a time. */
int oracle_pack(const uint8_t *e, uint64_t n, const uint8_t len[256], const uint32_t code[256],
                uint8_t *stream, uint64_t stream_cap, uint64_t *total_bits_out)
{
    uint64_t tb = 0;
    for (uint64_t i = 0; i < n; i++)
        tb += len[e[i]];
    uint64_t need = oracle_stream_bytes(tb);
    if (stream_cap < need)
        return OR_ENOMEM;
    memset(stream, 0, (size_t)need);
    uint64_t pos = 0;
    for (uint64_t i = 0; i < n; i++) {
        int l = len[e[i]];
        uint32_t c = code[e[i]];
        for (int b = l - 1; b >= 0; b--) {
            if ((c >> b) & 1u)
                stream[pos >> 3] |= (uint8_t)(0x80u >> (pos & 7));
            pos++;
        }
    }
    *total_bits_out = tb;
    return OR_OK;
}

/* Whole encoder: split, histogram, lengths, codes, pack. */
int oracle_encode(const uint16_t *u, uint64_t n, int cap, uint8_t *stream, uint64_t stream_cap,
                  uint8_t *mant, uint8_t len_out[256], uint64_t *total_bits_out)
{
    uint8_t *e = (uint8_t *)malloc(n ? (size_t)n : 1);
    if (!e)
        return OR_ENOMEM;
    oracle_split(u, n, e, mant);
    uint64_t hist[256];
    oracle_histogram(e, n, hist);
    int rc = oracle_code_lengths(hist, cap, len_out);
    if (rc != OR_OK) {
        free(e);
        return rc;
    }
    uint32_t code[256];
    oracle_canonical_codes(len_out, code);
    rc = oracle_pack(e, n, len_out, code, stream, stream_cap, total_bits_out);
    free(e);
    return rc;
}

/* ---- textbook canonical decoder state: per length, the first codeword,
 * the number of codewords, and where its symbols start in the list of
 * symbols sorted by (length, symbol). */
typedef struct {
    uint64_t first[33];
    uint64_t count[33];
    uint64_t base[33];
    uint8_t sorted[256];
    int k;
    int single;
} canon_dec;

static void canon_init(const uint8_t len[256], canon_dec *d)
{
    memset(d, 0, sizeof(*d));
    d->single = -1;
    for (int s = 0; s < 256; s++)
        if (len[s] > 0)
            d->count[len[s]]++;
    uint64_t c = 0, idx = 0;
    for (int l = 1; l <= 32; l++) {
        c = (c + d->count[l - 1]) << 1;
        d->first[l] = c;
        d->base[l] = idx;
        for (int s = 0; s < 256; s++)
            if (len[s] == l)
                d->sorted[idx++] = (uint8_t)s;
    }
    d->k = (int)idx;
}

/* Reads one codeword bit by bit starting at *pos; returns the symbol or -1. */
static int canon_read(const canon_dec *d, const uint8_t *stream, uint64_t total_bits, uint64_t *pos)
{
    uint64_t code = 0;
    for (int l = 1; l <= 32; l++) {
        if (*pos >= total_bits)
            return -1;
        uint64_t bit = (stream[*pos >> 3] >> (7 - (*pos & 7))) & 1u;
        code = (code << 1) | bit;
        (*pos)++;
        if (d->count[l] > 0 && code >= d->first[l] && code - d->first[l] < d->count[l])
            return d->sorted[d->base[l] + (code - d->first[l])];
    }
    return -1;
}

/* ---- bit-serial decoder: emits exactly n weights; the coded bits must be
 * used up exactly.  single_symbol is the exponent when the table has one
 * symbol (R3) and is ignored otherwise. */
int oracle_decode(const uint8_t *stream, uint64_t total_bits, const uint8_t len[256],
                  int single_symbol, const uint8_t *mant, uint64_t n, uint16_t *out)
{
    canon_dec d;
    canon_init(len, &d);
    if (d.k == 0) {
        if (total_bits != 0)
            return OR_ECORRUPT;
        if (n > 0 && (single_symbol < 0 || single_symbol > 255))
            return OR_EINVAL;
        for (uint64_t i = 0; i < n; i++)
            out[i] = oracle_join((uint8_t)single_symbol, mant[i]);
        return OR_OK;
    }
    uint64_t pos = 0;
    for (uint64_t i = 0; i < n; i++) {
        int s = canon_read(&d, stream, total_bits, &pos);
        if (s < 0)
            return OR_ECORRUPT;
        out[i] = oracle_join((uint8_t)s, mant[i]);
    }
    return pos == total_bits ? OR_OK : OR_ECORRUPT;
}

/* Decodes the exponent symbols only, from bit `start_bit`, for `count`
 * symbols (used to check a sampled tile of a large stream). */
int oracle_decode_symbols(const uint8_t *stream, uint64_t total_bits, const uint8_t len[256],
                          uint64_t start_bit, uint64_t count, uint8_t *sym_out)
{
    canon_dec d;
    canon_init(len, &d);
    if (d.k == 0)
        return count == 0 ? OR_OK : OR_EINVAL;
    uint64_t pos = start_bit;
    for (uint64_t i = 0; i < count; i++) {
        int s = canon_read(&d, stream, total_bits, &pos);
        if (s < 0)
            return OR_ECORRUPT;
        sym_out[i] = (uint8_t)s;
    }
    return OR_OK;
}

/* ---- R6: auxiliary arrays, from the list of code start positions. */
uint64_t oracle_n_windows(uint64_t total_bits, uint64_t W)
{
    return (total_bits + 8 * W - 1) / (8 * W);
}

int oracle_aux(const uint8_t *stream, uint64_t total_bits, const uint8_t len[256], uint64_t n,
               uint64_t W, uint64_t T, uint8_t *gap, uint64_t *out_start)
{
    if (W == 0 || T == 0)
        return OR_EINVAL;
    uint64_t nwin = oracle_n_windows(total_bits, W);
    uint64_t ntiles = (nwin + T - 1) / T;
    uint64_t t = 0, b = 0, count = 0, pos = 0;
    canon_dec d;
    canon_init(len, &d);
    /* visit the code starts in order; every window (tile) not yet given a
     * value takes the first start at or after its own first bit */
    while (pos < total_bits) {
        while (t < nwin && 8 * W * t <= pos) {
            gap[t] = (uint8_t)(pos - 8 * W * t);
            t++;
        }
        while (b < ntiles && 8 * W * T * b <= pos) {
            out_start[b] = count;
            b++;
        }
        if (canon_read(&d, stream, total_bits, &pos) < 0)
            return OR_ECORRUPT;
        count++;
        if (count > n)
            return OR_ECORRUPT;
    }
    if (total_bits > 0 && count != n)
        return OR_ECORRUPT;
    for (; t < nwin; t++)
        gap[t] = (uint8_t)(total_bits - 8 * W * t);
    for (; b < ntiles; b++)
        out_start[b] = n;
    out_start[ntiles] = n;
    return OR_OK;
}

/* ---- R7 (known-start chunks): codeword i starts at bit start(i), with
 * start(n) = total_bits.  For chunks of M codewords, chunk_bits[c] =
 * start(min(M(c+1), n)) - start(Mc); for groups of G chunks,
 * group_start[g] = start(MGg) and group_start[n_groups] = total_bits.
 * chunk_bits has n_groups * G entries; the ones past the last chunk are 0. */
int oracle_chunk_aux(const uint8_t *stream, uint64_t total_bits, const uint8_t len[256], uint64_t n,
                     uint64_t M, uint64_t G, uint32_t *chunk_bits, uint64_t *group_start)
{
    if (M == 0 || G == 0)
        return OR_EINVAL;
    uint64_t n_chunks = (n + M - 1) / M;
    uint64_t n_groups = (n_chunks + G - 1) / G;
    for (uint64_t c = 0; c < n_groups * G; c++)
        chunk_bits[c] = 0;
    canon_dec d;
    canon_init(len, &d);
    uint64_t pos = 0, chunk_start = 0;
    for (uint64_t i = 0; i < n; i++) {
        if (i % M == 0) {
            chunk_start = pos;
            if (i % (M * G) == 0)
                group_start[i / (M * G)] = pos;
        }
        if (total_bits > 0 && canon_read(&d, stream, total_bits, &pos) < 0)
            return OR_ECORRUPT;
        if ((i + 1) % M == 0 || i + 1 == n)
            chunk_bits[i / M] = (uint32_t)(pos - chunk_start);
    }
    if (pos != total_bits)
        return OR_ECORRUPT;
    group_start[n_groups] = total_bits;
    return OR_OK;
}

/* ======================================================================
 * rANS variant of the exponent coder (the ANS "bridge" of the ~1.5:1 page's
 * abstract; the LazyWeights write-up compares Huffman with rANS).  The pages
 * give no format; the readings taken here:
 *   R8  range ANS (Duda, "Asymmetric numeral systems", 2013) with a state x
 *       in [L, L * 2^16), L = 2^16, renormalised 16 bits at a time;
 *       symbol s with quantised frequency f_s and cumulative start c_s
 *       (sum of f over smaller symbols; the f_s sum to M = 2^scale_bits)
 *       encodes as x' = floor(x / f_s) * M + (x mod f_s) + c_s, after
 *       emitting the low 16 bits of x while x >= f_s * (L / M) * 2^16;
 *       decoding inverts it: slot = x mod M, s is the symbol whose
 *       [c_s, c_s + f_s) holds slot, x = f_s * floor(x / M) + slot - c_s,
 *       then while x < L: x = x * 2^16 + next word.
 *   R9  frequencies: f_s = max(1, floor(count_s * M / n)) for every present
 *       symbol, 0 for absent ones; the remainder M - sum f goes to the most
 *       frequent symbol (smallest symbol on ties) if positive; if negative,
 *       1 is taken repeatedly from the symbol with the largest f_s > 1
 *       (smallest symbol on ties).
 *   R10 interleaving: the symbols are cut into blocks of block_syms; in a
 *       block, symbol i belongs to state i mod I (I states, "lanes").  The
 *       encoder walks the block backwards (i = last .. 0), so that a decoder
 *       taking steps k = 0, 1, ... decodes symbols I k .. I k + I - 1 (one
 *       per state) and then renormalises the states in increasing state
 *       order, each taking the next word of the block.  A block is: I final
 *       encoder states (u32, little-endian), its words in decode order (u16,
 *       little-endian), zero padding to a multiple of 16 bytes.  Every state
 *       starts at L, so a decoder must end with every state at L and every
 *       word consumed.
 * ====================================================================== */

#define RANS_L 65536u

int oracle_rans_freqs(const uint64_t hist[256], int scale_bits, uint32_t freq[256])
{
    if (scale_bits < 8 || scale_bits > 16)
        return OR_EINVAL;
    const uint64_t M = 1ull << scale_bits;
    uint64_t n = 0;
    for (int s = 0; s < 256; s++)
        n += hist[s];
    for (int s = 0; s < 256; s++)
        freq[s] = 0;
    if (n == 0)
        return OR_OK;
    int64_t sum = 0;
    for (int s = 0; s < 256; s++) {
        if (!hist[s])
            continue;
        /* floor(count * M / n) without overflow: count <= n < 2^64, M <= 2^16 */
        const unsigned __int128 q = ((unsigned __int128)hist[s] * M) / n;
        freq[s] = q ? (uint32_t)q : 1u;
        sum += freq[s];
    }
    int64_t d = (int64_t)M - sum;
    if (d > 0) {
        int best = -1;
        for (int s = 0; s < 256; s++)
            if (hist[s] && (best < 0 || hist[s] > hist[best]))
                best = s;
        freq[best] += (uint32_t)d;
    }
    while (d < 0) {
        int best = -1;
        for (int s = 0; s < 256; s++)
            if (freq[s] > 1 && (best < 0 || freq[s] > freq[best]))
                best = s;
        if (best < 0)
            return OR_EINVAL; /* more symbols than M slots */
        freq[best]--;
        d++;
    }
    return OR_OK;
}

static void rans_cum(const uint32_t freq[256], uint32_t cum[257])
{
    cum[0] = 0;
    for (int s = 0; s < 256; s++)
        cum[s + 1] = cum[s] + freq[s];
}

/* Bytes of one block's encoding for `lanes` states and `words` words. */
static uint64_t rans_block_bytes(uint32_t lanes, uint64_t words)
{
    return (4ull * lanes + 2ull * words + 15) & ~15ull;
}

/* Encodes exponent symbols e[0..n) (every symbol must have freq > 0).
 * block_start receives n_blocks + 1 byte offsets. */
int oracle_rans_encode(const uint8_t *e, uint64_t n, const uint32_t freq[256], int scale_bits,
                       uint32_t lanes, uint32_t block_syms, uint8_t *out, uint64_t out_cap,
                       uint64_t *block_start, uint64_t *out_bytes)
{
    if (lanes < 1 || lanes > 64 || block_syms < lanes || block_syms % lanes || scale_bits < 8 ||
        scale_bits > 16)
        return OR_EINVAL;
    uint32_t cum[257];
    rans_cum(freq, cum);
    if (n && cum[256] != (1u << scale_bits))
        return OR_EINVAL;
    const uint64_t n_blocks = (n + block_syms - 1) / block_syms;
    uint16_t *stack = (uint16_t *)malloc(sizeof(uint16_t) * (block_syms + 1));
    if (!stack)
        return OR_ENOMEM;
    uint64_t pos = 0;
    for (uint64_t b = 0; b < n_blocks; b++) {
        block_start[b] = pos;
        const uint64_t i0 = b * block_syms;
        const uint64_t cnt = n - i0 < block_syms ? n - i0 : block_syms;
        uint32_t x[64];
        for (uint32_t j = 0; j < lanes; j++)
            x[j] = RANS_L;
        uint64_t words = 0;
        for (uint64_t ii = cnt; ii-- > 0;) {
            const uint32_t j = (uint32_t)(ii % lanes);
            const uint8_t s = e[i0 + ii];
            const uint32_t f = freq[s];
            if (f == 0) {
                free(stack);
                return OR_EINVAL;
            }
            const uint64_t x_max = ((uint64_t)(RANS_L >> scale_bits) << 16) * f;
            if (x[j] >= x_max) {
                stack[words++] = (uint16_t)(x[j] & 0xFFFFu);
                x[j] >>= 16;
            }
            x[j] = ((x[j] / f) << scale_bits) + (x[j] % f) + cum[s];
        }
        const uint64_t bytes = rans_block_bytes(lanes, words);
        if (pos + bytes > out_cap) {
            free(stack);
            return OR_ENOMEM;
        }
        uint8_t *p = out + pos;
        memset(p, 0, bytes);
        for (uint32_t j = 0; j < lanes; j++)
            for (int k = 0; k < 4; k++)
                p[4 * j + k] = (uint8_t)(x[j] >> (8 * k));
        for (uint64_t w = 0; w < words; w++) { /* decode order = reverse of emission */
            const uint16_t v = stack[words - 1 - w];
            p[4 * lanes + 2 * w] = (uint8_t)(v & 0xFF);
            p[4 * lanes + 2 * w + 1] = (uint8_t)(v >> 8);
        }
        pos += bytes;
    }
    block_start[n_blocks] = pos;
    *out_bytes = pos;
    free(stack);
    return OR_OK;
}

/* Decodes n symbols; OR_ECORRUPT if a block does not end with every state at
 * L and every word consumed, or reads past its end. */
int oracle_rans_decode(const uint8_t *stream, const uint64_t *block_start, uint64_t n,
                       const uint32_t freq[256], int scale_bits, uint32_t lanes, uint32_t block_syms,
                       uint8_t *e)
{
    if (lanes < 1 || lanes > 64 || block_syms < lanes || block_syms % lanes || scale_bits < 8 ||
        scale_bits > 16)
        return OR_EINVAL;
    uint32_t cum[257];
    rans_cum(freq, cum);
    const uint32_t M = 1u << scale_bits;
    if (n && cum[256] != M)
        return OR_EINVAL;
    const uint64_t n_blocks = (n + block_syms - 1) / block_syms;
    for (uint64_t b = 0; b < n_blocks; b++) {
        const uint8_t *p = stream + block_start[b];
        const uint64_t bytes = block_start[b + 1] - block_start[b];
        if (bytes < 4ull * lanes)
            return OR_ECORRUPT;
        const uint64_t max_words = (bytes - 4ull * lanes) / 2;
        const uint64_t i0 = b * block_syms;
        const uint64_t cnt = n - i0 < block_syms ? n - i0 : block_syms;
        uint32_t x[64];
        for (uint32_t j = 0; j < lanes; j++)
            x[j] = (uint32_t)p[4 * j] | ((uint32_t)p[4 * j + 1] << 8) | ((uint32_t)p[4 * j + 2] << 16) |
                   ((uint32_t)p[4 * j + 3] << 24);
        uint64_t w = 0;
        for (uint64_t k = 0; k * lanes < cnt; k++) {
            for (uint32_t j = 0; j < lanes && k * lanes + j < cnt; j++) {
                const uint32_t slot = x[j] & (M - 1);
                int s = 0;
                while (!(cum[s] <= slot && slot < cum[s + 1]))
                    s++;
                e[i0 + k * lanes + j] = (uint8_t)s;
                x[j] = freq[s] * (x[j] >> scale_bits) + slot - cum[s];
            }
            for (uint32_t j = 0; j < lanes && k * lanes + j < cnt; j++) {
                if (x[j] < RANS_L) {
                    if (w >= max_words)
                        return OR_ECORRUPT;
                    const uint32_t v = (uint32_t)p[4 * lanes + 2 * w] | ((uint32_t)p[4 * lanes + 2 * w + 1] << 8);
                    x[j] = (x[j] << 16) | v;
                    w++;
                }
            }
        }
        for (uint32_t j = 0; j < lanes; j++)
            if (x[j] != RANS_L)
                return OR_ECORRUPT;
        if (rans_block_bytes(lanes, w) != bytes)
            return OR_ECORRUPT;
    }
    return OR_OK;
}
