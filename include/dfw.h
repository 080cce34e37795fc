/*
 * dfw.h -- C ABI of libdfw: lossless entropy-coded bf16 weights, decoded on
 * an NVIDIA B200 (sm_100a).
 *
 * The method (sources are the pages this library restates; see each call):
 *   "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
 *   Inference via Dynamic-Length Float" (DFloat11), abstract -- bf16 weights
 *   carry low-entropy exponents; entropy coding assigns frequency-based
 *   variable-length codes; the GPU decoder (i) keeps compact lookup tables
 *   in on-chip SRAM, (ii) coordinates thread read/write positions in two
 *   phases with small auxiliary arrays, (iii) decompresses a whole
 *   transformer block at a time; the output is bit-for-bit identical.
 *   "From a Lossless (~1.5:1) Compression Algorithm for Llama2 7B Weights
 *   ...", abstract -- ~1.5:1 on Llama2-7B bf16 weights.
 *   The LazyWeights write-up (bedrocknews.com, arXiv 2611.17108v1) and the
 *   Huff-LLM abstract -- the entropy code is Huffman.
 *
 * FORMAT (the pages leave it open; this library fixes it):
 *   - Each bf16 bit pattern u splits into an exponent symbol
 *     e = (u >> 7) & 0xFF and a raw byte m = ((u >> 8) & 0x80) | (u & 0x7F);
 *     u = ((m & 0x80) << 8) | (e << 7) | (m & 0x7F).
 *   - The exponents get an optimal prefix code whose lengths are capped at
 *     `cap` bits (1..32), computed by package-merge with leaves ordered by
 *     (count, symbol) and leaves merged before packages on equal weight.
 *     One distinct exponent gets length 0 and an empty stream.
 *   - Codewords are canonical: assigned in (length, symbol) order as in
 *     RFC 1951 section 3.2.2.
 *   - The stream is the codewords of e[0], e[1], ... written MSB-first (the
 *     first bit is bit 7 of byte 0), zero-padded to a multiple of 64 bytes,
 *     followed by 16 zero guard bytes (DFW_STREAM_PAD).
 *   - The raw bytes m[0..n) are stored as they are, zero-padded to a
 *     multiple of 16 bytes (dfw_mant_bytes).
 *
 * DECODE PLAN (auxiliary arrays, DFloat11 abstract point (ii)):
 *   - The stream is cut into windows of W bytes; window t covers bits
 *     [8Wt, 8W(t+1)).  gap[t] (one byte) = distance from the window start to
 *     the first codeword that starts at or after it, or to total_bits if
 *     none does.  Since no codeword exceeds 32 bits, gap[t] < 32.
 *   - T consecutive windows form a tile, decoded by one CTA.
 *     out_start[b] (u64) = number of codewords that start before bit 8WTb,
 *     i.e. the output index of the tile's first weight; out_start[n_tiles]
 *     = n.
 *   - lut (DFloat11 abstract point (i): compact tables in on-chip SRAM) holds
 *     two parts.  First a fast table of 2^K 64-bit entries (K = fast_bits,
 *     8..12) keyed by the next K stream bits at a codeword start: it lists up
 *     to four whole codewords inside those K bits (their symbols, how many,
 *     the bits they use and where each ends) or marks an escape when the
 *     first codeword is longer than K bits.  Its symbols are stored rotated
 *     right by one bit, (e >> 1) | (e << 7) mod 256: bits 6..0 are then the
 *     bf16 pattern's high byte below the sign and bit 7 the top bit of its low
 *     byte, so the decoder assembles bf16 with byte masks alone.  Then a hierarchy of 256-entry
 *     tables keyed by successive bytes of the code: table 0 resolves every
 *     codeword of at most 8 bits and points to a subtable for longer ones (at
 *     most four levels for 32-bit codes); escapes are resolved through it.
 *
 * MEMORY AND OWNERSHIP: the caller allocates every buffer (host or device).
 * libdfw keeps no pointer after a call returns.  Device pointers must be
 * 16-byte aligned (DFW_EALIGN otherwise).  Decode calls are asynchronous on
 * the given CUDA stream; the caller keeps the buffers alive until the
 * stream's work completes.
 *
 * ERRORS: every call returns a dfw_status.  Host-side validation happens
 * before any launch.  Corruption that only the device can see (a tile whose
 * decoded symbol count disagrees with out_start, a table entry that points
 * outside the table, out_start out of order) is recorded in a per-device
 * status word, the damaged tile writes nothing, and dfw_check reports it.
 * Kernels never wait without bound and never trap.
 */
#ifndef DFW_H
#define DFW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dfw_status {
    DFW_OK = 0,
    DFW_EINVAL = 1,   /* an argument is out of range or inconsistent */
    DFW_ECAP = 2,     /* 2^cap is smaller than the number of distinct exponents */
    DFW_ENOMEM = 3,   /* a caller buffer is too small, or a host allocation failed */
    DFW_ECORRUPT = 4, /* stream, aux or table are inconsistent with each other */
    DFW_EALIGN = 5,   /* a device pointer is not 16-byte aligned */
    DFW_ECUDA = 6     /* a CUDA runtime call failed (launch or copy) */
} dfw_status;

#define DFW_FORMAT_VERSION 1u
#define DFW_MAX_CAP 32
#define DFW_STREAM_PAD 16 /* guard bytes after the 64-byte-rounded stream */

/* Code table and stream metadata written by dfw_encode / dfw_encode_multi. */
typedef struct dfw_table {
    uint32_t version;       /* DFW_FORMAT_VERSION */
    uint32_t cap;           /* length cap the lengths were built with */
    uint64_t n;             /* number of weights */
    uint64_t total_bits;    /* coded exponent bits (without padding) */
    uint64_t stream_bytes;  /* padded stream length in bytes */
    uint32_t n_symbols;     /* distinct exponents (0 only when n == 0) */
    uint32_t single_symbol; /* the exponent when n_symbols == 1, else 0 */
    uint8_t len[256];       /* code length per exponent, 0 = absent */
} dfw_table;

/* Shape of a decode plan, written by dfw_plan_query and completed by dfw_plan. */
typedef struct dfw_plan_info {
    uint32_t window_bytes;     /* W: bytes of stream per window */
    uint32_t tile_windows;     /* T: windows per tile (one tile per CTA) */
    uint64_t n_windows;        /* ceil(total_bits / 8W) windows; gap[] holds n_tiles * T bytes */
    uint64_t n_tiles;          /* ceil(n_windows / T): out_start[] has n_tiles + 1 */
    uint64_t max_tile_symbols; /* largest out_start[b+1] - out_start[b] (dfw_plan) */
    uint32_t lut_words;        /* u32 words of the LUT image: 2 * 2^fast_bits + 256 * lut_tables */
    uint32_t lut_tables;       /* 256-entry byte-keyed tables after the fast table */
    uint32_t fast_bits;        /* K: key width of the fast table (dfw_plan_query sets 10) */
    uint32_t reserved;         /* zero */
} dfw_plan_info;

/* Worst-case padded stream bytes for n weights (every code 32 bits long). */
uint64_t dfw_stream_bound(uint64_t n);

/* Padded raw-byte (sign+mantissa) array length for n weights. */
uint64_t dfw_mant_bytes(uint64_t n);

/*
 * dfw_encode -- split, histogram, capped canonical code, MSB-first packing.
 * Source: DFloat11 abstract (frequency-based dynamic-length encodings of
 * bf16 exponents); Huffman per the LazyWeights write-up.  Host only.
 *   bf16        host, n bf16 bit patterns (read only)
 *   cap         length cap, 1..32
 *   stream      host, stream_capacity bytes; receives table->stream_bytes
 *   mant        host, mant_capacity bytes; receives dfw_mant_bytes(n) bytes
 *   table       receives the code table and stream metadata
 *   n_threads   worker threads (0 = all hardware threads); the output is
 *               byte-identical for every thread count
 * Errors: DFW_EINVAL (null pointer, cap out of range), DFW_ECAP, DFW_ENOMEM
 * (table->stream_bytes then holds the size needed).
 */
dfw_status dfw_encode(const uint16_t *bf16, uint64_t n, int cap, uint8_t *stream,
                      uint64_t stream_capacity, uint8_t *mant, uint64_t mant_capacity,
                      dfw_table *table, int n_threads);

/*
 * dfw_encode_multi -- one code table over the concatenation of k tensors
 * (a transformer block; DFloat11 abstract point (iii)).  The stream and the
 * raw bytes are those of the concatenation in the given order.
 *   tensors[i]       host pointer to sizes[i] bf16 patterns
 *   tensor_offsets   host, k + 1 entries: prefix sums of sizes (output)
 * Other arguments and errors as dfw_encode.
 */
dfw_status dfw_encode_multi(const uint16_t *const *tensors, const uint64_t *sizes, int k, int cap,
                            uint8_t *stream, uint64_t stream_capacity, uint8_t *mant,
                            uint64_t mant_capacity, dfw_table *table, uint64_t *tensor_offsets,
                            int n_threads);

/*
 * dfw_plan_query -- sizes of the plan arrays for a table and (W, T), before
 * allocation.  Supported: W in {8, 16}, T in {128, 256, 512}, W * T <= 4096
 * (a tile's worst case must fit in shared memory).  Fills every
 * field of info except max_tile_symbols, with fast_bits = 10; a caller may
 * set fast_bits to another value in 8..12 and call again with it filled in
 * (a nonzero info->fast_bits on entry is kept).  Errors: DFW_EINVAL.
 */
dfw_status dfw_plan_query(const dfw_table *table, uint32_t window_bytes, uint32_t tile_windows,
                          dfw_plan_info *info);

/*
 * dfw_plan -- auxiliary arrays and LUT image for one stream (DFloat11
 * abstract points (i) and (ii)).  Host only; walks the stream once.
 *   stream      host, table->stream_bytes bytes
 *   gap         host, info->n_tiles * info->tile_windows bytes (output; the
 *               first n_windows are the gaps, the rest zero padding)
 *   out_start   host, info->n_tiles + 1 entries (output)
 *   lut         host, info->lut_words words (output)
 *   info        in: from dfw_plan_query; out: max_tile_symbols filled
 * Errors: DFW_EINVAL, DFW_ECORRUPT (the stream does not hold exactly
 * table->n codewords in table->total_bits bits).
 */
dfw_status dfw_plan(const uint8_t *stream, const dfw_table *table, uint8_t *gap,
                    uint64_t *out_start, uint32_t *lut, dfw_plan_info *info);

/*
 * dfw_decode -- bit-exact bf16 reconstruction on the GPU, asynchronous on
 * `cuda_stream` (a cudaStream_t; NULL = legacy default stream).
 * Source: DFloat11 abstract (two-phase kernel, SRAM LUTs, bit-exact output).
 *   d_stream     device, table->stream_bytes bytes
 *   d_mant       device, dfw_mant_bytes(n) bytes
 *   d_lut        device, info->lut_words words
 *   d_gap        device, info->n_tiles * info->tile_windows bytes
 *   d_out_start  device, info->n_tiles + 1 entries
 *   table, info  host structures from dfw_encode* and dfw_plan
 *   d_out        device, n bf16 patterns (output)
 * Errors: DFW_EINVAL, DFW_EALIGN, DFW_ECUDA; device-detected corruption
 * through dfw_check.
 */
dfw_status dfw_decode(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                      const uint8_t *d_gap, const uint64_t *d_out_start, const dfw_table *table,
                      const dfw_plan_info *info, uint16_t *d_out, void *cuda_stream);

/*
 * dfw_decode_block -- decodes the k tensors of one block (one shared table,
 * encoded by dfw_encode_multi) in one launch into one scratch buffer
 * (DFloat11 abstract point (iii)); tensor i lands at
 * d_scratch + tensor_offsets[i].
 *   tensor_offsets  host, k + 1 entries from dfw_encode_multi
 *   d_scratch       device, scratch_elems >= table->n bf16 slots
 * Other arguments and errors as dfw_decode.
 */
dfw_status dfw_decode_block(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                            const uint8_t *d_gap, const uint64_t *d_out_start,
                            const dfw_table *table, const dfw_plan_info *info,
                            const uint64_t *tensor_offsets, int k, uint16_t *d_scratch,
                            uint64_t scratch_elems, void *cuda_stream);

/*
 * dfw_check -- waits for `cuda_stream`, then reads and clears this device's
 * status word.  Returns DFW_ECORRUPT if any decode since the last check saw
 * corrupt input, DFW_ECUDA if the stream reported a CUDA error, else DFW_OK.
 * The word is shared by all streams of the device.
 */
dfw_status dfw_check(void *cuda_stream);

/* Bits of the device status word (what a kernel saw; sticky until read). */
#define DFW_ST_COUNT 1u   /* codewords ended elsewhere than the plan says */
#define DFW_ST_LUT 2u     /* a table entry or pointer is invalid */
#define DFW_ST_RANGE 4u   /* plan offsets out of order or out of range */
#define DFW_ST_TIMEOUT 8u /* a wait for a bulk copy gave up; the kernel returned early */
#define DFW_ST_CHECK 16u  /* checks build only: an index or copy range left its buffer (the access was skipped) */

/*
 * dfw_status_bits -- dfw_check, and the status bits it read and cleared in
 * *bits (0 when it returns DFW_OK; bits may be NULL).  Tells a timeout
 * (DFW_ST_TIMEOUT) from corrupt input.
 */
dfw_status dfw_status_bits(void *cuda_stream, uint32_t *bits);

/*
 * dfw_selftest_wait_timeout -- failure-path check with no fault: one warp
 * waits, with the bounded wait that every bulk-copy wait here uses, on an
 * mbarrier whose transaction no copy will complete.  The wait gives up at
 * its limit (2 s or 2^24 tries, whichever comes first) and the kernel sets
 * DFW_ST_TIMEOUT and returns, as a decode whose copy never landed would; the
 * context stays usable.  Asynchronous on cuda_stream (up to about 2 s of GPU
 * time); read the result with dfw_status_bits.  The pages describe no failure detection; this is the
 * library's own.  Errors: DFW_ECUDA if the launch fails.
 */
dfw_status dfw_selftest_wait_timeout(void *cuda_stream);

/*
 * dfw_checks_report -- the checks build (libdfw compiled with DFW_CHECKS,
 * the library's stand-in for a memory checker): every copy range, shared-
 * memory extent and output index the kernels compute is checked against its
 * buffer before use; a failing access is skipped and reported through
 * DFW_ST_CHECK and a site number (the first failing site is kept, sticky
 * until read).  *enabled = 1 in the checks build, 0 in the ordinary one
 * (whose kernels carry no checks); *site = the first failing site since the
 * last call, 0 if none, then cleared.  Synchronises the device.  The pages
 * describe no such build; it is the library's own.  Errors: DFW_EINVAL for
 * null pointers, DFW_ECUDA if reading the device word fails.
 */
dfw_status dfw_checks_report(uint32_t *enabled, uint32_t *site);

/*
 * KNOWN-START CHUNKS (a second decode plan over the same stream; the
 * "interleaved lanes" design of the LazyWeights write-up, Verified Facts
 * and body, realised with per-chunk bit offsets instead of separate lane
 * streams).  The codewords are cut into chunks of 64 (the last may be
 * shorter); chunk_bits[c] (u16) is the number of stream bits chunk c uses,
 * and group_start[g] (u64) is the first bit of chunk 32g, with
 * group_start[n_groups] = total_bits.  A warp decodes one group of 32
 * chunks: each lane finds its chunk's first bit by a warp prefix sum over
 * chunk_bits and decodes exactly its 64 codewords, so no count phase, no
 * block scan and no realignment of outputs are needed.
 */
typedef struct dfw_lanes_info {
    uint64_t n_chunks;        /* ceil(n / 64) */
    uint64_t n_groups;        /* ceil(n_chunks / 32); chunk_bits[] holds 32 * n_groups entries */
    uint32_t chunk_symbols;   /* 64 */
    uint32_t group_chunks;    /* 32 */
    uint32_t max_group_bytes; /* largest stream span a group reads, 16-byte aligned with guard (dfw_plan_lanes) */
    uint32_t lut_words;       /* as dfw_plan_info */
    uint32_t lut_tables;      /* as dfw_plan_info */
    uint32_t fast_bits;       /* as dfw_plan_info (dfw_plan_lanes_query sets 12 unless set) */
} dfw_lanes_info;

/* Sizes of the known-start plan arrays.  A nonzero info->fast_bits on entry
 * (8..12) is kept.  Errors: DFW_EINVAL. */
dfw_status dfw_plan_lanes_query(const dfw_table *table, dfw_lanes_info *info);

/*
 * dfw_plan_lanes -- chunk_bits (host, 32 * n_groups u16; padding zero),
 * group_start (host, n_groups + 1 u64) and the LUT image (host, lut_words
 * u32) for one stream; fills info->max_group_bytes.  Host only.
 * Errors: DFW_EINVAL, DFW_ECORRUPT (stream inconsistent with the table).
 */
dfw_status dfw_plan_lanes(const uint8_t *stream, const dfw_table *table, uint16_t *chunk_bits,
                          uint64_t *group_start, uint32_t *lut, dfw_lanes_info *info);

/*
 * dfw_decode_lanes -- bit-exact bf16 reconstruction from the known-start
 * plan, asynchronous on cuda_stream.  Device buffers: d_stream
 * (table->stream_bytes), d_mant (dfw_mant_bytes(n)), d_lut (lut_words),
 * d_chunk_bits (32 * n_groups u16), d_group_start (n_groups + 1 u64), d_out
 * (n bf16; 32-byte alignment lets the kernel store whole 32-byte sectors).
 * n must be below 2^38 (chunk indices are 32-bit; DFW_EINVAL otherwise).
 * Errors as dfw_decode; a group whose chunk bits disagree with
 * group_start, or whose codewords do not end where chunk_bits says, writes
 * nothing / is flagged through dfw_check.  Two closed forms of the code are
 * read in place instead (the plan and LUT are still checked on the host,
 * but not read on the device): two exponents with 1-bit codes (the stream
 * is a bitmap) and all 256 exponents with 8-bit codes (stream byte i is
 * exponent i); every stream is a valid code then, so nothing is flagged.
 */
dfw_status dfw_decode_lanes(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                            const uint16_t *d_chunk_bits, const uint64_t *d_group_start,
                            const dfw_table *table, const dfw_lanes_info *info, uint16_t *d_out,
                            void *cuda_stream);

/*
 * CONTAINER -- the encoded artefact (a tensor, or a block of tensors with
 * one table) as one byte buffer, to store it and decode it later.  The
 * pages ship entropy-coded models (DFloat11 abstract) but give no file
 * format; this one is the library's own.  All integers little-endian; every
 * section starts on a 16-byte boundary (zero padding between sections):
 *   0    8   magic "DFWBF16\0"
 *   8    4   DFW_FORMAT_VERSION
 *   12   4   flags: bit 0 = the known-start plan is present
 *   16   4   cap          20  4  n_symbols     24  4  single_symbol
 *   28   4   k (tensors, >= 1)
 *   32   8   n            40  8  total_bits    48  8  stream_bytes
 *   56   256 code lengths (dfw_table.len)
 *   then     (k + 1) u64 tensor offsets (first 0, last n)
 *   then     the stream (stream_bytes), then the raw bytes (dfw_mant_bytes(n))
 *   then     [plan] 32 * n_groups u16 chunk_bits, n_groups + 1 u64 group_start
 *   last 8   FNV-1a 64-bit hash of every byte before it
 * The LUT is not stored: dfw_lanes_lut rebuilds it from the lengths.
 */

/* Bytes of the container for this table and k tensors, with or without the
 * known-start plan; 0 for a bad argument. */
uint64_t dfw_container_bytes(const dfw_table *table, int k, int with_plan);

/*
 * dfw_container_write -- host: serialises an encoded tensor or block into
 * out (out_bytes >= dfw_container_bytes(...)).  tensor_offsets: k + 1
 * entries (NULL for k = 1); stream and mant as dfw_encode wrote them;
 * chunk_bits and group_start both NULL (no plan) or both as dfw_plan_lanes
 * wrote them.  Errors: DFW_EINVAL (bad table or arguments), DFW_ENOMEM (out
 * too small).
 */
dfw_status dfw_container_write(const dfw_table *table, int k, const uint64_t *tensor_offsets,
                               const uint8_t *stream, const uint8_t *mant, const uint16_t *chunk_bits,
                               const uint64_t *group_start, uint8_t *out, uint64_t out_bytes);

/* Where dfw_container_read found the sections: byte offsets into the buffer
 * (chunk_bits_at and group_start_at are 0 without a plan). */
typedef struct dfw_container_view {
    int32_t k;
    int32_t has_plan;
    uint64_t offsets_at, stream_at, mant_at, chunk_bits_at, group_start_at;
} dfw_container_view;

/*
 * dfw_container_read -- host: checks a container (magic, version, size,
 * hash, table, tensor offsets, and that the plan's chunk bits add up to its
 * group starts) and fills *table and *view; the data stay in buf.  Errors:
 * DFW_EINVAL (NULL arguments or another format version), DFW_ECORRUPT (any
 * check fails).
 */
dfw_status dfw_container_read(const uint8_t *buf, uint64_t bytes, dfw_table *table, dfw_container_view *view);

/*
 * dfw_lanes_scope -- one code-table scope of a sequence: the arguments of a
 * dfw_decode_lanes call other than the output and the stream (device
 * buffers as there; table and info in host memory).
 */
typedef struct dfw_lanes_scope {
    const uint8_t *d_stream;
    const uint8_t *d_mant;
    const uint32_t *d_lut;
    const uint16_t *d_chunk_bits;
    const uint64_t *d_group_start;
    const dfw_table *table;
    const dfw_lanes_info *info;
} dfw_lanes_scope;

/*
 * dfw_decode_lanes_seq -- k scopes decoded one after another into the same
 * output buffer: transformer-block-level decompression of a model, block by
 * block, into one scratch buffer (DFloat11 abstract, point (iii)).  The
 * result is exactly that of k dfw_decode_lanes calls in order on cuda_stream:
 * every byte of d_out ends as the last scope covering it wrote it.  What
 * differs is scheduling: one persistent launch serves up to
 * DFW_SEQ_MAX_SCOPES consecutive scopes (a run of a single scope uses
 * dfw_decode_lanes' kernel, which has no scope bookkeeping).  Its warps keep
 * the same 2048-weight output groups in every scope (group g of any scope is
 * written by the same threads), so a later scope's writes follow an earlier
 * one's in each thread's program order and no grid-wide barrier separates the
 * scopes; each
 * CTA switches fast tables between scopes, while its copies for the next
 * scope's first groups are already in flight.  A new launch starts when the
 * run limit is reached or a scope needs a smaller CTA (long codewords need
 * bigger stream slots); it is a programmatic dependent of the previous one
 * and holds its stores until that launch has completed.  Hence every scope's
 * inputs must be complete when the call is made (all earlier work on
 * cuda_stream counts) and no input may overlap d_out.
 *   scopes   host array of k scopes (k = 0 does nothing)
 *   d_out    max over scopes of n bf16, 16-byte aligned (32-byte alignment
 *            lets the kernel store whole 32-byte sectors)
 * Every scope is checked before the first launch; errors as
 * dfw_decode_lanes (nothing is launched on a host-side error); corrupt
 * streams or plans are flagged through dfw_check.  Asynchronous.
 */
#define DFW_SEQ_MAX_SCOPES 40 /* scopes one launch of dfw_decode_lanes_seq serves */

dfw_status dfw_decode_lanes_seq(int k, const dfw_lanes_scope *scopes, uint16_t *d_out, void *cuda_stream);

/*
 * dfw_decode_lanes_seq_launches -- how many kernel launches
 * dfw_decode_lanes_seq would make for these scopes (one per run of
 * consecutive scopes that share a CTA shape, at most DFW_SEQ_MAX_SCOPES per
 * run; empty scopes take none).  Host only: checks the scopes as the call
 * would and launches nothing.  Errors as dfw_decode_lanes_seq's host-side
 * checks; DFW_EINVAL for a null launches pointer.
 */
dfw_status dfw_decode_lanes_seq_launches(int k, const dfw_lanes_scope *scopes, int *launches);

/*
 * dfw_decode_gemv_lanes -- decode fused with its consumer: y_i = W_i x_i for
 * each of the k tensors of a scope (a transformer block's seven matrices, or
 * one), without writing the decoded weights anywhere.  Source: Huff-LLM
 * abstract (weights stay compressed up to the compute units) and the
 * LazyWeights write-up (decoding on demand, invisible to the consumer);
 * DFloat11 abstract point (iii) (per-block decompression).
 *   d_stream .. info    the scope's known-start plan, as dfw_decode_lanes
 *   k                   1..DFW_GEMV_MAX_TENSORS tensors
 *   tensor_offsets      host, k + 1 entries: tensor i is weights
 *                       [tensor_offsets[i], tensor_offsets[i+1]), first 0,
 *                       last n (as dfw_encode_multi writes them)
 *   cols                host, k entries: tensor i is a row-major matrix of
 *                       (size / cols[i]) rows x cols[i] columns; cols[i] a
 *                       multiple of 64 (so every 64-weight chunk lies in one
 *                       row); each tensor below 2^32 weights
 *   d_x                 host array of k device pointers: bf16 x_i, cols[i]
 *                       entries, 32-byte aligned
 *   d_y                 host array of k device pointers: fp32 y_i, one per row
 *   d_partial           device scratch, partial_elems >= n / 64 fp32 (16-byte
 *                       aligned): one partial dot product per chunk
 * Arithmetic: bf16 x bf16 products are exact; they are summed in fp32 with
 * fused multiply-adds, in an order fixed by the layout, so repeated calls
 * give identical bits; |y - exact| <= gamma(cols) * sum |w x| with
 * gamma(m) = m u / (1 - m u), u = 2^-24.  Asynchronous on cuda_stream (two
 * launches).  Errors: DFW_EINVAL, DFW_EALIGN, DFW_ENOMEM (partial too
 * small), DFW_ECUDA; corrupt plans through dfw_check (y then undefined).
 */
#define DFW_GEMV_MAX_TENSORS 8

dfw_status dfw_decode_gemv_lanes(const uint8_t *d_stream, const uint8_t *d_mant, const uint32_t *d_lut,
                                 const uint16_t *d_chunk_bits, const uint64_t *d_group_start,
                                 const dfw_table *table, const dfw_lanes_info *info, int k,
                                 const uint64_t *tensor_offsets, const uint32_t *cols,
                                 const uint16_t *const *d_x, float *const *d_y, float *d_partial,
                                 uint64_t partial_elems, void *cuda_stream);

/*
 * ENCODING ON THE GPU (two calls; same stream bytes as dfw_encode, and the
 * known-start plan's chunk_bits and group_start made on the way).  Source:
 * DFloat11 abstract (frequency-based codes for the bf16 exponents); the
 * LazyWeights write-up (Huffman; lanes with known starts).
 *
 * dfw_encode_device_scratch_bytes -- device scratch bytes the first call
 * needs (a few KB, whatever n).
 *
 * dfw_encode_device -- first call: splits the n bf16 patterns into raw bytes
 * and an exponent histogram on the GPU, builds the code on the host
 * (package-merge, canonical; exactly as dfw_encode), then counts each
 * chunk's bits and each group's start on the GPU.  Synchronises cuda_stream
 * twice (to read the histogram and the totals).
 *   d_bf16         device, n bf16 patterns (16-byte aligned)
 *   cap            length cap, 1..32
 *   d_mant         device, dfw_mant_bytes(n) bytes (output)
 *   d_chunk_bits   device, 32 * n_groups u16 (output)
 *   d_group_start  device, n_groups + 1 u64 (output)
 *   d_scratch      device, scratch_bytes >= dfw_encode_device_scratch_bytes(n)
 *   table          host, output: as dfw_encode (stream_bytes tells the caller
 *                  how large a stream to allocate for dfw_pack_device)
 *   info           host; in: fast_bits (0 = 12); out: as dfw_plan_lanes
 * n_groups = ceil(ceil(n / 64) / 32).  Errors: DFW_EINVAL, DFW_EALIGN,
 * DFW_ENOMEM (scratch too small), DFW_ECAP, DFW_ECUDA.
 *
 * dfw_pack_device -- second call: packs the codewords at the positions the
 * first call counted and writes the zero padding, so every one of the
 * stream's table->stream_bytes bytes is written (two launches: the words
 * neighbouring groups share are cleared first).  Asynchronous on cuda_stream.
 *   d_bf16, table, info, d_group_start   as returned by the first call
 *   d_stream   device, stream_capacity >= table->stream_bytes (output)
 * Errors: DFW_EINVAL, DFW_EALIGN, DFW_ENOMEM, DFW_ECUDA.
 *
 * dfw_lanes_lut -- the LUT image (host, info->lut_words u32) for a table and
 * info->fast_bits, without walking a stream.  Errors: DFW_EINVAL.
 */
uint64_t dfw_encode_device_scratch_bytes(uint64_t n);

dfw_status dfw_encode_device(const uint16_t *d_bf16, uint64_t n, int cap, uint8_t *d_mant,
                             uint16_t *d_chunk_bits, uint64_t *d_group_start, void *d_scratch,
                             uint64_t scratch_bytes, dfw_table *table, dfw_lanes_info *info,
                             void *cuda_stream);

dfw_status dfw_pack_device(const uint16_t *d_bf16, const dfw_table *table, const dfw_lanes_info *info,
                           const uint64_t *d_group_start, uint8_t *d_stream, uint64_t stream_capacity,
                           void *cuda_stream);

dfw_status dfw_lanes_lut(const dfw_table *table, const dfw_lanes_info *info, uint32_t *lut);

/*
 * dfw_encode_device_multi -- the first call for k scopes (the blocks of a
 * model, each with its own code), with the host's share of each scope
 * overlapped with the GPU's work on the next: pass 1 of scope i + 1 is
 * queued before the host waits for scope i's histogram, builds its code and
 * queues its counting passes.  The pages describe the encoder only as an
 * offline step; this call only schedules that step better.
 *   scopes         host array of k dfw_encode_scope: per scope the d_bf16, n,
 *                  d_mant, d_chunk_bits, d_group_start of dfw_encode_device
 *   cap            length cap, 1..32, for every scope
 *   d_scratch      device, scratch_bytes >= k * dfw_encode_device_scratch_bytes(0);
 *                  scope i uses the i-th such slice
 *   h_staging      host, staging_bytes >= dfw_encode_device_multi_staging_bytes(k),
 *                  8-byte aligned: where each scope's histogram and totals are
 *                  read back.  Page-locked memory (cudaHostAlloc) lets the copies
 *                  run ahead of the host; pageable memory gives the same results,
 *                  but each copy then waits for all earlier work
 *   tables, infos  host arrays of k: outputs (infos[i].fast_bits is read first),
 *                  each exactly what dfw_encode_device gives for scope i alone
 * Every scope is checked before anything is launched (an error then leaves
 * the device outputs untouched; tables and infos are unspecified).  An error
 * found later (DFW_ECAP: 2^cap is smaller
 * than a scope's number of exponents; DFW_ECUDA) stops the queueing; the
 * call still waits for the work already queued, and the outputs are then
 * unspecified.  In all cases cuda_stream is idle when the call returns (it
 * synchronises once per non-empty scope and once at the end).  Then
 * dfw_pack_device per scope, as after dfw_encode_device.  Errors: DFW_EINVAL,
 * DFW_EALIGN, DFW_ENOMEM (scratch or staging too small), DFW_ECAP, DFW_ECUDA.
 */
typedef struct dfw_encode_scope {
    const uint16_t *d_bf16;
    uint64_t n;
    uint8_t *d_mant;
    uint16_t *d_chunk_bits;
    uint64_t *d_group_start;
} dfw_encode_scope;

uint64_t dfw_encode_device_multi_staging_bytes(uint32_t k);

dfw_status dfw_encode_device_multi(uint32_t k, const dfw_encode_scope *scopes, int cap, void *d_scratch,
                                   uint64_t scratch_bytes, void *h_staging, uint64_t staging_bytes,
                                   dfw_table *tables, dfw_lanes_info *infos, void *cuda_stream);

/*
 * dfw_encode_device_noalloc -- dfw_encode_device without a scratch argument,
 * for callers that cannot allocate device memory when they encode: a serving
 * runtime that reserves all of the GPU's memory at start-up and allows no
 * allocation afterwards, or code that must not call cudaMalloc because the
 * call would synchronise the device or re-enter the caller's own allocator.
 * The pages describe no such call; it exists for those callers only.
 *
 * The scratch is an array of DFW_NOALLOC_SCRATCH_BYTES compiled into the
 * library: every GPU that uses the library holds one until the process
 * exits.  With lazy module loading (the CUDA runtime's default) the array
 * and the encoder's kernels are placed on a device when the library first
 * uses that device, not when the library is loaded, so a runtime that
 * reserves the GPU's memory up front should make one call (a warm-up) on
 * each device before it reserves.  The first call on a device also looks
 * up the array's device address (cudaGetSymbolAddress) and caches it; make
 * that first call before any stream capture begins.  The cached address
 * belongs to the device's context at that time: after cudaDeviceReset (or
 * anything else that destroys and re-creates the context) in the same
 * process the call is not supported.  All calls share the array and clear it before use,
 * so calls whose GPU work overlaps (two streams, two host threads) race on it:
 * the caller must not overlap them.  Arguments, outputs, synchronisation and
 * errors as dfw_encode_device; DFW_ENOMEM if the scratch that n needs
 * exceeded DFW_NOALLOC_SCRATCH_BYTES (the need is a fixed 10,496 bytes, so no
 * n reaches it today).  The call makes no cudaMalloc, cudaFree or other
 * device allocation; the inputs and outputs are the caller's.
 */
#define DFW_NOALLOC_SCRATCH_BYTES 16384

dfw_status dfw_encode_device_noalloc(const uint16_t *d_bf16, uint64_t n, int cap, uint8_t *d_mant,
                                     uint16_t *d_chunk_bits, uint64_t *d_group_start, dfw_table *table,
                                     dfw_lanes_info *info, void *cuda_stream);

/*
 * rANS VARIANT (the ANS coder of the ~1.5:1 page's abstract; the LazyWeights
 * write-up compares Huffman with rANS).  The pages fix no format; this one:
 *   - the same split: exponent symbols coded, raw bytes stored as they are;
 *   - frequencies quantised to M = 2^DFW_RANS_SCALE_BITS: floor(count M / n),
 *     at least 1 for a present exponent; a positive remainder goes to the
 *     most frequent exponent, a negative one is taken one unit at a time from
 *     the exponent with the largest frequency above 1 (smallest exponent on
 *     ties, both ways);
 *   - states x in [2^16, 2^32); exponent s (frequency f, cumulative start c)
 *     encodes as x' = floor(x / f) M + (x mod f) + c after emitting the low
 *     16 bits of x while x >= f (2^16 / M) 2^16; decoding inverts it and
 *     reloads 16 bits while x < 2^16;
 *   - blocks of DFW_RANS_BLOCK exponents, coded independently; in a block,
 *     exponent i belongs to state i mod DFW_RANS_LANES; the encoder runs
 *     backwards so a decoder takes steps k = 0, 1, ... (exponents 32k ..
 *     32k + 31, one per state) and then reloads the states that need it in
 *     increasing state order, each taking the next word;
 *   - a block is its 32 final encoder states (u32), its words in decoding
 *     order (u16), zero padding to 16 bytes; block_start[b] is its byte
 *     offset, block_start[n_blocks] the stream length.  Every state starts
 *     at 2^16, so a correct decode ends with every state at 2^16.
 */
#define DFW_RANS_SCALE_BITS 12
#define DFW_RANS_LANES 32
#define DFW_RANS_BLOCK 16384

typedef struct dfw_rans_table {
    uint32_t version;          /* DFW_FORMAT_VERSION */
    uint32_t scale_bits;       /* DFW_RANS_SCALE_BITS */
    uint32_t lanes;            /* DFW_RANS_LANES */
    uint32_t block_syms;       /* DFW_RANS_BLOCK */
    uint64_t n;                /* weights */
    uint64_t n_blocks;         /* ceil(n / block_syms) */
    uint64_t stream_bytes;     /* block_start[n_blocks] */
    uint32_t max_block_bytes;  /* largest block */
    uint32_t reserved;         /* zero */
    uint16_t freq[256];        /* quantised frequency per exponent (sum 2^scale_bits) */
} dfw_rans_table;

/* Worst-case rANS stream bytes for n weights. */
uint64_t dfw_rans_stream_bound(uint64_t n);

/*
 * dfw_rans_encode -- host: the k tensors' concatenation (one table), coded
 * as above; blocks are coded by n_threads threads (0 = all), the bytes are
 * the same for any thread count.
 *   stream       host, stream_capacity bytes (dfw_rans_stream_bound(n) suffices)
 *   mant         host, dfw_mant_bytes(n) raw bytes (output)
 *   block_start  host, n_blocks + 1 u64 (output)
 * Errors: DFW_EINVAL, DFW_ENOMEM (table->stream_bytes then holds the need).
 */
dfw_status dfw_rans_encode(const uint16_t *const *tensors, const uint64_t *sizes, int k,
                           uint8_t *stream, uint64_t stream_capacity, uint8_t *mant,
                           uint64_t mant_capacity, uint64_t *block_start, dfw_rans_table *table,
                           int n_threads);

/*
 * dfw_rans_decode -- GPU: one warp per block, 32 states decoded per step,
 * reloads ranked by warp ballot.  Device buffers d_stream (stream_bytes,
 * 16-byte aligned), d_mant (dfw_mant_bytes(n)), d_block_start (n_blocks + 1),
 * d_out (n bf16).  A block that does not end with every state at 2^16 and
 * every word used is flagged through dfw_check.  Errors as dfw_decode.
 */
dfw_status dfw_rans_decode(const uint8_t *d_stream, const uint8_t *d_mant, const uint64_t *d_block_start,
                           const dfw_rans_table *table, uint16_t *d_out, void *cuda_stream);

/* Static English text for a status code. */
const char *dfw_strerror(dfw_status status);

#ifdef __cplusplus
}
#endif

#endif /* DFW_H */
