/*
 * rans_b200.h -- C ABI of librans_b200: indexed 64-bit rANS entropy coding on
 * one NVIDIA B200 (sm_100a).
 *
 * What is coded (sources are page title + section):
 *   - rANS with a 64-bit state, 32-bit renormalisation words and 16-bit CDF
 *     precision ("torch_ans 0.3.0", Usage, variants table, rans64 row;
 *     "kompressor" README, Credits: CompressAI's ryg_rans-style coder).
 *   - One CDF row per symbol, chosen through an index array; rows given as
 *     cdfs / cdf_lengths / offsets ("torch_ans 0.3.0", Low-level API,
 *     rans_push and rans_pop).
 *   - Symbols outside a row's coded range [offset, offset + cdf_length - 2)
 *     take the row's escape bucket and are then sent as a zig-zag raw value
 *     in 4-bit bypass pieces (same section, "Range limit"; "kompressor"
 *     README, Correctness: the bypass path).
 *   - Many independent streams: contiguous chunks or spatial tiles ("kompressor"
 *     README, Why: zero cross-chunk dependency), each coded with W = 1, 2, 4,
 *     8 or 32 interleaved states sharing one word stream, symbol i on state
 *     i mod W ("torch_ans 0.3.0", Usage legend and FAQ: interleaved states
 *     share one bitstream; the 32-way form maps the states onto the lanes of
 *     a warp, the 2/4/8-way forms onto sub-warp lane groups).
 *   - Two coder formats: the 64/32/16 one described below (RANS_FMT_RANS64)
 *     and torch_ans's rans32_16 (RANS_FMT_RANS32_16: 32-bit state, 16-bit
 *     words, precision <= 15), each also alias-coded (RANS_FMT_ALIAS).
 *   - pmf -> quantised CDF rows ("torch_ans 0.3.0", High-level API,
 *     init_params) and Gaussian rows from a scale table ("kompressor" README,
 *     Getting Started: 64 CDF rows for the y latent).
 *
 * The RANS64 format: state bound L = 2^31 (initial encoder state, final decoder
 * state), symbol op renormalises when x >= 2^47 * freq, bypass op when
 * x >= 2^59; the stream of one chunk is its W lane states (low word, high
 * word; lane 0 first) followed by the renormalisation words in the order the
 * decoder consumes them, all little-endian 32-bit words.  The escape raw value
 * is 2(v - maxv) above the range and -2v - 1 below it; it is sent as a count
 * of 4-bit pieces (in pieces of at most 15, where 15 means "more follows"),
 * then the pieces, least significant first.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers unless a name says host_.
 *   - The caller allocates every buffer; the library never allocates device
 *     memory (sizes come from the *_bytes queries).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); all work
 *     is enqueued on it.  Only rans_tables_prepare, rans_alias_prepare and
 *     rans_get_status synchronise.
 *   - Argument errors detectable on the host return immediately with a
 *     negative status.  Errors found on the device (bad index, zero-width
 *     bucket, raw value beyond 60 bits, a malformed or truncated stream, output
 *     capacity) are recorded in the workspace's status word, first error wins,
 *     and are returned by rans_get_status; the outputs are then undefined.
 *     No kernel traps or asserts.
 */
#ifndef RANS_B200_H
#define RANS_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RANS_PRECISION 16
#define RANS_BYPASS_BITS 4

typedef enum rans_status {
    RANS_OK = 0,
    RANS_ERR_ARG = -1,        /* invalid argument (host-side or a bad chunking) */
    RANS_ERR_INDEX = -2,      /* an index outside [0, K) */
    RANS_ERR_ZERO_FREQ = -3,  /* a symbol maps to a bucket of width 0 */
    RANS_ERR_RANGE = -4,      /* an escape raw value of 2^60 or more */
    RANS_ERR_CAPACITY = -5,   /* an output or table buffer is too small */
    RANS_ERR_CORRUPT = -6,    /* a stream is truncated, too long or inconsistent */
    RANS_ERR_CUDA = -7,       /* a CUDA runtime call failed */
    RANS_ERR_TABLE = -8,      /* a malformed CDF row or pmf */
    RANS_ERR_TIMEOUT = -9     /* a bounded device wait gave up */
} rans_status;

/* Symbol element types. */
enum { RANS_SYM_INT32 = 0, RANS_SYM_UINT8 = 1, RANS_SYM_INT16 = 2 };

/* Chunking kinds. */
enum { RANS_CHUNK_CONTIG = 0, RANS_CHUNK_EXPLICIT = 1, RANS_CHUNK_TILED = 2 };

/*
 * Coder formats ("torch_ans 0.3.0", Usage, variants table):
 *   RANS_FMT_RANS64:    64-bit state, 32-bit little-endian stream words, CDF
 *                       rows summing to 2^16 (precision 16); lower state
 *                       bound 2^31; each state flushed as 2 words.
 *   RANS_FMT_RANS32_16: 32-bit state, 16-bit little-endian stream words, CDF
 *                       rows summing to 2^p with 1 <= p <= 15; lower state
 *                       bound 2^16 (the value for which one 16-bit word
 *                       restores a state below it); each state flushed as 2
 *                       words, so stream lengths are even.
 * Both code the same symbol -> op mapping (escape bucket, zig-zag raw value,
 * 4-bit bypass pieces); a bypass op renormalises at 2^59 / 2^28.  A table
 * set's precision picks the formats it serves: 16 -> RANS64, <= 15 ->
 * RANS32_16.
 */
enum { RANS_FMT_RANS64 = 0, RANS_FMT_RANS32_16 = 1 };

/*
 * RANS_FMT_ALIAS, or'ed into the format: alias-coded streams ("torch_ans
 * 0.3.0", Usage, Alias Coding: push and pop both change, pop finds the symbol
 * in constant time; Performance Tuning: a row's bucket count, cdf_length - 1,
 * must be a power of two; 1, 2, 4 or 8 interleaved states, no 32-way form).
 * The library's reading of the method (the pages give no construction):
 * the 2^p positions are cut into n = cdf_length - 1 slots of 2^p / n; Vose's
 * alias method (first-in first-out worklists of the symbols below and above
 * the slot width, each in ascending order) leaves slot j with d_j positions
 * of symbol j and the rest for an alias symbol; a symbol ranks its own slot's
 * positions first, then its alias parts in slot order.  The encoder codes
 * symbol s on the position of rank x mod f_s (x -> (x / f) 2^p + position),
 * the decoder reads symbol and rank from the slot of x mod 2^p
 * (x -> f (x >> p) + rank).  Needs alias tables (rans_alias_prepare).
 */
enum { RANS_FMT_ALIAS = 0x100 };

/*
 * How the n symbols are cut into streams, and how indexes map to symbols.
 *   CONTIG:   n_streams streams; stream k covers elements
 *             [k*ceil(n/S), min((k+1)*ceil(n/S), n)) (trailing streams may be
 *             empty).
 *   EXPLICIT: n_streams streams; stream k covers [stream_starts[k],
 *             stream_starts[k+1]) -- stream_starts is a device array of
 *             n_streams + 1 non-decreasing element offsets within [0, n].
 *   TILED:    the symbols are an NCHW tensor shape[0..3] = (B, C, H, W);
 *             one stream per (image, group of `group` channels, tile of
 *             tile_h x tile_w), ordered (b, g, tile row, tile column); inside a
 *             stream the elements go (channel, row, column); edge tiles are
 *             partial.  n must equal B*C*H*W.
 *   interleave: 1, 2, 4, 8 or 32 states per stream ("torch_ans 0.3.0",
 *             Usage, variants table: 1/2/4/8 for rans64, also 32 for
 *             rans32_16); symbol i of a stream codes on state i mod W.  32
 *             maps a stream onto a warp, the others onto one thread.  The
 *             float-latent entry points take 1 or 32.
 *   index_block: element p (flat position in the symbol array) uses row
 *             indexes[p / index_block]; 1 = one index per symbol; must be a
 *             power of two.
 *   format:   RANS_FMT_* (0, the zero-initialised default, is RANS64).
 */
typedef struct rans_chunking {
    int32_t kind;
    int32_t interleave;
    int64_t n_streams;
    const int64_t *stream_starts;
    int64_t shape[4];
    int64_t group, tile_h, tile_w;
    int64_t index_block;
    int32_t format;
    int32_t reserved;
} rans_chunking;

/*
 * A prepared table set, filled by rans_tables_prepare.  `blob` is the
 * caller's device buffer; the other fields describe its layout and are read
 * by the encoder and decoder.  The blob holds per-row metadata, every
 * bucket's (start, width) in 32 bits for the encoder, the CDF entries as
 * 16-bit starts for the decoder, and the decoder's lookup slots.  One table set serves both directions and every
 * chunking.  Treat the fields as opaque.
 */
typedef struct rans_tables {
    void *blob;
    uint64_t blob_bytes;
    int32_t K;              /* rows */
    int32_t max_buckets;    /* longest row's bucket count (cdf_length - 1) */
    int64_t n_buckets;      /* all rows' buckets */
    int64_t n_slots;        /* decode lookup slots */
    uint32_t meta_bytes, bucket_bytes, start_bytes, slot_bytes;  /* sections (16-B padded) */
    int32_t enc_in_smem;    /* encode table mode: 1 stages meta + buckets in shared
                               memory, 2 meta + 16-bit starts, 0 reads global */
    int32_t dec_in_smem;    /* decode table mode: 1 stages meta + starts + slots,
                               2 meta + starts (a binary search per lookup), 0 reads
                               global */
    int32_t device;         /* CUDA device the blob lives on */
    int32_t precision;      /* the rows sum to 2^precision */
    int32_t max_slot_log2;  /* log2 of the largest row's decode lookup slot count */
    void *alias;            /* alias tables (rans_alias_prepare), or NULL */
    uint64_t alias_bytes;
    uint64_t alias_remap_offset;  /* byte offset of the remap entries in `alias` */
} rans_tables;

/* ------------------------------------------------------------ status ---- */

/* A short English description of a status code (static storage). */
const char *rans_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
int rans_version(void);

/* ------------------------------------------------------- CDF tables ---- */

/*
 * Lengths and offsets of K Gaussian rows ("kompressor" README, Getting
 * Started: the y latent's 64 rows; "Benchmark notes", section 4: 200512 table
 * entries).  For tail mass t, m = -Phi^-1(t/2); row r has centre
 * c = ceil(scales[r] * m), cdf_length 2c + 3 and offset -c.
 *   scales:      device float[K], each > 0 and finite.
 *   cdf_lengths: device int32[K] out; a row that cannot be built gets a
 *                negative status instead of its length.
 *   offsets:     device int32[K] out.
 * Use it to size Lmax before rans_build_cdfs_from_scales.  Asynchronous.
 */
int rans_gaussian_lengths(const float *scales, int32_t K, double tail_mass,
                          int32_t *cdf_lengths, int32_t *offsets, void *stream);

/*
 * K Gaussian CDF rows.  Row r's pmf is Phi((0.5-|k|)/s) - Phi((-0.5-|k|)/s)
 * for k = -c..c (Phi in double, cast to float), followed by the tail mass
 * 2 Phi((-0.5-c)/s); the pmf is quantised as in rans_build_cdfs_from_pmfs,
 * to rows summing to 2^precision (1 <= precision <= 16).
 *   cdfs: device int32[K][Lmax] out; entries past a row's length are 0.
 *   cdf_lengths, offsets: device int32[K] out (as rans_gaussian_lengths);
 *   a row longer than Lmax, or one that cannot be quantised, gets a negative
 *   status as its length.  Asynchronous.
 */
int rans_build_cdfs_from_scales(const float *scales, int32_t K, double tail_mass,
                                int32_t precision, int32_t *cdfs, int32_t Lmax,
                                int32_t *cdf_lengths, int32_t *offsets, void *stream);

/*
 * K CDF rows from pmfs ("torch_ans 0.3.0", High-level API, init_params; FAQ:
 * rows are increasing positive integers up to 2^precision).  Row r takes
 * pmf_lengths[r] probabilities pmfs[r*pmf_stride ...] and then tail_mass[r];
 * with M = 2^precision (1 <= precision <= 16) each is scaled by M and
 * rounded half away from zero, the running sum is rescaled to
 * floor(M c / total), and every empty bucket then takes one unit from the
 * narrowest bucket wider than 1 (the first such on ties) -- scanning empty
 * buckets in ascending order.
 *   pmfs:        device float[K][pmf_stride].
 *   pmf_lengths: device int32[K], each in [0, pmf_stride].
 *   tail_mass:   device float[K].
 *   cdfs:        device int32[K][Lmax] out (Lmax >= max pmf_length + 2).
 *   cdf_lengths: device int32[K] out: pmf_length + 2, or a negative status for
 *                a row that cannot be built (negative or non-finite
 *                probability, total 0, nothing to steal from, too long).
 * Offsets are the caller's (they come with the pmfs).  Asynchronous.
 */
int rans_build_cdfs_from_pmfs(const float *pmfs, int32_t K, int32_t pmf_stride,
                              const int32_t *pmf_lengths, const float *tail_mass,
                              int32_t precision, int32_t *cdfs, int32_t Lmax,
                              int32_t *cdf_lengths, void *stream);

/* Upper bound on the blob size rans_tables_prepare needs for K rows of at
 * most Lmax entries. */
uint64_t rans_tables_bytes(int32_t K, int32_t Lmax);

/*
 * Validates CDF rows and lays out the coder's tables in `blob` (device,
 * blob_bytes >= rans_tables_bytes(K, Lmax)): per-row metadata, every bucket's
 * (start, width) packed in 32 bits, and a per-row lookup table mapping the
 * top bits of a decoder state's low 16 bits to its bucket.  Each row must
 * have 2 <= cdf_lengths[r] <= Lmax, cdf[0] = 0, cdf[len-1] = 2^precision
 * and strictly increasing entries; otherwise RANS_ERR_TABLE (or the negative
 * length left by a builder).  Rows of precision p < 16 are stored scaled to
 * 16 bits (entries times 2^(16-p)).  Synchronous (reads back the K lengths
 * and the validation status); fills *out.
 *   cdfs: device int32[K][Lmax]; cdf_lengths, offsets: device int32[K];
 *   precision: 16 (RANS64) or 1..15 (RANS32_16).
 */
int rans_tables_prepare(const int32_t *cdfs, int32_t K, int32_t Lmax,
                        const int32_t *cdf_lengths, const int32_t *offsets, int32_t precision,
                        void *blob, uint64_t blob_bytes, rans_tables *out, void *stream);

/*
 * Rebuilds a prepared table set in place from new CDF rows whose lengths (and
 * precision) equal the rows it was prepared from (for example a scale table rebuilt every
 * call): offsets, packed buckets and lookup slots are rewritten on the device
 * with the layout kept, with no host synchronisation.  A row whose length
 * differs, or a malformed row, records RANS_ERR_TABLE in the blob's status
 * word (read it with rans_get_status(tables->blob, stream)); the table set is
 * then unusable until prepared again.  Asynchronous.
 *   cdfs: device int32[K][Lmax]; cdf_lengths, offsets: device int32[K];
 *   tables: filled by rans_tables_prepare for the same K.
 */
int rans_tables_refresh(const int32_t *cdfs, int32_t K, int32_t Lmax,
                        const int32_t *cdf_lengths, const int32_t *offsets,
                        const rans_tables *tables, void *stream);

/*
 * rans_build_cdfs_from_scales (at the table set's precision) and
 * rans_tables_refresh from those rows, in one kernel launch: one CTA per row
 * quantises the row and rewrites its offset, packed buckets and lookup slots
 * from it.  Same outputs as the two calls: cdfs, cdf_lengths and offsets as
 * rans_build_cdfs_from_scales writes them, the table set as
 * rans_tables_refresh leaves it.  A row that cannot be built, or whose
 * length differs from the prepared layout, records RANS_ERR_TABLE in the
 * blob's status word (and its negative status as its length).  Asynchronous.
 *   scales: device float[K]; cdfs: device int32[K][Lmax] out;
 *   cdf_lengths, offsets: device int32[K] out;
 *   tables: prepared for the same K from Gaussian rows of the same lengths.
 */
int rans_tables_refresh_from_scales(const float *scales, int32_t K, double tail_mass,
                                    int32_t *cdfs, int32_t Lmax, int32_t *cdf_lengths,
                                    int32_t *offsets, const rans_tables *tables, void *stream);

/* Bytes of the alias tables of a prepared table set: 8 bytes per bucket
 * (slot words) and 2^precision 16-bit remap entries per row. */
uint64_t rans_alias_bytes(const rans_tables *tables);

/*
 * Builds the alias tables (see RANS_FMT_ALIAS) of a prepared table set from
 * the rows it was prepared from, into the caller's device buffer `alias`
 * (256-byte aligned, >= rans_alias_bytes), and records it in *tables.  Every
 * row's bucket count (cdf_length - 1) must be a power of two of at most 8192
 * (else RANS_ERR_ARG).  Synchronous: reads back the lengths and the status.
 *   cdfs, cdf_lengths: as for rans_tables_prepare (same rows).
 */
int rans_alias_prepare(const int32_t *cdfs, int32_t K, int32_t Lmax,
                       const int32_t *cdf_lengths, rans_tables *tables, void *alias,
                       uint64_t alias_bytes, void *stream);

/* ------------------------------------------------- sizes and queries ---- */

/* Number of streams the chunking makes of n symbols (< 0: invalid chunking). */
int64_t rans_num_streams(const rans_chunking *chunking, int64_t n);

/* Bytes of workspace rans_encode_with_indexes needs (status word, per-stream
 * lengths and a worst-case scratch slot per stream: 8 bytes per symbol plus
 * 16 * interleave + 16 per stream). */
uint64_t rans_encode_workspace_bytes(const rans_chunking *chunking, int64_t n);

/* Bytes of workspace rans_decode_with_indexes needs. */
uint64_t rans_decode_workspace_bytes(const rans_chunking *chunking, int64_t n);

/* An output capacity that can never be too small for n symbols. */
uint64_t rans_max_compressed_bytes(const rans_chunking *chunking, int64_t n);

/* ---------------------------------------------------- encode / decode ---- */

/*
 * encode_with_indexes ("torch_ans 0.3.0", Low-level API rans_push and
 * High-level API encode_with_indexes).  Codes the n symbols into one
 * byte string per stream, packed back to back in `out`; stream_offsets
 * receives S + 1 uint64 byte offsets (offsets[0] = 0, offsets[S] = total).
 * Each stream is coded symbol by symbol in reverse order into a worst-case
 * scratch slot of the workspace, then all streams are compacted into `out`
 * with a device prefix scan.
 *   symbols:   device array of n elements of sym_dtype (RANS_SYM_*).
 *   indexes:   device int32[ceil(n / index_block)], each in [0, tables->K).
 *   out:       device uint8[out_capacity].
 *   stream_offsets: device uint64[S + 1].
 *   workspace: device, >= rans_encode_workspace_bytes; 256-byte aligned.
 *   chunking->format picks the coder (RANS_FMT_*); the tables' precision
 *   must be 16 for RANS64 and at most 15 for RANS32_16 (else RANS_ERR_ARG).
 * Asynchronous; device errors via rans_get_status(workspace).
 */
int rans_encode_with_indexes(const void *symbols, int32_t sym_dtype, const int32_t *indexes,
                             int64_t n, const rans_tables *tables,
                             const rans_chunking *chunking, uint8_t *out,
                             uint64_t out_capacity, uint64_t *stream_offsets,
                             void *workspace, uint64_t workspace_bytes, void *stream);

/*
 * decode_with_indexes ("torch_ans 0.3.0", Low-level API rans_pop; the decoded
 * symbol is the row's last bucket whose CDF entry is <= the state's low
 * `precision` bits, the rule of the linear scan in "Benchmark notes" section
 * 4).
 *   in:             device uint8[in_bytes]: the packed streams, aligned to
 *                   the format's word (4 bytes, or 2 for RANS32_16).
 *   stream_offsets: device uint64[S + 1] from the encoder.
 *   indexes:        as for encode; must equal the encoder's.
 *   symbols_out:    device array of n elements of sym_dtype.
 *   workspace:      device, >= rans_decode_workspace_bytes; 256-byte aligned.
 * Every read is bounded by its stream's [offsets[k], offsets[k+1]); a stream
 * that does not end exactly where its words end with every lane back at the
 * initial state (2^31, or 2^16 for RANS32_16) is reported as
 * RANS_ERR_CORRUPT.  chunking->format and the tables' precision as for
 * encode.  Asynchronous.
 */
int rans_decode_with_indexes(const uint8_t *in, uint64_t in_bytes,
                             const uint64_t *stream_offsets, const int32_t *indexes,
                             int64_t n, const rans_tables *tables,
                             const rans_chunking *chunking, void *symbols_out,
                             int32_t sym_dtype, void *workspace, uint64_t workspace_bytes,
                             void *stream);

/*
 * rans_encode_with_indexes without a workspace argument, for callers that
 * cannot allocate device memory themselves (for example code inside a host
 * framework whose allocator owns all device memory, or a latency-critical path
 * on which a cudaMalloc, which may synchronise the device, is not allowed).
 * The pages have no counterpart: this is a packaging convenience of the
 * library.
 *   The workspace is a 32 MiB array inside the library that every GPU loading
 *   it keeps until exit; inputs needing more (rans_encode_workspace_bytes)
 *   return RANS_ERR_CAPACITY.  The first call in a device's CUDA context
 *   looks the array's device address up (call it once before any stream
 *   capture); after a device reset the new context's first call looks it up
 *   again.  All calls
 *   share the array: calls that overlap on the GPU race, so serialise them.
 *   Device errors cannot be read with rans_get_status here; instead
 *   stream_offsets[S] is set to UINT64_MAX.  Other arguments, outputs and
 *   results are those of rans_encode_with_indexes.  Allocates nothing.
 */
int rans_encode_with_indexes_noalloc(const void *symbols, int32_t sym_dtype,
                                     const int32_t *indexes, int64_t n,
                                     const rans_tables *tables,
                                     const rans_chunking *chunking, uint8_t *out,
                                     uint64_t out_capacity, uint64_t *stream_offsets,
                                     void *stream);

/* --------------------------------------------------- float latents ---- */

/*
 * The coder fed straight from a mean-scale model's float tensors (the y latent
 * of "Benchmark notes" section 3, whose per-stage breakdown shows the scales
 * mapped to table rows by CompressAI's build_indexes before the coder runs).
 * The pages name these steps without spelling them out; the library's reading:
 *   row:    for a scale s, the first of the K scale-table entries (increasing)
 *           that is >= max(s, scale_bound), a NaN scale counting as the bound;
 *           the last row when none of the first K - 1 entries is;
 *   symbol: y - mean in float32, rounded to the nearest integer, ties to even
 *           (mean 0 when `means` is NULL); a value that is not finite or not
 *           an int32 is RANS_ERR_RANGE;
 *   value:  the decoder returns float32(symbol) + mean, in float32.
 * The row of element i is what rans_encode_with_indexes takes as indexes[i]
 * and the symbol its symbols[i], so the streams are byte-identical to
 * encoding those.
 */

/* Rows of n scales (device float[n] in, device int32[n] out) for a K-entry
 * device scale table.  Asynchronous. */
int rans_build_indexes(const float *scales, int64_t n, const float *scale_table, int32_t K,
                       float scale_bound, int32_t *indexes, void *stream);

/*
 * encode_with_indexes from float latents, rows and symbols computed inside the
 * coder (no index or symbol array is written).
 *   y, scales:   device float[n]; means: device float[n] or NULL.
 *   scale_table: device float[table_len], table_len == tables->K: the scales
 *                the table rows were built from.
 *   chunking:    index_block must be 1 (one scale per element); format
 *                RANS64 (the float path codes the 64-bit format only).
 * Other arguments, outputs and errors as rans_encode_with_indexes.
 */
int rans_encode_from_scales(const float *y, const float *means, const float *scales,
                            int64_t n, const float *scale_table, int32_t table_len,
                            float scale_bound, const rans_tables *tables,
                            const rans_chunking *chunking, uint8_t *out,
                            uint64_t out_capacity, uint64_t *stream_offsets, void *workspace,
                            uint64_t workspace_bytes, void *stream);

/*
 * decode_with_indexes back to float values: values[i] = float32(symbol) +
 * means[i] (or the symbol alone when means is NULL), rows from the scales as
 * above.  values: device float[n].  Other arguments and errors as
 * rans_decode_with_indexes.
 */
int rans_decode_to_values(const uint8_t *in, uint64_t in_bytes, const uint64_t *stream_offsets,
                          const float *scales, const float *means, int64_t n,
                          const float *scale_table, int32_t table_len, float scale_bound,
                          const rans_tables *tables, const rans_chunking *chunking,
                          float *values, void *workspace, uint64_t workspace_bytes,
                          void *stream);

/* Synchronises `stream` and returns the first error recorded in `workspace`
 * (RANS_OK if none), then clears it. */
int rans_get_status(void *workspace, void *stream);

/* ------------------------------------------------------- diagnostics ---- */

/*
 * The encoder's division step on its own: q[i] = x[i] / f[i] and
 * r[i] = x[i] % f[i] for x < 2^47 f, 1 <= f <= 65536, computed the way the
 * encoder does (a double-precision quotient estimate and an exact integer
 * correction).  For tests.  Asynchronous.
 */
int rans_debug_divide(const uint64_t *x, const uint32_t *f, int64_t n, uint64_t *q,
                      uint32_t *r, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RANS_B200_H */
