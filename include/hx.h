/*
 * hx.h -- C ABI of the fixed-codebook entropy coder for 8-bit tensor symbols (e4m3 / INT8 bytes)
 * on NVIDIA B200 (sm_100a).
 *
 * Method. "Single-Stage Huffman Encoder for ML Compression" (abstract): a Huffman codebook is
 * fixed in advance from the average symbol distribution of previous batches, so the data path
 * runs no frequency pass, builds no codebook and ships no codebook with the data. "Quad Length
 * Codes for Lossless Compression of e4m3" (abstract, Tables 1-2): a variant whose code is a 3-bit
 * area prefix followed by a fixed-width index inside the area, driven by a 256-entry table.
 * "Lossless" is exact reconstruction of every input byte.
 *
 * Conventions for every call below.
 *  - Pointers named d_* are device memory; all others are host memory. Every buffer belongs to
 *    the caller: the library never allocates, frees or synchronises. Device work is enqueued on
 *    `stream` (a cudaStream_t passed as void*; NULL = the legacy default stream) in call order.
 *  - The return value (int) carries host-detected errors only: bad arguments, unsupported
 *    alignment, launch failures. 0 = enqueued. Errors found in the data on the device (an
 *    uncodable symbol, a corrupt stream, a codebook mismatch, a full output buffer) are OR-ed
 *    into the caller's device word *d_status, which the caller zeroes before and reads after the
 *    stream is synchronised. Data errors never trap the device: reads are clamped to the
 *    buffers' valid ranges, and no kernel waits for another block.
 *  - d_in / d_out / d_stream must be 16-byte aligned (as every torch allocation is); n < 2^32.
 *
 * Stream format (version 1). All integers little-endian; offsets from the stream start.
 *    0 u32 magic 0x31305848 ("HX01")   4 u8 version = 1   5 u8 kind (0 Huffman, 1 QLC)
 *    6 u8 lmax (Huffman: the build's limit; QLC: 11)       7 u8 0
 *    8 u32 chunk = 4096 symbols        12 u32 sub-streams per chunk = 8
 *   16 u64 n                           24 u64 n_chunks = ceil(n / 4096)
 *   32 u64 total_words                 40 u64 codebook hash (FNV-1a-64, see hx_codebook.hash)
 *   48 16 zero bytes
 *   64 u32 word_off[n_chunks + 1]: payload word where each chunk starts; [n_chunks] = total
 *    S = round_up(64 + 4 * (n_chunks + 1), 16): u16 sync[n_chunks][8]. sync[c][0] = the number
 *        of valid bits of chunk c; sync[c][k], k = 1..7, = bit offset of the chunk's symbol 512k
 *        (the bit count when the chunk has no symbol 512k).
 *    P = S + 16 * n_chunks = hx_payload_offset(n): u32 payload[total_words]. Codes are written
 *        most-significant bit first (bit 31 of a word comes first) and each chunk is zero-padded
 *        to a whole word; two zero guard words follow. Stream size = P + 4 * (total_words + 2).
 */
#ifndef HX_H
#define HX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status bits: host return values and the device status word use the same codes. */
typedef enum {
  HX_OK = 0,
  HX_ERR_ARG = 1,        /* invalid argument (null pointer, size, alignment, kind)          */
  HX_ERR_CUDA = 2,       /* a CUDA runtime call or kernel launch failed                      */
  HX_ERR_UNCODABLE = 4,  /* encode: an input byte has no code word (seen-only codebook)      */
  HX_ERR_CORRUPT = 8,    /* decode: the stream is malformed or does not decode exactly      */
  HX_ERR_CODEBOOK = 16,  /* decode: the stream was written with another codebook or kind    */
  HX_ERR_TIMEOUT = 32,   /* encode: a bounded wait for the chunks before one ran out          */
  HX_ERR_CAPACITY = 64   /* encode: out_cap is too small; header.total_words holds the need */
} hx_status;

enum { HX_KIND_HUFFMAN = 0, HX_KIND_QLC = 1, HX_KIND_SHANNONIC = 2, HX_KIND_EXPGOLOMB = 3 };
enum { HX_SHN_K = 16, HX_SHN_L = 128, HX_SHN_R = 7 }; /* Shannonic: ranges, tANS states, log2 L */
enum { HX_CHUNK = 4096, HX_SUBSTREAMS = 8, HX_LMAX_MAX = 12, HX_QLC_LMAX = 11 };
enum { HX_CB_SEEN_ONLY = 1 }; /* hx_build_codebook flag: no code for bytes with count 0 */

/* Bytes of the device table block that hx_codebook_upload writes and the codecs read. */
#define HX_TABLES_BYTES 10240

/* A codebook, built on the host. Huffman: len/code per byte value (canonical, RFC 1951 order).
 * QLC: qlc_bits[a] index bits of area a, areas hold ranks [qlc_start[a], qlc_start[a+1]),
 * rank2sym[r] the byte value of rank r; len/code are filled in as well (len = 3 + bits). */
typedef struct {
  uint8_t kind;          /* HX_KIND_HUFFMAN or HX_KIND_QLC                                */
  uint8_t lmax;          /* Huffman: length limit of the build; QLC: 11                   */
  uint8_t len[256];      /* code length in bits of each byte value, 0 = no code           */
  uint16_t code[256];    /* code word, right-aligned in len bits                          */
  uint8_t qlc_bits[8];   /* QLC only                                                      */
  uint16_t qlc_start[9]; /* QLC only                                                      */
  uint8_t rank2sym[256]; /* QLC only                                                      */
  uint64_t hash;         /* FNV-1a-64 of [kind, lmax, len[256]] (Huffman) or of
                            [kind, 11, qlc_bits[8], rank2sym[256]] (QLC) or of
                            [kind, 7, nr, lo[1..nr-1], f[0..nr)] (Shannonic, bytes); the stream
                            header carries it in place of the codebook                     */
  uint8_t sh_nr;         /* Shannonic only: number of ranges (1..16)                     */
  uint16_t sh_lo[HX_SHN_K + 1]; /* range r holds byte values sh_lo[r] .. sh_lo[r+1]-1       */
  uint8_t sh_f[HX_SHN_K]; /* tANS frequency of each range, summing to 128                 */
} hx_codebook;

/* Length-limited canonical Huffman codebook from summed counts.
 * "Single-Stage Huffman Encoder for ML Compression", abstract: the counts are the sum over
 * previous equal-size batches (the average distribution, up to scale). Every byte value gets a
 * code (weight max(count, 1)) unless flags has HX_CB_SEEN_ONLY. Lengths come from package-merge
 * (Larmore & Hirschberg 1990) with limit lmax in [1, 12]; ties: leaves by (count, byte value),
 * a leaf before a package of equal weight. Codes are canonical (RFC 1951 section 3.2.2).
 * counts: host u64[256]. Returns HX_ERR_ARG for a null pointer or an lmax the alphabet cannot
 * fit in (2^lmax < number of coded symbols). */
int hx_build_codebook(const uint64_t* counts, int lmax, uint32_t flags, hx_codebook* out);

/* Quad Length Code from counts. "Quad Length Codes for Lossless Compression of e4m3", abstract
 * and Tables 1-2: byte values ranked by count (descending, ties to the smaller value) fill 8
 * areas in order; area a codes its symbols as a (3 bits) followed by the rank inside the area
 * (qlc_bits[a] bits). Widths are non-decreasing, hold all 256 ranks, use at most max_distinct
 * distinct values (4 = "quad"; 1..8), and minimise the mean code length; ties go to the
 * lexicographically smallest width vector. flags must be 0. */
int hx_qlc_build(const uint64_t* counts, int max_distinct, uint32_t flags, hx_codebook* out);

/* Shannonic codebook from counts: the review page's range-partitioned coder. The 256 byte values
 * are split by dynamic programming into at most K (1..16) contiguous ranges minimising the sum
 * over ranges of W_r log2(W / W_r) + W_r ceil(log2 size_r) (range entropy plus fixed-width
 * offset bits; weights max(count, 1)); ties go to the smallest split point, then the fewest
 * ranges. The range index is coded by tANS with 128 states: frequencies
 * f_r = max(1, floor(128 W_r / W)), a shortfall given +1 at a time to the largest remainders
 * (ties to the lower range, cycling), an excess taken -1 at a time from the largest f_r > 1
 * (ties to the lower range); states spread with step 83. The offset inside the range takes
 * ceil(log2 size_r) bits. flags must be 0. */
int hx_shannonic_build(const uint64_t* counts, int K, uint32_t flags, hx_codebook* out);

/* Exp-Golomb codebook: the universal code the QLC page contrasts QLC with ("faster to decode
 * but [not exploiting] the symbol frequency distributions"), as a no-table reference point. A
 * byte b maps to an index v -- map 0 (sign-magnitude bytes such as e4m3): v = ((b & 0x7f) << 1)
 * | (b >> 7); map 1 (two's complement bytes such as INT8): zigzag, v = 2x for x >= 0, -2x - 1 for
 * x < 0 -- and v is coded by Exp-Golomb of order k: floor(log2(v / 2^k + 1)) zeros, then v + 2^k
 * in binary (ITU-T H.264 section 9.1 is order 0). order 5..8 keeps every code within 12 bits.
 * The codebook is a prefix code like a Huffman one (len/code filled, lmax = order); hash =
 * FNV-1a-64 of [3, order, map]. */
int hx_expgolomb_build(int order, int map, hx_codebook* out);

/* Pack a codebook into the HX_TABLES_BYTES table block in host memory (host_tables): the
 * encoder's code/length entry per byte value and the decoder's window table (for a QLC code the
 * window table is computed from the area widths and the rank table), plus the codebook's kind,
 * limit and hash. "Single-Stage Huffman Encoder for ML Compression", abstract: the sender and
 * the receiver hold the same fixed codebook, so this block is built once per codebook, never per
 * batch. The block's layout is private to the library. */
int hx_codebook_tables(const hx_codebook* cb, void* host_tables);

/* Pack and copy the table block to d_tables (HX_TABLES_BYTES of device memory) on `stream`.
 * cb may be released when the call returns. Same source as hx_codebook_tables. */
int hx_codebook_upload(const hx_codebook* cb, void* d_tables, void* stream);

/* Histogram of byte values: d_counts[v] += occurrences of v in d_in[0..n). d_counts is a
 * device u32[256] that accumulates (zero it first for a fresh count); n < 2^32.
 * "Single-Stage Huffman Encoder for ML Compression", abstract (the frequency analysis whose
 * running average defines the next fixed codebook). */
int hx_histogram(const uint8_t* d_in, uint64_t n, uint32_t* d_counts, void* stream);

/* Layout helpers (pure functions of n): offsets and sizes of the stream format above. The pages
 * fix no format; this one follows from decoding every chunk and sub-stream in parallel with no
 * codebook shipped (the stream format, no passage). */
uint64_t hx_payload_offset(uint64_t n);   /* P above                                         */
uint64_t hx_sync_offset(uint64_t n);      /* S above                                         */
uint64_t hx_encode_bound(uint64_t n);     /* largest stream for n bytes: P + 4*(1536*chunks+2) */
uint64_t hx_scratch_bytes(uint64_t n);    /* device scratch of an encode: 8*chunks + 16       */

/* Encode d_in[0..n) with the fixed Huffman codebook in d_tables into the stream d_out.
 * "Single-Stage Huffman Encoder for ML Compression", abstract (fixed codebook, nothing sent
 * but the coded data and a hash of the codebook). One pass over the input: each chunk's word
 * offset comes from the chunks before it through a bounded wait (see hx_encode_bounded).
 * d_out: out_cap bytes, at least hx_payload_offset(n) + 8. If the coded stream does not fit,
 * HX_ERR_CAPACITY is raised in *d_status, the header (with total_words) and the index are
 * still written, and no payload word is written at or past the space that out_cap leaves (the
 * chunks that fit may have written theirs). d_scratch: hx_scratch_bytes(n) bytes of device
 * memory, contents ignored on entry and clobbered (the call clears what it needs first). d_hist: NULL, or a device u32[256] that accumulates
 * the histogram of d_in (as hx_histogram) in the same pass. d_status: device u32.
 * Bytes with no code word raise HX_ERR_UNCODABLE and emit no bits. Tables of the wrong kind
 * raise HX_ERR_ARG in *d_status. */
int hx_encode(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out, uint64_t out_cap,
              void* d_scratch, uint32_t* d_hist, uint32_t* d_status, void* stream);

/* Decode the stream d_stream (stream_bytes bytes) into d_out[0..n_expected).
 * "Single-Stage Huffman Encoder for ML Compression", abstract: the receiver decodes with the
 * same fixed codebook the sender used, identified by the hash in the header; "Quad Length Codes
 * for Lossless Compression of e4m3", abstract: Huffman decoding is bit-sequential, which the
 * stream's 8 sub-streams per 4096-symbol chunk turn into independent runs.
 * The header must match: magic, version, chunk, sub-streams, n == n_expected (else
 * HX_ERR_CORRUPT), kind, lmax and hash == the tables' (else HX_ERR_CODEBOOK). Every chunk's
 * index entries are checked, and each of its 8 sub-streams must decode to exactly the bit
 * offset where the next one starts (else HX_ERR_CORRUPT; d_out is then unspecified).
 * Returns HX_ERR_CORRUPT at once when stream_bytes cannot hold the index for n_expected. */
int hx_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes, uint8_t* d_out,
              uint64_t n_expected, uint32_t* d_status, void* stream);

/* The same two calls for a QLC codebook (kind 1 tables): identical stream layout and rules.
 * "Quad Length Codes for Lossless Compression of e4m3", abstract: a code word is the 3-bit
 * area, then the area's fixed number of index bits; the index picks the symbol through a
 * 256-entry rank table. The GPU decoder folds these three steps into one lookup in a 4096-entry
 * window table that hx_codebook_tables precomputes from the area widths and the rank table. */
int hx_qlc_encode(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                  uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                  void* stream);
int hx_qlc_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes,
                  uint8_t* d_out, uint64_t n_expected, uint32_t* d_status, void* stream);

/* Decode with a set of table blocks: the device picks, by the codebook hash in the stream's
 * header, the block to decode with (the first of the right kind whose lmax and hash match), so
 * a receiver that keeps several codebook versions needs no host round trip to choose. d_tables:
 * a HOST array of n_tables device pointers (1 <= n_tables <= HX_MAX_TABLE_SET), each a
 * HX_TABLES_BYTES block; blocks that are not valid tables of this kind are skipped. No match
 * raises HX_ERR_CODEBOOK. Otherwise as hx_decode / hx_qlc_decode (kind 0 / 1), which are this
 * call with a set of one. "Single-Stage Huffman Encoder for ML Compression", abstract (sender and
 * receiver share the codebook; only its identity travels with the data). */
#define HX_MAX_TABLE_SET 8
int hx_decode_set(uint32_t kind, const void* const* d_tables, uint32_t n_tables,
                  const void* d_stream, uint64_t stream_bytes, uint8_t* d_out,
                  uint64_t n_expected, uint32_t* d_status, void* stream);

/* hx_encode (and hx_qlc_encode, hx_expgolomb_encode, hx_shannonic_encode) with its bounded wait
 * exposed, for failure-detection tests; the pages have no counterpart (they describe no GPU
 * encoder). The encoder reads its input once: each chunk (kind 2: each group of 4 chunks)
 * publishes its word count as soon as it has measured it, and learns its word offset from the
 * ones before it (they are always running, so the wait ends). Every such wait is still bounded:
 * after wait_ns nanoseconds (hx_encode uses 2 s) the chunk raises HX_ERR_TIMEOUT in *d_status and
 * writes no payload, and every chunk still waiting gives up at once; the kernel completes and the
 * context stays usable. withhold: a chunk (kind 2: a group) that never publishes its count
 * (UINT64_MAX: none), so that the ones after it time out. flush_rounds: with d_hist and kinds 0,
 * 1, 3, the chunks a warp codes between its flushes of the fused counts into d_hist (0: the 128
 * of hx_encode; at most 4096, else HX_ERR_ARG), so that a test can make the flush run often;
 * kind 2 counts into 32-bit tables per warp and flushes once. Other arguments and errors as
 * hx_encode. */
int hx_encode_bounded(uint32_t kind, const void* d_tables, const uint8_t* d_in, uint64_t n,
                      void* d_out, uint64_t out_cap, void* d_scratch, uint32_t* d_hist,
                      uint32_t* d_status, uint64_t wait_ns, uint64_t withhold,
                      uint32_t flush_rounds, void* stream);

/* Shannonic encode and decode (kind 2 tables): the same chunked stream, sub-stream framing and
 * index as hx_encode; inside a sub-stream the bits come from tANS run from its last symbol to
 * its first, starting in state 128: per symbol the offset (ceil(log2 size) bits), then the low
 * nb bits of the state (nb making state >> nb fall in [f_r, 2 f_r)), then the range's next
 * state; after the first symbol the final state minus 128 in 7 bits. The decoder reads each
 * sub-stream backwards from its end and must finish in state 128 exactly at its first bit (else
 * HX_ERR_CORRUPT). A sub-stream can take up to 15 bits per symbol: size d_out with
 * hx_shannonic_encode_bound(n). Arguments, scratch, histogram and status as hx_encode. */
uint64_t hx_shannonic_encode_bound(uint64_t n); /* P + 4*(1922*chunks + 2)                   */
int hx_shannonic_encode(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                        uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                        void* stream);
int hx_shannonic_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes,
                        uint8_t* d_out, uint64_t n_expected, uint32_t* d_status, void* stream);

/* Exp-Golomb encode and decode (kind 3 tables from hx_expgolomb_build): the prefix-code path of
 * hx_encode / hx_decode with the universal code; same stream, arguments and errors. */
int hx_expgolomb_encode(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                        uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                        void* stream);
int hx_expgolomb_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes,
                        uint8_t* d_out, uint64_t n_expected, uint32_t* d_status, void* stream);

/* Allocation-free encode. The pages have no counterpart to this call: it exists for callers
 * that cannot allocate device memory when they encode -- for example code that runs under a
 * framework whose caching allocator has already reserved the device's memory (a stray
 * cudaMalloc there can fail or fragment the pool), or a latency-critical path that cannot afford
 * the implicit device synchronisation of cudaMalloc/cudaFree. It behaves exactly like hx_encode
 * with Huffman tables (same stream, same status bits) but takes no scratch argument: its scratch
 * lives in a fixed device array inside the library, sized for n <= HX_NOALLOC_MAX_BYTES, that
 * every GPU which loads the library keeps until the process exits.
 *  - n > HX_NOALLOC_MAX_BYTES is refused with HX_ERR_ARG; nothing is enqueued.
 *  - The first call on a device looks up that array's device address (once per device, with
 *    the device current); make that first call before any stream capture on the device.
 *  - All calls share the one array, and each call clears what must start at zero. Calls whose
 *    work overlaps on the GPU (other streams, other host threads) race on it: serialise them.
 *  - It calls no cudaMalloc, cudaFree or other allocating routine. */
#define HX_NOALLOC_MAX_BYTES (128ull << 20)
int hx_encode_noalloc(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                      uint64_t out_cap, uint32_t* d_hist, uint32_t* d_status, void* stream);

/* ---- Online single-stage loop -----------------------------------------------------------
 * "Single-Stage Huffman Encoder for ML Compression", abstract: the codebook for a batch comes
 * from the average symbol distribution of previous batches, so the data path has no frequency
 * pass and no codebook build, and no codebook travels with the data. A session runs that loop:
 * batch t (the t-th hx_session_encode call, from 0) is coded with the codebook built from the
 * summed histograms of batches t-lag-m+1 .. t-lag (m = history), which the encoder itself
 * counted (the fused histogram); before any batch is observed, from initial_counts (NULL: all
 * ones). Drift refresh (the "Shannonic" review of range-partitioned coding: rebuild when the
 * code stops fitting the data): when batch j is observed, drift_j = mean code length of batch j
 * under the codebook that coded it / its entropy - 1; if drift > cfg.drift > 0 the history
 * restarts from batch j alone. The schedule depends only on the histograms, never on timing.
 *
 * hx_planner is that bookkeeping alone, on the host (no device): hx_planner_codebook(t) returns
 * batch t's codebook once batches 0 .. t-lag (and no later one) have been observed, in order,
 * with hx_planner_observe. */
typedef struct {
  uint32_t kind;          /* HX_KIND_HUFFMAN or HX_KIND_QLC                                   */
  uint32_t lmax;          /* Huffman: length limit 1..12 (0 = 12)                             */
  uint32_t max_distinct;  /* QLC: distinct widths 1..8 (0 = 4)                                */
  uint32_t flags;         /* Huffman: 0 or HX_CB_SEEN_ONLY; QLC: 0                            */
  uint32_t history;       /* m, batches summed: 1..64                                         */
  uint32_t lag;           /* batch t uses histograms of batches <= t - lag: 1..8              */
  double drift;           /* refresh threshold (fraction above entropy); <= 0: never refresh  */
} hx_session_config;

typedef struct {
  uint64_t hash;          /* codebook hash the batch was coded with                           */
  uint32_t slot;          /* device table slot that held it                                   */
  int32_t observed;       /* 1 once its histogram has been folded into the plan               */
  int32_t refreshed;      /* 1 if it triggered a drift refresh                                */
  uint32_t pad;
  uint64_t symbols;       /* bytes counted (once observed)                                    */
  double drift;           /* its drift (NaN until observed, or for an all-empty batch)        */
} hx_batch_info;

typedef struct hx_planner hx_planner;
int hx_planner_create(const hx_session_config* cfg, const uint64_t* initial_counts,
                      hx_planner** out);
int hx_planner_codebook(hx_planner* p, uint64_t batch, hx_codebook* out);
int hx_planner_observe(hx_planner* p, uint64_t batch, const uint64_t* counts, int* refreshed,
                       double* drift);
void hx_planner_destroy(hx_planner* p);

/* A session owns host state (the plan; pinned host buffers for lag + 1 histograms and one table
 * block per slot; CUDA events); the device memory is the caller's: d_slots, n_slots table blocks
 * of HX_TABLES_BYTES (lag + 1 <= n_slots <= HX_MAX_TABLE_SET, 16-byte aligned), which create
 * zeroes (cudaMemset, synchronous). Use a session from one host thread and one stream.
 *  - hx_session_encode: waits (host) for the histogram of batch t - lag if the device has not
 *    finished it, builds batch t's codebook when the history changed and uploads it to the next
 *    slot, zeroes d_hist (device u32[256]) and encodes into d_out with the fused histogram (as
 *    hx_encode / hx_qlc_encode: same arguments, scratch, status), then copies d_hist to the host.
 *  - hx_session_decode: hx_decode_set over the slots. A stream stays decodable until its slot is
 *    reused, n_slots codebook changes later (after that: HX_ERR_CODEBOOK).
 *  - hx_session_drain: folds every histogram still in flight (waits for the stream).
 *  - hx_session_batch_info: what batch t was coded with, and its drift once observed. */
typedef struct hx_session hx_session;
int hx_session_create(const hx_session_config* cfg, const uint64_t* initial_counts,
                      void* const* d_slots, uint32_t n_slots, hx_session** out);
int hx_session_encode(hx_session* s, const uint8_t* d_in, uint64_t n, void* d_out,
                      uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                      void* stream);
int hx_session_decode(hx_session* s, const void* d_stream, uint64_t stream_bytes, uint8_t* d_out,
                      uint64_t n_expected, uint32_t* d_status, void* stream);
int hx_session_drain(hx_session* s);
int hx_session_batch_info(const hx_session* s, uint64_t batch, hx_batch_info* out);
void hx_session_destroy(hx_session* s);

/* Measurement helpers (host, fp64). Shannon entropy -sum p log2 p of counts[256] in bits per
 * symbol ("Single-Stage Huffman Encoder for ML Compression", abstract: the ideal the fixed code
 * is compared with), and the mean code length sum count*len / sum count of a codebook (for a
 * Shannonic codebook the tANS ideal, log2(128 / f_r) + offset bits per symbol of range r). Both
 * return 0 for an all-zero histogram and -1 for a null pointer. */
double hx_entropy(const uint64_t* counts);
double hx_mean_length(const uint64_t* counts, const hx_codebook* cb);

/* Library format version (1) and a static description of a status code. */
int hx_version(void);
const char* hx_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* HX_H */
