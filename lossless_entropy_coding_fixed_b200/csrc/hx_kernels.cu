// CUDA kernels of the hx library (sm_100a) and the C entry points that launch them.
//
// The method: "Single-Stage Huffman Encoder for ML Compression" (abstract) -- a codebook fixed
// from earlier batches, so the coder runs with no frequency pass and ships no codebook; "Quad
// Length Codes for Lossless Compression of e4m3" (abstract, Tables 1-2) -- the area code.
//
//   k_histogram  byte histogram: 16-byte loads, four in flight per thread; one table of 32
//                copies per block in shared memory (lane l counts into copy l, so a warp's
//                atomics never conflict), one global atomic per non-empty bin and block.
//
//   k_encode     one pass over the input. A warp takes the next chunk from a counter and loads it
//                with coalesced 16-byte loads (16 bytes of each sub-stream per lane); the length
//                pass (one lookup per symbol in the lane's own copy of the length table, a shared
//                atomic that also counts the fused histogram) and a warp scan give the sync row
//                and the chunk's word count, which it publishes at once; the coding pass joins two
//                codes per 32-bit register, appends them to a 64-bit accumulator and ORs each
//                finished word into the warp's chunk buffer; a decoupled look-back over the
//                chunks before it (64 per round trip to L2, bounded wait) gives the chunk's word
//                offset, and the chunk leaves with coalesced stores.
//
//   k_decode     one thread per sub-stream (8 per chunk, 128 chunks per 1024-thread block). The
//                two payload words in use and a bit offset into them give the next 32 bits with
//                one funnel shift, enough for two codes; two more words are already requested
//                (predicated 4-byte loads, no lane-dependent branch). One lookup per symbol in
//                the 4096-entry shared table gives symbol and length for either kind (for a QLC
//                code it is precomputed from the area widths and the rank table). 32 decoded
//                bytes leave as one 32-byte store (a whole sector). Every sub-stream must end
//                exactly where the next one starts. Blocks whose sub-streams start crowded in one
//                bank of their lines (codes of one length) vote per warp and may read 16-byte
//                blocks instead.
//
//   k_sh_encode  the Shannonic range coder's encoder: tANS over range indices with one table
//                entry per step. A warp takes the next group of 4 chunks, runs one sub-stream per
//                lane and parks its bits in shared memory (a tANS sub-stream's length is known
//                only once it has been run), publishes the group's word count, learns its offset
//                by the same look-back as k_encode, and copies the chunks out with coalesced
//                stores; a group with a sub-stream too long for its region is coded again
//                straight into the payload.
//   k_sh_decode  reads each sub-stream backwards, one thread each, with 16-byte payload blocks
//                one block ahead and a 16-byte state entry per symbol.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "hx.h"
#include "hx_tables.h"

namespace {

constexpr uint32_t kMagic = 0x31305848u;  // "HX01"
constexpr uint32_t kChunk = HX_CHUNK;
constexpr uint32_t kSubLen = HX_CHUNK / HX_SUBSTREAMS;
constexpr int kDecThreads = 256;  // Shannonic decode: 8 threads per chunk, 32 chunks per block
constexpr int kHistThreads = 256;

__host__ __device__ inline uint64_t n_chunks_of(uint64_t n) { return (n + kChunk - 1) / kChunk; }
__host__ __device__ inline uint64_t sync_offset(uint64_t n) {
  return (64 + 4 * (n_chunks_of(n) + 1) + 15) / 16 * 16;
}
__host__ __device__ inline uint64_t payload_offset(uint64_t n) {
  return sync_offset(n) + 16 * n_chunks_of(n);
}

// ---------------------------------------------------------------------------------- histogram
// One table of 32 copies per block: bin v of copy l at word 32 v + l, lane l counting into copy l,
// so the 32 increments of a warp never share a bank; the copies are summed into the caller's
// counts at the end (one global atomic per non-empty bin and block).
static_assert(kHistThreads == 256, "k_histogram sums bin `tid` over the copies");
__global__ void __launch_bounds__(kHistThreads) k_histogram(const uint8_t* __restrict__ in,
                                                            uint64_t n, uint32_t* counts) {
  __shared__ uint32_t bins[256 * 32];
  const int tid = threadIdx.x, lane = tid & 31;
  for (int i = tid; i < 256 * 32; i += kHistThreads) bins[i] = 0;
  __syncthreads();
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(bins) + 4 * lane;
  auto count4 = [&](uint32_t w) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t a = __byte_perm(w, 0u, 0x4440u + j) * 128u + base;
      asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(a) : "memory");
    }
  };
  const uint64_t nvec = n / 16;
  const uint4* v = reinterpret_cast<const uint4*>(in);
  const uint64_t stride = (uint64_t)gridDim.x * kHistThreads;
  uint64_t i = blockIdx.x * (uint64_t)kHistThreads + tid;
  // four 16-byte loads in flight per thread, then their 64 bytes counted
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    uint4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = __ldcs(v + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      count4(x[u].x);
      count4(x[u].y);
      count4(x[u].z);
      count4(x[u].w);
    }
  }
  for (; i < nvec; i += stride) {
    const uint4 x = __ldcs(v + i);
    count4(x.x);
    count4(x.y);
    count4(x.z);
    count4(x.w);
  }
  if (blockIdx.x == 0)
    for (uint64_t i = nvec * 16 + tid; i < n; i += kHistThreads) atomicAdd(&bins[in[i] * 32 + lane], 1u);
  __syncthreads();
  uint32_t sum = 0;
  for (int l = 0; l < 32; ++l) sum += bins[tid * 32 + ((l + tid) & 31)];
  if (sum) atomicAdd(&counts[tid], sum);
}

// ---------------------------------------------------------------------------------- encode
// The arguments of an encode (k_encode for kinds 0, 1, 3; k_sh_encode for kind 2, whose
// look-back unit is a group of 4 chunks).
struct EncodeArgs {
  const hx::Tables* tables;
  const uint8_t* in;
  uint64_t n;
  uint8_t* out;
  uint64_t cap;
  uint32_t* hist;  // optional fused histogram
  uint32_t* status;
  uint32_t kind;
  uint64_t* look;     // scratch: each chunk's (group's) published word count or offset (zeroed)
  uint32_t* counter;  // scratch: next chunk (group) to take (zeroed)
  uint64_t wait_ns;   // limit of one chunk's wait for its predecessors
  uint64_t withhold;  // a chunk that publishes nothing (failure tests), else ~0
  uint32_t flush;     // fused histogram: a warp's chunks between its flushes of the counts
};

// Every header field but total_words.
__device__ inline void write_header(const EncodeArgs& a) {
  uint32_t* h32 = reinterpret_cast<uint32_t*>(a.out);
  uint64_t* h64 = reinterpret_cast<uint64_t*>(a.out);
  h32[0] = kMagic;
  h32[1] = 1u | (a.kind << 8) | (a.tables->lmax << 16);
  h32[2] = kChunk;
  h32[3] = HX_SUBSTREAMS;
  h64[2] = a.n;
  h64[3] = n_chunks_of(a.n);
  h64[5] = a.tables->hash;
  h64[6] = 0;
  h64[7] = 0;
  // zero the alignment gap between word_off[n_chunks] and the 16-byte aligned sync table
  const uint64_t gap = 64 + 4 * (n_chunks_of(a.n) + 1);
  for (uint64_t i = gap; i < sync_offset(a.n); i += 4) h32[i / 4] = 0;
}

// The tables' code word of byte value `sym` as (code, len); a damaged entry (a length above the
// limit or a code longer than its length) reads as no code word and raises HX_ERR_ARG.
__device__ inline uint32_t checked_code(const EncodeArgs& a, uint32_t sym, uint32_t* code) {
  const uint32_t t = a.tables->enc[sym];  // (code << 4) | len
  const uint32_t len = t & 15u, c = t >> 4;
  if (len > HX_LMAX_MAX || (c >> len) != 0) {
    atomicOr(a.status, (uint32_t)HX_ERR_ARG);
    *code = 0;
    return 0;
  }
  *code = c;
  return len;
}

// The 16 bytes of sub-stream k that lane `lane` codes: a 16-byte load for a whole chunk, byte
// loads (0 past the end) for the ragged last one. Returns how many of the 16 exist.
__device__ __forceinline__ uint32_t load16(const EncodeArgs& a, uint32_t c, uint32_t k,
                                           uint32_t lane, bool whole, uint4& v) {
  const uint64_t first = (uint64_t)c * kChunk + k * kSubLen + lane * 16;
  if (whole) {
    v = __ldg(reinterpret_cast<const uint4*>(a.in + first));
    return 16;
  }
  uint32_t w[4] = {0, 0, 0, 0};
  const uint32_t valid = first < a.n ? (uint32_t)min((uint64_t)16, a.n - first) : 0u;
  for (uint32_t j = 0; j < valid; ++j) w[j >> 2] |= (uint32_t)a.in[first + j] << (8 * (j & 3));
  v = make_uint4(w[0], w[1], w[2], w[3]);
  return valid;
}

constexpr uint32_t kMaxChunkWords = HX_CHUNK * HX_LMAX_MAX / 32;  // 1536: a chunk's largest size

// ---------------------------------------------------------------------------------- encode, one pass
// k_encode reads the input once. A warp takes the next chunk from a counter, loads it (16 bytes
// of each sub-stream per lane: every load instruction reads 512 contiguous bytes), sums the code
// lengths of its 16-symbol segments (with the fused histogram), scans them into the sync row, and
// publishes the chunk's word count at once. It then codes the chunk into its shared-memory buffer
// while the chunks before it finish, learns its word offset from them (a decoupled look-back:
// the nearest published offset plus the word counts in between), and copies the chunk out.
// Chunks are taken in order by running warps, each of which publishes its count before it waits,
// so every wait ends; each is still bounded (wait_ns), after which the chunk raises HX_ERR_TIMEOUT
// and writes no payload, and every later wait gives up at once.
constexpr int kEncThreads = 768;  // one block of 24 warps per SM sharing the two tables
constexpr uint32_t kEncWarps = kEncThreads / 32;
// 24-bit counts in the length table (bits 8-31; the length in bits 0-7, so 16 summed entries keep
// their bit count, at most 16 * 12, in the low byte). A warp that has taken `flush` chunks since
// its last flush clears the whole table into the histogram by itself (atomic ANDs beside the
// other warps' atomic adds), so between two flushes every warp takes fewer than `flush` chunks
// of 128 symbols per lane, and no entry grows by 2^24. The block's last counts go out once all
// its warps are done; no warp waits at a block barrier while chunks are left.
constexpr uint32_t kEncCountShift = 8;
constexpr uint32_t kEncFlushRounds = 128;     // `flush` of hx_encode (0.4 % of the work)
constexpr uint32_t kEncFlushRoundsMax = 4096;  // the largest `flush` hx_encode_bounded takes
static_assert(uint64_t(kEncWarps) * kEncFlushRoundsMax * 128 < (1ull << 24), "24-bit counts");
constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s
constexpr uint64_t kLookAgg = 1ull << 62;   // word count of the chunk alone
constexpr uint64_t kLookPre = 2ull << 62;   // word offset of the chunk's end (inclusive prefix)
constexpr uint64_t kLookValue = (1ull << 62) - 1;
constexpr int kLookLoads = 2;  // look-back loads per lane: a window of 64 chunks

// Two tables, entries [symbol][copy] with lane l using copy l (no bank conflicts): `len` =
// (count << 8) | len for the length pass (with the fused histogram the lookup is a shared atomic
// that adds 1 << 8), `code` = (code << 20) | len for the coding pass.
struct EncSmem {
  uint32_t len[256 * 32];
  uint32_t code[256 * 32];
  alignas(16) uint32_t buf[kEncWarps][kMaxChunkWords];  // each warp's chunk, zero between chunks
  uint32_t sink[kEncWarps][32];  // a word per lane for the stores a pair does not make
};

__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// 32-bit shared-memory addresses for the encoder's tables and buffers (no generic 64-bit address
// arithmetic): byte J of w picks the row of a [symbol][32] table with one byte permute and one
// multiply-add; `base` is the table's shared address plus 4 * lane.
template <int J>
__device__ __forceinline__ uint32_t row_addr(uint32_t w, uint32_t base) {
  return __byte_perm(w, 0u, 0x4440u + J) * 128u + base;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t atoms_add_u32(uint32_t a, uint32_t x) {
  uint32_t v;
  asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(v) : "r"(a), "r"(x) : "memory");
  return v;
}
__device__ __forceinline__ void reds_or_u32(uint32_t a, uint32_t x) {
  asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(a), "r"(x) : "memory");
}

// The bit count of the 16 bytes in v (count of them exist): the sum of their length-table entries
// ((count << 8) | len; the low 8 bits of the sum are the bit count, at most 16 * 12). With HIST
// each lookup is a shared atomic that also adds 1 to the entry's count.
template <bool HIST, bool COMPLETE, bool WHOLE>
__device__ __forceinline__ uint32_t lengths16(uint32_t base, const uint4& v, uint32_t count,
                                              bool& uncodable) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t sum = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (WHOLE || (uint32_t)(4 * q + j) < count) {
        const uint32_t a = j == 0   ? row_addr<0>(w[q], base)
                           : j == 1 ? row_addr<1>(w[q], base)
                           : j == 2 ? row_addr<2>(w[q], base)
                                    : row_addr<3>(w[q], base);
        const uint32_t e = HIST ? atoms_add_u32(a, 1u << kEncCountShift) : lds_u32(a);
        sum += e;
        if (!COMPLETE) uncodable |= (e & 0xffu) == 0;
      }
    }
  }
  return HIST ? sum & ((1u << kEncCountShift) - 1u) : sum;  // without HIST every count is 0
}

// Word offset of chunk c (c > 0) from the chunks before it, read 32 * kLookLoads at a time by
// the warp (each lane's loads are independent, so a window costs one round trip to L2): the sum
// of the counts back to (and including) the nearest published offset. ~0 when the wait ran out
// or another chunk's did. A chunk can only take an offset that was published within its window,
// so the window's width and the round trip's length bound how fast offsets travel down the
// chunks: 64 chunks and a one-instruction warp reduction measured 7 % faster than 32 and a
// shuffle reduction.
__device__ uint64_t lookback(const EncodeArgs& a, uint32_t c, uint32_t lane) {
  constexpr int NL = kLookLoads;
  uint64_t excl = 0;
  const uint64_t t0 = global_ns();
  for (int64_t base = (int64_t)c - 1; base >= 0; base -= 32 * NL) {
    int64_t i[NL];
    uint64_t v[NL];
#pragma unroll
    for (int r = 0; r < NL; ++r) {
      i[r] = base - 32 * r - (int64_t)lane;
      v[r] = i[r] >= 0 ? ld_relaxed_u64(a.look + i[r]) : kLookPre;  // before chunk 0: offset 0
    }
    uint32_t need[NL];
    bool found;
    for (;;) {
      uint32_t wait = 0;
      found = false;
#pragma unroll
      for (int r = 0; r < NL; ++r) {
        const uint32_t p = __ballot_sync(0xffffffffu, (v[r] >> 62) == 2);
        const uint32_t z = __ballot_sync(0xffffffffu, (v[r] >> 62) == 0);
        // lanes up to the nearest published offset, or all of them (none past it)
        need[r] = found ? 0u : p ? ((p & (0u - p)) << 1) - 1u : 0xffffffffu;
        wait |= z & need[r];
        found |= p != 0;
      }
      if (wait == 0) break;
      const bool out = global_ns() - t0 > a.wait_ns ||
                       (*reinterpret_cast<volatile uint32_t*>(a.status) & HX_ERR_TIMEOUT);
      if (__any_sync(0xffffffffu, out)) return ~0ull;
      __nanosleep(64);
#pragma unroll
      for (int r = 0; r < NL; ++r)
        if ((v[r] >> 62) == 0) v[r] = ld_relaxed_u64(a.look + i[r]);
    }
    // offsets and counts are below 2^32 (a stream holds fewer than 2^32 words), and so is the
    // window's sum: one warp reduction instruction
    uint32_t val = 0;
#pragma unroll
    for (int r = 0; r < NL; ++r) val += (need[r] >> lane) & 1u ? (uint32_t)(v[r] & kLookValue) : 0u;
    excl += __reduce_add_sync(0xffffffffu, val);
    if (found) break;
  }
  return excl;
}

// Codes the lane's 16 symbols of one sub-stream (bytes of v, `count` of them) as the bits
// [s, s + their length) of the chunk buffer, which is zero there: two codes are joined in a
// 32-bit register (at most 24 bits) and appended to a 64-bit accumulator; each finished word,
// and the unfinished last one, is OR-ed into the buffer (the pieces of neighbouring lanes share
// the first and the last word). Every pair makes one OR, into the lane's sink word when it
// finishes no word, so the loop has no branch.
template <bool WHOLE>
__device__ __forceinline__ void pack_segment(uint32_t base, const uint4& v, uint32_t count,
                                             uint32_t buf, uint32_t sink, uint32_t s) {
  uint32_t d = buf + 4 * (s >> 5) - sink, nacc = s & 31, hi = 0, lo = 0;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t e[4];
    e[0] = (WHOLE || 4 * q + 0 < (int)count) ? lds_u32(row_addr<0>(w[q], base)) : 0u;
    e[1] = (WHOLE || 4 * q + 1 < (int)count) ? lds_u32(row_addr<1>(w[q], base)) : 0u;
    e[2] = (WHOLE || 4 * q + 2 < (int)count) ? lds_u32(row_addr<2>(w[q], base)) : 0u;
    e[3] = (WHOLE || 4 * q + 3 < (int)count) ? lds_u32(row_addr<3>(w[q], base)) : 0u;
#pragma unroll
    for (int h = 0; h < 4; h += 2) {
      // The integer logic pipe is the busy one, so: the pair's length comes from one add (the
      // codes sit above bit 20), the shift by l1 is a wrapping funnel shift (it reads only
      // e[h + 1]'s low 5 bits, the length), and the bookkeeping is in multiply-adds: the word
      // goes to sink + f * d, d = (its address) - sink, f = 1 when a word is finished. The
      // codes' bits do not overlap, so the adds are ORs.
      const uint32_t pl = (e[h] + e[h + 1]) & 0xffu;
      const uint32_t pc = __funnelshift_l(0u, e[h] >> 20, e[h + 1]) + (e[h + 1] >> 20);
      hi = __funnelshift_l(lo, hi, pl);
      lo = (lo << pl) + pc;
      nacc += pl;
      const uint32_t f = nacc >> 5;  // 0 or 1: a pair adds at most 24 bits to at most 31
      nacc &= 31u;
      reds_or_u32(sink + f * d, __funnelshift_r(lo, hi, nacc));
      d += f * 4u;
    }
  }
  reds_or_u32(nacc ? sink + d : sink, lo << (32 - nacc));
}


// The chunk's word offset from the chunks before it, published as its end offset; false when
// the wait ran out (the chunk then writes no payload).
__device__ __forceinline__ bool chunk_offset(const EncodeArgs& a, uint32_t c, uint32_t words,
                                             uint32_t lane, uint64_t& off) {
  off = 0;
  if (c == 0) return true;
  off = lookback(a, c, lane);
  if (off == ~0ull) {
    if (lane == 0) atomicOr(a.status, (uint32_t)HX_ERR_TIMEOUT);
    return false;
  }
  if (lane == 0 && c != a.withhold) st_relaxed_u64(a.look + c, kLookPre | (off + words));
  return true;
}

// The coded chunk's words out at its offset, and its buffer cleared.
__device__ __forceinline__ void chunk_copy(const EncodeArgs& a, uint32_t c, uint32_t words,
                                           uint32_t* buf, uint32_t lane, uint64_t off,
                                           bool copy) {
  const uint64_t n = a.n;
  const uint32_t nchunks = (uint32_t)n_chunks_of(n);
  if (copy) {
    const uint64_t P = payload_offset(n);
    uint32_t* word_off = reinterpret_cast<uint32_t*>(a.out + 64);
    uint32_t* payload = reinterpret_cast<uint32_t*>(a.out + P);
    const uint64_t end = off + words;
    if (lane == 0) word_off[c] = (uint32_t)off;
    if (c + 1 == nchunks && lane == 0) {
      reinterpret_cast<uint64_t*>(a.out)[4] = end;
      word_off[nchunks] = (uint32_t)end;
    }
    // payload words that fit before the 2 guard words at the end of the caller's buffer
    const uint64_t room = a.cap >= P + 8 ? (a.cap - P - 8) / 4 : 0;
    if (end > room) {
      if (lane == 0) atomicOr(a.status, (uint32_t)HX_ERR_CAPACITY);
    } else {
      for (uint32_t i = lane; i < words; i += 32) payload[off + i] = buf[i];
      if (c + 1 == nchunks && lane < 2) payload[end + lane] = 0;
    }
  }
  __syncwarp();
  // leave the buffer zero for the next chunk
  uint4* b4 = reinterpret_cast<uint4*>(buf);
  for (uint32_t q = lane; q < (words + 3) / 4; q += 32) b4[q] = make_uint4(0, 0, 0, 0);
  __syncwarp();
}

// A coded chunk's way out (see k_encode): its word offset, then its words.
__device__ __forceinline__ void chunk_out(const EncodeArgs& a, uint32_t c, uint32_t words,
                                          uint32_t* buf, uint32_t lane) {
  __syncwarp();
  uint64_t off;
  const bool copy = chunk_offset(a, c, words, lane, off);
  chunk_copy(a, c, words, buf, lane, off, copy);
}

// One chunk by one warp (see k_encode).
template <bool HIST, bool COMPLETE, bool WHOLE>
__device__ __forceinline__ void encode_chunk(const EncodeArgs& a, EncSmem& sm, uint32_t c,
                                             uint32_t* buf, uint32_t* sink, bool& uncodable) {
  const uint32_t lane = threadIdx.x & 31, lane4 = lane * 4;
  const uint64_t n = a.n;
  const uint32_t nchunks = (uint32_t)n_chunks_of(n);
  uint32_t first[HX_SUBSTREAMS], row[HX_SUBSTREAMS];
  uint32_t run = 0;
  {
    // the length pass: 16 bytes of each sub-stream per lane (coalesced 512-byte loads)
    uint4 v[HX_SUBSTREAMS];
    uint32_t valid[HX_SUBSTREAMS];
#pragma unroll
    for (int k = 0; k < HX_SUBSTREAMS; ++k) valid[k] = load16(a, c, k, lane, WHOLE, v[k]);
    const uint32_t lenbase = (uint32_t)__cvta_generic_to_shared(sm.len) + lane4;
#pragma unroll
    for (int k = 0; k < HX_SUBSTREAMS; k += 2) {
      // two sub-streams per scan: bit counts < 2^16 in the two halves of a word
      const uint32_t b0 = lengths16<HIST, COMPLETE, WHOLE>(lenbase, v[k], valid[k], uncodable);
      const uint32_t b1 = lengths16<HIST, COMPLETE, WHOLE>(lenbase, v[k + 1], valid[k + 1],
                                                           uncodable);
      uint32_t incl = b0 | (b1 << 16);
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= (uint32_t)d) incl += t;
      }
      const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
      row[k] = run;
      first[k] = run + (incl & 0xffffu) - b0;
      run += tot & 0xffffu;
      row[k + 1] = run;
      first[k + 1] = run + (incl >> 16) - b1;
      run += tot >> 16;
    }
  }
  const uint32_t words = (run + 31) >> 5;
  // publish the word count before anything waits
  if (lane == 0 && c != a.withhold)
    st_relaxed_u64(a.look + c, (c == 0 ? kLookPre : kLookAgg) | words);
  if (lane == 0) {
    uint4* sync = reinterpret_cast<uint4*>(a.out + sync_offset(n));
    sync[c] = make_uint4(run | (row[1] << 16), row[2] | (row[3] << 16), row[4] | (row[5] << 16),
                         row[6] | (row[7] << 16));
  }
  // the coding pass, sub-stream by sub-stream; the lane's bytes again (from L2, where the first
  // load left them), one sub-stream ahead of the coding
  const uint32_t f01 = first[0] | (first[1] << 16), f23 = first[2] | (first[3] << 16);
  const uint32_t f45 = first[4] | (first[5] << 16), f67 = first[6] | (first[7] << 16);
  const uint32_t codebase = (uint32_t)__cvta_generic_to_shared(sm.code) + lane4;
  const uint32_t buf32 = (uint32_t)__cvta_generic_to_shared(buf);
  const uint32_t sink32 = (uint32_t)__cvta_generic_to_shared(sink);
  uint4 vn;
  uint32_t cn = load16(a, c, 0, lane, WHOLE, vn);
#pragma unroll 1
  for (uint32_t k = 0; k < HX_SUBSTREAMS; ++k) {
    const uint4 vk = vn;
    const uint32_t ck = cn;
    if (k + 1 < HX_SUBSTREAMS) cn = load16(a, c, k + 1, lane, WHOLE, vn);
    const uint32_t fw = k < 2 ? f01 : k < 4 ? f23 : k < 6 ? f45 : f67;
    pack_segment<WHOLE>(codebase, vk, ck, buf32, sink32, (fw >> (16 * (k & 1))) & 0xffffu);
  }
  chunk_out(a, c, words, buf, lane);
}


template <bool HIST, bool COMPLETE>
__device__ void encode_chunks(const EncodeArgs& a, EncSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t nchunks = (uint32_t)n_chunks_of(a.n);
  const uint32_t full_chunks = (uint32_t)(a.n / kChunk);
  uint32_t* buf = sm.buf[warp];
  uint32_t* sink = &sm.sink[warp][lane];
  for (uint32_t q = lane; q < kMaxChunkWords / 4; q += 32)
    reinterpret_cast<uint4*>(buf)[q] = make_uint4(0, 0, 0, 0);
  __syncwarp();
  bool uncodable = false;
  for (uint32_t r = 1;; ++r) {
    uint32_t c = 0;
    if (lane == 0) c = atomicAdd(a.counter, 1u);
    c = __shfl_sync(0xffffffffu, c, 0);
    if (c >= nchunks) break;
    // the chunk a warp will most likely take one round from now, into L2
    const uint64_t ahead = (uint64_t)c + gridDim.x * kEncWarps;
    if (lane == 0 && ahead < full_chunks)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.in + ahead * kChunk),
                   "r"(kChunk)
                   : "memory");
    if (c < full_chunks) encode_chunk<HIST, COMPLETE, true>(a, sm, c, buf, sink, uncodable);
    else encode_chunk<HIST, COMPLETE, false>(a, sm, c, buf, sink, uncodable);
    if (HIST && r % a.flush == 0) {
      // this warp clears every count into the histogram (the other warps keep counting)
      const uint32_t t0 = (uint32_t)__cvta_generic_to_shared(sm.len);
      for (int sym = 0; sym < 256; ++sym) {
        uint32_t old;
        asm volatile("atom.shared.and.b32 %0, [%1], %2;"
                     : "=r"(old)
                     : "r"(t0 + 4u * (32u * sym + lane)), "r"(0xffu)
                     : "memory");
        const uint32_t cnt = __reduce_add_sync(0xffffffffu, old >> kEncCountShift);
        if (lane == 0 && cnt) atomicAdd(&a.hist[sym], cnt);
      }
    }
  }
  if (HIST) {
    // the counts since the warps' last flushes, once every warp is done
    __syncthreads();
    for (int sym = tid; sym < 256; sym += kEncThreads) {
      uint32_t sum = 0;
      for (int l = 0; l < 32; ++l) sum += sm.len[sym * 32 + l] >> kEncCountShift;
      if (sum) atomicAdd(&a.hist[sym], sum);
    }
  }
  if (!COMPLETE && __any_sync(0xffffffffu, uncodable) && lane == 0)
    atomicOr(a.status, (uint32_t)HX_ERR_UNCODABLE);
}

__global__ void __launch_bounds__(kEncThreads, 1) k_encode(EncodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  EncSmem& sm = *reinterpret_cast<EncSmem*>(smem_raw);
  const int tid = threadIdx.x;
  if (a.tables->magic != hx::kTablesMagic || a.tables->kind != a.kind) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, (uint32_t)HX_ERR_ARG);
    return;
  }
  bool complete = true;
  for (int i = tid; i < 256 * 32; i += kEncThreads) {
    uint32_t code;
    const uint32_t len = checked_code(a, i / 32, &code);
    complete &= len != 0;
    sm.len[i] = len;
    sm.code[i] = (code << 20) | len;
  }
  complete = __syncthreads_and(complete);
  if (blockIdx.x == 0 && tid == 0) {
    write_header(a);
    if (a.n == 0) {  // no chunk writes the totals
      reinterpret_cast<uint64_t*>(a.out)[4] = 0;
      reinterpret_cast<uint32_t*>(a.out + 64)[0] = 0;
      if (a.cap >= payload_offset(0) + 8) {
        uint32_t* payload = reinterpret_cast<uint32_t*>(a.out + payload_offset(0));
        payload[0] = payload[1] = 0;
      }
    }
  }
  if (a.hist) {
    if (complete) encode_chunks<true, true>(a, sm);
    else encode_chunks<true, false>(a, sm);
  } else {
    if (complete) encode_chunks<false, true>(a, sm);
    else encode_chunks<false, false>(a, sm);
  }
}

// ---------------------------------------------------------------------------------- decode
// The decoder takes a set of table blocks and codes with the one whose hash the header names
// (hx_decode: a set of one).
constexpr int kMaxTableSet = HX_MAX_TABLE_SET;
struct DecodeArgs {
  const hx::Tables* set[kMaxTableSet];
  uint32_t nset;
  const uint8_t* st;
  uint64_t bytes;
  uint8_t* out;
  uint64_t n;
  uint32_t* status;
  uint32_t kind;
};

// Header checks shared by every block; returns total_words, or -status, and the table block the
// header's codebook hash picks. A set of one keeps the single-table order of checks: a block of
// the wrong kind is an argument error before the stream is looked at.
__device__ int64_t check_header(const DecodeArgs& a, const hx::Tables** picked) {
  const uint32_t* h32 = reinterpret_cast<const uint32_t*>(a.st);
  const uint64_t* h64 = reinterpret_cast<const uint64_t*>(a.st);
  const uint32_t vk = h32[1];
  if (a.nset == 1 && (a.set[0]->magic != hx::kTablesMagic || a.set[0]->kind != a.kind))
    return -(int64_t)HX_ERR_ARG;
  if (h32[0] != kMagic || (vk & 0xff) != 1 || h32[2] != kChunk || h32[3] != HX_SUBSTREAMS)
    return -(int64_t)HX_ERR_CORRUPT;
  if (((vk >> 8) & 0xff) != a.kind) return -(int64_t)HX_ERR_CODEBOOK;
  *picked = nullptr;
  for (uint32_t i = 0; i < a.nset && i < (uint32_t)kMaxTableSet; ++i) {
    const hx::Tables* t = a.set[i];
    if (t->magic == hx::kTablesMagic && t->kind == a.kind && ((vk >> 16) & 0xff) == t->lmax &&
        h64[5] == t->hash) {
      *picked = t;
      break;
    }
  }
  if (!*picked) return -(int64_t)HX_ERR_CODEBOOK;
  if (h64[2] != a.n || h64[3] != n_chunks_of(a.n)) return -(int64_t)HX_ERR_CORRUPT;
  const uint64_t P = payload_offset(a.n);
  const uint64_t total = h64[4];
  // the host guarantees bytes >= P + 8; the payload and its 2 guard words must fit
  if (total > (a.bytes - P) / 4 - 2 || total >= (1ull << 32)) return -(int64_t)HX_ERR_CORRUPT;
  return (int64_t)total;
}

// A sub-stream's payload words, MSB-first. The two words in use (w0:w1) and an offset bo < 32
// into w0 give the next 32 bits with one funnel shift -- enough for two codes of <= 12 bits, so
// every second symbol costs no extraction. Two further words are already requested (pf0, pf1);
// once bo passes 32 the words move up and one more is requested: one predicated 4-byte load
// per payload word. The word index is 32-bit, so an address is one multiply-add off the payload
// base. CHECKED readers treat words past the caller's buffer as 0; the others never reach them
// (checked once per sub-stream).
template <bool CHECKED>
struct SubstreamBits {
  const uint32_t* words;
  uint32_t wlimit;  // payload words inside the buffer (used when CHECKED)
  uint32_t wi;      // index of the next word to request
  uint32_t w0, w1, pf0, pf1;
  uint32_t bo;

  // a miss brings 256 bytes into L2: the rest of this sub-stream's line and the next one
  __device__ __forceinline__ static uint32_t load(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L2::256B.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
  }
  __device__ __forceinline__ uint32_t word(uint32_t i) const {
    if (CHECKED) return i < wlimit ? load(words + i) : 0u;
    return load(words + i);
  }
  __device__ __forceinline__ void start(uint32_t fw, uint32_t first_bo) {
    w0 = word(fw);
    w1 = word(fw + 1);
    pf0 = word(fw + 2);
    pf1 = word(fw + 3);
    wi = fw + 4;
    bo = first_bo;
  }
  __device__ __forceinline__ uint32_t peek() const { return __funnelshift_l(w1, w0, bo); }
  // after at most 24 more bits: bo < 56, so one word restores bo < 32
  __device__ __forceinline__ void advance(uint32_t nbits) {
    bo += nbits;
    if (bo >= 32) {
      bo -= 32;
      w0 = w1;
      w1 = pf0;
      pf0 = pf1;
      pf1 = word(wi++);
    }
  }
  // index (in payload bits) of the next bit not yet consumed
  __device__ __forceinline__ uint64_t position() const { return 32ull * (wi - 4) + bo; }
};
// Words a reader may request for one sub-stream: 4 at the start, then one per 32 bits of at
// most kSubLen codes of at most 15 bits (the table's length field).
constexpr uint32_t kReaderReach = 4 + (kSubLen * 15 + 31) / 32;

// The same w0:w1 window fed from 16-byte loads: a queue of the next `left` words (q0..q3, 1 to 4
// of them), refilled with one 16-byte block when it runs dry, so a lane requests a block every
// fourth word.
// The decoder uses it for warps whose lanes all read the same bank of their lines (sub-streams a
// multiple of 128 bytes apart advancing in step, as when every code has 8 bits), where it makes
// a quarter of the conflicted load requests. Unchecked only: the caller guarantees that every
// block it may request lies inside the buffer (kReaderReach16).
struct SubstreamBits16 {
  const uint4* blocks;  // the payload as 16-byte blocks (its base is 16-byte aligned)
  uint32_t bi;          // index of the next block to request
  uint32_t w0, w1, q0, q1, q2, q3, left;
  uint32_t bo;

  __device__ __forceinline__ static uint4 load(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
  }
  __device__ __forceinline__ uint32_t pull() {
    const uint32_t v = q0;
    q0 = q1;
    q1 = q2;
    q2 = q3;
    if (--left == 0) {
      const uint4 v = load(blocks + bi++);
      q0 = v.x;
      q1 = v.y;
      q2 = v.z;
      q3 = v.w;
      left = 4;
    }
    return v;
  }
  __device__ __forceinline__ void start(uint32_t fw, uint32_t first_bo) {
    bi = fw >> 2;
    const uint4 v = load(blocks + bi);
    bi += 1;
    q0 = v.x;
    q1 = v.y;
    q2 = v.z;
    q3 = v.w;
    left = 4;
    for (uint32_t r = fw & 3u; r > 0; --r) pull();
    w0 = pull();
    w1 = pull();
    bo = first_bo;
  }
  __device__ __forceinline__ uint32_t peek() const { return __funnelshift_l(w1, w0, bo); }
  __device__ __forceinline__ void advance(uint32_t nbits) {
    bo += nbits;
    if (bo >= 32) {
      bo -= 32;
      w0 = w1;
      w1 = pull();
    }
  }
  // the queue holds words 4 * bi - left .. 4 * bi - 1, so w0 is word 4 * bi - 2 - left
  __device__ __forceinline__ uint64_t position() const {
    return 32ull * (4ull * bi - 2 - left) + bo;
  }
};
// Words the 16-byte reader may request for a sub-stream whose first word is fw, counted from
// 4 * (fw / 4): one block at the start and one per 4 words taken, of at most 3 + 2 + one per 32
// bits of at most kSubLen codes of at most 15 bits.
constexpr uint32_t kReaderPulls16 = 3 + 2 + (31 + kSubLen * 15) / 32;
constexpr uint32_t kReaderReach16 = 4 * (1 + kReaderPulls16 / 4);
// a warp reads with 16-byte blocks when this many of its lanes start in one bank
constexpr uint32_t kCrowdedReaders = 16;

// The decode table in shared memory: for every 12-bit window, (symbol << 8) | hx::kDecValid |
// length of the code word it starts with; 0 when none does (an incomplete code). A warp's 32
// lookups hit random banks, about 3.8 wavefronts per lookup. For QLC and Exp-Golomb codes, whose
// few distinct lengths make the windows of a warp crowd more, the table is held 8 times, copy k
// confined to banks 4k .. 4k + 3 and read by lanes 4k .. 4k + 3, so only 4 lanes can meet in a
// bank (measured: QLC 0.918 -> 0.895 ms per GiB, Exp-Golomb 1.12 -> 0.94 ms; Huffman codes lose
// 2 % to the longer address arithmetic and the L1 the copies take, and keep the one table).
template <int COPIES>
struct DecLut;
template <>
struct DecLut<1> {
  const uint16_t* full;
  __device__ __forceinline__ uint32_t operator()(uint32_t x) const { return full[x >> 20]; }
};
template <>
struct DecLut<8> {
  // entry i of copy k at byte ((i >> 3) << 7) + (k << 4) + ((i & 7) << 1): each 128-byte row holds
  // 8 entries of every copy; `base` is the table's shared address + 16 * (lane / 4)
  uint32_t base;
  __device__ __forceinline__ uint32_t operator()(uint32_t x) const {
    const uint32_t a = base + ((x >> 23) << 7) + ((x >> 19) & 14u);
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
  }
};
// The copies go to the blocks of 1024 threads (large inputs); the smaller blocks of small inputs
// would spend more on filling 64 KB than the lookups gain (1 MiB of QLC: 28.8 -> 32.8 us).
template <int KIND, int THREADS>
__host__ __device__ constexpr int dec_copies() {
  return KIND == HX_KIND_HUFFMAN || THREADS != 1024 ? 1 : 8;
}
// dynamic shared memory of the decoder of a kind at block size index i (the one-table decoder's
// table is static)
constexpr size_t dec_lut_bytes(uint32_t kind, int i) {
  return kind == HX_KIND_HUFFMAN || i != 0 ? 0 : 8 * 4096 * 2;
}

// Two symbols from the reader: table entries (symbol << 8) | kDecValid | length for either kind
// (for a QLC table the length is 3 + the width of the area in the top 3 bits; the table holds it
// already). An entry of 0 (no code word starts the window) only occurs for an incomplete code:
// `valid` is the AND of the entries used, so its kDecValid bit ends up clear if any was 0.
template <bool COMPLETE, class Reader, class Lut>
__device__ __forceinline__ void decode_pair(Reader& rd, uint32_t& valid, const Lut& lut,
                                            uint32_t& e1, uint32_t& e2) {
  const uint32_t x = rd.peek();
  e1 = lut(x);
  const uint32_t l1 = e1 & 15u;
  e2 = lut(x << l1);
  const uint32_t l2 = e2 & 15u;
  if (!COMPLETE) valid &= e1 & e2;
  rd.advance(l1 + l2);
}

// 32 symbols -> 32 output bytes, one 32-byte streaming store (a whole sector) when the output is
// 32-byte aligned, else two 16-byte stores. The symbol bytes are gathered with byte permutes.
template <bool COMPLETE, class Reader, class Lut>
__device__ __forceinline__ void decode_group32(Reader& rd, uint32_t& valid, uint8_t* dst,
                                               bool out32, const Lut& lut) {
  uint32_t o[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t e1, e2, e3, e4;
    decode_pair<COMPLETE>(rd, valid, lut, e1, e2);
    decode_pair<COMPLETE>(rd, valid, lut, e3, e4);
    o[q] = __byte_perm(__byte_perm(e1, e2, 0x0051), __byte_perm(e3, e4, 0x0051), 0x5410);
  }
  if (out32) {
    asm volatile("st.global.cs.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(o[0]),
                 "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                 : "memory");
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    __stcs(d4, make_uint4(o[0], o[1], o[2], o[3]));
    __stcs(d4 + 1, make_uint4(o[4], o[5], o[6], o[7]));
  }
}

// Decodes `mine` symbols of one sub-stream from a started reader to dst; returns the reader's
// final bit position. Sets *invalid when a window started no code word.
template <bool COMPLETE, class Reader, class Lut>
__device__ __forceinline__ uint64_t decode_substream(Reader& rd, uint32_t mine, uint8_t* dst,
                                                     bool out32, bool& invalid,
                                                     const Lut& lut) {
  uint32_t valid = hx::kDecValid;
  const uint32_t groups = mine / 32;
  for (uint32_t g = 0; g < groups; ++g)
    decode_group32<COMPLETE>(rd, valid, dst + 32 * g, out32, lut);
  for (uint32_t i = groups * 32; i < mine; ++i) {
    const uint32_t e = lut(rd.peek());
    if (!COMPLETE) valid &= e;
    rd.advance(e & 15u);
    dst[i] = (uint8_t)(e >> 8);
  }
  invalid = !COMPLETE && (valid & hx::kDecValid) == 0;
  return rd.position();
}

// The block's chunks in a grid-stride loop, 8 lanes per chunk (one per sub-stream). COMPLETE:
// every window starts a code word, so no entry is checked. VOTE: the block's first chunk looked
// crowded (crowded_chunk), so the lanes about to decode vote on the 16-byte reader.
template <int THREADS, bool COMPLETE, bool VOTE, class Lut>
__device__ __forceinline__ void decode_chunks(const DecodeArgs& a, const Lut& lut,
                                              uint32_t total) {
  const int tid = threadIdx.x;
  const uint64_t n = a.n;
  const uint64_t nchunks = n_chunks_of(n);
  const uint64_t P = payload_offset(n);
  const uint32_t* word_off = reinterpret_cast<const uint32_t*>(a.st + 64);
  const uint4* sync = reinterpret_cast<const uint4*>(a.st + sync_offset(n));
  const uint32_t* words = reinterpret_cast<const uint32_t*>(a.st + P);
  // payload words inside the buffer, capped at 2^32 - 1 (no payload word lies beyond 2^32 - 2)
  const uint32_t wlimit = (uint32_t)min((a.bytes - P) / 4, (uint64_t)0xffffffffull);
  const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0;
  const bool blocks16 = (reinterpret_cast<uintptr_t>(words) & 15) == 0;
  const int k = tid & 7;

  for (uint64_t c = (uint64_t)blockIdx.x * (THREADS / 8) + (tid >> 3); c < nchunks;
       c += (uint64_t)gridDim.x * (THREADS / 8)) {
    const uint32_t w0 = __ldg(word_off + c), w1 = __ldg(word_off + c + 1);
    const uint4 sy = __ldg(sync + c);
    auto sync_at = [&](uint32_t i) -> uint32_t {  // u16 entry i of the chunk's sync row
      const uint32_t w = i < 2 ? sy.x : i < 4 ? sy.y : i < 6 ? sy.z : sy.w;
      return (w >> (16 * (i & 1))) & 0xffffu;
    };
    const uint32_t nbits = sy.x & 0xffffu;
    const uint32_t count = n - c * kChunk < kChunk ? (uint32_t)(n - c * kChunk) : kChunk;
    const uint32_t nsub = (count + kSubLen - 1) / kSubLen;
    bool bad = w0 > w1 || w1 > total || nbits > 32u * (w1 - w0) || (nbits + 31) / 32 != w1 - w0;
    const uint32_t mine = (uint32_t)k < nsub ? min(kSubLen, count - k * kSubLen) : 0u;
    if (mine == 0) {
      bad |= k > 0 && sync_at(k) != nbits;
    } else if (!bad) {
      const uint32_t start = k == 0 ? 0u : sync_at(k);
      const uint32_t end = (uint32_t)k + 1 < nsub ? sync_at(k + 1) : nbits;
      const uint64_t first_bit = 32ull * w0 + start;  // w0 <= total < 2^32
      bool invalid = false;
      uint8_t* dst = a.out + c * kChunk + (uint64_t)k * kSubLen;
      uint64_t pos;
      const uint32_t fw = (uint32_t)(first_bit >> 5), fbo = (uint32_t)(first_bit & 31);
      // VOTE: the lanes decoding now vote, and read 16-byte blocks when many of them start on
      // one bank
      bool crowded = false;
      if (VOTE) {
        const uint32_t voters = __activemask();
        crowded = __any_sync(voters,
                             __popc(__match_any_sync(voters, fw & 31u)) >= kCrowdedReaders);
      }
      if (VOTE && crowded && blocks16 &&
                 (uint64_t)(fw & ~3u) + kReaderReach16 <= wlimit) {
        SubstreamBits16 rd;
        rd.blocks = reinterpret_cast<const uint4*>(words);
        rd.start(fw, fbo);
        pos = decode_substream<COMPLETE>(rd, mine, dst, out32, invalid, lut);
      } else if ((uint64_t)fw + kReaderReach <= wlimit) {
        SubstreamBits<false> rd;
        rd.words = words;
        rd.wlimit = wlimit;
        rd.start(fw, fbo);
        pos = decode_substream<COMPLETE>(rd, mine, dst, out32, invalid, lut);
      } else {
        SubstreamBits<true> rd;
        rd.words = words;
        rd.wlimit = wlimit;
        rd.start(fw, fbo);
        pos = decode_substream<COMPLETE>(rd, mine, dst, out32, invalid, lut);
      }
      // the sub-stream must end exactly where the next one starts
      bad |= invalid || pos != 32ull * w0 + end;
    }
    if (bad) atomicOr(a.status, (uint32_t)HX_ERR_CORRUPT);
  }
}

// Whether the sub-streams of chunk c start crowded on one bank of their lines: 4 or more of its
// 8 first words equal modulo 32 (any flat code length does it: a sub-stream of 512 codes of L
// bits is 16 L words long; codes of mixed lengths do it by chance for about 1 chunk in 500).
// Read by one thread after the header checks.
__device__ bool crowded_chunk(const DecodeArgs& a, uint64_t c) {
  if (c >= n_chunks_of(a.n)) return false;
  const uint32_t w0 = reinterpret_cast<const uint32_t*>(a.st + 64)[c];
  const uint16_t* row = reinterpret_cast<const uint16_t*>(a.st + sync_offset(a.n)) + 8 * c;
  uint32_t bank[HX_SUBSTREAMS];
  for (int k = 0; k < HX_SUBSTREAMS; ++k)
    bank[k] = (w0 + ((k == 0 ? 0u : (uint32_t)row[k]) >> 5)) & 31u;
  for (int k = 0; k < HX_SUBSTREAMS; ++k) {
    int same = 0;
    for (int q = 0; q < HX_SUBSTREAMS; ++q) same += bank[q] == bank[k];
    if (same >= 4) return true;
  }
  return false;
}

// KIND is checked against the stream header and the tables; the symbol loop is the same. THREADS:
// one block of 1024 per SM for large inputs, with one copy of the table, the rest of the on-chip
// memory serving as L1 for the payload words; smaller blocks spread smaller inputs over more SMs
// (decode_common picks).
template <int KIND, int THREADS>
__global__ void __launch_bounds__(THREADS, 1024 / THREADS) k_decode(DecodeArgs a) {
  constexpr int kCopies = dec_copies<KIND, THREADS>();
  __shared__ __align__(16) uint16_t s_lut[kCopies == 1 ? 4096 : 8];
  extern __shared__ __align__(16) uint16_t s_lut_copies[];  // dec_lut_bytes(KIND, .) bytes
  __shared__ int64_t s_total;
  __shared__ const hx::Tables* s_tables;
  __shared__ bool s_crowded;
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_total = check_header(a, &s_tables);
    // the block's first chunk stands for the rest: a block whose chunks look crowded takes the
    // voting loop (the word-by-word loop alone runs faster elsewhere)
    s_crowded = s_total >= 0 && crowded_chunk(a, (uint64_t)blockIdx.x * (THREADS / 8));
  }
  __syncthreads();
  const int64_t total = s_total;
  if (total < 0) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, (uint32_t)(-total));
    return;
  }
  const hx::Tables* tables = s_tables;
  DecLut<kCopies> lut;
  if constexpr (kCopies == 1) {
    const uint4* src = reinterpret_cast<const uint4*>(tables->dec);
    uint4* dst = reinterpret_cast<uint4*>(s_lut);
    for (int i = tid; i < 4096 * 2 / 16; i += THREADS) dst[i] = src[i];
    lut.full = s_lut;
  } else {
    // entries 8r .. 8r + 7 fill bytes 16k .. 16k + 15 of row r in every copy k: one 16-byte load,
    // eight 16-byte stores
    const uint4* src = reinterpret_cast<const uint4*>(tables->dec);
    uint4* dst = reinterpret_cast<uint4*>(s_lut_copies);
    for (int r = tid; r < 4096 / 8; r += THREADS) {
      const uint4 v = src[r];
#pragma unroll
      for (int k = 0; k < 8; ++k) dst[8 * r + k] = v;
    }
    lut.base = (uint32_t)__cvta_generic_to_shared(s_lut_copies) + 16u * ((tid & 31) >> 2);
  }
  __syncthreads();
  const bool crowded = s_crowded;
  if (tables->complete) {
    if (crowded) decode_chunks<THREADS, true, true>(a, lut, (uint32_t)total);
    else decode_chunks<THREADS, true, false>(a, lut, (uint32_t)total);
  } else {
    if (crowded) decode_chunks<THREADS, false, true>(a, lut, (uint32_t)total);
    else decode_chunks<THREADS, false, false>(a, lut, (uint32_t)total);
  }
}

// ---------------------------------------------------------------------------------- shannonic
// The review page's range-partitioned coder: a byte's range index is coded by tANS with 128
// states (the table variant of asymmetric numeral systems), its offset inside the range in
// ceil(log2 size) bits. tANS runs from a sub-stream's last symbol to its first, so its bit count
// is known only after the whole sub-stream has been run: the encoder (k_sh_encode) parks each
// sub-stream's bits in shared memory until the offsets before it are known. The decoder,
// k_sh_decode, reads each sub-stream backwards.

constexpr int kShCopies = 16;  // symbol table copies: lane l reads copy l % 16 (<= 2-way)

// Encoder tables in shared memory: per byte value [byte][copy] one 8-byte entry, the step's
// fields (sh_sym) and the byte's offset in its range (sh_off), read with one load; the ranges'
// states (sh_enc). A row of 16 copies is 128 bytes, so lanes l and l + 16 share banks and a warp's
// lookup takes the 2 wavefronts its 256 bytes need.
struct ShEnc {
  uint2 ent[256 * kShCopies];
  uint8_t enc[128];
};

__device__ __forceinline__ void sh_load_tables(const hx::Tables* t, ShEnc& s) {
  for (int i = threadIdx.x; i < 256 * kShCopies; i += blockDim.x)
    s.ent[i] = make_uint2(t->sh_sym[i / kShCopies], t->sh_off[i / kShCopies]);
  for (int i = threadIdx.x; i < 128; i += blockDim.x) s.enc[i] = t->sh_enc[i];
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

// Shared addresses of the encoder tables for this lane: its copy of byte b's entry is at
// sym + 8 * kShCopies * b; `enc` is sh_enc's address - 128.
struct ShLane {
  uint32_t sym, enc;
};
__device__ __forceinline__ ShLane sh_lane(const ShEnc& s, uint32_t lane) {
  return {(uint32_t)__cvta_generic_to_shared(s.ent) + 8 * (lane % kShCopies),
          (uint32_t)__cvta_generic_to_shared(s.enc) - 128u};
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

// One tANS step from state x (in [128, 256)) with the byte's entry e: returns the bit count
// len = nb + ob it writes and moves x to the next state. The entry's key makes (x + key) >> 8 =
// len; x >> nb is (x << ob) >> len, and the ob in e's low bits is all a wrapping shift reads.
__device__ __forceinline__ uint32_t sh_next(uint32_t e, uint32_t& x, uint32_t enc, uint32_t& xo,
                                            uint32_t& hi) {
  const uint32_t len = (x * (1u << 20) + e) >> 28;
  xo = __funnelshift_l(0u, x, e);  // x << ob
  hi = xo >> len;                  // x >> nb, in [f, 2f)
  x = lds_u8(enc + __byte_perm(e, 0u, 0x4441) + hi);  // sh_enc[cum - f + hi]
  return len;
}

// The bits a step writes, (offset << nb) | (x mod 2^nb), from its entry e, the byte's offset,
// x << ob (xo), x >> nb (hi) and len: ((offset - hi) << len) + xo is the same value times 2^ob.
__device__ __forceinline__ uint32_t sh_value(uint32_t e, uint32_t off, uint32_t xo, uint32_t hi,
                                             uint32_t len) {
  return __funnelshift_r((((off - hi) << len) + xo), 0u, e);
}

// Symbols in sub-stream k of chunk c (0 past the end of the input).
__device__ __forceinline__ uint32_t sh_count(uint64_t n, uint32_t c, uint32_t k) {
  const uint64_t first = (uint64_t)c * kChunk + (uint64_t)k * kSubLen;
  return first < n ? (uint32_t)min((uint64_t)kSubLen, n - first) : 0u;
}

__device__ __forceinline__ void reds_add_u32(uint32_t a, uint32_t x) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(a), "r"(x) : "memory");
}

// Predicated stores (no branch around them).
__device__ __forceinline__ void st_global_if(bool p, uint32_t* a, uint32_t v) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %2, 0;\n @q st.global.u32 [%0], %1;\n}"
               ::"l"(a), "r"(v), "r"((uint32_t)p) : "memory");
}
__device__ __forceinline__ void st_global_v4_if(bool p, uint32_t* a, uint4 v) {
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.u32 q, %5, 0;\n @q st.global.v4.u32 [%0], {%1, %2, %3, %4};\n}"
      ::"l"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"((uint32_t)p) : "memory");
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_if(bool p, uint32_t a, uint32_t v) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %2, 0;\n @q st.shared.u32 [%0], %1;\n}"
               ::"r"(a), "r"(v), "r"((uint32_t)p) : "memory");
}

// Runs tANS over sub-stream k of chunk c (m symbols, from the last to the first) and hands its
// bits to put(value, len): two codes joined per call (at most 30 bits), the final state last.
// With HIST every byte is also counted at hist + 4 * byte (shared memory).
template <bool HIST, class Put>
__device__ __forceinline__ void sh_run(const EncodeArgs& a, const ShLane& tl, uint32_t c,
                                       uint32_t k, uint32_t m, uint32_t hist, Put&& put) {
  uint32_t state = 128;
  // the bits of byte `sym` (as sh_value) and their count
  auto code = [&](uint32_t sym, uint32_t& len) -> uint32_t {
    if (HIST) reds_add_u32(hist + 4u * sym, 1u);
    const uint2 eo = lds_v2(tl.sym + sym * (8 * kShCopies));
    uint32_t xo, xh;
    len = sh_next(eo.x, state, tl.enc, xo, xh);
    return sh_value(eo.x, eo.y, xo, xh, len);
  };
  if (m == kSubLen) {
    // a whole sub-stream: 16 bytes at a time from the end, the next 16 already requested
    const uint4* src =
        reinterpret_cast<const uint4*>(a.in + (uint64_t)c * kChunk + (uint64_t)k * kSubLen);
    uint4 nxt = __ldg(src + kSubLen / 16 - 1);
#pragma unroll 1
    for (int g = kSubLen / 16 - 1; g >= 0; --g) {
      const uint4 v = nxt;
      if (g > 0) nxt = __ldg(src + g - 1);
      const uint32_t w[4] = {v.w, v.z, v.y, v.x};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int h = 3; h > 0; h -= 2) {
          uint32_t l0, l1;
          const uint32_t v0 = code(__byte_perm(w[q], 0u, 0x4440 + h), l0);
          const uint32_t v1 = code(__byte_perm(w[q], 0u, 0x4440 + h - 1), l1);
          put((v0 << l1) | v1, l0 + l1);
        }
      }
    }
  } else if (m) {
    const uint64_t first = (uint64_t)c * kChunk + (uint64_t)k * kSubLen;
    for (uint32_t i = m; i-- > 0;) {
      uint32_t l;
      const uint32_t v = code((uint32_t)a.in[first + i], l);
      put(v, l);
    }
  }
  if (m) put(state - 128u, HX_SHN_R);
}

// Sub-stream k of chunk c (m > 0 symbols) coded again, straight into the payload: its bits start
// at bit s of the chunk, whose first word is woff; `last` when it ends the chunk. Finished words
// leave in aligned groups of 4 (one 16-byte store; q0..q2 hold the three words before the
// current one), those before the sub-stream's first whole group one by one, the stores predicated
// rather than branched around. The first word's earlier bits are stored as zeros; the last,
// unfinished word is stored whole when it ends the chunk, else returned in `tail` at `widx` for
// the caller to OR in once the sub-stream after it has stored that word.
__device__ __noinline__ void sh_write_direct(const EncodeArgs& a, const ShLane& tl, uint32_t c,
                                             uint32_t k, uint32_t m, uint32_t* payload,
                                             uint32_t woff, uint32_t s, bool last,
                                             uint32_t& widx, uint32_t& tail) {
  widx = woff + (s >> 5);
  uint32_t nacc = s & 31, hi = 0, lo = 0;
  const uint32_t gfirst = (widx + 3) & ~3u;
  uint32_t q0 = 0, q1 = 0, q2 = 0;
  sh_run<false>(a, tl, c, k, m, 0u, [&](uint32_t value, uint32_t len) {
    hi = __funnelshift_l(lo, hi, len);
    lo = (lo << len) | value;
    nacc += len;
    const bool full = nacc >= 32;
    nacc -= full ? 32u : 0u;
    const uint32_t w = __funnelshift_r(lo, hi, nacc);
    st_global_if(full && widx < gfirst, payload + widx, w);
    st_global_v4_if(full && widx >= gfirst && (widx & 3) == 3, payload + widx - 3,
                    make_uint4(q0, q1, q2, w));
    q0 = full ? q1 : q0;
    q1 = full ? q2 : q1;
    q2 = full ? w : q2;
    widx += full ? 1u : 0u;
  });
  // the finished words of the last, incomplete group
  const uint32_t g = max(gfirst, widx & ~3u);
  if (widx >= g + 1) payload[widx - 1] = q2;
  if (widx >= g + 2) payload[widx - 2] = q1;
  if (widx >= g + 3) payload[widx - 3] = q0;
  tail = nacc ? lo << (32 - nacc) : 0u;
  if (last && nacc) payload[widx] = tail;
}

// The one-pass encoder of kind 2. A warp takes the next group of 4 chunks from a counter, one
// sub-stream per lane, runs tANS over it and parks its bits in its own region of shared memory
// (a zero word, then up to kShPark words from bit 0), counting the fused histogram. From the bit
// counts it writes the sync rows and publishes the group's word count; it learns the group's word
// offset from the groups before it (the decoupled look-back of k_encode, over groups) and copies
// each chunk out, sub-stream by sub-stream, each lane shifting two consecutive payload words
// together from the parked words (the word before its pair from the lane before it). A word
// shared by two sub-streams is carried from one to the next and stored once. When any
// sub-stream of the group codes to more than kShPark words, its lane's writes have run into the
// regions after it (the last lane's into a guard area sized for the longest sub-stream), so every
// lane of the group codes its sub-stream again straight into the payload.

// warps per block (one block per SM): as many as the shared memory holds, with and without the
// fused histogram's tables
template <bool HIST>
__host__ __device__ constexpr int sh_enc_warps() { return HIST ? 12 : 13; }
constexpr uint32_t kShPark = 112;              // words: 7 bits per symbol
constexpr uint32_t kShStride = kShPark + 1;    // odd: the 32 regions start in 32 different banks
constexpr uint32_t kShSubMaxWords = (kSubLen * 15 + HX_SHN_R + 31) / 32;  // 241
constexpr uint32_t kShParkWords = 31 * kShStride + 1 + kShSubMaxWords;

template <bool HIST>
struct ShEncodeSmem {
  static constexpr int kWarps = sh_enc_warps<HIST>();
  ShEnc t;
  uint32_t hist[HIST ? kWarps : 1][256];
  alignas(16) uint32_t park[kWarps][kShParkWords];
};
static_assert(sizeof(ShEncodeSmem<true>) <= 227 * 1024, "one block per SM");
static_assert(sizeof(ShEncodeSmem<false>) <= 227 * 1024, "one block per SM");

template <bool HIST>
__device__ void sh_encode_groups(const EncodeArgs& a, ShEncodeSmem<HIST>& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint64_t n = a.n;
  const uint32_t nchunks = (uint32_t)n_chunks_of(n), ngroups = (nchunks + 3) / 4;
  const uint32_t full_chunks = (uint32_t)(n / kChunk);
  const uint64_t P = payload_offset(n);
  uint32_t* word_off = reinterpret_cast<uint32_t*>(a.out + 64);
  uint16_t* sync = reinterpret_cast<uint16_t*>(a.out + sync_offset(n));
  uint32_t* payload = reinterpret_cast<uint32_t*>(a.out + P);
  // payload words that fit before the 2 guard words at the end of the caller's buffer
  const uint64_t room = a.cap >= P + 8 ? (a.cap - P - 8) / 4 : 0;
  const ShLane tl = sh_lane(sm.t, lane);
  const uint32_t park = (uint32_t)__cvta_generic_to_shared(sm.park[warp]);
  const uint32_t hist = (uint32_t)__cvta_generic_to_shared(sm.hist[warp]);
  const uint32_t j = lane >> 3, k = lane & 7;
  const uint32_t region = park + 4u * kShStride * lane;
  for (;;) {
    uint32_t g = 0;
    if (lane == 0) g = atomicAdd(a.counter, 1u);
    g = __shfl_sync(0xffffffffu, g, 0);
    if (g >= ngroups) break;
    // the group this warp will most likely take next, into L2
    const uint64_t ahead = (uint64_t)g + gridDim.x * ShEncodeSmem<HIST>::kWarps;
    if (lane == 0 && 4 * ahead + 4 <= full_chunks)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.in + ahead * 4 * kChunk),
                   "r"(4 * kChunk)
                   : "memory");
    const uint32_t c = 4 * g + j;
    const uint32_t m = c < nchunks ? sh_count(n, c, k) : 0u;
    // tANS into the lane's region. pos counts the bits from the start of the zero word (32 +
    // the sub-stream's bits); hi:lo holds the last 64 of them, so the last finished word,
    // (pos >> 5) - 1, is hi:lo >> (pos mod 32) (a wrapping shift reads only pos's low 5 bits):
    // every append stores it, again and again until the next one is finished, with no
    // condition.
    uint32_t pos = 32, hi = 0, lo = 0;
    sh_run<HIST>(a, tl, c, k, m, hist, [&](uint32_t value, uint32_t len) {
      hi = __funnelshift_l(lo, hi, len);
      lo = (lo << len) | value;
      pos += len;
      sts_u32(region + ((pos >> 3) & ~3u) - 4u, __funnelshift_r(lo, hi, pos));
    });
    const uint32_t part = pos & 31u;  // the unfinished word's bits
    sts_if(part != 0, region + ((pos >> 3) & ~3u), part ? lo << (32 - part) : 0u);
    sts_u32(region, 0u);
    const uint32_t bits = pos - 32u;
    const bool spill = __any_sync(0xffffffffu, bits > 32u * kShPark);
    // the chunk's sync row: its bit count, then where sub-streams 1..7 start
    uint32_t incl = bits;
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, d, 8);
      if (k >= (uint32_t)d) incl += t;
    }
    const uint32_t s = incl - bits;
    const uint32_t cbits = __shfl_sync(0xffffffffu, incl, 7, 8);
    if (c < nchunks) sync[(uint64_t)c * HX_SUBSTREAMS + k] = (uint16_t)(k == 0 ? cbits : s);
    // the group's word count, published before the wait; each chunk's offset inside the group
    const uint32_t cw = (cbits + 31) >> 5;
    const uint32_t w0 = __shfl_sync(0xffffffffu, cw, 0), w1 = __shfl_sync(0xffffffffu, cw, 8);
    const uint32_t w2 = __shfl_sync(0xffffffffu, cw, 16), w3 = __shfl_sync(0xffffffffu, cw, 24);
    const uint32_t gw = w0 + w1 + w2 + w3;
    const uint32_t before = (j > 0 ? w0 : 0u) + (j > 1 ? w1 : 0u) + (j > 2 ? w2 : 0u);
    if (lane == 0 && g != a.withhold)
      st_relaxed_u64(a.look + g, (g == 0 ? kLookPre : kLookAgg) | gw);
    __syncwarp();
    uint64_t goff;
    const bool ok = chunk_offset(a, g, gw, lane, goff);
    // offsets are below 2^32 words (a stream holds fewer)
    const uint32_t coff = (uint32_t)goff + before;
    const bool fits = ok && (uint64_t)coff + cw <= room;
    if (ok && c < nchunks && k == 0) {
      word_off[c] = coff;
      if (c + 1 == nchunks) {
        reinterpret_cast<uint64_t*>(a.out)[4] = (uint64_t)coff + cw;
        word_off[nchunks] = coff + cw;
        if (fits) payload[coff + cw] = payload[coff + cw + 1] = 0;
      }
      if (!fits) atomicOr(a.status, (uint32_t)HX_ERR_CAPACITY);
    }
    if (!spill) {
      // chunk by chunk, sub-stream by sub-stream: the lanes take 32 consecutive output words
#pragma unroll 1
      for (uint32_t jj = 0; jj < 4; ++jj) {
        const uint32_t cc = 4 * g + jj;
        if (cc >= nchunks || !__shfl_sync(0xffffffffu, fits, 8 * jj)) continue;
        const uint32_t base = __shfl_sync(0xffffffffu, coff, 8 * jj);
        const uint32_t ctot = __shfl_sync(0xffffffffu, cbits, 8 * jj);
        uint32_t carry = 0;  // the unfinished word of the sub-stream before (its bits on top)
#pragma unroll 1
        for (uint32_t q = 0; q < HX_SUBSTREAMS; ++q) {
          const uint32_t src = 8 * jj + q;
          const uint32_t sq = __shfl_sync(0xffffffffu, s, src);
          const uint32_t bq = __shfl_sync(0xffffffffu, bits, src);
          if (bq == 0) continue;  // an empty sub-stream at the end of the input
          const uint32_t sh = sq & 31, e = sq + bq;
          const uint32_t nin = (bq + 31) >> 5, nout = ((e + 31) >> 5) - (sq >> 5);
          // its last word is finished by a later sub-stream: carried, not stored
          const bool open = (e & 31) != 0 && e < ctot;
          const uint32_t lim = nout - (open ? 1u : 0u);
          const uint32_t rq = park + 4u * kShStride * src + 4u;  // its word 0
          const uint32_t w0 = base + (sq >> 5);                   // the payload word of output 0
          // output word i = parked words i - 1 : i >> sh; before word 0 stand the carried bits
          uint32_t before = sh ? carry >> (32 - sh) : 0u;
          uint32_t wa = 0, wb = 0;
          for (uint32_t i0 = 0; i0 < nout; i0 += 64) {
            const uint32_t i = i0 + 2 * lane;
            const uint32_t ca = i < nin ? lds_u32(rq + 4u * i) : 0u;
            const uint32_t cb = i + 1 < nin ? lds_u32(rq + 4u * i + 4u) : 0u;
            uint32_t pa = __shfl_up_sync(0xffffffffu, cb, 1);
            if (lane == 0) pa = before;
            before = __shfl_sync(0xffffffffu, cb, 31);
            wa = __funnelshift_r(ca, pa, sh);
            wb = __funnelshift_r(cb, ca, sh);
            if (i < lim) payload[w0 + i] = wa;
            if (i + 1 < lim) payload[w0 + i + 1] = wb;
          }
          const uint32_t t = (nout - 1) & 63;  // the last word's place in the last round
          carry = open ? __shfl_sync(0xffffffffu, (t & 1) ? wb : wa, t >> 1) : 0u;
        }
      }
    } else {
      // a sub-stream outgrew its region: code the group again, straight into the payload
      const bool mine = fits && c < nchunks && m != 0;
      const bool last = m != 0 && s + bits == cbits;
      uint32_t widx = 0, tail = 0;
      if (mine) sh_write_direct(a, tl, c, k, m, payload, coff, s, last, widx, tail);
      __syncwarp();
      if (mine && !last && tail) atomicOr(payload + widx, tail);
    }
    __syncwarp();
  }
}

template <bool HIST>
__global__ void __launch_bounds__(32 * sh_enc_warps<HIST>(), 1) k_sh_encode(EncodeArgs a) {
  constexpr int kWarps = sh_enc_warps<HIST>(), kThreads = 32 * kWarps;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ShEncodeSmem<HIST>& sm = *reinterpret_cast<ShEncodeSmem<HIST>*>(smem_raw);
  const int tid = threadIdx.x;
  if (a.tables->magic != hx::kTablesMagic || a.tables->kind != a.kind) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, (uint32_t)HX_ERR_ARG);
    return;
  }
  sh_load_tables(a.tables, sm.t);
  if (HIST)
    for (int i = tid; i < kWarps * 256; i += kThreads) (&sm.hist[0][0])[i] = 0;
  if (blockIdx.x == 0 && tid == 0) {
    write_header(a);
    if (a.n == 0) {  // no group writes the totals
      reinterpret_cast<uint64_t*>(a.out)[4] = 0;
      reinterpret_cast<uint32_t*>(a.out + 64)[0] = 0;
      if (a.cap >= payload_offset(0) + 8) {
        uint32_t* payload = reinterpret_cast<uint32_t*>(a.out + payload_offset(0));
        payload[0] = payload[1] = 0;
      }
    }
  }
  __syncthreads();
  sh_encode_groups<HIST>(a, sm);
  if (HIST) {
    __syncthreads();
    for (int sym = tid; sym < 256; sym += kThreads) {
      uint32_t sum = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sum += sm.hist[HIST ? w : 0][sym];
      if (sum) atomicAdd(&a.hist[sym], sum);
    }
  }
}

// Reads a sub-stream backwards: the unread bits end at bit 32 * j + 32 - u of the payload (the
// last u, 0..31, bits of word j are read, MSB first); cur = word j, prv = word j - 1. The words below come
// in aligned 16-byte blocks: r is block rb, the one that holds the next word to come in, and the
// block below it is already requested (nx), so a block is moved only once it has had a whole
// block's worth of symbols to arrive. Words outside the caller's buffer read as 0.
// (j is signed: a reader that runs off the front of the payload must not wrap around; a payload
// holds fewer than 2^31 words, since n < 2^32 bytes at no more than 15 bits each.)
struct BackBits {
  const uint32_t* words;  // 16-byte aligned
  uint32_t wlimit;
  int32_t j, rb;
  uint32_t u, cur, prv;
  uint4 r, nx;
  __device__ __forceinline__ uint32_t word(int32_t i) const {
    return (uint32_t)i < wlimit ? __ldg(words + (uint32_t)i) : 0u;
  }
  __device__ __forceinline__ uint4 block(int32_t b) const {
    if (b >= 0 && 4u * (uint32_t)b + 4u <= wlimit)
      return __ldg(reinterpret_cast<const uint4*>(words) + b);
    return make_uint4(word(4 * b), word(4 * b + 1), word(4 * b + 2), word(4 * b + 3));
  }
  __device__ __forceinline__ void start(uint64_t end_bit) {
    const uint64_t last = end_bit - 1;  // the first bit to read (backwards)
    j = (int32_t)(last >> 5);
    u = 31u - (uint32_t)(last & 31);
    cur = word(j);
    prv = word(j - 1);
    rb = (j - 2) >> 2;  // floor: the block of word j - 2
    r = block(rb);
    nx = block(rb - 1);
  }
  // the 32 bits before the read position, the last of them in bit 0 (bits before the payload's
  // first word read as 0)
  __device__ __forceinline__ uint32_t peek() const { return __funnelshift_r(cur, prv, u); }
  __device__ __forceinline__ void advance() {
    --j;
    cur = prv;
    const int32_t i = j - 1;  // the word that comes in
    if ((i >> 2) != rb) {
      --rb;
      r = nx;
      nx = block(rb - 1);
    }
    const uint32_t lo = (i & 1) ? r.y : r.x, hi = (i & 1) ? r.w : r.z;
    prv = (i & 2) ? hi : lo;
  }
  // moves the read position back by len (<= 31) bits
  __device__ __forceinline__ void skip(uint32_t len) {
    u += len;
    if (u >= 32) {
      u -= 32;
      advance();
    }
  }
  // the `len` (<= 15) bits before the read position, MSB first
  __device__ __forceinline__ uint32_t read(uint32_t len) {
    const uint32_t v = peek() & ((1u << len) - 1u);
    skip(len);
    return v;
  }
  __device__ __forceinline__ int64_t position() const { return 32ll * j + 32 - u; }
};


__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}

// Decoding states in shared memory, [state][copy] with 16-byte entries: lane l reads copy l % 8,
// so the 8 lanes of each quarter of a warp read 8 different bank groups (no conflicts).
constexpr int kShDecCopies = 8;

// 5 resident blocks (48 registers): 6 would spill the reader's blocks
__global__ void __launch_bounds__(kDecThreads, 5) k_sh_decode(DecodeArgs a) {
  __shared__ __align__(16) uint4 s_dec[128 * kShDecCopies];
  __shared__ int64_t s_total;
  __shared__ const hx::Tables* s_tables;
  const int tid = threadIdx.x;
  if (tid == 0) s_total = check_header(a, &s_tables);
  __syncthreads();
  const int64_t total = s_total;
  if (total < 0) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, (uint32_t)(-total));
    return;
  }
  for (int i = tid; i < 128 * kShDecCopies; i += kDecThreads) {
    const uint32_t* d = s_tables->sh_dec[i / kShDecCopies];
    s_dec[i] = make_uint4(d[0], d[1], d[2], d[3]);
  }
  __syncthreads();
  // the entry of state x (in [128, 256)) is at tab + 16 * kShDecCopies * x
  const uint32_t tab = (uint32_t)__cvta_generic_to_shared(s_dec) + 16u * (tid % kShDecCopies) -
                       128u * 16u * kShDecCopies;
  const uint64_t n = a.n;
  const uint64_t nchunks = n_chunks_of(n);
  const uint64_t P = payload_offset(n);
  const uint32_t* word_off = reinterpret_cast<const uint32_t*>(a.st + 64);
  const uint4* sync = reinterpret_cast<const uint4*>(a.st + sync_offset(n));
  BackBits rd;
  rd.words = reinterpret_cast<const uint32_t*>(a.st + P);
  rd.wlimit = (uint32_t)min((a.bytes - P) / 4, (uint64_t)0xffffffffull);
  const uint32_t k = tid & 7;
  for (uint64_t c = (uint64_t)blockIdx.x * (kDecThreads / 8) + (tid >> 3); c < nchunks;
       c += (uint64_t)gridDim.x * (kDecThreads / 8)) {
    const uint32_t w0 = __ldg(word_off + c), w1 = __ldg(word_off + c + 1);
    const uint4 sy = __ldg(sync + c);
    auto sync_at = [&](uint32_t i) -> uint32_t {
      const uint32_t w = i < 2 ? sy.x : i < 4 ? sy.y : i < 6 ? sy.z : sy.w;
      return (w >> (16 * (i & 1))) & 0xffffu;
    };
    const uint32_t nbits = sy.x & 0xffffu;
    const uint32_t count = n - c * kChunk < kChunk ? (uint32_t)(n - c * kChunk) : kChunk;
    const uint32_t nsub = (count + kSubLen - 1) / kSubLen;
    bool bad = w0 > w1 || w1 > (uint32_t)total || nbits > 32u * (w1 - w0) ||
               (nbits + 31) / 32 != w1 - w0;
    const uint32_t mine = k < nsub ? min(kSubLen, count - k * kSubLen) : 0u;
    if (mine == 0) {
      bad |= k > 0 && sync_at(k) != nbits;
    } else if (!bad) {
      const uint32_t start = k == 0 ? 0u : sync_at(k);
      const uint32_t end = k + 1 < nsub ? sync_at(k + 1) : nbits;
      bad |= start >= end || end > nbits;
      if (!bad) {
        rd.start(32ull * w0 + end);
        uint32_t state = 128u + rd.read(HX_SHN_R);
        uint32_t over = 0;  // bit 31 set once an offset was not inside its range
        uint8_t* dst = a.out + c * kChunk + (uint64_t)k * kSubLen;
        // One symbol from x, the bits before the read position (the last in bit 0): the
        // state's low nb bits, before them the offset. Returns the byte (in the low 8 bits),
        // moves the state, and drops the symbol's bits from x, counting them in `used`.
        auto one = [&](uint32_t& x, uint32_t& used) -> uint32_t {
          const uint4 d = lds_v4(tab + 16u * kShDecCopies * state);
          const uint32_t v = x & d.x;       // offset and state bits
          x = __funnelshift_r(x, 0u, d.y);  // x >> (nb + ob)
          used += d.y;
          // the shifts by nb read d.z's low 5 bits
          const uint32_t off = __funnelshift_r(v, 0u, d.z);                  // v >> nb
          state = (d.z >> 16) + v - __funnelshift_l(0u, off, d.z);          // base + v mod 2^nb
          const uint32_t r = off * 0x10001u + d.w;
          over |= r;
          return r;
        };
        const uint32_t groups = mine / 16;
        for (uint32_t g = 0; g < groups; ++g) {
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t pair[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // two symbols take at most 30 of the 32 bits looked at
              uint32_t x = rd.peek(), used = 0;
              const uint32_t b0 = one(x, used);
              const uint32_t b1 = one(x, used);
              rd.skip(used);
              pair[h] = __byte_perm(b0, b1, 0x0040);
            }
            o[q] = __byte_perm(pair[0], pair[1], 0x5410);
          }
          __stcs(reinterpret_cast<uint4*>(dst + 16 * g), make_uint4(o[0], o[1], o[2], o[3]));
        }
        for (uint32_t i = groups * 16; i < mine; ++i) {
          uint32_t x = rd.peek(), used = 0;
          dst[i] = (uint8_t)one(x, used);
          rd.skip(used);
        }
        // the chain must end in state 128 exactly at the sub-stream's first bit
        bad |= (over >> 31) || state != 128u ||
               rd.position() != (int64_t)(32ull * w0 + start);
      }
    }
    if (bad) atomicOr(a.status, (uint32_t)HX_ERR_CORRUPT);
  }
}

// ---------------------------------------------------------------------------------- launch
// The prefix-code decoder's block sizes, and the kernel of a kind at size index i.
constexpr int kDecodeBlock[3] = {1024, 256, 64};
using DecodeKernel = void (*)(DecodeArgs);
template <int KIND>
DecodeKernel prefix_decoder_of(int i) {
  return i == 0 ? k_decode<KIND, 1024> : i == 1 ? k_decode<KIND, 256> : k_decode<KIND, 64>;
}
DecodeKernel prefix_decoder(uint32_t kind, int i) {
  return kind == HX_KIND_HUFFMAN ? prefix_decoder_of<HX_KIND_HUFFMAN>(i)
         : kind == HX_KIND_QLC   ? prefix_decoder_of<HX_KIND_QLC>(i)
                                 : prefix_decoder_of<HX_KIND_EXPGOLOMB>(i);
}

struct DeviceInfo {
  int sms = 0;
  int hist_per_sm = 0;
  int sh_encode_per_sm[2] = {0, 0};  // without, with the fused histogram
  int sh_decode_per_sm = 0;
  // prefix-code decode blocks per SM at 1024, 256, 64 threads: [0] Huffman, [1] QLC and
  // Exp-Golomb (whose 1024-thread blocks hold the 8 bank-confined table copies)
  int dec_per_sm[2][3] = {{0, 0, 0}, {0, 0, 0}};
  int enc_per_sm = 0;
};

// Sets the shared-memory carveout of `fn` to the smallest share that still holds `per_sm` blocks,
// the rest going to L1; keeps the default if that would lower the occupancy.
bool prefer_l1(int dev, const void* fn, int per_sm, int threads, size_t dyn_smem) {
  cudaFuncAttributes fa;
  int max_smem = 0;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess ||
      cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
          cudaSuccess ||
      max_smem <= 0)
    return false;
  // + the per-block reserve
  const long need = (long)per_sm * (long)(fa.sharedSizeBytes + dyn_smem + 1024);
  const int pct = (int)std::min<long>(100, (need * 100 + max_smem - 1) / max_smem + 1);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, pct) != cudaSuccess)
    return false;
  int now = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&now, fn, threads, dyn_smem) != cudaSuccess)
    return false;
  if (now < per_sm)
    return cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutDefault) == cudaSuccess;
  return true;
}

std::mutex g_info_mutex;
DeviceInfo g_info[64];

bool device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(g_info_mutex);
  DeviceInfo& d = g_info[dev];
  if (d.sms == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    for (uint32_t kind : {HX_KIND_HUFFMAN, HX_KIND_QLC, HX_KIND_EXPGOLOMB})
      for (int i = 0; i < 3; ++i)
        if (dec_lut_bytes(kind, i) &&
            cudaFuncSetAttribute(reinterpret_cast<const void*>(prefix_decoder(kind, i)),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dec_lut_bytes(kind, i)) != cudaSuccess)
          return false;
    for (int l = 0; l < 2; ++l) {
      const uint32_t kind = l == 0 ? HX_KIND_HUFFMAN : HX_KIND_QLC;
      for (int i = 0; i < 3; ++i)
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &d.dec_per_sm[l][i], reinterpret_cast<const void*>(prefix_decoder(kind, i)),
                kDecodeBlock[i], dec_lut_bytes(kind, i)) != cudaSuccess ||
            d.dec_per_sm[l][i] < 1)
          return false;
    }
    if (
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.hist_per_sm, k_histogram, kHistThreads,
                                                      0) != cudaSuccess ||
        cudaFuncSetAttribute(k_sh_encode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(ShEncodeSmem<false>)) != cudaSuccess ||
        cudaFuncSetAttribute(k_sh_encode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(ShEncodeSmem<true>)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &d.sh_encode_per_sm[0], k_sh_encode<false>, 32 * sh_enc_warps<false>(),
            sizeof(ShEncodeSmem<false>)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &d.sh_encode_per_sm[1], k_sh_encode<true>, 32 * sh_enc_warps<true>(),
            sizeof(ShEncodeSmem<true>)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.sh_decode_per_sm, k_sh_decode,
                                                      kDecThreads, 0) != cudaSuccess)
      return false;
    if (cudaFuncSetAttribute(k_encode, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(EncSmem)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.enc_per_sm, k_encode, kEncThreads,
                                                      sizeof(EncSmem)) != cudaSuccess ||
        d.enc_per_sm < 1)
      return false;
    if (d.sh_encode_per_sm[0] < 1 || d.sh_encode_per_sm[1] < 1 || d.sh_decode_per_sm < 1)
      return false;
    if (d.hist_per_sm < 1)
      return false;
    // The decoders' payload reads hit L1 most of the time: give L1 all the on-chip memory that
    // the resident decode blocks do not need for their tables.
    for (uint32_t kind : {HX_KIND_HUFFMAN, HX_KIND_QLC, HX_KIND_EXPGOLOMB})
      for (int i = 0; i < 3; ++i)
        if (!prefer_l1(dev, reinterpret_cast<const void*>(prefix_decoder(kind, i)),
                       d.dec_per_sm[kind == HX_KIND_HUFFMAN ? 0 : 1][i], kDecodeBlock[i],
                       dec_lut_bytes(kind, i)))
          return false;
    d.sms = sms;
  }
  *out = d;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int launched() { return cudaGetLastError() == cudaSuccess ? HX_OK : HX_ERR_CUDA; }

// Checks the arguments and fills the kernel arguments of one encode. Returns HX_OK or a host
// error.
int encode_args(uint32_t kind, const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                EncodeArgs* a, DeviceInfo* info) {
  if (!d_tables || !d_out || !d_scratch || !d_status || (n && !d_in)) return HX_ERR_ARG;
  if (kind != HX_KIND_HUFFMAN && kind != HX_KIND_QLC && kind != HX_KIND_SHANNONIC &&
      kind != HX_KIND_EXPGOLOMB)
    return HX_ERR_ARG;
  if (n >= (1ull << 32) || out_cap < payload_offset(n) + 8) return HX_ERR_ARG;
  if (!aligned16(d_in) || !aligned16(d_out) || !aligned16(d_scratch) || !aligned16(d_tables))
    return HX_ERR_ARG;
  if (!device_info(info)) return HX_ERR_CUDA;
  const uint32_t nchunks = (uint32_t)n_chunks_of(n);
  // scratch (hx_scratch_bytes): u64 look[nchunks] (kind 2 uses one per group of 4 chunks), then
  // the u32 counter
  *a = EncodeArgs{static_cast<const hx::Tables*>(d_tables), d_in, n, static_cast<uint8_t*>(d_out),
                  out_cap, d_hist, d_status, kind, static_cast<uint64_t*>(d_scratch),
                  reinterpret_cast<uint32_t*>(static_cast<uint64_t*>(d_scratch) + nchunks),
                  kDefaultWaitNs, ~0ull, kEncFlushRounds};
  return HX_OK;
}

// The single-pass encode: zero the look-back words and the counter, then one block per SM.
int launch_encode(const EncodeArgs& a, const DeviceInfo& info, cudaStream_t s) {
  const uint64_t nchunks = n_chunks_of(a.n);
  if (cudaMemsetAsync(a.look, 0, 8 * nchunks + 4, s) != cudaSuccess) return HX_ERR_CUDA;
  const uint32_t grid = (uint32_t)std::max<uint64_t>(
      1, std::min<uint64_t>((nchunks + kEncWarps - 1) / kEncWarps,
                            (uint64_t)info.sms * info.enc_per_sm));
  k_encode<<<grid, kEncThreads, sizeof(EncSmem), s>>>(a);
  return launched();
}

// The Shannonic encode: zero the look-back words and the counter, then one block per SM (a
// group of 4 chunks per warp and round).
int launch_shannonic(const EncodeArgs& a, const DeviceInfo& info, cudaStream_t s) {
  const uint64_t nchunks = n_chunks_of(a.n), ngroups = (nchunks + 3) / 4;
  const int hist = a.hist != nullptr;
  const uint64_t warps = hist ? sh_enc_warps<true>() : sh_enc_warps<false>();
  if (cudaMemsetAsync(a.look, 0, 8 * nchunks + 4, s) != cudaSuccess) return HX_ERR_CUDA;
  const uint32_t grid = (uint32_t)std::max<uint64_t>(
      1, std::min<uint64_t>((ngroups + warps - 1) / warps,
                            (uint64_t)info.sms * info.sh_encode_per_sm[hist]));
  if (hist) k_sh_encode<true><<<grid, 32 * warps, sizeof(ShEncodeSmem<true>), s>>>(a);
  else k_sh_encode<false><<<grid, 32 * warps, sizeof(ShEncodeSmem<false>), s>>>(a);
  return launched();
}

int encode_common(uint32_t kind, const void* d_tables, const uint8_t* d_in, uint64_t n,
                  void* d_out, uint64_t out_cap, void* d_scratch, uint32_t* d_hist,
                  uint32_t* d_status, void* stream, uint64_t wait_ns = kDefaultWaitNs,
                  uint64_t withhold = ~0ull, uint32_t flush = kEncFlushRounds) {
  EncodeArgs a;
  DeviceInfo info;
  const int rc = encode_args(kind, d_tables, d_in, n, d_out, out_cap, d_scratch, d_hist, d_status,
                             &a, &info);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  a.wait_ns = wait_ns;
  a.withhold = withhold;
  a.flush = flush;  // k_encode's; k_sh_encode's warps count into tables of their own
  return kind == HX_KIND_SHANNONIC ? launch_shannonic(a, info, s) : launch_encode(a, info, s);
}

int decode_common(uint32_t kind, const void* const* d_set, uint32_t nset, const void* d_stream,
                  uint64_t bytes, uint8_t* d_out, uint64_t n, uint32_t* d_status, void* stream) {
  if (!d_set || nset < 1 || nset > (uint32_t)kMaxTableSet) return HX_ERR_ARG;
  for (uint32_t i = 0; i < nset; ++i)
    if (!d_set[i] || !aligned16(d_set[i])) return HX_ERR_ARG;
  if (!d_stream || !d_status || (n && !d_out)) return HX_ERR_ARG;
  if (n >= (1ull << 32)) return HX_ERR_ARG;
  if (!aligned16(d_stream) || !aligned16(d_out)) return HX_ERR_ARG;
  if (bytes < payload_offset(n) + 8) return HX_ERR_CORRUPT;
  DeviceInfo info;
  if (!device_info(&info)) return HX_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint64_t nchunks = n_chunks_of(n);
  // prefix codes: blocks of 1024 from half a wave of them on (64 chunks per SM; the one table
  // copy per SM leaves the most L1 for the payload words), else of 256 from 16 chunks per SM, else
  // of 64 (small inputs over as many SMs as possible)
  int bi = 2;
  if (nchunks >= (uint64_t)info.sms * 64) bi = 0;
  else if (nchunks >= (uint64_t)info.sms * 16) bi = 1;
  const int threads = kind == HX_KIND_SHANNONIC ? kDecThreads : kDecodeBlock[bi];
  const int per_sm = kind == HX_KIND_SHANNONIC ? info.sh_decode_per_sm
                                               : info.dec_per_sm[kind == HX_KIND_HUFFMAN ? 0 : 1][bi];
  const uint64_t per_block = threads / 8;
  const uint64_t want = (nchunks + per_block - 1) / per_block;
  const uint32_t grid =
      (uint32_t)std::max<uint64_t>(1, std::min<uint64_t>(want, (uint64_t)info.sms * per_sm));
  DecodeArgs a{};
  for (uint32_t i = 0; i < nset; ++i) a.set[i] = static_cast<const hx::Tables*>(d_set[i]);
  a.nset = nset;
  a.st = static_cast<const uint8_t*>(d_stream);
  a.bytes = bytes;
  a.out = d_out;
  a.n = n;
  a.status = d_status;
  a.kind = kind;
  if (kind == HX_KIND_SHANNONIC)
    k_sh_decode<<<grid, kDecThreads, 0, s>>>(a);
  else
    prefix_decoder(kind, bi)<<<grid, threads, dec_lut_bytes(kind, bi), s>>>(a);
  return launched();
}

}  // namespace

// Scratch of hx_encode_noalloc: the single-pass encoder's look-back words (8 bytes per chunk)
// and its chunk counter, for HX_NOALLOC_MAX_BYTES of input. Host code must not pass this name to
// a kernel (on the host it is only a stand-in); its device address comes from
// cudaGetSymbolAddress, once per device.
constexpr uint64_t kNoallocScratch = 8 * (HX_NOALLOC_MAX_BYTES / HX_CHUNK) + 16;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratch];

namespace {
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64];  // device address of g_noalloc_scratch, per device
}  // namespace

extern "C" {

uint64_t hx_scratch_bytes(uint64_t n) { return 8 * n_chunks_of(n) + 16; }

// For callers that cannot allocate device memory at encode time (a framework's caching
// allocator owns the device memory, or a path that cannot take cudaMalloc's implicit
// synchronisation): hx_encode with Huffman tables, its scratch in g_noalloc_scratch. The first
// call on a device fetches that array's address with the device current; every call clears the
// words it uses there first (a cudaMemsetAsync, which allocates nothing), and calls that overlap
// on the GPU race on the shared array.
int hx_encode_noalloc(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                      uint64_t out_cap, uint32_t* d_hist, uint32_t* d_status, void* stream) {
  if (n > HX_NOALLOC_MAX_BYTES) return HX_ERR_ARG;
  static_assert(sizeof(g_noalloc_scratch) >= 8 * (HX_NOALLOC_MAX_BYTES / HX_CHUNK) + 4,
                "scratch array smaller than the look-back words and counter of the limit");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HX_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HX_ERR_CUDA;
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return encode_common(HX_KIND_HUFFMAN, d_tables, d_in, n, d_out, out_cap, scratch, d_hist,
                       d_status, stream);
}

int hx_codebook_upload(const hx_codebook* cb, void* d_tables, void* stream) {
  if (!d_tables) return HX_ERR_ARG;
  alignas(16) static thread_local unsigned char host[HX_TABLES_BYTES];
  const int rc = hx_codebook_tables(cb, host);
  if (rc) return rc;
  // pageable source: the copy has consumed `host` when the call returns
  if (cudaMemcpyAsync(d_tables, host, HX_TABLES_BYTES, cudaMemcpyHostToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return HX_ERR_CUDA;
  return HX_OK;
}

int hx_histogram(const uint8_t* d_in, uint64_t n, uint32_t* d_counts, void* stream) {
  if (!d_counts || (n && !d_in) || n >= (1ull << 32) || !aligned16(d_in)) return HX_ERR_ARG;
  if (n == 0) return HX_OK;
  DeviceInfo info;
  if (!device_info(&info)) return HX_ERR_CUDA;
  const uint64_t want = (n / 16 + kHistThreads - 1) / kHistThreads;
  const uint32_t grid = (uint32_t)std::max<uint64_t>(
      1, std::min<uint64_t>(want, (uint64_t)info.sms * info.hist_per_sm));
  k_histogram<<<grid, kHistThreads, 0, static_cast<cudaStream_t>(stream)>>>(d_in, n, d_counts);
  return launched();
}

int hx_encode(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out, uint64_t out_cap,
              void* d_scratch, uint32_t* d_hist, uint32_t* d_status, void* stream) {
  return encode_common(HX_KIND_HUFFMAN, d_tables, d_in, n, d_out, out_cap, d_scratch, d_hist,
                       d_status, stream);
}

int hx_qlc_encode(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                  uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                  void* stream) {
  return encode_common(HX_KIND_QLC, d_tables, d_in, n, d_out, out_cap, d_scratch, d_hist,
                       d_status, stream);
}

int hx_encode_bounded(uint32_t kind, const void* d_tables, const uint8_t* d_in, uint64_t n,
                      void* d_out, uint64_t out_cap, void* d_scratch, uint32_t* d_hist,
                      uint32_t* d_status, uint64_t wait_ns, uint64_t withhold,
                      uint32_t flush_rounds, void* stream) {
  if (flush_rounds > kEncFlushRoundsMax) return HX_ERR_ARG;
  return encode_common(kind, d_tables, d_in, n, d_out, out_cap, d_scratch, d_hist, d_status,
                       stream, wait_ns, withhold, flush_rounds ? flush_rounds : kEncFlushRounds);
}

int hx_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes, uint8_t* d_out,
              uint64_t n_expected, uint32_t* d_status, void* stream) {
  return decode_common(HX_KIND_HUFFMAN, &d_tables, 1, d_stream, stream_bytes, d_out, n_expected,
                       d_status, stream);
}

int hx_qlc_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes,
                  uint8_t* d_out, uint64_t n_expected, uint32_t* d_status, void* stream) {
  return decode_common(HX_KIND_QLC, &d_tables, 1, d_stream, stream_bytes, d_out, n_expected,
                       d_status, stream);
}

int hx_shannonic_encode(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                        uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                        void* stream) {
  return encode_common(HX_KIND_SHANNONIC, d_tables, d_in, n, d_out, out_cap, d_scratch, d_hist,
                       d_status, stream);
}

int hx_shannonic_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes,
                        uint8_t* d_out, uint64_t n_expected, uint32_t* d_status, void* stream) {
  return decode_common(HX_KIND_SHANNONIC, &d_tables, 1, d_stream, stream_bytes, d_out, n_expected,
                       d_status, stream);
}

int hx_expgolomb_encode(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                        uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                        void* stream) {
  return encode_common(HX_KIND_EXPGOLOMB, d_tables, d_in, n, d_out, out_cap, d_scratch, d_hist,
                       d_status, stream);
}

int hx_expgolomb_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes,
                        uint8_t* d_out, uint64_t n_expected, uint32_t* d_status, void* stream) {
  return decode_common(HX_KIND_EXPGOLOMB, &d_tables, 1, d_stream, stream_bytes, d_out,
                       n_expected, d_status, stream);
}

int hx_decode_set(uint32_t kind, const void* const* d_tables, uint32_t n_tables,
                  const void* d_stream, uint64_t stream_bytes, uint8_t* d_out,
                  uint64_t n_expected, uint32_t* d_status, void* stream) {
  if (kind != HX_KIND_HUFFMAN && kind != HX_KIND_QLC && kind != HX_KIND_SHANNONIC &&
      kind != HX_KIND_EXPGOLOMB)
    return HX_ERR_ARG;
  return decode_common(kind, d_tables, n_tables, d_stream, stream_bytes, d_out, n_expected,
                       d_status, stream);
}

}  // extern "C"
