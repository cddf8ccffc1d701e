// CUDA kernels of the hx library (sm_100a) and the C entry points that launch them.
//
//   k_histogram   byte histogram: 16-byte loads, one private 256-bin table per warp in shared
//                 memory, one global atomic per non-empty bin and block.
//   k_encode      one 4096-symbol chunk per block iteration (persistent grid, chunks taken in
//                 order from an atomic ticket): code/length lookup from a shared-memory table,
//                 warp + block prefix sums of the code lengths (warp k = sub-stream k, so the
//                 warp prefixes are the sync offsets), packing through a 64-bit accumulator into
//                 shared memory, the chunk's word offset from a single-pass decoupled look-back
//                 scan (Merrill & Garland 2016) with a bounded wait, then coalesced word stores.
//   k_decode      one thread per sub-stream (8 per chunk, 32 chunks per 256-thread block): a
//                 64-bit bit window refilled from the payload, one lookup per symbol in the
//                 4096-entry shared-memory table (Huffman) or a 3-bit area + index read (QLC),
//                 16 output bytes per 16-byte store. Every sub-stream must end exactly where the
//                 next one starts.
//
// The method: "Single-Stage Huffman Encoder for ML Compression" (abstract) -- a codebook fixed
// from earlier batches, so the coder runs with no frequency pass and ships no codebook; "Quad
// Length Codes for Lossless Compression of e4m3" (abstract, Tables 1-2) -- the area code.
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
constexpr uint32_t kMaxChunkWords = HX_CHUNK * HX_LMAX_MAX / 32;  // 1536
constexpr int kEncThreads = 256;  // 16 symbols per thread; warp k codes sub-stream k
constexpr int kDecThreads = 256;  // 8 threads per chunk, 32 chunks per block
constexpr int kHistThreads = 256;
constexpr unsigned long long kLookbackLimitNs = 1000000000ull;  // 1 s bound on any wait

// look-back flag word: [63:62] state, [61:0] value (words)
constexpr unsigned long long kFlagAggregate = 1ull << 62;
constexpr unsigned long long kFlagInclusive = 2ull << 62;
constexpr unsigned long long kFlagValue = (1ull << 62) - 1;

__host__ __device__ inline uint64_t n_chunks_of(uint64_t n) { return (n + kChunk - 1) / kChunk; }
__host__ __device__ inline uint64_t sync_offset(uint64_t n) {
  return (64 + 4 * (n_chunks_of(n) + 1) + 15) / 16 * 16;
}
__host__ __device__ inline uint64_t payload_offset(uint64_t n) {
  return sync_offset(n) + 16 * n_chunks_of(n);
}

__device__ inline unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ inline void st_relaxed(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ inline unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------------- histogram
__global__ void __launch_bounds__(kHistThreads) k_histogram(const uint8_t* __restrict__ in,
                                                            uint64_t n, uint32_t* counts) {
  __shared__ uint32_t bins[kHistThreads / 32][256];
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < (kHistThreads / 32) * 256; i += kHistThreads) (&bins[0][0])[i] = 0;
  __syncthreads();
  uint32_t* mine = bins[warp];
  const uint64_t nvec = n / 16;
  const uint4* v = reinterpret_cast<const uint4*>(in);
  for (uint64_t i = blockIdx.x * (uint64_t)kHistThreads + tid; i < nvec;
       i += (uint64_t)gridDim.x * kHistThreads) {
    const uint4 x = __ldcs(v + i);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      atomicAdd(&mine[w[j] & 0xff], 1u);
      atomicAdd(&mine[(w[j] >> 8) & 0xff], 1u);
      atomicAdd(&mine[(w[j] >> 16) & 0xff], 1u);
      atomicAdd(&mine[w[j] >> 24], 1u);
    }
  }
  if (blockIdx.x == 0)
    for (uint64_t i = nvec * 16 + tid; i < n; i += kHistThreads) atomicAdd(&mine[in[i]], 1u);
  __syncthreads();
  uint32_t sum = 0;
#pragma unroll
  for (int w = 0; w < kHistThreads / 32; ++w) sum += bins[w][tid];
  if (sum) atomicAdd(&counts[tid], sum);
}

// ---------------------------------------------------------------------------------- encode
struct EncodeArgs {
  const hx::Tables* tables;
  const uint8_t* in;
  uint64_t n;
  uint8_t* out;
  uint64_t cap;
  unsigned long long* flags;  // scratch: one look-back word per chunk
  uint32_t* ticket;           // scratch: next chunk to take
  uint32_t* hist;             // optional fused histogram
  uint32_t* status;
  uint32_t kind;
};

// Every header field but total_words (written by the block that codes the last chunk).
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

// Decoupled look-back: publish this chunk's word count, then add up predecessors until one
// with an inclusive prefix is found. Chunks are taken in ticket order, so every predecessor is
// already running and will publish; the wait is still bounded (HX_ERR_TIMEOUT).
__device__ uint32_t chunk_word_offset(const EncodeArgs& a, uint32_t c, uint32_t words) {
  if (c == 0) {
    st_relaxed(a.flags, kFlagInclusive | words);
    return 0;
  }
  st_relaxed(a.flags + c, kFlagAggregate | words);
  unsigned long long excl = 0;
  int64_t j = (int64_t)c - 1;
  unsigned long long t0 = 0;
  while (j >= 0) {
    const unsigned long long f = ld_relaxed(a.flags + j);
    const unsigned long long state = f & ~kFlagValue;
    if (state == 0) {
      const unsigned long long now = global_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kLookbackLimitNs) {
        atomicOr(a.status, (uint32_t)HX_ERR_TIMEOUT);
        break;
      }
      __nanosleep(64);
      continue;
    }
    excl += f & kFlagValue;
    if (state == kFlagInclusive) break;
    --j;
  }
  st_relaxed(a.flags + c, kFlagInclusive | (excl + words));
  return (uint32_t)excl;
}

__global__ void __launch_bounds__(kEncThreads) k_encode(EncodeArgs a) {
  __shared__ uint32_t s_lut[256];
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_buf[kMaxChunkWords];
  __shared__ uint32_t s_warp_bits[kEncThreads / 32];
  __shared__ uint32_t s_chunk, s_offset;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint64_t n = a.n;
  const uint32_t nchunks = (uint32_t)n_chunks_of(n);
  if (a.tables->magic != hx::kTablesMagic || a.tables->kind != a.kind) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, (uint32_t)HX_ERR_ARG);
    return;
  }
  {
    uint32_t e = a.tables->enc[tid];
    if ((e & 15u) > HX_LMAX_MAX) {  // keeps a damaged table block inside the staging buffer
      e = 0;
      atomicOr(a.status, (uint32_t)HX_ERR_ARG);
    }
    s_lut[tid] = e;
  }
  s_hist[tid] = 0;
  if (blockIdx.x == 0 && tid == 0 && nchunks == 0) {
    write_header(a);
    reinterpret_cast<uint64_t*>(a.out)[4] = 0;
    reinterpret_cast<uint32_t*>(a.out + 64)[0] = 0;
    const uint64_t P = payload_offset(0);
    if (P + 8 <= a.cap) {
      reinterpret_cast<uint32_t*>(a.out + P)[0] = 0;
      reinterpret_cast<uint32_t*>(a.out + P)[1] = 0;
    } else {
      atomicOr(a.status, (uint32_t)HX_ERR_CAPACITY);
    }
  }
  const uint64_t P = payload_offset(n);
  uint32_t* word_off = reinterpret_cast<uint32_t*>(a.out + 64);
  uint4* sync = reinterpret_cast<uint4*>(a.out + sync_offset(n));
  uint32_t* payload = reinterpret_cast<uint32_t*>(a.out + P);
  const bool want_hist = a.hist != nullptr;
  bool uncodable = false;

  for (;;) {
    if (tid == 0) s_chunk = atomicAdd(a.ticket, 1u);
    for (int i = tid; i < (int)kMaxChunkWords; i += kEncThreads) s_buf[i] = 0;
    __syncthreads();
    const uint32_t c = s_chunk;
    if (c >= nchunks) break;
    const uint64_t base = (uint64_t)c * kChunk;
    const uint32_t count = n - base < kChunk ? (uint32_t)(n - base) : kChunk;
    const uint32_t first = (uint32_t)tid * 16;

    // 16 symbols of this thread
    uint32_t w[4];
    if (count == kChunk) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(a.in + base) + tid);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t x = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const uint32_t i = first + 4 * q + b;
          if (i < count) x |= (uint32_t)a.in[base + i] << (8 * b);
        }
        w[q] = x;
      }
    }
    const uint32_t valid = count > first ? min(16u, count - first) : 0u;
    uint32_t e[16];
    uint32_t bits = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t sym = (w[j >> 2] >> (8 * (j & 3))) & 0xff;
      const bool here = (uint32_t)j < valid;
      const uint32_t ent = here ? s_lut[sym] : 0u;
      uncodable |= here && (ent & 15u) == 0;
      if (want_hist && here) atomicAdd(&s_hist[sym], 1u);
      e[j] = ent;
      bits += ent & 15u;
    }

    // bit offset of this thread inside the chunk: warp scan, then the warps before it
    uint32_t incl = bits;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += t;
    }
    if (lane == 31) s_warp_bits[warp] = incl;
    __syncthreads();
    uint32_t warp_base = 0, total = 0;
#pragma unroll
    for (int k = 0; k < kEncThreads / 32; ++k) {
      const uint32_t t = s_warp_bits[k];
      warp_base += k < warp ? t : 0u;
      total += t;
    }
    const uint32_t off = warp_base + incl - bits;

    // pack: whole words this thread owns are stored, shared boundary words are OR-ed
    if (bits) {
      uint32_t widx = off >> 5;
      const uint32_t lead = off & 31;
      uint64_t acc = 0;
      uint32_t nacc = lead;
      bool first_word = true;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t len = e[j] & 15u;
        acc = (acc << len) | (e[j] >> 4);
        nacc += len;
        if (nacc >= 32) {
          nacc -= 32;
          const uint32_t word = (uint32_t)(acc >> nacc);
          if (first_word && lead) atomicOr(&s_buf[widx], word);
          else s_buf[widx] = word;
          first_word = false;
          ++widx;
        }
      }
      if (nacc) atomicOr(&s_buf[widx], (uint32_t)(acc << (32 - nacc)));
    }
    const uint32_t words = (total + 31) >> 5;
    __syncthreads();

    if (tid == 0) s_offset = chunk_word_offset(a, c, words);
    __syncthreads();
    const uint32_t woff = s_offset;
    const bool fits = P + 4ull * ((uint64_t)woff + words + 2) <= a.cap;
    if (fits) {
      for (uint32_t i = tid; i < words; i += kEncThreads) payload[woff + i] = s_buf[i];
    }
    if (tid == 0) {
      word_off[c] = woff;
      uint32_t pre[HX_SUBSTREAMS];
      uint32_t acc = 0;
#pragma unroll
      for (int k = 0; k < HX_SUBSTREAMS; ++k) {
        pre[k] = acc;
        acc += s_warp_bits[k];
      }
      sync[c] = make_uint4(total | (pre[1] << 16), pre[2] | (pre[3] << 16), pre[4] | (pre[5] << 16),
                           pre[6] | (pre[7] << 16));
      if (!fits) atomicOr(a.status, (uint32_t)HX_ERR_CAPACITY);
      if (c == 0) write_header(a);
      if (c == nchunks - 1) {
        const uint32_t end = woff + words;
        word_off[nchunks] = end;
        reinterpret_cast<uint64_t*>(a.out)[4] = end;
        if (fits) {
          payload[end] = 0;
          payload[end + 1] = 0;
        }
      }
    }
    __syncthreads();
  }
  if (uncodable) atomicOr(a.status, (uint32_t)HX_ERR_UNCODABLE);
  if (want_hist) {
    __syncthreads();
    if (s_hist[tid]) atomicAdd(&a.hist[tid], s_hist[tid]);
  }
}

__global__ void k_zero_scratch(unsigned long long* flags, uint32_t nchunks, uint32_t* ticket) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < nchunks) flags[i] = 0;
  if (i == 0) *ticket = 0;
}

// ---------------------------------------------------------------------------------- decode
struct DecodeArgs {
  const hx::Tables* tables;
  const uint8_t* st;
  uint64_t bytes;
  uint8_t* out;
  uint64_t n;
  uint32_t* status;
  uint32_t kind;
};

// Header checks shared by every block; returns total_words, or -1 after raising the status.
__device__ int64_t check_header(const DecodeArgs& a) {
  const uint32_t* h32 = reinterpret_cast<const uint32_t*>(a.st);
  const uint64_t* h64 = reinterpret_cast<const uint64_t*>(a.st);
  const uint32_t vk = h32[1];
  if (a.tables->magic != hx::kTablesMagic || a.tables->kind != a.kind) return -(int64_t)HX_ERR_ARG;
  if (h32[0] != kMagic || (vk & 0xff) != 1 || h32[2] != kChunk || h32[3] != HX_SUBSTREAMS)
    return -(int64_t)HX_ERR_CORRUPT;
  if (((vk >> 8) & 0xff) != a.kind || ((vk >> 16) & 0xff) != a.tables->lmax ||
      h64[5] != a.tables->hash)
    return -(int64_t)HX_ERR_CODEBOOK;
  if (h64[2] != a.n || h64[3] != n_chunks_of(a.n)) return -(int64_t)HX_ERR_CORRUPT;
  const uint64_t P = payload_offset(a.n);
  const uint64_t total = h64[4];
  // the host guarantees bytes >= P + 8; the payload and its 2 guard words must fit
  if (total > (a.bytes - P) / 4 - 2 || total >= (1ull << 32)) return -(int64_t)HX_ERR_CORRUPT;
  return (int64_t)total;
}

template <int KIND>
__global__ void __launch_bounds__(kDecThreads) k_decode(DecodeArgs a) {
  __shared__ __align__(16) uint16_t s_lut[KIND == HX_KIND_HUFFMAN ? 4096 : 2];
  __shared__ uint8_t s_r2s[256];
  __shared__ uint32_t s_area[8];
  __shared__ int64_t s_total;
  const int tid = threadIdx.x;
  if (tid == 0) s_total = check_header(a);
  if (KIND == HX_KIND_HUFFMAN) {
    const uint4* src = reinterpret_cast<const uint4*>(a.tables->dec);
    uint4* dst = reinterpret_cast<uint4*>(s_lut);
    for (int i = tid; i < 4096 * 2 / 16; i += kDecThreads) dst[i] = src[i];
  } else {
    s_r2s[tid] = a.tables->rank2sym[tid];
    if (tid < 8) s_area[tid] = a.tables->qlc_area[tid];
  }
  __syncthreads();
  const int64_t total = s_total;
  if (total < 0) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, (uint32_t)(-total));
    return;
  }
  const uint32_t qbits = a.tables->qlc_bits_packed;
  const uint64_t n = a.n;
  const uint64_t nchunks = n_chunks_of(n);
  const uint32_t* word_off = reinterpret_cast<const uint32_t*>(a.st + 64);
  const uint4* sync = reinterpret_cast<const uint4*>(a.st + sync_offset(n));
  const uint32_t* payload = reinterpret_cast<const uint32_t*>(a.st + payload_offset(n));
  const uint32_t last_word = (uint32_t)total + 1;  // the second guard word
  const int k = tid & 7;

  for (uint64_t c = (uint64_t)blockIdx.x * (kDecThreads / 8) + (tid >> 3); c < nchunks;
       c += (uint64_t)gridDim.x * (kDecThreads / 8)) {
    const uint32_t w0 = __ldg(word_off + c), w1 = __ldg(word_off + c + 1);
    const uint4 sy = __ldg(sync + c);
    auto sync_at = [&](uint32_t i) -> uint32_t {  // u16 entry i of the chunk's sync row
      const uint32_t w = i < 2 ? sy.x : i < 4 ? sy.y : i < 6 ? sy.z : sy.w;
      return (w >> (16 * (i & 1))) & 0xffffu;
    };
    const uint32_t nbits = sy.x & 0xffffu;
    const uint32_t count = n - c * kChunk < kChunk ? (uint32_t)(n - c * kChunk) : kChunk;
    const uint32_t nsub = (count + kSubLen - 1) / kSubLen;
    bool bad = w0 > w1 || w1 > (uint32_t)total || nbits > 32u * (w1 - w0) ||
               (nbits + 31) / 32 != w1 - w0;
    const uint32_t mine = (uint32_t)k < nsub ? min(kSubLen, count - k * kSubLen) : 0u;
    if (mine == 0) {
      bad |= k > 0 && sync_at(k) != nbits;
    } else if (!bad) {
      const uint32_t start = k == 0 ? 0u : sync_at(k);
      const uint32_t end = (uint32_t)k + 1 < nsub ? sync_at(k + 1) : nbits;
      uint32_t widx = w0 + (start >> 5);
      auto fetch = [&](uint32_t i) -> uint32_t { return __ldg(payload + min(i, last_word)); };
      uint64_t win = ((uint64_t)fetch(widx) << 32) | fetch(widx + 1);
      win <<= (start & 31);
      int avail = 64 - (int)(start & 31);
      widx += 2;
      uint32_t used = 0;
      bool invalid = false;
      uint8_t* dst = a.out + c * kChunk + (uint64_t)k * kSubLen;

      auto step = [&]() -> uint32_t {
        if (avail < 32) {
          win |= (uint64_t)fetch(widx++) << (32 - avail);
          avail += 32;
        }
        uint32_t sym, len;
        if (KIND == HX_KIND_HUFFMAN) {
          const uint32_t e = s_lut[win >> 52];
          len = e >> 8;
          sym = e & 0xff;
          invalid |= len == 0;
        } else {
          const uint32_t area = (uint32_t)(win >> 61);
          const uint32_t b = (qbits >> (4 * area)) & 15u;
          const uint32_t idx = (uint32_t)(win >> (61 - b)) & ((1u << b) - 1u);
          const uint32_t info = s_area[area];
          invalid |= idx >= ((info >> 9) & 511u);
          sym = s_r2s[((info & 511u) + idx) & 255u];
          len = 3 + b;
        }
        win <<= len;
        avail -= (int)len;
        used += len;
        return sym;
      };

      const uint32_t groups = mine / 16;
      for (uint32_t g = 0; g < groups; ++g) {
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v = step();
          v |= step() << 8;
          v |= step() << 16;
          v |= step() << 24;
          o[q] = v;
        }
        reinterpret_cast<uint4*>(dst)[g] = make_uint4(o[0], o[1], o[2], o[3]);
      }
      for (uint32_t i = groups * 16; i < mine; ++i) dst[i] = (uint8_t)step();
      bad |= invalid || start + used != end;
    }
    if (bad) atomicOr(a.status, (uint32_t)HX_ERR_CORRUPT);
  }
}

// ---------------------------------------------------------------------------------- launch
struct DeviceInfo {
  int sms = 0;
  int enc_per_sm = 0, huff_per_sm = 0, qlc_per_sm = 0, hist_per_sm = 0;
};

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
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.enc_per_sm, k_encode, kEncThreads, 0) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.huff_per_sm, k_decode<HX_KIND_HUFFMAN>,
                                                      kDecThreads, 0) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.qlc_per_sm, k_decode<HX_KIND_QLC>,
                                                      kDecThreads, 0) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.hist_per_sm, k_histogram, kHistThreads,
                                                      0) != cudaSuccess)
      return false;
    d.sms = sms;
  }
  *out = d;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int launched() { return cudaGetLastError() == cudaSuccess ? HX_OK : HX_ERR_CUDA; }

int encode_common(uint32_t kind, const void* d_tables, const uint8_t* d_in, uint64_t n,
                  void* d_out, uint64_t out_cap, void* d_scratch, uint32_t* d_hist,
                  uint32_t* d_status, void* stream) {
  if (!d_tables || !d_out || !d_scratch || !d_status || (n && !d_in)) return HX_ERR_ARG;
  if (n >= (1ull << 32) || out_cap < payload_offset(n) + 8) return HX_ERR_ARG;
  if (!aligned16(d_in) || !aligned16(d_out) || !aligned16(d_scratch) || !aligned16(d_tables))
    return HX_ERR_ARG;
  DeviceInfo info;
  if (!device_info(&info)) return HX_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint32_t nchunks = (uint32_t)n_chunks_of(n);
  auto* flags = static_cast<unsigned long long*>(d_scratch);
  auto* ticket = reinterpret_cast<uint32_t*>(flags + nchunks);
  k_zero_scratch<<<(nchunks + 255) / 256 + (nchunks == 0), 256, 0, s>>>(flags, nchunks, ticket);
  EncodeArgs a{static_cast<const hx::Tables*>(d_tables), d_in, n, static_cast<uint8_t*>(d_out),
               out_cap, flags, ticket, d_hist, d_status, kind};
  const uint32_t grid =
      (uint32_t)std::max<uint64_t>(1, std::min<uint64_t>(nchunks, (uint64_t)info.sms * info.enc_per_sm));
  k_encode<<<grid, kEncThreads, 0, s>>>(a);
  return launched();
}

int decode_common(uint32_t kind, const void* d_tables, const void* d_stream, uint64_t bytes,
                  uint8_t* d_out, uint64_t n, uint32_t* d_status, void* stream) {
  if (!d_tables || !d_stream || !d_status || (n && !d_out)) return HX_ERR_ARG;
  if (n >= (1ull << 32)) return HX_ERR_ARG;
  if (!aligned16(d_stream) || !aligned16(d_out) || !aligned16(d_tables)) return HX_ERR_ARG;
  if (bytes < payload_offset(n) + 8) return HX_ERR_CORRUPT;
  DeviceInfo info;
  if (!device_info(&info)) return HX_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint64_t nchunks = n_chunks_of(n);
  const uint64_t per_block = kDecThreads / 8;
  const int per_sm = kind == HX_KIND_HUFFMAN ? info.huff_per_sm : info.qlc_per_sm;
  const uint64_t want = (nchunks + per_block - 1) / per_block;
  const uint32_t grid =
      (uint32_t)std::max<uint64_t>(1, std::min<uint64_t>(want, (uint64_t)info.sms * per_sm));
  DecodeArgs a{static_cast<const hx::Tables*>(d_tables), static_cast<const uint8_t*>(d_stream),
               bytes, d_out, n, d_status, kind};
  if (kind == HX_KIND_HUFFMAN)
    k_decode<HX_KIND_HUFFMAN><<<grid, kDecThreads, 0, s>>>(a);
  else
    k_decode<HX_KIND_QLC><<<grid, kDecThreads, 0, s>>>(a);
  return launched();
}

}  // namespace

extern "C" {

uint64_t hx_scratch_bytes(uint64_t n) { return 8 * n_chunks_of(n) + 16; }

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

int hx_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes, uint8_t* d_out,
              uint64_t n_expected, uint32_t* d_status, void* stream) {
  return decode_common(HX_KIND_HUFFMAN, d_tables, d_stream, stream_bytes, d_out, n_expected,
                       d_status, stream);
}

int hx_qlc_decode(const void* d_tables, const void* d_stream, uint64_t stream_bytes,
                  uint8_t* d_out, uint64_t n_expected, uint32_t* d_status, void* stream) {
  return decode_common(HX_KIND_QLC, d_tables, d_stream, stream_bytes, d_out, n_expected, d_status,
                       stream);
}

}  // extern "C"
