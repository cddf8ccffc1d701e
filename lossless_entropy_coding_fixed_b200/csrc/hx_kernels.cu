// CUDA kernels of the hx library (sm_100a) and the C entry points that launch them.
//
// The method: "Single-Stage Huffman Encoder for ML Compression" (abstract) -- a codebook fixed
// from earlier batches, so the coder runs with no frequency pass and ships no codebook; "Quad
// Length Codes for Lossless Compression of e4m3" (abstract, Tables 1-2) -- the area code.
//
//   k_histogram  byte histogram: 16-byte loads, one private 256-bin table per warp in shared
//                memory, one global atomic per non-empty bin and block.
//
//   k_encode     persistent; one 4096-symbol chunk per block iteration, encoder block e of E
//                taking chunks e, e+E, e+2E, ... Input chunks arrive in a 3-stage shared-memory
//                ring by bulk asynchronous copies (cp.async.bulk + mbarrier), issued as soon as a
//                stage is free. The code/length table is replicated 16 times ([symbol][copy]),
//                so a warp's 32 lookups meet at most two to a bank; its high bits count the
//                symbols, so a single shared atomic both reads the code and adds to the fused
//                histogram.
//                Warp prefix sums of the code lengths (warp k = sub-stream k: the warp prefixes
//                are the sync offsets) and packing through a 64-bit accumulator into a shared
//                output buffer; the chunk's size goes out at once as a flag word. A chunk is
//                stored a few iterations later, when every block has published the sizes of its
//                wave: each block sums the wave's sizes itself (no serial scan, no dedicated
//                block) and keeps a running total of earlier waves, which gives the offset.
//
//   k_decode     one thread per sub-stream (8 per chunk, 32 chunks per 256-thread block). The
//                payload is read word by word, a few words ahead of use (predicated loads, no
//                lane-dependent branch); a 64-bit bit window feeds one lookup per symbol in the
//                4096-entry shared table, which gives symbol and length for either kind (for a
//                QLC code it is precomputed from the area widths and the rank table). 32
//                decoded bytes leave as two 16-byte stores (a whole 32-byte sector). Every
//                sub-stream must end exactly where the next one starts.
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
constexpr int kStages = 3;        // encode input ring
constexpr int kLag = 2;           // encode: a chunk is stored kLag iterations after it is coded
constexpr int kLutCopies = 16;    // encode: table copies; lane l reads copy l % kLutCopies
constexpr int kOutBufs = kLag + 2;  // encode output buffers
// 12-bit counters; a copy gains at most 16 per chunk from each lane that reads it
constexpr uint32_t kHistFlushChunks = 4095 / (16 * (32 / kLutCopies));
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s bound on any wait

// per-chunk flag word: [63:62] state, [61:0] value. The block that codes a chunk publishes its
// size in words (kFlagSize).
constexpr unsigned long long kFlagSize = 1ull << 62;
constexpr unsigned long long kFlagValue = (1ull << 62) - 1;
constexpr uint32_t kMaxEncodeBlocks = 2 * kEncThreads;  // a wave's sizes: two per thread

__host__ __device__ inline uint64_t n_chunks_of(uint64_t n) { return (n + kChunk - 1) / kChunk; }
__host__ __device__ inline uint64_t sync_offset(uint64_t n) {
  return (64 + 4 * (n_chunks_of(n) + 1) + 15) / 16 * 16;
}
__host__ __device__ inline uint64_t payload_offset(uint64_t n) {
  return sync_offset(n) + 16 * n_chunks_of(n);
}

// ---------------------------------------------------------------------------------- PTX helpers
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
__device__ inline uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ inline void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bulk copy global -> shared (no multicast), completion counted on `bar`.
__device__ inline void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ inline void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ inline void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Wait for phase `parity` of `bar`; false after kWaitLimitNs.
__device__ inline bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > kWaitLimitNs) return false;
  return true;
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

struct EncSmem {
  // [symbol][copy]: (code << 20) | (count << 8) | len. Lane l reads copy l % kLutCopies, so a
  // warp's lookups meet at most 32 / kLutCopies to a bank; len in the low byte lets 16 entries
  // be summed into a bit count (16 * 12 < 256); the code comes out with one shift.
  uint32_t lut[256 * kLutCopies];
  alignas(128) uint8_t in[kStages][kChunk];
  uint32_t out[kOutBufs][kMaxChunkWords];
  alignas(16) uint32_t warp_bits[kOutBufs][kEncThreads / 32];
  alignas(8) uint32_t wave_red[2][2 * (kEncThreads / 32)];  // per warp (total, prefix), by parity
  uint64_t bar[kStages];
  uint32_t stop;  // a bulk copy did not complete in time
};

// Every header field but total_words (written by the block that finishes the last chunk).
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

// Size flag of chunk c, waiting (bounded in time) until its block has published it.
__device__ uint32_t wait_chunk_size(const EncodeArgs& a, uint32_t c, unsigned long long f) {
  if ((f & ~kFlagValue) == kFlagSize) return (uint32_t)(f & kFlagValue);
  const unsigned long long t0 = global_ns();
  while (true) {
    __nanosleep(32);
    f = ld_relaxed(a.flags + c);
    if ((f & ~kFlagValue) == kFlagSize) return (uint32_t)(f & kFlagValue);
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(a.status, (uint32_t)HX_ERR_TIMEOUT);
      return 0;
    }
  }
}

// The 16 symbols of one thread -> table entries (and the fused histogram); returns the summed
// entries, whose low byte is the thread's bit count. FULL: all 16 symbols exist.
template <bool HIST, bool FULL>
__device__ __forceinline__ uint32_t lookup16(uint32_t* lut_lane, const uint32_t w[4],
                                             uint32_t valid, uint32_t e[16]) {
  uint32_t sum = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t sym = (w[j >> 2] >> (8 * (j & 3))) & 0xffu;
    uint32_t ent = 0;
    if (FULL || (uint32_t)j < valid) {
      uint32_t* slot = lut_lane + sym * kLutCopies;
      ent = HIST ? atomicAdd(slot, 1u << 8) : *slot;
    }
    e[j] = ent;
    sum += ent;
  }
  return sum;
}

// Pack 16 (code, len) entries MSB-first starting at bit `off` of buf: two codes are joined in a
// 32-bit register (<= 24 bits), then appended to a 64-bit accumulator (hi:lo) with funnel
// shifts. Every finished word is OR-ed into the zeroed buffer (the first and last may be shared
// with neighbours), so the emit is one predicated step with no lane-dependent branch.
__device__ __forceinline__ void pack16(const uint32_t e[16], uint32_t off, uint32_t* buf) {
  uint32_t widx = off >> 5;
  uint32_t nacc = off & 31;  // the first bits belong to the previous thread (zeros here)
  uint32_t hi = 0, lo = 0;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const uint32_t e0 = e[2 * p], e1 = e[2 * p + 1];
    const uint32_t l1 = e1 & 0xffu;
    const uint32_t pl = (e0 & 0xffu) + l1;
    const uint32_t pc = ((e0 >> 20) << l1) | (e1 >> 20);
    hi = __funnelshift_l(lo, hi, pl);
    lo = (lo << pl) | pc;
    nacc += pl;
    const bool full = nacc >= 32;
    nacc -= full ? 32u : 0u;
    if (full) atomicOr(&buf[widx], __funnelshift_r(lo, hi, nacc));
    widx += full ? 1u : 0u;
  }
  if (nacc) atomicOr(&buf[widx], lo << (32 - nacc));
}

// Encoder block e of E takes chunks e, e + E, e + 2E, ... in order: iteration k codes chunk
// kE + e, and the chunks kE .. kE + E - 1 form wave k. Stage k % kStages of the input ring
// holds the chunk of iteration k, loaded by a bulk copy kStages iterations ahead.
//
// Word offsets without a serial scan: a chunk is stored kLag iterations after it is coded.
// Then every block reads the sizes that all blocks published for that wave (two per thread,
// requested before the symbol work), and one block-wide sum gives both the wave's total and
// the words of the chunks before its own in the wave. Each block adds the wave totals up as it
// goes, so the offset of its chunk is that running total plus its in-wave prefix. All blocks
// are resident (cooperative launch), so every size a block waits for is being computed.
template <bool HIST, bool COMPLETE>
__device__ void encode_chunks(const EncodeArgs& a, EncSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint64_t n = a.n;
  const uint32_t nchunks = (uint32_t)n_chunks_of(n);
  const uint32_t full_chunks = (uint32_t)(n / kChunk);
  const uint32_t E = gridDim.x, eb = blockIdx.x;
  const uint64_t P = payload_offset(n);
  uint32_t* word_off = reinterpret_cast<uint32_t*>(a.out + 64);
  uint4* sync = reinterpret_cast<uint4*>(a.out + sync_offset(n));
  uint32_t* payload = reinterpret_cast<uint32_t*>(a.out + P);
  uint32_t* lut_lane = sm.lut + lane % kLutCopies;
  auto chunk_of = [&](uint32_t k) -> uint32_t { return k * E + eb; };

  // stage k % kStages <- chunk of iteration k (bulk copy for a full chunk; else a plain arrive)
  auto issue = [&](uint32_t k) {
    const uint32_t c = chunk_of(k);
    uint64_t* bar = &sm.bar[k % kStages];
    if (c < full_chunks) {
      mbar_arrive_expect_tx(bar, kChunk);
      bulk_load(sm.in[k % kStages], a.in + (uint64_t)c * kChunk, kChunk, bar);
    } else {
      mbar_arrive(bar);
    }
  };
  // only thread 0 waits on a stage; the block barrier after it hands the stage to every thread
  auto await_stage = [&](uint32_t k) {
    if (chunk_of(k) < nchunks && !mbar_wait(&sm.bar[k % kStages], (k / kStages) & 1u)) {
      sm.stop = 1;
      atomicOr(a.status, (uint32_t)HX_ERR_TIMEOUT);
    }
  };
  // size flags of wave w that this thread sums: its chunks tid and tid + kEncThreads
  auto load_wave = [&](uint32_t w, unsigned long long f[2]) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t j = (uint32_t)tid + i * kEncThreads;
      const uint64_t c = (uint64_t)w * E + j;
      f[i] = (j < E && c < nchunks) ? ld_relaxed(a.flags + c) : kFlagSize;
    }
  };
  // this thread's part of the wave total and of the block's in-wave prefix, reduced per warp
  auto reduce_wave = [&](uint32_t w, unsigned long long f[2], uint32_t parity) {
    uint32_t tot = 0, pre = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t j = (uint32_t)tid + i * kEncThreads;
      const uint32_t v = wait_chunk_size(a, w * E + j, f[i]);
      tot += v;
      pre += j < eb ? v : 0u;
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
      tot += __shfl_xor_sync(0xffffffffu, tot, d);
      pre += __shfl_xor_sync(0xffffffffu, pre, d);
    }
    if (lane == 0) {
      sm.wave_red[parity][2 * warp] = tot;
      sm.wave_red[parity][2 * warp + 1] = pre;
    }
  };
  if (tid == 0) {
    sm.stop = 0;
    for (uint32_t k = 0; k < (uint32_t)kStages; ++k) issue(k);
    await_stage(0);
    if (nchunks == 0 && eb == 0) {  // an empty stream: header, index and guards only
      write_header(a);
      reinterpret_cast<uint64_t*>(a.out)[4] = 0;
      word_off[0] = 0;
      payload[0] = 0;  // the host checked cap >= P + 8
      payload[1] = 0;
    }
  }
  __syncthreads();

  bool uncodable = false;
  uint32_t since_flush = 0;
  uint64_t running = 0;  // words of all waves before the one being stored

  // Stores of the chunk of iteration k (output buffer k % kOutBufs); its wave's sums are in
  // wave_red[parity]. Every thread computes the same offset.
  auto store_chunk = [&](uint32_t k, uint32_t parity) {
    // lanes 0..7 fetch one warp's (total, prefix) pair each; a shuffle sum spreads the result
    uint2 wr = lane < kEncThreads / 32
                   ? *reinterpret_cast<const uint2*>(&sm.wave_red[parity][2 * lane])
                   : make_uint2(0u, 0u);
#pragma unroll
    for (int d = 4; d > 0; d >>= 1) {
      wr.x += __shfl_xor_sync(0xffffffffu, wr.x, d);
      wr.y += __shfl_xor_sync(0xffffffffu, wr.y, d);
    }
    const uint32_t wave_total = __shfl_sync(0xffffffffu, wr.x, 0);
    const uint32_t before = __shfl_sync(0xffffffffu, wr.y, 0);
    const uint64_t woff = running + before;
    running += wave_total;
    const int b = (int)(k % kOutBufs);
    const uint32_t c = chunk_of(k);
    const uint4 t0 = *reinterpret_cast<const uint4*>(&sm.warp_bits[b][0]);
    const uint4 t1 = *reinterpret_cast<const uint4*>(&sm.warp_bits[b][4]);
    const uint32_t total = t0.x + t0.y + t0.z + t0.w + t1.x + t1.y + t1.z + t1.w;
    const uint32_t words = (total + 31) >> 5;
    const bool fits = P + 4ull * (woff + words + 2) <= a.cap;
    uint32_t* buf = sm.out[b];
    for (uint32_t i = tid; i < words; i += kEncThreads) {
      if (fits) payload[woff + i] = buf[i];
      buf[i] = 0;
    }
    if (tid == 0) {
      const uint32_t p1 = t0.x, p2 = p1 + t0.y, p3 = p2 + t0.z, p4 = p3 + t0.w;
      const uint32_t p5 = p4 + t1.x, p6 = p5 + t1.y, p7 = p6 + t1.z;
      sync[c] = make_uint4(total | (p1 << 16), p2 | (p3 << 16), p4 | (p5 << 16), p6 | (p7 << 16));
      word_off[c] = (uint32_t)woff;
      if (!fits) atomicOr(a.status, (uint32_t)HX_ERR_CAPACITY);
      if (c == 0) write_header(a);
      if (c == nchunks - 1) {  // the last chunk closes the index
        const uint64_t end = woff + words;
        word_off[nchunks] = (uint32_t)end;
        reinterpret_cast<uint64_t*>(a.out)[4] = end;
        if (fits) {
          payload[end] = 0;
          payload[end + 1] = 0;
        }
      }
    }
  };

  auto flush_hist = [&]() {  // counts in the lane tables -> global, then clear them
    __syncthreads();
    uint32_t sum = 0;
    for (int l = 0; l < kLutCopies; ++l) {
      const uint32_t e = sm.lut[tid * kLutCopies + l];
      sum += (e >> 8) & 0xfffu;
      sm.lut[tid * kLutCopies + l] = e & ~(0xfffu << 8);
    }
    if (sum) atomicAdd(&a.hist[tid], sum);
    __syncthreads();
  };

  uint32_t k = 0;
  for (;; ++k) {
    const uint32_t c = chunk_of(k);
    if (c >= nchunks || sm.stop) break;  // uniform: sm.stop is set before a block barrier
    const int s = (int)(k % kStages);
    const int ob = (int)(k % kOutBufs);
    const bool lagged = k >= kLag;
    unsigned long long wf[2];
    if (lagged) load_wave(k - kLag, wf);  // answers are needed only after the symbol work

    uint32_t w[4];
    uint32_t e[16];
    uint32_t sum;
    if (c < full_chunks) {
      const uint4 v = reinterpret_cast<const uint4*>(sm.in[s])[tid];
      w[0] = v.x;
      w[1] = v.y;
      w[2] = v.z;
      w[3] = v.w;
      sum = lookup16<HIST, true>(lut_lane, w, 16, e);
      if (!COMPLETE)
#pragma unroll
        for (int j = 0; j < 16; ++j) uncodable |= (e[j] & 0xffu) == 0;
    } else {  // the ragged last chunk, from global memory
      const uint64_t base = (uint64_t)c * kChunk;
      const uint32_t first = (uint32_t)tid * 16;
      const uint32_t count = (uint32_t)(n - base);
      const uint32_t valid = count > first ? min(16u, count - first) : 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t x = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if ((uint32_t)(4 * q + b) < valid)
            x |= (uint32_t)a.in[base + first + 4 * q + b] << (8 * b);
        w[q] = x;
      }
      sum = lookup16<HIST, false>(lut_lane, w, valid, e);
      if (!COMPLETE)
#pragma unroll
        for (int j = 0; j < 16; ++j) uncodable |= (uint32_t)j < valid && (e[j] & 0xffu) == 0;
    }
    const uint32_t bits = sum & 0xffu;
    uint32_t incl = bits;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += t;
    }
    if (lane == 31) sm.warp_bits[ob][warp] = incl;
    if (lagged) reduce_wave(k - kLag, wf, k & 1);
    if (tid == 0) await_stage(k + 1);
    __syncthreads();  // warp totals and wave sums ready; stage s read; next stage handed over

    // lanes 0..7 hold the warp totals; a shuffle scan gives this warp's base and the total
    uint32_t wt = lane < kEncThreads / 32 ? sm.warp_bits[ob][lane] : 0u;
#pragma unroll
    for (int d = 1; d < kEncThreads / 32; d <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, wt, d);
      if (lane >= d) wt += t;
    }
    const uint32_t warp_base = __shfl_sync(0xffffffffu, wt, (warp + 31) & 31) & (warp ? ~0u : 0u);
    const uint32_t total = __shfl_sync(0xffffffffu, wt, kEncThreads / 32 - 1);
    if (tid == 0) {
      st_relaxed(a.flags + c, kFlagSize | ((total + 31) >> 5));
      fence_proxy_async();  // this stage's generic reads before the async refill
      issue(k + kStages);
    }
    if (bits) pack16(e, warp_base + incl - bits, sm.out[ob]);
    if (lagged) store_chunk(k - kLag, k & 1);
    if (HIST && ++since_flush == kHistFlushChunks) {
      flush_hist();
      since_flush = 0;
    }
  }
  if (tid == 0 && sm.stop)  // timed out: let copies still in flight land
    for (uint32_t j = 0; j < (uint32_t)kStages; ++j)
      if (chunk_of(k + j) < full_chunks)
        mbar_wait(&sm.bar[(k + j) % kStages], ((k + j) / kStages) & 1u);
  // drain: the last kLag coded chunks
  for (uint32_t j = k > kLag ? k - kLag : 0; j < k; ++j) {
    unsigned long long wf[2];
    load_wave(j, wf);
    __syncthreads();
    reduce_wave(j, wf, 0);
    __syncthreads();
    store_chunk(j, 0);
  }
  if (!COMPLETE && uncodable) atomicOr(a.status, (uint32_t)HX_ERR_UNCODABLE);
  if (HIST) flush_hist();
}

__global__ void __launch_bounds__(kEncThreads, 3) k_encode(EncodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  EncSmem& sm = *reinterpret_cast<EncSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const uint32_t nchunks = (uint32_t)n_chunks_of(a.n);
  if (a.tables->magic != hx::kTablesMagic || a.tables->kind != a.kind) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, (uint32_t)HX_ERR_ARG);
    return;
  }
  bool complete = true;
  for (int i = tid; i < 256 * kLutCopies; i += kEncThreads) {
    const uint32_t t = a.tables->enc[i / kLutCopies];  // (code << 4) | len
    uint32_t e = ((t >> 4) << 20) | (t & 15u);
    if ((t & 15u) > HX_LMAX_MAX || t > 0xffffu) {  // a damaged table block stays harmless
      e = 0;
      atomicOr(a.status, (uint32_t)HX_ERR_ARG);
    }
    complete &= (e & 0xffu) != 0;
    sm.lut[i] = e;
  }
  for (int i = tid; i < kOutBufs * (int)kMaxChunkWords; i += kEncThreads) (&sm.out[0][0])[i] = 0;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.bar[s], 1);
    fence_barrier_init();
  }
  complete = __syncthreads_and(complete);
  if (a.hist) {
    if (complete) encode_chunks<true, true>(a, sm);
    else encode_chunks<true, false>(a, sm);
  } else {
    if (complete) encode_chunks<false, true>(a, sm);
    else encode_chunks<false, false>(a, sm);
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

// Header checks shared by every block; returns total_words, or -status.
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

// Payload words of one sub-stream, MSB-first, through a 64-bit bit window held as two 32-bit
// halves (wh:wl) whose top `avail` bits are valid. The next kPrefetch words are already
// requested (pf[]): a refill takes pf[0] and requests one more word -- one predicated load and
// register moves, no branch that depends on the other lanes. Words past the caller's buffer
// read as 0.
constexpr int kPrefetch = 2;
struct SubstreamReader {
  const uint32_t* words;
  uint64_t wlimit;  // payload words inside the buffer
  uint64_t wi;      // index of the word in pf[0]
  uint32_t pf[kPrefetch];
  uint32_t wh, wl;
  int avail;

  __device__ __forceinline__ uint32_t word(uint64_t i) const {
    return i < wlimit ? __ldg(words + i) : 0u;
  }
  // afterwards >= 32 valid bits: room for two codes of <= 12 bits
  __device__ __forceinline__ void refill() {
    if (avail < 32) {
      const uint32_t w = pf[0];
#pragma unroll
      for (int i = 0; i + 1 < kPrefetch; ++i) pf[i] = pf[i + 1];
      pf[kPrefetch - 1] = word(wi + kPrefetch);
      ++wi;
      wh |= w >> avail;                            // the word lands at bits [32-avail, 64-avail)
      wl |= __funnelshift_lc(0u, w, 32 - avail);  // its low part (nothing when avail == 0)
      avail += 32;
    }
  }
  __device__ __forceinline__ void consume(uint32_t len) {  // len <= 15
    wh = __funnelshift_l(wl, wh, len);
    wl <<= len;
    avail -= (int)len;
  }
  __device__ void start(uint64_t first_bit) {
    const uint64_t fw = first_bit >> 5;
    const uint32_t sh = (uint32_t)(first_bit & 31);
    wh = word(fw);
    wl = word(fw + 1);
    wi = fw + 2;
#pragma unroll
    for (int i = 0; i < kPrefetch; ++i) pf[i] = word(wi + i);
    wh = __funnelshift_l(wl, wh, sh);
    wl <<= sh;
    avail = 64 - (int)sh;
  }
  // index (in payload bits) of the next bit not yet consumed
  __device__ uint64_t position() const { return 32 * wi - (uint64_t)avail; }
};

// One symbol from the top of the window: the 4096-entry table gives (symbol << 8) | length for
// both kinds. For a QLC table the length is 3 + the width of the area in the top 3 bits; the
// table holds it already, so reading it there costs less than recomputing it. An entry of 0
// (no code word starts the window) only occurs for an incomplete code.
template <bool COMPLETE>
__device__ __forceinline__ uint32_t next_symbol(SubstreamReader& rd, bool& invalid,
                                                const uint16_t* lut) {
  const uint32_t e = lut[rd.wh >> 20];
  const uint32_t len = e & 15u;
  if (!COMPLETE) invalid |= len == 0;
  rd.consume(len);
  return e;
}

// 32 symbols -> 32 output bytes (two 16-byte streaming stores, one whole sector). Each symbol's
// byte is moved into place with one byte permute.
template <bool COMPLETE>
__device__ __forceinline__ void decode_group32(SubstreamReader& rd, bool& invalid, uint4* d4,
                                               const uint16_t* lut) {
  uint32_t o[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    rd.refill();
    uint32_t v = next_symbol<COMPLETE>(rd, invalid, lut) >> 8;
    v = __byte_perm(v, next_symbol<COMPLETE>(rd, invalid, lut), 0x3250);
    rd.refill();
    v = __byte_perm(v, next_symbol<COMPLETE>(rd, invalid, lut), 0x3510);
    v = __byte_perm(v, next_symbol<COMPLETE>(rd, invalid, lut), 0x5210);
    o[q] = v;
  }
  __stcs(d4, make_uint4(o[0], o[1], o[2], o[3]));
  __stcs(d4 + 1, make_uint4(o[4], o[5], o[6], o[7]));
}

template <bool COMPLETE>
__device__ void decode_chunks(const DecodeArgs& a, const uint16_t* lut, uint32_t total) {
  const int tid = threadIdx.x;
  const uint64_t n = a.n;
  const uint64_t nchunks = n_chunks_of(n);
  const uint64_t P = payload_offset(n);
  const uint32_t* word_off = reinterpret_cast<const uint32_t*>(a.st + 64);
  const uint4* sync = reinterpret_cast<const uint4*>(a.st + sync_offset(n));
  SubstreamReader rd;
  rd.words = reinterpret_cast<const uint32_t*>(a.st + P);
  rd.wlimit = (a.bytes - P) / 4;  // payload words inside the buffer
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
    bool bad = w0 > w1 || w1 > total || nbits > 32u * (w1 - w0) || (nbits + 31) / 32 != w1 - w0;
    const uint32_t mine = (uint32_t)k < nsub ? min(kSubLen, count - k * kSubLen) : 0u;
    if (mine == 0) {
      bad |= k > 0 && sync_at(k) != nbits;
    } else if (!bad) {
      const uint32_t start = k == 0 ? 0u : sync_at(k);
      const uint32_t end = (uint32_t)k + 1 < nsub ? sync_at(k + 1) : nbits;
      const uint64_t first_bit = 32ull * w0 + start;
      rd.start(first_bit);
      bool invalid = false;
      uint8_t* dst = a.out + c * kChunk + (uint64_t)k * kSubLen;
      const uint32_t groups = mine / 32;
      for (uint32_t g = 0; g < groups; ++g)
        decode_group32<COMPLETE>(rd, invalid, reinterpret_cast<uint4*>(dst + 32 * g), lut);
      for (uint32_t i = groups * 32; i < mine; ++i) {
        rd.refill();
        dst[i] = (uint8_t)(next_symbol<COMPLETE>(rd, invalid, lut) >> 8);
      }
      // the sub-stream must end exactly where the next one starts
      bad |= invalid || rd.position() != 32ull * w0 + end;
    }
    if (bad) atomicOr(a.status, (uint32_t)HX_ERR_CORRUPT);
  }
}

// KIND is checked against the stream header and the tables; the symbol loop is the same.
template <int KIND>
__global__ void __launch_bounds__(kDecThreads, 5) k_decode(DecodeArgs a) {
  __shared__ __align__(16) uint16_t s_lut[4096];
  __shared__ int64_t s_total;
  const int tid = threadIdx.x;
  if (tid == 0) s_total = check_header(a);
  const uint4* src = reinterpret_cast<const uint4*>(a.tables->dec);
  uint4* dst = reinterpret_cast<uint4*>(s_lut);
  for (int i = tid; i < 4096 * 2 / 16; i += kDecThreads) dst[i] = src[i];
  __syncthreads();
  const int64_t total = s_total;
  if (total < 0) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(a.status, (uint32_t)(-total));
    return;
  }
  if (a.tables->complete)
    decode_chunks<true>(a, s_lut, (uint32_t)total);
  else
    decode_chunks<false>(a, s_lut, (uint32_t)total);
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
    if (cudaFuncSetAttribute(k_encode, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(EncSmem)) != cudaSuccess)
      return false;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.enc_per_sm, k_encode, kEncThreads,
                                                      sizeof(EncSmem)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.huff_per_sm, k_decode<HX_KIND_HUFFMAN>,
                                                      kDecThreads, 0) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.qlc_per_sm, k_decode<HX_KIND_QLC>,
                                                      kDecThreads, 0) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.hist_per_sm, k_histogram, kHistThreads,
                                                      0) != cudaSuccess)
      return false;
    if (d.enc_per_sm < 1 || d.huff_per_sm < 1 || d.qlc_per_sm < 1 || d.hist_per_sm < 1)
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
  // blocks take chunks round-robin and wait for each other's sizes: all must be resident at
  // once (cooperative launch), and a wave's sizes are summed two per thread
  const uint32_t grid = (uint32_t)std::max<uint64_t>(
      1, std::min<uint64_t>({(uint64_t)nchunks, (uint64_t)info.sms * info.enc_per_sm,
                             (uint64_t)kMaxEncodeBlocks}));
  void* params[] = {&a};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(k_encode), dim3(grid),
                                  dim3(kEncThreads), params, sizeof(EncSmem), s) != cudaSuccess)
    return launched() | HX_ERR_CUDA;
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

// Scratch of hx_encode_noalloc: one flag word per chunk plus the ticket, for up to
// HX_NOALLOC_MAX_BYTES of input. Host code must not pass this name to a kernel (on the host it is
// only a stand-in); its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[8 * (HX_NOALLOC_MAX_BYTES / HX_CHUNK) + 16];

namespace {
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64];  // device address of g_noalloc_scratch, per device
}  // namespace

extern "C" {

uint64_t hx_scratch_bytes(uint64_t n) { return 8 * n_chunks_of(n) + 16; }

// For callers that cannot allocate device memory at encode time (a framework's caching
// allocator owns the device memory, or a path that cannot take cudaMalloc's implicit
// synchronisation): hx_encode with Huffman tables, its scratch in g_noalloc_scratch. The first
// call on a device fetches that array's address with the device current; every call zeroes the
// part it uses (k_zero_scratch) and calls that overlap on the GPU race on the shared array.
int hx_encode_noalloc(const void* d_tables, const uint8_t* d_in, uint64_t n, void* d_out,
                      uint64_t out_cap, uint32_t* d_hist, uint32_t* d_status, void* stream) {
  if (n > HX_NOALLOC_MAX_BYTES) return HX_ERR_ARG;
  static_assert(sizeof(g_noalloc_scratch) >= 8 * (HX_NOALLOC_MAX_BYTES / HX_CHUNK) + 16,
                "scratch array smaller than hx_scratch_bytes(HX_NOALLOC_MAX_BYTES)");
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
