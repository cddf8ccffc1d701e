// Oracle for the fixed-codebook entropy coder of 8-bit tensor symbols.
//
// TEST INFRASTRUCTURE ONLY. This file is the plain, slow, obviously correct CPU definition of
// every result the CUDA library computes. Only the tests, the smoke check and the benchmark's
// CPU-baseline leg may load it. It shares no code, header, table or constant generator with the
// library: the stream format below is written out a second time from its specification.
//
// Method sources:
//   [SSH] "Single-Stage Huffman Encoder for ML Compression", abstract: a Huffman codebook fixed
//         in advance from the average distribution of previous batches; no per-shard frequency
//         pass and no codebook sent with the data.
//   [QLC] "Quad Length Codes for Lossless Compression of e4m3", abstract and Tables 1-2: a 3-bit
//         area prefix selects one of 8 areas; each area holds a run of symbols ranked by
//         probability and codes them with a fixed number of index bits.
//   [PM]  Larmore & Hirschberg (1990), package-merge for length-limited prefix codes.
//   [RFC] RFC 1951 section 3.2.2, canonical Huffman codes from code lengths.
//   [SHN] the "Shannonic" review page (method and runtime sections): the 256 byte values split
//         by dynamic programming into at most K = 16 contiguous ranges that minimise the range
//         entropy plus the fixed-width offset bits; the range index is coded by 128-state tANS
//         (J. Duda, asymmetric numeral systems, table variant), the offset in ceil(log2 size)
//         bits.
//   [EG]  the QLC page's contrast case, universal Exp-Golomb codes: order k codes v >= 0 as
//         floor(log2(v / 2^k + 1)) zeros, then v + 2^k in binary (ITU-T H.264 section 9.1
//         is the order-0 case); a byte is first mapped to v by its sign and magnitude.
//
// Readings where the pages are silent (all stated once more in the design notes):
//   - averaging over equal-size batches == summing their counts; every byte gets a code
//     (weight max(w,1)) unless seen-only is asked for;
//   - package-merge ties: leaves sorted by (weight, symbol); a leaf goes before a package of
//     equal weight; packages keep creation order;
//   - QLC widths are non-decreasing over areas, at most `max_distinct` distinct widths (4, the
//     "quad"), area a (0-based) has code a in 3 bits; ties between equal-cost width vectors go
//     to the lexicographically smallest; ranking ties go to the smaller symbol.
//
// Stream format (version 1), all little-endian, offsets from the stream start:
//   0   u32 magic 0x31305848 ("HX01")     4 u8 version=1   5 u8 kind (0 Huffman, 1 QLC)
//   6   u8 lmax   7 u8 0                  8 u32 chunk=4096 12 u32 substreams=8
//   16  u64 n     24 u64 n_chunks = ceil(n/4096)   32 u64 total_words   40 u64 codebook hash
//   48  16 zero bytes
//   64  u32 word_off[n_chunks+1]          (words from the payload start)
//   S = round_up_16(64 + 4*(n_chunks+1)): u16 sync[n_chunks][8]; [0] = the chunk's bit count,
//       [k] = bit offset of symbol 512k inside the chunk (= the bit count if it does not exist)
//   P = S + 16*n_chunks: u32 payload[total_words], MSB-first (bit 31 of word 0 first), each
//       chunk zero-padded to a whole word; then 2 zero guard words.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

constexpr uint32_t kMagic = 0x31305848u;
constexpr uint8_t kVersion = 1;
constexpr uint64_t kChunk = 4096;
constexpr uint64_t kSubstreams = 8;
constexpr uint64_t kSubLen = 512;
constexpr int kLmaxCap = 12;
constexpr int kQlcLmax = 11;

// status bits, same meaning as the library's
constexpr int kErrArg = 1, kErrUncodable = 4, kErrCorrupt = 8, kErrCodebook = 16, kErrCapacity = 64;

uint64_t n_chunks_of(uint64_t n) { return (n + kChunk - 1) / kChunk; }
uint64_t sync_offset(uint64_t n) { return (64 + 4 * (n_chunks_of(n) + 1) + 15) / 16 * 16; }
uint64_t payload_offset(uint64_t n) { return sync_offset(n) + 16 * n_chunks_of(n); }

uint32_t rd32(const uint8_t* p) { uint32_t v; std::memcpy(&v, p, 4); return v; }
uint64_t rd64(const uint8_t* p) { uint64_t v; std::memcpy(&v, p, 8); return v; }
uint16_t rd16(const uint8_t* p) { uint16_t v; std::memcpy(&v, p, 2); return v; }
void wr32(uint8_t* p, uint32_t v) { std::memcpy(p, &v, 4); }
void wr64(uint8_t* p, uint64_t v) { std::memcpy(p, &v, 8); }
void wr16(uint8_t* p, uint16_t v) { std::memcpy(p, &v, 2); }

// FNV-1a, 64-bit: offset basis 14695981039346656037, prime 1099511628211.
uint64_t fnv1a(const std::vector<uint8_t>& bytes) {
  uint64_t h = 14695981039346656037ull;
  for (uint8_t b : bytes) { h ^= b; h *= 1099511628211ull; }
  return h;
}

// ---- [PM] package-merge: optimal code lengths with no length above lmax -----------------------
struct Item {
  uint64_t w;
  std::vector<int> occurrences;  // how many times each symbol's leaf sits inside this item
};

// weights: 256 entries; symbols with weight 0 get no code. Returns false if impossible.
bool package_merge(const uint64_t* weights, int lmax, uint8_t* len_out) {
  std::memset(len_out, 0, 256);
  std::vector<Item> leaves;
  for (int s = 0; s < 256; ++s) {
    if (weights[s] == 0) continue;
    Item it{weights[s], std::vector<int>(256, 0)};
    it.occurrences[s] = 1;
    leaves.push_back(it);
  }
  const int m = (int)leaves.size();
  if (m == 0) return true;
  if (m == 1) {  // a one-symbol alphabet still needs one bit per symbol
    for (int s = 0; s < 256; ++s) if (weights[s]) len_out[s] = 1;
    return true;
  }
  if (lmax < 1 || lmax > kLmaxCap || (1 << lmax) < m) return false;
  // leaves in (weight, symbol) order: they were pushed in symbol order, so a stable sort works
  std::stable_sort(leaves.begin(), leaves.end(),
                   [](const Item& a, const Item& b) { return a.w < b.w; });

  std::vector<Item> list = leaves;  // the list of the deepest level, lmax
  for (int level = lmax - 1; level >= 1; --level) {
    // package: pair up neighbours of the list below, an odd last item is dropped
    std::vector<Item> packages;
    for (size_t i = 0; i + 1 < list.size(); i += 2) {
      Item p{list[i].w + list[i + 1].w, std::vector<int>(256, 0)};
      for (int s = 0; s < 256; ++s)
        p.occurrences[s] = list[i].occurrences[s] + list[i + 1].occurrences[s];
      packages.push_back(p);
    }
    // merge with the leaves; on equal weight the leaf comes first
    std::vector<Item> merged;
    size_t a = 0, b = 0;
    while (a < leaves.size() || b < packages.size()) {
      if (b == packages.size() || (a < leaves.size() && leaves[a].w <= packages[b].w))
        merged.push_back(leaves[a++]);
      else
        merged.push_back(packages[b++]);
    }
    list.swap(merged);
  }
  // the cheapest 2m-2 items of the top list; a symbol's length counts its leaf's appearances
  std::vector<int> length(256, 0);
  for (int i = 0; i < 2 * m - 2; ++i)
    for (int s = 0; s < 256; ++s) length[s] += list[i].occurrences[s];
  for (int s = 0; s < 256; ++s) len_out[s] = (uint8_t)length[s];
  return true;
}

// ---- [RFC] canonical codes --------------------------------------------------------------------
void canonical_codes(const uint8_t* len, uint32_t* code) {
  int count[kLmaxCap + 2] = {0};
  for (int s = 0; s < 256; ++s) count[len[s]]++;
  count[0] = 0;
  uint32_t next[kLmaxCap + 2] = {0};
  uint32_t c = 0;
  for (int l = 1; l <= kLmaxCap; ++l) {
    c = (c + count[l - 1]) << 1;
    next[l] = c;
  }
  for (int s = 0; s < 256; ++s) code[s] = len[s] ? next[len[s]]++ : 0;
}

// ---- [QLC] exhaustive search of the area widths --------------------------------------------
struct Qlc {
  uint8_t bits[8];
  uint16_t start[9];
  uint8_t rank2sym[256];
};

bool qlc_search(const uint64_t* weights, int max_distinct, Qlc* q) {
  if (max_distinct < 1 || max_distinct > 8) return false;
  // rank symbols: weight descending, ties to the smaller symbol
  std::vector<int> order(256);
  for (int s = 0; s < 256; ++s) order[s] = s;
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return weights[a] > weights[b]; });
  // every non-decreasing width vector b[0..7] in [0,8]^8, visited in lexicographic order
  int b[8];
  bool have = false;
  unsigned __int128 best_cost = 0;
  int best[8] = {0};
  for (int i = 0; i < 8; ++i) b[i] = 0;
  while (true) {
    uint64_t capacity = 0;
    for (int i = 0; i < 8; ++i) capacity += 1ull << b[i];
    int distinct = 1;
    for (int i = 1; i < 8; ++i) if (b[i] != b[i - 1]) ++distinct;
    if (capacity >= 256 && distinct <= max_distinct) {
      // cost = sum over ranks of weight * (3 + width of the rank's area)
      unsigned __int128 cost = 0;
      int r = 0;
      for (int a = 0; a < 8 && r < 256; ++a) {
        int take = (int)std::min<uint64_t>(1ull << b[a], (uint64_t)(256 - r));
        for (int k = 0; k < take; ++k, ++r)
          cost += (unsigned __int128)weights[order[r]] * (unsigned)(3 + b[a]);
      }
      if (!have || cost < best_cost) {
        have = true;
        best_cost = cost;
        std::memcpy(best, b, sizeof best);
      }
    }
    // next non-decreasing vector: bump the last position that can grow, reset the tail to it
    int i = 7;
    while (i >= 0 && b[i] == 8) --i;
    if (i < 0) break;
    int v = b[i] + 1;
    for (int j = i; j < 8; ++j) b[j] = v;
  }
  if (!have) return false;
  int r = 0;
  for (int a = 0; a < 8; ++a) {
    q->bits[a] = (uint8_t)best[a];
    q->start[a] = (uint16_t)r;
    r += (int)std::min<uint64_t>(1ull << best[a], (uint64_t)(256 - r));
  }
  q->start[8] = (uint16_t)r;
  for (int k = 0; k < 256; ++k) q->rank2sym[k] = (uint8_t)order[k];
  return true;
}

void qlc_codes(const Qlc& q, uint8_t* len, uint32_t* code) {
  for (int a = 0; a < 8; ++a)
    for (int r = q.start[a]; r < q.start[a + 1]; ++r) {
      int s = q.rank2sym[r];
      len[s] = (uint8_t)(3 + q.bits[a]);
      code[s] = ((uint32_t)a << q.bits[a]) | (uint32_t)(r - q.start[a]);
    }
}

// ---- bit-serial writer / reader -------------------------------------------------------------
struct BitWriter {
  std::vector<uint32_t> words;
  uint64_t nbits = 0;
  void put(uint32_t code, int len) {
    for (int i = len - 1; i >= 0; --i) {  // most significant bit first
      uint32_t bit = (code >> i) & 1u;
      if (nbits % 32 == 0) words.push_back(0);
      words.back() |= bit << (31 - nbits % 32);
      ++nbits;
    }
  }
};

struct BitReader {
  const uint8_t* payload;  // first word of the chunk
  uint64_t limit;          // valid bits of the chunk
  uint64_t pos = 0;
  bool past_end = false;
  int get() {
    if (pos >= limit) { past_end = true; return 0; }
    uint32_t w = rd32(payload + 4 * (pos / 32));
    int bit = (int)((w >> (31 - pos % 32)) & 1u);
    ++pos;
    return bit;
  }
};

struct Header {
  uint8_t kind, lmax;
  uint64_t hash;
};

// Encode x[0..n) with per-symbol (len, code) into the framing above. Returns status bits.
int encode(const Header& h, const uint8_t* len, const uint32_t* code, const uint8_t* x, uint64_t n,
           uint8_t* out, uint64_t cap, uint64_t* written) {
  const uint64_t nc = n_chunks_of(n), S = sync_offset(n), P = payload_offset(n);
  *written = 0;
  if (cap < P) return kErrCapacity;
  int status = 0;
  std::vector<uint32_t> word_off(nc + 1, 0);
  std::vector<uint16_t> sync(nc * kSubstreams, 0);
  std::vector<uint32_t> payload;
  for (uint64_t c = 0; c < nc; ++c) {
    BitWriter bw;
    const uint64_t lo = c * kChunk, hi = std::min(n, lo + kChunk);
    uint16_t starts[kSubstreams] = {0};
    for (uint64_t i = lo; i < hi; ++i) {
      if ((i - lo) % kSubLen == 0) starts[(i - lo) / kSubLen] = (uint16_t)bw.nbits;
      const uint8_t s = x[i];
      if (len[s] == 0) { status |= kErrUncodable; continue; }
      bw.put(code[s], len[s]);
    }
    const uint64_t nsub = (hi - lo + kSubLen - 1) / kSubLen;
    sync[c * kSubstreams + 0] = (uint16_t)bw.nbits;
    for (uint64_t k = 1; k < kSubstreams; ++k)
      sync[c * kSubstreams + k] = k < nsub ? starts[k] : (uint16_t)bw.nbits;
    word_off[c] = (uint32_t)payload.size();
    payload.insert(payload.end(), bw.words.begin(), bw.words.end());
  }
  word_off[nc] = (uint32_t)payload.size();
  const uint64_t total = payload.size();
  const uint64_t need = P + 4 * (total + 2);
  // the header is written whenever it fits, so a caller can learn the size it needs
  std::memset(out, 0, (size_t)std::min<uint64_t>(cap, P));
  wr32(out + 0, kMagic);
  out[4] = kVersion;
  out[5] = h.kind;
  out[6] = h.lmax;
  out[7] = 0;
  wr32(out + 8, (uint32_t)kChunk);
  wr32(out + 12, (uint32_t)kSubstreams);
  wr64(out + 16, n);
  wr64(out + 24, nc);
  wr64(out + 32, total);
  wr64(out + 40, h.hash);
  if (need > cap) return status | kErrCapacity;
  for (uint64_t c = 0; c <= nc; ++c) wr32(out + 64 + 4 * c, word_off[c]);
  for (uint64_t i = 0; i < nc * kSubstreams; ++i) wr16(out + S + 2 * i, sync[i]);
  for (uint64_t w = 0; w < total; ++w) wr32(out + P + 4 * w, payload[w]);
  wr32(out + P + 4 * total, 0);
  wr32(out + P + 4 * total + 4, 0);
  *written = need;
  return status;
}

// One-symbol decoders. Each returns the symbol, or -1 when no code word matches.
struct CanonicalDecoder {  // [RFC] inverse: first code and first index of every length, no table
  int lmax;
  int count[kLmaxCap + 1] = {0};
  int64_t first_code[kLmaxCap + 1] = {0};
  int first_index[kLmaxCap + 1] = {0};
  std::vector<int> sorted;  // symbols by (length, symbol)
  explicit CanonicalDecoder(const uint8_t* len, int lmax_) : lmax(lmax_) {
    for (int s = 0; s < 256; ++s) if (len[s]) count[len[s]]++;
    int64_t c = 0;
    int idx = 0;
    for (int l = 1; l <= kLmaxCap; ++l) {  // count[0] stays 0: the same recurrence as encoding
      c = (c + count[l - 1]) << 1;
      first_code[l] = c;
      first_index[l] = idx;
      idx += count[l];
    }
    for (int l = 1; l <= kLmaxCap; ++l)
      for (int s = 0; s < 256; ++s) if (len[s] == l) sorted.push_back(s);
  }
  int next(BitReader& br) const {
    int64_t code = 0;
    for (int l = 1; l <= lmax; ++l) {
      code = (code << 1) | br.get();
      if (br.past_end) return -1;
      const int64_t d = code - first_code[l];
      if (d >= 0 && d < count[l]) return sorted[first_index[l] + (int)d];
    }
    return -1;
  }
};

struct QlcDecoder {  // [QLC]: 3 area bits, then the area's index bits
  Qlc q;
  int next(BitReader& br) const {
    int a = 0;
    for (int i = 0; i < 3; ++i) a = (a << 1) | br.get();
    int idx = 0;
    for (int i = 0; i < q.bits[a]; ++i) idx = (idx << 1) | br.get();
    if (br.past_end) return -1;
    const int r = q.start[a] + idx;
    if (r >= q.start[a + 1]) return -1;
    return q.rank2sym[r];
  }
};

template <class Dec>
int decode(const Header& h, const Dec& dec, const uint8_t* st, uint64_t bytes, uint8_t* out,
           uint64_t n_expected) {
  if (bytes < 64) return kErrCorrupt;
  if (rd32(st) != kMagic || st[4] != kVersion || rd32(st + 8) != kChunk ||
      rd32(st + 12) != kSubstreams)
    return kErrCorrupt;
  if (st[5] != h.kind || st[6] != h.lmax || rd64(st + 40) != h.hash) return kErrCodebook;
  const uint64_t n = rd64(st + 16);
  if (n != n_expected || rd64(st + 24) != n_chunks_of(n)) return kErrCorrupt;
  const uint64_t nc = n_chunks_of(n), S = sync_offset(n), P = payload_offset(n);
  const uint64_t total = rd64(st + 32);
  // the stream holds the payload and its 2 guard words; word offsets are u32
  if (P > bytes || (bytes - P) / 4 < 2 || total > (bytes - P) / 4 - 2 || total >= (1ull << 32))
    return kErrCorrupt;
  int status = 0;
  for (uint64_t c = 0; c < nc; ++c) {
    const uint64_t lo = c * kChunk, hi = std::min(n, lo + kChunk);
    const uint32_t w0 = rd32(st + 64 + 4 * c), w1 = rd32(st + 64 + 4 * (c + 1));
    const uint8_t* sy = st + S + 16 * c;
    const uint64_t nbits = rd16(sy);
    if (w0 > w1 || w1 > total || nbits > 32ull * (w1 - w0) || (nbits + 31) / 32 != w1 - w0) {
      status |= kErrCorrupt;
      continue;
    }
    BitReader br{st + P + 4ull * w0, nbits};
    const uint64_t nsub = (hi - lo + kSubLen - 1) / kSubLen;
    bool bad = false;
    for (uint64_t i = lo; i < hi && !bad; ++i) {
      const uint64_t k = (i - lo) / kSubLen;
      if ((i - lo) % kSubLen == 0 && k > 0 && br.pos != rd16(sy + 2 * k)) bad = true;
      const int s = dec.next(br);
      if (s < 0) bad = true;
      else out[i] = (uint8_t)s;
    }
    if (!bad && br.pos != nbits) bad = true;
    for (uint64_t k = nsub; k < kSubstreams && !bad; ++k)
      if (k > 0 && rd16(sy + 2 * k) != nbits) bad = true;
    if (bad) status |= kErrCorrupt;
  }
  return status;
}

// ---- [SHN] range partition + 128-state tANS --------------------------------------------------
// Readings (the page gives the objective, K = 16 and L = 128, not the details):
//   - ranges are contiguous in byte value; weights max(count, 1) (every byte codable); at most K
//     ranges; cost of range [a, b) with weight W_ab (of W in all) is
//     W_ab * log2(W / W_ab) + W_ab * ceil(log2(b - a)), summed; the dynamic programme takes, for
//     each prefix, the smallest split point reaching the strict minimum, and the smallest range
//     count reaching it;
//   - tANS frequencies: f_r = max(1, floor(W_r L / W)); a shortfall goes +1 at a time to the
//     largest remainders W_r L mod W (ties to the lower range, cycling), an excess -1 at a time
//     from the largest f_r > 1 (ties to the lower range);
//   - spread: positions 0, 83, 166 mod 128, ... (step L/2 + L/8 + 3) take range 0 f_0 times,
//     then range 1, ...; decoding state L + u holds range spread[u], and the k-th state of range
//     r (in increasing u) is reached from x_s = f_r + k;
//   - a sub-stream is encoded from its last symbol to its first, starting in state L: the offset
//     (ceil(log2 size) bits), then the low nb bits of the state (nb making state >> nb fall in
//     [f_r, 2 f_r)), then the state becomes the k-th state of the range, k = (state >> nb) - f_r;
//     after the first symbol the state minus L goes out in 7 bits. Bits are appended MSB-first,
//     so a decoder reads each sub-stream backwards from its end and must finish in state L
//     exactly at the sub-stream's first bit.
constexpr int kShR = 7, kShL = 1 << kShR, kShK = 16, kShStep = kShL / 2 + kShL / 8 + 3;
constexpr uint8_t kKindShannonic = 2;

int ceil_log2(int v) {
  int b = 0;
  while ((1 << b) < v) ++b;
  return b;
}

// Optimal partition of weights[0..n) into at most K contiguous ranges; lo[0..nr] boundaries.
int partition(const uint64_t* w, int n, int K, int* lo) {
  std::vector<uint64_t> P(n + 1, 0);
  for (int i = 0; i < n; ++i) P[i + 1] = P[i] + w[i];
  const double W = (double)P[n];
  auto cost = [&](int a, int b) {
    const uint64_t wab = P[b] - P[a];
    if (wab == 0) return 0.0;
    return (double)wab * std::log2(W / (double)wab) + (double)wab * (double)ceil_log2(b - a);
  };
  const double inf = 1e300;
  std::vector<std::vector<double>> best(K + 1, std::vector<double>(n + 1, inf));
  std::vector<std::vector<int>> from(K + 1, std::vector<int>(n + 1, -1));
  for (int b = 1; b <= n; ++b) best[1][b] = cost(0, b), from[1][b] = 0;
  for (int k = 2; k <= K; ++k)
    for (int b = k; b <= n; ++b)
      for (int a = k - 1; a < b; ++a) {
        const double c = best[k - 1][a] + cost(a, b);
        if (c < best[k][b]) best[k][b] = c, from[k][b] = a;
      }
  int kbest = 1;
  for (int k = 2; k <= K && k <= n; ++k)
    if (best[k][n] < best[kbest][n]) kbest = k;
  int b = n;
  for (int k = kbest; k >= 1; --k) {
    lo[k] = b;
    b = from[k][b];
  }
  lo[0] = 0;
  return kbest;
}

struct Shn {
  int nr;
  int lo[kShK + 1];
  int f[kShK];
  int spread[kShL];
  int range_of[256];
};

void shn_tables(Shn& t) {
  int pos = 0;
  for (int r = 0; r < t.nr; ++r)
    for (int j = 0; j < t.f[r]; ++j) {
      t.spread[pos] = r;
      pos = (pos + kShStep) % kShL;
    }
  for (int r = 0; r < t.nr; ++r)
    for (int v = t.lo[r]; v < t.lo[r + 1]; ++v) t.range_of[v] = r;
}

void normalise(const uint64_t* wr, int nr, int* f) {
  uint64_t W = 0;
  for (int r = 0; r < nr; ++r) W += wr[r];
  int sum = 0;
  std::vector<uint64_t> rem(nr);
  for (int r = 0; r < nr; ++r) {
    const uint64_t q = wr[r] * kShL / W;
    rem[r] = wr[r] * kShL - q * W;
    f[r] = std::max<int>(1, (int)q);
    sum += f[r];
  }
  while (sum < kShL) {  // largest remainder first, ties to the lower range; then cycle
    std::vector<int> order(nr);
    for (int r = 0; r < nr; ++r) order[r] = r;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return rem[a] > rem[b]; });
    for (int i = 0; i < nr && sum < kShL; ++i) ++f[order[i]], ++sum;
  }
  while (sum > kShL) {
    int big = -1;
    for (int r = 0; r < nr; ++r)
      if (f[r] > 1 && (big < 0 || f[r] > f[big])) big = r;
    --f[big];
    --sum;
  }
}

bool shn_build(const uint64_t* counts, int K, bool cover_all, Shn& t) {
  uint64_t w[256];
  for (int s = 0; s < 256; ++s) w[s] = cover_all ? std::max<uint64_t>(counts[s], 1) : counts[s];
  uint64_t W = 0;
  for (int s = 0; s < 256; ++s) W += w[s];
  if (W == 0 || K < 1 || K > kShK) return false;
  t.nr = partition(w, 256, K, t.lo);
  uint64_t wr[kShK] = {0};
  for (int r = 0; r < t.nr; ++r)
    for (int v = t.lo[r]; v < t.lo[r + 1]; ++v) wr[r] += w[v];
  for (int r = 0; r < t.nr; ++r)
    if (wr[r] == 0) return false;  // seen-only weights left a range empty
  normalise(wr, t.nr, t.f);
  shn_tables(t);
  return true;
}

uint64_t shn_hash(const Shn& t) {
  std::vector<uint8_t> b = {kKindShannonic, (uint8_t)kShR, (uint8_t)t.nr};
  for (int r = 1; r < t.nr; ++r) b.push_back((uint8_t)t.lo[r]);
  for (int r = 0; r < t.nr; ++r) b.push_back((uint8_t)t.f[r]);
  return fnv1a(b);
}

// The k-th decoding state of range r (k from 0, increasing u).
int shn_state_of(const Shn& t, int r, int k) {
  for (int u = 0; u < kShL; ++u)
    if (t.spread[u] == r && k-- == 0) return kShL + u;
  return -1;
}

int floor_log2(int v) {
  int b = -1;
  while (v) v >>= 1, ++b;
  return b;
}

void shn_encode_substream(const Shn& t, const uint8_t* x, uint64_t m, BitWriter& bw) {
  int state = kShL;
  for (uint64_t i = m; i-- > 0;) {
    const int s = x[i], r = t.range_of[s];
    bw.put((uint32_t)(s - t.lo[r]), ceil_log2(t.lo[r + 1] - t.lo[r]));
    int nb = 0;
    while ((state >> nb) >= 2 * t.f[r]) ++nb;  // state >> nb lands in [f_r, 2 f_r)
    bw.put((uint32_t)(state & ((1 << nb) - 1)), nb);
    state = shn_state_of(t, r, (state >> nb) - t.f[r]);
  }
  bw.put((uint32_t)(state - kShL), kShR);
}

struct BackReader {  // reads a sub-stream from its end towards its first bit
  const uint8_t* payload;
  uint64_t start, pos;
  bool past = false;
  uint32_t get(int nb) {
    if (pos - start < (uint64_t)nb) { past = true; return 0; }
    uint32_t v = 0;
    for (uint64_t q = pos - nb; q < pos; ++q)
      v = (v << 1) | ((rd32(payload + 4 * (q / 32)) >> (31 - q % 32)) & 1u);
    pos -= nb;
    return v;
  }
};

// Decodes m symbols of a sub-stream occupying chunk bits [start, end); false if it is not one.
bool shn_decode_substream(const Shn& t, const uint8_t* payload, uint64_t start, uint64_t end,
                          uint8_t* out, uint64_t m) {
  int next[kShK];
  for (int r = 0; r < t.nr; ++r) next[r] = t.f[r];
  int dec_xs[kShL];  // x_s of each decoding state
  for (int u = 0; u < kShL; ++u) dec_xs[u] = next[t.spread[u]]++;
  BackReader br{payload, start, end};
  int state = kShL + (int)br.get(kShR);
  for (uint64_t i = 0; i < m; ++i) {
    const int u = state - kShL, r = t.spread[u], xs = dec_xs[u];
    const int nb = kShR - floor_log2(xs);
    const int low = (int)br.get(nb);
    const int off = (int)br.get(ceil_log2(t.lo[r + 1] - t.lo[r]));
    if (br.past || t.lo[r] + off >= t.lo[r + 1]) return false;
    out[i] = (uint8_t)(t.lo[r] + off);
    state = (xs << nb) + low;
  }
  return state == kShL && br.pos == start;
}

int shn_encode(const Shn& t, const uint8_t* x, uint64_t n, uint8_t* out, uint64_t cap,
               uint64_t* written) {
  const uint64_t nc = n_chunks_of(n), S = sync_offset(n), P = payload_offset(n);
  *written = 0;
  if (cap < P) return kErrCapacity;
  std::vector<uint32_t> word_off(nc + 1, 0);
  std::vector<uint16_t> sync(nc * kSubstreams, 0);
  std::vector<uint32_t> payload;
  for (uint64_t c = 0; c < nc; ++c) {
    BitWriter bw;
    const uint64_t lo = c * kChunk, hi = std::min(n, lo + kChunk);
    const uint64_t nsub = (hi - lo + kSubLen - 1) / kSubLen;
    uint16_t starts[kSubstreams] = {0};
    for (uint64_t k = 0; k < nsub; ++k) {
      starts[k] = (uint16_t)bw.nbits;
      const uint64_t a = lo + k * kSubLen, b = std::min(hi, a + kSubLen);
      shn_encode_substream(t, x + a, b - a, bw);
    }
    sync[c * kSubstreams + 0] = (uint16_t)bw.nbits;
    for (uint64_t k = 1; k < kSubstreams; ++k)
      sync[c * kSubstreams + k] = k < nsub ? starts[k] : (uint16_t)bw.nbits;
    word_off[c] = (uint32_t)payload.size();
    payload.insert(payload.end(), bw.words.begin(), bw.words.end());
  }
  word_off[nc] = (uint32_t)payload.size();
  const uint64_t total = payload.size();
  const uint64_t need = P + 4 * (total + 2);
  std::memset(out, 0, (size_t)std::min<uint64_t>(cap, P));
  wr32(out + 0, kMagic);
  out[4] = kVersion;
  out[5] = kKindShannonic;
  out[6] = (uint8_t)kShR;
  out[7] = 0;
  wr32(out + 8, (uint32_t)kChunk);
  wr32(out + 12, (uint32_t)kSubstreams);
  wr64(out + 16, n);
  wr64(out + 24, nc);
  wr64(out + 32, total);
  wr64(out + 40, shn_hash(t));
  if (need > cap) return kErrCapacity;
  for (uint64_t c = 0; c <= nc; ++c) wr32(out + 64 + 4 * c, word_off[c]);
  for (uint64_t i = 0; i < nc * kSubstreams; ++i) wr16(out + S + 2 * i, sync[i]);
  for (uint64_t w = 0; w < total; ++w) wr32(out + P + 4 * w, payload[w]);
  wr32(out + P + 4 * total, 0);
  wr32(out + P + 4 * total + 4, 0);
  *written = need;
  return 0;
}

int shn_decode(const Shn& t, const uint8_t* st, uint64_t bytes, uint8_t* out, uint64_t n_expected) {
  if (bytes < 64) return kErrCorrupt;
  if (rd32(st) != kMagic || st[4] != kVersion || rd32(st + 8) != kChunk ||
      rd32(st + 12) != kSubstreams)
    return kErrCorrupt;
  if (st[5] != kKindShannonic || st[6] != kShR || rd64(st + 40) != shn_hash(t)) return kErrCodebook;
  const uint64_t n = rd64(st + 16);
  if (n != n_expected || rd64(st + 24) != n_chunks_of(n)) return kErrCorrupt;
  const uint64_t nc = n_chunks_of(n), S = sync_offset(n), P = payload_offset(n);
  const uint64_t total = rd64(st + 32);
  if (P > bytes || (bytes - P) / 4 < 2 || total > (bytes - P) / 4 - 2 || total >= (1ull << 32))
    return kErrCorrupt;
  int status = 0;
  for (uint64_t c = 0; c < nc; ++c) {
    const uint64_t lo = c * kChunk, hi = std::min(n, lo + kChunk);
    const uint32_t w0 = rd32(st + 64 + 4 * c), w1 = rd32(st + 64 + 4 * (c + 1));
    const uint8_t* sy = st + S + 16 * c;
    const uint64_t nbits = rd16(sy);
    if (w0 > w1 || w1 > total || nbits > 32ull * (w1 - w0) || (nbits + 31) / 32 != w1 - w0) {
      status |= kErrCorrupt;
      continue;
    }
    const uint64_t nsub = (hi - lo + kSubLen - 1) / kSubLen;
    bool bad = false;
    for (uint64_t k = 0; k < kSubstreams && !bad; ++k) {
      const uint64_t a = k == 0 ? 0 : rd16(sy + 2 * k);
      if (k >= nsub) {
        if (k > 0 && a != nbits) bad = true;
        continue;
      }
      const uint64_t b = k + 1 < nsub ? rd16(sy + 2 * (k + 1)) : nbits;
      const uint64_t s0 = lo + k * kSubLen, s1 = std::min(hi, s0 + kSubLen);
      if (a > b || b > nbits ||
          !shn_decode_substream(t, st + P + 4ull * w0, a, b, out + s0, s1 - s0))
        bad = true;
    }
    if (bad) status |= kErrCorrupt;
  }
  return status;
}

bool shn_from(int nr, const int* lo, const int* f, Shn& t) {
  if (nr < 1 || nr > kShK || lo[0] != 0 || lo[nr] != 256) return false;
  int sum = 0;
  for (int r = 0; r < nr; ++r) {
    if (lo[r + 1] <= lo[r] || f[r] < 1) return false;
    sum += f[r];
  }
  if (sum != kShL) return false;
  t.nr = nr;
  for (int r = 0; r <= nr; ++r) t.lo[r] = lo[r];
  for (int r = 0; r < nr; ++r) t.f[r] = f[r];
  shn_tables(t);
  return true;
}

// ---- [EG] Exp-Golomb over a sign/magnitude index ----------------------------------------------
// map 0 (sign-magnitude bytes, e4m3): v = (magnitude << 1) | sign; map 1 (two's complement,
// INT8): v = 2x for x >= 0 and -2x - 1 for x < 0 (zigzag).
constexpr uint8_t kKindExpGolomb = 3;

int eg_index(int byte, int map) {
  if (map == 0) return ((byte & 0x7f) << 1) | (byte >> 7);
  const int x = byte >= 128 ? byte - 256 : byte;
  return x >= 0 ? 2 * x : -2 * x - 1;
}

void eg_codes(int order, int map, uint8_t* len, uint32_t* code) {
  for (int b = 0; b < 256; ++b) {
    const uint32_t v = (uint32_t)eg_index(b, map) + (1u << order);
    int top = 0;  // bits of v + 2^k
    while ((v >> top) > 1) ++top;
    len[b] = (uint8_t)(2 * top - order + 1);  // (top - order) zeros, then top + 1 bits
    code[b] = v;
  }
}

uint64_t eg_hash(int order, int map) {
  return fnv1a({kKindExpGolomb, (uint8_t)order, (uint8_t)map});
}

struct EgDecoder {  // [EG]: count zeros, then read that many + order + 1 bits
  int order;
  int byte_of[512];  // index v -> byte (-1: no byte has it)
  EgDecoder(int order_, int map) : order(order_) {
    for (int v = 0; v < 512; ++v) byte_of[v] = -1;
    for (int b = 0; b < 256; ++b) byte_of[eg_index(b, map)] = b;
  }
  int next(BitReader& br) const {
    int zeros = 0;
    while (br.get() == 0) {
      if (br.past_end || ++zeros > 16) return -1;
    }
    if (br.past_end) return -1;
    uint32_t v = 1;
    for (int i = 0; i < zeros + order; ++i) v = (v << 1) | (uint32_t)br.get();
    if (br.past_end) return -1;
    v -= 1u << order;
    return v < 512 ? byte_of[v] : -1;
  }
};

}  // namespace

// ================================ C entry points (ctypes) ====================================
extern "C" {

// counts[256] = occurrences of each byte value in x[0..n)
void orc_histogram(const uint8_t* x, uint64_t n, uint64_t* counts) {
  for (int s = 0; s < 256; ++s) counts[s] = 0;
  for (uint64_t i = 0; i < n; ++i) counts[x[i]]++;
}

// [SSH] weights from the summed counts of the prior batches; cover_all gives every byte >= 1.
// Returns 0, or kErrArg when lmax is out of range for the alphabet.
int orc_huffman_lengths(const uint64_t* counts, int lmax, int cover_all, uint8_t* len) {
  uint64_t w[256];
  for (int s = 0; s < 256; ++s) w[s] = cover_all ? std::max<uint64_t>(counts[s], 1) : counts[s];
  return package_merge(w, lmax, len) ? 0 : kErrArg;
}

void orc_canonical_codes(const uint8_t* len, uint32_t* code) { canonical_codes(len, code); }

// [QLC] widths, area starts, rank table, and the resulting per-symbol lengths and codes.
int orc_qlc_build(const uint64_t* counts, int max_distinct, uint8_t* bits, uint16_t* start,
                  uint8_t* rank2sym, uint8_t* len, uint32_t* code) {
  Qlc q;
  if (!qlc_search(counts, max_distinct, &q)) return kErrArg;
  std::memcpy(bits, q.bits, 8);
  std::memcpy(start, q.start, sizeof q.start);
  std::memcpy(rank2sym, q.rank2sym, 256);
  qlc_codes(q, len, code);
  return 0;
}

// FNV-1a-64 of an arbitrary byte string (exposed so that tests can pin it to published vectors).
uint64_t orc_fnv1a(const uint8_t* bytes, uint64_t n) {
  return fnv1a(std::vector<uint8_t>(bytes, bytes + n));
}

// Hash that the stream header carries in place of the codebook.
// Huffman: FNV-1a-64 of [0, lmax, len[0..255]]; QLC: of [1, 11, bits[0..7], rank2sym[0..255]].
uint64_t orc_hash_huffman(int lmax, const uint8_t* len) {
  std::vector<uint8_t> b{0, (uint8_t)lmax};
  b.insert(b.end(), len, len + 256);
  return fnv1a(b);
}
uint64_t orc_hash_qlc(const uint8_t* bits, const uint8_t* rank2sym) {
  std::vector<uint8_t> b{1, (uint8_t)kQlcLmax};
  b.insert(b.end(), bits, bits + 8);
  b.insert(b.end(), rank2sym, rank2sym + 256);
  return fnv1a(b);
}

uint64_t orc_payload_offset(uint64_t n) { return payload_offset(n); }
uint64_t orc_sync_offset(uint64_t n) { return sync_offset(n); }
uint64_t orc_encode_bound(uint64_t n) { return payload_offset(n) + 4 * (n_chunks_of(n) * 1536 + 2); }

int orc_encode_huffman(int lmax, const uint8_t* len, const uint8_t* x, uint64_t n, uint8_t* out,
                       uint64_t cap, uint64_t* written) {
  uint32_t code[256];
  canonical_codes(len, code);
  Header h{0, (uint8_t)lmax, orc_hash_huffman(lmax, len)};
  return encode(h, len, code, x, n, out, cap, written);
}

int orc_decode_huffman(int lmax, const uint8_t* len, const uint8_t* stream, uint64_t bytes,
                       uint8_t* out, uint64_t n) {
  Header h{0, (uint8_t)lmax, orc_hash_huffman(lmax, len)};
  CanonicalDecoder dec(len, lmax);
  return decode(h, dec, stream, bytes, out, n);
}

int orc_encode_qlc(const uint8_t* bits, const uint16_t* start, const uint8_t* rank2sym,
                   const uint8_t* x, uint64_t n, uint8_t* out, uint64_t cap, uint64_t* written) {
  Qlc q;
  std::memcpy(q.bits, bits, 8);
  std::memcpy(q.start, start, sizeof q.start);
  std::memcpy(q.rank2sym, rank2sym, 256);
  uint8_t len[256] = {0};
  uint32_t code[256] = {0};
  qlc_codes(q, len, code);
  Header h{1, (uint8_t)kQlcLmax, orc_hash_qlc(bits, rank2sym)};
  return encode(h, len, code, x, n, out, cap, written);
}

int orc_decode_qlc(const uint8_t* bits, const uint16_t* start, const uint8_t* rank2sym,
                   const uint8_t* stream, uint64_t bytes, uint8_t* out, uint64_t n) {
  QlcDecoder dec;
  std::memcpy(dec.q.bits, bits, 8);
  std::memcpy(dec.q.start, start, sizeof dec.q.start);
  std::memcpy(dec.q.rank2sym, rank2sym, 256);
  Header h{1, (uint8_t)kQlcLmax, orc_hash_qlc(bits, rank2sym)};
  return decode(h, dec, stream, bytes, out, n);
}

// Shannon entropy of the counts, bits per symbol (fp64).
double orc_entropy(const uint64_t* counts) {
  double total = 0;
  for (int s = 0; s < 256; ++s) total += (double)counts[s];
  if (total == 0) return 0;
  double h = 0;
  for (int s = 0; s < 256; ++s)
    if (counts[s]) {
      const double p = (double)counts[s] / total;
      h -= p * std::log2(p);
    }
  return h;
}

// Mean code length in bits per symbol of data with these counts (payload bits only).
double orc_mean_length(const uint64_t* counts, const uint8_t* len) {
  double total = 0, bits = 0;
  for (int s = 0; s < 256; ++s) {
    total += (double)counts[s];
    bits += (double)counts[s] * len[s];
  }
  return total ? bits / total : 0;
}

// [SHN] builder, partition (for any alphabet size, so tests can search small ones exhaustively),
// hash, bound, encode and decode. lo: nr + 1 boundaries, f: nr frequencies (sum 128).
int orc_shannonic_build(const uint64_t* counts, int K, int cover_all, int* nr, int* lo, int* f) {
  Shn t;
  if (!counts || !nr || !lo || !f || !shn_build(counts, K, cover_all != 0, t)) return kErrArg;
  *nr = t.nr;
  for (int r = 0; r <= t.nr; ++r) lo[r] = t.lo[r];
  for (int r = 0; r < t.nr; ++r) f[r] = t.f[r];
  return 0;
}
int orc_shannonic_partition(const uint64_t* w, int n, int K, int* lo) {
  if (!w || !lo || n < 1 || K < 1) return -1;
  return partition(w, n, K, lo);
}
int orc_shannonic_normalise(const uint64_t* wr, int nr, int* f) {
  if (!wr || !f || nr < 1 || nr > kShL) return kErrArg;
  normalise(wr, nr, f);
  return 0;
}
uint64_t orc_hash_shannonic(int nr, const int* lo, const int* f) {
  Shn t;
  return shn_from(nr, lo, f, t) ? shn_hash(t) : 0;
}
uint64_t orc_shannonic_encode_bound(uint64_t n) {
  // per sub-stream at most 512 * (8 offset + 7 state) + 7 bits: 1922 words per chunk
  return payload_offset(n) + 4 * (n_chunks_of(n) * 1922 + 2);
}
int orc_encode_shannonic(int nr, const int* lo, const int* f, const uint8_t* x, uint64_t n,
                         uint8_t* out, uint64_t cap, uint64_t* written) {
  Shn t;
  if (!shn_from(nr, lo, f, t)) return kErrArg;
  return shn_encode(t, x, n, out, cap, written);
}
int orc_decode_shannonic(int nr, const int* lo, const int* f, const uint8_t* stream,
                         uint64_t bytes, uint8_t* out, uint64_t n) {
  Shn t;
  if (!shn_from(nr, lo, f, t)) return kErrArg;
  return shn_decode(t, stream, bytes, out, n);
}

// [EG] per-byte code words, hash, encode and decode.
int orc_expgolomb_codes(int order, int map, uint8_t* len, uint32_t* code) {
  if (order < 0 || order > 8 || (map != 0 && map != 1) || !len || !code) return kErrArg;
  eg_codes(order, map, len, code);
  return 0;
}
uint64_t orc_hash_expgolomb(int order, int map) { return eg_hash(order, map); }
int orc_encode_expgolomb(int order, int map, const uint8_t* x, uint64_t n, uint8_t* out,
                         uint64_t cap, uint64_t* written) {
  uint8_t len[256];
  uint32_t code[256];
  if (orc_expgolomb_codes(order, map, len, code)) return kErrArg;
  Header h{kKindExpGolomb, (uint8_t)order, eg_hash(order, map)};
  return encode(h, len, code, x, n, out, cap, written);
}
int orc_decode_expgolomb(int order, int map, const uint8_t* stream, uint64_t bytes, uint8_t* out,
                         uint64_t n) {
  if (order < 0 || order > 8 || (map != 0 && map != 1)) return kErrArg;
  Header h{kKindExpGolomb, (uint8_t)order, eg_hash(order, map)};
  EgDecoder dec(order, map);
  return decode(h, dec, stream, bytes, out, n);
}

}  // extern "C"
