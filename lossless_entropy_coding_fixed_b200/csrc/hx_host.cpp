// Host side of the hx library: codebook construction (package-merge, canonical codes, the QLC
// area search), the codebook hash and the device table block. Runs on the CPU, off the data
// path: "Single-Stage Huffman Encoder for ML Compression" (abstract) builds the codebook once
// from earlier batches, so nothing here sits between a batch and its coded stream.
#include <algorithm>
#include <cmath>
#include <cstddef>
#include <cstring>
#include <vector>

#include "hx.h"
#include "hx_tables.h"

namespace {

constexpr uint64_t kFnvBasis = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

uint64_t fnv1a_update(uint64_t h, const uint8_t* p, size_t n) {
  for (size_t i = 0; i < n; ++i) h = (h ^ p[i]) * kFnvPrime;
  return h;
}

// ---- package-merge (Larmore & Hirschberg 1990) ------------------------------------------
// Items live in a node pool: a leaf names its symbol, a package names its two parts. The
// selected items are expanded once at the end to count how often each leaf appears.
struct PmNode {
  uint64_t weight;
  int symbol;  // >= 0 for a leaf
  int part0, part1;
};

bool lengths_by_package_merge(const uint64_t w[256], int lmax, uint8_t len[256]) {
  std::memset(len, 0, 256);
  // leaves first (pool[0..m)), then each row's packages; a row holds at most 2m - 1 <= 511 items
  constexpr int kPool = 256 + (HX_LMAX_MAX - 1) * 256;
  std::vector<PmNode> pool;
  pool.reserve(kPool);
  int leaves[256];
  size_t m = 0;
  for (int s = 0; s < 256; ++s)
    if (w[s]) {
      leaves[m++] = (int)pool.size();
      pool.push_back({w[s], s, -1, -1});
    }
  if (m == 0) return true;
  if (m == 1) {
    len[pool[leaves[0]].symbol] = 1;
    return true;
  }
  if (lmax < 1 || lmax > HX_LMAX_MAX || (size_t(1) << lmax) < m) return false;
  std::stable_sort(leaves, leaves + m,
                   [&](int a, int b) { return pool[a].weight < pool[b].weight; });
  int rows[2][512];
  int* row = rows[0];
  int* next = rows[1];
  size_t nrow = m;
  std::copy(leaves, leaves + m, row);
  for (int depth = 1; depth < lmax; ++depth) {
    // this row's packages, in order; then merge them with the leaves (a leaf first on a tie)
    const size_t npk = nrow / 2, first = pool.size();
    for (size_t i = 0; i < npk; ++i) {
      const int a = row[2 * i], b = row[2 * i + 1];
      pool.push_back({pool[a].weight + pool[b].weight, -1, a, b});
    }
    size_t li = 0, pi = 0, k = 0;
    while (li < m || pi < npk) {
      const bool take_leaf =
          pi == npk || (li < m && pool[leaves[li]].weight <= pool[first + pi].weight);
      next[k++] = take_leaf ? leaves[li++] : (int)(first + pi++);
    }
    std::swap(row, next);
    nrow = k;
  }
  // the first 2m - 2 items of the top row; a leaf's length is how often it occurs in them
  int stack[2 * HX_LMAX_MAX + 2];
  for (size_t i = 0; i < 2 * m - 2; ++i) {
    int sp = 0;
    stack[sp++] = row[i];
    while (sp) {
      const PmNode& nd = pool[stack[--sp]];
      if (nd.symbol >= 0) {
        len[nd.symbol]++;
      } else {
        stack[sp++] = nd.part0;
        stack[sp++] = nd.part1;
      }
    }
  }
  return true;
}

// Canonical code words from lengths, RFC 1951 section 3.2.2: shorter codes first, and within
// one length in increasing symbol order.
void canonical(const uint8_t len[256], uint16_t code[256]) {
  uint32_t per_len[HX_LMAX_MAX + 1] = {0};
  for (int s = 0; s < 256; ++s)
    if (len[s]) per_len[len[s]]++;
  uint32_t first[HX_LMAX_MAX + 1] = {0};
  uint32_t v = 0;
  for (int l = 1; l <= HX_LMAX_MAX; ++l) {
    v = (v + per_len[l - 1]) << 1;
    first[l] = v;
  }
  for (int s = 0; s < 256; ++s) code[s] = len[s] ? (uint16_t)first[len[s]]++ : 0;
}

// ---- QLC area search -------------------------------------------------------------------
struct QlcSearch {
  unsigned __int128 prefix[257];  // prefix[r] = total weight of ranks < r
  int max_distinct;
  int cur[8];
  int best[8];
  bool found = false;
  unsigned __int128 best_cost = 0;

  // Width vectors are visited depth-first with non-decreasing widths: lexicographic order, so
  // the first vector reaching the minimum is the smallest one.
  void visit(int area, int min_width, int distinct, int covered, unsigned __int128 cost) {
    // costs only grow along a path, and a later vector of equal cost never replaces the best
    if (found && cost >= best_cost) return;
    if (covered == 256 && area < 8) {
      // every completion costs the same; the smallest repeats the last width (no new value)
      for (int a = area; a < 8; ++a) cur[a] = min_width;
      area = 8;
    }
    if (area == 8) {
      if (covered == 256 && (!found || cost < best_cost)) {
        found = true;
        best_cost = cost;
        std::memcpy(best, cur, sizeof cur);
      }
      return;
    }
    for (int b = min_width; b <= 8; ++b) {
      const int d = distinct + ((area == 0 || b != cur[area - 1]) ? 1 : 0);
      if (d > max_distinct) continue;
      const int take = std::min(1 << b, 256 - covered);
      cur[area] = b;
      visit(area + 1, b, d, covered + take,
            cost + (prefix[covered + take] - prefix[covered]) * (unsigned)(3 + b));
    }
  }
};

int fill_qlc(const uint64_t counts[256], int max_distinct, hx_codebook* out) {
  int rank[256];
  for (int s = 0; s < 256; ++s) rank[s] = s;
  std::stable_sort(rank, rank + 256, [&](int a, int b) { return counts[a] > counts[b]; });
  QlcSearch q;
  q.max_distinct = max_distinct;
  q.prefix[0] = 0;
  for (int r = 0; r < 256; ++r) q.prefix[r + 1] = q.prefix[r] + counts[rank[r]];
  q.visit(0, 0, 0, 0, 0);
  if (!q.found) return HX_ERR_ARG;
  std::memset(out, 0, sizeof *out);
  out->kind = HX_KIND_QLC;
  out->lmax = HX_QLC_LMAX;
  int r = 0;
  for (int a = 0; a < 8; ++a) {
    out->qlc_bits[a] = (uint8_t)q.best[a];
    out->qlc_start[a] = (uint16_t)r;
    const int take = std::min(1 << q.best[a], 256 - r);
    for (int i = 0; i < take; ++i, ++r) {
      const int s = rank[r];
      out->len[s] = (uint8_t)(3 + q.best[a]);
      out->code[s] = (uint16_t)((a << q.best[a]) | i);
    }
  }
  out->qlc_start[8] = (uint16_t)r;
  for (int i = 0; i < 256; ++i) out->rank2sym[i] = (uint8_t)rank[i];
  const uint8_t head[2] = {HX_KIND_QLC, HX_QLC_LMAX};
  uint64_t h = fnv1a_update(kFnvBasis, head, 2);
  h = fnv1a_update(h, out->qlc_bits, 8);
  out->hash = fnv1a_update(h, out->rank2sym, 256);
  return HX_OK;
}

// ---- Shannonic: range partition + 128-state tANS (the review page's method) ------------------
constexpr int kShR = HX_SHN_R, kShL = HX_SHN_L, kShK = HX_SHN_K;
constexpr int kShStep = kShL / 2 + kShL / 8 + 3;  // 83: odd, so it visits every state

int bits_for(int size) {  // ceil(log2 size)
  int b = 0;
  while ((1 << b) < size) ++b;
  return b;
}

// Minimal sum over ranges of W_r log2(W / W_r) + W_r ceil(log2 size_r), over partitions of the
// 256 values into at most K contiguous ranges. best[k][b]: the first b values in k ranges; the
// split point and range count are the smallest reaching the strict minimum.
int shannonic_partition(const uint64_t w[256], int K, uint16_t lo[kShK + 1]) {
  uint64_t pre[257];
  pre[0] = 0;
  for (int v = 0; v < 256; ++v) pre[v + 1] = pre[v] + w[v];
  const double W = (double)pre[256];
  auto cost = [&](int a, int b) -> double {
    const uint64_t wab = pre[b] - pre[a];
    if (wab == 0) return 0.0;
    return (double)wab * std::log2(W / (double)wab) + (double)wab * (double)bits_for(b - a);
  };
  static thread_local double best[kShK + 1][257];
  static thread_local int split[kShK + 1][257];
  for (int b = 1; b <= 256; ++b) {
    best[1][b] = cost(0, b);
    split[1][b] = 0;
  }
  for (int k = 2; k <= K; ++k)
    for (int b = k; b <= 256; ++b) {
      best[k][b] = 1e300;
      split[k][b] = -1;
      for (int a = k - 1; a < b; ++a) {
        const double c = best[k - 1][a] + cost(a, b);
        if (c < best[k][b]) {
          best[k][b] = c;
          split[k][b] = a;
        }
      }
    }
  int kk = 1;
  for (int k = 2; k <= K; ++k)
    if (best[k][256] < best[kk][256]) kk = k;
  int b = 256;
  for (int k = kk; k >= 1; --k) {
    lo[k] = (uint16_t)b;
    b = split[k][b];
  }
  lo[0] = 0;
  return kk;
}

// tANS frequencies summing to 128 from the ranges' weights.
void shannonic_frequencies(const uint64_t* wr, int nr, uint8_t* f) {
  uint64_t W = 0;
  for (int r = 0; r < nr; ++r) W += wr[r];
  int fi[kShK], sum = 0;
  uint64_t rem[kShK];
  for (int r = 0; r < nr; ++r) {
    const uint64_t q = wr[r] * (uint64_t)kShL / W;
    rem[r] = wr[r] * (uint64_t)kShL - q * W;
    fi[r] = q > 0 ? (int)q : 1;
    sum += fi[r];
  }
  if (sum < kShL) {
    int order[kShK];
    for (int r = 0; r < nr; ++r) order[r] = r;
    std::stable_sort(order, order + nr, [&](int a, int b) { return rem[a] > rem[b]; });
    for (int i = 0; sum < kShL; i = (i + 1) % nr, ++sum) ++fi[order[i]];
  }
  while (sum > kShL) {
    int big = -1;
    for (int r = 0; r < nr; ++r)
      if (fi[r] > 1 && (big < 0 || fi[r] > fi[big])) big = r;
    --fi[big];
    --sum;
  }
  for (int r = 0; r < nr; ++r) f[r] = (uint8_t)fi[r];
}

uint64_t shannonic_hash(const hx_codebook& cb) {
  uint8_t bytes[3 + 2 * kShK];
  size_t n = 0;
  bytes[n++] = HX_KIND_SHANNONIC;
  bytes[n++] = (uint8_t)kShR;
  bytes[n++] = cb.sh_nr;
  for (int r = 1; r < cb.sh_nr; ++r) bytes[n++] = (uint8_t)cb.sh_lo[r];
  for (int r = 0; r < cb.sh_nr; ++r) bytes[n++] = cb.sh_f[r];
  return fnv1a_update(kFnvBasis, bytes, n);
}

bool shannonic_valid(const hx_codebook& cb) {
  if (cb.sh_nr < 1 || cb.sh_nr > kShK || cb.sh_lo[0] != 0 || cb.sh_lo[cb.sh_nr] != 256)
    return false;
  int sum = 0;
  for (int r = 0; r < cb.sh_nr; ++r) {
    if (cb.sh_lo[r + 1] <= cb.sh_lo[r] || cb.sh_f[r] < 1) return false;
    sum += cb.sh_f[r];
  }
  return sum == kShL;
}

int shannonic_tables(const hx_codebook& cb, hx::Tables* t) {
  if (!shannonic_valid(cb)) return HX_ERR_ARG;
  const int nr = cb.sh_nr;
  int spread[kShL];
  for (int r = 0, pos = 0; r < nr; ++r)
    for (int j = 0; j < cb.sh_f[r]; ++j) {
      spread[pos] = r;
      pos = (pos + kShStep) % kShL;
    }
  int cum[kShK + 1];
  cum[0] = 0;
  for (int r = 0; r < nr; ++r) cum[r + 1] = cum[r] + cb.sh_f[r];
  int seen[kShK] = {0};
  for (int u = 0; u < kShL; ++u) {
    const int r = spread[u];
    const int xs = cb.sh_f[r] + seen[r];  // the seen[r]-th state of range r
    t->sh_enc[cum[r] + seen[r]] = (uint8_t)(kShL + u);
    ++seen[r];
    int lg = 0;
    while ((2 << lg) <= xs) ++lg;
    const int nb = kShR - lg;
    const int size = cb.sh_lo[r + 1] - cb.sh_lo[r];
    const int tot = nb + bits_for(size);
    t->sh_dec[u][0] = (1u << tot) - 1u;
    t->sh_dec[u][1] = (uint32_t)tot;
    t->sh_dec[u][2] = (uint32_t)nb | ((uint32_t)(xs << nb) << 16);
    t->sh_dec[u][3] = (uint32_t)cb.sh_lo[r] | ((uint32_t)(0x8000 - size) << 16);
  }
  for (int r = 0; r < nr; ++r) {
    int lg = 0;
    while ((2 << lg) <= cb.sh_f[r]) ++lg;
    const int k = kShR - lg, f = cb.sh_f[r];
    const int size = cb.sh_lo[r + 1] - cb.sh_lo[r], ob = bits_for(size);
    // (k << 8) - (f << k) + 256 ob lies in [-255, 3840): stored as 12 bits, two's complement
    const uint32_t key = (uint32_t)((k << 8) - (f << k) + 256 * ob) & 0xfffu;
    for (int v = cb.sh_lo[r]; v < cb.sh_lo[r + 1]; ++v) {
      t->sh_sym[v] = (uint32_t)ob | ((uint32_t)(cum[r] - f + 128) << 8) | (key << 20);
      t->sh_off[v] = (uint8_t)(v - cb.sh_lo[r]);
    }
  }
  return HX_OK;
}

}  // namespace

extern "C" {

int hx_build_codebook(const uint64_t* counts, int lmax, uint32_t flags, hx_codebook* out) {
  if (!counts || !out || (flags & ~(uint32_t)HX_CB_SEEN_ONLY)) return HX_ERR_ARG;
  uint64_t w[256];
  for (int s = 0; s < 256; ++s)
    w[s] = (flags & HX_CB_SEEN_ONLY) ? counts[s] : std::max<uint64_t>(counts[s], 1);
  hx_codebook cb;
  std::memset(&cb, 0, sizeof cb);
  if (!lengths_by_package_merge(w, lmax, cb.len)) return HX_ERR_ARG;
  cb.kind = HX_KIND_HUFFMAN;
  cb.lmax = (uint8_t)lmax;
  canonical(cb.len, cb.code);
  const uint8_t head[2] = {HX_KIND_HUFFMAN, (uint8_t)lmax};
  cb.hash = fnv1a_update(fnv1a_update(kFnvBasis, head, 2), cb.len, 256);
  *out = cb;
  return HX_OK;
}

int hx_qlc_build(const uint64_t* counts, int max_distinct, uint32_t flags, hx_codebook* out) {
  if (!counts || !out || flags || max_distinct < 1 || max_distinct > 8) return HX_ERR_ARG;
  return fill_qlc(counts, max_distinct, out);
}

int hx_expgolomb_build(int order, int map, hx_codebook* out) {
  if (!out || order < 5 || order > 8 || (map != 0 && map != 1)) return HX_ERR_ARG;
  hx_codebook cb;
  std::memset(&cb, 0, sizeof cb);
  cb.kind = HX_KIND_EXPGOLOMB;
  cb.lmax = (uint8_t)order;
  for (int b = 0; b < 256; ++b) {
    int v;
    if (map == 0) {
      v = ((b & 0x7f) << 1) | (b >> 7);
    } else {
      const int x = (int)(int8_t)(uint8_t)b;
      v = x >= 0 ? 2 * x : -2 * x - 1;
    }
    const uint32_t w = (uint32_t)v + (1u << order);  // written after (bits of w) - order - 1 zeros
    int top = 0;
    while ((w >> (top + 1)) != 0) ++top;
    cb.len[b] = (uint8_t)(2 * top - order + 1);
    cb.code[b] = (uint16_t)w;
  }
  const uint8_t bytes[3] = {HX_KIND_EXPGOLOMB, (uint8_t)order, (uint8_t)map};
  cb.hash = fnv1a_update(kFnvBasis, bytes, 3);
  *out = cb;
  return HX_OK;
}

int hx_shannonic_build(const uint64_t* counts, int K, uint32_t flags, hx_codebook* out) {
  if (!counts || !out || flags || K < 1 || K > kShK) return HX_ERR_ARG;
  uint64_t w[256];
  for (int v = 0; v < 256; ++v) w[v] = std::max<uint64_t>(counts[v], 1);
  hx_codebook cb;
  std::memset(&cb, 0, sizeof cb);
  cb.kind = HX_KIND_SHANNONIC;
  cb.lmax = (uint8_t)kShR;
  cb.sh_nr = (uint8_t)shannonic_partition(w, K, cb.sh_lo);
  uint64_t wr[kShK] = {0};
  for (int r = 0; r < cb.sh_nr; ++r)
    for (int v = cb.sh_lo[r]; v < cb.sh_lo[r + 1]; ++v) wr[r] += w[v];
  shannonic_frequencies(wr, cb.sh_nr, cb.sh_f);
  cb.hash = shannonic_hash(cb);
  *out = cb;
  return HX_OK;
}

uint64_t hx_shannonic_encode_bound(uint64_t n) {
  const uint64_t chunks = (n + HX_CHUNK - 1) / HX_CHUNK;
  // a sub-stream: at most 512 symbols of 8 offset + 7 state bits, then 7 bits of final state
  const uint64_t words = (HX_SUBSTREAMS * (512 * 15 + 7) + 31) / 32;
  return hx_payload_offset(n) + 4 * (chunks * words + 2);
}

int hx_codebook_tables(const hx_codebook* cb, void* host_tables) {
  if (!cb || !host_tables) return HX_ERR_ARG;
  if (cb->kind != HX_KIND_HUFFMAN && cb->kind != HX_KIND_QLC && cb->kind != HX_KIND_SHANNONIC &&
      cb->kind != HX_KIND_EXPGOLOMB)
    return HX_ERR_ARG;
  std::memset(host_tables, 0, HX_TABLES_BYTES);
  hx::Tables* t = static_cast<hx::Tables*>(host_tables);
  if (cb->kind == HX_KIND_SHANNONIC) {
    const int rc = shannonic_tables(*cb, t);
    if (rc) return rc;
    t->complete = 0;
    t->kind = cb->kind;
    t->lmax = cb->lmax;
    t->magic = hx::kTablesMagic;
    t->hash = cb->hash;
    return HX_OK;
  }
  for (int s = 0; s < 256; ++s) {
    const int l = cb->len[s];
    if (l > HX_LMAX_MAX || (l && (cb->code[s] >> l))) return HX_ERR_ARG;
    t->enc[s] = ((uint32_t)cb->code[s] << 4) | (uint32_t)l;
    if (!l) continue;
    const uint32_t lo = (uint32_t)cb->code[s] << (HX_LMAX_MAX - l);
    const uint32_t hi = lo + (1u << (HX_LMAX_MAX - l));
    for (uint32_t wv = lo; wv < hi; ++wv) {
      if (t->dec[wv]) return HX_ERR_ARG;  // not a prefix code
      t->dec[wv] = (uint16_t)((s << 8) | hx::kDecValid | l);
    }
  }
  if (cb->kind == HX_KIND_QLC) {
    std::memcpy(t->rank2sym, cb->rank2sym, 256);
    for (int a = 0; a < 8; ++a) {
      const uint32_t first = cb->qlc_start[a], fill = cb->qlc_start[a + 1] - cb->qlc_start[a];
      if (cb->qlc_bits[a] > 8 || cb->qlc_start[a + 1] < cb->qlc_start[a] ||
          fill > (1u << cb->qlc_bits[a]))
        return HX_ERR_ARG;
      t->qlc_area[a] = first | (fill << 9) | ((uint32_t)cb->qlc_bits[a] << 18);
      t->qlc_bits_packed |= (uint32_t)cb->qlc_bits[a] << (4 * a);
    }
  }
  t->complete = 1;
  for (int wv = 0; wv < 4096; ++wv)
    if (!t->dec[wv]) t->complete = 0;
  t->kind = cb->kind;
  t->lmax = cb->lmax;
  t->magic = hx::kTablesMagic;
  t->hash = cb->hash;
  return HX_OK;
}

uint64_t hx_sync_offset(uint64_t n) {
  const uint64_t chunks = (n + HX_CHUNK - 1) / HX_CHUNK;
  return (64 + 4 * (chunks + 1) + 15) / 16 * 16;
}

uint64_t hx_payload_offset(uint64_t n) {
  return hx_sync_offset(n) + 16 * ((n + HX_CHUNK - 1) / HX_CHUNK);
}

uint64_t hx_encode_bound(uint64_t n) {
  const uint64_t chunks = (n + HX_CHUNK - 1) / HX_CHUNK;
  return hx_payload_offset(n) + 4 * (chunks * (HX_CHUNK * HX_LMAX_MAX / 32) + 2);
}

double hx_entropy(const uint64_t* counts) {
  if (!counts) return -1;
  long double total = 0;
  for (int s = 0; s < 256; ++s) total += counts[s];
  if (total == 0) return 0;
  double h = 0;
  for (int s = 0; s < 256; ++s)
    if (counts[s]) {
      const double p = (double)(counts[s] / total);
      h -= p * std::log2(p);
    }
  return h;
}

double hx_mean_length(const uint64_t* counts, const hx_codebook* cb) {
  if (!counts || !cb) return -1;
  long double total = 0, bits = 0;
  if (cb->kind == HX_KIND_SHANNONIC) {  // tANS codes range r in log2(128 / f_r) bits on average
    if (!shannonic_valid(*cb)) return -1;
    for (int r = 0; r < cb->sh_nr; ++r) {
      const double len = std::log2((double)kShL / cb->sh_f[r]) +
                         bits_for(cb->sh_lo[r + 1] - cb->sh_lo[r]);
      for (int s = cb->sh_lo[r]; s < cb->sh_lo[r + 1]; ++s) {
        total += counts[s];
        bits += (long double)counts[s] * len;
      }
    }
    return total == 0 ? 0 : (double)(bits / total);
  }
  for (int s = 0; s < 256; ++s) {
    total += counts[s];
    bits += (long double)counts[s] * cb->len[s];
  }
  return total == 0 ? 0 : (double)(bits / total);
}

int hx_version(void) { return 1; }

const char* hx_status_string(int code) {
  switch (code) {
    case HX_OK: return "ok";
    case HX_ERR_ARG: return "invalid argument";
    case HX_ERR_CUDA: return "CUDA error";
    case HX_ERR_UNCODABLE: return "input byte without a code word";
    case HX_ERR_CORRUPT: return "corrupt stream";
    case HX_ERR_CODEBOOK: return "stream written with another codebook";
    case HX_ERR_TIMEOUT: return "a bounded device wait ran out";
    case HX_ERR_CAPACITY: return "output buffer too small";
    default: return "several errors (bit set)";
  }
}

}  // extern "C"
