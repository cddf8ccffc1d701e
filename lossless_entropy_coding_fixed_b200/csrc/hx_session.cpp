// Online single-stage loop: the planner (host bookkeeping, no device) and the session that runs
// it around the device encoder and decoder.
//
// "Single-Stage Huffman Encoder for ML Compression" (abstract): the codebook for a batch comes
// from the average distribution of earlier batches, so no frequency pass or codebook build sits
// on the data path. Here the earlier batches' histograms are the encoder's own fused histograms;
// batch t is coded with the codebook of the histograms of batches t - lag - m + 1 .. t - lag, so
// the host rebuilds while the device codes the batches in between, and the schedule does not
// depend on timing. "Shannonic" (the review of the range-partitioned coder): the codebook is
// rebuilt when the data drifts away from it -- here, when a batch's coded length exceeds its own
// entropy by more than a set fraction, the history restarts from that batch.
#include <cuda_runtime.h>

#include <cmath>
#include <condition_variable>
#include <cstring>
#include <deque>
#include <limits>
#include <map>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#include "hx.h"

struct hx_planner {
  hx_session_config cfg;
  uint64_t initial[256];
  std::deque<std::vector<uint64_t>> history;  // observed batches, oldest first (at most m)
  uint64_t next_obs = 0;                       // next batch to observe
  std::map<uint64_t, hx_codebook> issued;      // codebooks handed out, not yet observed
  bool cached = false;                         // `current` matches the history
  hx_codebook current;
};

// The session's host work (waiting for a batch's histogram, folding it into the plan, building
// and packing the next codebook) runs on a worker thread, so the calling thread only enqueues
// device work; hx_session_encode(t) waits only if batch t's codebook is not ready yet.
struct hx_session {
  hx_planner plan;  // the worker's
  int device = 0;
  void* slots[HX_MAX_TABLE_SET];        // device table blocks (caller's memory)
  uint64_t slot_hash[HX_MAX_TABLE_SET];  // 0 = empty
  uint32_t nslots = 0, cur = 0;
  unsigned char* staging = nullptr;     // pinned: one table block per slot
  uint32_t* hist_host = nullptr;        // pinned: lag + 1 histograms in flight
  cudaEvent_t* events = nullptr;        // one per in-flight histogram
  uint32_t ring = 0;                    // lag + 1
  uint64_t batch = 0;                   // next batch to encode (caller's thread)

  struct Ready {
    hx_codebook cb;
    std::vector<unsigned char> tables;
  };
  std::mutex mu;
  std::condition_variable cv;
  uint64_t enqueued = 0;             // batches whose histogram copy is enqueued
  uint64_t folded = 0;               // batches the worker has folded
  std::map<uint64_t, Ready> ready;   // codebooks built for batches not yet encoded
  std::vector<hx_batch_info> info;
  int error = HX_OK;                 // first error of the worker
  bool stop = false;
  std::thread worker;
};

namespace {

int check_config(const hx_session_config* c) {
  if (!c) return HX_ERR_ARG;
  if (c->kind != HX_KIND_HUFFMAN && c->kind != HX_KIND_QLC) return HX_ERR_ARG;
  if (c->kind == HX_KIND_HUFFMAN && (c->lmax > HX_LMAX_MAX || (c->flags & ~HX_CB_SEEN_ONLY)))
    return HX_ERR_ARG;
  if (c->kind == HX_KIND_QLC && (c->max_distinct > 8 || c->flags)) return HX_ERR_ARG;
  if (c->history < 1 || c->history > 64 || c->lag < 1 || c->lag > 8) return HX_ERR_ARG;
  if (std::isnan(c->drift)) return HX_ERR_ARG;
  return HX_OK;
}

int build(const hx_session_config& c, const uint64_t* counts, hx_codebook* out) {
  if (c.kind == HX_KIND_HUFFMAN)
    return hx_build_codebook(counts, c.lmax ? (int)c.lmax : HX_LMAX_MAX, c.flags, out);
  return hx_qlc_build(counts, c.max_distinct ? (int)c.max_distinct : 4, 0, out);
}

int planner_init(hx_planner* p, const hx_session_config* cfg, const uint64_t* initial) {
  const int rc = check_config(cfg);
  if (rc) return rc;
  p->cfg = *cfg;
  for (int s = 0; s < 256; ++s) p->initial[s] = initial ? initial[s] : 1;
  return HX_OK;
}

int planner_codebook(hx_planner* p, uint64_t t, hx_codebook* out) {
  // every batch up to t - lag must have been observed, and none after it
  const uint64_t need = t + 1 > p->cfg.lag ? t + 1 - p->cfg.lag : 0;
  if (p->next_obs != need) return HX_ERR_ARG;
  if (!p->cached) {
    uint64_t sum[256] = {0};
    if (p->history.empty()) {
      std::memcpy(sum, p->initial, sizeof sum);
    } else {
      for (const auto& h : p->history)
        for (int s = 0; s < 256; ++s) sum[s] += h[s];
    }
    const int rc = build(p->cfg, sum, &p->current);
    if (rc) return rc;
    p->cached = true;
  }
  p->issued[t] = p->current;
  *out = p->current;
  return HX_OK;
}

int planner_observe(hx_planner* p, uint64_t j, const uint64_t* counts, int* refreshed,
                    double* drift) {
  if (!counts || j != p->next_obs) return HX_ERR_ARG;
  double d = std::numeric_limits<double>::quiet_NaN();
  bool refresh = false;
  auto it = p->issued.find(j);
  if (it != p->issued.end()) {
    const double H = hx_entropy(counts);
    if (H > 0) {
      d = hx_mean_length(counts, &it->second) / H - 1.0;
      refresh = p->cfg.drift > 0 && d > p->cfg.drift;
    }
    p->issued.erase(it);
  }
  if (refresh) p->history.clear();
  p->history.emplace_back(counts, counts + 256);
  while (p->history.size() > p->cfg.history) p->history.pop_front();
  p->cached = false;
  ++p->next_obs;
  if (refreshed) *refreshed = refresh ? 1 : 0;
  if (drift) *drift = d;
  return HX_OK;
}

// Worker: builds and packs the codebook of batch t into the ready map.
int session_prepare(hx_session* s, uint64_t t) {
  hx_session::Ready r;
  int rc = planner_codebook(&s->plan, t, &r.cb);
  if (rc) return rc;
  r.tables.resize(HX_TABLES_BYTES);
  rc = hx_codebook_tables(&r.cb, r.tables.data());
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(s->mu);
  s->ready.emplace(t, std::move(r));
  return HX_OK;
}

// Worker: folds the histogram of batch j (its copy to pinned memory has been enqueued).
int session_fold(hx_session* s, uint64_t j) {
  const uint32_t r = (uint32_t)(j % s->ring);
  if (cudaEventSynchronize(s->events[r]) != cudaSuccess) return HX_ERR_CUDA;
  uint64_t counts[256];
  uint64_t total = 0;
  for (int v = 0; v < 256; ++v) total += counts[v] = s->hist_host[r * 256 + v];
  int refreshed = 0;
  double drift = 0;
  const int rc = planner_observe(&s->plan, j, counts, &refreshed, &drift);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(s->mu);
  hx_batch_info& b = s->info[j];
  b.observed = 1;
  b.refreshed = refreshed;
  b.drift = drift;
  b.symbols = total;
  return HX_OK;
}

void session_worker(hx_session* s) {
  cudaSetDevice(s->device);
  int rc = HX_OK;
  // batches 0 .. lag-1 are coded before any histogram is back
  for (uint64_t t = 0; t < s->plan.cfg.lag && rc == HX_OK; ++t) rc = session_prepare(s, t);
  for (uint64_t j = 0; rc == HX_OK; ++j) {
    {
      std::unique_lock<std::mutex> lock(s->mu);
      s->cv.notify_all();
      s->cv.wait(lock, [&] { return s->enqueued > j || s->stop; });
      if (s->enqueued <= j) break;  // stopped with nothing left to fold
    }
    rc = session_fold(s, j);
    if (rc == HX_OK) rc = session_prepare(s, j + s->plan.cfg.lag);
    std::lock_guard<std::mutex> lock(s->mu);
    s->folded = j + 1;
  }
  std::lock_guard<std::mutex> lock(s->mu);
  if (rc != HX_OK && s->error == HX_OK) s->error = rc;
  s->stop = true;
  s->cv.notify_all();
}

void session_free(hx_session* s) {
  if (s->worker.joinable()) {
    {
      std::lock_guard<std::mutex> lock(s->mu);
      s->stop = true;
    }
    s->cv.notify_all();
    s->worker.join();
  }
  if (s->events)
    for (uint32_t i = 0; i < s->ring; ++i)
      if (s->events[i]) cudaEventDestroy(s->events[i]);
  delete[] s->events;
  if (s->staging) cudaFreeHost(s->staging);
  if (s->hist_host) cudaFreeHost(s->hist_host);
  delete s;
}

}  // namespace

extern "C" {

int hx_planner_create(const hx_session_config* cfg, const uint64_t* initial_counts,
                      hx_planner** out) {
  if (!out) return HX_ERR_ARG;
  *out = nullptr;
  hx_planner* p = new (std::nothrow) hx_planner();
  if (!p) return HX_ERR_ARG;
  const int rc = planner_init(p, cfg, initial_counts);
  if (rc) {
    delete p;
    return rc;
  }
  *out = p;
  return HX_OK;
}

int hx_planner_codebook(hx_planner* p, uint64_t batch, hx_codebook* out) {
  if (!p || !out) return HX_ERR_ARG;
  return planner_codebook(p, batch, out);
}

int hx_planner_observe(hx_planner* p, uint64_t batch, const uint64_t* counts, int* refreshed,
                       double* drift) {
  if (!p) return HX_ERR_ARG;
  return planner_observe(p, batch, counts, refreshed, drift);
}

void hx_planner_destroy(hx_planner* p) { delete p; }

int hx_session_create(const hx_session_config* cfg, const uint64_t* initial_counts,
                      void* const* d_slots, uint32_t n_slots, hx_session** out) {
  if (!out) return HX_ERR_ARG;
  *out = nullptr;
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!d_slots || n_slots < cfg->lag + 1 || n_slots > HX_MAX_TABLE_SET) return HX_ERR_ARG;
  for (uint32_t i = 0; i < n_slots; ++i)
    if (!d_slots[i] || (reinterpret_cast<uintptr_t>(d_slots[i]) & 15)) return HX_ERR_ARG;
  hx_session* s = new (std::nothrow) hx_session();
  if (!s) return HX_ERR_ARG;
  rc = planner_init(&s->plan, cfg, initial_counts);
  if (rc) {
    delete s;
    return rc;
  }
  s->nslots = n_slots;
  for (uint32_t i = 0; i < n_slots; ++i) {
    s->slots[i] = d_slots[i];
    s->slot_hash[i] = 0;
  }
  s->ring = cfg->lag + 1;
  s->events = new (std::nothrow) cudaEvent_t[s->ring]();
  if (!s->events ||
      cudaMallocHost(reinterpret_cast<void**>(&s->staging), (size_t)n_slots * HX_TABLES_BYTES) !=
          cudaSuccess ||
      cudaMallocHost(reinterpret_cast<void**>(&s->hist_host), (size_t)s->ring * 256 * 4) !=
          cudaSuccess) {
    session_free(s);
    return HX_ERR_CUDA;
  }
  for (uint32_t i = 0; i < s->ring; ++i)
    if (cudaEventCreateWithFlags(&s->events[i], cudaEventDisableTiming) != cudaSuccess) {
      session_free(s);
      return HX_ERR_CUDA;
    }
  // no slot holds a table yet: a zeroed block is never picked by hx_decode_set
  for (uint32_t i = 0; i < n_slots; ++i)
    if (cudaMemset(d_slots[i], 0, HX_TABLES_BYTES) != cudaSuccess) {
      session_free(s);
      return HX_ERR_CUDA;
    }
  if (cudaGetDevice(&s->device) != cudaSuccess) {
    session_free(s);
    return HX_ERR_CUDA;
  }
  try {
    s->worker = std::thread(session_worker, s);
  } catch (...) {
    session_free(s);
    return HX_ERR_ARG;
  }
  *out = s;
  return HX_OK;
}

void hx_session_destroy(hx_session* s) {
  if (s) session_free(s);
}

int hx_session_encode(hx_session* s, const uint8_t* d_in, uint64_t n, void* d_out,
                      uint64_t out_cap, void* d_scratch, uint32_t* d_hist, uint32_t* d_status,
                      void* stream) {
  if (!s || !d_hist) return HX_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint64_t t = s->batch;
  // 1. batch t's codebook, built by the worker from the histograms up to batch t - lag
  hx_session::Ready r;
  {
    std::unique_lock<std::mutex> lock(s->mu);
    s->cv.wait(lock, [&] { return s->ready.count(t) || s->stop; });
    auto it = s->ready.find(t);
    if (it == s->ready.end()) return s->error ? s->error : HX_ERR_ARG;
    r = std::move(it->second);
    s->ready.erase(it);
  }
  // 2. uploaded to the next slot when it changed
  int rc;
  if (s->slot_hash[s->cur] != r.cb.hash) {
    const uint32_t next = s->slot_hash[s->cur] == 0 ? s->cur : (s->cur + 1) % s->nslots;
    unsigned char* host = s->staging + (size_t)next * HX_TABLES_BYTES;
    std::memcpy(host, r.tables.data(), HX_TABLES_BYTES);
    if (cudaMemcpyAsync(s->slots[next], host, HX_TABLES_BYTES, cudaMemcpyHostToDevice, st) !=
        cudaSuccess)
      return HX_ERR_CUDA;
    s->cur = next;
    s->slot_hash[next] = r.cb.hash;
  }
  // 3. encode with it, counting this batch's histogram
  if (cudaMemsetAsync(d_hist, 0, 256 * sizeof(uint32_t), st) != cudaSuccess) return HX_ERR_CUDA;
  rc = s->plan.cfg.kind == HX_KIND_HUFFMAN
           ? hx_encode(s->slots[s->cur], d_in, n, d_out, out_cap, d_scratch, d_hist, d_status,
                       stream)
           : hx_qlc_encode(s->slots[s->cur], d_in, n, d_out, out_cap, d_scratch, d_hist,
                           d_status, stream);
  if (rc) return rc;
  // 4. the histogram goes to the host, where the worker folds it
  const uint32_t ri = (uint32_t)(t % s->ring);
  if (cudaMemcpyAsync(s->hist_host + (size_t)ri * 256, d_hist, 256 * sizeof(uint32_t),
                      cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaEventRecord(s->events[ri], st) != cudaSuccess)
    return HX_ERR_CUDA;
  hx_batch_info b{};
  b.hash = r.cb.hash;
  b.slot = s->cur;
  b.drift = std::numeric_limits<double>::quiet_NaN();
  {
    std::lock_guard<std::mutex> lock(s->mu);
    s->info.push_back(b);
    s->enqueued = t + 1;
  }
  s->cv.notify_all();
  s->batch = t + 1;
  return HX_OK;
}

int hx_session_decode(hx_session* s, const void* d_stream, uint64_t stream_bytes, uint8_t* d_out,
                      uint64_t n_expected, uint32_t* d_status, void* stream) {
  if (!s) return HX_ERR_ARG;
  return hx_decode_set(s->plan.cfg.kind, s->slots, s->nslots, d_stream, stream_bytes, d_out,
                       n_expected, d_status, stream);
}

int hx_session_drain(hx_session* s) {
  if (!s) return HX_ERR_ARG;
  std::unique_lock<std::mutex> lock(s->mu);
  s->cv.wait(lock, [&] { return s->folded >= s->enqueued || s->stop; });
  return s->error;
}

int hx_session_batch_info(const hx_session* s, uint64_t batch, hx_batch_info* out) {
  if (!s || !out) return HX_ERR_ARG;
  hx_session* m = const_cast<hx_session*>(s);
  std::lock_guard<std::mutex> lock(m->mu);
  if (batch >= m->info.size()) return HX_ERR_ARG;
  *out = m->info[batch];
  return HX_OK;
}

}  // extern "C"
