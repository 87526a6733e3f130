// Host driver of one decode layer: the whole five-stage sequence in native
// code, so the per-layer host cost is the launches and (when the layer is not
// fully resident) one small device->host copy and its synchronisation -- or,
// for one token, a wait on a word the routing kernel writes to host memory
// after the active list itself.
//
//   route -> sort -> [lookup -> misses to host -> LRU step -> pinned installs on
//   the side stream + table upload -> FFN of the resident experts (writes y),
//   overlapping the copies -> compute stream waits] -> FFN (of the installed
//   experts, adding to y; or of every expert, writing y)
//
// RFC "How the prototype works": each layer copies its routing to the host
// once; misses become one host-to-device copy per expert; when every expert
// is resident the layer never synchronises with the host.
//
// Guessed prefetch (same page, item "Reads": the next two layers' experts are
// guessed by running their routers on the current hidden states and read in
// the background; PR #50717 commit note: install_ahead skips guessed reads
// still in flight instead of waiting for them).  moe_decode_layer_ahead routes
// the guessed layers' logits (top-k, L = 0) next to the layer's own stages, so
// their ids come back with the layer's one synchronisation; the guessed
// misses get slots reserved in the cache and their copies start on an `ahead`
// stream of their own, one event per batch.  At the start of a layer its
// landed batches are entered into the table (an event query, never a wait);
// batches still in flight are skipped and stay reserved.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstring>
#include <vector>

#include <cuda_runtime.h>

#include "moe.h"

extern "C" moe_status moe_internal_expert_ffn(const uint16_t* x, int32_t T, const moe_layer_desc* d,
                                              const void* pool, int32_t n_slots, const int32_t* slot_table,
                                              const int32_t* ids, const float* w, const int32_t* offsets,
                                              const int32_t* pairs, const int32_t* active, const int32_t* n_active,
                                              const uint16_t* x_sorted, int32_t pass_begin, int32_t pass_len,
                                              float* y_accum, void* ws, size_t ws_bytes, int32_t* dev_err,
                                              cudaStream_t stream, int overwrite);
extern "C" moe_status moe_internal_route_sort_lookup(
    const float* logits, int32_t T, const moe_layer_desc* d, float L, const int32_t* slot_table, int32_t n_shared,
    const float* shared_w, int32_t n_slots, int32_t* ids, float* w, int32_t* offsets, int32_t* pairs,
    int32_t* active, int32_t* n_active, int32_t* slots, int32_t* miss, int32_t* n_miss, int32_t* dev_err,
    cudaStream_t stream, int32_t* host_meta, int32_t seq);

struct moe_prefetch {
  struct Batch {
    cudaEvent_t ev;
    std::vector<int32_t> slots;
  };
  std::vector<std::vector<Batch>> q;  // [layer]: guessed copies in flight, oldest first
  std::vector<cudaEvent_t> spare;     // recycled events
  std::vector<uint8_t> dirty;         // [layer]: host table changed by reservations since the last upload
  int64_t guessed = 0, started = 0, entered = 0, wasted = 0, skipped = 0;
};

namespace {

// Whether the device addresses host memory p at the same pointer (page-locked
// memory from cudaHostAlloc / cudaMallocHost under unified addressing).
// Checked on every call: a cached answer could outlive the allocation.
bool device_maps_host(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost && a.devicePointer == p;
}

// Sequence words of the one-token routing kernel's host writes: distinct
// from every count the copy-back path leaves in the same word (<= 1032).
int32_t next_host_seq() {
  static std::atomic<uint32_t> n{0};
  return (int32_t)(0x40000000u | (n.fetch_add(1, std::memory_order_relaxed) & 0x3fffffffu));
}

// Wait until the routing kernel has published the active list to host
// memory (host_meta[1] == seq).  Bounded: the stream's state is polled every
// 1024 reads, and a stream that has failed or finished without the word, or
// a wait past kHostWaitSeconds, ends it with an error.
constexpr double kHostWaitSeconds = 5.0;
moe_status wait_host_seq(const int32_t* host_meta, int32_t seq, cudaStream_t stream) {
  const volatile int32_t* word = host_meta + 1;
  const auto t0 = std::chrono::steady_clock::now();
  for (uint32_t i = 1; *word != seq; ++i) {
    if ((i & 1023u) == 0) {
      const cudaError_t e = cudaStreamQuery(stream);
      if (e == cudaSuccess) {
        if (*word == seq) break;
        return MOE_ERR_CUDA;  // the stream drained, the word never came
      }
      if (e != cudaErrorNotReady) return MOE_ERR_CUDA;
      if (std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count() > kHostWaitSeconds)
        return MOE_ERR_TIMEOUT;
    }
#if defined(__x86_64__)
    __builtin_ia32_pause();
#endif
  }
  std::atomic_thread_fence(std::memory_order_acquire);
  return MOE_OK;
}

struct Guess {
  moe_prefetch* pf;
  const moe_guess* g;
  int32_t n;
  const moe_guess_buffers* gb;
  cudaStream_t ahead;
};

// Enter the landed guessed copies of `layer` into the table; upload it on
// `stream` if reservations or entries changed it.
moe_status retire(moe_prefetch* pf, moe_cache* cache, int32_t layer, const moe_layer_ctx* lc, cudaStream_t stream) {
  auto& q = pf->q[layer];
  size_t done = 0;
  for (; done < q.size(); ++done) {
    const cudaError_t e = cudaEventQuery(q[done].ev);
    if (e == cudaErrorNotReady) break;  // this batch and the later ones are still in flight: skipped
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    for (int32_t slot : q[done].slots) {
      int32_t in = 0;
      if (moe_cache_commit(cache, layer, slot, &in) != MOE_OK) return MOE_ERR_INVALID;
      pf->entered += in;
      pf->wasted += 1 - in;
    }
    pf->spare.push_back(q[done].ev);
    pf->dirty[layer] = 1;
  }
  for (size_t i = done; i < q.size(); ++i) pf->skipped += (int64_t)q[i].slots.size();
  q.erase(q.begin(), q.begin() + (ptrdiff_t)done);
  if (pf->dirty[layer]) {
    const int32_t E0 = lc->desc->E;
    std::memcpy(lc->table_stage, moe_cache_table(cache, layer), sizeof(int32_t) * (size_t)E0);
    if (cudaMemcpyAsync(lc->table_dev, lc->table_stage, sizeof(int32_t) * (size_t)E0, cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    pf->dirty[layer] = 0;
  }
  return MOE_OK;
}

// The guessed layers' experts (ids back on the host): reserve slots for the
// misses and start their copies on the ahead stream.
moe_status start_guesses(const Guess& G, moe_cache* cache, int32_t T) {
  thread_local std::vector<int32_t> want, out_e, out_s;
  thread_local std::vector<const void*> rows;
  for (int32_t gi = 0; gi < G.n; ++gi) {
    const moe_guess& g = G.g[gi];
    const int32_t k = g.lc->desc->k, E0 = g.lc->desc->E;
    const int32_t* ids = G.gb->ids_host + (size_t)gi * G.gb->stride;
    const int32_t top = g.top > 0 && g.top < k ? g.top : k;  // ids are in rank order per token
    want.clear();
    for (int32_t t = 0; t < T; ++t) want.insert(want.end(), ids + (size_t)t * k, ids + (size_t)t * k + top);
    std::sort(want.begin(), want.end());
    want.erase(std::unique(want.begin(), want.end()), want.end());
    while (!want.empty() && (want.back() >= E0 || want.back() < 0)) want.pop_back();
    G.pf->guessed += (int64_t)want.size();
    out_e.resize(want.size());
    out_s.resize(want.size());
    int32_t n = 0;
    moe_status s = moe_cache_reserve(cache, g.layer, want.data(), (int32_t)want.size(), out_e.data(), out_s.data(), &n);
    if (s != MOE_OK) return s;
    if (n == 0) continue;
    rows.resize(n);
    for (int32_t i = 0; i < n; ++i) rows[i] = g.lc->bank_rows[out_e[i]];
    s = moe_install_slots(g.lc->pool, g.lc->slot_bytes, g.lc->n_slots, rows.data(), out_s.data(), n, G.ahead,
                          nullptr);
    if (s != MOE_OK) return s;
    cudaEvent_t ev;
    if (!G.pf->spare.empty()) {
      ev = G.pf->spare.back();
      G.pf->spare.pop_back();
    } else if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
      return MOE_ERR_CUDA;
    }
    if (cudaEventRecord(ev, G.ahead) != cudaSuccess) return MOE_ERR_CUDA;
    G.pf->q[g.layer].push_back({ev, std::vector<int32_t>(out_s.begin(), out_s.begin() + n)});
    G.pf->dirty[g.layer] = 1;  // victims left the table
    G.pf->started += n;
  }
  return MOE_OK;
}

moe_status decode_layer(moe_cache* cache, int32_t layer, const moe_layer_ctx* lc, const moe_step_buffers* b,
                        const uint16_t* x, const float* logits, int32_t T, float L, float* y, cudaStream_t stream,
                        cudaStream_t side, cudaEvent_t installed, int32_t* n_installed, const Guess* G) {
  if (!cache || !lc || !b || !lc->desc || !y || !x || !logits) return MOE_ERR_INVALID;
  const moe_layer_desc* d0 = lc->desc;  // the routed experts
  const int32_t ns = lc->n_shared;
  if (ns < 0 || ns > 8) return MOE_ERR_INVALID;
  // the widened layer: shared experts E0 .. E0 + ns - 1 after the routed ones
  moe_layer_desc dw = *d0;
  dw.E += ns;
  dw.k += ns;
  const moe_layer_desc* d = &dw;
  if (T < 1 || T > b->max_tokens || T > 64) return MOE_ERR_INVALID;
  const int32_t E = d->E, E0 = d0->E;
  if (n_installed) *n_installed = 0;
  int32_t* n_active = b->meta;
  int32_t* n_miss = b->meta + 1;
  int32_t* active = b->meta + 2;
  int32_t* miss = b->meta + 2 + E;
  // where the FFN runs on the tensor-core grouped GEMM (above the fused decode kernel's range; BF16
  // experts always), it reads x sorted by expert
  uint16_t* xs =
      (b->x_sorted && moe_ffn_kernel_path(d, T, 1) == MOE_PATH_TC_PREFILL) ? b->x_sorted : nullptr;
  // one token without sorted x: routing, sort and lookup in one launch
  const bool one = T == 1 && !xs;
  if (one && ns == 0 && !(G && G->n > 0) && moe_cache_resident(cache, layer) >= E0) {
    // a fully resident layer: the FFN launch routes the token itself (the host needs none of it)
    const moe_status r = moe_route_expert_ffn(x, logits, T, d0, L, lc->pool, lc->n_slots, lc->table_dev, b->ids,
                                              b->w, b->offsets, b->pairs, active, n_active, b->slots, miss, n_miss,
                                              y, b->ws, b->ws_bytes, b->dev_err, stream);
    if (r != MOE_ERR_UNSUPPORTED) return r;
  }
  moe_status s = MOE_OK;
  const bool guessing = G && G->n > 0;
  const bool resident = moe_cache_resident(cache, layer) >= E0;
  // the host needs the active list: for one token the routing kernel writes it
  // straight to host memory, with no copy back or stream synchronisation
  int32_t* host_meta = nullptr;
  int32_t seq = 0;
  if (one && !resident && !guessing && device_maps_host(b->meta_host)) {
    host_meta = b->meta_host;
    seq = next_host_seq();
  }
  if (one) {
    s = moe_internal_route_sort_lookup(logits, T, d0, L, lc->table_dev, ns, lc->shared_w, lc->n_slots, b->ids,
                                       b->w, b->offsets, b->pairs, active, n_active, b->slots, miss, n_miss,
                                       b->dev_err, stream, host_meta, seq);
    if (s != MOE_OK) return s;
  } else {
    s = ns ? moe_route_shared(logits, T, d0, L, lc->table_dev, ns, lc->shared_w, b->ids, b->w, stream)
           : moe_route(logits, T, d0, L, lc->table_dev, b->ids, b->w, stream);
    if (s != MOE_OK) return s;
    s = moe_sort(b->ids, xs ? x : nullptr, T, d, b->offsets, b->pairs, active, n_active, xs, b->ws, b->ws_bytes,
                 stream);
    if (s != MOE_OK) return s;
  }
  // the guessed layers' top-k, on the same synchronisation as the layer's own lookup
  if (guessing) {
    for (int32_t gi = 0; gi < G->n; ++gi) {
      const moe_guess& g = G->g[gi];
      int32_t* gids = G->gb->ids + (size_t)gi * G->gb->stride;
      s = moe_route(g.logits, T, g.lc->desc, 0.0f, nullptr, gids, G->gb->w + (size_t)gi * G->gb->stride, stream);
      if (s != MOE_OK) return s;
      if (cudaMemcpyAsync(G->gb->ids_host + (size_t)gi * G->gb->stride, gids,
                          sizeof(int32_t) * (size_t)T * g.lc->desc->k, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
  }
  if (resident && guessing) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    s = start_guesses(*G, cache, T);
    if (s != MOE_OK) return s;
  }
  if (!resident) {
    if (!one) {
      s = moe_slot_lookup(lc->table_dev, active, n_active, 0, E, lc->n_slots, b->slots, miss, n_miss, b->dev_err,
                          stream);
      if (s != MOE_OK) return s;
    }
    if (host_meta) {
      s = wait_host_seq(host_meta, seq, stream);
      if (s != MOE_OK) return s;
    } else {
      if (cudaMemcpyAsync(b->meta_host, b->meta, sizeof(int32_t) * (size_t)(2 + E), cudaMemcpyDeviceToHost,
                          stream) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    }
    const int32_t na = b->meta_host[0];
    if (na < ns || na > E) return MOE_ERR_INVALID;
    thread_local std::vector<int32_t> out_e, out_s;
    thread_local std::vector<const void*> rows;
    out_e.resize(E);
    out_s.resize(E);
    int32_t n = 0;
    // the active list is ascending: every token's shared experts are its last
    // ns entries, and the cache manages the routed ones only
    s = moe_cache_step(cache, layer, b->meta_host + 2, na - ns, out_e.data(), out_s.data(), &n);
    if (s != MOE_OK) return s;
    if (guessing) {  // after this layer's own misses have their slots
      s = start_guesses(*G, cache, T);
      if (s != MOE_OK) return s;
    }
    if (n > 0) {
      rows.resize(n);
      for (int32_t i = 0; i < n; ++i) rows[i] = lc->bank_rows[out_e[i]];
      s = moe_install_slots(lc->pool, lc->slot_bytes, lc->n_slots, rows.data(), out_s.data(), n, side, nullptr);
      if (s != MOE_OK) return s;
      std::memcpy(lc->table_stage, moe_cache_table(cache, layer), sizeof(int32_t) * (size_t)E0);
      if (cudaMemcpyAsync(lc->table_dev, lc->table_stage, sizeof(int32_t) * (size_t)E0, cudaMemcpyHostToDevice,
                          side) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaEventRecord(installed, side) != cudaSuccess) return MOE_ERR_CUDA;
      if (n_installed) *n_installed = n;
      // The experts that were resident keep their slots (the LRU step never
      // evicts an expert of the step), so their FFN runs while the copies land:
      // the pass is reordered as [resident..., installed...] (both ascending)
      // in the host copy's miss region, which has been read, and goes to the
      // device slots buffer, which the lookup no longer needs.
      int32_t* order = b->meta_host + 2 + E;
      const int32_t* act = b->meta_host + 2;
      int32_t nr = 0;
      for (int32_t i = 0, m = 0; i < na; ++i) {
        if (m < n && out_e[m] == act[i]) {
          ++m;
          continue;
        }
        order[nr++] = act[i];
      }
      for (int32_t i = 0; i < n; ++i) order[nr + i] = out_e[i];
      if (cudaMemcpyAsync(b->slots, order, sizeof(int32_t) * (size_t)na, cudaMemcpyHostToDevice, stream) !=
          cudaSuccess)
        return MOE_ERR_CUDA;
      if (nr > 0) {
        s = moe_internal_expert_ffn(x, T, d, lc->pool, lc->n_slots, lc->table_dev, b->ids, b->w, b->offsets,
                                    b->pairs, b->slots, n_active, xs, 0, nr, y, b->ws, b->ws_bytes, b->dev_err,
                                    stream, 1);
        if (s != MOE_OK) return s;
      }
      if (cudaStreamWaitEvent(stream, installed, 0) != cudaSuccess) return MOE_ERR_CUDA;
      return moe_internal_expert_ffn(x, T, d, lc->pool, lc->n_slots, lc->table_dev, b->ids, b->w, b->offsets,
                                     b->pairs, b->slots, n_active, xs, nr, n, y, b->ws, b->ws_bytes,
                                     b->dev_err, stream, nr > 0 ? 0 : 1);
    }
  }
  // one pass over every active expert, writing y (no separate zeroing)
  return moe_internal_expert_ffn(x, T, d, lc->pool, lc->n_slots, lc->table_dev, b->ids, b->w, b->offsets, b->pairs,
                                 active, n_active, xs, 0, E, y, b->ws, b->ws_bytes, b->dev_err, stream, 1);
}

}  // namespace

extern "C" {

moe_status moe_decode_layer(moe_cache* cache, int32_t layer, const moe_layer_ctx* lc, const moe_step_buffers* b,
                            const uint16_t* x, const float* logits, int32_t T, float L, float* y,
                            cudaStream_t stream, cudaStream_t side, cudaEvent_t installed, int32_t* n_installed) {
  return decode_layer(cache, layer, lc, b, x, logits, T, L, y, stream, side, installed, n_installed, nullptr);
}

moe_status moe_prefetch_create(int32_t n_layers, moe_prefetch** out) {
  if (!out || n_layers < 1) return MOE_ERR_INVALID;
  moe_prefetch* p = new moe_prefetch();
  p->q.resize(n_layers);
  p->dirty.assign(n_layers, 0);
  *out = p;
  return MOE_OK;
}

void moe_prefetch_destroy(moe_prefetch* p) {
  if (!p) return;
  for (auto& q : p->q)
    for (auto& b : q) cudaEventDestroy(b.ev);
  for (cudaEvent_t e : p->spare) cudaEventDestroy(e);
  delete p;
}

void moe_prefetch_stats(const moe_prefetch* p, int64_t* guessed, int64_t* started, int64_t* entered,
                        int64_t* wasted, int64_t* skipped) {
  if (!p) return;
  if (guessed) *guessed = p->guessed;
  if (started) *started = p->started;
  if (entered) *entered = p->entered;
  if (wasted) *wasted = p->wasted;
  if (skipped) *skipped = p->skipped;
}

moe_status moe_decode_layer_ahead(moe_cache* cache, moe_prefetch* pf, int32_t layer, const moe_layer_ctx* lc,
                                  const moe_step_buffers* b, const uint16_t* x, const float* logits, int32_t T,
                                  float L, float* y, cudaStream_t stream, cudaStream_t side, cudaEvent_t installed,
                                  int32_t* n_installed, const moe_guess* guesses, int32_t n_guesses,
                                  const moe_guess_buffers* gb, cudaStream_t ahead) {
  if (!cache || !pf || layer < 0 || layer >= (int32_t)pf->q.size() || !lc || !lc->desc) return MOE_ERR_INVALID;
  if (n_guesses < 0 || n_guesses > 2 || (n_guesses > 0 && (!guesses || !gb))) return MOE_ERR_INVALID;
  for (int32_t i = 0; i < n_guesses; ++i) {
    const moe_guess& g = guesses[i];
    if (!g.lc || !g.lc->desc || !g.logits || g.layer < 0 || g.layer >= (int32_t)pf->q.size() || g.layer == layer)
      return MOE_ERR_INVALID;
    if ((int64_t)T * g.lc->desc->k > gb->stride) return MOE_ERR_CAPACITY;
  }
  moe_status s = retire(pf, cache, layer, lc, stream);
  if (s != MOE_OK) return s;
  const Guess G{pf, guesses, n_guesses, gb, ahead};
  return decode_layer(cache, layer, lc, b, x, logits, T, L, y, stream, side, installed, n_installed, &G);
}

}  // extern "C"
