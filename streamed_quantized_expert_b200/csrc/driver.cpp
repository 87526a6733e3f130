// Host driver of one decode layer: the whole five-stage sequence in native
// code, so the per-layer host cost is the launches and (when the layer is not
// fully resident) one small device->host copy and its synchronisation.
//
//   route -> sort -> [lookup -> misses to host -> LRU step -> pinned installs on
//   the side stream + table upload -> FFN of the resident experts (writes y),
//   overlapping the copies -> compute stream waits] -> FFN (of the installed
//   experts, adding to y; or of every expert, writing y)
//
// RFC "How the prototype works": each layer copies its routing to the host
// once; misses become one host-to-device copy per expert; when every expert
// is resident the layer never synchronises with the host.
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

extern "C" moe_status moe_decode_layer(moe_cache* cache, int32_t layer, const moe_layer_ctx* lc,
                                       const moe_step_buffers* b, const uint16_t* x, const float* logits,
                                       int32_t T, float L, float* y, cudaStream_t stream, cudaStream_t side,
                                       cudaEvent_t installed, int32_t* n_installed) {
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
  moe_status s = ns ? moe_route_shared(logits, T, d0, L, lc->table_dev, ns, lc->shared_w, b->ids, b->w, stream)
                    : moe_route(logits, T, d0, L, lc->table_dev, b->ids, b->w, stream);
  if (s != MOE_OK) return s;
  // from 32 tokens the FFN runs on the tensor-core grouped GEMM, which reads x sorted by expert
  uint16_t* xs = (T >= 32 && b->x_sorted) ? b->x_sorted : nullptr;
  s = moe_sort(b->ids, xs ? x : nullptr, T, d, b->offsets, b->pairs, active, n_active, xs, b->ws, b->ws_bytes,
               stream);
  if (s != MOE_OK) return s;
  if (moe_cache_resident(cache, layer) < E0) {
    s = moe_slot_lookup(lc->table_dev, active, n_active, 0, E, lc->n_slots, b->slots, miss, n_miss, b->dev_err,
                        stream);
    if (s != MOE_OK) return s;
    if (cudaMemcpyAsync(b->meta_host, b->meta, sizeof(int32_t) * (size_t)(2 + E), cudaMemcpyDeviceToHost,
                        stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
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
