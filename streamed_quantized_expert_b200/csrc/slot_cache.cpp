// Host slot cache: one LRU per (size class, layer) over the layer's own range
// of its class pool (1bit-MONSTER engine PR #137 "expert slots in size
// classes": each class has its own slots and LRU, one LRU per layer with
// --per-layer, every layer keeps the same share of its experts, empty slots
// sit at the back of the LRU and are taken first).  Host memory only.
//
// Guessed prefetch (RFC "How the prototype works", item "Reads": the next two
// layers' experts are guessed and read in the background): moe_cache_reserve
// takes slots for guessed experts the way a step takes them for misses, but
// leaves the experts out of the table while their copies are in flight; a
// reserved slot is never a victim; moe_cache_commit enters the expert once
// its copy has landed (or frees the slot if the expert was installed
// elsewhere meanwhile).
#include <cstdint>
#include <algorithm>
#include <vector>

#include "moe.h"

struct moe_cache {
  int32_t E = 0, n_layers = 0, S = 0;
  std::vector<int32_t> layer_class, layer_base, class_slots;
  std::vector<std::vector<int32_t>> table;  // [layer][E]
  std::vector<std::vector<int32_t>> owner;  // [layer][S]: expert in slot base+i, or -1
  std::vector<std::vector<int64_t>> stamp;  // [layer][S]: last use, 0 = never used
  std::vector<std::vector<int32_t>> pend;   // [layer][S]: expert whose guessed copy is in flight, or -1
  std::vector<uint8_t> used;                // scratch [S]
  std::vector<int32_t> resident;            // [layer]: experts with a slot
  int64_t clock = 0, hits = 0, misses = 0, evictions = 0;
};

extern "C" {

moe_status moe_cache_create(int32_t E, int32_t n_layers, const int32_t* layer_class, int32_t slots_per_layer,
                            moe_cache** out) {
  if (!out || E < 1 || n_layers < 1 || slots_per_layer < 1) return MOE_ERR_INVALID;
  moe_cache* c = new moe_cache();
  c->E = E;
  c->n_layers = n_layers;
  c->S = slots_per_layer;
  c->layer_class.assign(n_layers, 0);
  int32_t ncls = 1;
  for (int32_t l = 0; l < n_layers; ++l) {
    const int32_t k = layer_class ? layer_class[l] : 0;
    if (k < 0 || k > 255) {
      delete c;
      return MOE_ERR_INVALID;
    }
    c->layer_class[l] = k;
    if (k + 1 > ncls) ncls = k + 1;
  }
  c->class_slots.assign(ncls, 0);
  c->layer_base.assign(n_layers, 0);
  for (int32_t l = 0; l < n_layers; ++l) {
    c->layer_base[l] = c->class_slots[c->layer_class[l]];
    c->class_slots[c->layer_class[l]] += slots_per_layer;
  }
  c->table.assign(n_layers, std::vector<int32_t>(E, -1));
  c->owner.assign(n_layers, std::vector<int32_t>(slots_per_layer, -1));
  c->stamp.assign(n_layers, std::vector<int64_t>(slots_per_layer, 0));
  c->pend.assign(n_layers, std::vector<int32_t>(slots_per_layer, -1));
  c->used.assign(slots_per_layer, 0);
  c->resident.assign(n_layers, 0);
  *out = c;
  return MOE_OK;
}

void moe_cache_destroy(moe_cache* c) { delete c; }

const int32_t* moe_cache_table(const moe_cache* c, int32_t layer) {
  if (!c || layer < 0 || layer >= c->n_layers) return nullptr;
  return c->table[layer].data();
}

int32_t moe_cache_layer_base(const moe_cache* c, int32_t layer) {
  if (!c || layer < 0 || layer >= c->n_layers) return -1;
  return c->layer_base[layer];
}

int32_t moe_cache_class_slots(const moe_cache* c, int32_t cls) {
  if (!c || cls < 0 || cls >= (int32_t)c->class_slots.size()) return 0;
  return c->class_slots[cls];
}

moe_status moe_cache_place(moe_cache* c, int32_t layer, const int32_t* experts, const int32_t* slots, int32_t n) {
  if (!c || layer < 0 || layer >= c->n_layers || n < 0 || (n > 0 && (!experts || !slots))) return MOE_ERR_INVALID;
  const int32_t base = c->layer_base[layer];
  for (int32_t i = 0; i < n; ++i) {
    const int32_t e = experts[i], s = slots[i] - base;
    if (e < 0 || e >= c->E || s < 0 || s >= c->S) return MOE_ERR_INVALID;
    auto& tab = c->table[layer];
    auto& own = c->owner[layer];
    if (own[s] >= 0) {
      tab[own[s]] = -1;
      --c->resident[layer];
    }
    if (tab[e] >= 0) {
      own[tab[e] - base] = -1;
      --c->resident[layer];
    }
    own[s] = e;
    tab[e] = base + s;
    ++c->resident[layer];
    c->stamp[layer][s] = ++c->clock;  // placed slots are more recent than empty ones
  }
  return MOE_OK;
}

moe_status moe_cache_step(moe_cache* c, int32_t layer, const int32_t* pass_experts, int32_t n_pass,
                          int32_t* out_experts, int32_t* out_slots, int32_t* n_out) {
  if (!c || layer < 0 || layer >= c->n_layers || n_pass < 0 || !n_out) return MOE_ERR_INVALID;
  if (n_pass > 0 && (!pass_experts || !out_experts || !out_slots)) return MOE_ERR_INVALID;
  const int32_t base = c->layer_base[layer];
  auto& tab = c->table[layer];
  auto& own = c->owner[layer];
  auto& stp = c->stamp[layer];
  std::fill(c->used.begin(), c->used.end(), 0);
  for (int32_t s = 0; s < c->S; ++s) c->used[s] = c->pend[layer][s] >= 0;  // copies in flight: no victims
  for (int32_t i = 0; i < n_pass; ++i) {
    const int32_t e = pass_experts[i];
    if (e < 0 || e >= c->E) return MOE_ERR_INVALID;
    if (tab[e] >= 0) {
      c->used[tab[e] - base] = 1;
      stp[tab[e] - base] = ++c->clock;
      ++c->hits;
    }
  }
  moe_status st = MOE_OK;
  int32_t n = 0;
  for (int32_t i = 0; i < n_pass; ++i) {
    const int32_t e = pass_experts[i];
    if (tab[e] >= 0) continue;
    ++c->misses;
    int32_t best = -1;
    for (int32_t s = 0; s < c->S; ++s) {
      if (c->used[s]) continue;
      if (best < 0 || stp[s] < stp[best]) best = s;
    }
    out_experts[n] = e;
    if (best < 0) {
      out_slots[n++] = -1;
      st = MOE_ERR_CAPACITY;
      continue;
    }
    if (own[best] >= 0) {
      tab[own[best]] = -1;
      ++c->evictions;
      --c->resident[layer];
    }
    own[best] = e;
    tab[e] = base + best;
    ++c->resident[layer];
    c->used[best] = 1;
    stp[best] = ++c->clock;
    out_slots[n++] = base + best;
  }
  *n_out = n;
  return st;
}

moe_status moe_cache_reserve(moe_cache* c, int32_t layer, const int32_t* experts, int32_t n, int32_t* out_experts,
                             int32_t* out_slots, int32_t* n_out) {
  if (!c || layer < 0 || layer >= c->n_layers || n < 0 || !n_out) return MOE_ERR_INVALID;
  if (n > 0 && (!experts || !out_experts || !out_slots)) return MOE_ERR_INVALID;
  const int32_t base = c->layer_base[layer];
  auto& tab = c->table[layer];
  auto& own = c->owner[layer];
  auto& stp = c->stamp[layer];
  auto& pnd = c->pend[layer];
  int32_t m = 0;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t e = experts[i];
    if (e < 0 || e >= c->E) return MOE_ERR_INVALID;
    if (tab[e] >= 0) continue;  // resident already
    bool in_flight = false;
    for (int32_t s = 0; s < c->S && !in_flight; ++s) in_flight = pnd[s] == e;
    if (in_flight) continue;
    // the least recently used slot without a copy in flight (empty slots first)
    int32_t best = -1;
    for (int32_t s = 0; s < c->S; ++s) {
      if (pnd[s] >= 0) continue;
      if (best < 0 || stp[s] < stp[best]) best = s;
    }
    if (best < 0) break;  // every slot has a copy in flight
    if (own[best] >= 0) {
      tab[own[best]] = -1;
      ++c->evictions;
      --c->resident[layer];
      own[best] = -1;
    }
    pnd[best] = e;
    stp[best] = ++c->clock;
    out_experts[m] = e;
    out_slots[m++] = base + best;
  }
  *n_out = m;
  return MOE_OK;
}

moe_status moe_cache_commit(moe_cache* c, int32_t layer, int32_t slot, int32_t* entered) {
  if (!c || layer < 0 || layer >= c->n_layers) return MOE_ERR_INVALID;
  const int32_t s = slot - c->layer_base[layer];
  if (s < 0 || s >= c->S || c->pend[layer][s] < 0) return MOE_ERR_INVALID;
  const int32_t e = c->pend[layer][s];
  c->pend[layer][s] = -1;
  auto& tab = c->table[layer];
  if (tab[e] < 0) {  // the guess is now resident
    c->owner[layer][s] = e;
    tab[e] = slot;
    ++c->resident[layer];
    c->stamp[layer][s] = ++c->clock;
    if (entered) *entered = 1;
  } else {  // installed elsewhere while the copy was in flight: the slot is free again
    c->stamp[layer][s] = 0;
    if (entered) *entered = 0;
  }
  return MOE_OK;
}

int32_t moe_cache_resident(const moe_cache* c, int32_t layer) {
  if (!c || layer < 0 || layer >= c->n_layers) return -1;
  return c->resident[layer];
}

void moe_cache_stats(const moe_cache* c, int64_t* hits, int64_t* misses, int64_t* evictions) {
  if (!c) return;
  if (hits) *hits = c->hits;
  if (misses) *misses = c->misses;
  if (evictions) *evictions = c->evictions;
}

}  // extern "C"
