// libmoe C ABI: argument checks, workspace carving and launches.  Every
// entry point validates before launching anything and returns a moe_status;
// see include/moe.h for the contract of each call.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

using namespace moe;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status check_desc(const moe_layer_desc* d) {
  if (!d) return MOE_ERR_INVALID;
  if (d->E < 1 || d->k < 1 || d->k > d->E || d->H < 1 || d->I < 1) return MOE_ERR_INVALID;
  if (d->group != 32 && d->group != 64 && d->group != 128) return MOE_ERR_UNSUPPORTED;
  auto bits_ok = [](int b) { return b == 3 || b == 4 || b == 6 || b == 16; };  // 16: BF16 experts
  if (!bits_ok(d->bits_gu) || !bits_ok(d->bits_down)) return MOE_ERR_UNSUPPORTED;
  if (d->H % d->group || d->I % d->group) return MOE_ERR_INVALID;
  if (d->E > 1024 || d->k > 32) return MOE_ERR_UNSUPPORTED;
  if (d->H > 1 << 16 || d->I > 1 << 16) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

thread_local const char* g_last_cuda_error = "no error";

std::atomic<long long> g_wait_limit{kDefaultWaitCycles};

moe_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  g_last_cuda_error = cudaGetErrorName(e);
  return MOE_ERR_CUDA;
}

int device_sms() {
  static int cached[128] = {0};
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 128 && cached[dev] > 0) return cached[dev];
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  if (dev >= 0 && dev < 128) cached[dev] = sms;
  return sms;
}

// Workspace: [control block (kWsControlBytes)][tagged h words][sort scratch |
// FFN scratch].  The control block (the single-launch decode kernel's epoch
// and arrival count) and the tagged h words (that kernel's h, each word
// carrying its launch's tag) persist from call to call and are zeroed
// together, once, before the first call; they sit at the same place for
// every T.  The sort and FFN scratch overlap (different calls,
// stream-ordered).
struct WsCarve {
  size_t sort, hb, h, o, tag, total;
};

// tc: the call may run the tensor-core path (x_sorted given), whose per-pair
// outputs need o from kTcMinTokens tokens; without it o is needed above 64.
WsCarve carve(const moe_layer_desc& d, int T, bool tc = true) {
  WsCarve c{};
  const int64_t np = (int64_t)T * d.k;
  // the single-launch decode kernel's tagged h words, for its largest call
  // (T * k <= 64): at the same place for every T, written by nothing else
  const int64_t np_tag = 8 * (int64_t)d.k < 64 ? 8 * (int64_t)d.k : 64;
  c.tag = (size_t)round_up(np_tag * padded_k(d.I) * 8, 256);
  c.sort = (size_t)round_up((int64_t)sort_ws_bytes((int)np, d.E), 256);
  // h (bf16, rows padded to 128-blocks) and its per-8-column partial sums
  c.hb = (size_t)round_up(np * padded_k(d.I) * 2, 256);
  c.h = c.hb + (size_t)round_up(np * padded_k(d.I), 256);
  // o: per-pair outputs of the tensor-core path (T >= kTcMinTokens) and of the GEMV path for T > 64
  c.o = ((tc && (T >= kTcMinTokens || bf16_experts(d))) || T > kFusedMaxTokens) ? (size_t)round_up(np * d.H * 4, 256)
                                                                                  : 0;
  const size_t ffn = c.h + c.o;
  c.total = kWsControlBytes + c.tag + (c.sort > ffn ? c.sort : ffn);
  return c;
}

}  // namespace

long long moe::wait_limit_cycles() { return g_wait_limit.load(std::memory_order_relaxed); }

extern "C" {

void moe_set_wait_limit_cycles(int64_t cycles) {
  g_wait_limit.store(cycles > 0 ? (long long)cycles : kDefaultWaitCycles, std::memory_order_relaxed);
}

const char* moe_last_cuda_error(void) { return g_last_cuda_error; }

int32_t moe_ffn_kernel_path(const moe_layer_desc* d, int32_t T, int32_t has_x_sorted) {
  if (check_desc(d) != MOE_OK || T < 1 || !ffn_decode_supported(*d)) return -1;
  return ffn_kernel_path(*d, T, has_x_sorted != 0, device_sms());
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_NOT_RESIDENT: return "expert not resident";
    case MOE_ERR_CAPACITY: return "capacity exceeded";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

size_t moe_slot_bytes(const moe_layer_desc* d) {
  if (check_desc(d) != MOE_OK) return 0;
  return (size_t)make_layout(*d).slot_bytes;
}

moe_status moe_slot_layout(const moe_layer_desc* d, moe_slot_layout_t* out) {
  moe_status s = check_desc(d);
  if (s != MOE_OK) return s;
  if (!out) return MOE_ERR_INVALID;
  const Layout L = make_layout(*d);
  out->gate_up = (uint64_t)L.gu;
  out->down = (uint64_t)L.d;
  out->gate_up_tile_bytes = (uint64_t)L.tile_gu;
  out->down_tile_bytes = (uint64_t)L.tile_d;
  out->slot_bytes = (uint64_t)L.slot_bytes;
  return MOE_OK;
}

size_t moe_workspace_bytes(const moe_layer_desc* d, int32_t max_tokens) {
  if (check_desc(d) != MOE_OK || max_tokens < 0) return 0;
  return carve(*d, max_tokens).total;
}

// Workspace bytes of a call that passes no x_sorted (the GEMV / fused kernels).
// Head of the workspace that persists from call to call (control block and
// tagged h words): the bytes moe_expert_ffn_noalloc clears before each call.
__attribute__((visibility("hidden"))) size_t moe_internal_workspace_persistent_bytes(const moe_layer_desc* d) {
  if (check_desc(d) != MOE_OK) return 0;
  return kWsControlBytes + carve(*d, 1).tag;
}

__attribute__((visibility("hidden"))) size_t moe_internal_workspace_bytes_no_tc(const moe_layer_desc* d,
                                                                               int32_t max_tokens) {
  if (check_desc(d) != MOE_OK || max_tokens < 0) return 0;
  return carve(*d, max_tokens, false).total;
}

moe_status moe_route(const float* logits, int32_t T, const moe_layer_desc* d, float L, const int32_t* slot_table,
                     int32_t* ids, float* w, cudaStream_t stream) {
  moe_status s = check_desc(d);
  if (s != MOE_OK) return s;
  if (T < 0 || !(L >= 0.0f) || L > 1e30f) return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (!logits || !ids || !w) return MOE_ERR_INVALID;
  if (L > 0.0f && !slot_table) return MOE_ERR_INVALID;
  return cuda_status(launch_route(logits, T, d->E, d->k, L, slot_table, ids, w, 0, nullptr, stream));
}

moe_status moe_route_shared(const float* logits, int32_t T, const moe_layer_desc* d, float L,
                            const int32_t* slot_table, int32_t n_shared, const float* shared_w, int32_t* ids,
                            float* w, cudaStream_t stream) {
  moe_status s = check_desc(d);
  if (s != MOE_OK) return s;
  if (T < 0 || !(L >= 0.0f) || L > 1e30f || n_shared < 0 || n_shared > kMaxShared) return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (!logits || !ids || !w) return MOE_ERR_INVALID;
  if (L > 0.0f && !slot_table) return MOE_ERR_INVALID;
  return cuda_status(launch_route(logits, T, d->E, d->k, L, slot_table, ids, w, n_shared, shared_w, stream));
}

moe_status moe_sort(const int32_t* ids, const uint16_t* x, int32_t T, const moe_layer_desc* d, int32_t* offsets,
                    int32_t* pairs, int32_t* active, int32_t* n_active, uint16_t* x_sorted, void* ws,
                    size_t ws_bytes, cudaStream_t stream) {
  moe_status s = check_desc(d);
  if (s != MOE_OK) return s;
  if (T < 0 || (int64_t)T * d->k > (1 << 24)) return MOE_ERR_INVALID;
  if (!offsets || !active || !n_active) return MOE_ERR_INVALID;
  if (T > 0 && (!ids || !pairs)) return MOE_ERR_INVALID;
  if (x && (!x_sorted || !aligned(x, 16) || !aligned(x_sorted, 16) || d->H % 8)) return MOE_ERR_INVALID;
  const WsCarve c = carve(*d, T);
  if (c.sort > 0 && (!ws || ws_bytes < c.total)) return MOE_ERR_CAPACITY;
  void* scratch = c.sort > 0 ? static_cast<char*>(ws) + kWsControlBytes + c.tag : nullptr;
  return cuda_status(launch_sort(ids, x, T, d->k, d->E, d->H, offsets, pairs, active, n_active, x_sorted, scratch,
                                 stream));
}

// moe_route_sort_lookup that also publishes n_active and the active list to
// host_meta (page-locked host memory the device addresses at the same
// pointer; NULL: not at all) and then seq to host_meta[1] (used by the
// decode driver in place of a copy back and a stream synchronisation).
__attribute__((visibility("hidden"))) moe_status moe_internal_route_sort_lookup(
    const float* logits, int32_t T, const moe_layer_desc* d, float L, const int32_t* slot_table, int32_t n_shared,
    const float* shared_w, int32_t n_slots, int32_t* ids, float* w, int32_t* offsets, int32_t* pairs,
    int32_t* active, int32_t* n_active, int32_t* slots, int32_t* miss, int32_t* n_miss, int32_t* dev_err,
    cudaStream_t stream, int32_t* host_meta, int32_t seq) {
  moe_status s = check_desc(d);
  if (s != MOE_OK) return s;
  if (T < 0 || !(L >= 0.0f) || L > 1e30f || n_slots < 0 || n_shared < 0 || n_shared > kMaxShared)
    return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (T != 1 || d->k + n_shared > 32) return MOE_ERR_UNSUPPORTED;  // the widened layer, as moe_sort takes it
  if (!logits || !slot_table || !ids || !w || !offsets || !pairs || !active || !n_active || !slots || !miss ||
      !n_miss)
    return MOE_ERR_INVALID;
  return cuda_status(launch_route_sort_lookup(logits, d->E, d->k, L, slot_table, n_shared, shared_w, n_slots, ids, w,
                                              offsets, pairs, active, n_active, slots, miss, n_miss, dev_err,
                                              stream, host_meta, seq));
}

moe_status moe_route_sort_lookup(const float* logits, int32_t T, const moe_layer_desc* d, float L,
                                 const int32_t* slot_table, int32_t n_shared, const float* shared_w,
                                 int32_t n_slots, int32_t* ids, float* w, int32_t* offsets, int32_t* pairs,
                                 int32_t* active, int32_t* n_active, int32_t* slots, int32_t* miss,
                                 int32_t* n_miss, int32_t* dev_err, cudaStream_t stream) {
  return moe_internal_route_sort_lookup(logits, T, d, L, slot_table, n_shared, shared_w, n_slots, ids, w, offsets,
                                        pairs, active, n_active, slots, miss, n_miss, dev_err, stream, nullptr, 0);
}

moe_status moe_slot_lookup(const int32_t* slot_table, const int32_t* active, const int32_t* n_active,
                           int32_t pass_begin, int32_t pass_len, int32_t n_slots, int32_t* slots, int32_t* miss,
                           int32_t* n_miss, int32_t* dev_err, cudaStream_t stream) {
  if (!slot_table || !active || !n_active || !slots || !miss || !n_miss) return MOE_ERR_INVALID;
  if (pass_begin < 0 || pass_len < 0 || n_slots < 0) return MOE_ERR_INVALID;
  return cuda_status(launch_lookup(slot_table, active, n_active, pass_begin, pass_len, n_slots, slots, miss, n_miss,
                                   dev_err, stream));
}

moe_status moe_install_slots(void* pool, size_t slot_bytes, int32_t n_slots, const void* const* host_rows,
                             const int32_t* slots, int32_t n, cudaStream_t side, cudaEvent_t done) {
  if (n < 0) return MOE_ERR_INVALID;
  if (n > 0 && (!pool || !host_rows || !slots || slot_bytes == 0)) return MOE_ERR_INVALID;
  for (int32_t i = 0; i < n; ++i)
    if (slots[i] < 0 || slots[i] >= n_slots || !host_rows[i]) return MOE_ERR_INVALID;
  for (int32_t i = 0; i < n; ++i) {
    char* dst = static_cast<char*>(pool) + (size_t)slots[i] * slot_bytes;
    cudaError_t e = cudaMemcpyAsync(dst, host_rows[i], slot_bytes, cudaMemcpyHostToDevice, side);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (done && cudaEventRecord(done, side) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

// moe_expert_ffn with a choice of y semantics: overwrite = 1 writes y = the
// pass's result (used by the decode driver, whose single pass covers every
// active expert, so that y needs no separate zeroing); 0 adds to y.
__attribute__((visibility("hidden"))) moe_status moe_internal_expert_ffn(
    const uint16_t* x, int32_t T, const moe_layer_desc* d, const void* pool, int32_t n_slots,
    const int32_t* slot_table, const int32_t* ids, const float* w, const int32_t* offsets, const int32_t* pairs,
    const int32_t* active, const int32_t* n_active, const uint16_t* x_sorted, int32_t pass_begin, int32_t pass_len,
    float* y_accum, void* ws, size_t ws_bytes, int32_t* dev_err, cudaStream_t stream, int overwrite) {
  moe_status s = check_desc(d);
  if (s != MOE_OK) return s;
  if (T < 0 || pass_begin < 0 || pass_len < 0 || n_slots < 0) return MOE_ERR_INVALID;
  if (T == 0 || pass_len == 0) return MOE_OK;
  if (!x || !pool || !slot_table || !ids || !w || !offsets || !pairs || !active || !n_active || !y_accum)
    return MOE_ERR_INVALID;
  if (!aligned(pool, 256) || !aligned(x, 16) || !aligned(ws, 256)) return MOE_ERR_INVALID;
  if ((int64_t)T * d->k > (1 << 24)) return MOE_ERR_UNSUPPORTED;
  if (!ffn_decode_supported(*d)) return MOE_ERR_UNSUPPORTED;
  if (bf16_experts(*d) && (!x_sorted || !ffn_prefill_tc_shape_ok(*d))) return MOE_ERR_UNSUPPORTED;
  const WsCarve c = carve(*d, T, x_sorted != nullptr);
  if (!ws || ws_bytes < c.total) return MOE_ERR_CAPACITY;
  FfnArgs a{};
  a.x = x;
  a.T = T;
  a.E = d->E;
  a.k = d->k;
  a.H = d->H;
  a.I = d->I;
  a.g = d->group;
  a.pool = static_cast<const uint8_t*>(pool);
  a.L = make_layout(*d);
  a.slot_bytes = a.L.slot_bytes;
  a.n_slots = n_slots;
  a.table = slot_table;
  a.ids = ids;
  a.w = w;
  a.offsets = offsets;
  a.pairs = pairs;
  a.active = active;
  a.n_active = n_active;
  a.x_sorted = x_sorted;
  a.pass_begin = pass_begin;
  a.pass_len = pass_len;
  a.y = y_accum;
  a.ctl = static_cast<unsigned*>(ws);
  char* const scr = static_cast<char*>(ws) + kWsControlBytes + c.tag;  // sort | FFN scratch
  a.h = reinterpret_cast<uint16_t*>(scr);
  a.hpart = reinterpret_cast<float*>(scr + c.hb);
  a.o = c.o ? reinterpret_cast<float*>(scr + c.h) : nullptr;
  a.htag = static_cast<char*>(ws) + kWsControlBytes;
  a.dev_err = dev_err;
  a.y_overwrite = overwrite ? 1 : 0;
  a.wait_limit = wait_limit_cycles();
  return cuda_status(launch_ffn_decode(a, *d, device_sms(), stream));
}

moe_status moe_expert_ffn(const uint16_t* x, int32_t T, const moe_layer_desc* d, const void* pool, int32_t n_slots,
                          const int32_t* slot_table, const int32_t* ids, const float* w, const int32_t* offsets,
                          const int32_t* pairs, const int32_t* active, const int32_t* n_active,
                          const uint16_t* x_sorted, int32_t pass_begin, int32_t pass_len, float* y_accum, void* ws,
                          size_t ws_bytes, int32_t* dev_err, cudaStream_t stream) {
  return moe_internal_expert_ffn(x, T, d, pool, n_slots, slot_table, ids, w, offsets, pairs, active, n_active,
                                 x_sorted, pass_begin, pass_len, y_accum, ws, ws_bytes, dev_err, stream, 0);
}

moe_status moe_route_expert_ffn(const uint16_t* x, const float* logits, int32_t T, const moe_layer_desc* d, float L,
                                const void* pool, int32_t n_slots, const int32_t* slot_table, int32_t* ids, float* w,
                                int32_t* offsets, int32_t* pairs, int32_t* active, int32_t* n_active, int32_t* slots,
                                int32_t* miss, int32_t* n_miss, float* y, void* ws, size_t ws_bytes, int32_t* dev_err,
                                cudaStream_t stream) {
  moe_status s = check_desc(d);
  if (s != MOE_OK) return s;
  if (T < 1 || n_slots < 0 || !(L >= 0.0f) || L > 1e30f) return MOE_ERR_INVALID;
  if (!x || !logits || !pool || !slot_table || !ids || !w || !offsets || !pairs || !active || !n_active || !slots ||
      !miss || !n_miss || !y)
    return MOE_ERR_INVALID;
  if (!aligned(pool, 256) || !aligned(x, 16) || !aligned(ws, 256)) return MOE_ERR_INVALID;
  if (T != 1 || d->E > kRouteMaxExperts || bf16_experts(*d) || !ffn_decode_supported(*d)) return MOE_ERR_UNSUPPORTED;
  const WsCarve c = carve(*d, T, false);
  if (!ws || ws_bytes < c.total) return MOE_ERR_CAPACITY;
  FfnArgs a{};
  a.x = x;
  a.T = T;
  a.E = d->E;
  a.k = d->k;
  a.H = d->H;
  a.I = d->I;
  a.g = d->group;
  a.pool = static_cast<const uint8_t*>(pool);
  a.L = make_layout(*d);
  a.slot_bytes = a.L.slot_bytes;
  a.n_slots = n_slots;
  a.table = slot_table;
  a.pass_begin = 0;
  a.pass_len = d->E;
  a.y = y;
  a.ctl = static_cast<unsigned*>(ws);
  char* const scr = static_cast<char*>(ws) + kWsControlBytes + c.tag;
  a.h = reinterpret_cast<uint16_t*>(scr);
  a.hpart = reinterpret_cast<float*>(scr + c.hb);
  a.htag = static_cast<char*>(ws) + kWsControlBytes;
  a.dev_err = dev_err;
  a.y_overwrite = 1;
  a.wait_limit = wait_limit_cycles();
  a.logits = logits;
  a.route_L = L;
  a.r_ids = ids;
  a.r_w = w;
  a.r_offsets = offsets;
  a.r_pairs = pairs;
  a.r_active = active;
  a.r_n_active = n_active;
  a.r_slots = slots;
  a.r_miss = miss;
  a.r_n_miss = n_miss;
  const cudaError_t e = launch_ffn_route_fused(a, *d, device_sms(), stream);
  if (e == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
  return cuda_status(e);
}

moe_status moe_dequant_slot(const void* pool, int32_t slot, const moe_layer_desc* d, float* out_fp32,
                            uint16_t* out_bf16, cudaStream_t stream) {
  moe_status s = check_desc(d);
  if (s != MOE_OK) return s;
  if (!pool || slot < 0 || (!out_fp32 && !out_bf16)) return MOE_ERR_INVALID;
  const Layout L = make_layout(*d);
  const uint8_t* base = static_cast<const uint8_t*>(pool) + (int64_t)slot * L.slot_bytes;
  return cuda_status(launch_dequant_slot(base, *d, L, out_fp32, out_bf16, stream));
}

moe_status moe_quantize_rows(const float* w, int32_t rows, int32_t K, int32_t group, int32_t bits,
                             int32_t gate_up_I, uint8_t* proj, cudaStream_t stream) {
  if (rows < 0 || K < 1 || rows % 16) return MOE_ERR_INVALID;
  if (gate_up_I < 0 || (gate_up_I > 0 && (rows != 2 * gate_up_I || gate_up_I % 8))) return MOE_ERR_INVALID;
  if (group != 32 && group != 64 && group != 128) return MOE_ERR_UNSUPPORTED;
  if (bits != 3 && bits != 4 && bits != 6 && bits != 16) return MOE_ERR_UNSUPPORTED;
  if (K % group) return MOE_ERR_INVALID;
  if (rows == 0) return MOE_OK;
  if (!w || !proj || !aligned(proj, 16)) return MOE_ERR_INVALID;
  return cuda_status(launch_quantize(w, rows, K, group, bits, gate_up_I, proj, stream));
}

moe_status moe_router_logits(const uint16_t* x, int32_t T, const uint16_t* W, const float* bias, float scale,
                             int32_t E, int32_t H, float* logits, cudaStream_t stream) {
  if (T < 0 || E < 1 || H < 8 || H % 8 || !(scale == scale)) return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (!x || !W || !logits || !aligned(x, 16) || !aligned(W, 16)) return MOE_ERR_INVALID;
  if (T > 65535) return MOE_ERR_UNSUPPORTED;
  return cuda_status(launch_router(x, W, bias, scale, T, E, H, logits, stream));
}

moe_status moe_exp_portable(const float* x, int64_t n, float* out, cudaStream_t stream) {
  if (n < 0 || (n > 0 && (!x || !out))) return MOE_ERR_INVALID;
  return cuda_status(launch_exp(x, n, out, stream));
}

}  // extern "C"
