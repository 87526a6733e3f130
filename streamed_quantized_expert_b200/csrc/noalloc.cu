// moe_expert_ffn_noalloc: moe_expert_ffn with its scratch in a fixed device
// array, for callers that cannot allocate device memory themselves.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes that
// every GPU loading this library holds until the process exits.  In host code
// the array's name is only a host-side stand-in: its device address is looked
// up once per device with cudaGetSymbolAddress (with that device current) on
// the first call made on that device, and then passed to the kernels.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB
static __device__ __align__(256) uint8_t g_ffn_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

moe_status scratch_of_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ffn_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" size_t moe_internal_workspace_bytes_no_tc(const moe_layer_desc* d, int32_t max_tokens);
extern "C" size_t moe_internal_workspace_persistent_bytes(const moe_layer_desc* d);

extern "C" size_t moe_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" moe_status moe_expert_ffn_noalloc(const uint16_t* x, int32_t T, const moe_layer_desc* d,
                                             const void* pool, int32_t n_slots, const int32_t* slot_table,
                                             const int32_t* ids, const float* w, const int32_t* offsets,
                                             const int32_t* pairs, const int32_t* active, const int32_t* n_active,
                                             int32_t pass_begin, int32_t pass_len, float* y_accum,
                                             int32_t* dev_err, cudaStream_t stream) {
  const size_t need = moe_internal_workspace_bytes_no_tc(d, T);  // no x_sorted is passed below
  if (need == 0 || T < 0) return MOE_ERR_INVALID;
  if (T > moe::kFusedMaxTokens || need > kNoAllocScratchBytes) return MOE_ERR_CAPACITY;
  void* scratch = nullptr;
  const moe_status s = scratch_of_current_device(&scratch);
  if (s != MOE_OK) return s;
  // The array keeps whatever the previous call (on any stream, with any
  // layer description) left in it.  Its head -- the control block and the
  // tagged h words, which a workspace keeps from call to call -- is cleared
  // in stream order, so that every call starts from a zeroed workspace and
  // depends on no earlier one.
  const size_t head = moe_internal_workspace_persistent_bytes(d);
  if (head == 0 || head > need) return MOE_ERR_INVALID;
  if (cudaMemsetAsync(scratch, 0, head, stream) != cudaSuccess) return MOE_ERR_CUDA;
  return moe_expert_ffn(x, T, d, pool, n_slots, slot_table, ids, w, offsets, pairs, active, n_active, nullptr,
                        pass_begin, pass_len, y_accum, scratch, kNoAllocScratchBytes, dev_err, stream);
}
