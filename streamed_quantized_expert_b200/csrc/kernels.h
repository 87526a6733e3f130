// Internal launcher declarations shared by the libmoe translation units.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"
#include "moe.h"

namespace moe {

constexpr int kFusedMaxTokens = 64;  // decode down kernel combines in shared memory up to this T
constexpr int kTcMinTokens = 1;  // with x_sorted the FFN runs on the tcgen05 grouped GEMM wherever the fused
                                 // decode kernel does not apply (it matches or beats the GEMV kernels at every
                                 // such T measured: 7 to 32 tokens, Flash- and Coder-like shapes)
constexpr int kMaxShared = 8;  // shared experts per layer (moe_route_shared)
// BF16 experts (a 16-bit projection): only the tensor-core grouped GEMM runs them
inline bool bf16_experts(const moe_layer_desc& d) { return d.bits_gu == 16 || d.bits_down == 16; }
constexpr int kRouteBlockMaxTokens = 64;  // up to this T, routing takes a block (8 warps) per token

struct FfnArgs {
  const uint16_t* x;
  int T;
  int E, k, H, I, g;
  const uint8_t* pool;
  int64_t slot_bytes;
  int n_slots;
  const int32_t* table;
  const int32_t* ids;
  const float* w;
  const int32_t* offsets;
  const int32_t* pairs;
  const int32_t* active;
  const int32_t* n_active;
  const uint16_t* x_sorted;
  int pass_begin, pass_len;
  float* y;
  uint16_t* h;    // workspace: [T*k][I] bf16 by sorted position (two-kernel path); the fused kernel
                  // uses [T*k][padded I] by flat pair, scaled by 2^-a of the down pair slot
  float* hpart;   // workspace: [T*k][padded I / 8] float pairs (unused by the fused kernel)
  void* htag;     // workspace (fused kernel): [T*k][padded I] 64-bit words (bf16 h, launch tag)
  float* o;     // workspace: [T*k][H] fp32, by flat pair index (T > kFusedMaxTokens)
  int32_t* dev_err;
  unsigned* ctl;    // workspace control block (the fused kernel's 64-bit launch ticket counter)
  int y_overwrite;  // 1: y = result (single pass over all experts); 0: y += result
  Layout L;
  // filled by the launcher
  int64_t q_gu, q_d, tile_gu, tile_d, rb_gu, rb_d;
  int ng_gu, ng_d, nblk_gu, nblk_d;
  int gu_stage_bytes, d_stage_bytes, gu_nstage, d_nstage;
  int xh_stage_bytes;  // fused kernel: shared region for x' and its sums, then (at h_stage_off) h
  int h_stage_off;
  long long wait_limit;  // clock-cycle limit of every bounded device wait (wait_limit_cycles())
  // route mode of the fused decode kernel (moe_route_expert_ffn, one token):
  // the kernel routes it from logits [E] itself (ids / w / offsets / pairs /
  // active / n_active above are then unused) and its CTA 0 writes the
  // routing, the sort and the slot lookup to the r_ buffers
  const float* logits;
  float route_L;
  int32_t* r_ids;
  float* r_w;
  int32_t* r_offsets;
  int32_t* r_pairs;
  int32_t* r_active;
  int32_t* r_n_active;
  int32_t* r_slots;
  int32_t* r_miss;
  int32_t* r_n_miss;
};
// experts a layer may have for the fused decode kernel to route its token itself
constexpr int kRouteMaxExperts = 1024;

// Launch with programmatic stream serialization, so the kernel's CTAs can be
// scheduled while the previous kernel in the stream drains; every kernel
// calls griddepcontrol.wait before reading what earlier kernels wrote.
template <typename... Args>
inline cudaError_t launch_pdl(const void* func, int grid, int block, size_t smem, cudaStream_t st,
                              const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* argv[] = {const_cast<void*>(static_cast<const void*>(&args))...};
  return cudaLaunchKernelExC(&cfg, func, argv);
}

cudaError_t launch_router(const uint16_t* x, const uint16_t* W, const float* bias, float scale, int T, int E, int H,
                          float* logits, cudaStream_t st);
cudaError_t launch_route(const float* logits, int T, int E, int k, float L, const int32_t* table, int32_t* ids,
                         float* w, int n_shared, const float* shared_w, cudaStream_t st);
size_t sort_ws_bytes(int n, int E);
cudaError_t launch_sort(const int32_t* ids, const uint16_t* x, int T, int k, int E, int H, int32_t* offsets,
                        int32_t* pairs, int32_t* active, int32_t* n_active, uint16_t* x_sorted, void* ws,
                        cudaStream_t st);
cudaError_t launch_lookup(const int32_t* table, const int32_t* active, const int32_t* n_active, int pass_begin,
                          int pass_len, int n_slots, int32_t* slots, int32_t* miss, int32_t* n_miss,
                          int32_t* dev_err, cudaStream_t st);
cudaError_t launch_route_sort_lookup(const float* logits, int E, int k, float L, const int32_t* table, int ns,
                                     const float* sw, int n_slots, int32_t* ids, float* w, int32_t* offsets,
                                     int32_t* pairs, int32_t* active, int32_t* n_active, int32_t* slots,
                                     int32_t* miss, int32_t* n_miss, int32_t* dev_err, cudaStream_t st,
                                     int32_t* host_meta = nullptr, int32_t seq = 0);
cudaError_t launch_exp(const float* x, int64_t n, float* out, cudaStream_t st);
cudaError_t launch_quantize(const float* w, int rows, int K, int g, int b, int gu_I, uint8_t* q, cudaStream_t st);
cudaError_t launch_dequant_slot(const uint8_t* slot, const moe_layer_desc& d, const Layout& L, float* out32,
                                uint16_t* out16, cudaStream_t st);
bool ffn_decode_supported(const moe_layer_desc& d);
cudaError_t launch_ffn_decode(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st);
cudaError_t launch_ffn_route_fused(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st);
cudaError_t launch_ffn_fused(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st);
cudaError_t launch_ffn_prefill_tc(const FfnArgs& a, const moe_layer_desc& d, int num_sms, cudaStream_t st);
bool ffn_fused_plan(FfnArgs& a, const moe_layer_desc& d, int num_sms, size_t& smem);
bool ffn_prefill_tc_shape_ok(const moe_layer_desc& d);
int ffn_kernel_path(const moe_layer_desc& d, int T, bool has_x_sorted, int num_sms);
__global__ void combine_kernel(const FfnArgs a);
int combine_grid(int T, int H, int num_sms);
constexpr size_t kWsControlBytes = 512;  // head of the workspace: the fused kernel's launch ticket counter
constexpr long long kDefaultWaitCycles = 4000000000ll;  // about 2 s at the top SM clock
// Limit of the bounded device waits of kernels launched from now on
// (moe_set_wait_limit_cycles; kDefaultWaitCycles unless a test lowered it).
long long wait_limit_cycles();

}  // namespace moe
