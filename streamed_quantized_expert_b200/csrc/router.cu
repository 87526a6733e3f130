// Router projection: logits[t][e] = scale * (x_t . W_e) + bias_e, bf16 x and
// W, fp32 accumulation.  The install-ahead path evaluates the routers of the
// next layers on the current hidden state with it (RFC "How the prototype
// works", item "Reads": the next two layers' experts are guessed by running
// their routers on the current hidden states).
//
// One warp per (token, expert): 16-byte loads of x and of the expert's row,
// the lanes' partial sums reduced by shuffles in a fixed order
// (deterministic).  The row of W is read once per token; decode-sized T
// makes this a plain HBM stream of E x H x 2 bytes.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void __launch_bounds__(256) router_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ W,
                                                     const float* __restrict__ bias, float scale, int T, int E,
                                                     int H, float* __restrict__ logits) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5), t = blockIdx.y;
  pdl_wait();
  pdl_launch_dependents();
  if (e >= E || t >= T) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  const uint4* wr = reinterpret_cast<const uint4*>(W + (size_t)e * H);
  float acc = 0.f;
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 a = __ldg(xr + c), b = __ldg(wr + c);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc = fmaf(bf16_lo(av[u]), bf16_lo(bv[u]), acc);
      acc = fmaf(bf16_hi(av[u]), bf16_hi(bv[u]), acc);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) logits[(size_t)t * E + e] = fmaf(scale, acc, bias ? bias[e] : 0.f);
}

cudaError_t launch_router(const uint16_t* x, const uint16_t* W, const float* bias, float scale, int T, int E, int H,
                          float* logits, cudaStream_t st) {
  const dim3 grid((unsigned)((E + 7) / 8), (unsigned)T);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, router_kernel, x, W, bias, scale, T, E, H, logits);
}

}  // namespace moe
