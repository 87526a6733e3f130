// Device helpers shared by the decode FFN kernels (two-kernel and fused).
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRedBatch = 8;          // (item, token tile) entries reduced across warps at a time
constexpr int kDenseMaxTokens = 8;    // T <= 8: every token gets its own MMA column
constexpr int kMaxCtaExperts = 64;    // per-CTA expert metadata table
constexpr int kHStageMax = 24 * 1024; // h staged in shared memory up to this many bytes
constexpr int kDnKSplit = 4;          // down: warps split K four ways, the rest take experts in turn
constexpr int kFuConsumers = 16;      // fused kernel consumer warps

struct RedMeta {
  int ei;    // CTA-local expert index
  int pos;   // first sorted position of the token tile (tile mode)
  int ntok;  // tokens in the tile
  int jt;    // 8-row tile of the intermediate dimension
};

struct ExpMeta {
  int e;     // expert id
  int slot;  // slot in the pool (may be invalid: the expert is skipped)
  int pos0;  // first sorted position of the expert's pairs
  int cnt;   // pairs routed to the expert
};

template <int B>
__device__ __forceinline__ void load_unit(const uint8_t* p, uint32_t (&w)[B]) {
  if constexpr (B == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x;
    w[1] = v.y;
    w[2] = v.z;
    w[3] = v.w;
  } else if constexpr (B == 6) {
    const uint2* q = reinterpret_cast<const uint2*>(p);
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const uint2 v = q[i];
      w[2 * i] = v.x;
      w[2 * i + 1] = v.y;
    }
  } else {
    const uint32_t* q = reinterpret_cast<const uint32_t*>(p);
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = q[i];
  }
}

__device__ __forceinline__ uint32_t bf2_scale_eighth(uint32_t v) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v);
  h = __hmul2(h, __floats2bfloat162_rn(0.125f, 0.125f));
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t ld_pair(const uint16_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

// B fragments (x of the token in column g8, scaled by 2^-a) for one 128-block
// and the per-group sums sum x and sum 128 x 2^-a, delivered for the two
// token columns this thread's C fragment covers (2 t4, 2 t4 + 1).
template <int B, int GS>
__device__ __forceinline__ void load_b_block(const uint16_t* row, int kb, int K, int t4, uint32_t (&bf)[8][2],
                                             float (&xs)[8 / GS][2], float (&xo)[8 / GS][2]) {
  float sx[8 / GS], so[8 / GS];
#pragma unroll
  for (int G = 0; G < 8 / GS; ++G) sx[G] = so[G] = 0.0f;
  // all sixteen loads first, so that they are in flight together
  uint32_t vv[8][2];
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int klo = kb * 128 + 16 * s + 2 * t4, khi = klo + 8;
    vv[s][0] = (row != nullptr && klo < K) ? ld_pair(row + klo) : 0u;
    vv[s][1] = (row != nullptr && khi < K) ? ld_pair(row + khi) : 0u;
  }
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    uint32_t v0 = vv[s][0], v1 = vv[s][1];
    const float x0 = bf16_lo(v0) + bf16_hi(v0), x1 = bf16_lo(v1) + bf16_hi(v1);
    if (PairShift<B>::a(2 * s) == 3) v0 = bf2_scale_eighth(v0);
    if (PairShift<B>::a(2 * s + 1) == 3) v1 = bf2_scale_eighth(v1);
    bf[s][0] = v0;
    bf[s][1] = v1;
    sx[s / GS] += x0 + x1;
    so[s / GS] += 128.0f * (bf16_lo(v0) + bf16_hi(v0) + bf16_lo(v1) + bf16_hi(v1));
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int G = 0; G < 8 / GS; ++G) {
    sx[G] += __shfl_xor_sync(0xffffffffu, sx[G], 1);
    sx[G] += __shfl_xor_sync(0xffffffffu, sx[G], 2);
    so[G] += __shfl_xor_sync(0xffffffffu, so[G], 1);
    so[G] += __shfl_xor_sync(0xffffffffu, so[G], 2);
    xs[G][0] = __shfl_sync(0xffffffffu, sx[G], 8 * (lane & 3));
    xs[G][1] = __shfl_sync(0xffffffffu, sx[G], 8 * (lane & 3) + 4);
    xo[G][0] = __shfl_sync(0xffffffffu, so[G], 8 * (lane & 3));
    xo[G][1] = __shfl_sync(0xffffffffu, so[G], 8 * (lane & 3) + 4);
  }
}

// Offset of this thread's unit (unit t4 of block 0, row g8) inside an 8-row
// group in shared memory; block kb adds kb * 32 units.
template <int B>
__device__ __forceinline__ int thread_unit_off(int t4, int g8) {
  return (8 * t4 + unit_sigma<B>(t4, g8)) * 4 * B;
}

// One 128-block of a 16-row tile: 8-row groups ga (A rows 0-7) and gb (rows
// 8-15) in shared memory; uoff = thread_unit_off; sbA / sbB point at the
// tile's (scale, bias) words of rows g8 / 8+g8 (group gi at [16 gi]);
// accumulate the group epilogues into acc.
template <int B, int GS>
__device__ __forceinline__ void block_mma(const uint8_t* ga, const uint8_t* gb, const uint32_t* sbA,
                                          const uint32_t* sbB, int kb, int uoff, const uint32_t (&bf)[8][2],
                                          const float (&xs)[8 / GS][2], const float (&xo)[8 / GS][2],
                                          float (&acc)[4]) {
  uint32_t wa[B], wb[B], pa[16], pb[16];
  load_unit<B>(ga + kb * 128 * B + uoff, wa);
  load_unit<B>(gb + kb * 128 * B + uoff, wb);
  unpack_unit<B>(wa, pa);
  unpack_unit<B>(wb, pb);
#pragma unroll
  for (int G = 0; G < 8 / GS; ++G) {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ss = 0; ss < GS; ++ss) {
      const int s = G * GS + ss;
      const uint32_t af[4] = {pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1]};
      mma_bf16(d, af, bf[s][0], bf[s][1]);
    }
    const int gi = kb * (8 / GS) + G;
    const uint32_t wA = sbA[gi * 16], wB = sbB[gi * 16];
    const float sA = bf16_lo(wA), bA = bf16_hi(wA), sB = bf16_lo(wB), bB = bf16_hi(wB);
    acc[0] += sA * (d[0] - xo[G][0]) + bA * xs[G][0];
    acc[1] += sA * (d[1] - xo[G][1]) + bA * xs[G][1];
    acc[2] += sB * (d[2] - xo[G][0]) + bB * xs[G][0];
    acc[3] += sB * (d[3] - xo[G][1]) + bB * xs[G][1];
  }
}

__device__ __forceinline__ int pass_count(const FfnArgs& a) {
  int n = *a.n_active - a.pass_begin;
  if (n > a.pass_len) n = a.pass_len;
  return n > 0 ? n : 0;
}

__device__ __forceinline__ bool slot_ok(const FfnArgs& a, int slot) { return slot >= 0 && slot < a.n_slots; }

__device__ __forceinline__ void flag_slot(const FfnArgs& a, int slot) {
  if (a.dev_err) atomicOr(a.dev_err, slot < 0 ? MOE_DEV_ERR_NOT_RESIDENT : MOE_DEV_ERR_SLOT_RANGE);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Named barrier over the consumer warps only (the producer warp never joins).
__device__ __forceinline__ void consumers_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Thread i (of nthreads) fills meta[i] for pass entry first + i; in dense mode
// also tokpos[i][t] = sorted position of (expert, token t) or -1, and (if
// wtab) wtab[i][t] = its routing weight (0 if absent).  The loads of all
// entries are independent, so the table costs a couple of L2 round trips.
template <bool DENSE>
__device__ __forceinline__ void load_expert_meta(const FfnArgs& a, int first, int n, ExpMeta* meta, int* tokpos,
                                                 float* wtab, int nthreads) {
  for (int i = threadIdx.x; i < n; i += nthreads) {
    const int e = a.active[a.pass_begin + first + i];
    ExpMeta m;
    m.e = e;
    m.slot = a.table[e];
    m.pos0 = a.offsets[e];
    m.cnt = a.offsets[e + 1] - m.pos0;
    meta[i] = m;
    if (DENSE) {
      for (int t = 0; t < kDenseMaxTokens; ++t) {
        tokpos[i * kDenseMaxTokens + t] = -1;
        if (wtab) wtab[i * kDenseMaxTokens + t] = 0.f;
      }
      for (int p = m.pos0; p < m.pos0 + m.cnt; ++p) {
        const int pf = a.pairs[p];
        const int t = pf / a.k;
        tokpos[i * kDenseMaxTokens + t] = p;
        if (wtab) wtab[i * kDenseMaxTokens + t] = a.w[pf];
      }
    }
  }
}

// T <= 8 tokens with every routed pair fitting the per-CTA tables: one MMA
// column per token for every expert.
inline bool dense_mode(const FfnArgs& a) { return a.T <= kDenseMaxTokens && a.T * a.k <= kMaxCtaExperts; }

// Opt a kernel into the large dynamic shared-memory carve-out once per
// (kernel, device); the attribute call is not free on the launch path.  Each
// caller passes its own flag word (one per kernel instantiation).
inline cudaError_t ensure_smem_attr(const void* kern, int (&done_mask)[4]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 128 && ((__atomic_load_n(&done_mask[dev >> 5], __ATOMIC_RELAXED) >> (dev & 31)) & 1)) return cudaSuccess;
  // dynamic limit = the device's per-block opt-in maximum minus the kernel's static shared memory
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaFuncAttributes fa;
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kern);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
  // the whole carve-out as shared memory
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e == cudaSuccess && dev < 128) __atomic_fetch_or(&done_mask[dev >> 5], 1 << (dev & 31), __ATOMIC_RELAXED);
  return e;
}


}  // namespace moe
