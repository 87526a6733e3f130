// Quantization into the slot row format (input preparation: the RFC's
// one-time quantize_experts, which writes experts in MLX's affine format; and
// the rounding of BF16 experts to their bf16 rows) and the test-only
// dequantisation of a slot through the FFN's code unpackers.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// Word index (unit p * b + word in unit) and bit of code bit j of input kk of
// a 128-input block.
__device__ __forceinline__ void block_bit(int kk, int b, int j, int& word, int& bit) {
  const int s = kk >> 4, r16 = kk & 15;
  const int h = r16 >> 3, p = (r16 & 7) >> 1;
  const int i = 2 * s + h;
  int wi, bi;
  if (b == 4) {
    wi = i >> 2;
    bi = 4 * (i & 3) + j;
  } else if (b == 3) {
    if (i < 15) {
      wi = i / 5;
      bi = 3 * (i % 5) + j;
    } else {
      wi = j;
      bi = 15;
    }
  } else {
    if (i < 12) {
      wi = i >> 1;
      bi = 6 * (i & 1) + j;
    } else if (j < 4) {
      wi = i - 12;
      bi = 12 + j;
    } else {
      wi = 4 + ((i - 12) >> 1);
      bi = 12 + 2 * ((i - 12) & 1) + (j - 4);
    }
  }
  word = p * b + wi;
  bit = bi + ((kk & 1) ? 16 : 0);
}

__device__ __forceinline__ int64_t unit_off(int b, int64_t row, int64_t u, int64_t rb, int64_t tile) {
  return b == 3 ? unit_offset<3>(row, u, rb, tile) : b == 4 ? unit_offset<4>(row, u, rb, tile)
                                                            : unit_offset<6>(row, u, rb, tile);
}

// One warp per (row, 128-block); lane owns inputs 4*lane .. 4*lane+3.
// gu_I > 0: the rows are a gate/up matrix (gate rows 0..gu_I-1, then up
// rows), written to their storage rows; else row r is storage row r.
__global__ void __launch_bounds__(256) quantize_kernel(const float* __restrict__ w, int rows, int K, int g, int b,
                                                       int gu_I, uint8_t* __restrict__ q) {
  __shared__ uint32_t s_words[8][24];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = (int)(padded_k(K) / 128);
  const int64_t task = (int64_t)blockIdx.x * 8 + warp;
  if (task >= (int64_t)rows * nblk) return;
  const int r = (int)(task / nblk), blk = (int)(task % nblk);
  const int k0 = blk * 128 + 4 * lane;
  float v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = (k0 + i < K) ? w[(int64_t)r * K + k0 + i] : 0.0f;
  // group min / max over the g/4 lanes of the group
  float mn = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
  float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
  const int lanes_per_group = g / 4;
  for (int o = 1; o < lanes_per_group; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const int qmax = (1 << b) - 1;
  const bool group_padded = (blk * 128 + (lane / lanes_per_group) * g) >= K;
  uint16_t sh = 0, bh = 0;
  if (!group_padded) {
    sh = f32_to_bf16_rne(__fdiv_rn(__fsub_rn(mx, mn), (float)qmax));
    bh = f32_to_bf16_rne(mn);
  }
  const float sf = __uint_as_float((uint32_t)sh << 16), bf = __uint_as_float((uint32_t)bh << 16);
  if (lane < 4 * b) s_words[warp][lane] = 0u;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int code = 0;
    if (!group_padded && k0 + i < K && sf != 0.0f) {
      float t = rintf(__fdiv_rn(__fsub_rn(v[i], bf), sf));
      t = fminf(fmaxf(t, 0.0f), (float)qmax);
      code = (int)t;
    }
    for (int j = 0; j < b; ++j) {
      if ((code >> j) & 1) {
        int word, bit;
        block_bit(4 * lane + i, b, j, word, bit);
        atomicOr(&s_words[warp][word], 1u << bit);
      }
    }
  }
  __syncwarp();
  const int64_t rb = row_bytes(K, b), tile = tile_bytes(K, g, b);
  const int srow = gu_I > 0 ? gate_up_row(r, gu_I) : r;
  if (lane < 4 * b) {
    const int p = lane / b, wi = lane % b;
    reinterpret_cast<uint32_t*>(q + unit_off(b, srow, 4 * blk + p, rb, tile))[wi] = s_words[warp][lane];
  }
  if (lane % lanes_per_group == 0) {
    const int gi = (blk * 128 + 4 * lane) / g;
    *reinterpret_cast<uint32_t*>(q + sb_offset(srow, gi, rb, tile)) = (uint32_t)sh | ((uint32_t)bh << 16);
  }
}

// BF16 experts: the rows rounded to bf16 (nearest even), row-major in storage
// row order, each row padded with zeros to whole 128-input blocks.  One thread
// per (row, pair of inputs).
__global__ void __launch_bounds__(256) bf16_rows_kernel(const float* __restrict__ w, int rows, int K, int gu_I,
                                                        uint8_t* __restrict__ q) {
  const int Kp = (int)padded_k(K);
  const int64_t task = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (task >= (int64_t)rows * (Kp / 2)) return;
  const int r = (int)(task / (Kp / 2)), k = 2 * (int)(task % (Kp / 2));
  const float v0 = k < K ? w[(int64_t)r * K + k] : 0.0f, v1 = k + 1 < K ? w[(int64_t)r * K + k + 1] : 0.0f;
  const int srow = gu_I > 0 ? gate_up_row(r, gu_I) : r;
  reinterpret_cast<uint32_t*>(q + (int64_t)srow * Kp * 2)[k / 2] =
      (uint32_t)f32_to_bf16_rne(v0) | ((uint32_t)f32_to_bf16_rne(v1) << 16);
}

// BF16 experts (test): the stored values, logical row order.
__global__ void bf16_dequant_kernel(const uint8_t* __restrict__ qbase, int rows, int K, int gu_I,
                                    float* __restrict__ out32, uint16_t* __restrict__ out16) {
  const int64_t task = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (task >= (int64_t)rows * K) return;
  const int lr = (int)(task / K), k = (int)(task % K);
  const int r = gu_I > 0 ? gate_up_row(lr, gu_I) : lr;
  const uint16_t v = reinterpret_cast<const uint16_t*>(qbase + (int64_t)r * padded_k(K) * 2)[k];
  if (out32) out32[task] = __uint_as_float((uint32_t)v << 16);
  if (out16) out16[task] = v;
}

// Dequantise rows of one projection: one thread per (storage row, unit),
// through the same unpack_unit<B> the FFN kernels use.  out[r][k] = fmaf(s,
// q, b), r the logical row (gu_I > 0: gate/up row order).
template <int B>
__global__ void dequant_kernel(const uint8_t* __restrict__ qbase, int rows, int K, int g, int gu_I,
                               float* __restrict__ out32, uint16_t* __restrict__ out16) {
  const int nunit = (int)(padded_k(K) / 32);
  const int64_t task = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (task >= (int64_t)rows * nunit) return;
  const int lr = (int)(task / nunit), u = (int)(task % nunit);
  const int r = gu_I > 0 ? gate_up_row(lr, gu_I) : lr;  // storage row
  const int blk = u >> 2, t = u & 3;
  const int64_t rb = row_bytes(K, B), tile = tile_bytes(K, g, B);
  const uint32_t* wp = reinterpret_cast<const uint32_t*>(qbase + unit_offset<B>(r, u, rb, tile));
  uint32_t wv[B];
#pragma unroll
  for (int i = 0; i < B; ++i) wv[i] = wp[i];
  uint32_t p[16];
  unpack_unit<B>(wv, p);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int a = PairShift<B>::a(i);
    const int k = blk * 128 + pair_input(i, t);
    if (k >= K) continue;  // K is a multiple of 32, so k+1 < K too
    const uint32_t sbw = *reinterpret_cast<const uint32_t*>(qbase + sb_offset(r, k / g, rb, tile));
    const float s = bf16_lo(sbw), bb = bf16_hi(sbw);
    const float v0 = __fmaf_rn(s, pair_lo_q(p[i], a), bb);
    const float v1 = __fmaf_rn(s, pair_hi_q(p[i], a), bb);
    if (out32) {
      out32[(int64_t)lr * K + k] = v0;
      out32[(int64_t)lr * K + k + 1] = v1;
    }
    if (out16) {
      out16[(int64_t)lr * K + k] = f32_to_bf16_rne(v0);
      out16[(int64_t)lr * K + k + 1] = f32_to_bf16_rne(v1);
    }
  }
}

template <int B>
static void launch_dq(const uint8_t* q, int rows, int K, int g, int gu_I, float* o32, uint16_t* o16,
                      cudaStream_t st) {
  const int64_t n = (int64_t)rows * (padded_k(K) / 32);
  dequant_kernel<B><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(q, rows, K, g, gu_I, o32, o16);
}

static void dq_dispatch(int b, const uint8_t* q, int rows, int K, int g, int gu_I, float* o32, uint16_t* o16,
                        cudaStream_t st) {
  if (b == 3) launch_dq<3>(q, rows, K, g, gu_I, o32, o16, st);
  else if (b == 4) launch_dq<4>(q, rows, K, g, gu_I, o32, o16, st);
  else if (b == 6) launch_dq<6>(q, rows, K, g, gu_I, o32, o16, st);
  else {
    const int64_t n = (int64_t)rows * K;
    bf16_dequant_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(q, rows, K, gu_I, o32, o16);
  }
}

cudaError_t launch_dequant_slot(const uint8_t* slot, const moe_layer_desc& d, const Layout& L, float* out32,
                                uint16_t* out16, cudaStream_t st) {
  const int64_t n_gu = (int64_t)2 * d.I * d.H;
  dq_dispatch(d.bits_gu, slot + L.gu, 2 * d.I, d.H, d.group, d.I, out32, out16, st);
  dq_dispatch(d.bits_down, slot + L.d, d.H, d.I, d.group, 0, out32 ? out32 + n_gu : nullptr,
              out16 ? out16 + n_gu : nullptr, st);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const float* w, int rows, int K, int g, int b, int gu_I, uint8_t* q, cudaStream_t st) {
  if (b == 16) {
    const int64_t n = (int64_t)rows * (padded_k(K) / 2);
    if (n == 0) return cudaSuccess;
    bf16_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(w, rows, K, gu_I, q);
    return cudaGetLastError();
  }
  const int64_t tasks = (int64_t)rows * (padded_k(K) / 128);
  if (tasks == 0) return cudaSuccess;
  quantize_kernel<<<(unsigned)((tasks + 7) / 8), 256, 0, st>>>(w, rows, K, g, b, gu_I, q);
  return cudaGetLastError();
}

}  // namespace moe
