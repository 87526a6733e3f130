// Shared device helpers for libmoe (sm_100a).
//
// Slot format: see include/moe.h.  This header holds the layout arithmetic,
// the packed-code unpackers used by every kernel that reads a slot, and thin
// inline-PTX wrappers (mbarrier, bulk async copy, HMMA).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------------------
// Layout
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }
__host__ __device__ constexpr int64_t padded_k(int64_t K) { return round_up(K, 128); }
__host__ __device__ constexpr int64_t row_bytes(int64_t K, int bits) { return padded_k(K) * bits / 8; }
__host__ __device__ constexpr int64_t row_groups(int64_t K, int g) { return padded_k(K) / g; }

struct Layout {
  int64_t gu, d;            // byte offsets of the gate_up and down projections in a slot
  int64_t rb_gu, rb_d;      // code bytes of one row
  int ng_gu, ng_d;          // (scale, bias) groups per (padded) row
  int nblk_gu, nblk_d;      // 128-input blocks per row
  int64_t tile_gu, tile_d;  // bytes of one 16-row tile: codes, then scale/bias words
  int64_t slot_bytes;
};

// bits = 16: unquantized BF16 experts, rows of bf16 values (row-major, padded
// to whole 128-input blocks with zeros), no (scale, bias) words.
__host__ __device__ constexpr int64_t tile_bytes(int64_t K, int g, int bits) {
  return 16 * row_bytes(K, bits) + (bits == 16 ? 0 : 16 * row_groups(K, g) * 4);
}

inline Layout make_layout(const moe_layer_desc& d) {
  Layout L{};
  L.rb_gu = row_bytes(d.H, d.bits_gu);
  L.rb_d = row_bytes(d.I, d.bits_down);
  L.ng_gu = (int)row_groups(d.H, d.group);
  L.ng_d = (int)row_groups(d.I, d.group);
  L.nblk_gu = (int)(padded_k(d.H) / 128);
  L.nblk_d = (int)(padded_k(d.I) / 128);
  L.tile_gu = tile_bytes(d.H, d.group, d.bits_gu);
  L.tile_d = tile_bytes(d.I, d.group, d.bits_down);
  L.gu = 0;
  L.d = round_up((int64_t)(2 * d.I / 16) * L.tile_gu, 256);
  L.slot_bytes = round_up(L.d + (int64_t)(d.H / 16) * L.tile_d, 256);
  return L;
}

// ---------------------------------------------------------------------------
// Packed codes -> bf16 pairs
// ---------------------------------------------------------------------------
// A unit holds 16 input pairs.  unpack_unit<B> turns the unit's B words into
// 16 registers, register i = bf16x2 (low: even input, high: odd input) with
// value 128 + q * 2^a(i) in each half: the code lands in the low mantissa
// bits of bf16 128.0 (0x4300), at bit offset a(i) (0 or 3).  Consumers either
// subtract the offset per group (tensor-core GEMV) or convert to the exact q.
constexpr uint32_t kMagic = 0x43004300u;
// The same codes under the fp16 magic 1024.0 (0x6400): 1024 + q * 2^a in each
// half (q * 2^a < 1024 for every width), for fp16 tensor-core operands.
constexpr uint32_t kMagic16 = 0x64006400u;

// (a & mask) | c  in one LOP3 (truth table 0xEA = (A & B) | C).
template <uint32_t MASK>
__device__ __forceinline__ uint32_t andor(uint32_t a, uint32_t c) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "n"(MASK), "r"(c));
  return r;
}

template <int B>
struct PairShift;  // a(i): 0 or 3 per pair index

template <>
struct PairShift<4> {
  static __host__ __device__ constexpr int a(int i) { return (i % 4) & 1 ? 3 : 0; }
};
template <>
struct PairShift<3> {
  static __host__ __device__ constexpr int a(int i) { return (i < 15 && ((i % 5) == 1 || (i % 5) == 3)) ? 3 : 0; }
};
template <>
struct PairShift<6> {
  static __host__ __device__ constexpr int a(int) { return 0; }
};

template <int B, uint32_t M = kMagic>
struct Unpack;

template <int B, uint32_t M = kMagic>
__device__ __forceinline__ void unpack_unit(const uint32_t (&w)[B], uint32_t (&p)[16]) {
  Unpack<B, M>::run(w, p);
}

template <uint32_t kMagic>
struct Unpack<4, kMagic> {
static __device__ __forceinline__ void run(const uint32_t (&w)[4], uint32_t (&p)[16]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t v = w[k];
    const uint32_t v8 = v >> 8;
    p[4 * k + 0] = andor<0x000F000Fu>(v, kMagic);       // bits 0..3, a = 0
    p[4 * k + 1] = andor<0x00780078u>(v >> 1, kMagic);  // bits 4..7 -> 3..6, a = 3
    p[4 * k + 2] = andor<0x000F000Fu>(v8, kMagic);      // bits 8..11 -> 0..3, a = 0
    p[4 * k + 3] = andor<0x00780078u>(v8 >> 1, kMagic); // bits 12..15 -> 3..6, a = 3
  }
}
};

template <uint32_t kMagic>
struct Unpack<3, kMagic> {
static __device__ __forceinline__ void run(const uint32_t (&w)[3], uint32_t (&p)[16]) {
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const uint32_t v = w[k];
    const uint32_t v6 = v >> 6;
    p[5 * k + 0] = andor<0x00070007u>(v, kMagic);        // bits 0..2, a = 0
    p[5 * k + 1] = andor<0x00380038u>(v, kMagic);        // bits 3..5, a = 3
    p[5 * k + 2] = andor<0x00070007u>(v6, kMagic);       // bits 6..8 -> 0..2, a = 0
    p[5 * k + 3] = andor<0x00380038u>(v6, kMagic);       // bits 9..11 -> 3..5, a = 3
    p[5 * k + 4] = andor<0x00070007u>(v >> 12, kMagic);  // bits 12..14 -> 0..2, a = 0
  }
  // pair 15: code bit j is bit 15 (31) of word j
  uint32_t t = andor<0x00010001u>(w[0] >> 15, kMagic);
  t = andor<0x00020002u>(w[1] >> 14, t);
  p[15] = andor<0x00040004u>(w[2] >> 13, t);
}
};

template <uint32_t kMagic>
struct Unpack<6, kMagic> {
static __device__ __forceinline__ void run(const uint32_t (&w)[6], uint32_t (&p)[16]) {
#pragma unroll
  for (int k = 0; k < 6; ++k) {
    p[2 * k + 0] = andor<0x003F003Fu>(w[k], kMagic);       // bits 0..5
    p[2 * k + 1] = andor<0x003F003Fu>(w[k] >> 6, kMagic);  // bits 6..11
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    // low 4 code bits at 12..15 of word m; high 2 at 12+2(m%2).. of word 4+m/2
    uint32_t t = andor<0x000F000Fu>(w[m] >> 12, kMagic);
    p[12 + m] = andor<0x00300030u>(w[4 + m / 2] >> (8 + 2 * (m % 2)), t);
  }
}
};

// bf16x2 (128 + q*2^a) -> exact q of the low / high half as float.
__device__ __forceinline__ float pair_lo_q(uint32_t p, int a) {
  return (__uint_as_float(p << 16) - 128.0f) * (a ? 0.125f : 1.0f);
}
__device__ __forceinline__ float pair_hi_q(uint32_t p, int a) {
  return (__uint_as_float(p & 0xFFFF0000u) - 128.0f) * (a ? 0.125f : 1.0f);
}

// Rows are stored in tiles of 16 (codes of two 8-row groups, then the tile's
// scale/bias words).  Inside a group (unit-major) unit u of row r sits at unit
// position 8u + sigma(u, r), which keeps the per-thread unit loads of the GEMV
// kernels free of shared-memory bank conflicts.
template <int B>
__host__ __device__ constexpr int unit_sigma(int u, int r) {
  return B == 3 ? r : B == 4 ? (r + 2 * (u & 3)) & 7 : (r + 4 * ((u >> 1) & 1)) & 7;
}

// Byte offset of unit u of row `row` from the start of its projection.
template <int B>
__host__ __device__ constexpr int64_t unit_offset(int64_t row, int64_t u, int64_t row_bytes, int64_t tile) {
  return (row >> 4) * tile + ((row >> 3) & 1) * 8 * row_bytes + (8 * u + unit_sigma<B>((int)u, (int)(row & 7))) * 4 * B;
}

// Byte offset of the (scale, bias) word of (row, group gi) from the start of
// its projection: group-major inside the row's tile, after the tile's codes.
__host__ __device__ constexpr int64_t sb_offset(int64_t row, int64_t gi, int64_t row_bytes, int64_t tile) {
  return (row >> 4) * tile + 16 * row_bytes + 4 * (gi * 16 + (row & 15));
}

// Storage row of logical gate/up row R (blocks of 16: 8 gate rows, 8 up rows).
__host__ __device__ constexpr int gate_up_row(int R, int I) {
  return 16 * ((R < I ? R : R - I) >> 3) + (R < I ? 0 : 8) + ((R < I ? R : R - I) & 7);
}

// Logical input (within a 128-block) of register i's even member for unit t:
// i = 2s + h  ->  16s + 2t + 8h.
__host__ __device__ constexpr int pair_input(int i, int t) { return 16 * (i >> 1) + 2 * t + 8 * (i & 1); }

// ---------------------------------------------------------------------------
// bf16 helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// fp32 -> fp16 bits, round to nearest even, saturating at +-65504 (the
// tensor-core path's operands: sorted activations and h).
__device__ __forceinline__ uint16_t f32_to_f16_sat(float f) {
  f = fminf(fmaxf(f, -65504.0f), 65504.0f);
  return __half_as_ushort(__float2half_rn(f));
}

// ---------------------------------------------------------------------------
// HMMA m16n8k16, bf16 inputs, fp32 accumulate
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// mbarrier + bulk async copy (global -> shared)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// Non-blocking test of a barrier phase (about 20 cycles when it is complete).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// One potentially blocking test of a barrier phase.  The waiting thread may be
// suspended (up to suspend_ns) until the phase completes, so waiting warps do
// not poll the barrier while the bulk copies that complete it are in flight.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t suspend_ns = 200000u) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait on a barrier phase: gives up (returns false) after about
// `limit_cycles` SM clock cycles (default 4e9: about 2 s at the top clock), so
// a copy that never lands cannot keep the GPU busy; the caller records
// MOE_DEV_ERR_TIMEOUT and returns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  long long limit_cycles) {
  if (mbar_test(bar, parity)) return true;  // non-blocking test: the common already-complete case
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > limit_cycles) return false;
  }
}

// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) from global to
// shared memory, completing as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Programmatic dependent launch controls.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

}  // namespace moe
