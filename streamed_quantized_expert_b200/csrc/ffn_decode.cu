// Stages 4 + 5 for decode-sized token counts: the quantized SwiGLU expert FFN
// read straight from the slot pool (RFC "How the prototype works": quantized
// experts through gather_qmm on the pool; experts "gated, concatenated,
// untransposed, no bias"), then the weighted combine.
//
// Design (B200): the projections are GEMVs with a handful of tokens, bound by
// HBM.  Each CTA streams its share of expert rows into shared memory with
// bulk async copies (one per row, padded rows so the per-thread unit loads
// are bank-conflict free) behind mbarriers.  Warps turn packed codes into
// bf16 pairs (128 + q*2^a) with one LOP3 per two codes and feed them, with no
// per-weight arithmetic, to HMMA m16n8k16 against x pre-scaled by 2^-a.  The
// scale, bias and 128-offset are applied once per (row, group, token):
//   sum_k (s q_k + b) x_k = s * (D_g - 128 sum_k x_k 2^-a_k) + b * sum_k x_k.
// gate and up rows sit in the same 16-row MMA tile (rows 0-7 gate, 8-15 up),
// so every thread holds gate and up of the same output and applies SwiGLU in
// registers.  The down kernel owns output rows across all of the pass's
// experts, so the combine is a plain deterministic sum (no atomics).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {


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
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int klo = kb * 128 + 16 * s + 2 * t4, khi = klo + 8;
    uint32_t v0 = 0u, v1 = 0u;
    if (row) {
      if (klo < K) v0 = ld_pair(row + klo);
      if (khi < K) v1 = ld_pair(row + khi);
    }
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

// One 128-block of a 16-row tile: rows ra (A rows 0-7) and rb (rows 8-15) in
// shared memory, unit t4; accumulate the group epilogues into acc.
template <int B, int GS>
__device__ __forceinline__ void block_mma(const uint8_t* ra, const uint8_t* rbp, const uint32_t* sbA,
                                          const uint32_t* sbB, int kb, int t4, const uint32_t (&bf)[8][2],
                                          const float (&xs)[8 / GS][2], const float (&xo)[8 / GS][2],
                                          float (&acc)[4]) {
  uint32_t wa[B], wb[B], pa[16], pb[16];
  load_unit<B>(ra + (kb * 4 + t4) * 4 * B, wa);
  load_unit<B>(rbp + (kb * 4 + t4) * 4 * B, wb);
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
    const uint32_t wA = sbA[gi], wB = sbB[gi];
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

// ---------------------------------------------------------------------------
// gate/up + SwiGLU:  h[pos][j] = silu(gate_j . x_t) * (up_j . x_t)
// Work item = (active expert of the pass, 8 consecutive j) = a 16-row MMA
// tile (8 gate rows, 8 up rows).  Each CTA takes a contiguous range of items.
// Warp 8 is the producer: it streams every item's rows into a ring of shared
// memory stages (full/empty mbarriers).  Warps 0-7 split K (BPW 128-blocks
// each, x fragments stay in registers while the token set is unchanged) and
// run through all their items without CTA-wide barriers; partial sums are
// reduced across warps once per batch of kRedBatch (item, token-tile) entries.
// ---------------------------------------------------------------------------
constexpr int kGuConsumers = 8;
constexpr int kGuThreads = (kGuConsumers + 1) * 32;
constexpr int kRedBatch = 8;

struct RedMeta {
  int pos;   // first sorted position of the token tile
  int ntok;  // tokens in the tile
  int jt;    // 8-row tile of the intermediate dimension
  int pad;
};

template <int B, int BPW, int GS>
__global__ void __launch_bounds__(kGuThreads, 1) ffn_gu_kernel(const FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const int NST = a.gu_nstage, SB = a.gu_stage_bytes, SR = a.sr_gu;
  float* red = reinterpret_cast<float*>(smem + (size_t)NST * SB);  // [kRedBatch][8 warps][32][4]
  RedMeta* meta = reinterpret_cast<RedMeta*>(red + kRedBatch * kGuConsumers * 32 * 4);
  uint64_t* full = reinterpret_cast<uint64_t*>(meta + kRedBatch);
  uint64_t* empty = full + NST;

  pdl_wait();
  const int n_act = pass_count(a);
  const int jt_n = a.I / 8;
  const int n_items = n_act * jt_n;
  const int i0 = (int)(((int64_t)n_items * blockIdx.x) / gridDim.x);
  const int i1 = (int)(((int64_t)n_items * (blockIdx.x + 1)) / gridDim.x);
  const int my_items = i1 - i0;
  pdl_launch_dependents();
  if (my_items <= 0) return;
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGuConsumers);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kGuConsumers) {  // producer
    if (lane == 0) {
      const uint32_t sbb = 8u * a.ng_gu * 4u;
      for (int r = 0; r < my_items; ++r) {
        const int s = r % NST;
        if (r >= NST && !mbar_wait_bounded(&empty[s], (uint32_t)(((r / NST) - 1) & 1))) {
          if (a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
          // the consumers will time out on full[s]; nothing more is issued
          break;
        }
        const int item = i0 + r;
        const int jt = item % jt_n;
        const int slot = a.table[a.active[a.pass_begin + item / jt_n]];
        uint8_t* st = smem + (size_t)s * SB;
        if (!slot_ok(a, slot)) {
          mbar_arrive_expect_tx(&full[s], 0);
          continue;
        }
        const uint8_t* base = a.pool + (int64_t)slot * a.slot_bytes;
        mbar_arrive_expect_tx(&full[s], 16u * (uint32_t)a.rb_gu + 2u * sbb);
        for (int rr = 0; rr < 16; ++rr) {
          const int grow = (rr < 8 ? 0 : a.I) + jt * 8 + (rr & 7);
          bulk_g2s(st + rr * SR, base + a.q_gu + (int64_t)grow * a.rb_gu, (uint32_t)a.rb_gu, &full[s]);
        }
        uint8_t* sbd = st + 16 * SR;
        bulk_g2s(sbd, base + a.sb_gu + (int64_t)jt * sbb, sbb, &full[s]);
        bulk_g2s(sbd + sbb, base + a.sb_gu + (int64_t)(a.I + jt * 8) * a.ng_gu * 4, sbb, &full[s]);
      }
    }
    return;
  }

  // consumers
  uint32_t bf[BPW][8][2];
  float xs[BPW][8 / GS][2], xo[BPW][8 / GS][2];
  int cached_tok = -2;
  bool timed_out = false;
  int nent = 0;  // entries in the current reduction batch

  auto flush = [&]() {
    consumers_sync(kGuConsumers * 32);
    for (int idx = tid; idx < nent * 64; idx += kGuConsumers * 32) {
      const int en = idx >> 6, j = (idx >> 3) & 7, n = idx & 7;
      const RedMeta m = meta[en];
      if (n >= m.ntok) continue;
      const int src = 4 * j + (n >> 1), c = n & 1;
      const float* rp = red + (size_t)en * kGuConsumers * 32 * 4;
      float gate = 0.f, up = 0.f;
#pragma unroll
      for (int w = 0; w < kGuConsumers; ++w) {
        gate += rp[(w * 32 + src) * 4 + c];
        up += rp[(w * 32 + src) * 4 + 2 + c];
      }
      const float hv = gate / (1.0f + expf(-gate)) * up;
      a.h[(int64_t)(m.pos + n) * a.I + m.jt * 8 + j] = f32_to_bf16_rne(hv);
    }
    consumers_sync(kGuConsumers * 32);
    nent = 0;
  };

  for (int r = 0; r < my_items; ++r) {
    const int s = r % NST;
    const int item = i0 + r;
    const int jt = item % jt_n;
    const int e = a.active[a.pass_begin + item / jt_n];
    const int slot = a.table[e];
    const bool ok = slot_ok(a, slot);
    if (!ok && tid == 0 && jt == 0) flag_slot(a, slot);
    // a wait that runs out marks the warp; it keeps walking the items (no
    // waits, no math) so that every consumer reaches the same batch barriers
    if (!timed_out && !mbar_wait_bounded(&full[s], (uint32_t)((r / NST) & 1))) timed_out = true;
    const uint8_t* st = smem + (size_t)s * SB;
    const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 16 * SR);
    const int pos0 = a.offsets[e], cnt_e = ok ? a.offsets[e + 1] - pos0 : 0;
    for (int tt = 0; tt * 8 < cnt_e; ++tt) {
      const int ntok = min(8, cnt_e - tt * 8);
      const int my_tok = g8 < ntok ? a.pairs[pos0 + tt * 8 + g8] / a.k : -1;
      if (!__all_sync(0xffffffffu, my_tok == cached_tok)) {
        const uint16_t* xrow = my_tok >= 0 ? a.x + (int64_t)my_tok * a.H : nullptr;
#pragma unroll
        for (int bi = 0; bi < BPW; ++bi) load_b_block<B, GS>(xrow, warp * BPW + bi, a.H, t4, bf[bi], xs[bi], xo[bi]);
        cached_tok = my_tok;
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int bi = 0; bi < BPW; ++bi) {
        const int kb = warp * BPW + bi;
        if (kb < a.nblk_gu && !timed_out)
          block_mma<B, GS>(st + g8 * SR, st + (8 + g8) * SR, sbs + g8 * a.ng_gu, sbs + (8 + g8) * a.ng_gu, kb, t4,
                           bf[bi], xs[bi], xo[bi], acc);
      }
      *reinterpret_cast<float4*>(&red[(((size_t)nent * kGuConsumers + warp) * 32 + lane) * 4]) =
          make_float4(acc[0], acc[1], acc[2], acc[3]);
      if (warp == 0 && lane == 0) meta[nent] = RedMeta{pos0 + tt * 8, ntok, jt, 0};
      if (++nent == kRedBatch) flush();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  // every consumer warp reaches here with the same nent (same items, same order)
  if (nent > 0) flush();
  if (timed_out && lane == 0 && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------
// down (+ combine).  CTA owns 16 output rows.  Warp 4 is the producer: it
// streams the pass's experts' 16-row slices into a ring of stages as soon as
// the CTA starts -- before waiting for the gate/up kernel, since the slots do
// not depend on it.  Warps 0-3 split K (128-blocks round-robin) over every
// expert of the pass.
// FUSED (T <= 64): y[t][rows] += sum_j w[t,j] o_{t,j}   (deterministic order)
// else           : o[pair][rows] = o_{t,j}   (combined by combine_kernel)
// ---------------------------------------------------------------------------
constexpr int kDnConsumers = 4;
constexpr int kDnThreads = (kDnConsumers + 1) * 32;

template <int B, int GS, bool FUSED>
__global__ void __launch_bounds__(kDnThreads, 1) ffn_down_kernel(const FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const int NST = a.d_nstage, SB = a.d_stage_bytes, SR = a.sr_d;
  float* ypart = reinterpret_cast<float*>(smem + (size_t)NST * SB);  // [4 warps][T][16]
  const int ypart_n = FUSED ? kDnConsumers * a.T * 16 : 0;
  uint64_t* full = reinterpret_cast<uint64_t*>(ypart + ypart_n);
  uint64_t* empty = full + NST;

  // the pass's experts and their slots were written before the gate/up kernel
  // started, so they can be read before waiting on it
  int n_act = *a.n_active - a.pass_begin;
  if (n_act > a.pass_len) n_act = a.pass_len;
  const int n_rt = a.H / 16;
  const int rt = blockIdx.x;
  if (rt >= n_rt || n_act <= 0) {
    pdl_wait();
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDnConsumers);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kDnConsumers) {  // producer
    if (lane == 0) {
      const uint32_t sbb = 16u * a.ng_d * 4u;
      for (int r = 0; r < n_act; ++r) {
        const int s = r % NST;
        if (r >= NST && !mbar_wait_bounded(&empty[s], (uint32_t)(((r / NST) - 1) & 1))) {
          if (a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
          break;
        }
        const int slot = a.table[a.active[a.pass_begin + r]];
        uint8_t* st = smem + (size_t)s * SB;
        if (!slot_ok(a, slot)) {
          mbar_arrive_expect_tx(&full[s], 0);
          continue;
        }
        const uint8_t* base = a.pool + (int64_t)slot * a.slot_bytes;
        mbar_arrive_expect_tx(&full[s], 16u * (uint32_t)a.rb_d + sbb);
        for (int rr = 0; rr < 16; ++rr)
          bulk_g2s(st + rr * SR, base + a.q_d + (int64_t)(rt * 16 + rr) * a.rb_d, (uint32_t)a.rb_d, &full[s]);
        bulk_g2s(st + 16 * SR, base + a.sb_d + (int64_t)rt * sbb, sbb, &full[s]);
      }
    }
    pdl_wait();
    return;
  }

  pdl_wait();  // h (gate/up output) and y are ready
  if (FUSED) {
    for (int i = tid; i < ypart_n; i += kDnConsumers * 32) ypart[i] = 0.f;
    consumers_sync(kDnConsumers * 32);
  }
  bool timed_out = false;
  float acc1[4] = {0.f, 0.f, 0.f, 0.f};  // T == 1: every expert feeds the same token
  const bool single = FUSED && a.T == 1;
  // FUSED: the 4 warps split K of every expert.  Otherwise each warp owns
  // whole experts (r % 4 == warp), so o is written once, without atomics.
  const int kb0 = FUSED ? warp : 0, kbs = FUSED ? kDnConsumers : 1;
  for (int r = 0; r < n_act; ++r) {
    const int s = r % NST;
    const int e = a.active[a.pass_begin + r];
    const bool ok = slot_ok(a, a.table[e]);
    // every warp waits on every stage before releasing it, which keeps the
    // phases of the empty barriers in order
    if (!timed_out && !mbar_wait_bounded(&full[s], (uint32_t)((r / NST) & 1))) timed_out = true;
    const uint8_t* st = smem + (size_t)s * SB;
    const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 16 * SR);
    const bool mine = FUSED || (r % kDnConsumers) == warp;
    const int pos0 = a.offsets[e], cnt_e = (ok && mine && !timed_out) ? a.offsets[e + 1] - pos0 : 0;
    for (int tt = 0; tt * 8 < cnt_e; ++tt) {
      const int ntok = min(8, cnt_e - tt * 8);
      const uint16_t* hrow = g8 < ntok ? a.h + (int64_t)(pos0 + tt * 8 + g8) * a.I : nullptr;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int kb = kb0; kb < a.nblk_d; kb += kbs) {
        uint32_t bf[8][2];
        float xs[8 / GS][2], xo[8 / GS][2];
        load_b_block<B, GS>(hrow, kb, a.I, t4, bf, xs, xo);
        block_mma<B, GS>(st + g8 * SR, st + (8 + g8) * SR, sbs + g8 * a.ng_d, sbs + (8 + g8) * a.ng_d, kb, t4, bf,
                         xs, xo, acc);
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int n = 2 * t4 + c;
        if (n < ntok) {
          const int pf = a.pairs[pos0 + tt * 8 + n];
          if (FUSED) {
            const float wg = a.w[pf];
            if (single) {
              acc1[c] += wg * acc[c];
              acc1[2 + c] += wg * acc[2 + c];
            } else {
              float* yp = ypart + ((size_t)warp * a.T + pf / a.k) * 16;
              yp[g8] += wg * acc[c];
              yp[8 + g8] += wg * acc[2 + c];
            }
          } else {
            float* op = a.o + (int64_t)pf * a.H + rt * 16;
            op[g8] = acc[c];
            op[8 + g8] = acc[2 + c];
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (timed_out && lane == 0 && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
  if (FUSED) {
    consumers_sync(kDnConsumers * 32);  // all ypart updates done before the single-token write
    if (single) {
      // only column 0 (t4 == 0, c == 0) carries token 0
      if (t4 == 0) {
        ypart[(size_t)warp * 16 + g8] = acc1[0];
        ypart[(size_t)warp * 16 + 8 + g8] = acc1[2];
      }
    }
    consumers_sync(kDnConsumers * 32);
    for (int i = tid; i < a.T * 16; i += kDnConsumers * 32) {
      const int tok = i >> 4, row = i & 15;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kDnConsumers; ++w) sum += ypart[((size_t)w * a.T + tok) * 16 + row];
      a.y[(int64_t)tok * a.H + rt * 16 + row] += sum;
    }
  }
}

// y[t][r] += sum_j [expert of (t,j) in the pass] w[t,j] * o[t*k+j][r], j ascending.
__global__ void combine_kernel(const FfnArgs a) {
  pdl_wait();
  const int n_act = pass_count(a);
  if (n_act == 0) return;
  const int e_lo = a.active[a.pass_begin], e_hi = a.active[a.pass_begin + n_act - 1];
  const int64_t total = (int64_t)a.T * a.H;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / a.H), r = (int)(i % a.H);
    float s = 0.f;
    for (int j = 0; j < a.k; ++j) {
      const int pf = t * a.k + j;
      const int e = a.ids[pf];
      if (e >= e_lo && e <= e_hi && slot_ok(a, a.table[e])) s += a.w[pf] * a.o[(int64_t)pf * a.H + r];
    }
    a.y[i] += s;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int smem_row_stride(int64_t rb, int bits) {
  // words per row congruent to 12 (3-bit units), 16 (4-bit) or 24 (6-bit)
  // mod 32: the per-thread unit loads of 8 rows x 4 units hit distinct banks
  const int target = bits == 3 ? 12 : bits == 4 ? 16 : 24;
  int sr = (int)round_up(rb, 16);
  while (((sr / 4) & 31) != target) sr += 16;
  return sr;
}

size_t ffn_ws_bytes(const moe_layer_desc& d, int T) {
  const int64_t np = (int64_t)T * d.k;
  size_t b = (size_t)round_up(np * d.I * 2, 256);  // h (bf16)
  if (T > kFusedMaxTokens) b += (size_t)round_up(np * d.H * 4, 256);  // o (fp32)
  return b;
}

// Opt a kernel into the large dynamic shared-memory carve-out once per
// (kernel, device); the attribute call is not free on the launch path.  Each
// caller passes its own flag word (one per kernel instantiation).
static cudaError_t ensure_smem_attr(const void* kern, int (&done_mask)[4]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 128 && ((__atomic_load_n(&done_mask[dev >> 5], __ATOMIC_RELAXED) >> (dev & 31)) & 1)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess && dev < 128) __atomic_fetch_or(&done_mask[dev >> 5], 1 << (dev & 31), __ATOMIC_RELAXED);
  return e;
}

template <int B, int BPW, int GS>
static cudaError_t launch_gu(const FfnArgs& a, int grid, size_t smem, cudaStream_t st) {
  static int done[4] = {0, 0, 0, 0};
  const void* kern = reinterpret_cast<const void*>(ffn_gu_kernel<B, BPW, GS>);
  cudaError_t e = ensure_smem_attr(kern, done);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, kGuThreads, smem, st, a);
}

template <int B, int GS, bool F>
static cudaError_t launch_dn(const FfnArgs& a, int grid, size_t smem, cudaStream_t st) {
  static int done[4] = {0, 0, 0, 0};
  const void* kern = reinterpret_cast<const void*>(ffn_down_kernel<B, GS, F>);
  cudaError_t e = ensure_smem_attr(kern, done);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, kDnThreads, smem, st, a);
}

template <int B, int BPW>
static cudaError_t gu_by_gs(const FfnArgs& a, int gs, int grid, size_t smem, cudaStream_t st) {
  if (gs == 2) return launch_gu<B, BPW, 2>(a, grid, smem, st);
  if (gs == 4) return launch_gu<B, BPW, 4>(a, grid, smem, st);
  return launch_gu<B, BPW, 8>(a, grid, smem, st);
}

template <int B>
static cudaError_t gu_by_bpw(const FfnArgs& a, int bpw, int gs, int grid, size_t smem, cudaStream_t st) {
  if (bpw == 1) return gu_by_gs<B, 1>(a, gs, grid, smem, st);
  if (bpw == 2) return gu_by_gs<B, 2>(a, gs, grid, smem, st);
  return gu_by_gs<B, 4>(a, gs, grid, smem, st);
}

template <int B, bool F>
static cudaError_t dn_by_gs(const FfnArgs& a, int gs, int grid, size_t smem, cudaStream_t st) {
  if (gs == 2) return launch_dn<B, 2, F>(a, grid, smem, st);
  if (gs == 4) return launch_dn<B, 4, F>(a, grid, smem, st);
  return launch_dn<B, 8, F>(a, grid, smem, st);
}

template <bool F>
static cudaError_t dn_by_bits(const FfnArgs& a, int bits, int gs, int grid, size_t smem, cudaStream_t st) {
  if (bits == 3) return dn_by_gs<3, F>(a, gs, grid, smem, st);
  if (bits == 4) return dn_by_gs<4, F>(a, gs, grid, smem, st);
  return dn_by_gs<6, F>(a, gs, grid, smem, st);
}

bool ffn_decode_supported(const moe_layer_desc& d) {
  const int nblk = (int)(padded_k(d.H) / 128);
  return nblk <= kGuConsumers * 4 && d.H % 16 == 0 && d.I % 8 == 0;
}

// Shared-memory budgets: the gate/up and down kernels of one layer are sized
// to be resident on an SM together (the down kernel starts early and streams
// its weights while gate/up finishes).
constexpr size_t kGuSmemCap = 150 * 1024;
constexpr size_t kDnSmemCap = 72 * 1024;

cudaError_t launch_ffn_decode(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st) {
  const Layout& L = a.L;
  a.q_gu = L.q_gu;
  a.q_d = L.q_d;
  a.sb_gu = L.sb_gu;
  a.sb_d = L.sb_d;
  a.rb_gu = L.rb_gu;
  a.rb_d = L.rb_d;
  a.ng_gu = L.ng_gu;
  a.ng_d = L.ng_d;
  a.nblk_gu = L.nblk_gu;
  a.nblk_d = L.nblk_d;
  a.sr_gu = smem_row_stride(L.rb_gu, d.bits_gu);
  a.sr_d = smem_row_stride(L.rb_d, d.bits_down);
  a.gu_stage_bytes = (int)round_up(16 * a.sr_gu + 16 * L.ng_gu * 4, 128);
  a.d_stage_bytes = (int)round_up(16 * a.sr_d + 16 * L.ng_d * 4, 128);
  const int gs = d.group / 16;
  const int nblk = L.nblk_gu;
  const int bpw = nblk <= kGuConsumers ? 1 : nblk <= 2 * kGuConsumers ? 2 : 4;
  const int max_pass = a.pass_len < d.E ? a.pass_len : d.E;

  // gate/up: 148 CTAs (or fewer items), stages for every item of a CTA if they fit
  const int64_t items = (int64_t)max_pass * (d.I / 8);
  int grid = (int)(items < num_sms ? items : num_sms);
  if (grid < 1) grid = 1;
  const size_t red_bytes = (size_t)kRedBatch * kGuConsumers * 32 * 4 * sizeof(float) + kRedBatch * sizeof(RedMeta);
  const int64_t items_per_cta = (items + grid - 1) / grid;
  int nst = (int)((kGuSmemCap - red_bytes) / (a.gu_stage_bytes + 16));
  if (nst > items_per_cta) nst = (int)items_per_cta;
  if (nst > 32) nst = 32;
  if (nst < 1) return cudaErrorInvalidConfiguration;
  a.gu_nstage = nst;
  const size_t gu_smem = (size_t)nst * a.gu_stage_bytes + red_bytes + (size_t)nst * 16;

  const bool fused = a.T <= kFusedMaxTokens;
  const size_t ypart = fused ? (size_t)kDnConsumers * a.T * 16 * sizeof(float) : 0;
  int dnst = (int)((kDnSmemCap - ypart) / (a.d_stage_bytes + 16));
  if (dnst > max_pass) dnst = max_pass;
  if (dnst > 32) dnst = 32;
  if (dnst < 2) dnst = 2;
  a.d_nstage = dnst;
  const size_t dn_smem = (size_t)dnst * a.d_stage_bytes + ypart + (size_t)dnst * 16;

  cudaError_t e = cudaSuccess;
  if (d.bits_gu == 3) e = gu_by_bpw<3>(a, bpw, gs, grid, gu_smem, st);
  else if (d.bits_gu == 4) e = gu_by_bpw<4>(a, bpw, gs, grid, gu_smem, st);
  else e = gu_by_bpw<6>(a, bpw, gs, grid, gu_smem, st);
  if (e != cudaSuccess) return e;

  const int n_rt = d.H / 16;
  if (fused) e = dn_by_bits<true>(a, d.bits_down, gs, n_rt, dn_smem, st);
  else e = dn_by_bits<false>(a, d.bits_down, gs, n_rt, dn_smem, st);
  if (e != cudaSuccess || fused) return e;
  const int64_t total = (int64_t)a.T * d.H;
  int cgrid = (int)((total + 255) / 256);
  if (cgrid > num_sms * 8) cgrid = num_sms * 8;
  return launch_pdl(reinterpret_cast<const void*>(combine_kernel), cgrid, 256, 0, st, a);
}

}  // namespace moe
