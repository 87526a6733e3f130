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
#include "ffn_common.cuh"
#include "kernels.h"

namespace moe {


// ---------------------------------------------------------------------------
// gate/up + SwiGLU:  h[pos][j] = silu(gate_j . x_t) * (up_j . x_t)
// Work item = (active expert of the pass, 8 consecutive j) = a 16-row MMA
// tile (8 gate rows, 8 up rows).  Each CTA takes a contiguous range of items.
// Warp 8 is the producer: it streams every item's rows into a ring of shared
// memory stages (full/empty mbarriers).  Warps 0-7 split K (BPW 128-blocks
// each, x fragments in registers) and run through all their items without
// CTA-wide barriers; partial sums are reduced across warps once per batch of
// kRedBatch entries.  DENSE (T <= 8): MMA column n is token n for every
// expert, so x is loaded once per kernel; otherwise columns are the expert's
// own tokens, 8 at a time.
// ---------------------------------------------------------------------------
constexpr int kGuConsumers = 8;
constexpr int kGuThreads = (kGuConsumers + 1) * 32;

template <int B, int BPW, int GS, bool DENSE>
__global__ void __launch_bounds__(kGuThreads, 1) ffn_gu_kernel(const FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const int NST = a.gu_nstage, SB = a.gu_stage_bytes;
  const int GRP = 8 * (int)a.rb_gu;  // bytes of an 8-row group
  const int uoff = thread_unit_off<B>(t4, g8);
  float* red = reinterpret_cast<float*>(smem + (size_t)NST * SB);  // [kRedBatch][8 warps][32][4]
  RedMeta* rmeta = reinterpret_cast<RedMeta*>(red + kRedBatch * kGuConsumers * 32 * 4);
  ExpMeta* emeta = reinterpret_cast<ExpMeta*>(rmeta + kRedBatch);
  int* tokpos = reinterpret_cast<int*>(emeta + kMaxCtaExperts);  // [kMaxCtaExperts][8]
  uint64_t* full = reinterpret_cast<uint64_t*>(tokpos + kMaxCtaExperts * kDenseMaxTokens);
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
  const int e_first = i0 / jt_n;
  const int n_exp = (i1 - 1) / jt_n - e_first + 1;  // <= kMaxCtaExperts (checked by the launcher)
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGuConsumers);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kGuConsumers) {  // producer: finds its experts' slots itself and starts the copies at once
    if (lane == 0) {
      const uint32_t tb = (uint32_t)a.tile_gu;
      int cur_ai = -1, slot = -1;
      for (int r = 0; r < my_items; ++r) {
        const int s = r % NST;
        if (r >= NST && !mbar_wait_bounded(&empty[s], (uint32_t)(((r / NST) - 1) & 1), a.wait_limit)) {
          if (a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
          break;  // the consumers time out on full[s]; nothing more is issued
        }
        const int item = i0 + r;
        const int jt = item % jt_n;
        if (item / jt_n != cur_ai) {
          cur_ai = item / jt_n;
          slot = a.table[a.active[a.pass_begin + cur_ai]];
        }
        uint8_t* st = smem + (size_t)s * SB;
        if (!slot_ok(a, slot)) {
          mbar_arrive_expect_tx(&full[s], 0);
          continue;
        }
        // tile jt = storage rows 16 jt .. 16 jt + 15 = gate rows 8 jt.. then up rows 8 jt..
        const uint8_t* base = a.pool + (int64_t)slot * a.slot_bytes;
        mbar_arrive_expect_tx(&full[s], tb);
        bulk_g2s(st, base + a.q_gu + (int64_t)jt * tb, tb, &full[s]);
      }
    }
    return;
  }

  // consumers: the experts' metadata (loaded while the first copies fly)
  load_expert_meta<DENSE>(a, e_first, n_exp, emeta, tokpos, nullptr, kGuConsumers * 32);
  consumers_sync(kGuConsumers * 32);

  // consumers
  uint32_t bf[BPW][8][2];
  float xs[BPW][8 / GS][2], xo[BPW][8 / GS][2];
  int cached_tok = -2;
  bool timed_out = false;
  int nent = 0;  // entries in the current reduction batch

  if (DENSE) {  // column g8 = token g8 for every expert: load x once
    const uint16_t* xrow = g8 < a.T ? a.x + (int64_t)g8 * a.H : nullptr;
#pragma unroll
    for (int bi = 0; bi < BPW; ++bi) load_b_block<B, GS>(xrow, warp * BPW + bi, a.H, t4, bf[bi], xs[bi], xo[bi]);
  }

  auto flush = [&]() {
    consumers_sync(kGuConsumers * 32);
    for (int idx = tid; idx < nent * 64; idx += kGuConsumers * 32) {
      const int en = idx >> 6, j = (idx >> 3) & 7, n = idx & 7;
      const RedMeta m = rmeta[en];
      int pos;
      if (DENSE) {
        pos = n < a.T ? tokpos[m.ei * kDenseMaxTokens + n] : -1;
      } else {
        pos = n < m.ntok ? m.pos + n : -1;
      }
      if (pos < 0) continue;
      const int src = 4 * j + (n >> 1), c = n & 1;
      const float* rp = red + (size_t)en * kGuConsumers * 32 * 4;
      float gate = 0.f, up = 0.f;
#pragma unroll
      for (int w = 0; w < kGuConsumers; ++w) {
        gate += rp[(w * 32 + src) * 4 + c];
        up += rp[(w * 32 + src) * 4 + 2 + c];
      }
      const float hv = gate / (1.0f + expf(-gate)) * up;
      a.h[(int64_t)pos * a.I + m.jt * 8 + j] = f32_to_bf16_rne(hv);
    }
    consumers_sync(kGuConsumers * 32);
    nent = 0;
  };

  for (int r = 0; r < my_items; ++r) {
    const int s = r % NST;
    const int item = i0 + r;
    const int jt = item % jt_n;
    const int ei = item / jt_n - e_first;
    const ExpMeta em = emeta[ei];
    const bool ok = slot_ok(a, em.slot);
    if (!ok && tid == 0 && jt == 0) flag_slot(a, em.slot);
    // a wait that runs out marks the warp; it keeps walking the items (no
    // waits, no math) so that every consumer reaches the same batch barriers
    if (!timed_out && !mbar_wait_bounded(&full[s], (uint32_t)((r / NST) & 1), a.wait_limit)) timed_out = true;
    const uint8_t* st = smem + (size_t)s * SB;
    const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
    const int n_tiles = !ok ? 0 : DENSE ? 1 : (em.cnt + 7) / 8;
    for (int tt = 0; tt < n_tiles; ++tt) {
      const int ntok = DENSE ? a.T : min(8, em.cnt - tt * 8);
      if (!DENSE) {
        const int my_tok = g8 < ntok ? a.pairs[em.pos0 + tt * 8 + g8] / a.k : -1;
        if (!__all_sync(0xffffffffu, my_tok == cached_tok)) {
          const uint16_t* xrow = my_tok >= 0 ? a.x + (int64_t)my_tok * a.H : nullptr;
#pragma unroll
          for (int bi = 0; bi < BPW; ++bi)
            load_b_block<B, GS>(xrow, warp * BPW + bi, a.H, t4, bf[bi], xs[bi], xo[bi]);
          cached_tok = my_tok;
        }
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int bi = 0; bi < BPW; ++bi) {
        const int kb = warp * BPW + bi;
        if (kb < a.nblk_gu && !timed_out)
          block_mma<B, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf[bi], xs[bi],
                           xo[bi], acc);
      }
      *reinterpret_cast<float4*>(&red[(((size_t)nent * kGuConsumers + warp) * 32 + lane) * 4]) =
          make_float4(acc[0], acc[1], acc[2], acc[3]);
      if (warp == 0 && lane == 0) rmeta[nent] = RedMeta{ei, em.pos0 + tt * 8, ntok, jt};
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
// not depend on it.  Warps 0-3 split K (128-blocks round-robin).
// DENSE (T <= 8): column n = token n; h rows are staged in shared memory when
//   they fit; y[t][rows] += sum over experts of w * o, summed in registers in
//   expert order, then over the K-split warps in warp order.
// FUSED (T <= 64): per-warp partial y in shared memory, summed in warp order.
// else: o[pair][rows] = o_{t,j} (combined by combine_kernel); each warp owns
//   whole experts.
// ---------------------------------------------------------------------------
constexpr int kDnConsumers = 8;
constexpr int kDnThreads = (kDnConsumers + 1) * 32;

template <int B, int GS, int MODE>  // MODE 0: dense, 1: fused token tiles, 2: per-pair output
__global__ void __launch_bounds__(kDnThreads, 1) ffn_down_kernel(const FfnArgs a) {
  constexpr bool DENSE = MODE == 0, FUSED = MODE <= 1;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const int NST = a.d_nstage, SB = a.d_stage_bytes;
  const int GRP = 8 * (int)a.rb_d;  // bytes of an 8-row group
  const int uoff = thread_unit_off<B>(t4, g8);
  uint8_t* hst = smem + (size_t)NST * SB;  // staged h (DENSE), kHStageMax bytes
  float* ypart = reinterpret_cast<float*>(hst + (DENSE ? kHStageMax : 0));  // [4][T][16] or [4][32][4]
  const int ypart_n = DENSE ? kDnConsumers * 32 * 4 : MODE == 1 ? kDnConsumers * a.T * 16 : 0;
  const bool overwrite = a.y_overwrite != 0;
  ExpMeta* emeta = reinterpret_cast<ExpMeta*>(ypart + ypart_n);
  int* tokpos = reinterpret_cast<int*>(emeta + kMaxCtaExperts);
  float* wtab = reinterpret_cast<float*>(tokpos + kMaxCtaExperts * kDenseMaxTokens);
  uint64_t* full = reinterpret_cast<uint64_t*>(wtab + kMaxCtaExperts * kDenseMaxTokens);
  uint64_t* empty = full + NST;

  // the pass's experts, slots and routing were written before the gate/up
  // kernel started, so they can be read before waiting on it
  int n_act = *a.n_active - a.pass_begin;
  if (n_act > a.pass_len) n_act = a.pass_len;
  const int n_rt = a.H / 16;
  const int rt = blockIdx.x;
  if (rt >= n_rt || n_act <= 0) {
    pdl_wait();
    if (rt < n_rt && a.y_overwrite)
      for (int i = threadIdx.x; i < a.T * 16; i += blockDim.x) a.y[(int64_t)(i >> 4) * a.H + rt * 16 + (i & 15)] = 0.f;
    return;
  }
  const int n_meta = n_act < kMaxCtaExperts ? n_act : kMaxCtaExperts;
  load_expert_meta<DENSE>(a, 0, n_meta, emeta, tokpos, wtab, kDnThreads);
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
      const uint32_t tb = (uint32_t)a.tile_d;
      for (int r = 0; r < n_act; ++r) {
        const int s = r % NST;
        if (r >= NST && !mbar_wait_bounded(&empty[s], (uint32_t)(((r / NST) - 1) & 1), a.wait_limit)) {
          if (a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
          break;
        }
        const int slot = r < n_meta ? emeta[r].slot : a.table[a.active[a.pass_begin + r]];
        uint8_t* st = smem + (size_t)s * SB;
        if (!slot_ok(a, slot)) {
          mbar_arrive_expect_tx(&full[s], 0);
          continue;
        }
        const uint8_t* base = a.pool + (int64_t)slot * a.slot_bytes;
        mbar_arrive_expect_tx(&full[s], tb);
        bulk_g2s(st, base + a.q_d + (int64_t)rt * tb, tb, &full[s]);
      }
    }
    pdl_wait();
    return;
  }

  pdl_wait();  // h (gate/up output) and y are ready
  const int np = a.T * a.k;
  const bool h_staged = DENSE && (size_t)np * a.I * 2 <= (size_t)kHStageMax;
  if (h_staged) {
    // h is read by every CTA: plain coalesced copy into shared memory
    const uint4* src = reinterpret_cast<const uint4*>(a.h);
    uint4* dst = reinterpret_cast<uint4*>(hst);
    for (int i = tid; i < np * a.I / 8; i += kDnConsumers * 32) dst[i] = src[i];
  }
  if (MODE == 1)
    for (int i = tid; i < ypart_n; i += kDnConsumers * 32) ypart[i] = 0.f;
  consumers_sync(kDnConsumers * 32);

  bool timed_out = false;
  float yacc[4] = {0.f, 0.f, 0.f, 0.f};  // DENSE: (row g8 | g8+8) x (token 2t4 | 2t4+1)
  const int kb0 = FUSED ? (warp % kDnKSplit) : 0, kbs = FUSED ? kDnKSplit : 1;
  const int egrp = FUSED ? kDnConsumers / kDnKSplit : kDnConsumers;  // warp groups taking experts in turn
  const int my_grp = FUSED ? warp / kDnKSplit : warp;
  for (int r = 0; r < n_act; ++r) {
    const int s = r % NST;
    ExpMeta em;
    if (r < n_meta) {
      em = emeta[r];
    } else {
      em.e = a.active[a.pass_begin + r];
      em.slot = a.table[em.e];
      em.pos0 = a.offsets[em.e];
      em.cnt = a.offsets[em.e + 1] - em.pos0;
    }
    const bool ok = slot_ok(a, em.slot);
    // every warp waits on every stage before releasing it, which keeps the
    // phases of the empty barriers in order
    if (!timed_out && !mbar_wait_bounded(&full[s], (uint32_t)((r / NST) & 1), a.wait_limit)) timed_out = true;
    const uint8_t* st = smem + (size_t)s * SB;
    const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
    const bool mine = (r % egrp) == my_grp;
    const bool run = ok && mine && !timed_out;
    if (DENSE) {
      if (run) {
        const int pos = g8 < a.T ? tokpos[r * kDenseMaxTokens + g8] : -1;
        const uint16_t* hrow = pos < 0 ? nullptr
                               : h_staged ? reinterpret_cast<const uint16_t*>(hst) + (size_t)pos * a.I
                                          : a.h + (int64_t)pos * a.I;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = kb0; kb < a.nblk_d; kb += kbs) {
          uint32_t bf[8][2];
          float xs[8 / GS][2], xo[8 / GS][2];
          load_b_block<B, GS>(hrow, kb, a.I, t4, bf, xs, xo);
          block_mma<B, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs, xo, acc);
        }
        const float w0 = wtab[r * kDenseMaxTokens + 2 * t4], w1 = wtab[r * kDenseMaxTokens + 2 * t4 + 1];
        yacc[0] += w0 * acc[0];
        yacc[1] += w1 * acc[1];
        yacc[2] += w0 * acc[2];
        yacc[3] += w1 * acc[3];
      }
    } else {
      const int cnt_e = run ? em.cnt : 0;
      for (int tt = 0; tt * 8 < cnt_e; ++tt) {
        const int ntok = min(8, cnt_e - tt * 8);
        const uint16_t* hrow = g8 < ntok ? a.h + (int64_t)(em.pos0 + tt * 8 + g8) * a.I : nullptr;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = kb0; kb < a.nblk_d; kb += kbs) {
          uint32_t bf[8][2];
          float xs[8 / GS][2], xo[8 / GS][2];
          load_b_block<B, GS>(hrow, kb, a.I, t4, bf, xs, xo);
          block_mma<B, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs, xo, acc);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int n = 2 * t4 + c;
          if (n < ntok) {
            const int pf = a.pairs[em.pos0 + tt * 8 + n];
            if (FUSED) {
              const float wg = a.w[pf];
              float* yp = ypart + ((size_t)warp * a.T + pf / a.k) * 16;
              yp[g8] += wg * acc[c];
              yp[8 + g8] += wg * acc[2 + c];
            } else {
              float* op = a.o + (int64_t)pf * a.H + rt * 16;
              op[g8] = acc[c];
              op[8 + g8] = acc[2 + c];
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (timed_out && lane == 0 && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
  if (DENSE) {
    *reinterpret_cast<float4*>(&ypart[(warp * 32 + lane) * 4]) = make_float4(yacc[0], yacc[1], yacc[2], yacc[3]);
    consumers_sync(kDnConsumers * 32);
    for (int i = tid; i < a.T * 16; i += kDnConsumers * 32) {
      const int tok = i >> 4, row = i & 15;
      // value of (row, token) sits at lane 4*(row&7) + tok/2, component (row>>3)*2 + (tok&1)
      const int src = 4 * (row & 7) + (tok >> 1), c = (row >> 3) * 2 + (tok & 1);
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kDnConsumers; ++w) sum += ypart[(w * 32 + src) * 4 + c];
      float* yp = a.y + (int64_t)tok * a.H + rt * 16 + row;
      *yp = overwrite ? sum : *yp + sum;
    }
  } else if (MODE == 1) {
    consumers_sync(kDnConsumers * 32);
    for (int i = tid; i < a.T * 16; i += kDnConsumers * 32) {
      const int tok = i >> 4, row = i & 15;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kDnConsumers; ++w) sum += ypart[((size_t)w * a.T + tok) * 16 + row];
      float* yp = a.y + (int64_t)tok * a.H + rt * 16 + row;
      *yp = overwrite ? sum : *yp + sum;
    }
  }
}

// y[t][r] += sum_j [expert of (t,j) in the pass] w[t,j] * o[t*k+j][r], j ascending.
// One warp per (token, 256-column chunk): lane j tests pair j (k <= 32) and a
// ballot gives the token's pairs in this pass; a token with none is skipped
// (its y row is not touched unless y is overwritten).  Each lane sums two
// groups of 4 columns, so a warp issues its loads together.
constexpr int kCombineChunk = 256;

__global__ void combine_kernel(const FfnArgs a) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t w0 = (int64_t)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int64_t nw = (int64_t)((gridDim.x * blockDim.x) >> 5);
  const int nch = (a.H + kCombineChunk - 1) / kCombineChunk;
  const int n_act = pass_count(a);
  const int e_lo = n_act > 0 ? a.active[a.pass_begin] : 1, e_hi = n_act > 0 ? a.active[a.pass_begin + n_act - 1] : 0;
  const bool vec = (reinterpret_cast<uintptr_t>(a.y) & 15) == 0;
  for (int64_t it = w0; it < (int64_t)a.T * nch; it += nw) {
    const int t = (int)(it / nch), ch = (int)(it % nch);
    bool in = false;
    float wj = 0.f;
    if (lane < a.k) {
      const int pf = t * a.k + lane;
      const int e = a.ids[pf];
      in = e >= e_lo && e <= e_hi && slot_ok(a, a.table[e]);
      wj = a.w[pf];
    }
    const unsigned mask = __ballot_sync(0xffffffffu, in);
    if (mask == 0u && !a.y_overwrite) continue;
    float* yrow = a.y + (int64_t)t * a.H;
    float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    const int c0 = ch * kCombineChunk + 4 * lane;
    for (unsigned m = mask; m; m &= m - 1) {
      const int j = __ffs(m) - 1;
      const float wv = __shfl_sync(0xffffffffu, wj, j);  // mask is warp-uniform
      const float* orow = a.o + ((int64_t)t * a.k + j) * a.H;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = c0 + 128 * h;
        if (c < a.H) {
          const float4 o = *reinterpret_cast<const float4*>(orow + c);
          acc[h].x += wv * o.x;
          acc[h].y += wv * o.y;
          acc[h].z += wv * o.z;
          acc[h].w += wv * o.w;
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = c0 + 128 * h;
      if (c >= a.H) continue;
      if (vec) {
        float4* yp = reinterpret_cast<float4*>(yrow + c);
        if (!a.y_overwrite) {
          const float4 y0 = *yp;
          acc[h].x += y0.x;
          acc[h].y += y0.y;
          acc[h].z += y0.z;
          acc[h].w += y0.w;
        }
        *yp = acc[h];
      } else {
        const float v[4] = {acc[h].x, acc[h].y, acc[h].z, acc[h].w};
        for (int q = 0; q < 4; ++q) yrow[c + q] = a.y_overwrite ? v[q] : yrow[c + q] + v[q];
      }
    }
  }
}

// Grid of the combine: one warp per (token, column chunk), 8 warps per block.
int combine_grid(int T, int H, int num_sms) {
  const int64_t items = (int64_t)T * ((H + kCombineChunk - 1) / kCombineChunk);
  int64_t g = (items + 7) / 8;
  if (g > (int64_t)num_sms * 16) g = (int64_t)num_sms * 16;
  return g < 1 ? 1 : (int)g;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int B, int BPW, int GS>
static cudaError_t launch_gu(const FfnArgs& a, int grid, size_t smem, cudaStream_t st) {
  static int done[4] = {0, 0, 0, 0};
  static int done_d[4] = {0, 0, 0, 0};
  const bool dense = dense_mode(a);
  const void* kern = dense ? reinterpret_cast<const void*>(ffn_gu_kernel<B, BPW, GS, true>)
                           : reinterpret_cast<const void*>(ffn_gu_kernel<B, BPW, GS, false>);
  cudaError_t e = ensure_smem_attr(kern, dense ? done_d : done);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, kGuThreads, smem, st, a);
}

template <int B, int GS, int F>
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

template <int B, int F>
static cudaError_t dn_by_gs(const FfnArgs& a, int gs, int grid, size_t smem, cudaStream_t st) {
  if (gs == 2) return launch_dn<B, 2, F>(a, grid, smem, st);
  if (gs == 4) return launch_dn<B, 4, F>(a, grid, smem, st);
  return launch_dn<B, 8, F>(a, grid, smem, st);
}

template <int F>
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

// 0: fused single-launch decode; 1: gate/up + down GEMV kernels (mma.sync);
// 2: tcgen05 grouped GEMM (prefill) -- the choice launch_ffn_decode makes
// for a call covering every expert of the layer.
int ffn_kernel_path(const moe_layer_desc& d, int T, bool has_x_sorted, int num_sms) {
  // BF16 experts run on the tensor-core grouped GEMM only, at any T
  if (bf16_experts(d)) return has_x_sorted && ffn_prefill_tc_shape_ok(d) ? 2 : -1;
  FfnArgs a{};
  a.T = T;
  a.pass_len = d.E;
  a.L = make_layout(d);
  unsigned ctl_stub = 0;
  a.ctl = &ctl_stub;  // the plan only checks that a control block and the tagged h region exist
  a.htag = &ctl_stub;
  size_t smem = 0;
  if (ffn_fused_plan(a, d, num_sms, smem)) return 0;
  if (T >= kTcMinTokens && has_x_sorted && ffn_prefill_tc_shape_ok(d)) return 2;
  return 1;
}

// The fused decode kernel in route mode only (a.logits set): no other path routes.
cudaError_t launch_ffn_route_fused(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st) {
  const Layout& L = a.L;
  a.q_gu = L.gu;
  a.q_d = L.d;
  a.tile_gu = L.tile_gu;
  a.tile_d = L.tile_d;
  a.rb_gu = L.rb_gu;
  a.rb_d = L.rb_d;
  a.ng_gu = L.ng_gu;
  a.ng_d = L.ng_d;
  a.nblk_gu = L.nblk_gu;
  a.nblk_d = L.nblk_d;
  return launch_ffn_fused(a, d, num_sms, st);
}

cudaError_t launch_ffn_decode(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st) {
  const Layout& L = a.L;
  if (bf16_experts(d)) {
    a.q_gu = L.gu;
    a.q_d = L.d;
    return launch_ffn_prefill_tc(a, d, num_sms, st);
  }
  {
    FfnArgs f = a;
    f.q_gu = L.gu;
    f.q_d = L.d;
    f.tile_gu = L.tile_gu;
    f.tile_d = L.tile_d;
    f.rb_gu = L.rb_gu;
    f.rb_d = L.rb_d;
    f.ng_gu = L.ng_gu;
    f.ng_d = L.ng_d;
    f.nblk_gu = L.nblk_gu;
    f.nblk_d = L.nblk_d;
    const cudaError_t e = launch_ffn_fused(f, d, num_sms, st);
    if (e != cudaErrorNotSupported) return e;
  }
  a.q_gu = L.gu;
  a.q_d = L.d;
  a.tile_gu = L.tile_gu;
  a.tile_d = L.tile_d;
  a.rb_gu = L.rb_gu;
  a.rb_d = L.rb_d;
  a.ng_gu = L.ng_gu;
  a.ng_d = L.ng_d;
  a.nblk_gu = L.nblk_gu;
  a.nblk_d = L.nblk_d;
  if (a.T >= kTcMinTokens) {  // tensor-core grouped GEMM (needs x_sorted)
    const cudaError_t e = launch_ffn_prefill_tc(a, d, num_sms, st);
    if (e != cudaErrorNotSupported) return e;
  }
  a.gu_stage_bytes = (int)round_up(L.tile_gu, 128);
  a.d_stage_bytes = (int)round_up(L.tile_d, 128);
  const int gs = d.group / 16;
  const int nblk = L.nblk_gu;
  const int bpw = nblk <= kGuConsumers ? 1 : nblk <= 2 * kGuConsumers ? 2 : 4;
  // at most T*k experts are active, however long the pass
  int max_pass = a.pass_len < d.E ? a.pass_len : d.E;
  if ((int64_t)a.T * d.k < max_pass) max_pass = a.T * d.k;

  // gate/up: 148 CTAs (or fewer items), stages for every item of a CTA if they fit
  const int64_t items = (int64_t)max_pass * (d.I / 8);
  int grid = (int)(items < num_sms ? items : num_sms);
  if (grid < 1) grid = 1;
  const size_t meta_bytes = (size_t)kMaxCtaExperts * (sizeof(ExpMeta) + kDenseMaxTokens * 2 * sizeof(int));
  const size_t red_bytes = (size_t)kRedBatch * kGuConsumers * 32 * 4 * sizeof(float) + kRedBatch * sizeof(RedMeta);
  const int64_t items_per_cta = (items + grid - 1) / grid;
  if (items_per_cta / (d.I / 8) + 2 > kMaxCtaExperts) return cudaErrorInvalidConfiguration;
  int nst = (int)((kGuSmemCap - red_bytes - meta_bytes) / (a.gu_stage_bytes + 16));
  if (nst > items_per_cta) nst = (int)items_per_cta;
  if (nst > 32) nst = 32;
  if (nst < 1) return cudaErrorInvalidConfiguration;
  a.gu_nstage = nst;
  const size_t gu_smem = (size_t)nst * a.gu_stage_bytes + red_bytes + meta_bytes + (size_t)nst * 16;

  const bool dense = dense_mode(a);
  const int mode = dense ? 0 : a.T <= kFusedMaxTokens ? 1 : 2;
  const size_t ypart = mode == 0 ? (size_t)kDnConsumers * 32 * 4 * sizeof(float) + kHStageMax
                       : mode == 1 ? (size_t)kDnConsumers * a.T * 16 * sizeof(float) : 0;
  int dnst = (int)((kDnSmemCap - ypart - meta_bytes) / (a.d_stage_bytes + 16));
  if (dnst > max_pass) dnst = max_pass;
  if (dnst > 32) dnst = 32;
  if (dnst < 2) dnst = 2;
  a.d_nstage = dnst;
  const size_t dn_smem = (size_t)dnst * a.d_stage_bytes + ypart + meta_bytes + (size_t)dnst * 16;

  cudaError_t e = cudaSuccess;
  if (d.bits_gu == 3) e = gu_by_bpw<3>(a, bpw, gs, grid, gu_smem, st);
  else if (d.bits_gu == 4) e = gu_by_bpw<4>(a, bpw, gs, grid, gu_smem, st);
  else e = gu_by_bpw<6>(a, bpw, gs, grid, gu_smem, st);
  if (e != cudaSuccess) return e;

  const int n_rt = d.H / 16;
  if (mode == 0) e = dn_by_bits<0>(a, d.bits_down, gs, n_rt, dn_smem, st);
  else if (mode == 1) e = dn_by_bits<1>(a, d.bits_down, gs, n_rt, dn_smem, st);
  else e = dn_by_bits<2>(a, d.bits_down, gs, n_rt, dn_smem, st);
  if (e != cudaSuccess || mode < 2) return e;
  return launch_pdl(reinterpret_cast<const void*>(combine_kernel), combine_grid(a.T, d.H, num_sms), 256, 0, st, a);
}

}  // namespace moe
