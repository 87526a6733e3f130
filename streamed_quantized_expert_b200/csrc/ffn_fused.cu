// Decode FFN in one launch (T <= 8 tokens, every routed pair in the per-CTA
// tables): gate/up + SwiGLU, a grid-wide barrier, then down + combine.
//
// One CTA per SM, all co-resident (cooperative launch).  At kernel start the
// producer warp of each CTA issues the bulk copies of everything the CTA will
// read: its gate/up tiles (one 16-row tile per (expert, 8 j) item, one copy
// each) and its 16-row slice of every active expert's down projection (one
// copy per expert).  The down weights therefore stream in while gate/up
// computes, and the layer pays for one launch and one memory latency instead
// of two.  The barrier between the phases is a counter + generation pair in
// the workspace, bounded by a clock limit (MOE_DEV_ERR_TIMEOUT on expiry).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ffn_common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kFuThreads = (kFuConsumers + 1) * 32;

// Grid barrier on two words in global memory: ctl[0] counts arrivals, ctl[1]
// is the generation.  The last CTA to arrive resets the count and bumps the
// generation, so the words are back to (0, g+1) after every barrier.  Called
// by one thread per CTA.  Returns false if the wait ran out.
__device__ __forceinline__ bool grid_barrier(unsigned* ctl, unsigned nblocks, long long limit_cycles) {
  volatile unsigned* vgen = ctl + 1;
  const unsigned g0 = *vgen;
  __threadfence();
  const unsigned prev = atomicAdd(ctl, 1u);
  if (prev == nblocks - 1) {
    atomicExch(ctl, 0u);
    __threadfence();
    atomicAdd(ctl + 1, 1u);
    return true;
  }
  const long long t0 = clock64();
  while (*vgen == g0) {
    if (clock64() - t0 > limit_cycles) return false;
    __nanosleep(64);
  }
  __threadfence();
  return true;
}

template <int BG, int BD, int BPW, int GS>
__global__ void __launch_bounds__(kFuThreads, 1) ffn_fused_kernel(const FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const int NSG = a.gu_nstage, SBG = a.gu_stage_bytes, NSD = a.d_nstage, SBD = a.d_stage_bytes;
  uint8_t* gst = smem;                                  // gate/up stages
  uint8_t* dst_ = gst + (size_t)NSG * SBG;              // down stages
  uint8_t* hst = dst_ + (size_t)NSD * SBD;              // staged h (kHStageMax)
  float* red = reinterpret_cast<float*>(hst + kHStageMax);                     // [kRedBatch][8][32][4]
  float* ypart = red + kRedBatch * kFuConsumers * 32 * 4;                      // [8][32][4]
  RedMeta* rmeta = reinterpret_cast<RedMeta*>(ypart + kFuConsumers * 32 * 4);  // [kRedBatch]
  ExpMeta* gmeta = reinterpret_cast<ExpMeta*>(rmeta + kRedBatch);             // gate/up experts of this CTA
  int* gtok = reinterpret_cast<int*>(gmeta + kMaxCtaExperts);                  // [64][8]
  ExpMeta* dmeta = reinterpret_cast<ExpMeta*>(gtok + kMaxCtaExperts * kDenseMaxTokens);  // pass experts
  int* dtok = reinterpret_cast<int*>(dmeta + kMaxCtaExperts);
  float* dw = reinterpret_cast<float*>(dtok + kMaxCtaExperts * kDenseMaxTokens);
  uint64_t* gfull = reinterpret_cast<uint64_t*>(dw + kMaxCtaExperts * kDenseMaxTokens);
  uint64_t* gempty = gfull + NSG;
  uint64_t* dfull = gempty + NSG;
  uint64_t* dempty = dfull + NSD;

  pdl_wait();
  const int n_act = pass_count(a);  // <= T*k <= kMaxCtaExperts (dense mode)
  const int jt_n = a.I / 8;
  const int n_items = n_act * jt_n;
  const int i0 = (int)(((int64_t)n_items * blockIdx.x) / gridDim.x);
  const int i1 = (int)(((int64_t)n_items * (blockIdx.x + 1)) / gridDim.x);
  const int my_items = i1 - i0;
  const int n_rt = a.H / 16;
  const int rt = blockIdx.x;  // the launcher makes gridDim.x >= n_rt
  const bool has_rt = rt < n_rt;
  const int n_dn = has_rt ? n_act : 0;
  const int e_first = my_items > 0 ? i0 / jt_n : 0;
  const int n_gexp = my_items > 0 ? (i1 - 1) / jt_n - e_first + 1 : 0;
  if (tid == 0) {
    for (int s = 0; s < NSG; ++s) {
      mbar_init(&gfull[s], 1);
      mbar_init(&gempty[s], kFuConsumers);
    }
    for (int s = 0; s < NSD; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dempty[s], kFuConsumers);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kFuConsumers) {  // producer
    if (lane == 0) {
      const uint32_t tbg = (uint32_t)a.tile_gu, tbd = (uint32_t)a.tile_d;
      int cur_ai = -1, gslot = -1;
      auto issue_gu = [&](int r) -> bool {
        const int s = r % NSG;
        if (r >= NSG && !mbar_wait_bounded(&gempty[s], (uint32_t)(((r / NSG) - 1) & 1))) return false;
        const int item = i0 + r;
        if (item / jt_n != cur_ai) {
          cur_ai = item / jt_n;
          gslot = a.table[a.active[a.pass_begin + cur_ai]];
        }
        if (!slot_ok(a, gslot)) {
          mbar_arrive_expect_tx(&gfull[s], 0);
          return true;
        }
        mbar_arrive_expect_tx(&gfull[s], tbg);
        bulk_g2s(gst + (size_t)s * SBG, a.pool + (int64_t)gslot * a.slot_bytes + a.q_gu + (int64_t)(item % jt_n) * tbg,
                 tbg, &gfull[s]);
        return true;
      };
      auto issue_dn = [&](int r) -> bool {
        const int s = r % NSD;
        if (r >= NSD && !mbar_wait_bounded(&dempty[s], (uint32_t)(((r / NSD) - 1) & 1))) return false;
        const int slot = a.table[a.active[a.pass_begin + r]];
        if (!slot_ok(a, slot)) {
          mbar_arrive_expect_tx(&dfull[s], 0);
          return true;
        }
        mbar_arrive_expect_tx(&dfull[s], tbd);
        bulk_g2s(dst_ + (size_t)s * SBD, a.pool + (int64_t)slot * a.slot_bytes + a.q_d + (int64_t)rt * tbd, tbd,
                 &dfull[s]);
        return true;
      };
      // everything that fits goes out at once; the rest as stages free up
      bool ok = true;
      int rg = 0, rd = 0;
      for (; ok && rg < my_items && rg < NSG; ++rg) ok = issue_gu(rg);
      for (; ok && rd < n_dn && rd < NSD; ++rd) ok = issue_dn(rd);
      for (; ok && rg < my_items; ++rg) ok = issue_gu(rg);
      for (; ok && rd < n_dn; ++rd) ok = issue_dn(rd);
      if (!ok && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
    }
    return;
  }

  // consumers: metadata of this CTA's gate/up experts and of the pass's experts
  load_expert_meta<true>(a, e_first, n_gexp, gmeta, gtok, nullptr, kFuConsumers * 32);
  if (has_rt) load_expert_meta<true>(a, 0, n_act, dmeta, dtok, dw, kFuConsumers * 32);
  consumers_sync(kFuConsumers * 32);
  bool timed_out = false;

  // ---------------- phase 1: gate/up + SwiGLU -> h ----------------
  {
    const int GRP = 8 * (int)a.rb_gu;
    const int uoff = thread_unit_off<BG>(t4, g8);
    uint32_t bf[BPW][8][2];
    float xs[BPW][8 / GS][2], xo[BPW][8 / GS][2];
    const uint16_t* xrow = g8 < a.T ? a.x + (int64_t)g8 * a.H : nullptr;
#pragma unroll
    for (int bi = 0; bi < BPW; ++bi) load_b_block<BG, GS>(xrow, warp * BPW + bi, a.H, t4, bf[bi], xs[bi], xo[bi]);
    int nent = 0;
    auto flush = [&]() {
      consumers_sync(kFuConsumers * 32);
      for (int idx = tid; idx < nent * 64; idx += kFuConsumers * 32) {
        const int en = idx >> 6, j = (idx >> 3) & 7, n = idx & 7;
        const RedMeta m = rmeta[en];
        const int pos = n < a.T ? gtok[m.ei * kDenseMaxTokens + n] : -1;
        if (pos < 0) continue;
        const int src = 4 * j + (n >> 1), c = n & 1;
        const float* rp = red + (size_t)en * kFuConsumers * 32 * 4;
        float gate = 0.f, up = 0.f;
#pragma unroll
        for (int w = 0; w < kFuConsumers; ++w) {
          gate += rp[(w * 32 + src) * 4 + c];
          up += rp[(w * 32 + src) * 4 + 2 + c];
        }
        a.h[(int64_t)pos * a.I + m.jt * 8 + j] = f32_to_bf16_rne(gate / (1.0f + expf(-gate)) * up);
      }
      consumers_sync(kFuConsumers * 32);
      nent = 0;
    };
    for (int r = 0; r < my_items; ++r) {
      const int s = r % NSG;
      const int item = i0 + r;
      const int jt = item % jt_n;
      const int ei = item / jt_n - e_first;
      const bool ok = slot_ok(a, gmeta[ei].slot);
      if (!ok && tid == 0 && jt == 0) flag_slot(a, gmeta[ei].slot);
      if (!timed_out && !mbar_wait_bounded(&gfull[s], (uint32_t)((r / NSG) & 1))) timed_out = true;
      if (ok) {
        const uint8_t* st = gst + (size_t)s * SBG;
        const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int bi = 0; bi < BPW; ++bi) {
          const int kb = warp * BPW + bi;
          if (kb < a.nblk_gu && !timed_out)
            block_mma<BG, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf[bi], xs[bi], xo[bi], acc);
        }
        *reinterpret_cast<float4*>(&red[(((size_t)nent * kFuConsumers + warp) * 32 + lane) * 4]) =
            make_float4(acc[0], acc[1], acc[2], acc[3]);
        if (warp == 0 && lane == 0) rmeta[nent] = RedMeta{ei, 0, a.T, jt};
        if (++nent == kRedBatch) flush();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&gempty[s]);
    }
    if (nent > 0) flush();
  }

  // ---------------- grid barrier: every h row is written ----------------
  __threadfence();
  consumers_sync(kFuConsumers * 32);
  __shared__ int s_barrier_ok;
  if (tid == 0) s_barrier_ok = grid_barrier(a.ctl, gridDim.x, 4000000000ll) ? 1 : 0;
  consumers_sync(kFuConsumers * 32);
  if (!s_barrier_ok) timed_out = true;

  // ---------------- phase 2: down + combine -> y ----------------
  if (has_rt) {
    const int GRP = 8 * (int)a.rb_d;
    const int uoff = thread_unit_off<BD>(t4, g8);
    const int np = a.T * a.k;
    const bool h_staged = (size_t)np * a.I * 2 <= (size_t)kHStageMax;
    if (h_staged && !timed_out) {
      const uint4* src = reinterpret_cast<const uint4*>(a.h);
      uint4* dstp = reinterpret_cast<uint4*>(hst);
      for (int i = tid; i < np * a.I / 8; i += kFuConsumers * 32) dstp[i] = __ldcg(src + i);
    }
    consumers_sync(kFuConsumers * 32);
    // warps w and w+4 split K the same way; the two halves take experts in turn
    const int kq = warp % kDnKSplit, grp = warp / kDnKSplit, ngrp = kFuConsumers / kDnKSplit;
    float yacc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < n_dn; ++r) {
      const int s = r % NSD;
      const ExpMeta em = dmeta[r];
      if (!timed_out && !mbar_wait_bounded(&dfull[s], (uint32_t)((r / NSD) & 1))) timed_out = true;
      if (slot_ok(a, em.slot) && (r % ngrp) == grp && !timed_out) {
        const uint8_t* st = dst_ + (size_t)s * SBD;
        const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
        const int pos = g8 < a.T ? dtok[r * kDenseMaxTokens + g8] : -1;
        const uint16_t* hrow = pos < 0 ? nullptr
                               : h_staged ? reinterpret_cast<const uint16_t*>(hst) + (size_t)pos * a.I
                                          : a.h + (int64_t)pos * a.I;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = kq; kb < a.nblk_d; kb += kDnKSplit) {
          uint32_t bf[8][2];
          float xs[8 / GS][2], xo[8 / GS][2];
          load_b_block<BD, GS>(hrow, kb, a.I, t4, bf, xs, xo);
          block_mma<BD, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs, xo, acc);
        }
        const float w0 = dw[r * kDenseMaxTokens + 2 * t4], w1 = dw[r * kDenseMaxTokens + 2 * t4 + 1];
        yacc[0] += w0 * acc[0];
        yacc[1] += w1 * acc[1];
        yacc[2] += w0 * acc[2];
        yacc[3] += w1 * acc[3];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[s]);
    }
    *reinterpret_cast<float4*>(&ypart[(warp * 32 + lane) * 4]) = make_float4(yacc[0], yacc[1], yacc[2], yacc[3]);
    consumers_sync(kFuConsumers * 32);
    for (int i = tid; i < a.T * 16; i += kFuConsumers * 32) {
      const int tok = i >> 4, row = i & 15;
      const int src = 4 * (row & 7) + (tok >> 1), c = (row >> 3) * 2 + (tok & 1);
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kFuConsumers; ++w) sum += ypart[(w * 32 + src) * 4 + c];
      float* yp = a.y + (int64_t)tok * a.H + rt * 16 + row;
      *yp = a.y_overwrite ? sum : *yp + sum;
    }
  }
  if (timed_out && lane == 0 && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------
template <int BG, int BD, int BPW, int GS>
static cudaError_t launch_fused_t(const FfnArgs& a, int grid, size_t smem, cudaStream_t st) {
  static int done[4] = {0, 0, 0, 0};
  const void* kern = reinterpret_cast<const void*>(ffn_fused_kernel<BG, BD, BPW, GS>);
  cudaError_t e = ensure_smem_attr(kern, done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)kFuThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  void* argv[] = {const_cast<void*>(static_cast<const void*>(&a))};
  // co-residency of every CTA is required (grid barrier): always cooperative;
  // early launch behind the previous kernel as well where the driver accepts
  // the combination (remembered after the first refusal)
  static int pdl_refused = 0;
  if (!__atomic_load_n(&pdl_refused, __ATOMIC_RELAXED)) {
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelExC(&cfg, kern, argv);
    if (e != cudaErrorInvalidValue && e != cudaErrorNotSupported) return e;
    (void)cudaGetLastError();  // a refused launch configuration is not sticky
    __atomic_store_n(&pdl_refused, 1, __ATOMIC_RELAXED);
  }
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, kern, argv);
}

template <int BG, int BD, int BPW>
static cudaError_t fused_gs(const FfnArgs& a, int gs, int grid, size_t smem, cudaStream_t st) {
  if (gs == 2) return launch_fused_t<BG, BD, BPW, 2>(a, grid, smem, st);
  if (gs == 4) return launch_fused_t<BG, BD, BPW, 4>(a, grid, smem, st);
  return launch_fused_t<BG, BD, BPW, 8>(a, grid, smem, st);
}

template <int BG, int BD>
static cudaError_t fused_bpw(const FfnArgs& a, int bpw, int gs, int grid, size_t smem, cudaStream_t st) {
  if (bpw == 1) return fused_gs<BG, BD, 1>(a, gs, grid, smem, st);
  return fused_gs<BG, BD, 2>(a, gs, grid, smem, st);
}

template <int BG>
static cudaError_t fused_bd(const FfnArgs& a, int bd, int bpw, int gs, int grid, size_t smem, cudaStream_t st) {
  if (bd == 3) return fused_bpw<BG, 3>(a, bpw, gs, grid, smem, st);
  if (bd == 4) return fused_bpw<BG, 4>(a, bpw, gs, grid, smem, st);
  return fused_bpw<BG, 6>(a, bpw, gs, grid, smem, st);
}

// Returns cudaErrorNotSupported when the fused path does not apply (the
// caller then uses the two-kernel path).
cudaError_t launch_ffn_fused(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st) {
  if (!(a.T <= kDenseMaxTokens && a.T * d.k <= kMaxCtaExperts) || a.ctl == nullptr) return cudaErrorNotSupported;
  const int nblk = a.L.nblk_gu;
  if (nblk > 2 * kFuConsumers) return cudaErrorNotSupported;
  const int bpw = nblk <= kFuConsumers ? 1 : 2;
  const int n_rt = d.H / 16;
  if (n_rt > num_sms) return cudaErrorNotSupported;
  const int grid = num_sms;
  int max_pass = a.pass_len < d.E ? a.pass_len : d.E;
  if (a.T * d.k < max_pass) max_pass = a.T * d.k;
  a.gu_stage_bytes = (int)round_up(a.L.tile_gu, 128);
  a.d_stage_bytes = (int)round_up(a.L.tile_d, 128);
  const int64_t items_per_cta = ((int64_t)max_pass * (d.I / 8) + grid - 1) / grid;
  const size_t fixed = (size_t)kHStageMax + (size_t)kRedBatch * kFuConsumers * 32 * 4 * 4 +
                       (size_t)kFuConsumers * 32 * 4 * 4 + kRedBatch * sizeof(RedMeta) +
                       2 * (size_t)kMaxCtaExperts * (sizeof(ExpMeta) + kDenseMaxTokens * 2 * sizeof(int));
  const size_t cap = 220 * 1024;
  if (fixed + a.gu_stage_bytes + a.d_stage_bytes + 64 > cap) return cudaErrorNotSupported;
  // down stages: every expert of the pass if possible, else half the room
  int nsd = max_pass;
  int nsg = (int)(items_per_cta < 1 ? 1 : items_per_cta);
  while ((size_t)nsd * a.d_stage_bytes + (size_t)nsg * a.gu_stage_bytes + fixed + 16 * (nsd + nsg) > cap) {
    if (nsg > nsd && nsg > 2) --nsg;
    else if (nsd > 2) --nsd;
    else if (nsg > 1) --nsg;
    else return cudaErrorNotSupported;
  }
  a.gu_nstage = nsg;
  a.d_nstage = nsd;
  const size_t smem = (size_t)nsg * a.gu_stage_bytes + (size_t)nsd * a.d_stage_bytes + fixed + 16 * (nsd + nsg);
  const int gs = d.group / 16;
  if (d.bits_gu == 3) return fused_bd<3>(a, d.bits_down, bpw, gs, grid, smem, st);
  if (d.bits_gu == 4) return fused_bd<4>(a, d.bits_down, bpw, gs, grid, smem, st);
  return fused_bd<6>(a, d.bits_down, bpw, gs, grid, smem, st);
}

}  // namespace moe
