// Decode FFN in one launch (T <= 8 tokens, every routed pair in the per-CTA
// tables): gate/up + SwiGLU, a grid-wide barrier, then down + combine.
//
// One CTA per SM, all co-resident (cooperative launch).  At kernel start
// every CTA reads the pass's tables in one round of independent loads (the
// active expert list, the routed ids and weights), then the producer warp
// resolves the slots (one more round) and its 32 lanes issue, in parallel, the
// bulk copies of everything the CTA will read: its gate/up tiles (one 16-row
// tile per (expert, 8 j) item) and its 16-row slice of every active expert's
// down projection.  The down weights therefore stream in while gate/up
// computes, and the layer pays for one launch and one memory latency instead
// of two.  No sorted pair order is needed: h rows are indexed by the flat
// (token, rank) pair, and each expert's tokens are found in the routed ids.
// The barrier between the phases is a monotonic 64-bit arrival counter in the
// workspace (release add, acquire poll), bounded by a clock limit
// (MOE_DEV_ERR_TIMEOUT on expiry).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ffn_common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kFuThreads = (kFuConsumers + 1) * 32;
// per-pass tables in shared memory: active ids, slots, routed ids, routed
// weights (kMaxCtaExperts each) and the (expert, token) -> pair map
constexpr size_t kFuTableBytes =
    (size_t)kMaxCtaExperts * (3 * sizeof(int) + sizeof(float)) + (size_t)kMaxCtaExperts * kDenseMaxTokens * sizeof(int);

// Grid barrier on a 64-bit arrival counter that only grows: every launch
// adds gridDim.x, so a launch starts with the counter at a multiple of the
// grid size (zero-initialised workspace) and each CTA waits for the next
// multiple above its own arrival.  Called by one thread per CTA after a
// CTA-wide barrier; the release add publishes the CTA's global writes and the
// acquire load makes the other CTAs' writes visible.  Returns false if the
// wait ran out (the counter is then no longer aligned: the caller must zero
// the control block before the next launch).
__device__ __forceinline__ bool grid_barrier(unsigned long long* ctr, unsigned nblocks, long long limit_cycles) {
  unsigned long long old, cur;
  asm volatile("atom.add.release.gpu.u64 %0, [%1], 1;" : "=l"(old) : "l"(ctr) : "memory");
  const unsigned long long target = old - old % nblocks + nblocks;
  const long long t0 = clock64();
  for (;;) {
    asm volatile("ld.acquire.gpu.u64 %0, [%1];" : "=l"(cur) : "l"(ctr) : "memory");
    if ((long long)(cur - target) >= 0) return true;
    if (clock64() - t0 > limit_cycles) return false;
  }
}

// Named barrier 2 over all threads of the CTA: the producer warp arrives once
// the slot table is written, the consumer warps wait on it.
__device__ __forceinline__ void tables_arrive() { asm volatile("bar.arrive 2, %0;" ::"n"(kFuThreads) : "memory"); }
__device__ __forceinline__ void tables_sync() { asm volatile("bar.sync 2, %0;" ::"n"(kFuThreads) : "memory"); }

template <int BG, int BD, int BPW, int GS>
__global__ void __launch_bounds__(kFuThreads, 1) ffn_fused_kernel(const FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const int NSG = a.gu_nstage, SBG = a.gu_stage_bytes, NSD = a.d_nstage, SBD = a.d_stage_bytes;
  uint8_t* gst = smem;                                  // gate/up stages
  uint8_t* dst_ = gst + (size_t)NSG * SBG;              // down stages
  uint8_t* hst = dst_ + (size_t)NSD * SBD;              // staged x, later staged h
  float* red = reinterpret_cast<float*>(hst + a.xh_stage_bytes);               // [kRedBatch][8][32][4]
  float* ypart = red + kRedBatch * kFuConsumers * 32 * 4;                      // [8][32][4]
  RedMeta* rmeta = reinterpret_cast<RedMeta*>(ypart + kFuConsumers * 32 * 4);  // [kRedBatch]
  int* s_act = reinterpret_cast<int*>(rmeta + kRedBatch);  // pass entry -> expert id
  int* s_slot = s_act + kMaxCtaExperts;                    // pass entry -> slot
  int* s_ids = s_slot + kMaxCtaExperts;                    // flat pair -> expert id
  float* s_w = reinterpret_cast<float*>(s_ids + kMaxCtaExperts);  // flat pair -> routing weight
  int* s_tok = reinterpret_cast<int*>(s_w + kMaxCtaExperts);      // [entry][token] -> flat pair or -1
  uint64_t* gfull = reinterpret_cast<uint64_t*>(s_tok + kMaxCtaExperts * kDenseMaxTokens);
  uint64_t* gempty = gfull + NSG;
  uint64_t* dfull = gempty + NSG;
  uint64_t* dempty = dfull + NSD;
  __shared__ int s_nact;

  pdl_wait();
  // one round of independent loads: pass length, active list, routed pairs
  const int np = a.T * a.k;  // <= kMaxCtaExperts (dense mode)
  int cap = a.E - a.pass_begin;
  if (cap > a.pass_len) cap = a.pass_len;
  if (cap > kMaxCtaExperts) cap = kMaxCtaExperts;
  if (tid == 0) s_nact = pass_count(a);
  for (int i = tid; i < cap; i += kFuThreads) s_act[i] = a.active[a.pass_begin + i];
  for (int p = tid; p < np; p += kFuThreads) {
    s_ids[p] = a.ids[p];
    s_w[p] = a.w[p];
  }
  // x -> shared memory in the same round (x is 16-byte aligned and H a
  // multiple of 32, so x is a whole number of 16-byte words)
  {
    const int nx = a.T * a.H / 8;
    uint4* xd = reinterpret_cast<uint4*>(hst);
    for (int b0 = tid; b0 < nx; b0 += 4 * kFuThreads) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (b0 + u * kFuThreads < nx) v[u] = __ldg(reinterpret_cast<const uint4*>(a.x) + b0 + u * kFuThreads);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (b0 + u * kFuThreads < nx) xd[b0 + u * kFuThreads] = v[u];
    }
  }
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
  // consumers: x fragments of the gate/up blocks, from shared memory
  uint32_t xbf[BPW][8][2];
  float xs[BPW][8 / GS][2], xo[BPW][8 / GS][2];
  if (warp < kFuConsumers) {
    const uint16_t* xrow = g8 < a.T ? reinterpret_cast<const uint16_t*>(hst) + g8 * a.H : nullptr;
#pragma unroll
    for (int bi = 0; bi < BPW; ++bi) load_b_block<BG, GS>(xrow, warp * BPW + bi, a.H, t4, xbf[bi], xs[bi], xo[bi]);
  }
  const int n_act = s_nact < cap ? s_nact : cap;
  const int jt_n = a.I / 8;
  const int n_items = n_act * jt_n;
  const int i0 = (int)(((int64_t)n_items * blockIdx.x) / gridDim.x);
  const int i1 = (int)(((int64_t)n_items * (blockIdx.x + 1)) / gridDim.x);
  const int my_items = i1 - i0;
  const int n_rt = a.H / 16;
  const int rt = blockIdx.x;  // the launcher makes gridDim.x >= n_rt
  const bool has_rt = rt < n_rt;
  const int n_dn = has_rt ? n_act : 0;
  const int Ip = a.nblk_d * 128;  // h row stride: the intermediate size padded to whole 128-blocks

  if (warp == kFuConsumers) {  // producer
    // second round of loads: the slots of the pass's experts
    for (int i = lane; i < n_act; i += 32) {
      const int e = s_act[i];
      s_slot[i] = (e >= 0 && e < a.E) ? a.table[e] : -1;
    }
    __syncwarp();
    tables_arrive();
    {
      const uint32_t tbg = (uint32_t)a.tile_gu, tbd = (uint32_t)a.tile_d;
      auto issue_gu = [&](int r) -> bool {
        const int s = r % NSG;
        if (r >= NSG && !mbar_wait_bounded(&gempty[s], (uint32_t)(((r / NSG) - 1) & 1))) return false;
        const int item = i0 + r;
        const int gslot = s_slot[item / jt_n];
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
        const int slot = s_slot[r];
        if (!slot_ok(a, slot)) {
          mbar_arrive_expect_tx(&dfull[s], 0);
          return true;
        }
        mbar_arrive_expect_tx(&dfull[s], tbd);
        bulk_g2s(dst_ + (size_t)s * SBD, a.pool + (int64_t)slot * a.slot_bytes + a.q_d + (int64_t)rt * tbd, tbd,
                 &dfull[s]);
        return true;
      };
      // everything that fits goes out at once, one copy per lane; the rest
      // (lane 0) as stages free up
      const int ng0 = my_items < NSG ? my_items : NSG, nd0 = n_dn < NSD ? n_dn : NSD;
      for (int r = lane; r < ng0; r += 32) issue_gu(r);
      for (int r = lane; r < nd0; r += 32) issue_dn(r);
      if (lane == 0) {
        bool ok = true;
        for (int r = ng0; ok && r < my_items; ++r) ok = issue_gu(r);
        for (int r = nd0; ok && r < n_dn; ++r) ok = issue_dn(r);
        if (!ok && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
      }
    }
    return;
  }

  // consumers: (entry, token) -> flat pair map from the routed ids (a token
  // routes to an expert at most once)
  for (int i = tid; i < n_act * kDenseMaxTokens; i += kFuConsumers * 32) {
    const int r = i / kDenseMaxTokens, t = i % kDenseMaxTokens;
    int p = -1;
    if (t < a.T) {
      const int e = s_act[r];
      for (int j = 0; j < a.k; ++j)
        if (s_ids[t * a.k + j] == e) p = t * a.k + j;
    }
    s_tok[i] = p;
  }
  tables_sync();  // slots written by the producer; pair map by all consumers
  if (blockIdx.x == 0)
    for (int i = tid; i < n_act; i += kFuConsumers * 32)
      if (!slot_ok(a, s_slot[i])) flag_slot(a, s_slot[i]);
  bool timed_out = false;

  // ---------------- phase 1: gate/up + SwiGLU -> h ----------------
  {
    const int GRP = 8 * (int)a.rb_gu;
    const int uoff = thread_unit_off<BG>(t4, g8);
    const bool all_blocks = (warp + 1) * BPW <= a.nblk_gu;
    int nent = 0;
    auto flush = [&]() {
      consumers_sync(kFuConsumers * 32);
      // eight consecutive lanes hold the eight columns of one (entry, token);
      // h is stored scaled by 2^-a of its down pair slot (exact: a power of
      // two), with the partial sums (sum h, sum 128 h 2^-a) of the eight
      for (int idx = tid; idx < nent * 64; idx += kFuConsumers * 32) {
        const int en = idx >> 6, n = (idx >> 3) & 7, j = idx & 7;
        const RedMeta m = rmeta[en];
        const int pos = s_tok[m.ei * kDenseMaxTokens + n];  // -1 for absent tokens
        const int src = 4 * j + (n >> 1), c = n & 1;
        const float* rp = red + (size_t)en * kFuConsumers * 32 * 4;
        float gate = 0.f, up = 0.f;
#pragma unroll
        for (int w = 0; w < kFuConsumers; ++w) {
          gate += rp[(w * 32 + src) * 4 + c];
          up += rp[(w * 32 + src) * 4 + 2 + c];
        }
        const float hv = gate / (1.0f + expf(-gate)) * up;
        const int kcol = m.jt * 8 + j, kk = kcol & 127;
        const bool eighth = PairShift<BD>::a(2 * (kk >> 4) + ((kk & 15) >> 3)) == 3;
        const uint16_t hb = f32_to_bf16_rne(eighth ? hv * 0.125f : hv);
        const float hsv = __uint_as_float((uint32_t)hb << 16);
        float sx = eighth ? 8.0f * hsv : hsv, so = 128.0f * hsv;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          sx += __shfl_xor_sync(0xffffffffu, sx, o);
          so += __shfl_xor_sync(0xffffffffu, so, o);
        }
        if (pos >= 0) {
          a.h[(int64_t)pos * Ip + kcol] = hb;
          if (j == 0) *reinterpret_cast<float2*>(a.hpart + 2 * ((int64_t)pos * (Ip / 8) + m.jt)) = make_float2(sx, so);
        }
      }
      consumers_sync(kFuConsumers * 32);
      nent = 0;
    };
    // stage / parity and (expert entry, 8-row tile) advance incrementally
    int s = 0, jt = i0 % jt_n, ei = i0 / jt_n;
    uint32_t ph = 0;
    for (int r = 0; r < my_items; ++r) {
      const bool ok = slot_ok(a, s_slot[ei]);
      if (!timed_out && !mbar_wait_bounded(&gfull[s], ph)) timed_out = true;
      if (ok) {
        const uint8_t* st = gst + (size_t)s * SBG;
        const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (!timed_out) {
          if (all_blocks) {  // straight-line: the blocks' chains interleave
#pragma unroll
            for (int bi = 0; bi < BPW; ++bi)
              block_mma<BG, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, warp * BPW + bi, uoff, xbf[bi], xs[bi], xo[bi],
                                acc);
          } else {
#pragma unroll
            for (int bi = 0; bi < BPW; ++bi)
              if (warp * BPW + bi < a.nblk_gu)
                block_mma<BG, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, warp * BPW + bi, uoff, xbf[bi], xs[bi],
                                  xo[bi], acc);
          }
        }
        *reinterpret_cast<float4*>(&red[(((size_t)nent * kFuConsumers + warp) * 32 + lane) * 4]) =
            make_float4(acc[0], acc[1], acc[2], acc[3]);
        if (warp == 0 && lane == 0) rmeta[nent] = RedMeta{ei, 0, a.T, jt};
        if (++nent == kRedBatch) flush();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&gempty[s]);
      if (++s == NSG) {
        s = 0;
        ph ^= 1u;
      }
      if (++jt == jt_n) {
        jt = 0;
        ++ei;
      }
    }
    if (nent > 0) flush();
  }

  // ---------------- grid barrier: every h row is written ----------------
  consumers_sync(kFuConsumers * 32);
  __shared__ int s_barrier_ok;
  if (tid == 0)
    s_barrier_ok = grid_barrier(reinterpret_cast<unsigned long long*>(a.ctl), gridDim.x, 4000000000ll) ? 1 : 0;
  consumers_sync(kFuConsumers * 32);
  if (!s_barrier_ok) timed_out = true;

  // ---------------- phase 2: down + combine -> y ----------------
  if (has_rt) {
    const int GRP = 8 * (int)a.rb_d;
    const int uoff = thread_unit_off<BD>(t4, g8);
    // h (already scaled by 2^-a) -> shared memory, padding columns zeroed,
    // and per (pair, group) the epilogue sums from the per-8-column partials
    const int ngd = Ip / a.g;
    uint16_t* hs = reinterpret_cast<uint16_t*>(hst);
    float2* hsum = reinterpret_cast<float2*>(hst + (size_t)np * Ip * 2);
    if (!timed_out) {
      const int cpr = Ip / 8, nh = np * cpr;
      const bool padded = Ip != a.I;
      const uint4* hsrc = reinterpret_cast<const uint4*>(a.h);
      for (int b0 = tid; b0 < nh; b0 += 4 * kFuConsumers * 32) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = b0 + u * kFuConsumers * 32;
          v[u] = (i < nh && (!padded || 8 * (i % cpr) < a.I)) ? __ldcg(hsrc + i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (b0 + u * kFuConsumers * 32 < nh) reinterpret_cast<uint4*>(hs)[b0 + u * kFuConsumers * 32] = v[u];
      }
      const int cpg = a.g / 8, jt_i = a.I / 8;  // partials per group; 8-column tiles of I
      // task = p * ngd + G, stepped by the thread count without dividing
      const int dp = (kFuConsumers * 32) / ngd, dG = (kFuConsumers * 32) % ngd;
      int p = tid / ngd, G = tid % ngd;
      for (int task = tid; task < np * ngd; task += kFuConsumers * 32) {
        const float4* src = reinterpret_cast<const float4*>(a.hpart + 2 * ((int64_t)p * cpr + G * cpg));
        float sx = 0.f, so = 0.f;
        for (int c0 = 0; c0 < cpg / 2; c0 += 8) {
          float4 v[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            v[c] = (c0 + c < cpg / 2 && G * cpg + 2 * (c0 + c) < jt_i) ? __ldcg(src + c0 + c)
                                                                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            sx += v[c].x + v[c].z;
            so += v[c].y + v[c].w;
          }
        }
        hsum[task] = make_float2(sx, so);
        p += dp;
        G += dG;
        if (G >= ngd) {
          G -= ngd;
          ++p;
        }
      }
    }
    consumers_sync(kFuConsumers * 32);
    // warps w and w+4 split K the same way; the two halves take experts in
    // turn.  A window of 2 * ngrp experts gives every warp two experts whose
    // load / unpack / MMA chains are independent and run interleaved (one
    // expert per window when fewer stages than that are resident).
    const int kq = warp % kDnKSplit, grp = warp / kDnKSplit, ngrp = kFuConsumers / kDnKSplit;
    const int win = NSD >= 2 * ngrp ? 2 * ngrp : ngrp;
    float yacc[4] = {0.f, 0.f, 0.f, 0.f};
    // B fragments (token column g8) and epilogue sums (columns 2 t4, 2 t4 + 1)
    // of expert entry r, 128-block kb; absent tokens read zeros
    auto frag = [&](int r, int kb, uint32_t(&bf)[8][2], float(&xs)[8 / GS][2], float(&xo)[8 / GS][2]) {
      const int pb = s_tok[r * kDenseMaxTokens + g8];
      const int p0 = s_tok[r * kDenseMaxTokens + 2 * t4], p1 = s_tok[r * kDenseMaxTokens + 2 * t4 + 1];
      const uint16_t* row = pb < 0 ? nullptr : hs + (size_t)pb * Ip + kb * 128 + 2 * t4;
#pragma unroll
      for (int st = 0; st < 8; ++st) {
        bf[st][0] = row ? ld_pair(row + 16 * st) : 0u;
        bf[st][1] = row ? ld_pair(row + 16 * st + 8) : 0u;
      }
#pragma unroll
      for (int G = 0; G < 8 / GS; ++G) {
        const int gi = kb * (8 / GS) + G;
        const float2 v0 = p0 < 0 ? make_float2(0.f, 0.f) : hsum[p0 * ngd + gi];
        const float2 v1 = p1 < 0 ? make_float2(0.f, 0.f) : hsum[p1 * ngd + gi];
        xs[G][0] = v0.x;
        xo[G][0] = v0.y;
        xs[G][1] = v1.x;
        xo[G][1] = v1.y;
      }
    };
    auto combine = [&](int r, const float (&acc)[4]) {
      const int p0 = s_tok[r * kDenseMaxTokens + 2 * t4], p1 = s_tok[r * kDenseMaxTokens + 2 * t4 + 1];
      const float w0 = p0 >= 0 ? s_w[p0] : 0.f, w1 = p1 >= 0 ? s_w[p1] : 0.f;
      yacc[0] += w0 * acc[0];
      yacc[1] += w1 * acc[1];
      yacc[2] += w0 * acc[2];
      yacc[3] += w1 * acc[3];
    };
    // stage and parity of the window's first expert (win <= NSD: a window
    // wraps around the stages at most once)
    int s0 = 0;
    uint32_t ph0 = 0;
    auto stage_of = [&](int q) -> int { return s0 + q < NSD ? s0 + q : s0 + q - NSD; };
    for (int r0 = 0; r0 < n_dn; r0 += win) {
      const int r1 = r0 + win < n_dn ? r0 + win : n_dn;
      for (int q = 0; q < r1 - r0; ++q)
        if (!timed_out && !mbar_wait_bounded(&dfull[stage_of(q)], s0 + q < NSD ? ph0 : ph0 ^ 1u)) timed_out = true;
      const int ra = r0 + grp, rb = r0 + ngrp + grp;
      const bool va = !timed_out && ra < r1 && slot_ok(a, s_slot[ra]);
      const bool vb = !timed_out && win > ngrp && rb < r1 && slot_ok(a, s_slot[rb]);
      if (va && vb) {
        const uint8_t* sta = dst_ + (size_t)stage_of(grp) * SBD;
        const uint8_t* stb = dst_ + (size_t)stage_of(ngrp + grp) * SBD;
        const uint32_t* sba = reinterpret_cast<const uint32_t*>(sta + 2 * GRP);
        const uint32_t* sbb = reinterpret_cast<const uint32_t*>(stb + 2 * GRP);
        float acca[4] = {0.f, 0.f, 0.f, 0.f}, accb[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = kq; kb < a.nblk_d; kb += kDnKSplit) {
          uint32_t bfa[8][2], bfb[8][2];
          float xsa[8 / GS][2], xoa[8 / GS][2], xsb[8 / GS][2], xob[8 / GS][2];
          frag(ra, kb, bfa, xsa, xoa);
          frag(rb, kb, bfb, xsb, xob);
          block_mma<BD, GS>(sta, sta + GRP, sba + g8, sba + 8 + g8, kb, uoff, bfa, xsa, xoa, acca);
          block_mma<BD, GS>(stb, stb + GRP, sbb + g8, sbb + 8 + g8, kb, uoff, bfb, xsb, xob, accb);
        }
        combine(ra, acca);
        combine(rb, accb);
      } else if (va || vb) {
        const int rr = va ? ra : rb;
        const uint8_t* st = dst_ + (size_t)stage_of(rr - r0) * SBD;
        const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = kq; kb < a.nblk_d; kb += kDnKSplit) {
          uint32_t bf[8][2];
          float xs1[8 / GS][2], xo1[8 / GS][2];
          frag(rr, kb, bf, xs1, xo1);
          block_mma<BD, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs1, xo1, acc);
        }
        combine(rr, acc);
      }
      __syncwarp();
      if (lane == 0)
        for (int q = 0; q < r1 - r0; ++q) mbar_arrive(&dempty[stage_of(q)]);
      s0 += win;
      if (s0 >= NSD) {
        s0 -= NSD;
        ph0 ^= 1u;
      }
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
// Stage sizes and counts of the fused kernel for this call (into a), its
// shared memory; false when the fused path does not apply.
bool ffn_fused_plan(FfnArgs& a, const moe_layer_desc& d, int num_sms, size_t& smem) {
  if (!(a.T <= kDenseMaxTokens && a.T * d.k <= kMaxCtaExperts) || a.ctl == nullptr) return false;
  if (a.L.nblk_gu > 2 * kFuConsumers) return false;
  if (d.H / 16 > num_sms) return false;
  const int grid = num_sms;
  int max_pass = a.pass_len < d.E ? a.pass_len : d.E;
  if (a.T * d.k < max_pass) max_pass = a.T * d.k;
  a.gu_stage_bytes = (int)round_up(a.L.tile_gu, 128);
  a.d_stage_bytes = (int)round_up(a.L.tile_d, 128);
  const int64_t items_per_cta = ((int64_t)max_pass * (d.I / 8) + grid - 1) / grid;
  {
    // x in the gate/up phase, then h (scaled, rows padded to 128-blocks) and
    // the per-(pair, group) sums in the down phase
    const size_t np = (size_t)a.T * d.k, Ip = (size_t)a.L.nblk_d * 128;
    const size_t xb = (size_t)a.T * d.H * 2, hb = np * Ip * 2 + np * (Ip / d.group) * 8;
    a.xh_stage_bytes = (int)round_up((int64_t)(xb > hb ? xb : hb), 128);
  }
  const size_t fixed = (size_t)a.xh_stage_bytes + (size_t)kRedBatch * kFuConsumers * 32 * 4 * 4 +
                       (size_t)kFuConsumers * 32 * 4 * 4 + kRedBatch * sizeof(RedMeta) +
                       kFuTableBytes;
  const size_t cap = 220 * 1024;
  if (fixed + a.gu_stage_bytes + a.d_stage_bytes + 64 > cap) return false;
  // down stages: every expert of the pass if possible, else half the room; at
  // least one per down warp group, so that a window of experts never waits on
  // a stage it has not released
  constexpr int kMinDn = kFuConsumers / kDnKSplit;
  int nsd = max_pass > kMinDn ? max_pass : kMinDn;
  int nsg = (int)(items_per_cta < 1 ? 1 : items_per_cta);
  while ((size_t)nsd * a.d_stage_bytes + (size_t)nsg * a.gu_stage_bytes + fixed + 16 * (nsd + nsg) > cap) {
    if (nsg > nsd && nsg > 2) --nsg;
    else if (nsd > kMinDn) --nsd;
    else if (nsg > 1) --nsg;
    else return false;
  }
  a.gu_nstage = nsg;
  a.d_nstage = nsd;
  smem = (size_t)nsg * a.gu_stage_bytes + (size_t)nsd * a.d_stage_bytes + fixed + 16 * (nsd + nsg);
  return true;
}

cudaError_t launch_ffn_fused(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st) {
  size_t smem = 0;
  if (!ffn_fused_plan(a, d, num_sms, smem)) return cudaErrorNotSupported;
  const int grid = num_sms;
  const int bpw = a.L.nblk_gu <= kFuConsumers ? 1 : 2;
  const int gs = d.group / 16;
  if (d.bits_gu == 3) return fused_bd<3>(a, d.bits_down, bpw, gs, grid, smem, st);
  if (d.bits_gu == 4) return fused_bd<4>(a, d.bits_down, bpw, gs, grid, smem, st);
  return fused_bd<6>(a, d.bits_down, bpw, gs, grid, smem, st);
}

}  // namespace moe
