// Decode FFN in one launch (T <= 8 tokens, every routed pair in the per-CTA
// tables): gate/up + SwiGLU -> h, then down + weighted combine -> y.
//
// One CTA per SM, all co-resident (cooperative launch), in two roles:
//   * gate/up CTAs (blockIdx.x >= n_dn) take the pass's gate/up items -- a
//     16-row tile (8 gate + 8 up rows) of one expert -- in rounds: item
//     i = r * n_gu + c.  Items run expert-major, so each round finishes the
//     next experts of the pass.  After every pair of items a CTA writes their
//     h columns and adds the item count to each expert's readiness counter
//     (release);
//   * down CTAs (blockIdx.x < n_dn) own rt_per_dn 16-row tiles of the down
//     projection: at kernel start they copy those rows of every active
//     expert (one contiguous bulk copy per expert), then take the experts as
//     their counters report complete (acquire), several at once, and
//     accumulate w * (W_d h) for every token in registers; y is written once.
// The role split is chosen on the host so that every SM streams about the
// same number of bytes.  There is no grid-wide barrier: the down work of the
// first experts overlaps the gate/up work of the last, and a layer costs one
// launch and one metadata round trip.  The producer warp of every CTA reads
// the pass's active experts and the whole expert -> slot table in one round
// of independent loads, then its 32 lanes issue the CTA's bulk copies in
// parallel.
//
// Control block (head of the workspace): one readiness counter per pass
// entry and the down CTAs' departure count.  Every launch starts with them at
// zero; the last down CTA to leave sets them back to zero.  A readiness wait
// is bounded (MOE_DEV_ERR_TIMEOUT) and needs the counter to equal the
// expert's item count exactly, so a counter left over by an interrupted
// launch is reported, not silently used.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ffn_common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kFuThreads = (kFuConsumers + 1) * 32;
constexpr int kFuRtMax = 4;  // 16-row down tiles per down CTA
constexpr int kFuRedFloats = kRedBatch * kFuConsumers * 32 * 4;
static_assert(kFuConsumers * kFuRtMax * 32 * 4 <= kFuRedFloats, "down partial sums fit the reduction buffer");
// control block words
constexpr int kCtlReady = 0;                // uint32 [kMaxCtaExperts]
constexpr int kCtlDepart = kMaxCtaExperts;  // uint32
static_assert((kCtlDepart + 1) * 4 <= (int)kWsControlBytes, "control block size");
// per-pass tables in shared memory: active ids, slots, routed ids, routed
// weights (kMaxCtaExperts each) and the (entry, token) -> flat pair map
constexpr size_t kFuTableBytes =
    (size_t)kMaxCtaExperts * (3 * sizeof(int) + sizeof(float)) + (size_t)kMaxCtaExperts * kDenseMaxTokens * sizeof(int);

__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Named barrier 2 over all threads of the CTA: the producer warp arrives once
// the pass tables are in shared memory, the consumer warps wait on it.
__device__ __forceinline__ void tables_arrive() { asm volatile("bar.arrive 2, %0;" ::"n"(kFuThreads) : "memory"); }
__device__ __forceinline__ void tables_sync() { asm volatile("bar.sync 2, %0;" ::"n"(kFuThreads) : "memory"); }

template <int BG, int BD, int BPW, int GS>
__global__ void __launch_bounds__(kFuThreads, 1) ffn_fused_kernel(const FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const bool dn_role = (int)blockIdx.x < a.fu_n_dn;
  const int NS = dn_role ? a.d_nstage : a.gu_nstage;
  const int SB = dn_role ? a.d_stage_bytes : a.gu_stage_bytes;
  uint8_t* stg = smem;                                         // stages of the CTA's role
  uint8_t* xh = stg + (size_t)a.fu_stage_area;                 // gate/up: x [T][H]; down: h rows + sums
  float* red = reinterpret_cast<float*>(xh + a.xh_stage_bytes);                 // partial sums
  RedMeta* rmeta = reinterpret_cast<RedMeta*>(red + kFuRedFloats);              // [kRedBatch]
  int* s_act = reinterpret_cast<int*>(rmeta + kRedBatch);      // pass entry -> expert id
  int* s_slot = s_act + kMaxCtaExperts;                        // pass entry -> slot
  int* s_ids = s_slot + kMaxCtaExperts;                        // flat pair -> expert id
  float* s_w = reinterpret_cast<float*>(s_ids + kMaxCtaExperts);  // flat pair -> routing weight
  int* s_tok = reinterpret_cast<int*>(s_w + kMaxCtaExperts);      // [entry][token] -> flat pair or -1
  uint64_t* full = reinterpret_cast<uint64_t*>(s_tok + kMaxCtaExperts * kDenseMaxTokens);
  uint64_t* empty = full + NS;
  int* s_table = reinterpret_cast<int*>(empty + NS);           // expert -> slot, [E]
  __shared__ int s_nact;
  __shared__ unsigned long long s_ready;
  __shared__ int s_timeout, s_npl;
  __shared__ int s_plist[kMaxCtaExperts];
  unsigned* ready = a.ctl + kCtlReady;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFuConsumers);
    }
    fence_barrier_init();
    s_timeout = 0;
  }
  __syncthreads();
  pdl_wait();
  const int np = a.T * a.k;  // <= kMaxCtaExperts (dense mode)
  int cap = a.E - a.pass_begin;
  if (cap > a.pass_len) cap = a.pass_len;
  if (cap > kMaxCtaExperts) cap = kMaxCtaExperts;
  if (cap < 0) cap = 0;
  const int jt_n = a.I / 8;
  const int n_gu = (int)gridDim.x - a.fu_n_dn;
  const int n_rt = a.H / 16;
  const int rt0 = (int)blockIdx.x * a.fu_rt_per_dn;
  const int nrt = dn_role ? (n_rt - rt0 < a.fu_rt_per_dn ? n_rt - rt0 : a.fu_rt_per_dn) : 0;
  const int Ip = a.nblk_d * 128;  // h row stride: the intermediate size padded to whole 128-blocks

  if (warp == kFuConsumers) {
    // ---------------- producer: pass tables, then the CTA's bulk copies ----------------
    const int na_raw = *a.n_active;
    int act_v[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int i = lane + 32 * q;
      act_v[q] = i < cap ? a.active[a.pass_begin + i] : -1;
    }
    for (int e0 = 0; e0 < a.E; e0 += 512) {  // the table in one round (two for E > 512)
      int v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int e = e0 + lane + 32 * u;
        v[u] = e < a.E ? a.table[e] : -1;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int e = e0 + lane + 32 * u;
        if (e < a.E) s_table[e] = v[u];
      }
    }
    int n_act = na_raw - a.pass_begin;
    if (n_act > cap) n_act = cap;
    if (n_act < 0) n_act = 0;
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int i = lane + 32 * q;
      if (i < cap) s_act[i] = act_v[q];
      if (i < n_act) {
        const int e = act_v[q];
        s_slot[i] = (e >= 0 && e < a.E) ? s_table[e] : -1;
      }
    }
    if (lane == 0) s_nact = n_act;
    __syncwarp();
    tables_arrive();
    const int64_t sbytes = a.slot_bytes;
    bool ok = true;
    if (dn_role) {
      // entry i: rows rt0*16 .. (rt0+nrt)*16 of its down projection, one copy
      const uint32_t bytes = (uint32_t)(nrt * a.tile_d);
      auto issue = [&](int i) -> bool {
        const int s = i % NS;
        if (i >= NS && !mbar_wait_bounded(&empty[s], (uint32_t)(((i / NS) - 1) & 1), a.wait_limit)) return false;
        const int slot = s_slot[i];
        if (!slot_ok(a, slot) || nrt <= 0) {
          mbar_arrive_expect_tx(&full[s], 0);
          return true;
        }
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(stg + (size_t)s * SB, a.pool + (int64_t)slot * sbytes + a.q_d + (int64_t)rt0 * a.tile_d, bytes,
                 &full[s]);
        return true;
      };
      const int n0 = n_act < NS ? n_act : NS;
      for (int i = lane; i < n0; i += 32) issue(i);
      if (lane == 0)
        for (int i = n0; ok && i < n_act; ++i) ok = issue(i);
    } else {
      const int gi = (int)blockIdx.x - a.fu_n_dn;
      const int n_items = n_act * jt_n;
      const int my_items = gi < n_items ? (n_items - gi + n_gu - 1) / n_gu : 0;
      const uint32_t bytes = (uint32_t)a.tile_gu;
      auto issue = [&](int q) -> bool {
        const int s = q % NS;
        if (q >= NS && !mbar_wait_bounded(&empty[s], (uint32_t)(((q / NS) - 1) & 1), a.wait_limit)) return false;
        const int item = gi + q * n_gu;
        const int slot = s_slot[item / jt_n];
        if (!slot_ok(a, slot)) {
          mbar_arrive_expect_tx(&full[s], 0);
          return true;
        }
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(stg + (size_t)s * SB, a.pool + (int64_t)slot * sbytes + a.q_gu + (int64_t)(item % jt_n) * bytes,
                 bytes, &full[s]);
        return true;
      };
      const int n0 = my_items < NS ? my_items : NS;
      for (int q = lane; q < n0; q += 32) issue(q);
      if (lane == 0)
        for (int q = n0; ok && q < my_items; ++q) ok = issue(q);
    }
    if (!ok && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
    return;
  }

  // ---------------- consumers ----------------
  for (int p = tid; p < np; p += kFuConsumers * 32) {
    s_ids[p] = a.ids[p];
    s_w[p] = a.w[p];
  }
  if (!dn_role) {  // x -> shared memory, in the producer's round (H a multiple of 32: whole 16-byte words)
    const int nx = a.T * a.H / 8;
    uint4* xd = reinterpret_cast<uint4*>(xh);
    for (int b0 = tid; b0 < nx; b0 += 4 * kFuConsumers * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (b0 + u * kFuConsumers * 32 < nx)
          v[u] = __ldg(reinterpret_cast<const uint4*>(a.x) + b0 + u * kFuConsumers * 32);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (b0 + u * kFuConsumers * 32 < nx) xd[b0 + u * kFuConsumers * 32] = v[u];
    }
  }
  tables_sync();  // the producer's pass tables
  const int n_act = s_nact;
  // (entry, token) -> flat pair from the routed ids (a token routes to an expert at most once)
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
  if (blockIdx.x == 0)
    for (int i = tid; i < n_act; i += kFuConsumers * 32)
      if (!slot_ok(a, s_slot[i])) flag_slot(a, s_slot[i]);
  consumers_sync(kFuConsumers * 32);
  pdl_launch_dependents();
  bool timed_out = false;

  if (!dn_role) {
    // ---------------- gate/up + SwiGLU -> h, item pairs ----------------
    const int gi = (int)blockIdx.x - a.fu_n_dn;
    const int n_items = n_act * jt_n;
    const int my_items = gi < n_items ? (n_items - gi + n_gu - 1) / n_gu : 0;
    uint32_t xbf[BPW][8][2];
    float xs[BPW][8 / GS][2], xo[BPW][8 / GS][2];
    {
      const uint16_t* xrow = g8 < a.T ? reinterpret_cast<const uint16_t*>(xh) + g8 * a.H : nullptr;
#pragma unroll
      for (int bi = 0; bi < BPW; ++bi) load_b_block<BG, GS>(xrow, warp * BPW + bi, a.H, t4, xbf[bi], xs[bi], xo[bi]);
    }
    const int GRP = 8 * (int)a.rb_gu;
    const int uoff = thread_unit_off<BG>(t4, g8);
    const bool all_blocks = (warp + 1) * BPW <= a.nblk_gu;
    auto item_mma = [&](const uint8_t* st, float (&acc)[4]) {
      const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
#pragma unroll
      for (int bi = 0; bi < BPW; ++bi)
        if (all_blocks || warp * BPW + bi < a.nblk_gu)
          block_mma<BG, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, warp * BPW + bi, uoff, xbf[bi], xs[bi], xo[bi],
                            acc);
    };
    const int nflush = a.T * 8;  // (token, column) pairs of one entry
    for (int q = 0; q < my_items; q += 2) {
      const bool two = q + 1 < my_items;
      const int it0 = gi + q * n_gu, it1 = it0 + n_gu;
      const int e0 = it0 / jt_n, e1 = two ? it1 / jt_n : 0;
      const bool ok0 = slot_ok(a, s_slot[e0]), ok1 = two && slot_ok(a, s_slot[e1]);
      const int s0 = q % NS, s1 = (q + 1) % NS;
      if (!timed_out && !mbar_wait_bounded(&full[s0], (uint32_t)((q / NS) & 1), a.wait_limit)) timed_out = true;
      if (two && !timed_out && !mbar_wait_bounded(&full[s1], (uint32_t)(((q + 1) / NS) & 1), a.wait_limit))
        timed_out = true;
      float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
      if (!timed_out) {
        if (ok0 && ok1) {  // the two items' load / unpack / MMA chains interleave
          const uint8_t* st0 = stg + (size_t)s0 * SB;
          const uint8_t* st1 = stg + (size_t)s1 * SB;
          const uint32_t* sb0 = reinterpret_cast<const uint32_t*>(st0 + 2 * GRP);
          const uint32_t* sb1 = reinterpret_cast<const uint32_t*>(st1 + 2 * GRP);
#pragma unroll
          for (int bi = 0; bi < BPW; ++bi)
            if (all_blocks || warp * BPW + bi < a.nblk_gu) {
              block_mma<BG, GS>(st0, st0 + GRP, sb0 + g8, sb0 + 8 + g8, warp * BPW + bi, uoff, xbf[bi], xs[bi],
                                xo[bi], acc0);
              block_mma<BG, GS>(st1, st1 + GRP, sb1 + g8, sb1 + 8 + g8, warp * BPW + bi, uoff, xbf[bi], xs[bi],
                                xo[bi], acc1);
            }
        } else {
          if (ok0) item_mma(stg + (size_t)s0 * SB, acc0);
          if (ok1) item_mma(stg + (size_t)s1 * SB, acc1);
        }
      }
      int nent = 0;
      if (ok0) {
        *reinterpret_cast<float4*>(&red[((size_t)warp * 32 + lane) * 4]) =
            make_float4(acc0[0], acc0[1], acc0[2], acc0[3]);
        if (tid == 0) rmeta[0] = RedMeta{e0, 0, a.T, it0 % jt_n};
        nent = 1;
      }
      if (ok1) {
        *reinterpret_cast<float4*>(&red[(((size_t)nent * kFuConsumers + warp) * 32 + lane) * 4]) =
            make_float4(acc1[0], acc1[1], acc1[2], acc1[3]);
        if (tid == 0) rmeta[nent] = RedMeta{e1, 0, a.T, it1 % jt_n};
        ++nent;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s0]);
        if (two) mbar_arrive(&empty[s1]);
      }
      if (nent == 0) continue;
      consumers_sync(kFuConsumers * 32);
      // eight consecutive lanes hold the eight columns of one (entry, token);
      // h is stored scaled by 2^-a of its down pair slot (exact: a power of
      // two), with the partial sums (sum h, sum 128 h 2^-a) of the eight
      for (int base = warp * 32; base < nent * nflush; base += kFuConsumers * 32) {
        const int idx = base + lane;
        const bool act = idx < nent * nflush;
        const int en = act ? idx / nflush : 0, n = act ? (idx % nflush) >> 3 : 0, j = idx & 7;
        const RedMeta m = rmeta[en];
        const int pos = act ? s_tok[m.ei * kDenseMaxTokens + n] : -1;  // -1 for absent tokens
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
      // publish: the items' h columns are written (CTA barrier, then a release add per item)
      if (tid == 0)
        for (int en = 0; en < nent; ++en) red_release_add(ready + rmeta[en].ei, 1u);
    }
  } else if (nrt > 0) {
    // ---------------- down + combine -> y, experts as they complete ----------------
    const int ngd = Ip / a.g;
    uint16_t* hs = reinterpret_cast<uint16_t*>(xh);
    float2* hsum = reinterpret_cast<float2*>(xh + (size_t)np * Ip * 2);
    const int GRP = 8 * (int)a.rb_d;
    const int uoff = thread_unit_off<BD>(t4, g8);
    const int kq = warp % kDnKSplit, grp = warp / kDnKSplit, ngrp = kFuConsumers / kDnKSplit;
    float yacc[kFuRtMax][4];
#pragma unroll
    for (int r = 0; r < kFuRtMax; ++r) yacc[r][0] = yacc[r][1] = yacc[r][2] = yacc[r][3] = 0.f;
    // entries still to take (all of the pass: an entry whose slot is not
    // valid is taken at once and skipped, so that its stage is released)
    unsigned long long pending = n_act >= 64 ? ~0ull : ((1ull << n_act) - 1ull);
    int low = 0;  // lowest entry not yet taken (the stages hold entries low .. low + NS - 1)
    const long long t0 = clock64();
    const int cpr = Ip / 8, cpg = a.g / 8, jt_i = a.I / 8;
    while (pending != 0ull) {
      // which entries of the window have every gate/up item published
      if (warp == 0) {
        unsigned long long m = 0ull;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int i = lane + 32 * q;
          bool r = false;
          if (i < n_act && i < low + NS && ((pending >> i) & 1ull))
            r = !slot_ok(a, s_slot[i]) || ld_acquire_u32(ready + i) == (unsigned)jt_n;
          m |= (unsigned long long)__ballot_sync(0xffffffffu, r) << (32 * q);
        }
        if (lane == 0) {
          s_ready = m;
          s_npl = 0;
          if (m == 0ull && clock64() - t0 > a.wait_limit) s_timeout = 1;
        }
      }
      consumers_sync(kFuConsumers * 32);
      const unsigned long long now = s_ready;
      if (s_timeout) {
        timed_out = true;
        break;
      }
      if (now == 0ull) {
        __nanosleep(64);
        continue;
      }
      // the flat pairs of the newly complete experts
      for (int i2 = tid; i2 < n_act * kDenseMaxTokens; i2 += kFuConsumers * 32) {
        const int e = i2 / kDenseMaxTokens;
        const int p = s_tok[i2];
        if (p >= 0 && ((now >> e) & 1ull) && slot_ok(a, s_slot[e])) s_plist[atomicAdd(&s_npl, 1)] = p;
      }
      consumers_sync(kFuConsumers * 32);
      const int npl = s_npl;
      // their h rows (already scaled by 2^-a; padding columns zeroed) and the
      // per-(pair, group) epilogue sums from the per-8-column partials, all
      // loads of a thread in flight together
      for (int b0 = tid; b0 < npl * cpr; b0 += 4 * kFuConsumers * 32) {
        uint4 v[4];
        int dst[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = b0 + u * kFuConsumers * 32;
          dst[u] = -1;
          v[u] = make_uint4(0u, 0u, 0u, 0u);
          if (idx < npl * cpr) {
            const int p = s_plist[idx / cpr], c = idx % cpr;
            dst[u] = p * cpr + c;
            if (8 * c < a.I) v[u] = __ldcg(reinterpret_cast<const uint4*>(a.h + (int64_t)p * Ip) + c);
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (dst[u] >= 0) reinterpret_cast<uint4*>(hs)[dst[u]] = v[u];
      }
      for (int task = tid; task < npl * ngd; task += kFuConsumers * 32) {
        const int p = s_plist[task / ngd], G = task % ngd;
        const float2* src = reinterpret_cast<const float2*>(a.hpart) + (int64_t)p * cpr + G * cpg;
        float2 v[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          v[c] = (c < cpg && G * cpg + c < jt_i) ? __ldcg(src + c) : make_float2(0.f, 0.f);
        float sx = 0.f, so = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          sx += v[c].x;
          so += v[c].y;
        }
        hsum[p * ngd + G] = make_float2(sx, so);
      }
      consumers_sync(kFuConsumers * 32);
      // warps w and w + kDnKSplit split K the same way; the groups take the
      // ready experts in turn, each over all of the CTA's row tiles
      int nth = 0;
      for (int i = low; i < n_act; ++i) {
        if (!((now >> i) & 1ull)) continue;
        const bool valid = slot_ok(a, s_slot[i]);
        const bool mine = valid && (nth % ngrp) == grp;
        nth += valid ? 1 : 0;
        const int s = i % NS;
        if (!timed_out && !mbar_wait_bounded(&full[s], (uint32_t)((i / NS) & 1), a.wait_limit)) timed_out = true;
        if (mine && !timed_out) {
          const uint8_t* st = stg + (size_t)s * SB;
          const int pb = s_tok[i * kDenseMaxTokens + g8];
          const int p0 = s_tok[i * kDenseMaxTokens + 2 * t4], p1 = s_tok[i * kDenseMaxTokens + 2 * t4 + 1];
          const float w0 = p0 >= 0 ? s_w[p0] : 0.f, w1 = p1 >= 0 ? s_w[p1] : 0.f;
          float acc[kFuRtMax][4];
#pragma unroll
          for (int r = 0; r < kFuRtMax; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
          for (int kb = kq; kb < a.nblk_d; kb += kDnKSplit) {
            uint32_t bf[8][2];
            float xs1[8 / GS][2], xo1[8 / GS][2];
            const uint16_t* row = pb < 0 ? nullptr : hs + (size_t)pb * Ip + kb * 128 + 2 * t4;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              bf[u][0] = row ? ld_pair(row + 16 * u) : 0u;
              bf[u][1] = row ? ld_pair(row + 16 * u + 8) : 0u;
            }
#pragma unroll
            for (int G = 0; G < 8 / GS; ++G) {
              const int gi2 = kb * (8 / GS) + G;
              const float2 v0 = p0 < 0 ? make_float2(0.f, 0.f) : hsum[p0 * ngd + gi2];
              const float2 v1 = p1 < 0 ? make_float2(0.f, 0.f) : hsum[p1 * ngd + gi2];
              xs1[G][0] = v0.x;
              xo1[G][0] = v0.y;
              xs1[G][1] = v1.x;
              xo1[G][1] = v1.y;
            }
#pragma unroll
            for (int r = 0; r < kFuRtMax; ++r)
              if (r < nrt) {
                const uint8_t* tile = st + (size_t)r * a.tile_d;
                const uint32_t* sbs = reinterpret_cast<const uint32_t*>(tile + 2 * GRP);
                block_mma<BD, GS>(tile, tile + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs1, xo1, acc[r]);
              }
          }
#pragma unroll
          for (int r = 0; r < kFuRtMax; ++r) {
            yacc[r][0] += w0 * acc[r][0];
            yacc[r][1] += w1 * acc[r][1];
            yacc[r][2] += w0 * acc[r][2];
            yacc[r][3] += w1 * acc[r][3];
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      pending &= ~now;
      while (low < n_act && !((pending >> low) & 1ull)) ++low;
      consumers_sync(kFuConsumers * 32);  // s_ready, s_plist and the h rows are read
    }
    // y rows of the CTA's tiles: the sum over the warps (fixed order)
#pragma unroll
    for (int r = 0; r < kFuRtMax; ++r)
      if (r < nrt)
        *reinterpret_cast<float4*>(&red[(((size_t)r * kFuConsumers + warp) * 32 + lane) * 4]) =
            make_float4(yacc[r][0], yacc[r][1], yacc[r][2], yacc[r][3]);
    consumers_sync(kFuConsumers * 32);
    for (int i = tid; i < nrt * a.T * 16; i += kFuConsumers * 32) {
      const int r = i / (a.T * 16), rem = i % (a.T * 16), tok = rem >> 4, row = rem & 15;
      const int src = 4 * (row & 7) + (tok >> 1), c = (row >> 3) * 2 + (tok & 1);
      const float* rp = red + (size_t)r * kFuConsumers * 32 * 4;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kFuConsumers; ++w) sum += rp[(w * 32 + src) * 4 + c];
      float* yp = a.y + (int64_t)tok * a.H + (rt0 + r) * 16 + row;
      *yp = a.y_overwrite ? sum : *yp + sum;
    }
  }
  if (dn_role) {
    // the last down CTA to leave zeroes the control block for the next launch
    consumers_sync(kFuConsumers * 32);
    if (tid == 0) {
      unsigned* depart = a.ctl + kCtlDepart;
      __threadfence();
      const unsigned old = atomicAdd(depart, 1u);
      if (old == (unsigned)a.fu_n_dn - 1u) {
        for (int i = 0; i < kMaxCtaExperts; ++i) ready[i] = 0u;
        *depart = 0u;
        __threadfence();
      }
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
  // co-residency of every CTA is required (the down CTAs wait for the gate/up
  // CTAs): always cooperative; early launch behind the previous kernel as
  // well where the driver accepts the combination (remembered after the
  // first refusal)
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

// Role split, stage counts and shared memory of the fused kernel for this
// call (into a); false when the fused path does not apply (the caller then
// uses the two-kernel path).
bool ffn_fused_plan(FfnArgs& a, const moe_layer_desc& d, int num_sms, size_t& smem) {
  if (!(a.T <= kDenseMaxTokens && a.T * d.k <= kMaxCtaExperts) || a.ctl == nullptr) return false;
  if (a.L.nblk_gu > 2 * kFuConsumers || d.E > 1024 || d.I % 8) return false;
  const int grid = num_sms;
  const int n_rt = d.H / 16, jt_n = d.I / 8;
  int max_pass = a.pass_len < d.E ? a.pass_len : d.E;
  if (a.T * d.k < max_pass) max_pass = a.T * d.k;
  if (max_pass < 1) max_pass = 1;
  // down CTAs in proportion to the down projection's share of the bytes
  const double gu_b = (double)jt_n * a.L.tile_gu, dn_b = (double)n_rt * a.L.tile_d;
  int want = (int)(grid * dn_b / (gu_b + dn_b) + 0.5);
  if (want < 1) want = 1;
  int rpd = (n_rt + want - 1) / want;
  if (rpd > kFuRtMax) return false;
  const int n_dn = (n_rt + rpd - 1) / rpd;
  if (n_dn >= grid) return false;
  const int n_gu = grid - n_dn;
  a.fu_n_dn = n_dn;
  a.fu_rt_per_dn = rpd;
  a.gu_stage_bytes = (int)round_up(a.L.tile_gu, 128);
  a.d_stage_bytes = (int)round_up((int64_t)rpd * a.L.tile_d, 128);
  {
    // x in the gate/up CTAs; h (scaled, rows padded to 128-blocks) and the
    // per-(pair, group) sums in the down CTAs
    const size_t np = (size_t)a.T * d.k, Ip = (size_t)a.L.nblk_d * 128;
    const size_t xb = (size_t)a.T * d.H * 2, hb = np * Ip * 2 + np * (Ip / d.group) * 8;
    a.xh_stage_bytes = (int)round_up((int64_t)(xb > hb ? xb : hb), 128);
  }
  const size_t fixed = (size_t)a.xh_stage_bytes + (size_t)kFuRedFloats * 4 + kRedBatch * sizeof(RedMeta) +
                       kFuTableBytes + (size_t)d.E * 4 + 16;
  const size_t cap = 220 * 1024;
  if (fixed + (size_t)2 * a.gu_stage_bytes + 32 > cap) return false;
  const size_t area = cap - fixed;
  const int64_t items_per_cta = ((int64_t)max_pass * jt_n + n_gu - 1) / n_gu;
  int nsg = (int)(area / (a.gu_stage_bytes + 16));
  if (nsg > items_per_cta) nsg = (int)items_per_cta;
  if (nsg < 2) nsg = 2;
  int nsd = (int)(area / (a.d_stage_bytes + 16));
  if (nsd > max_pass) nsd = max_pass;
  if (nsd < 1) return false;
  a.gu_nstage = nsg;
  a.d_nstage = nsd;
  const size_t sg = (size_t)nsg * a.gu_stage_bytes, sd = (size_t)nsd * a.d_stage_bytes;
  a.fu_stage_area = (int)round_up((int64_t)(sg > sd ? sg : sd), 128);
  const int nbar = nsg > nsd ? nsg : nsd;
  smem = (size_t)a.fu_stage_area + fixed + 16 * (size_t)nbar;
  return smem <= cap + 16 * (size_t)nbar;
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
