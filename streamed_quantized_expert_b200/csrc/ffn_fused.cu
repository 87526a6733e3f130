// Decode FFN in one launch (T <= 8 tokens, every routed pair in the per-CTA
// tables): gate/up + SwiGLU -> h, then down + weighted combine -> y.
//
// One CTA per SM, all co-resident (cooperative launch); a producer warp and
// 16 consumer warps per CTA.  Every CTA first takes a contiguous range of the
// pass's gate/up items (a 16-row tile: 8 gate + 8 up rows of one expert;
// items run expert-major), then -- if it owns one -- a 16-row tile of the
// down projection for every active expert.  The ranges are weighted so that
// each SM streams about the same number of bytes (CTAs without a down tile
// take more gate/up items).  There is no grid-wide barrier: after every pair
// of items a CTA writes their h columns and adds the item count to each
// expert's readiness counter (release); a CTA's down work takes the experts
// in order as their counters report every item written (acquire), so the
// down work of the first experts overlaps the gate/up work of the last.
//
// Before the dependency wait (programmatic dependent launch) every CTA asks
// L2 for the pass's tables, x and the expert -> slot table, so that the
// metadata round after the wait hits L2.  The producer warp then reads the
// active experts and the whole slot table in one round of independent loads
// and its 32 lanes issue, in parallel, one bulk copy per gate/up item and one
// per expert for the down tile, so the down weights stream in while gate/up
// computes.  The consumer warps form four groups of four; group g takes the
// CTA's items g, g + 4, ... and splits K over its warps, so four items are in
// flight at once and every barrier of the gate/up phase is group-local.  A
// group reduces its four warps' partial sums with shuffles, writes the item's
// h columns, and hands the item to the producer warp, which makes the writes
// visible (release) and adds to the expert's readiness counter, so no
// consumer waits on that fence.
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
constexpr int kFuDnGroups = kFuConsumers / kDnKSplit;  // warp groups taking down experts in turn
constexpr int kGuGroups = 4;                            // gate/up warp groups (one item each at a time)
constexpr int kGuGroupWarps = kFuConsumers / kGuGroups;
constexpr int kGuPubRing = 32;                          // items a group can hand over before they are published
constexpr int kFuRedFloats = kFuConsumers * 32 * 4;     // one item per group: [warp][lane][4]
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
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Named barrier 2 over all threads of the CTA: the producer warp arrives once
// the pass tables are in shared memory, the consumer warps wait on it.
__device__ __forceinline__ void tables_arrive() { asm volatile("bar.arrive 2, %0;" ::"n"(kFuThreads) : "memory"); }
__device__ __forceinline__ void tables_sync() { asm volatile("bar.sync 2, %0;" ::"n"(kFuThreads) : "memory"); }
// Named barriers 3 .. 6: one per gate/up warp group.
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, %1;" ::"r"(3 + g), "n"(kGuGroupWarps * 32) : "memory");
}
__device__ __forceinline__ int ld_volatile_shared(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

// First gate/up item of CTA c (c = grid: the item count): every CTA's quota
// is the pass's bytes / grid, less the bytes of its down tile for the CTAs
// that own one, in gate/up items (closed form of the prefix sum).
__device__ __forceinline__ int fu_item_bound(int c, int n_items, int n_act, const FfnArgs& a) {
  const int64_t G = gridDim.x, nd = a.H / 16;
  const int64_t dn = (int64_t)n_act * a.tile_d;                // bytes of one down tile over the pass
  const int64_t tot = (int64_t)n_items * a.tile_gu + nd * dn;  // bytes of the pass
  int64_t f = (int64_t)c * tot - (c < nd ? c : nd) * G * dn;   // prefix * G, in bytes
  if (f < 0) f = 0;
  const int64_t v = f / (G * a.tile_gu);
  return v > n_items ? n_items : (int)v;
}

template <int BG, int BD, int BPW, int GS>
__global__ void __launch_bounds__(kFuThreads, 1) ffn_fused_kernel(const FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const int NSG = a.gu_nstage, SBG = a.gu_stage_bytes, NSD = a.d_nstage, SBD = a.d_stage_bytes;
  uint8_t* gst = smem;                                            // gate/up stages
  uint8_t* dst_ = gst + (size_t)NSG * SBG;                        // down stages
  uint8_t* xh = dst_ + (size_t)NSD * SBD;                         // x [T][H], then h rows + sums
  float* red = reinterpret_cast<float*>(xh + a.xh_stage_bytes);   // partial sums [warps][32][4]
  int* s_act = reinterpret_cast<int*>(red + kFuRedFloats);        // pass entry -> expert id
  int* s_slot = s_act + kMaxCtaExperts;                           // pass entry -> slot
  int* s_ids = s_slot + kMaxCtaExperts;                           // flat pair -> expert id
  float* s_w = reinterpret_cast<float*>(s_ids + kMaxCtaExperts);  // flat pair -> routing weight
  int* s_tok = reinterpret_cast<int*>(s_w + kMaxCtaExperts);      // [entry][token] -> flat pair or -1
  uint64_t* gfull = reinterpret_cast<uint64_t*>(s_tok + kMaxCtaExperts * kDenseMaxTokens);
  uint64_t* gempty = gfull + NSG;
  uint64_t* dfull = gempty + NSG;
  uint64_t* dempty = dfull + NSD;
  int* s_table = reinterpret_cast<int*>(dempty + NSD);  // expert -> slot, [E]
  __shared__ int s_nact, s_i0, s_i1;
  __shared__ unsigned long long s_ready;
  __shared__ int s_timeout, s_npl;
  __shared__ int s_plist[kMaxCtaExperts];
  __shared__ int s_pub_e[kGuGroups][kGuPubRing];  // per group: entries of its written items, in order
  __shared__ int s_pub_cnt[kGuGroups];             // items a group has handed over
  unsigned* ready = a.ctl + kCtlReady;
  const int np = a.T * a.k;  // <= kMaxCtaExperts (dense mode)

  // ask L2 for what the metadata round reads; nothing is read into the SM
  // before the dependency wait (the previous kernel may still write it)
  if (warp == kFuConsumers) {
    for (int e = 32 * lane; e < a.E; e += 32 * 32) prefetch_l2(a.table + e);
    if (lane == 0) prefetch_l2(a.n_active);
    if (lane < 2) prefetch_l2(a.active + a.pass_begin + 32 * lane);
    if (lane == 2) prefetch_l2(a.ids);
    if (lane == 3) prefetch_l2(a.w);
  } else {
    const int nx = a.T * a.H * 2;  // bytes of x
    for (int b = 128 * tid; b < nx; b += 128 * kFuConsumers * 32)
      prefetch_l2(reinterpret_cast<const uint8_t*>(a.x) + b);
  }
  if (tid == 0) {
    for (int s = 0; s < NSG; ++s) {
      mbar_init(&gfull[s], 1);
      mbar_init(&gempty[s], kGuGroupWarps);
    }
    for (int s = 0; s < NSD; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dempty[s], kFuConsumers);
    }
    fence_barrier_init();
    s_timeout = 0;
    for (int g = 0; g < kGuGroups; ++g) s_pub_cnt[g] = 0;
  }
  __syncthreads();
  pdl_wait();
  int cap = a.E - a.pass_begin;
  if (cap > a.pass_len) cap = a.pass_len;
  if (cap > kMaxCtaExperts) cap = kMaxCtaExperts;
  if (cap < 0) cap = 0;
  const int jt_n = a.I / 8;
  const int n_rt = a.H / 16;
  const int rt = blockIdx.x;  // the CTA's down tile, if rt < n_rt
  const bool has_rt = rt < n_rt;
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
    const int n_items = n_act * jt_n;
    const int i0 = fu_item_bound(blockIdx.x, n_items, n_act, a);
    const int i1 = fu_item_bound(blockIdx.x + 1, n_items, n_act, a);
    if (lane == 0) {
      s_nact = n_act;
      s_i0 = i0;
      s_i1 = i1;
    }
    __syncwarp();
    tables_arrive();
    const int my_items = i1 - i0, n_dn = has_rt ? n_act : 0;
    const uint32_t tbg = (uint32_t)a.tile_gu, tbd = (uint32_t)a.tile_d;
    auto issue_gu = [&](int r) -> bool {
      const int s = r % NSG;
      if (r >= NSG && !mbar_wait_bounded(&gempty[s], (uint32_t)(((r / NSG) - 1) & 1), a.wait_limit)) return false;
      const int item = i0 + r;
      const int slot = s_slot[item / jt_n];
      if (!slot_ok(a, slot)) {
        mbar_arrive_expect_tx(&gfull[s], 0);
        return true;
      }
      mbar_arrive_expect_tx(&gfull[s], tbg);
      bulk_g2s(gst + (size_t)s * SBG, a.pool + (int64_t)slot * a.slot_bytes + a.q_gu + (int64_t)(item % jt_n) * tbg,
               tbg, &gfull[s]);
      return true;
    };
    auto issue_dn = [&](int i) -> bool {
      const int s = i % NSD;
      if (i >= NSD && !mbar_wait_bounded(&dempty[s], (uint32_t)(((i / NSD) - 1) & 1), a.wait_limit)) return false;
      const int slot = s_slot[i];
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
    for (int i = lane; i < nd0; i += 32) issue_dn(i);
    bool ok = true;
    if (lane == 0) {
      for (int r = ng0; ok && r < my_items; ++r) ok = issue_gu(r);
      for (int i = nd0; ok && i < n_dn; ++i) ok = issue_dn(i);
    }
    // publish service: lane 1 + g makes gate/up group g's h writes visible
    // (fence) and adds each written item to its expert's readiness counter
    // (lane 0 may still be refilling stages, which waits on the consumers)
    if (lane >= 1 && lane <= kGuGroups) {
      const int g = lane - 1;
      const int n_g = my_items > g ? (my_items - g + kGuGroups - 1) / kGuGroups : 0;
      int done = 0;
      const long long t0 = clock64();
      while (ok && done < n_g) {
        const int c = ld_volatile_shared(&s_pub_cnt[g]);
        if (c == done) {
          if (clock64() - t0 > a.wait_limit) ok = false;
          continue;
        }
        __threadfence();
        for (; done < c; ++done) {
          const int e = s_pub_e[g][done % kGuPubRing];
          if (e >= 0) atomicAdd(ready + e, 1u);
        }
      }
    }
    if (!ok && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
    return;
  }

  // ---------------- consumers ----------------
  for (int p = tid; p < np; p += kFuConsumers * 32) {
    s_ids[p] = a.ids[p];
    s_w[p] = a.w[p];
  }
  {
    // x' = x 2^-a (exact: a power of two; a by input position within its
    // 128-block) -> shared memory, with the per-(group, token) sums
    // sum x and 128 sum x' that the group epilogues apply
    const int nx = a.T * a.H / 8;  // 16-byte words of x (H a multiple of 32)
    const int wpg = a.g / 8;       // words per group: consecutive lanes, aligned
    uint4* xd = reinterpret_cast<uint4*>(xh);
    float* xsum = reinterpret_cast<float*>(xh + (size_t)a.T * a.H * 2);
    for (int base = warp * 32; base < nx; base += kFuConsumers * 32) {
      const int idx = base + lane;
      const bool act = idx < nx;
      uint4 v = act ? __ldg(reinterpret_cast<const uint4*>(a.x) + idx) : make_uint4(0u, 0u, 0u, 0u);
      const int t = idx / (a.H / 8), k = (idx % (a.H / 8)) * 8, kk = k & 127;
      const bool eighth = PairShift<BG>::a(2 * (kk >> 4) + ((kk & 15) >> 3)) == 3;
      uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float sx = 0.f, so = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        sx += bf16_lo(w4[u]) + bf16_hi(w4[u]);
        if (eighth) w4[u] = bf2_scale_eighth(w4[u]);
        so += bf16_lo(w4[u]) + bf16_hi(w4[u]);
      }
      for (int o = 1; o < wpg; o <<= 1) {
        sx += __shfl_xor_sync(0xffffffffu, sx, o);
        so += __shfl_xor_sync(0xffffffffu, so, o);
      }
      if (act) {
        xd[idx] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        if ((idx % wpg) == 0) {
          const int G = k / a.g;
          xsum[(G * a.T + t) * 2] = sx;
          xsum[(G * a.T + t) * 2 + 1] = 128.0f * so;
        }
      }
    }
  }
  tables_sync();  // the producer's pass tables
  const int n_act = s_nact, i0 = s_i0, i1 = s_i1;
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
  consumers_sync(kFuConsumers * 32);  // x in shared memory, pair map written
  bool timed_out = false;

  // ---------------- gate/up + SwiGLU -> h, one item per warp group ----------------
  {
    const int gg = warp / kGuGroupWarps, wg = warp % kGuGroupWarps;  // group, warp within the group
    const uint16_t* xrow = g8 < a.T ? reinterpret_cast<const uint16_t*>(xh) + g8 * a.H : nullptr;
    const float* xsum = reinterpret_cast<const float*>(xh + (size_t)a.T * a.H * 2);
    const int GRP = 8 * (int)a.rb_gu;
    const int uoff = thread_unit_off<BG>(t4, g8);
    const int n0 = 2 * t4 < a.T ? 2 * t4 : 0, n1 = 2 * t4 + 1 < a.T ? 2 * t4 + 1 : 0;  // C fragment columns
    const int my_items = i1 - i0;
    int handed = 0;
    for (int q = gg; q < my_items; q += kGuGroups) {
      const int it = i0 + q, e = it / jt_n, jt = it % jt_n;
      const int s = q % NSG;
      const bool ok = slot_ok(a, s_slot[e]);
      if (!timed_out && !mbar_wait_bounded(&gfull[s], (uint32_t)((q / NSG) & 1), a.wait_limit)) timed_out = true;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (!timed_out) {
        const uint8_t* st = gst + (size_t)s * SBG;
        const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
        for (int kb = wg; kb < a.nblk_gu; kb += kGuGroupWarps) {
          uint32_t bf[8][2];
          float xs[8 / GS][2], xo[8 / GS][2];
          const uint16_t* row = xrow ? xrow + kb * 128 + 2 * t4 : nullptr;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            bf[u][0] = row ? ld_pair(row + 16 * u) : 0u;
            bf[u][1] = row ? ld_pair(row + 16 * u + 8) : 0u;
          }
#pragma unroll
          for (int G = 0; G < 8 / GS; ++G) {
            const int gi = kb * (8 / GS) + G;
            xs[G][0] = xsum[(gi * a.T + n0) * 2];
            xo[G][0] = xsum[(gi * a.T + n0) * 2 + 1];
            xs[G][1] = xsum[(gi * a.T + n1) * 2];
            xo[G][1] = xsum[(gi * a.T + n1) * 2 + 1];
          }
          block_mma<BG, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs, xo, acc);
        }
      }
      *reinterpret_cast<float4*>(&red[((size_t)warp * 32 + lane) * 4]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&gempty[s]);
      group_sync(gg);
      // warp wg takes tokens wg, wg + 4, ...: lane 4 j + w holds column j's
      // gate/up partial of the group's warp w; shuffles sum the four warps,
      // then (sum h, sum 128 h 2^-a) over the eight columns
      for (int n = wg; n < a.T; n += kGuGroupWarps) {
        const int j = lane >> 2, w = lane & 3;
        const float* rp = red + ((size_t)(gg * kGuGroupWarps + w) * 32 + 4 * j + (n >> 1)) * 4;
        float gate = rp[n & 1], up = rp[2 + (n & 1)];
        gate += __shfl_xor_sync(0xffffffffu, gate, 1);
        up += __shfl_xor_sync(0xffffffffu, up, 1);
        gate += __shfl_xor_sync(0xffffffffu, gate, 2);
        up += __shfl_xor_sync(0xffffffffu, up, 2);
        const float hv = gate / (1.0f + expf(-gate)) * up;
        const int kcol = jt * 8 + j, kk = kcol & 127;
        const bool eighth = PairShift<BD>::a(2 * (kk >> 4) + ((kk & 15) >> 3)) == 3;
        const uint16_t hb = f32_to_bf16_rne(eighth ? hv * 0.125f : hv);
        const float hsv = __uint_as_float((uint32_t)hb << 16);
        float sx = eighth ? 8.0f * hsv : hsv, so = 128.0f * hsv;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          sx += __shfl_xor_sync(0xffffffffu, sx, o);
          so += __shfl_xor_sync(0xffffffffu, so, o);
        }
        const int pos = s_tok[e * kDenseMaxTokens + n];  // -1: the token does not route here
        if (ok && !timed_out && pos >= 0) {
          if (w == 0) a.h[(int64_t)pos * Ip + kcol] = hb;
          if (lane == 0) *reinterpret_cast<float2*>(a.hpart + 2 * ((int64_t)pos * (Ip / 8) + jt)) = make_float2(sx, so);
        }
      }
      group_sync(gg);  // the item's h columns are written; red is free again
      if (wg == 0 && lane == 0) {  // hand the item to the producer warp's publish service
        s_pub_e[gg][handed % kGuPubRing] = ok && !timed_out ? e : -1;
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&s_pub_cnt[gg]) = handed + 1;
      }
      ++handed;
    }
  }
  consumers_sync(kFuConsumers * 32);  // every group is done with x' and red

  // ---------------- down + combine -> y, experts in order as they complete ----------------
  if (has_rt) {
    const int ngd = Ip / a.g;
    uint16_t* hs = reinterpret_cast<uint16_t*>(xh);
    float2* hsum = reinterpret_cast<float2*>(xh + (size_t)np * Ip * 2);
    const int GRP = 8 * (int)a.rb_d;
    const int uoff = thread_unit_off<BD>(t4, g8);
    const int kq = warp % kDnKSplit, grp = warp / kDnKSplit;
    float yacc[4] = {0.f, 0.f, 0.f, 0.f};
    unsigned long long pending = n_act >= 64 ? ~0ull : ((1ull << n_act) - 1ull);
    int low = 0;  // lowest entry not yet taken (the stages hold entries low .. low + NSD - 1)
    const long long t0 = clock64();
    const int cpr = Ip / 8, cpg = a.g / 8, jt_i = a.I / 8;
    while (pending != 0ull) {
      // the run of entries from the lowest pending one whose every gate/up
      // item is published (an entry whose slot is not valid counts as done);
      // taking entries in order keeps each warp's sum order fixed
      if (warp == 0) {
        unsigned long long m = 0ull;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int i = lane + 32 * q;
          bool r = false;
          if (i < n_act && i < low + NSD && ((pending >> i) & 1ull))
            r = !slot_ok(a, s_slot[i]) || ld_acquire_u32(ready + i) == (unsigned)jt_n;
          m |= (unsigned long long)__ballot_sync(0xffffffffu, r) << (32 * q);
        }
        const unsigned long long run = ~(m >> low);
        const int len = run == 0ull ? 64 - low : __ffsll((long long)run) - 1;
        const unsigned long long take = len >= 64 ? ~0ull : (((1ull << len) - 1ull) << low);
        if (lane == 0) {
          s_ready = take;
          s_npl = 0;
          if (take == 0ull && clock64() - t0 > a.wait_limit) s_timeout = 1;
        }
      }
      consumers_sync(kFuConsumers * 32);
      const unsigned long long now = s_ready;
      if (s_timeout) {
        timed_out = true;
        break;
      }
      if (now == 0ull) {
        __nanosleep(32);
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
      for (int b0 = tid; b0 < npl * cpr; b0 += 2 * kFuConsumers * 32) {
        uint4 v[2];
        int dsti[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = b0 + u * kFuConsumers * 32;
          dsti[u] = -1;
          v[u] = make_uint4(0u, 0u, 0u, 0u);
          if (idx < npl * cpr) {
            const int p = s_plist[idx / cpr], c = idx % cpr;
            dsti[u] = p * cpr + c;
            if (8 * c < a.I) v[u] = __ldcg(reinterpret_cast<const uint4*>(a.h + (int64_t)p * Ip) + c);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (dsti[u] >= 0) reinterpret_cast<uint4*>(hs)[dsti[u]] = v[u];
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
      // warps w, w + kDnKSplit, ... split K the same way; entry i belongs to
      // warp group i % kFuDnGroups
      for (int i = low; i < n_act; ++i) {
        if (!((now >> i) & 1ull)) continue;
        const int s = i % NSD;
        if (!timed_out && !mbar_wait_bounded(&dfull[s], (uint32_t)((i / NSD) & 1), a.wait_limit)) timed_out = true;
        if (!timed_out && slot_ok(a, s_slot[i]) && (i % kFuDnGroups) == grp) {
          const uint8_t* st = dst_ + (size_t)s * SBD;
          const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
          const int pb = s_tok[i * kDenseMaxTokens + g8];
          const int p0 = s_tok[i * kDenseMaxTokens + 2 * t4], p1 = s_tok[i * kDenseMaxTokens + 2 * t4 + 1];
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
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
            block_mma<BD, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs1, xo1, acc);
          }
          const float w0 = p0 >= 0 ? s_w[p0] : 0.f, w1 = p1 >= 0 ? s_w[p1] : 0.f;
          yacc[0] += w0 * acc[0];
          yacc[1] += w1 * acc[1];
          yacc[2] += w0 * acc[2];
          yacc[3] += w1 * acc[3];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&dempty[s]);
      }
      pending &= ~now;
      while (low < n_act && !((pending >> low) & 1ull)) ++low;
      consumers_sync(kFuConsumers * 32);  // s_ready, s_plist and the h rows are read
    }
    // y rows of the CTA's tile: the sum over the warps (fixed order)
    *reinterpret_cast<float4*>(&red[((size_t)warp * 32 + lane) * 4]) = make_float4(yacc[0], yacc[1], yacc[2], yacc[3]);
    consumers_sync(kFuConsumers * 32);
    for (int i = tid; i < a.T * 16; i += kFuConsumers * 32) {
      const int tok = i >> 4, row = i & 15;
      const int src = 4 * (row & 7) + (tok >> 1), c = (row >> 3) * 2 + (tok & 1);
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kFuConsumers; ++w) sum += red[(w * 32 + src) * 4 + c];
      float* yp = a.y + (int64_t)tok * a.H + rt * 16 + row;
      *yp = a.y_overwrite ? sum : *yp + sum;
    }
    // the last CTA with a down tile to leave zeroes the control block for the next launch
    consumers_sync(kFuConsumers * 32);
    if (tid == 0) {
      unsigned* depart = a.ctl + kCtlDepart;
      __threadfence();
      const unsigned old = atomicAdd(depart, 1u);
      if (old == (unsigned)n_rt - 1u) {
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
  // co-residency of every CTA is required (down work waits for other CTAs'
  // gate/up items): always cooperative; early launch behind the previous
  // kernel as well where the driver accepts the combination (remembered after
  // the first refusal)
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

// Stage sizes and counts of the fused kernel for this call (into a), its
// shared memory; false when the fused path does not apply (the caller then
// uses the two-kernel path).
bool ffn_fused_plan(FfnArgs& a, const moe_layer_desc& d, int num_sms, size_t& smem) {
  if (!(a.T <= kDenseMaxTokens && a.T * d.k <= kMaxCtaExperts) || a.ctl == nullptr) return false;
  if (a.L.nblk_gu > 2 * kFuConsumers || d.E > 1024 || d.I % 8) return false;
  if (d.H / 16 > num_sms) return false;
  const int grid = num_sms;
  int max_pass = a.pass_len < d.E ? a.pass_len : d.E;
  if (a.T * d.k < max_pass) max_pass = a.T * d.k;
  if (max_pass < 1) max_pass = 1;
  a.gu_stage_bytes = (int)round_up(a.L.tile_gu, 128);
  a.d_stage_bytes = (int)round_up(a.L.tile_d, 128);
  {
    // x' and its per-(group, token) sums in the gate/up phase; h (scaled,
    // rows padded to 128-blocks) and the per-(pair, group) sums in the down phase
    const size_t np = (size_t)a.T * d.k, Ip = (size_t)a.L.nblk_d * 128;
    const size_t xb = (size_t)a.T * d.H * 2 + (size_t)(d.H / d.group) * a.T * 8;
    const size_t hb = np * Ip * 2 + np * (Ip / d.group) * 8;
    a.xh_stage_bytes = (int)round_up((int64_t)(xb > hb ? xb : hb), 128);
  }
  // the most gate/up items a CTA can get: a CTA without a down tile takes the
  // whole quota of (gate/up + down bytes) / grid
  const int n_rt = d.H / 16, jt_n = d.I / 8;
  const double tot = (double)max_pass * jt_n * a.L.tile_gu + (double)n_rt * max_pass * a.L.tile_d;
  const int64_t items_max = (int64_t)(tot / grid / a.L.tile_gu) + 2;
  if ((items_max + kGuGroups - 1) / kGuGroups > kGuPubRing) return false;
  const size_t fixed = (size_t)a.xh_stage_bytes + (size_t)kFuRedFloats * 4 + kFuTableBytes + (size_t)d.E * 4 + 16;
  const size_t cap = 220 * 1024;
  constexpr int kMinDn = kFuDnGroups;
  if (fixed + 2 * (size_t)a.gu_stage_bytes + kMinDn * (size_t)a.d_stage_bytes + 64 > cap) return false;
  // down stages: every expert of the pass if possible; gate/up stages: every
  // item of the CTA if possible, at least two (a pair is computed at once)
  int nsd = max_pass > kMinDn ? max_pass : kMinDn;
  int nsg = (int)(items_max < 2 ? 2 : items_max);
  while ((size_t)nsd * a.d_stage_bytes + (size_t)nsg * a.gu_stage_bytes + fixed + 16 * (nsd + nsg) > cap) {
    if (nsg > nsd && nsg > 2) --nsg;
    else if (nsd > kMinDn) --nsd;
    else if (nsg > 2) --nsg;
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
