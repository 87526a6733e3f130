// Decode FFN in one launch (T <= 8 tokens, every routed pair in the per-CTA
// tables): gate/up + SwiGLU -> h, then down + weighted combine -> y.
//
// One CTA per SM, all co-resident (cooperative launch); a producer warp and
// 16 consumer warps per CTA.  Every CTA first takes a contiguous range of the
// pass's gate/up items (a 16-row tile: 8 gate + 8 up rows of one expert;
// items run expert-major), then -- if it owns one -- a 16-row tile of the
// down projection for every active expert.  The ranges are weighted so that
// each SM streams about the same number of bytes (CTAs without a down tile
// take more gate/up items).
//
// Before the dependency wait (programmatic dependent launch) every CTA asks
// L2 for the pass's tables, x and the expert -> slot table, so that the
// metadata round after the wait hits L2.  The producer warp then reads the
// active experts and the whole slot table in one round of independent loads
// and its 32 lanes issue, in parallel, one bulk copy per gate/up item and one
// per expert for the down tile, so the down weights stream in while gate/up
// computes.
// The CTA's arrival on the launch's control word is taken by a consumer
// lane, off the producer's path to its first copy.
//
// Gate/up: warp pair m takes the CTA's items m, m + 8, ...; each warp of the
// pair runs half of K, one adds the other's partial sums (a pair barrier), so
// an item's gate and up sums end in registers, SwiGLU runs there, and the
// warp writes the item's h columns.  Each h value is one 64-bit word: the
// bf16 value and a 32-bit tag of this launch, so h needs no fence and no
// flag -- the down side reads the words until every tag it needs is this
// launch's.
//
// Down: tasks (pass entry i, 128-input block kb) go round-robin over the 16
// warps; a task reads its entry's h slice (spinning on the tags, bounded),
// stages it in the warp's shared scratch with its per-group sums, and runs
// the CTA's 16-row tile over that block.  The warps' partial sums of y meet
// once, in a fixed order, at the end (deterministic).
// With one token and every entry's down tile resident at once, a warp's
// tasks (at most three) read their h blocks together -- one round of global
// reads instead of one per task -- then compute back to back.
//
// Stage rings (when a CTA's items or entries outnumber its stages): several
// warps consume the uses of one stage, so a consumer could reach use u of a
// stage while use u - 2 is still being read elsewhere -- where a barrier's
// phase parity cannot tell use u from use u - 2.  So the producer also
// records in shared memory, per stage, how many uses it has issued; a
// consumer first waits until use u is issued (then the barrier is in use u's
// phase: use u + 1 needs this consumer's own release) and only then for the
// phase.  A wait that runs out marks the CTA aborted: the producer issues
// no further copy, the consumers skip every later wait, and the producer
// waits (with a long limit of its own) for every copy it did issue before
// it leaves.
//
// Launch tag: the control block (head of the workspace) holds one 64-bit
// word, the launch epoch (high half) and the arrivals of the running launch
// (low half).  Every CTA adds one arrival once its dependency wait is over
// (so the previous launch has completed); the CTA that completes the count
// turns it into the next epoch with zero arrivals.  All CTAs of a launch thus
// see the same epoch, and the tag is a bijective 32-bit mix (MurmurHash3's
// finaliser) of the epoch plus one: never 0, so a zeroed workspace holds no
// valid word, and unlike a small integer no plausible leftover of other
// scratch (small counts, bf16 pairs) matches it.  The count is complete after every launch, a timed
// out one included.  A control block that was not (an arrival count at or
// past the grid: every CTA reports MOE_DEV_ERR_TIMEOUT and skips its work; a
// count below it: the CTAs split over two tags and the down side's reads run
// out) stays so until the whole workspace is zeroed.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ffn_common.cuh"
#include "route_block.cuh"
#include "kernels.h"

namespace moe {

constexpr int kFuThreads = (kFuConsumers + 1) * 32;
constexpr int kFuPairs = kFuConsumers / 2;              // gate/up warp pairs
constexpr int kFuRedFloats = kFuConsumers * 32 * 4;     // [warp][lane][4]: pair partials, then y partials
constexpr int kFuScratchRowWords = 64 + 4;              // one token's 128-column h block, fragment order, padded
constexpr int kFuScratchPerTok = kFuScratchRowWords * 4 + 8 * 8;  // bytes per warp and row: h block + group sums
constexpr int kFuFastTasks = 3;  // one-token down: tasks per warp read together
static_assert(8 <= (int)kWsControlBytes, "control block size");
constexpr unsigned long long kEpochOne = 1ull << 32;
// per-pass tables in shared memory: active ids, slots, routed ids, routed
// weights (kMaxCtaExperts each) and the (entry, token) -> flat pair map
constexpr size_t kFuTableBytes =
    (size_t)kMaxCtaExperts * (3 * sizeof(int) + sizeof(float)) + (size_t)kMaxCtaExperts * kDenseMaxTokens * sizeof(int);

__device__ __forceinline__ unsigned fmix32(unsigned h) {
  h ^= h >> 16;
  h *= 0x85ebca6bu;
  h ^= h >> 13;
  h *= 0xc2b2ae35u;
  h ^= h >> 16;
  return h;
}
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
__device__ __forceinline__ void st_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Two tagged h words; each 64-bit element is read as one access, so a word's
// value and tag always come from the same store.
__device__ __forceinline__ void ld_volatile_2w(const uint64_t* p, uint64_t& w0, uint64_t& w1) {
  asm volatile("ld.volatile.global.v2.u64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p) : "memory");
}

// MMA fragment order of a bf16 row vector in shared memory: the pair
// (k, k + 1), k even, of 128-input block kb is 32-bit word
// ((kb * 4 + t4) * 8 + s) * 2 + half, s = k's 16-input step in the block,
// half = which 8 of the step, t4 = the pair within those 8.  So the 16 words
// lane t4 takes as B fragments for a block are contiguous (four 16-byte
// loads instead of sixteen 4-byte ones: the shared-memory instruction queue,
// not the tensor pipe, bounds this loop).  Rows are Kp + 8 elements apart, so
// consecutive rows start on different banks.
__device__ __forceinline__ int frag_word(int k) {
  const int kb = k >> 7, kk = k & 127;
  return ((kb * 4 + ((kk >> 1) & 3)) * 8 + (kk >> 4)) * 2 + ((kk >> 3) & 1);
}
__host__ __device__ constexpr int frag_rows_bytes(int rows, int Kp) { return rows * (Kp + 8) * 2; }
__device__ __forceinline__ void load_frag(const uint4* row, int kb, int t4, uint32_t (&bf)[8][2]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 v = row ? row[(kb * 4 + t4) * 4 + j] : make_uint4(0u, 0u, 0u, 0u);
    bf[2 * j][0] = v.x;
    bf[2 * j][1] = v.y;
    bf[2 * j + 1][0] = v.z;
    bf[2 * j + 1][1] = v.w;
  }
}

// Named barrier 2 over all threads of the CTA: the producer warp arrives once
// the pass tables are in shared memory, the consumer warps wait on it.
__device__ __forceinline__ void tables_arrive() { asm volatile("bar.arrive 2, %0;" ::"n"(kFuThreads) : "memory"); }
__device__ __forceinline__ void tables_sync() { asm volatile("bar.sync 2, %0;" ::"n"(kFuThreads) : "memory"); }
// Route mode: named barrier 12 is the routing threads' own (warps 0-7, the
// block routing function's barrier); on named barrier 11 they arrive once the
// token's ids and weights are in shared memory and the producer waits.
constexpr int kRouteWarps = 8;
__device__ __forceinline__ void routed_arrive() {
  asm volatile("bar.arrive 11, %0;" ::"n"(32 * (kRouteWarps + 1)) : "memory");
}
__device__ __forceinline__ void routed_sync() {
  asm volatile("bar.sync 11, %0;" ::"n"(32 * (kRouteWarps + 1)) : "memory");
}
// Named barriers 3 .. 10: one per gate/up warp pair.
__device__ __forceinline__ void pair_sync(int m) { asm volatile("bar.sync %0, 64;" ::"r"(3 + m) : "memory"); }

// First gate/up item of CTA c (c = grid: the item count), CTAs c < H / 16
// owning a down tile.  Every CTA's quota is the pass's bytes / grid, less the
// bytes of its down tile for the CTAs that own one (closed form of the prefix
// sum, in gate/up items); where one down tile alone is more than the quota,
// the down CTAs take no item and the others share the items evenly.
__device__ __forceinline__ int fu_item_bound(int c, int n_items, int n_act, const FfnArgs& a) {
  const int64_t G = gridDim.x, nd = a.H / 16;
  const int64_t dn = (int64_t)n_act * a.tile_d;                // bytes of one down tile over the pass
  const int64_t tot = (int64_t)n_items * a.tile_gu + nd * dn;  // bytes of the pass
  int64_t v;
  if (dn * G <= tot) {
    int64_t f = (int64_t)c * tot - (c < nd ? c : nd) * G * dn;  // prefix * G, in bytes
    if (f < 0) f = 0;
    v = f / (G * a.tile_gu);
  } else {
    v = c > nd ? (int64_t)(c - nd) * n_items / (G - nd) : 0;
  }
  return v > n_items ? n_items : (int)v;
}

// RT: route mode (moe_route_expert_ffn, one token): consumer warps 0-7 route
// it with the routing kernels' block function (same ids, order and weights),
// the producer forms the active list from the routed ids, and CTA 0 writes
// the routing, the sort and the lookup for the caller.
template <int BG, int BD, int BPW, int GS, bool RT>
__global__ void __launch_bounds__(kFuThreads, 1) ffn_fused_kernel(const FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, t4 = lane & 3, g8 = lane >> 2;
  const int NSG = a.gu_nstage, SBG = a.gu_stage_bytes, NSD = a.d_nstage, SBD = a.d_stage_bytes;
  uint8_t* gst = smem;                                            // gate/up stages
  uint8_t* dst_ = gst + (size_t)NSG * SBG;                        // down stages
  uint8_t* xh = dst_ + (size_t)NSD * SBD;                         // x' [T][H] + sums, then warp scratch
  float* red = reinterpret_cast<float*>(xh + a.xh_stage_bytes);   // [warp][lane][4]
  int* s_act = reinterpret_cast<int*>(red + kFuRedFloats);        // pass entry -> expert id
  int* s_slot = s_act + kMaxCtaExperts;                           // pass entry -> slot
  int* s_ids = s_slot + kMaxCtaExperts;                           // flat pair -> expert id
  float* s_w = reinterpret_cast<float*>(s_ids + kMaxCtaExperts);  // flat pair -> routing weight
  int* s_tok = reinterpret_cast<int*>(s_w + kMaxCtaExperts);      // [entry][token] -> flat pair or -1
  uint64_t* gfull = reinterpret_cast<uint64_t*>(s_tok + kMaxCtaExperts * kDenseMaxTokens);
  uint64_t* gempty = gfull + NSG;
  uint64_t* dfull = gempty + NSG;
  uint64_t* dempty = dfull + NSD;
  int* s_iss = reinterpret_cast<int*>(dempty + NSD);   // uses issued, per stage: gate/up [NSG], down [NSD]
  int* s_table = s_iss + NSG + NSD;                      // expert -> slot, [E]
  __shared__ int s_nact, s_i0, s_i1;
  __shared__ unsigned s_tag;
  __shared__ int s_abort;  // a wait of this CTA ran out
  __shared__ unsigned s_mask[kRouteMaxExperts / 32];  // route mode: the routed experts, as bits
  const int np = a.T * a.k;  // <= kMaxCtaExperts (dense mode)
  uint64_t* htag = reinterpret_cast<uint64_t*>(a.htag);  // [T*k][padded I] tagged h words

  // ask L2 for what the metadata round reads; nothing is read into the SM
  // before the dependency wait (the previous kernel may still write it)
  if (warp == kFuConsumers) {
    for (int e = 32 * lane; e < a.E; e += 32 * 32) prefetch_l2(a.table + e);
    if (RT) {  // the token's logits (the routing's input) instead of the routing
      for (int b = 128 * lane; b < a.E * 4; b += 128 * 32) prefetch_l2(reinterpret_cast<const uint8_t*>(a.logits) + b);
    } else {
      if (lane == 0) prefetch_l2(a.n_active);
      if (lane < 2) prefetch_l2(a.active + a.pass_begin + 32 * lane);
      if (lane == 2) prefetch_l2(a.ids);
      if (lane == 3) prefetch_l2(a.w);
    }
  } else {
    const int nx = a.T * a.H * 2;  // bytes of x
    for (int b = 128 * tid; b < nx; b += 128 * kFuConsumers * 32)
      prefetch_l2(reinterpret_cast<const uint8_t*>(a.x) + b);
  }
  if (tid == 0) {
    for (int s = 0; s < NSG; ++s) {
      mbar_init(&gfull[s], 1);
      mbar_init(&gempty[s], 1);
    }
    for (int s = 0; s < NSD; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dempty[s], a.nblk_d);
    }
    fence_barrier_init();
    s_abort = 0;
  }
  for (int s = tid; s < NSG + NSD; s += kFuThreads) s_iss[s] = 0;
  __syncthreads();
  volatile int* abort_flag = &s_abort;
  // until the producer has issued use u of stage idx (bounded)
  auto issued = [&](int idx, int u) -> bool {
    const volatile int* c = s_iss + idx;
    const long long t0 = clock64();
    while (*c <= u) {
      if (clock64() - t0 > a.wait_limit) return false;
      __nanosleep(32);
    }
    return true;
  };
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
    int na_raw = 0;
    int act_v[2] = {-1, -1};
    if (!RT) {
      na_raw = *a.n_active;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = lane + 32 * q;
        act_v[q] = i < cap ? a.active[a.pass_begin + i] : -1;
      }
    } else {
      s_mask[lane] = 0u;
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
    if (RT) {
      // the routed experts ascending (k distinct of E <= 1024): a bit each, then a warp scan
      routed_sync();
      if (lane < np) atomicOr(&s_mask[s_ids[lane] >> 5], 1u << (s_ids[lane] & 31));
      __syncwarp();
      const unsigned m = s_mask[lane];
      int incl = __popc(m);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int pos = incl - __popc(m);
      for (unsigned b = m; b; b &= b - 1) s_act[pos++] = 32 * lane + __ffs(b) - 1;
      na_raw = __shfl_sync(0xffffffffu, incl, 31);
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = lane + 32 * q;
        act_v[q] = i < na_raw ? s_act[i] : -1;
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
      if (r >= NSG) {  // a refill: the stage's previous item released, and no abort
        if (!mbar_wait_bounded(&gempty[s], (uint32_t)(((r / NSG) - 1) & 1), a.wait_limit) || *abort_flag) return false;
      }
      const int item = i0 + r;
      const int slot = s_slot[item / jt_n];
      if (!slot_ok(a, slot)) {
        mbar_arrive_expect_tx(&gfull[s], 0);
      } else {
        mbar_arrive_expect_tx(&gfull[s], tbg);
        bulk_g2s(gst + (size_t)s * SBG,
                 a.pool + (int64_t)slot * a.slot_bytes + a.q_gu + (int64_t)(item % jt_n) * tbg, tbg, &gfull[s]);
      }
      reinterpret_cast<volatile int*>(s_iss)[s] = r / NSG + 1;
      return true;
    };
    auto issue_dn = [&](int i) -> bool {
      const int s = i % NSD;
      if (i >= NSD) {
        if (!mbar_wait_bounded(&dempty[s], (uint32_t)(((i / NSD) - 1) & 1), a.wait_limit) || *abort_flag) return false;
      }
      const int slot = s_slot[i];
      if (!slot_ok(a, slot)) {
        mbar_arrive_expect_tx(&dfull[s], 0);
      } else {
        mbar_arrive_expect_tx(&dfull[s], tbd);
        bulk_g2s(dst_ + (size_t)s * SBD, a.pool + (int64_t)slot * a.slot_bytes + a.q_d + (int64_t)rt * tbd, tbd,
                 &dfull[s]);
      }
      reinterpret_cast<volatile int*>(s_iss)[NSG + s] = i / NSD + 1;
      return true;
    };
    // everything that fits goes out at once, one copy per lane; the rest
    // (lane 0) as stages free up
    const int ng0 = my_items < NSG ? my_items : NSG, nd0 = n_dn < NSD ? n_dn : NSD;
    for (int r = lane; r < ng0; r += 32) issue_gu(r);
    for (int i = lane; i < nd0; i += 32) issue_dn(i);
    __syncwarp();
    if (lane == 0) {
      bool ok = true;
      int ng = ng0, nd = nd0;  // copies issued (each completes its stage's phase)
      while (ok && ng < my_items) {
        if (issue_gu(ng)) ++ng;
        else ok = false;
      }
      while (ok && nd < n_dn) {
        if (issue_dn(nd)) ++nd;
        else ok = false;
      }
      if (!ok) *abort_flag = 1;
      // every copy issued lands before the CTA can leave
      bool landed = true;
      for (int s = 0; s < NSG && s < ng; ++s) {
        const int last = s + ((ng - 1 - s) / NSG) * NSG;  // last item issued on stage s
        landed &= mbar_wait_bounded(&gfull[s], (uint32_t)((last / NSG) & 1), kDefaultWaitCycles);
      }
      for (int s = 0; s < NSD && s < nd; ++s) {
        const int last = s + ((nd - 1 - s) / NSD) * NSD;
        landed &= mbar_wait_bounded(&dfull[s], (uint32_t)((last / NSD) & 1), kDefaultWaitCycles);
      }
      if ((!ok || !landed) && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
    }
    return;
  }

  // ---------------- consumers ----------------
  // this CTA's arrival on the launch's control word (its result is needed only
  // when the tag is published, before the table barrier)
  unsigned long long cw = 0ull;
  if (warp == 0 && lane == 0) {
    unsigned long long* ctr = reinterpret_cast<unsigned long long*>(a.ctl);
    cw = atomicAdd(ctr, 1ull);
    if ((unsigned)cw == gridDim.x - 1u) atomicAdd(ctr, kEpochOne - gridDim.x);  // the next launch's epoch
  }
  if (!RT) {
    for (int p = tid; p < np; p += kFuConsumers * 32) {
      s_ids[p] = a.ids[p];
      s_w[p] = a.w[p];
    }
  } else if (warp < kRouteWarps) {
    // route the token: every CTA the same, bit for bit
    route_select_token<kRouteMaxExperts / 256, 12>(a.logits, a.E, a.k, a.route_L, a.table, s_ids, s_w, 0, 1.0f);
    routed_arrive();
  }
  {
    // x' = x 2^-a (exact: a power of two; a by input position within its
    // 128-block) -> shared memory in MMA fragment order (frag_word), with
    // the per-(group, token) sums sum x and 128 sum x' that the group
    // epilogues apply; columns past H, tokens past T and groups past H are 0
    const int nx = a.T * a.H / 8;  // 16-byte words of x (H a multiple of 32)
    const int wpg = a.g / 8;       // words per group: consecutive lanes, aligned
    const int Kp = a.nblk_gu * 128, rw = (Kp + 8) / 2;  // padded row, row stride in words
    uint32_t* xw = reinterpret_cast<uint32_t*>(xh);
    float* xq = reinterpret_cast<float*>(xh + frag_rows_bytes(a.T, Kp));
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
        uint32_t* dst = xw + t * rw + frag_word(k);  // the four pairs are four t4 lanes apart
#pragma unroll
        for (int u = 0; u < 4; ++u) dst[16 * u] = w4[u];
        if ((idx % wpg) == 0) {
          const int G = k / a.g;
          xq[(G * 8 + t) * 2] = sx;
          xq[(G * 8 + t) * 2 + 1] = 128.0f * so;
        }
      }
    }
    const int npad = (Kp - a.H) / 2;  // pair words past H, per row
    for (int i = tid; i < a.T * npad; i += kFuConsumers * 32)
      xw[(i / npad) * rw + frag_word(a.H + 2 * (i % npad))] = 0u;
    for (int i = tid; i < (Kp / a.g) * 8; i += kFuConsumers * 32)
      if (i % 8 >= a.T || i / 8 >= a.H / a.g) xq[2 * i] = xq[2 * i + 1] = 0.f;
  }
  if (warp == 0 && lane == 0) {
    unsigned tg = 0u;  // 0: a count this launch cannot complete -- no valid tag, no work
    if ((unsigned)cw < gridDim.x) {
      const unsigned t = (unsigned)(cw >> 32) + 1u;
      tg = fmix32(t == 0u ? 1u : t);  // fmix32 maps only 0 to 0
    } else {
      *abort_flag = 1;
      if (a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
    }
    s_tag = tg;
  }
  tables_sync();  // the producer's pass tables (and the tag)
  const int n_act = s_nact, i0 = s_i0, i1 = s_i1;
  const unsigned tag = s_tag;
  if (RT && blockIdx.x == 0) {
    // the caller's copy of the routing, the sort and the lookup (as
    // moe_route_sort_lookup writes them): one token, so its k experts are
    // distinct and pair j of rank r in expert order sits at position r
    if (tid < np) {
      const int e = s_ids[tid];
      int r = 0;
      for (int q = 0; q < np; ++q) r += s_ids[q] < e;
      a.r_ids[tid] = e;
      a.r_w[tid] = s_w[tid];
      a.r_pairs[r] = tid;
    }
    for (int e = tid; e <= a.E; e += kFuConsumers * 32) {
      int r = 0;
      for (int q = 0; q < np; ++q) r += s_ids[q] < e;
      a.r_offsets[e] = r;
    }
    if (warp == 1) {
      const bool in = lane < n_act;
      const int e = in ? s_act[lane] : -1;
      const int sl = in ? s_slot[lane] : 0;
      if (in) {
        a.r_active[lane] = e;
        a.r_slots[lane] = sl;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, in && sl < 0);
      if (in && sl < 0) a.r_miss[__popc(bal & ((1u << lane) - 1u))] = e;
      if (lane == 0) {
        *a.r_n_active = n_act;
        *a.r_n_miss = __popc(bal);
      }
    }
  }
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
  consumers_sync(kFuConsumers * 32);  // x' in shared memory, pair map written
  bool timed_out = tag == 0u;

  // ---------------- gate/up + SwiGLU -> h: one item per warp pair ----------------
  {
    const int m = warp >> 1, hw = warp & 1;  // pair, half of K
    const int Kp = a.nblk_gu * 128;
    const uint4* xrow = g8 < a.T ? reinterpret_cast<const uint4*>(xh) + g8 * ((Kp + 8) / 8) : nullptr;
    const float4* xq4 = reinterpret_cast<const float4*>(xh + frag_rows_bytes(a.T, Kp));
    const int GRP = 8 * (int)a.rb_gu;
    const int uoff = thread_unit_off<BG>(t4, g8);
    const int my_items = i1 - i0;
    int pass = 0;
    for (int q = m; q < my_items; q += kFuPairs, ++pass) {
      const int it = i0 + q, e = it / jt_n, jt = it % jt_n;
      const int s = q % NSG;
      const bool ok = slot_ok(a, s_slot[e]);
      // use q / NSG of the stage issued (so the barrier is in its phase), then its data
      timed_out |= *abort_flag != 0;
      if (!timed_out && !issued(s, q / NSG)) timed_out = true;
      if (!timed_out && !mbar_wait_bounded(&gfull[s], (uint32_t)((q / NSG) & 1), a.wait_limit)) timed_out = true;
      if (timed_out) *abort_flag = 1;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (!timed_out && ok) {
        const uint8_t* st = gst + (size_t)s * SBG;
        const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
#pragma unroll 2
        for (int kb = hw; kb < a.nblk_gu; kb += 2) {
          uint32_t bf[8][2];
          float xs[8 / GS][2], xo[8 / GS][2];
          load_frag(xrow, kb, t4, bf);
#pragma unroll
          for (int G = 0; G < 8 / GS; ++G) {
            const float4 q = xq4[(kb * (8 / GS) + G) * 4 + t4];  // tokens 2 t4, 2 t4 + 1
            xs[G][0] = q.x;
            xo[G][0] = q.y;
            xs[G][1] = q.z;
            xo[G][1] = q.w;
          }
          block_mma<BG, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs, xo, acc);
        }
      }
      // pair reduction: the odd warp's partial sums go through shared memory
      // (double-buffered by item, so one barrier per item suffices)
      float* pr = red + ((size_t)((m * 2 + (pass & 1)) * 32 + lane)) * 4;
      if (hw == 1) *reinterpret_cast<float4*>(pr) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      pair_sync(m);
      if (hw == 1) continue;
      {
        const float4 o = *reinterpret_cast<const float4*>(pr);
        acc[0] += o.x;
        acc[1] += o.y;
        acc[2] += o.z;
        acc[3] += o.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&gempty[s]);
      // lane (j = g8, t4) holds gate (acc[c]) and up (acc[2 + c]) of column
      // jt * 8 + j for token 2 t4 + c; h is stored scaled by 2^-a of its
      // down pair slot (exact: a power of two), tagged with this launch
      const int kcol = jt * 8 + g8, kk = kcol & 127;
      const bool eighth = PairShift<BD>::a(2 * (kk >> 4) + ((kk & 15) >> 3)) == 3;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int n = 2 * t4 + c;
        const int pos = n < a.T ? s_tok[e * kDenseMaxTokens + n] : -1;  // -1: the token does not route here
        if (ok && !timed_out && pos >= 0) {
          const float gate = acc[c], up = acc[2 + c];
          const float hv = gate / (1.0f + expf(-gate)) * up;
          const uint16_t hb = f32_to_bf16_rne(eighth ? hv * 0.125f : hv);
          st_u64(htag + (int64_t)pos * Ip + kcol, ((uint64_t)tag << 32) | hb);
        }
      }
    }
  }

  // ---------------- down + combine -> y: (entry, K block) tasks over the warps ----------------
  if (has_rt) {
    const int GRP = 8 * (int)a.rb_d;
    const int uoff = thread_unit_off<BD>(t4, g8);
    const int nb = a.nblk_d;
    constexpr int GPB = 8 / GS;  // groups per 128-block
    const int srows = a.T > kFuFastTasks ? a.T : kFuFastTasks;  // scratch rows per warp
    uint32_t* hsc = reinterpret_cast<uint32_t*>(xh + a.h_stage_off + (size_t)warp * srows * kFuScratchPerTok);
    float2* gsum = reinterpret_cast<float2*>(hsc + srows * kFuScratchRowWords);  // [row][group of the block]
    float yacc[4] = {0.f, 0.f, 0.f, 0.f};
    const int ntask = n_act * nb;
    // One token whose down tiles are all resident at once (every entry has its
    // own stage, each used once): a warp's tasks (at most kFuFastTasks) read
    // their h blocks together -- one round of global reads instead of one
    // per task -- then wait for their tiles and compute back to back.
    const bool fast = a.T == 1 && n_act <= NSD && ntask <= kFuConsumers * kFuFastTasks;
    if (fast && !timed_out) {
      uint64_t fw[kFuFastTasks][4];
      int fi[kFuFastTasks], fkb[kFuFastTasks];
      bool fv[kFuFastTasks];
#pragma unroll
      for (int j = 0; j < kFuFastTasks; ++j) {
        const int task = warp + kFuConsumers * j;
        fi[j] = task < ntask ? task / nb : 0;
        fkb[j] = task < ntask ? task % nb : 0;
        const int p = task < ntask ? s_tok[fi[j] * kDenseMaxTokens] : -1;
        fv[j] = task < ntask && slot_ok(a, s_slot[fi[j]]) && p >= 0;
        fw[j][0] = fw[j][1] = fw[j][2] = fw[j][3] = 0ull;
        if (fv[j]) {
          const uint64_t* src = htag + (int64_t)p * Ip + fkb[j] * 128 + 4 * lane;
          ld_volatile_2w(src, fw[j][0], fw[j][1]);
          ld_volatile_2w(src + 2, fw[j][2], fw[j][3]);
        }
      }
      const long long t0 = clock64();
      for (;;) {
        bool fresh[kFuFastTasks];
        bool all = true;
#pragma unroll
        for (int j = 0; j < kFuFastTasks; ++j) {
          fresh[j] = true;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            fresh[j] &= !fv[j] || fkb[j] * 128 + 4 * lane + q >= a.I || (unsigned)(fw[j][q] >> 32) == tag;
          all &= fresh[j];
        }
        if (__all_sync(0xffffffffu, all)) break;
        if (clock64() - t0 > a.wait_limit) {
          timed_out = true;
          break;
        }
        __nanosleep(32);
#pragma unroll
        for (int j = 0; j < kFuFastTasks; ++j)
          if (!fresh[j]) {
            const uint64_t* src = htag + (int64_t)s_tok[fi[j] * kDenseMaxTokens] * Ip + fkb[j] * 128 + 4 * lane;
            ld_volatile_2w(src, fw[j][0], fw[j][1]);
            ld_volatile_2w(src + 2, fw[j][2], fw[j][3]);
          }
      }
      // stage each task's block (its own scratch row) and its per-group sums
      const int kk = (4 * lane) & 127;
      const bool eighth = PairShift<BD>::a(2 * (kk >> 4) + ((kk & 15) >> 3)) == 3;
      const int lpg = a.g / 4;  // lanes per group (8, 16 or 32)
#pragma unroll
      for (int j = 0; j < kFuFastTasks; ++j) {
        if (!fv[j]) continue;  // warp-uniform
        const int c0 = fkb[j] * 128 + 4 * lane;
        const uint32_t h0 = c0 < a.I ? (uint32_t)(fw[j][0] & 0xFFFFu) : 0u;
        const uint32_t h1 = c0 + 1 < a.I ? (uint32_t)(fw[j][1] & 0xFFFFu) : 0u;
        const uint32_t h2 = c0 + 2 < a.I ? (uint32_t)(fw[j][2] & 0xFFFFu) : 0u;
        const uint32_t h3 = c0 + 3 < a.I ? (uint32_t)(fw[j][3] & 0xFFFFu) : 0u;
        uint32_t* dst = hsc + j * kFuScratchRowWords + frag_word(4 * lane);  // pairs one t4 apart
        dst[0] = h0 | (h1 << 16);
        dst[16] = h2 | (h3 << 16);
        const float v = __uint_as_float(h0 << 16) + __uint_as_float(h1 << 16) + __uint_as_float(h2 << 16) +
                        __uint_as_float(h3 << 16);
        float sx = eighth ? 8.0f * v : v, so = 128.0f * v;
        for (int o = 1; o < lpg; o <<= 1) {
          sx += __shfl_xor_sync(0xffffffffu, sx, o);
          so += __shfl_xor_sync(0xffffffffu, so, o);
        }
        if ((lane % lpg) == 0) gsum[j * GPB + lane / lpg] = make_float2(sx, so);
      }
      __syncwarp();
      // the tasks' down tiles: entry i on stage i, its first and only use
#pragma unroll
      for (int j = 0; j < kFuFastTasks; ++j) {
        if (!fv[j] || timed_out) continue;
        if (!issued(NSG + fi[j], 0) || !mbar_wait_bounded(&dfull[fi[j]], 0u, a.wait_limit)) timed_out = true;
      }
      if (timed_out) *abort_flag = 1;
#pragma unroll
      for (int j = 0; j < kFuFastTasks; ++j) {
        if (!fv[j] || timed_out) continue;
        const int i = fi[j];
        const uint8_t* st = dst_ + (size_t)i * SBD;
        const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
        const int pb = s_tok[i * kDenseMaxTokens + g8];
        const int p0 = s_tok[i * kDenseMaxTokens + 2 * t4], p1 = s_tok[i * kDenseMaxTokens + 2 * t4 + 1];
        uint32_t bf[8][2];
        float xs1[GPB][2], xo1[GPB][2];
        load_frag(pb < 0 ? nullptr : reinterpret_cast<const uint4*>(hsc + j * kFuScratchRowWords), 0, t4, bf);
#pragma unroll
        for (int G = 0; G < GPB; ++G) {
          const float2 v0 = p0 < 0 ? make_float2(0.f, 0.f) : gsum[j * GPB + G];
          xs1[G][0] = v0.x;
          xo1[G][0] = v0.y;
          xs1[G][1] = 0.f;  // token 1 does not exist
          xo1[G][1] = 0.f;
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        block_mma<BD, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, fkb[j], uoff, bf, xs1, xo1, acc);
        const float w0 = p0 >= 0 ? s_w[p0] : 0.f, w1 = p1 >= 0 ? s_w[p1] : 0.f;
        yacc[0] += w0 * acc[0];
        yacc[1] += w1 * acc[1];
        yacc[2] += w0 * acc[2];
        yacc[3] += w1 * acc[3];
      }
    }
    for (int task = fast ? ntask : warp; task < ntask; task += kFuConsumers) {
      const int i = task / nb, kb = task % nb;
      const int s = i % NSD;
      const bool ok = slot_ok(a, s_slot[i]);
      timed_out |= *abort_flag != 0;
      if (ok && !timed_out) {
        // the entry's h words of this block, for each of its tokens: read
        // until every tag is this launch's (bounded), then stage the values
        // and the block's per-group sums (sum h, sum 128 h 2^-a)
        const long long t0 = clock64();
        for (int t = 0; t < a.T && !timed_out; ++t) {
          const int p = s_tok[i * kDenseMaxTokens + t];
          if (p < 0) continue;
          const int c0 = kb * 128 + 4 * lane;  // this lane's four columns
          const uint64_t* src = htag + (int64_t)p * Ip + c0;
          uint64_t w[4];
          for (;;) {
            ld_volatile_2w(src, w[0], w[1]);
            ld_volatile_2w(src + 2, w[2], w[3]);
            bool fresh = true;
#pragma unroll
            for (int j = 0; j < 4; ++j) fresh &= (unsigned)(w[j] >> 32) == tag || c0 + j >= a.I;
            if (__all_sync(0xffffffffu, fresh)) break;
            if (clock64() - t0 > a.wait_limit) {
              timed_out = true;
              break;
            }
            __nanosleep(32);
          }
          const uint32_t h0 = c0 < a.I ? (uint32_t)(w[0] & 0xFFFFu) : 0u;
          const uint32_t h1 = c0 + 1 < a.I ? (uint32_t)(w[1] & 0xFFFFu) : 0u;
          const uint32_t h2 = c0 + 2 < a.I ? (uint32_t)(w[2] & 0xFFFFu) : 0u;
          const uint32_t h3 = c0 + 3 < a.I ? (uint32_t)(w[3] & 0xFFFFu) : 0u;
          uint32_t* dst = hsc + t * kFuScratchRowWords + frag_word(4 * lane);  // pairs one t4 apart
          dst[0] = h0 | (h1 << 16);
          dst[16] = h2 | (h3 << 16);
          // per-group sums: the four columns share a pair slot, so one scale
          const int kk = (4 * lane) & 127;
          const bool eighth = PairShift<BD>::a(2 * (kk >> 4) + ((kk & 15) >> 3)) == 3;
          const float v = __uint_as_float(h0 << 16) + __uint_as_float(h1 << 16) + __uint_as_float(h2 << 16) +
                          __uint_as_float(h3 << 16);
          float sx = eighth ? 8.0f * v : v, so = 128.0f * v;
          // group G of the block covers lanes G * g / 4 .. (G + 1) * g / 4 - 1
          const int lpg = a.g / 4;  // lanes per group (8, 16 or 32)
          for (int o = 1; o < lpg; o <<= 1) {
            sx += __shfl_xor_sync(0xffffffffu, sx, o);
            so += __shfl_xor_sync(0xffffffffu, so, o);
          }
          if ((lane % lpg) == 0) gsum[t * GPB + lane / lpg] = make_float2(sx, so);
        }
        __syncwarp();
        if (!timed_out && !issued(NSG + s, i / NSD)) timed_out = true;
        if (!timed_out && !mbar_wait_bounded(&dfull[s], (uint32_t)((i / NSD) & 1), a.wait_limit)) timed_out = true;
        if (timed_out) *abort_flag = 1;
      }
      if (ok && !timed_out) {
        const uint8_t* st = dst_ + (size_t)s * SBD;
        const uint32_t* sbs = reinterpret_cast<const uint32_t*>(st + 2 * GRP);
        const int pb = s_tok[i * kDenseMaxTokens + g8];
        const int p0 = s_tok[i * kDenseMaxTokens + 2 * t4], p1 = s_tok[i * kDenseMaxTokens + 2 * t4 + 1];
        uint32_t bf[8][2];
        float xs1[GPB][2], xo1[GPB][2];
        load_frag(pb < 0 ? nullptr : reinterpret_cast<const uint4*>(hsc + g8 * kFuScratchRowWords), 0, t4, bf);
#pragma unroll
        for (int G = 0; G < GPB; ++G) {
          const float2 v0 = p0 < 0 ? make_float2(0.f, 0.f) : gsum[(2 * t4) * GPB + G];
          const float2 v1 = p1 < 0 ? make_float2(0.f, 0.f) : gsum[(2 * t4 + 1) * GPB + G];
          xs1[G][0] = v0.x;
          xo1[G][0] = v0.y;
          xs1[G][1] = v1.x;
          xo1[G][1] = v1.y;
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        block_mma<BD, GS>(st, st + GRP, sbs + g8, sbs + 8 + g8, kb, uoff, bf, xs1, xo1, acc);
        const float w0 = p0 >= 0 ? s_w[p0] : 0.f, w1 = p1 >= 0 ? s_w[p1] : 0.f;
        yacc[0] += w0 * acc[0];
        yacc[1] += w1 * acc[1];
        yacc[2] += w0 * acc[2];
        yacc[3] += w1 * acc[3];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[s]);
    }
    // y rows of the CTA's tile: the sum over the warps (fixed order)
    consumers_sync(kFuConsumers * 32);  // the pair partials in red are read
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
  }
  if (timed_out && lane == 0 && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------
template <int BG, int BD, int BPW, int GS, bool RT>
static cudaError_t launch_fused_t(const FfnArgs& a, int grid, size_t smem, cudaStream_t st) {
  static int done[4] = {0, 0, 0, 0};
  const void* kern = reinterpret_cast<const void*>(ffn_fused_kernel<BG, BD, BPW, GS, RT>);
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
  const bool rt = a.logits != nullptr;
  if (gs == 2) return rt ? launch_fused_t<BG, BD, BPW, 2, true>(a, grid, smem, st)
                         : launch_fused_t<BG, BD, BPW, 2, false>(a, grid, smem, st);
  if (gs == 4) return rt ? launch_fused_t<BG, BD, BPW, 4, true>(a, grid, smem, st)
                         : launch_fused_t<BG, BD, BPW, 4, false>(a, grid, smem, st);
  return rt ? launch_fused_t<BG, BD, BPW, 8, true>(a, grid, smem, st)
            : launch_fused_t<BG, BD, BPW, 8, false>(a, grid, smem, st);
}

template <int BG>
static cudaError_t fused_bd(const FfnArgs& a, int bd, int gs, int grid, size_t smem, cudaStream_t st) {
  if (bd == 3) return fused_gs<BG, 3, 1>(a, gs, grid, smem, st);
  if (bd == 4) return fused_gs<BG, 4, 1>(a, gs, grid, smem, st);
  return fused_gs<BG, 6, 1>(a, gs, grid, smem, st);
}

// Stage sizes and counts of the fused kernel for this call (into a), its
// shared memory; false when the fused path does not apply (the caller then
// uses the two-kernel path).
bool ffn_fused_plan(FfnArgs& a, const moe_layer_desc& d, int num_sms, size_t& smem) {
  if (!(a.T <= kDenseMaxTokens && a.T * d.k <= kMaxCtaExperts) || a.ctl == nullptr || a.htag == nullptr)
    return false;
  if (d.E > 1024 || d.I % 8 || d.H / 16 > num_sms) return false;
  const int grid = num_sms;
  int max_pass = a.pass_len < d.E ? a.pass_len : d.E;
  if (a.T * d.k < max_pass) max_pass = a.T * d.k;
  if (max_pass < 1) max_pass = 1;
  a.gu_stage_bytes = (int)round_up(a.L.tile_gu, 128);
  a.d_stage_bytes = (int)round_up(a.L.tile_d, 128);
  // x' (fragment order) and its per-(group, token) sums, tokens padded to 8;
  // then each warp's h block scratch
  const int Kx = (int)padded_k(d.H);
  const size_t xb = (size_t)round_up((int64_t)frag_rows_bytes(a.T, Kx) + (int64_t)(Kx / d.group) * 8 * 8, 128);
  a.h_stage_off = (int)xb;
  const int srows = a.T > kFuFastTasks ? a.T : kFuFastTasks;  // each warp's scratch rows
  a.xh_stage_bytes = (int)round_up((int64_t)xb + (int64_t)kFuConsumers * srows * kFuScratchPerTok, 128);
  // the most gate/up items a CTA can get: a CTA without a down tile takes the
  // whole quota of (gate/up + down bytes) / grid, or the items / (CTAs
  // without a down tile) where a down tile is more than the quota (which case
  // applies does not depend on the number of experts)
  const int n_rt = d.H / 16, jt_n = d.I / 8;
  const double tot = (double)max_pass * jt_n * a.L.tile_gu + (double)n_rt * max_pass * a.L.tile_d;
  const bool even = (double)max_pass * a.L.tile_d * grid <= tot;
  const int64_t items_max =
      even ? (int64_t)(tot / grid / a.L.tile_gu) + 2 : (int64_t)max_pass * jt_n / (grid - n_rt) + 2;
  const size_t fixed = (size_t)a.xh_stage_bytes + (size_t)kFuRedFloats * 4 + kFuTableBytes + (size_t)d.E * 4 + 16;
  const size_t cap = 220 * 1024;
  if (fixed + (size_t)a.gu_stage_bytes + (size_t)a.d_stage_bytes + 64 > cap) return false;
  // down stages: every expert of the pass if possible; gate/up stages: every
  // item of the CTA if possible
  int nsd = max_pass;
  int nsg = (int)(items_max < 1 ? 1 : items_max);
  while ((size_t)nsd * a.d_stage_bytes + (size_t)nsg * a.gu_stage_bytes + fixed + 20 * (nsd + nsg) > cap) {
    if (nsg > nsd && nsg > 1) --nsg;
    else if (nsd > 1) --nsd;
    else if (nsg > 1) --nsg;
    else return false;
  }
  a.gu_nstage = nsg;
  a.d_nstage = nsd;
  smem = (size_t)nsg * a.gu_stage_bytes + (size_t)nsd * a.d_stage_bytes + fixed + 20 * (nsd + nsg);
  return true;
}

cudaError_t launch_ffn_fused(FfnArgs a, const moe_layer_desc& d, int num_sms, cudaStream_t st) {
  size_t smem = 0;
  if (!ffn_fused_plan(a, d, num_sms, smem)) return cudaErrorNotSupported;
  // route mode: one token, one pass over every expert
  if (a.logits != nullptr &&
      (a.T != 1 || d.E > kRouteMaxExperts || d.k > 32 || a.pass_begin != 0 || a.pass_len < d.E || !a.r_ids ||
       !a.r_w || !a.r_offsets || !a.r_pairs || !a.r_active || !a.r_n_active || !a.r_slots || !a.r_miss ||
       !a.r_n_miss))
    return cudaErrorNotSupported;
  const int grid = num_sms;
  const int gs = d.group / 16;
  if (d.bits_gu == 3) return fused_bd<3>(a, d.bits_down, gs, grid, smem, st);
  if (d.bits_gu == 4) return fused_bd<4>(a, d.bits_down, gs, grid, smem, st);
  return fused_bd<6>(a, d.bits_down, gs, grid, smem, st);
}

}  // namespace moe
