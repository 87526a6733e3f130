// Routing of one token by a block of 256 threads (stage 1: route_topk with
// cache-aware substitution, BigMoeOnEdge's commit note: resident experts'
// scores raised by L x the token's score range, top-k taken again), shared by
// the routing kernels and the stage kernels that route a token themselves, so
// that all give the same ids, order and weights bit for bit.
#pragma once

#include <cfloat>
#include <climits>

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// exp for routing: Cody & Waite reduction x = n ln2 + r (ln2 split into a
// 15-significant-bit head and a tail, both applied with fma), e^r by the
// degree-7 Taylor polynomial in Horner form, 2^n through the exponent field.
// Every operation is an explicit round-to-nearest intrinsic, so the compiler
// cannot contract or reorder: the result is a fixed function of x that a CPU
// evaluation of the same steps reproduces bit for bit.  Domain x <= 0;
// x < -87 gives 0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float route_exp(float x) {
  if (!(x >= -87.0f)) return 0.0f;
  if (x > 0.0f) x = 0.0f;
  const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));  // x * log2(e)
  float r = __fmaf_rn(-n, 0x1.62e400p-1f, x);          // ln2 head
  r = __fmaf_rn(-n, 0x1.7f7d1cp-20f, r);               // ln2 tail
  float p = 0x1.a01a02p-13f;                            // 1/7!
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);                 // 1/6!
  p = __fmaf_rn(p, r, 0x1.111112p-7f);                  // 1/5!
  p = __fmaf_rn(p, r, 0x1.555556p-5f);                  // 1/4!
  p = __fmaf_rn(p, r, 0x1.555556p-3f);                  // 1/3!
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int ni = (int)n;  // [-126, 0]
  return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

// Key order: (u' desc, l desc, e asc).
__device__ __forceinline__ bool key_better(float au, float al, int ae, float bu, float bl, int be) {
  return au > bu || (au == bu && (al > bl || (al == bl && ae < be)));
}

// The barrier of the 256 routing threads: the whole block (BAR < 0), or named
// barrier BAR over threads 0..255 of a larger block.
template <int BAR>
__device__ __forceinline__ void route_bar() {
  if constexpr (BAR < 0) {
    __syncthreads();
  } else {
    asm volatile("bar.sync %0, 256;" ::"n"(BAR) : "memory");
  }
}

// One block (8 warps) per token, for decode-sized T: thread i owns experts
// e = i + 256 m.  The top-k is a radix select on a 64-bit key whose order is
// the selection order: high word = bits of u' (non-negative floats order as
// their bit patterns), low word = l mapped to an order-preserving unsigned
// (-0 taken as +0, so that equal logits compare equal), ties on the whole key
// broken by the lower expert id.  Eight-bit digits from the top: each pass
// histograms the digit of the experts still tied with the selection boundary,
// finds the digit value that holds the k-th best, takes every expert above
// it and keeps the tied ones; a pass whose boundary bucket is exactly the
// number still to take ends the select (usually after two or three passes).
// The chosen experts are then put in key order by counting, for each, the
// chosen ones with a better key.  Same ids, order and weights as route_kernel.
__device__ __forceinline__ uint32_t ordered_logit(float l) {
  uint32_t b = __float_as_uint(l);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ uint32_t key_digit(uint32_t k1, uint32_t k2, int d) {
  return d < 4 ? (k1 >> (24 - 8 * d)) & 0xFFu : (k2 >> (56 - 8 * d)) & 0xFFu;
}

__device__ __forceinline__ bool key_before(uint32_t a1, uint32_t a2, int ae, uint32_t b1, uint32_t b2, int be) {
  return a1 > b1 || (a1 == b1 && (a2 > b2 || (a2 == b2 && ae < be)));
}

// The 256 threads of the block route the token of logits row `l`: ids_row /
// w_row receive its k experts in key order and their weights, then the ns
// shared experts (ids E.., weight sw_t).
template <int NPT, int BAR = -1>
__device__ __forceinline__ void route_select_token(const float* __restrict__ l, int E, int k, float L,
                                                   const int32_t* __restrict__ table, int32_t* __restrict__ ids_row,
                                                   float* __restrict__ w_row, int ns, float sw_t) {
  __shared__ float s_red[8];
  __shared__ uint32_t s_hist[256];
  __shared__ int s_ctl[3];  // boundary digit, experts still to take, boundary bucket size
  __shared__ int s_warp[8];
  __shared__ int s_nsel;
  __shared__ uint32_t s_k1[32], s_k2[32];
  __shared__ int s_e[32];
  __shared__ float s_u[32];
  __shared__ int s_oe[32];
  __shared__ float s_ou[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float lv[NPT], u[NPT];
  bool res[NPT];
  float lmax = -FLT_MAX;
#pragma unroll
  for (int m = 0; m < NPT; ++m) {
    const int e = tid + 256 * m;
    lv[m] = e < E ? l[e] : -FLT_MAX;
    res[m] = (L > 0.0f && table != nullptr && e < E) ? table[e] >= 0 : false;
    lmax = fmaxf(lmax, lv[m]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if (lane == 0) s_red[warp] = lmax;
  if (tid == 0) s_nsel = 0;
  route_bar<BAR>();
  lmax = s_red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) lmax = fmaxf(lmax, s_red[w]);
  float umin = FLT_MAX;
#pragma unroll
  for (int m = 0; m < NPT; ++m) {
    const int e = tid + 256 * m;
    u[m] = e < E ? route_exp(__fsub_rn(lv[m], lmax)) : 0.0f;
    if (e < E) umin = fminf(umin, u[m]);
  }
  float boost = 0.0f;
  if (L > 0.0f && table != nullptr) {
#pragma unroll
    for (int o = 16; o; o >>= 1) umin = fminf(umin, __shfl_xor_sync(0xffffffffu, umin, o));
    route_bar<BAR>();  // every warp has read s_red
    if (lane == 0) s_red[warp] = umin;
    route_bar<BAR>();
    umin = s_red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) umin = fminf(umin, s_red[w]);
    boost = __fmul_rn(L, __fsub_rn(1.0f, umin));
  }
  uint32_t k1[NPT], k2[NPT];
  bool cand[NPT], sel[NPT];
#pragma unroll
  for (int m = 0; m < NPT; ++m) {
    const int e = tid + 256 * m;
    k1[m] = __float_as_uint(res[m] ? __fadd_rn(u[m], boost) : u[m]);
    k2[m] = ordered_logit(lv[m]);
    cand[m] = e < E;
    sel[m] = false;
  }
  int need = k;  // experts still to take among the candidates
  bool done = false;
  for (int d = 0; d < 8 && !done; ++d) {
    s_hist[tid] = 0u;
    route_bar<BAR>();
#pragma unroll
    for (int m = 0; m < NPT; ++m) {
      const uint32_t dig = cand[m] ? key_digit(k1[m], k2[m], d) : 0x100u;
      const uint32_t peers = __match_any_sync(0xffffffffu, dig);
      if (cand[m] && lane == __ffs(peers) - 1) atomicAdd(&s_hist[dig], (uint32_t)__popc(peers));
    }
    route_bar<BAR>();
    if (warp == 0) {  // lane i covers bins 255 - 8 i down to 248 - 8 i
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = s_hist[255 - 8 * lane - i];
        tot += c[i];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t above = incl - tot;
      if (above < (uint32_t)need && (uint32_t)need <= incl) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above + c[i] >= (uint32_t)need) {
            s_ctl[0] = 255 - 8 * lane - i;
            s_ctl[1] = need - (int)above;
            s_ctl[2] = (int)c[i];
            break;
          }
          above += c[i];
        }
      }
    }
    route_bar<BAR>();
    const uint32_t bd = (uint32_t)s_ctl[0];
    need = s_ctl[1];
    done = s_ctl[2] == need;  // the whole boundary bucket is taken
#pragma unroll
    for (int m = 0; m < NPT; ++m) {
      if (!cand[m]) continue;
      const uint32_t dig = key_digit(k1[m], k2[m], d);
      if (dig > bd || (done && dig == bd)) {
        sel[m] = true;
        cand[m] = false;
      } else if (dig < bd) {
        cand[m] = false;
      }
    }
  }
  if (!done) {  // the candidates left share the whole key: take the `need` lowest expert ids
    int base = 0;
#pragma unroll
    for (int m = 0; m < NPT; ++m) {
      const uint32_t bal = __ballot_sync(0xffffffffu, cand[m]);
      route_bar<BAR>();  // s_warp free
      if (lane == 0) s_warp[warp] = __popc(bal);
      route_bar<BAR>();
      int before = 0, total = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        before += w < warp ? s_warp[w] : 0;
        total += s_warp[w];
      }
      const int rank = base + before + __popc(bal & ((1u << lane) - 1u));
      if (cand[m] && rank < need) sel[m] = true;
      base += total;
    }
  }
  // the k chosen experts, then each one's position in key order
#pragma unroll
  for (int m = 0; m < NPT; ++m)
    if (sel[m]) {
      const int i = atomicAdd(&s_nsel, 1);
      s_k1[i] = k1[m];
      s_k2[i] = k2[m];
      s_e[i] = tid + 256 * m;
      s_u[i] = u[m];
    }
  route_bar<BAR>();
  if (warp == 0) {
    int pos = 0;
    const bool mine = lane < k;
    const uint32_t a1 = mine ? s_k1[lane] : 0u, a2 = mine ? s_k2[lane] : 0u;
    const int ae = mine ? s_e[lane] : 0;
    for (int i = 0; i < k; ++i) pos += key_before(s_k1[i], s_k2[i], s_e[i], a1, a2, ae) ? 1 : 0;
    if (mine) {
      s_oe[pos] = ae;
      s_ou[pos] = s_u[lane];
    }
    __syncwarp();
    const float my_u = mine ? s_ou[lane] : 0.0f;
    float sum = my_u;
#pragma unroll
    for (int o = 16; o; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, o));
    if (mine) {  // the row: the top-k, then the shared experts
      ids_row[lane] = s_oe[lane];
      w_row[lane] = __fdiv_rn(my_u, sum);
    }
    if (lane < ns) {
      ids_row[k + lane] = E + lane;
      w_row[k + lane] = sw_t;
    }
  }
}

}  // namespace moe
