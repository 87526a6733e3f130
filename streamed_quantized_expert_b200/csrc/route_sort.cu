// Stages 1-3: route_topk (+ cache-aware substitution), moe_sort, slot lookup.
//
// Stage 1 follows BigMoeOnEdge's commit note on cache-aware substitution
// (resident experts' scores raised by L x the token's score range, top-k taken
// again, the same number of experts runs).  Stage 2 follows the transformers
// PR #50717 notes and the RFC's "Prefill" item (tokens sorted by expert, 64
// experts per pass).  Stage 3 follows the RFC's "Cache" item (per-layer
// expert -> slot table over one preallocated pool).
#include <cfloat>
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "route_block.cuh"

namespace moe {

__global__ void exp_kernel(const float* __restrict__ x, int64_t n, float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = route_exp(x[i]);
}

// One warp per token; lane owns experts e = 32*i + lane.
template <int NPL>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int T, int E, int k, float L,
                                                    const int32_t* __restrict__ table, int32_t* __restrict__ ids,
                                                    float* __restrict__ wout, int ns, const float* __restrict__ sw) {
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  pdl_wait();
  pdl_launch_dependents();
  if (t >= T) return;
  const float* l = logits + (size_t)t * E;
  float lv[NPL], u[NPL], up[NPL];
  float lmax = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = 32 * i + lane;
    lv[i] = e < E ? l[e] : -FLT_MAX;
    lmax = fmaxf(lmax, lv[i]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = 32 * i + lane;
    u[i] = e < E ? route_exp(__fsub_rn(lv[i], lmax)) : -1.0f;
    up[i] = u[i];
  }
  if (L > 0.0f && table != nullptr) {
    float umin = FLT_MAX;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (32 * i + lane < E) umin = fminf(umin, u[i]);
#pragma unroll
    for (int o = 16; o; o >>= 1) umin = fminf(umin, __shfl_xor_sync(0xffffffffu, umin, o));
    const float boost = __fmul_rn(L, __fsub_rn(1.0f, umin));
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = 32 * i + lane;
      if (e < E && table[e] >= 0) up[i] = __fadd_rn(u[i], boost);
    }
  }
  uint32_t taken = 0;
  int my_e = 0;
  float my_u = 0.0f;
  for (int j = 0; j < k; ++j) {
    float bu = -FLT_MAX, bl = -FLT_MAX, bw = 0.0f;
    int be = INT_MAX;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = 32 * i + lane;
      if (e < E && !((taken >> i) & 1u) && key_better(up[i], lv[i], e, bu, bl, be)) {
        bu = up[i];
        bl = lv[i];
        be = e;
        bw = u[i];
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ou = __shfl_xor_sync(0xffffffffu, bu, o);
      const float ol = __shfl_xor_sync(0xffffffffu, bl, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      const float ow = __shfl_xor_sync(0xffffffffu, bw, o);
      if (key_better(ou, ol, oe, bu, bl, be)) {
        bu = ou;
        bl = ol;
        be = oe;
        bw = ow;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == j) {
      my_e = be;
      my_u = bw;
    }
  }
  float s = lane < k ? my_u : 0.0f;
#pragma unroll
  for (int o = 16; o; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
  const int ks = k + ns;  // output row: the top-k, then the shared experts
  if (lane < k) {
    ids[(size_t)t * ks + lane] = my_e;
    wout[(size_t)t * ks + lane] = __fdiv_rn(my_u, s);
  }
  if (lane < ns) {
    ids[(size_t)t * ks + k + lane] = E + lane;
    wout[(size_t)t * ks + k + lane] = sw ? sw[t] : 1.0f;
  }
}

template <int NPT>
__global__ void __launch_bounds__(256) route_select_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                           float L, const int32_t* __restrict__ table,
                                                           int32_t* __restrict__ ids, float* __restrict__ wout, int ns,
                                                           const float* __restrict__ sw) {
  const int t = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  if (t >= T) return;
  const int ks = k + ns;  // output row: the top-k, then the shared experts
  route_select_token<NPT>(logits + (size_t)t * E, E, k, L, table, ids + (size_t)t * ks, wout + (size_t)t * ks, ns,
                          (ns > 0 && sw) ? sw[t] : 1.0f);
}

// One decode token's stages 1-3 in one block: route (as route_select_kernel,
// with ns shared experts E .. E + ns - 1 of weight sw after the top k), then
// the sort of its k + ns pairs (distinct experts: the active list is the
// routed experts ascending, then the shared ones; pair j of rank r sits at
// position r) and the slot lookup over the whole active list (as
// sort_small_kernel and lookup_kernel write them for T = 1).  With host_meta
// (page-locked host memory the device can address), warp 1 also writes
// n_active to host_meta[0] and the active list to host_meta[2 ..], then, once
// those writes are visible system-wide, seq to host_meta[1]: the host waits
// for seq there instead of copying the list back and synchronising.
template <int NPT>
__global__ void __launch_bounds__(256) route_sort_lookup_kernel(
    const float* __restrict__ logits, int E, int k, float L, const int32_t* __restrict__ table, int ns,
    const float* __restrict__ sw, int n_slots, int32_t* __restrict__ ids, float* __restrict__ w,
    int32_t* __restrict__ offsets, int32_t* __restrict__ pairs, int32_t* __restrict__ active,
    int32_t* __restrict__ n_active, int32_t* __restrict__ slots, int32_t* __restrict__ miss,
    int32_t* __restrict__ n_miss, int32_t* __restrict__ dev_err, int32_t* host_meta, int32_t seq) {
  __shared__ int s_sel[32];  // the token's experts, rank order (k + ns <= 32)
  __shared__ int s_act[32];  // ascending
  const int tid = threadIdx.x, n = k + ns, Ew = E + ns;
  pdl_wait();
  pdl_launch_dependents();
  route_select_token<NPT>(logits, E, k, L, table, ids, w, ns, (ns > 0 && sw) ? sw[0] : 1.0f);
  __syncthreads();  // the block's own global writes of ids are visible to it
  if (tid < n) s_sel[tid] = ids[tid];
  __syncthreads();
  if (tid < n) {
    const int e = s_sel[tid];
    int r = 0;
    for (int j = 0; j < n; ++j) r += s_sel[j] < e;
    s_act[r] = e;
    active[r] = e;
    pairs[r] = tid;
  }
  for (int e = tid; e <= Ew; e += 256) {
    int c = 0;
    for (int j = 0; j < n; ++j) c += s_sel[j] < e;
    offsets[e] = c;
  }
  __syncthreads();
  if (tid < 32) {  // lookup: one lane per active expert (k + ns <= 32)
    const bool in = tid < n;
    const int e = in ? s_act[tid] : -1;
    const int sl = in ? table[e] : 0;
    if (in) slots[tid] = sl;
    if (in && sl >= n_slots && dev_err) atomicOr(dev_err, MOE_DEV_ERR_SLOT_RANGE);
    const unsigned bal = __ballot_sync(0xffffffffu, in && sl < 0);
    if (in && sl < 0) miss[__popc(bal & ((1u << tid) - 1u))] = e;
    if (tid == 0) {
      *n_active = n;
      *n_miss = __popc(bal);
    }
  } else if (tid < 64 && host_meta) {
    const int lane = tid - 32;
    if (lane < n) host_meta[2 + lane] = s_act[lane];
    if (lane == 0) host_meta[0] = n;
    __threadfence_system();
    __syncwarp();
    if (lane == 0) *reinterpret_cast<volatile int32_t*>(host_meta + 1) = seq;
  }
}

// ---------------------------------------------------------------------------
// moe_sort
// ---------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ int block_excl_scan(int v, int* total, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int excl = x - v + (warp ? s_warp[warp - 1] : 0);
  if (total) *total = s_warp[31];
  __syncthreads();
  return excl;
}

// Offsets + active list from per-expert totals held one per thread.
__device__ void write_offsets_active(int cnt, int E, int n, int32_t* offsets, int32_t* active, int32_t* n_active,
                                     int* s_warp, int* s_off) {
  const int e = threadIdx.x;
  const int off = block_excl_scan(e < E ? cnt : 0, nullptr, s_warp);
  if (e < E) {
    offsets[e] = off;
    s_off[e] = off;
  }
  if (e == 0) offsets[E] = n;
  int na = 0;
  const int apos = block_excl_scan((e < E && cnt > 0) ? 1 : 0, &na, s_warp);
  if (e < E && cnt > 0) active[apos] = e;
  if (e == 0) *n_active = na;
}

// Whole sort in one CTA when T*k <= 1024.
__global__ void __launch_bounds__(1024) sort_small_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                          int32_t* __restrict__ offsets, int32_t* __restrict__ pairs,
                                                          int32_t* __restrict__ active, int32_t* __restrict__ n_active) {
  __shared__ int s_hist[1024];
  __shared__ int s_off[1024];
  __shared__ int s_ids[1024];
  __shared__ int s_warp[32];
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  s_hist[tid] = 0;
  __syncthreads();
  int e = -1;
  if (tid < n) {
    e = ids[tid];
    s_ids[tid] = e;
    atomicAdd(&s_hist[e], 1);
  }
  __syncthreads();
  write_offsets_active(s_hist[tid], E, n, offsets, active, n_active, s_warp, s_off);
  __syncthreads();
  if (tid < n) {
    int rank = 0;
    for (int i = 0; i < tid; ++i) rank += (s_ids[i] == e);
    pairs[s_off[e] + rank] = tid;
  }
}

// Large sorts: chunks of 1024 pairs.  (1) per-chunk histograms.
__global__ void __launch_bounds__(1024) sort_hist_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                         int32_t* __restrict__ chunk_hist) {
  __shared__ int s_hist[1024];
  pdl_wait();
  pdl_launch_dependents();
  s_hist[threadIdx.x] = 0;
  __syncthreads();
  const int i = blockIdx.x * 1024 + threadIdx.x;
  if (i < n) atomicAdd(&s_hist[ids[i]], 1);
  __syncthreads();
  if ((int)threadIdx.x < E) chunk_hist[(size_t)blockIdx.x * E + threadIdx.x] = s_hist[threadIdx.x];
}

// (2) offsets, active, and per-chunk bases (in place over chunk_hist).
__global__ void __launch_bounds__(1024) sort_scan_kernel(int32_t* __restrict__ chunk_hist, int nchunk, int n, int E,
                                                         int32_t* __restrict__ offsets, int32_t* __restrict__ active,
                                                         int32_t* __restrict__ n_active) {
  __shared__ int s_off[1024];
  __shared__ int s_warp[32];
  const int e = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  int tot = 0;
  if (e < E)
    for (int c = 0; c < nchunk; ++c) tot += chunk_hist[(size_t)c * E + e];
  write_offsets_active(tot, E, n, offsets, active, n_active, s_warp, s_off);
  if (e < E) {
    int run = s_off[e];
    for (int c = 0; c < nchunk; ++c) {
      const int v = chunk_hist[(size_t)c * E + e];
      chunk_hist[(size_t)c * E + e] = run;
      run += v;
    }
  }
}

// (3) stable scatter inside each chunk.
__global__ void __launch_bounds__(1024) sort_scatter_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                            const int32_t* __restrict__ chunk_base,
                                                            int32_t* __restrict__ pairs) {
  __shared__ int s_ids[1024];
  __shared__ int s_base[1024];
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x * 1024 + threadIdx.x;
  const int e = i < n ? ids[i] : -1;
  s_ids[threadIdx.x] = e;
  if ((int)threadIdx.x < E) s_base[threadIdx.x] = chunk_base[(size_t)blockIdx.x * E + threadIdx.x];
  __syncthreads();
  if (i < n) {
    int rank = 0;
    for (int j = 0; j < (int)threadIdx.x; ++j) rank += (s_ids[j] == e);
    pairs[s_base[e] + rank] = i;
  }
}

// x_sorted[i] = fp16(x[pairs[i] / k]) (the tensor-core path's operand type):
// one warp per row, 16-byte loads and stores, bf16 -> fp16 round to nearest
// even, saturating at +-65504.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  return (uint32_t)f32_to_f16_sat(bf16_lo(v)) | ((uint32_t)f32_to_f16_sat(bf16_hi(v)) << 16);
}

__global__ void gather_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ pairs, int n, int k,
                                   int H, uint16_t* __restrict__ xs) {
  const int lane = threadIdx.x & 31;
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= n) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(pairs[row] / k) * H);
  uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)row * H);
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 v = src[c];
    dst[c] = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
  }
}

// ---------------------------------------------------------------------------
// slot lookup
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) lookup_kernel(const int32_t* __restrict__ table,
                                                      const int32_t* __restrict__ active,
                                                      const int32_t* __restrict__ n_active, int pass_begin,
                                                      int pass_len, int n_slots, int32_t* __restrict__ slots,
                                                      int32_t* __restrict__ miss, int32_t* __restrict__ n_miss,
                                                      int32_t* __restrict__ dev_err) {
  __shared__ int s_warp[32];
  pdl_wait();
  pdl_launch_dependents();
  const int na = *n_active;
  int end = pass_begin + pass_len;
  if (end > na) end = na;
  const int cnt = end > pass_begin ? end - pass_begin : 0;
  const int i = threadIdx.x;
  int e = -1, s = 0;
  if (i < cnt) {
    e = active[pass_begin + i];
    s = table[e];
    slots[i] = s;
    if (s >= n_slots && dev_err) atomicOr(dev_err, MOE_DEV_ERR_SLOT_RANGE);
  }
  const bool is_miss = (i < cnt) && s < 0;
  int nm = 0;
  const int pos = block_excl_scan(is_miss ? 1 : 0, &nm, s_warp);
  if (is_miss) miss[pos] = e;
  if (i == 0) *n_miss = nm;
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_route(const float* logits, int T, int E, int k, float L, const int32_t* table, int32_t* ids,
                         float* w, int n_shared, const float* shared_w, cudaStream_t st) {
  if (T <= kRouteBlockMaxTokens && E <= 1024) {  // decode sizes: a block per token
    const void* kb = E <= 256 ? reinterpret_cast<const void*>(route_select_kernel<1>)
                     : E <= 512 ? reinterpret_cast<const void*>(route_select_kernel<2>)
                                : reinterpret_cast<const void*>(route_select_kernel<4>);
    return launch_pdl(kb, T, 256, 0, st, logits, T, E, k, L, table, ids, w, n_shared, shared_w);
  }
  const int blocks = (T + 7) / 8;
  const void* kern = E <= 32    ? reinterpret_cast<const void*>(route_kernel<1>)
                     : E <= 128 ? reinterpret_cast<const void*>(route_kernel<4>)
                     : E <= 512 ? reinterpret_cast<const void*>(route_kernel<16>)
                                : reinterpret_cast<const void*>(route_kernel<32>);
  return launch_pdl(kern, blocks, 256, 0, st, logits, T, E, k, L, table, ids, w, n_shared, shared_w);
}

cudaError_t launch_route_sort_lookup(const float* logits, int E, int k, float L, const int32_t* table, int ns,
                                     const float* sw, int n_slots, int32_t* ids, float* w, int32_t* offsets,
                                     int32_t* pairs, int32_t* active, int32_t* n_active, int32_t* slots,
                                     int32_t* miss, int32_t* n_miss, int32_t* dev_err, cudaStream_t st,
                                     int32_t* host_meta, int32_t seq) {
  const void* kb = E <= 256 ? reinterpret_cast<const void*>(route_sort_lookup_kernel<1>)
                   : E <= 512 ? reinterpret_cast<const void*>(route_sort_lookup_kernel<2>)
                              : reinterpret_cast<const void*>(route_sort_lookup_kernel<4>);
  return launch_pdl(kb, 1, 256, 0, st, logits, E, k, L, table, ns, sw, n_slots, ids, w, offsets, pairs, active,
                    n_active, slots, miss, n_miss, dev_err, host_meta, seq);
}

size_t sort_ws_bytes(int n, int E) { return n <= 1024 ? 0 : (size_t)((n + 1023) / 1024) * E * sizeof(int32_t); }

cudaError_t launch_sort(const int32_t* ids, const uint16_t* x, int T, int k, int E, int H, int32_t* offsets,
                        int32_t* pairs, int32_t* active, int32_t* n_active, uint16_t* x_sorted, void* ws,
                        cudaStream_t st) {
  const int n = T * k;
  if (n <= 1024) {
    cudaError_t e = launch_pdl(reinterpret_cast<const void*>(sort_small_kernel), 1, 1024, 0, st, ids, n, E, offsets,
                               pairs, active, n_active);
    if (e != cudaSuccess) return e;
  } else {
    const int nchunk = (n + 1023) / 1024;
    int32_t* ch = static_cast<int32_t*>(ws);
    sort_hist_kernel<<<nchunk, 1024, 0, st>>>(ids, n, E, ch);
    sort_scan_kernel<<<1, 1024, 0, st>>>(ch, nchunk, n, E, offsets, active, n_active);
    sort_scatter_kernel<<<nchunk, 1024, 0, st>>>(ids, n, E, ch, pairs);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (x && x_sorted && n > 0) {
    gather_rows_kernel<<<(n + 7) / 8, 256, 0, st>>>(x, pairs, n, k, H, x_sorted);
    err = cudaGetLastError();
  }
  return err;
}

cudaError_t launch_lookup(const int32_t* table, const int32_t* active, const int32_t* n_active, int pass_begin,
                          int pass_len, int n_slots, int32_t* slots, int32_t* miss, int32_t* n_miss,
                          int32_t* dev_err, cudaStream_t st) {
  return launch_pdl(reinterpret_cast<const void*>(lookup_kernel), 1, 1024, 0, st, table, active, n_active, pass_begin,
                    pass_len, n_slots, slots, miss, n_miss, dev_err);
}

cudaError_t launch_exp(const float* x, int64_t n, float* out, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  exp_kernel<<<(int)blocks, 256, 0, st>>>(x, n, out);
  return cudaGetLastError();
}

}  // namespace moe
