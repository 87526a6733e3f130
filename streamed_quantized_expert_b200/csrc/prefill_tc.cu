// Expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM), fed by TMA:
// the grouped GEMM of a pass's experts over their sorted tokens, for prefill
// chunks and batched decode (above the fused decode kernel's range, when x sorted
// by expert is given).
//
// Two launches per pass of at most 64 experts (a longer pass runs as several),
// one persistent CTA per SM, each looping over tiles of (expert, 128 weight
// rows, up to 128 tokens):
//   gate/up: GU[rows, tokens] = deq(W_gu[e])[rows, H] . X_sorted[tokens, H]^T,
//            then h[token][j] = silu(gate_j) * up_j (bf16), j = intermediate;
//   down:    O[rows, tokens]  = deq(W_d[e])[rows, I] . h[tokens, I]^T,
//            o[pair][row] = O (fp32), summed per token by the combine kernel.
// The weight rows are the MMA's M side (the "swap AB" arrangement for grouped
// expert GEMMs: a token count per expert of tens to hundreds fits N, which
// steps by 16, where it would leave most of a 128-row M tile empty).
//
// Warp roles (832 threads):
//   0-15  dequant: warp w = (group w / 4, TMEM lane quadrant w % 4), lane =
//         weight row; for quantized codes the four warps of a group take whole
//         rows of every fourth 128-input block (landed by TMA): unpack the
//         row's codes once, w = fma(scale, q, bias) in fp16x2 with one
//         rounding, and store its 64 fp16 pairs to the A operand in TMEM with
//         four tcgen05.st (lane = row, column = input / 2); BF16 rows: warp w
//         converts K quarter w / 4 of its rows of every block;
//   16-23 epilogue: TMEM -> registers (warp i reads TMEM lanes 32 (i % 4)..;
//         the two warps of a quadrant take alternate 16-column chunks);
//   24    producer: TMA loads of codes, (scale, bias) words and token rows;
//   25    MMA issuer (one thread): tcgen05.mma kind::f16 (fp16 x fp16 -> fp32
//        in TMEM) with A from TMEM and B (token rows) from shared memory,
//        M = 128, N = tokens rounded up to 16, K = 16 per instruction;
//        tcgen05.commit frees stages and publishes accumulators.
// The operands are fp16 (11 significant bits): the token rows come sorted and
// converted by moe_sort, h is written in fp16 by the gate/up epilogue, and the
// weights are dequantised to fp16, so each rounding is 4x finer than bf16's.
// BF16 experts (16-bit slots: rows of bf16 values) take the same path: TMA
// brings 128 rows x 128 inputs with the 128-byte swizzle and the "dequant"
// warps convert each row's quarter to fp16 on its way into TMEM (exact for
// normal fp16 magnitudes).
// Accumulators are double-buffered in TMEM (2 x 128 columns), so the epilogue
// of one tile overlaps the MMAs of the next; the two A buffers take 2 x 64
// more columns.  With A in TMEM, shared memory carries only the TMA traffic
// and the MMA's B reads (the dequantised tile never goes through it).
//
// Every wait is bounded; a wait that runs out sets a CTA-wide abort flag and
// MOE_DEV_ERR_TIMEOUT, the roles leave their loops, the producer waits for
// the copies it issued, the MMA thread waits for its MMAs, and TMEM is freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "ffn_common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kPfBM = 128;      // weight rows per tile (MMA M)
constexpr int kPfBN = 128;      // tokens per tile (MMA N), at most; a launch takes 64 or 128
constexpr int kPfABufs = 4;     // dequantised A buffers (in TMEM)
constexpr int kPfDqWarps = 16;  // one per 8-row group of the 128-row tile
constexpr int kPfEpiWarps = 8;  // two per TMEM lane quadrant, taking alternate 16-column chunks
constexpr int kPfEpiWarp0 = kPfDqWarps, kPfProdWarp = kPfEpiWarp0 + kPfEpiWarps, kPfMmaWarp = kPfProdWarp + 1;
constexpr int kPfThreads = (kPfMmaWarp + 1) * 32;
constexpr int kPfTmemCols = 512;  // two accumulators of NB fp32 columns, then the A buffers
constexpr int kPfAcols = 64;       // one A buffer: 128 inputs as fp16 pairs, 128 lanes = rows
static_assert(2 * kPfBN + kPfABufs * kPfAcols <= kPfTmemCols, "TMEM columns");
static_assert(kPfABufs == 4 && kPfDqWarps == 16, "dequant warps: one group of four (one per TMEM lane quadrant) per A buffer");
// load stages (codes + scale/bias + token rows of NB rows) that fit the
// shared memory: a tile of at most 64 tokens has half the token bytes per
// stage, so its ring is deeper (the ring, not the arithmetic, paces the
// stages when the tokens per expert are few)
__host__ __device__ constexpr int pf_stages(int bits, int nb) {
  return nb == 64 ? (bits == 16 ? 4 : bits == 6 ? 7 : 8) : (bits == 16 ? 3 : bits == 6 ? 4 : 5);
}

struct PfEntry {
  int slot;    // slot of the expert (tiles skipped when not resident)
  int pos0;    // first sorted position of its tokens
  int cnt;     // tokens
  int tile0;   // first tile of the entry in the CTA-wide tile order
};

struct PfArgs {
  int T, k, H, I, g, E;
  int K;            // reduction length: H (gate/up) or I (down)
  int nkb;          // 128-input blocks of K
  int mtiles;       // 128-row tiles of the weight rows: 2I/128 or H/128
  int n_slots;
  const int32_t* table;
  const int32_t* active;
  const int32_t* n_active;
  const int32_t* offsets;
  const int32_t* pairs;
  int pass_begin, pass_len;
  uint16_t* h;      // [T*k][I] bf16 by sorted position (gate/up writes, down reads through its map)
  float* o;         // [T*k][H] fp32 by flat pair (down writes)
  int32_t* dev_err;
  long long wait_limit;  // clock-cycle limit of every bounded wait
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(tm), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
          "r"(smem_addr(dst)),
      "l"(tm), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* tm, int x, int y, int z, int w,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(smem_addr(dst)),
      "l"(tm), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tmap_prefetch(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tm) : "memory");
}

// Shared-memory matrix descriptor of a 128-byte swizzled K-major operand
// whose 8-row groups are 1024 bytes apart (rows of 64 bf16): start address
// >> 4 in bits 0-13, leading byte offset 16 B (unused by swizzled K-major) in
// bits 16-29, stride byte offset 1024 B in bits 32-45, descriptor version 1
// in bits 46-47, swizzle mode 2 (128 B) in bits 61-63.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and
// B fp16 (bits 7-9 = 0, bits 10-12 = 0), both K-major (bits 15, 16 = 0),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__device__ __forceinline__ uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D (TMEM, fp32) (+)= A . B^T, M x N x 16: A (M x 16 fp16: lane m, columns k / 2) in TMEM at a_tmem,
// B (N x 16 fp16, K-major, 128-byte swizzled) in shared memory; kind::f16.
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::
          "r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 TMEM lanes x 16 consecutive 32-bit columns: thread i of the warp gets
// lane (base lane + i), columns col..col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Thread i of the warp writes v to lane (base lane + i), columns col..col+15.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ bool slot_ok_pf(int n_slots, int slot) { return slot >= 0 && slot < n_slots; }

// Bounded wait that also gives up once another role of the CTA has aborted.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        long long limit_cycles) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity, 20000u)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit_cycles) {
      *abort_flag = 1;
      return false;
    }
  }
}

// BF16 experts: K quarter cq of row r from the stage's two 64-input halves
// (128 rows x 128 bytes each, 128-byte swizzle: 16-byte chunk c of row r sits
// at chunk c ^ (r % 8)), converted to fp16 pairs (pair index = TMEM column).
__device__ __forceinline__ void pf_bf16_quarter(int cq, const uint8_t* cs, uint32_t ta, int r) {
  const uint8_t* row = cs + (cq >> 1) * (128 * 128) + r * 128;
  uint32_t out[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = (cq & 1) * 4 + j;
    const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * (c ^ (r & 7)));
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u)
      out[4 * j + u] = (uint32_t)f32_to_f16_sat(bf16_lo(w4[u])) | ((uint32_t)f32_to_f16_sat(bf16_hi(w4[u])) << 16);
  }
  tmem_st16(ta + 16 * cq, out);
}

// The whole 128-input block of weight row r (0..127 of the tile) -> 64 fp16
// pairs at TMEM columns 0..63 of this thread's lane (ta: the warp's lanes, A
// buffer column 0).  Codes: the tile's 16 8-row groups, each 4 units x 8 rows
// x B words (unit t of row rr at word (8 t + sigma) B), loaded once;
// scale/bias: per 16-row tile, GPB groups of 16 words.  Pair i = 2 s + h' of
// unit t holds inputs 16 s + 2 t + 8 h' (+1), i.e. TMEM column 8 s + 4 h' + t:
// K quarter cq (inputs 32 cq .. 32 cq + 31, a single group) is pairs
// i = 4 cq + m of every unit, at columns 16 cq + 4 m + t.  Each weight is
// scale * q + bias in fp16 with one rounding: bf16 scale and bias -> fp16
// (exact for normal fp16 magnitudes), codes unpacked onto the fp16 magic 1024
// so that q = p - 1024 exactly.
template <int B, int GPB>
__device__ __forceinline__ void pf_dequant_row(const uint8_t* cs, const uint32_t* sbs, uint32_t ta, int r) {
  const int g8 = r >> 3, rr = r & 7;
  uint32_t w[4][B];
#pragma unroll
  for (int t = 0; t < 4; ++t) load_unit<B>(cs + (g8 * 32 + 8 * t + unit_sigma<B>(t, rr)) * 4 * B, w[t]);
  const uint32_t m = kMagic16;
  const __half2 m1024 = *reinterpret_cast<const __half2*>(&m);
#pragma unroll
  for (int cq = 0; cq < 4; ++cq) {
    const int gi = (cq * GPB) / 4;  // the quarter's (single) group within the block
    const uint32_t word = sbs[(r >> 4) * 16 * GPB + gi * 16 + (r & 15)];
    const float sf = bf16_lo(word), bf = bf16_hi(word);
    const __half2 sc = __half2half2(__float2half_rn(sf));
    const __half2 sc8 = __half2half2(__float2half_rn(sf * 0.125f));
    const __half2 bi = __half2half2(__float2half_rn(bf));
    uint32_t out[16];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint32_t p[16];
      unpack_unit<B, kMagic16>(w[t], p);
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) {
        const int i = 4 * cq + mm;
        const __half2 scale = PairShift<B>::a(i) == 3 ? sc8 : sc;
        const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&p[i]), m1024);
        const __half2 v = __hfma2(scale, q, bi);
        out[4 * mm + t] = *reinterpret_cast<const uint32_t*>(&v);
      }
    }
    tmem_st16(ta + 16 * cq, out);
  }
}

struct PfTile {
  int ent, mt, nt, n;  // entry, 128-row tile, token tile, tokens in the tile
  int slot, row0;      // slot; first sorted position of the tile's tokens
};

template <int B, int GPB, bool GU, int NB>
__global__ void __launch_bounds__(kPfThreads, 1)
    pf_gemm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_sb,
                   const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_b64,
                   const __grid_constant__ CUtensorMap tm_b128, const PfArgs a) {
  extern __shared__ uint8_t pf_smem_raw[];
  constexpr int kCodesBytes = 2048 * B;   // 16 groups x 4 units x 8 rows x B words (B = 16: 128 x 128 bf16)
  constexpr int kSbBytes = B == 16 ? 0 : 512 * GPB;  // 8 tiles x 16 GPB words
  constexpr int kPfStages = pf_stages(B, NB);
  constexpr int kXHalf = NB * 128;  // one 64-input half of a token stage: NB rows x 128 B
  constexpr int kAcol = 2 * NB;     // first TMEM column of the A buffers
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pf_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xst = base;                                           // [stage][2 halves][128 rows][128 B]
  uint8_t* cst = xst + kPfStages * 2 * kXHalf;                 // [stage] codes
  uint8_t* sbst = cst + kPfStages * kCodesBytes;                 // [stage] scale/bias words
  uint64_t* bars = reinterpret_cast<uint64_t*>(sbst + kPfStages * kSbBytes);
  uint64_t* full = bars;                        // producer (expect_tx) -> dequant, MMA
  uint64_t* empty = full + kPfStages;           // MMA commit -> producer
  uint64_t* afull = empty + kPfStages;          // dequant warps (TMEM stores done) -> MMA
  uint64_t* aempty = afull + kPfABufs;          // MMA commit -> dequant
  uint64_t* accfull = aempty + kPfABufs;        // MMA commit -> epilogue
  uint64_t* accempty = accfull + 2;             // epilogue threads -> MMA
  uint64_t* drain = accempty + 2;               // MMA commit at exit
  __shared__ PfEntry s_ent[kMaxCtaExperts];
  __shared__ int s_nent, s_ntiles;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  if (tid == 0) {
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kPfABufs; ++b) {
      // quantized codes: the four warps of the buffer's block group; BF16 rows: all sixteen
      mbar_init(&afull[b], B == 16 ? kPfDqWarps : kPfDqWarps / kPfABufs);
      mbar_init(&aempty[b], 1);
    }
    for (int c = 0; c < 2; ++c) {
      mbar_init(&accfull[c], 1);
      mbar_init(&accempty[c], kPfEpiWarps * 32);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    s_abort = 0;
  }
  if (warp == kPfMmaWarp) {  // TMEM: two accumulators of NB columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem)),
                 "r"(kPfTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == kPfProdWarp && lane == 0) {
    tmap_prefetch(&tm_q);
    tmap_prefetch(&tm_sb);
    tmap_prefetch(&tm_b);
    tmap_prefetch(&tm_b64);
    tmap_prefetch(&tm_b128);
  }
  pdl_wait();
  // the pass's experts and their tiles (token tiles x row tiles, row tile
  // fastest): the active list is read next to its length (one round), then
  // the experts' slots and token ranges (a second), and the tile offsets are a
  // warp scan
  if (warp == 0) {
    int cap = a.E - a.pass_begin;
    if (cap > a.pass_len) cap = a.pass_len;
    if (cap > kMaxCtaExperts) cap = kMaxCtaExperts;
    if (cap < 0) cap = 0;
    const int na = *a.n_active;
    int ev[2];
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) ev[qq] = lane + 32 * qq < cap ? a.active[a.pass_begin + lane + 32 * qq] : -1;
    int n = na - a.pass_begin;
    if (n > cap) n = cap;
    if (n < 0) n = 0;
    int tiles[2];
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
      const int i = lane + 32 * qq, e = ev[qq];
      const bool in = i < n && e >= 0 && e < a.E;
      PfEntry en;
      en.slot = in ? a.table[e] : -1;
      en.pos0 = in ? a.offsets[e] : 0;
      en.cnt = in ? a.offsets[e + 1] - en.pos0 : 0;
      tiles[qq] = slot_ok_pf(a.n_slots, en.slot) ? ((en.cnt + NB - 1) / NB) * a.mtiles : 0;
      if (i < n) {
        en.slot = (e >= 0 && e < a.E) ? en.slot : -1;
        s_ent[i] = en;
        if (blockIdx.x == 0 && !slot_ok_pf(a.n_slots, en.slot) && a.dev_err)
          atomicOr(a.dev_err, en.slot < 0 ? MOE_DEV_ERR_NOT_RESIDENT : MOE_DEV_ERR_SLOT_RANGE);
      }
    }
    // exclusive prefix of the tile counts over entries 0..63 (entry i = lane + 32 qq)
    int incl0 = tiles[0], incl1 = tiles[1];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u0 = __shfl_up_sync(0xffffffffu, incl0, o), u1 = __shfl_up_sync(0xffffffffu, incl1, o);
      if (lane >= o) {
        incl0 += u0;
        incl1 += u1;
      }
    }
    const int tot0 = __shfl_sync(0xffffffffu, incl0, 31);
    if (lane < n) s_ent[lane].tile0 = incl0 - tiles[0];
    if (lane + 32 < n) s_ent[lane + 32].tile0 = tot0 + incl1 - tiles[1];
    const int total = tot0 + __shfl_sync(0xffffffffu, incl1, 31);
    if (lane == 0) {
      s_nent = n;
      s_ntiles = total;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  const int nent = s_nent, ntiles = s_ntiles;
  // tile t's entry: each role visits its tiles in increasing order, so the
  // scan resumes from the entry of the role's previous tile (hint)
  auto tile_at = [&](int t, int& hint) -> PfTile {
    int i = hint;
    while (i + 1 < nent && s_ent[i + 1].tile0 <= t) ++i;
    hint = i;
    const PfEntry en = s_ent[i];
    const int local = t - en.tile0;
    PfTile tl;
    tl.ent = i;
    tl.nt = local / a.mtiles;
    tl.mt = local - tl.nt * a.mtiles;
    tl.n = en.cnt - tl.nt * NB < NB ? en.cnt - tl.nt * NB : NB;
    tl.slot = en.slot;
    tl.row0 = en.pos0 + tl.nt * NB;
    return tl;
  };

  if (warp == kPfProdWarp) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int s = 0, ent_hint = 0;
      uint32_t ph = 0, issued = 0, last_ph = 0;  // per-stage bit masks for the exit drain
      for (int t = blockIdx.x; t < ntiles && !s_abort; t += gridDim.x) {
        const PfTile tl = tile_at(t, ent_hint);
        // the tile's token rows: one box of 32, 64 or 128 rows per 64-column half
        // (rows past the expert's tokens are loaded and never read by the MMA)
        const int brows = tl.n <= 32 ? 32 : tl.n <= 64 ? 64 : 128;
        const CUtensorMap* tmb = brows == 32 ? &tm_b : brows == 64 ? &tm_b64 : &tm_b128;
        const uint32_t bytes = kCodesBytes + kSbBytes + (uint32_t)brows * 2 * 128;
        bool ok = true;
        for (int kb = 0; kb < a.nkb; ++kb) {
          if (!pf_wait(&empty[s], ph ^ 1u, &s_abort, a.wait_limit)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], bytes);
          if constexpr (B == 16) {  // (input, row, slot) boxes of 64 x 128 x 1
            tma_load_3d(cst + s * kCodesBytes, &tm_q, kb * 128, tl.mt * kPfBM, tl.slot, &full[s]);
            tma_load_3d(cst + s * kCodesBytes + 128 * 128, &tm_q, kb * 128 + 64, tl.mt * kPfBM, tl.slot, &full[s]);
          } else {
            tma_load_4d(cst + s * kCodesBytes, &tm_q, kb * 32 * B, 0, tl.mt * 8, tl.slot, &full[s]);
            tma_load_3d(sbst + s * kSbBytes, &tm_sb, kb * 16 * GPB, tl.mt * 8, tl.slot, &full[s]);
          }
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            tma_load_2d(xst + (s * 2 + hf) * kXHalf, tmb, kb * 128 + hf * 64, tl.row0, &full[s]);
          issued |= 1u << s;
          last_ph = (last_ph & ~(1u << s)) | (ph << s);
          if (++s == kPfStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
      }
      // every copy issued lands before the CTA can exit
      for (int q = 0; q < kPfStages; ++q)
        if ((issued >> q) & 1u) mbar_wait_bounded(&full[q], (last_ph >> q) & 1u, a.wait_limit);
    }
  } else if (warp == kPfMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int s = 0, ab = 0, c = 0, ent_hint = 0;
      uint32_t ph = 0, pa = 0, pc = 0;
      bool issued_any = false;
      for (int t = blockIdx.x; t < ntiles && !s_abort; t += gridDim.x) {
        const PfTile tl = tile_at(t, ent_hint);
        const int npad = (tl.n + 15) & ~15;
        const uint32_t idesc = idesc_f16(kPfBM, npad);
        if (!pf_wait(&accempty[c], pc ^ 1u, &s_abort, a.wait_limit)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(c * NB);
        bool ok = true;
        for (int kb = 0; kb < a.nkb; ++kb) {
          // operands of the block's 8 MMAs, formed before the waits so that
          // the issue loop is the MMAs alone (the thread shares its
          // sub-partition's issue slots with the dequant warps)
          const uint32_t a_tm = tmem_base + (uint32_t)(kAcol + ab * kPfAcols);
          const uint64_t bd0 = sw128_desc(smem_addr(xst + s * 2 * kXHalf));  // + (offset >> 4): no carry (< 2^18 B)
          const uint32_t acc0 = kb != 0 ? 1u : 0u;
          if (!pf_wait(&full[s], ph, &s_abort, a.wait_limit) || !pf_wait(&afull[ab], pa, &s_abort, a.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            umma_bf16_ta(d, a_tm + 8 * k16, bd0 + (uint64_t)(((k16 >> 2) * kXHalf + (k16 & 3) * 32) >> 4), idesc,
                         k16 != 0 ? 1u : acc0);
          issued_any = true;
          umma_commit(&empty[s]);
          umma_commit(&aempty[ab]);
          if (++s == kPfStages) {
            s = 0;
            ph ^= 1u;
          }
          if (++ab == kPfABufs) {
            ab = 0;
            pa ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&accfull[c]);
        if (++c == 2) {
          c = 0;
          pc ^= 1u;
        }
      }
      if (issued_any) {  // every MMA issued completes before TMEM is freed
        umma_commit(drain);
        mbar_wait_bounded(drain, 0, a.wait_limit);
      }
    }
  } else if (warp < kPfDqWarps) {
    // ---------------- dequant ----------------
    // Quantized codes: warp = (block group sel, TMEM lane quadrant q), lane =
    // weight row; the four warps of group sel dequantise whole rows of every
    // fourth block of the CTA's block sequence (block b when b % 4 == sel)
    // into A buffer sel, so a row's code words are loaded once and four blocks
    // are in flight.  BF16 rows (nothing to unpack, nothing loaded twice):
    // every warp takes K quarter sel of its quadrant's rows of every block.
    constexpr bool kRowGroups = B != 16;
    const int q = warp & 3, sel = warp >> 2, r = 32 * q + lane;
    int b = 0;  // position in the CTA's block sequence
    for (int t = blockIdx.x; t < ntiles && !s_abort; t += gridDim.x) {
      bool ok = true;
      for (int kb = 0; kb < a.nkb; ++kb, ++b) {
        if (kRowGroups && (b & (kPfABufs - 1)) != sel) continue;
        const int s = b % kPfStages, ab = b & (kPfABufs - 1);
        const uint32_t ph = (uint32_t)((b / kPfStages) & 1), pa = (uint32_t)((b / kPfABufs) & 1);
        if (!pf_wait(&full[s], ph, &s_abort, a.wait_limit) || !pf_wait(&aempty[ab], pa ^ 1u, &s_abort, a.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(kAcol + ab * kPfAcols);
        if constexpr (B == 16)
          pf_bf16_quarter(sel, cst + s * kCodesBytes, ta, r);
        else
          pf_dequant_row<B, GPB>(cst + s * kCodesBytes, reinterpret_cast<const uint32_t*>(sbst + s * kSbBytes), ta, r);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[ab]);
      }
      if (!ok) break;
    }
  } else {
    // ---------------- epilogue (TMEM lanes 32 (warp % 4) ..) ----------------
    const int q = warp & 3, r = 32 * q + lane, eh = (warp - kPfEpiWarp0) >> 2;  // quadrant, row, chunk parity
    int c = 0, ent_hint = 0;
    uint32_t pc = 0;
    for (int t = blockIdx.x; t < ntiles && !s_abort; t += gridDim.x) {
      const PfTile tl = tile_at(t, ent_hint);
      if (!pf_wait(&accfull[c], pc, &s_abort, a.wait_limit)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(c * NB);
      // the tile's pair indices (down) in registers: lane l holds columns l, 32 + l, ...
      int pidx[NB / 32];
      if (!GU) {
#pragma unroll
        for (int q4 = 0; q4 < NB / 32; ++q4)
          pidx[q4] = 32 * q4 + lane < tl.n ? a.pairs[tl.row0 + 32 * q4 + lane] : 0;
      }
      const bool gate = (r & 15) < 8;  // storage rows: 16-row blocks of 8 gate rows then 8 up rows
      const int j = tl.mt * (kPfBM / 2) + (r >> 4) * 8 + (r & 7);
      const int row = tl.mt * kPfBM + r;
#pragma unroll
      for (int nb = 0; nb < NB / 32; ++nb) {
        if (32 * nb >= tl.n) break;
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          const int n0 = 32 * nb + 16 * hb;
          if (n0 >= tl.n) break;
          if (hb != eh) continue;  // the other warp of this quadrant takes this chunk
          uint32_t v[16];
          tmem_ld16(taddr + (uint32_t)n0, v);
          tmem_ld_wait();
          if (GU) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float x = __uint_as_float(v[i]);
              const float u = __shfl_xor_sync(0xffffffffu, x, 8);
              if (gate && n0 + i < tl.n)
                a.h[(int64_t)(tl.row0 + n0 + i) * a.I + j] = f32_to_f16_sat(__fdividef(x, 1.0f + __expf(-x)) * u);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int pf = __shfl_sync(0xffffffffu, pidx[nb], 16 * hb + i);
              if (n0 + i < tl.n) a.o[(int64_t)pf * a.H + row] = __uint_as_float(v[i]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&accempty[c]);
      if (++c == 2) {
        c = 0;
        pc ^= 1u;
      }
    }
  }
  pdl_launch_dependents();
  if (s_abort && tid == 0 && a.dev_err) atomicOr(a.dev_err, MOE_DEV_ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kPfMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kPfTmemCols)
                 : "memory");
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* addr, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
  const auto fn = tmap_encoder();
  if (!fn) return false;
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(m, dt, (cuuint32_t)rank, const_cast<void*>(addr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Maps of one projection of the pool: codes as 32-bit words (8-row group
// words, half, 16-row tile, slot) and the (scale, bias) words (tile words,
// tile, slot); a box is one 128-input block of a 128-row tile.
bool encode_proj(CUtensorMap* q, CUtensorMap* sb, const uint8_t* proj, int64_t rb, int64_t tile, int ng, int rows,
                 int bits, int gpb, int64_t slot_bytes, int n_slots) {
  const cuuint64_t qd[4] = {(cuuint64_t)(2 * rb), 2, (cuuint64_t)(rows / 16), (cuuint64_t)n_slots};
  const cuuint64_t qs[3] = {(cuuint64_t)(8 * rb), (cuuint64_t)tile, (cuuint64_t)slot_bytes};
  const cuuint32_t qb[4] = {(cuuint32_t)(32 * bits), 2, 8, 1};
  if (!encode(q, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, proj, qd, qs, qb, CU_TENSOR_MAP_SWIZZLE_NONE)) return false;
  const cuuint64_t sd[3] = {(cuuint64_t)(16 * ng), (cuuint64_t)(rows / 16), (cuuint64_t)n_slots};
  const cuuint64_t ss[2] = {(cuuint64_t)tile, (cuuint64_t)slot_bytes};
  const cuuint32_t sbx[3] = {(cuuint32_t)(16 * gpb), 8, 1};
  return encode(sb, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, proj + 16 * rb, sd, ss, sbx, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// BF16 experts: a projection's rows of bf16 values as (input, row, slot),
// boxes of 64 inputs (128 bytes, 128-byte swizzle) x 128 rows x 1 slot.
bool encode_proj_bf16(CUtensorMap* q, const uint8_t* proj, int64_t kp, int rows, int64_t slot_bytes, int n_slots) {
  const cuuint64_t d[3] = {(cuuint64_t)kp, (cuuint64_t)rows, (cuuint64_t)n_slots};
  const cuuint64_t st[2] = {(cuuint64_t)kp * 2, (cuuint64_t)slot_bytes};
  const cuuint32_t b[3] = {64, (cuuint32_t)kPfBM, 1};
  return encode(q, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, proj, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Token rows (fp16 [rows][cols], row-major) for the MMA's B operand: boxes of
// 64 columns (128 bytes, 128-byte swizzle) x box_rows rows.
bool encode_rows(CUtensorMap* m, const uint16_t* base, int64_t rows, int cols, int box_rows) {
  const cuuint64_t d[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t s[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t b[2] = {64, (cuuint32_t)box_rows};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, d, s, b, CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t pf_smem_bytes(int bits, int gpb, int nb) {
  const size_t ns = (size_t)pf_stages(bits, nb);
  return 1024 + ns * 2 * (size_t)nb * 128 + ns * 2048 * bits + (bits == 16 ? 0 : ns * 512 * gpb) +
         (2 * ns + 2 * kPfABufs + 5) * 8;
}

template <int B, int GPB, bool GU, int NB>
cudaError_t launch_pf_t(const CUtensorMap& q, const CUtensorMap& sb, const CUtensorMap (&bm)[3], const PfArgs& pa,
                        int grid, cudaStream_t st) {
  static int done[4] = {0, 0, 0, 0};
  const void* kern = reinterpret_cast<const void*>(pf_gemm_kernel<B, GPB, GU, NB>);
  const size_t smem = pf_smem_bytes(B, GPB, NB);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev >= 128) return cudaErrorNotSupported;
  if (!((__atomic_load_n(&done[dev >> 5], __ATOMIC_RELAXED) >> (dev & 31)) & 1)) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&done[dev >> 5], 1 << (dev & 31), __ATOMIC_RELAXED);
  }
  return launch_pdl(kern, grid, kPfThreads, smem, st, q, sb, bm[0], bm[1], bm[2], pa);
}

template <int B, bool GU, int NB>
cudaError_t launch_pf_gpb(int gpb, const CUtensorMap& q, const CUtensorMap& sb, const CUtensorMap (&bm)[3],
                          const PfArgs& pa, int grid, cudaStream_t st) {
  if (gpb == 1) return launch_pf_t<B, 1, GU, NB>(q, sb, bm, pa, grid, st);
  if (gpb == 2) return launch_pf_t<B, 2, GU, NB>(q, sb, bm, pa, grid, st);
  return launch_pf_t<B, 4, GU, NB>(q, sb, bm, pa, grid, st);
}

template <bool GU, int NB>
cudaError_t launch_pf_nb(int bits, int gpb, const CUtensorMap& q, const CUtensorMap& sb, const CUtensorMap (&bm)[3],
                         const PfArgs& pa, int grid, cudaStream_t st) {
  if (bits == 3) return launch_pf_gpb<3, GU, NB>(gpb, q, sb, bm, pa, grid, st);
  if (bits == 4) return launch_pf_gpb<4, GU, NB>(gpb, q, sb, bm, pa, grid, st);
  if (bits == 16) return launch_pf_t<16, 1, GU, NB>(q, sb, bm, pa, grid, st);
  return launch_pf_gpb<6, GU, NB>(gpb, q, sb, bm, pa, grid, st);
}

template <bool GU>
cudaError_t launch_pf(int bits, int gpb, int nb, const CUtensorMap& q, const CUtensorMap& sb,
                      const CUtensorMap (&bm)[3], const PfArgs& pa, int grid, cudaStream_t st) {
  return nb == 64 ? launch_pf_nb<GU, 64>(bits, gpb, q, sb, bm, pa, grid, st)
                  : launch_pf_nb<GU, 128>(bits, gpb, q, sb, bm, pa, grid, st);
}

}  // namespace

bool ffn_prefill_tc_shape_ok(const moe_layer_desc& d) {
  return d.H % 128 == 0 && d.I % 128 == 0 && (d.group == 32 || d.group == 64 || d.group == 128) &&
         tmap_encoder() != nullptr;
}

static bool ffn_prefill_tc_supported(const FfnArgs& a, const moe_layer_desc& d) {
  return a.x_sorted != nullptr && a.o != nullptr && a.n_slots > 0 && ffn_prefill_tc_shape_ok(d);
}

// gate/up + SwiGLU -> h, down -> o (per pair), combine -> y; returns
// cudaErrorNotSupported when the shapes or inputs do not fit this path.
cudaError_t launch_ffn_prefill_tc(const FfnArgs& a, const moe_layer_desc& d, int num_sms, cudaStream_t st) {
  if (!ffn_prefill_tc_supported(a, d)) return cudaErrorNotSupported;
  const Layout& L = a.L;
  const int gpb = 128 / d.group;
  const int64_t np = (int64_t)a.T * d.k;
  CUtensorMap q_gu, sb_gu, q_d, sb_d, xm[3], hm[3];
  auto proj_maps = [&](CUtensorMap* q, CUtensorMap* sb, int64_t off, int64_t rb, int64_t tile, int ng, int rows,
                       int bits, int64_t K) {
    if (bits == 16) {
      *sb = CUtensorMap{};  // no scale/bias words
      return encode_proj_bf16(q, a.pool + off, padded_k(K), rows, L.slot_bytes, a.n_slots);
    }
    return encode_proj(q, sb, a.pool + off, rb, tile, ng, rows, bits, gpb, L.slot_bytes, a.n_slots);
  };
  if (!proj_maps(&q_gu, &sb_gu, L.gu, L.rb_gu, L.tile_gu, L.ng_gu, 2 * d.I, d.bits_gu, d.H) ||
      !proj_maps(&q_d, &sb_d, L.d, L.rb_d, L.tile_d, L.ng_d, d.H, d.bits_down, d.I) ||
      !encode_rows(&xm[0], a.x_sorted, np, d.H, 32) || !encode_rows(&xm[1], a.x_sorted, np, d.H, 64) ||
      !encode_rows(&xm[2], a.x_sorted, np, d.H, 128) || !encode_rows(&hm[0], a.h, np, d.I, 32) ||
      !encode_rows(&hm[1], a.h, np, d.I, 64) || !encode_rows(&hm[2], a.h, np, d.I, 128))
    return cudaErrorInvalidValue;
  PfArgs pa{};
  pa.T = a.T;
  pa.k = d.k;
  pa.H = d.H;
  pa.I = d.I;
  pa.g = d.group;
  pa.E = d.E;
  pa.n_slots = a.n_slots;
  pa.table = a.table;
  pa.active = a.active;
  pa.n_active = a.n_active;
  pa.offsets = a.offsets;
  pa.pairs = a.pairs;
  pa.pass_begin = a.pass_begin;
  pa.pass_len = a.pass_len;
  pa.h = a.h;
  pa.o = a.o;
  pa.dev_err = a.dev_err;
  pa.wait_limit = a.wait_limit;
  const int grid = num_sms;
  // tokens per tile: 64 when an expert averages at most 48 of the chunk's
  // pairs (the deeper load ring pays more than the second token tile of a
  // crowded expert costs), else 128
  const int nb = np <= 48LL * d.E ? 64 : 128;
  // a CTA's tile table holds kMaxCtaExperts experts: longer passes run as
  // several gate/up + down launches over consecutive sub-ranges (sub-ranges
  // past the active list find no experts), then one combine over the pass
  const int pass_end = a.pass_len < d.E - a.pass_begin ? a.pass_begin + a.pass_len : d.E;
  for (int pb = a.pass_begin; pb < pass_end; pb += kMaxCtaExperts) {
    pa.pass_begin = pb;
    pa.pass_len = pass_end - pb < kMaxCtaExperts ? pass_end - pb : kMaxCtaExperts;
    pa.K = d.H;
    pa.nkb = L.nblk_gu;
    pa.mtiles = 2 * d.I / kPfBM;
    cudaError_t e = launch_pf<true>(d.bits_gu, gpb, nb, q_gu, sb_gu, xm, pa, grid, st);
    if (e != cudaSuccess) return e;
    pa.K = d.I;
    pa.nkb = L.nblk_d;
    pa.mtiles = d.H / kPfBM;
    e = launch_pf<false>(d.bits_down, gpb, nb, q_d, sb_d, hm, pa, grid, st);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(reinterpret_cast<const void*>(combine_kernel), combine_grid(a.T, d.H, num_sms), 256, 0, st, a);
}

}  // namespace moe
