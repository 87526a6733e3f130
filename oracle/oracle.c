/*
 * Oracle for the streamed, quantized routed-expert FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * CPU statement of what the GPU path computes.  Only the test-suite, the
 * package smoke check and the CPU-baseline leg of the benchmark may load it.
 * It shares no code, header or constant table with the CUDA library; the two
 * meet only on the byte layouts written down below and in the ABI header.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no contraction: every float operation below rounds exactly once, in the
 * order written).
 *
 * Sources (web pages on expert offload for MoE models):
 *  - "RFC: stream MoE experts from disk in from_pretrained", section "How the
 *    prototype works": one device pool of expert slots shared by all layers,
 *    a per-layer expert->slot table, quantized experts in MLX's affine format
 *    with one contiguous row per expert, experts that are "gated,
 *    concatenated, untransposed, no bias", sorted prefill in groups of 64
 *    experts.
 *  - huggingface/transformers PR #50717 "POC: Experts offload", commit notes:
 *    the expert->slot tables live on the host; sorted prefill runs 64 experts
 *    at a time.
 *  - BigMoeOnEdge, commit note on cache-aware substitution: before a decode
 *    routing is committed, every expert already in the cache gets its score
 *    raised by L times the token's score range and the top-k is taken again;
 *    the same number of experts runs.
 *  - 1bit-MONSTER engine PR #137 "expert slots in size classes": layers are
 *    grouped by the bytes one expert needs (the sum of its aligned read
 *    windows); each group has its own slots and LRU; empty slots are taken
 *    first.
 *
 * Readings of the pages (where they are silent) are stated at each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32                                                        */
/* ------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round-to-nearest-even from fp32 to bf16 (NaN kept quiet). */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* exp for routing: one fixed sequence of fp32 operations                */
/* ------------------------------------------------------------------ */
/*
 * The routing scores are softmax probabilities (BigMoeOnEdge note: "score
 * range", "top-k is taken again").  Which experts win is decided by comparing
 * floats, so the GPU and this oracle must evaluate exp identically.  The
 * function is written from its mathematics, not from any vendor library:
 *   Cody & Waite range reduction  x = n*ln2 + r,  n = rint(x*log2(e)),
 *   with ln2 split into hi (15 significant bits) + lo, both applied by fma;
 *   e^r by the degree-7 Taylor polynomial in Horner form (fma per step);
 *   scaling by 2^n through the exponent field.
 * Domain: x <= 0 (inputs are l - max l).  x < -87 returns 0 (e^-87 is still
 * a normal float, so every returned value is normal).
 */
#define ORC_LOG2E 0x1.715476p+0f
#define ORC_LN2_HI 0x1.62e400p-1f  /* 0.693145751953125 */
#define ORC_LN2_LO 0x1.7f7d1cp-20f /* ln2 - ln2_hi rounded to float */

float orc_exp_portable(float x) {
  if (!(x >= -87.0f)) return 0.0f;
  if (x > 0.0f) x = 0.0f;
  float n = rintf(x * ORC_LOG2E);
  float r = fmaf(-n, ORC_LN2_HI, x);
  r = fmaf(-n, ORC_LN2_LO, r);
  /* Taylor coefficients 1/k!, k = 7..0, each rounded to float */
  float p = 0x1.a01a02p-13f;      /* 1/5040 */
  p = fmaf(p, r, 0x1.6c16c2p-10f); /* 1/720 */
  p = fmaf(p, r, 0x1.111112p-7f);  /* 1/120 */
  p = fmaf(p, r, 0x1.555556p-5f);  /* 1/24 */
  p = fmaf(p, r, 0x1.555556p-3f);  /* 1/6 */
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  int32_t ni = (int32_t)n; /* in [-126, 0] */
  uint32_t bits = (uint32_t)(ni + 127) << 23;
  float s;
  memcpy(&s, &bits, 4);
  return p * s;
}

void orc_exp_portable_range(const float* x, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_exp_portable(x[i]);
}

/* Every float in [lo_bits .. hi_bits] interpreted as negative floats walking
 * from -0 downward: out[i] = exp(float with bits (0x80000000 | (start + i))). */
void orc_exp_portable_neg_bits(uint32_t start, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) {
    uint32_t b = 0x80000000u | (start + (uint32_t)i);
    float x;
    memcpy(&x, &b, 4);
    out[i] = orc_exp_portable(x);
  }
}

/* ------------------------------------------------------------------ */
/* Stage 1: route_topk (+ cache-aware substitution)                      */
/* ------------------------------------------------------------------ */
/*
 * Per token t:
 *   u_e  = exp(l_e - max_e l)                     (softmax up to its sum)
 *   with L > 0 (decode only):  u'_e = u_e + L * (1 - min_e u) * [e resident]
 *     (1 - min u is the token's score range in u units: max u = exp(0) = 1;
 *      the boost scales with the softmax sum, so selecting on u' selects the
 *      same experts as boosting the normalised softmax)
 *   top-k by the key (u' desc, l desc, e asc)
 *   w_j = u_{e_j} / sum_j u_{e_j}    (the unboosted scores: substitution
 *     changes which experts run, not how they are weighted)
 * Readings (the note does not spell these out): the score range is taken
 * over all E experts of the token; "resident" is slot_table[e] >= 0 before
 * this step's installs, the same mask for every token of the call.
 * Every comparison uses the fp32 values; the weights are formed in double.
 */
void orc_route(const float* logits, int32_t T, int32_t E, int32_t k, float L, const int32_t* slot_table,
               int32_t* ids, double* w, float* u_out) {
  float* u = (float*)malloc(sizeof(float) * (size_t)E);
  float* up = (float*)malloc(sizeof(float) * (size_t)E);
  unsigned char* taken = (unsigned char*)malloc((size_t)E);
  for (int32_t t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    float lmax = l[0];
    for (int32_t e = 1; e < E; ++e)
      if (l[e] > lmax) lmax = l[e];
    for (int32_t e = 0; e < E; ++e) u[e] = orc_exp_portable(l[e] - lmax);
    if (L > 0.0f && slot_table) {
      float umin = u[0];
      for (int32_t e = 1; e < E; ++e)
        if (u[e] < umin) umin = u[e];
      float range = 1.0f - umin;
      float boost = L * range;
      for (int32_t e = 0; e < E; ++e) up[e] = (slot_table[e] >= 0) ? (u[e] + boost) : u[e];
    } else {
      for (int32_t e = 0; e < E; ++e) up[e] = u[e];
    }
    memset(taken, 0, (size_t)E);
    for (int32_t j = 0; j < k; ++j) {
      int32_t best = -1;
      for (int32_t e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || up[e] > up[best] || (up[e] == up[best] && l[e] > l[best])) best = e;
        /* equal (u', l): the lower id was met first and stays */
      }
      taken[best] = 1;
      ids[(size_t)t * k + j] = best;
    }
    double sum = 0.0;
    for (int32_t j = 0; j < k; ++j) sum += (double)u[ids[(size_t)t * k + j]];
    for (int32_t j = 0; j < k; ++j) w[(size_t)t * k + j] = (double)u[ids[(size_t)t * k + j]] / sum;
    if (u_out) memcpy(u_out + (size_t)t * E, u, sizeof(float) * (size_t)E);
  }
  free(u);
  free(up);
  free(taken);
}

/* ------------------------------------------------------------------ */
/* Stage 2: moe_sort                                                     */
/* ------------------------------------------------------------------ */
/*
 * Tokens grouped by expert (transformers PR #50717 notes; RFC "Prefill").
 * The T*k (token, rank) pairs are identified by their flat index t*k + j.
 * Stable counting sort by expert: key expert ascending, ties by flat index.
 *   offsets[e] = number of pairs routed to experts < e   (offsets[E] = T*k)
 *   pairs[offsets[e] ..] = flat indices routed to e, ascending
 *   active = experts with at least one pair, ascending; *n_active = count
 * Prefill pass p covers active[64p .. 64p+64).
 */
void orc_sort(const int32_t* ids, int32_t T, int32_t k, int32_t E, int32_t* offsets, int32_t* pairs,
              int32_t* active, int32_t* n_active) {
  int64_t n = (int64_t)T * k;
  int32_t* count = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  for (int64_t i = 0; i < n; ++i) count[ids[i]] += 1;
  int32_t run = 0;
  for (int32_t e = 0; e < E; ++e) {
    offsets[e] = run;
    pos[e] = run;
    run += count[e];
  }
  offsets[E] = run;
  for (int64_t i = 0; i < n; ++i) pairs[pos[ids[i]]++] = (int32_t)i;
  int32_t na = 0;
  for (int32_t e = 0; e < E; ++e)
    if (count[e] > 0) active[na++] = e;
  *n_active = na;
  free(count);
  free(pos);
}

/* ------------------------------------------------------------------ */
/* Stage 3: expert -> slot lookup                                        */
/* ------------------------------------------------------------------ */
/*
 * RFC "How the prototype works": a per-layer expert -> slot table over one
 * preallocated pool.  For the pass [pass_begin, pass_begin + pass_len) of the
 * active list (clipped to n_active):
 *   slots[i] = table[active[pass_begin + i]]   (-1 = not resident)
 *   miss     = the pass's experts whose slot is -1, ascending
 * Returns 1 in *bad if a slot id is >= n_slots (corrupt table), else 0.
 */
void orc_slot_lookup(const int32_t* table, const int32_t* active, int32_t n_active, int32_t pass_begin,
                     int32_t pass_len, int32_t n_slots, int32_t* slots, int32_t* miss, int32_t* n_miss,
                     int32_t* bad) {
  int32_t end = pass_begin + pass_len;
  if (end > n_active) end = n_active;
  int32_t nm = 0;
  *bad = 0;
  for (int32_t i = pass_begin; i < end; ++i) {
    int32_t s = table[active[i]];
    slots[i - pass_begin] = s;
    if (s < 0) miss[nm++] = active[i];
    else if (s >= n_slots) *bad = 1;
  }
  *n_miss = nm;
}

/* ------------------------------------------------------------------ */
/* Slot format                                                           */
/* ------------------------------------------------------------------ */
/*
 * The RFC says only "MLX's affine format, one contiguous row per expert".
 * Bit layout (a reading; the pages give none):
 *
 * A weight row of K inputs is padded to Kp = K rounded up to 128; padded
 * groups have scale = bias = 0 (so they dequantise to exactly 0).  The row is
 * cut into blocks of 128 inputs; block B is 4 units, unit p in 0..3, each unit
 * 32 codes in b 32-bit little-endian words (4b bytes).  Unit p of block B
 * holds, for s = 0..7, the two input pairs
 *     (128B + 16s + 2p,     +1)      -> pair index i = 2s
 *     (128B + 16s + 2p + 8, +1)      -> pair index i = 2s + 1
 * The even input of a pair sits in the low 16-bit half of a word, the odd
 * input at the same bit offset in the high half (bit + 16).  Within a unit:
 *   b = 4: pair i in word i/4 at bits 4*(i%4) .. +3
 *   b = 3: pair i < 15 in word i/5 at bits 3*(i%5) .. +2;
 *          pair 15: code bit j (j = 0,1,2) is bit 15 of word j
 *   b = 6: pair i < 12 in word i/2 at bits 6*(i%2) .. +5;
 *          pair i >= 12, m = i - 12: code bits 0..3 at bits 12..15 of
 *          word m; code bits 4,5 at bits 12 + 2*(m%2) + {0,1} of word 4+m/2
 * Rows are stored in tiles of 16 consecutive rows.  A tile is the rows'
 * codes (16 * row_bytes bytes) followed by their (scale, bias) words (16 *
 * Kp/g words); consecutive tiles are adjacent.  Codes: the tile's rows form
 * two groups of 8 (rows 0-7, rows 8-15), each 8 * row_bytes bytes; inside a
 * group, unit u (= 4B + p) of row r (0..7) sits at unit position
 * 8u + sigma(u, r) (unit positions are 4b bytes apart), with
 *   b = 3: sigma = r
 *   b = 4: sigma = (r + 2 (u mod 4)) mod 8
 *   b = 6: sigma = (r + 4 ((u / 2) mod 2)) mod 8
 * Scale/bias: per group of g inputs a (scale, bias) pair of bf16 in one
 * 32-bit word, scale in the low half; inside a tile group-major: the word of
 * (row r, group gi) is word gi*16 + r.
 *
 * A slot (one expert) is two projections, each starting on a 256-byte
 * boundary: gate_up (2I rows; row order: blocks of 16, block m = gate rows
 * 8m..8m+7 then up rows 8m..8m+7, so tile m is one block) then down (H rows).
 * The slot's byte size is the end rounded to 256 -- the "sum of its aligned
 * read windows" that keys its size class (1bit-MONSTER PR #137).
 */
static int64_t orc_round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

/* b = 16: unquantized BF16 experts (RFC "stream MoE experts from disk in
 * from_pretrained", "How the prototype works", item "Cache": BF16 experts run
 * through the grouped experts kernel).  Reading: a BF16 projection is its
 * rows of K bf16 values, row-major, each row padded to a multiple of 128
 * inputs with zeros, rows in the same storage order as the quantized formats,
 * no scale/bias words. */
int orc_bits_supported(int32_t b) { return b == 3 || b == 4 || b == 6 || b == 16; }

int64_t orc_row_bytes(int32_t K, int32_t b) { return orc_round_up(K, 128) * b / 8; }

int64_t orc_row_groups(int32_t K, int32_t g) { return orc_round_up(K, 128) / g; }

/* Bytes of one 16-row tile of a projection with K inputs per row. */
int64_t orc_tile_bytes(int32_t K, int32_t g, int32_t b) {
  return 16 * orc_row_bytes(K, b) + (b == 16 ? 0 : 16 * orc_row_groups(K, g) * 4);
}

/* off[0] = gate_up projection, off[1] = down projection, off[2] = gate_up
 * tile bytes, off[3] = down tile bytes, off[4] = slot bytes. */
void orc_slot_layout(int32_t H, int32_t I, int32_t g, int32_t b_gu, int32_t b_d, int64_t* off) {
  int64_t o = 0;
  off[0] = 0;
  o += (int64_t)(2 * I / 16) * orc_tile_bytes(H, g, b_gu);
  o = orc_round_up(o, 256);
  off[1] = o;
  o += (int64_t)(H / 16) * orc_tile_bytes(I, g, b_d);
  o = orc_round_up(o, 256);
  off[2] = orc_tile_bytes(H, g, b_gu);
  off[3] = orc_tile_bytes(I, g, b_d);
  off[4] = o; /* slot bytes */
}

static uint32_t orc_load_word(const uint8_t* p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}

static void orc_store_word(uint8_t* p, uint32_t v) {
  p[0] = (uint8_t)v;
  p[1] = (uint8_t)(v >> 8);
  p[2] = (uint8_t)(v >> 16);
  p[3] = (uint8_t)(v >> 24);
}

/* Position of code bit j of input k of row `row` of a projection (rows of
 * row_bytes code bytes, tiles of tile_bytes): byte offset of its 32-bit word
 * from the projection's start, and the bit inside that word. */
static void orc_code_bit(int32_t row, int64_t row_bytes, int64_t tile_bytes, int32_t k, int32_t b, int32_t j,
                         int64_t* word_byte, int32_t* bit) {
  int32_t blk = k / 128, kk = k % 128;
  int32_t s = kk / 16, r16 = kk % 16;
  int32_t h = r16 / 8;
  int32_t p = (r16 % 8) / 2;
  int32_t odd = k & 1;
  int32_t i = 2 * s + h;
  int64_t u = (int64_t)blk * 4 + p;
  int32_t r = row % 8;
  int32_t sigma;
  if (b == 3) sigma = r;
  else if (b == 4) sigma = (r + 2 * (int32_t)(u % 4)) % 8;
  else sigma = (r + 4 * (int32_t)((u / 2) % 2)) % 8;
  int64_t pos = 8 * u + sigma; /* unit position inside the 8-row group */
  int32_t wi, bi;
  if (b == 4) {
    wi = i / 4;
    bi = 4 * (i % 4) + j;
  } else if (b == 3) {
    if (i < 15) {
      wi = i / 5;
      bi = 3 * (i % 5) + j;
    } else {
      wi = j;
      bi = 15;
    }
  } else { /* b == 6 */
    if (i < 12) {
      wi = i / 2;
      bi = 6 * (i % 2) + j;
    } else {
      int32_t m = i - 12;
      if (j < 4) {
        wi = m;
        bi = 12 + j;
      } else {
        wi = 4 + m / 2;
        bi = 12 + 2 * (m % 2) + (j - 4);
      }
    }
  }
  *word_byte = (int64_t)(row / 16) * tile_bytes + (int64_t)((row % 16) / 8) * 8 * row_bytes + pos * 4 * b + 4 * wi;
  *bit = bi + (odd ? 16 : 0);
}

/* Code of input k of row `row` in a projection of K inputs per row (b = 16:
 * the bf16 bits of the weight, little-endian at row * row_bytes + 2 k). */
int32_t orc_get_code(const uint8_t* proj, int32_t K, int32_t g, int32_t row, int32_t k, int32_t b) {
  int64_t rb = orc_row_bytes(K, b), tb = orc_tile_bytes(K, g, b);
  if (b == 16) {
    const uint8_t* e = proj + (int64_t)row * rb + 2 * (int64_t)k;
    return (int32_t)((uint32_t)e[0] | ((uint32_t)e[1] << 8));
  }
  int32_t q = 0;
  for (int32_t j = 0; j < b; ++j) {
    int64_t wb;
    int32_t bit;
    orc_code_bit(row, rb, tb, k, b, j, &wb, &bit);
    q |= (int32_t)((orc_load_word(proj + wb) >> bit) & 1u) << j;
  }
  return q;
}

void orc_set_code(uint8_t* proj, int32_t K, int32_t g, int32_t row, int32_t k, int32_t b, int32_t q) {
  int64_t rb = orc_row_bytes(K, b), tb = orc_tile_bytes(K, g, b);
  if (b == 16) {
    uint8_t* e = proj + (int64_t)row * rb + 2 * (int64_t)k;
    e[0] = (uint8_t)q;
    e[1] = (uint8_t)(q >> 8);
    return;
  }
  for (int32_t j = 0; j < b; ++j) {
    int64_t wb;
    int32_t bit;
    orc_code_bit(row, rb, tb, k, b, j, &wb, &bit);
    uint32_t v = orc_load_word(proj + wb);
    v &= ~(1u << bit);
    v |= (uint32_t)((q >> j) & 1) << bit;
    orc_store_word(proj + wb, v);
  }
}

/* Byte offset of the (scale, bias) word of (row, group gi) from the
 * projection's start. */
int64_t orc_sb_offset(int32_t row, int64_t gi, int32_t K, int32_t g, int32_t b) {
  return (int64_t)(row / 16) * orc_tile_bytes(K, g, b) + 16 * orc_row_bytes(K, b) + 4 * (gi * 16 + row % 16);
}

static uint32_t orc_get_sb(const uint8_t* proj, int32_t row, int64_t gi, int32_t K, int32_t g, int32_t b) {
  return orc_load_word(proj + orc_sb_offset(row, gi, K, g, b));
}

/* Storage row of logical gate/up row R (gate rows 0..I-1, up rows I..2I-1). */
int32_t orc_gate_up_row(int32_t R, int32_t I) {
  int32_t j = R < I ? R : R - I;
  return 16 * (j / 8) + (R < I ? 0 : 8) + j % 8;
}

/* ------------------------------------------------------------------ */
/* Quantization (input preparation; RFC: quantize_experts writes MLX's    */
/* affine format)                                                        */
/* ------------------------------------------------------------------ */
/*
 * Plain min/max affine, per group of g consecutive inputs of a row (a
 * reading: MLX's exact edge rules are not on the pages):
 *   scale = bf16_rne((max - min) / (2^b - 1)),  bias = bf16_rne(min)
 *   q = clamp(rint((w - bias) / scale), 0, 2^b - 1), using the rounded scale
 *   and bias; q = 0 when scale == 0.
 * All arithmetic in fp32, one rounding per operation.
 * w: [rows, K] fp32 in storage row order (rows a multiple of 16).  proj:
 * (rows/16) * tile_bytes(K, g, b) bytes, the tiles above (zeroed here).
 */
void orc_quantize_rows(const float* w, int32_t rows, int32_t K, int32_t g, int32_t b, uint8_t* proj) {
  int64_t ng = orc_row_groups(K, g);
  int32_t qmax = (1 << b) - 1;
  memset(proj, 0, (size_t)((rows / 16) * orc_tile_bytes(K, g, b)));
  if (b == 16) {  /* BF16 experts: the weights rounded to bf16 (nearest even) */
    for (int32_t r = 0; r < rows; ++r)
      for (int32_t k = 0; k < K; ++k) orc_set_code(proj, K, g, r, k, 16, orc_f32_to_bf16(w[(int64_t)r * K + k]));
    return;
  }
  for (int32_t r = 0; r < rows; ++r) {
    const float* wr = w + (int64_t)r * K;
    for (int64_t gi = 0; gi < ng; ++gi) {
      int32_t k0 = (int32_t)(gi * g);
      if (k0 >= K) {
        orc_store_word(proj + orc_sb_offset(r, gi, K, g, b), 0u);
        continue;
      }
      float mn = wr[k0], mx = wr[k0];
      for (int32_t k = k0; k < k0 + g; ++k) {
        if (wr[k] < mn) mn = wr[k];
        if (wr[k] > mx) mx = wr[k];
      }
      uint16_t sh = orc_f32_to_bf16((mx - mn) / (float)qmax);
      uint16_t bh = orc_f32_to_bf16(mn);
      float sf = orc_bf16_to_f32(sh), bf = orc_bf16_to_f32(bh);
      for (int32_t k = k0; k < k0 + g; ++k) {
        int32_t q = 0;
        if (sf != 0.0f) {
          float t = rintf((wr[k] - bf) / sf);
          if (t < 0.0f) t = 0.0f;
          if (t > (float)qmax) t = (float)qmax;
          q = (int32_t)t;
        }
        orc_set_code(proj, K, g, r, k, b, q);
      }
      orc_store_word(proj + orc_sb_offset(r, gi, K, g, b), (uint32_t)sh | ((uint32_t)bh << 16));
    }
  }
}

/* ------------------------------------------------------------------ */
/* Dequantization (bit-exact target)                                     */
/* ------------------------------------------------------------------ */
/* deq = fma(scale, q, bias) in fp32: one rounding.  Rows of K (unpadded), in
 * storage order. */
void orc_dequant_rows(const uint8_t* proj, int32_t rows, int32_t K, int32_t g, int32_t b, float* out) {
  for (int32_t r = 0; r < rows; ++r) {
    for (int32_t k = 0; k < K; ++k) {
      if (b == 16) {  /* BF16 experts: the stored value itself */
        out[(int64_t)r * K + k] = orc_bf16_to_f32((uint16_t)orc_get_code(proj, K, g, r, k, 16));
        continue;
      }
      uint32_t sbw = orc_get_sb(proj, r, k / g, K, g, b);
      float s = orc_bf16_to_f32((uint16_t)(sbw & 0xffffu));
      float bb = orc_bf16_to_f32((uint16_t)(sbw >> 16));
      int32_t c = orc_get_code(proj, K, g, r, k, b);
      out[(int64_t)r * K + k] = fmaf(s, (float)c, bb);
    }
  }
}

/* Whole slot: gate_up [2I, H] (logical row order: gate then up) and down
 * [H, I], fp32. */
void orc_dequant_slot(const uint8_t* slot, int32_t H, int32_t I, int32_t g, int32_t b_gu, int32_t b_d,
                      float* gate_up, float* down) {
  int64_t off[5];
  orc_slot_layout(H, I, g, b_gu, b_d, off);
  float* tmp = (float*)malloc(sizeof(float) * (size_t)2 * I * H);
  orc_dequant_rows(slot + off[0], 2 * I, H, g, b_gu, tmp);
  for (int32_t R = 0; R < 2 * I; ++R)
    memcpy(gate_up + (int64_t)R * H, tmp + (int64_t)orc_gate_up_row(R, I) * H, sizeof(float) * (size_t)H);
  free(tmp);
  orc_dequant_rows(slot + off[1], H, I, g, b_d, down);
}

/* ------------------------------------------------------------------ */
/* Stages 4 + 5: expert FFN (SwiGLU) and weighted combine                */
/* ------------------------------------------------------------------ */
/*
 * For each token t in the list and each rank j (ascending):
 *   e = ids[t,j];  W_gu = deq(slot of e) [2I, H];  W_d = deq [H, I]
 *   gu = W_gu x_t;  h = silu(gu[0..I)) * gu[I..2I);  o = W_d h
 *   y_t += w[t,j] * o
 * silu(z) = z / (1 + exp(-z)).  Accumulation in double (the dequantised
 * weights are fp32 values, x is bf16; both exact in double).
 * expert_slot[e]: pointer to expert e's slot bytes (its cache slot).
 * tok: list of n_tok token indices to evaluate; y: [n_tok, H] double.
 */
void orc_expert_ffn(const uint16_t* x, int32_t H, int32_t I, int32_t g, int32_t b_gu, int32_t b_d,
                    int32_t k, const uint8_t* const* expert_slot, const int32_t* ids, const double* w,
                    const int32_t* tok, int32_t n_tok, double* y) {
  /* Each expert's weights are dequantised once per distinct slot and reused
   * for every (token, rank) it serves; o_{t,j} is kept per (t, j) and y_t is
   * summed over j in rank order at the end. */
  int64_t npair = (int64_t)n_tok * k;
  float* wgu = (float*)malloc(sizeof(float) * (size_t)2 * I * H);
  float* wd = (float*)malloc(sizeof(float) * (size_t)H * I);
  double* xd = (double*)malloc(sizeof(double) * (size_t)H);
  double* h = (double*)malloc(sizeof(double) * (size_t)I);
  double* o = (double*)malloc(sizeof(double) * (size_t)(npair > 0 ? npair : 1) * H);
  unsigned char* done = (unsigned char*)calloc((size_t)(npair > 0 ? npair : 1), 1);
  for (int64_t p = 0; p < npair; ++p) {
    if (done[p]) continue;
    int32_t tp = tok[p / k];
    const uint8_t* slot = expert_slot[ids[(int64_t)tp * k + p % k]];
    orc_dequant_slot(slot, H, I, g, b_gu, b_d, wgu, wd);
    for (int64_t q = p; q < npair; ++q) {
      int32_t t = tok[q / k];
      if (done[q] || expert_slot[ids[(int64_t)t * k + q % k]] != slot) continue;
      done[q] = 1;
      for (int32_t c = 0; c < H; ++c) xd[c] = (double)orc_bf16_to_f32(x[(int64_t)t * H + c]);
      for (int32_t r = 0; r < I; ++r) {
        double a = 0.0, u = 0.0;
        for (int32_t c = 0; c < H; ++c) {
          a += (double)wgu[(int64_t)r * H + c] * xd[c];
          u += (double)wgu[(int64_t)(I + r) * H + c] * xd[c];
        }
        h[r] = a / (1.0 + exp(-a)) * u;
      }
      for (int32_t r = 0; r < H; ++r) {
        double acc = 0.0;
        for (int32_t c = 0; c < I; ++c) acc += (double)wd[(int64_t)r * I + c] * h[c];
        o[q * H + r] = acc;
      }
    }
  }
  for (int32_t ti = 0; ti < n_tok; ++ti) {
    int32_t t = tok[ti];
    for (int32_t r = 0; r < H; ++r) {
      double acc = 0.0;
      for (int32_t j = 0; j < k; ++j) acc += w[(int64_t)t * k + j] * o[((int64_t)ti * k + j) * H + r];
      y[(int64_t)ti * H + r] = acc;
    }
  }
  free(wgu);
  free(wd);
  free(xd);
  free(h);
  free(o);
  free(done);
}

/* ------------------------------------------------------------------ */
/* Host slot cache: LRU per (size class, layer)                          */
/* ------------------------------------------------------------------ */
/*
 * 1bit-MONSTER PR #137: each size class has its own slots and LRU, one LRU
 * per layer with --per-layer; every layer keeps the same share of its
 * experts; empty slots sit at the back of the LRU and are taken first.
 * Reading: one LRU per (class, layer) over that layer's own slot range.
 * Plain array model: stamp[s] = last use (0 = never used, so empty slots are
 * the least recent); owner[s] = expert in slot s or -1.
 *   touch(hits): stamp the hit experts' slots, ascending expert order
 *   assign(misses): for each miss, ascending, take the slot with the lowest
 *     (stamp, slot id) among slots not used by the current pass; evict its
 *     owner (table[owner] = -1), install the miss there.
 * Returns the number of misses that found no slot (capacity error).
 */
int32_t orc_lru_step(int32_t E, int32_t n_slots, int32_t slot_base, int32_t* table, int32_t* owner,
                     int64_t* stamp, int64_t* clock, const int32_t* pass_experts, int32_t n_pass,
                     int32_t* assigned /*[n_pass]: slot for each miss in order, or -1*/, int32_t* n_assigned) {
  unsigned char* used = (unsigned char*)calloc((size_t)n_slots, 1);
  int32_t fail = 0, na = 0;
  for (int32_t i = 0; i < n_pass; ++i) {
    int32_t e = pass_experts[i];
    int32_t s = table[e];
    if (s >= 0) {
      used[s - slot_base] = 1;
      stamp[s - slot_base] = ++(*clock);
    }
  }
  for (int32_t i = 0; i < n_pass; ++i) {
    int32_t e = pass_experts[i];
    if (table[e] >= 0) continue;
    int32_t best = -1;
    for (int32_t s = 0; s < n_slots; ++s) {
      if (used[s]) continue;
      if (best < 0 || stamp[s] < stamp[best]) best = s;
    }
    if (best < 0) {
      assigned[na++] = -1;
      ++fail;
      continue;
    }
    if (owner[best] >= 0) table[owner[best]] = -1;
    owner[best] = e;
    table[e] = slot_base + best;
    used[best] = 1;
    stamp[best] = ++(*clock);
    assigned[na++] = slot_base + best;
  }
  *n_assigned = na;
  free(used);
  (void)E;
  return fail;
}
