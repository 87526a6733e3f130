/*
 * moe.h -- C ABI of libmoe: the routed-expert FFN run out of a bounded,
 * slot-indexed device expert cache, for NVIDIA B200 (sm_100a).
 *
 * The path, in five stages, follows web pages on streaming MoE experts:
 *   1. moe_route        router softmax -> top-k -> renormalise, with optional
 *                       cache-aware substitution (BigMoeOnEdge, commit note on
 *                       cache-aware substitution)
 *   2. moe_sort         tokens grouped by expert; prefill runs at most 64
 *                       experts per pass (transformers PR #50717 "POC:
 *                       Experts offload" notes; RFC "stream MoE experts from
 *                       disk in from_pretrained", section "How the prototype
 *                       works", item "Prefill")
 *   3. moe_slot_lookup  per-layer expert -> slot table over one preallocated
 *                       pool, with a miss list (RFC, "How the prototype
 *                       works", items "Cache" and "Reads")
 *      moe_install_slots  one host-to-device copy per missed expert from
 *                       pinned host rows (RFC, items "Reads" and "Host tier")
 *   4+5. moe_expert_ffn fused group-wise affine dequant (w = scale*q + bias)
 *                       feeding the SwiGLU gate/up/down projections straight
 *                       from the slot pool (RFC: quantized experts through
 *                       gather_qmm on the pool; experts "gated, concatenated,
 *                       untransposed, no bias"), then the weighted combine of
 *                       the k expert outputs per token.
 *   Size classes: layers whose experts need the same bytes share one pool
 *   with its own slots (1bit-MONSTER engine PR #137 "expert slots in size
 *   classes"); the host side of that is the moe_cache_* functions.
 *
 * Conventions for every call:
 *   - Device pointers are raw CUDA device addresses; "host" pointers are
 *     ordinary (or pinned, where stated) host memory.  bf16 tensors are passed
 *     as uint16_t bit patterns.  All arrays are dense, row-major.
 *   - The library allocates no device memory and keeps no state between
 *     calls (the host slot cache object lives in host memory; the one fixed
 *     device array is the scratch of moe_expert_ffn_noalloc).  The caller owns
 *     every buffer, stream and event.
 *   - Every device call is asynchronous on the given stream and does not
 *     synchronise with the host.
 *   - Argument errors are found before anything is launched and return
 *     MOE_ERR_INVALID or MOE_ERR_UNSUPPORTED; launch failures return
 *     MOE_ERR_CUDA.  Data errors found on the device (a slot id of -1 or past
 *     the pool reaching the FFN, a wait that ran out) are OR-ed into the
 *     caller's int32 *dev_err word (MOE_DEV_ERR_* bits); the offending work
 *     item is skipped, nothing traps.  The caller reads dev_err after its
 *     next synchronisation.
 *
 * Slot format (one expert = one slot; the pages name "MLX's affine format,
 * one contiguous row per expert" but give no bit layout -- this one is
 * chosen so that the GPU unpacks two codes per logic operation):
 *   A weight row of K inputs is padded to Kp = K rounded up to 128 (padded
 *   groups have scale = bias = 0).  Each block of 128 inputs is 4 units of 32
 *   codes; unit p holds, for s = 0..7, the input pairs (128B+16s+2p, +1) and
 *   (128B+16s+2p+8, +1) as pair indices 2s and 2s+1, the even input in the
 *   low 16-bit half of a 32-bit word and the odd input at the same offset in
 *   the high half.  Rows are stored in tiles of 16 consecutive rows; a tile
 *   is the rows' codes (16*Kp*b/8 bytes) followed by their (scale, bias)
 *   words, and consecutive tiles are adjacent.  The codes are two groups of
 *   8 rows; inside a group, unit u = 4B+p of row r (0..7) is at unit position
 *   8u + sigma(u, r) (4b bytes per position), sigma = r for b=3,
 *   (r + 2(u mod 4)) mod 8 for b=4, (r + 4((u/2) mod 2)) mod 8 for b=6 -- so a
 *   tile is one contiguous copy and the GEMV's per-thread unit loads from
 *   shared memory are bank-conflict free.  A unit is b little-endian words:
 *     b=4: pair i in word i/4, bits 4*(i%4)..+3
 *     b=3: pair i<15 in word i/5, bits 3*(i%5)..+2; pair 15: bit j of the
 *          code is bit 15 of word j
 *     b=6: pair i<12 in word i/2, bits 6*(i%2)..+5; pair 12+m: code bits 0..3
 *          at bits 12..15 of word m, bits 4..5 at bits 12+2*(m%2)+{0,1} of
 *          word 4+m/2
 *   Per group of g inputs, one 32-bit word: bf16 scale (low half), bf16 bias
 *   (high half); inside a tile the words are group-major (word (r, gi) at
 *   gi*16 + r).  A slot is two projections, each 256-byte aligned:
 *     gate_up [2I rows]  storage row order: blocks of 16 rows, block m =
 *             gate rows 8m..8m+7 then up rows 8m..8m+7 (one tile per block)
 *     down    [H rows]
 *   slot_bytes = end of the down projection rounded to 256.  Dequantised weight
 *   = fmaf(scale, q, bias) in fp32 (one rounding).
 * BF16 experts (b = 16; RFC "How the prototype works", item "Cache": BF16
 * experts run through the grouped experts kernel): a projection is its rows
 * of bf16 values, row-major (row r at r * Kp * 2 bytes), zero-padded to Kp,
 * in the same storage row order, with no scale/bias words; a tile is 16 rows.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,      /* bad argument (null pointer, size, alignment) */
  MOE_ERR_CUDA = 2,         /* a CUDA runtime call or launch failed */
  MOE_ERR_UNSUPPORTED = 3,  /* valid request outside what is built (bits, group, sizes) */
  MOE_ERR_NOT_RESIDENT = 4, /* an expert needed by the call has no slot */
  MOE_ERR_CAPACITY = 5,     /* no free slot / buffer too small */
  MOE_ERR_TIMEOUT = 6       /* a bounded device wait ran out */
} moe_status;

/* Bits OR-ed into the caller's device int32 *dev_err. */
#define MOE_DEV_ERR_NOT_RESIDENT 1 /* slot id -1 reached the FFN: pair skipped */
#define MOE_DEV_ERR_SLOT_RANGE 2   /* slot id >= n_slots: pair skipped */
#define MOE_DEV_ERR_TIMEOUT 4      /* bounded wait on a copy barrier ran out */
#define MOE_DEV_ERR_BAD_EXPERT 8   /* an expert id outside [0, E) */

/* Shapes of one MoE layer.  Limits: 1 <= k <= E <= 1024; H and I multiples of
 * group; group in {32, 64, 128}; bits in {3, 4, 6}, or 16 for a BF16
 * projection (unquantized; group then only checks H and I).  A layer with a
 * 16-bit projection runs on the tensor-core grouped GEMM only: its
 * moe_expert_ffn calls need x_sorted at every T and H, I multiples of 128
 * (else MOE_ERR_UNSUPPORTED). */
typedef struct {
  int32_t E;         /* experts in the layer */
  int32_t k;         /* experts per token (top-k) */
  int32_t H;         /* hidden size: input of gate/up, output of down */
  int32_t I;         /* expert intermediate size */
  int32_t group;     /* inputs per (scale, bias) group */
  int32_t bits_gu;   /* code width of the gate/up projection (16: bf16 values) */
  int32_t bits_down; /* code width of the down projection (16: bf16 values) */
} moe_layer_desc;

/* Byte offsets of the two projections in a slot, their 16-row tile sizes, and
 * the slot size (the size-class key of 1bit-MONSTER PR #137: "the sum of its
 * aligned read windows"). */
typedef struct {
  uint64_t gate_up, down, gate_up_tile_bytes, down_tile_bytes, slot_bytes;
} moe_slot_layout_t;

/* Slot byte size for d, or 0 if d is invalid. */
size_t moe_slot_bytes(const moe_layer_desc* d);

/* Projection offsets and tile sizes for d.  Returns MOE_ERR_INVALID or
 * MOE_ERR_UNSUPPORTED for a bad d. */
moe_status moe_slot_layout(const moe_layer_desc* d, moe_slot_layout_t* out);

/* Device workspace needed by moe_sort and moe_expert_ffn for up to
 * max_tokens tokens (0 if d is invalid).  One buffer of this size may be
 * shared by the two calls when they run in stream order.  Zero the whole
 * buffer once after allocating it (e.g. cudaMemset).  Its head -- a 512-byte
 * control block (the single-launch decode FFN's launch epoch and arrival
 * count) and that kernel's h words, each tagged with its launch -- carries
 * over from call to call; every launch leaves the head consistent, also one
 * whose waits ran out.  Only a launch cut short on the device (its context
 * lost) or foreign writes can leave it otherwise; a later call then reports
 * MOE_DEV_ERR_TIMEOUT instead of using stale values -- zero the whole buffer
 * after a reported timeout.  Calls with different layer descriptions may
 * share the buffer if it is large enough for each. */
size_t moe_workspace_bytes(const moe_layer_desc* d, int32_t max_tokens);

/* Stage 1.  Cache-aware top-k (BigMoeOnEdge note: every expert already in
 * the cache gets its score raised by L times the token's score range, then
 * the top-k is taken again; the same number of experts runs).
 *   logits     device fp32 [T, E], finite
 *   L          substitution strength; 0 = plain top-k.  Meant for decode.
 *   slot_table device int32 [E], this layer's expert -> slot (-1 = absent),
 *              read before this step's installs; may be NULL when L == 0.
 *   ids        device int32 [T, k], experts in rank order
 *   w          device fp32 [T, k], u_e / sum over the chosen u (unboosted)
 * Per token: u_e = exp(l_e - max l) with a fixed fp32 exp (range reduction by
 * ln2 + degree-7 Taylor) so that ids match a CPU evaluation bit for bit;
 * u'_e = u_e + L*(1 - min u) for resident e; key (u' desc, l desc, e asc).
 * T = 0 is a no-op. */
moe_status moe_route(const float* logits, int32_t T, const moe_layer_desc* d, float L,
                     const int32_t* slot_table, int32_t* ids, float* w, cudaStream_t stream);

/* Stage 1 for a layer with always-on shared experts (BigMoeOnEdge
 * docs/limitations.md, "Limitations", bullet "Shared experts stay resident":
 * the routed experts stream, the shared expert stays resident).  The top-k
 * of moe_route, then n_shared (0..8) shared experts appended to every token:
 *   ids  device int32 [T, k + n_shared]: the top-k in rank order, then the
 *        expert ids E, E+1, ..., E+n_shared-1
 *   w    device fp32 [T, k + n_shared]: the top-k weights (normalised over
 *        the top-k only), then shared_w[t] for each shared expert, or 1 when
 *        shared_w is NULL (device fp32 [T], e.g. a per-token gate)
 * The layer's other calls then take the widened description (E + n_shared
 * experts, k + n_shared per token) and a slot table of E + n_shared entries
 * whose last n_shared entries hold the shared experts' slots, so the shared
 * experts run in the same moe_expert_ffn launch as the routed ones.  Keeping
 * those slots resident is the caller's (moe_cache manages routed experts
 * only).  n_shared outside 0..8 returns MOE_ERR_INVALID. */
moe_status moe_route_shared(const float* logits, int32_t T, const moe_layer_desc* d, float L,
                            const int32_t* slot_table, int32_t n_shared, const float* shared_w, int32_t* ids,
                            float* w, cudaStream_t stream);

/* Stage 2.  Stable counting sort of the T*k (token, rank) pairs by expert.
 *   ids      device int32 [T, k]
 *   x        device bf16 [T, H] or NULL; when given, x_sorted is written
 *   offsets  device int32 [E+1]: pairs of expert e are offsets[e]..offsets[e+1]
 *   pairs    device int32 [T*k]: flat index t*k+j, by expert then flat index
 *   active   device int32 [E]: experts with >= 1 pair, ascending
 *   n_active device int32 [1]
 *   x_sorted device fp16 [T*k, H]: x_sorted[i] = x[pairs[i] / k] converted
 *            to fp16 (round to nearest even, saturating at +-65504), the
 *            operand type of the tensor-core grouped GEMM (if x)
 *   ws       device workspace of ws_bytes >= moe_workspace_bytes(d, T)
 * Prefill pass p covers active[64p .. 64p+64). */
moe_status moe_sort(const int32_t* ids, const uint16_t* x, int32_t T, const moe_layer_desc* d,
                    int32_t* offsets, int32_t* pairs, int32_t* active, int32_t* n_active,
                    uint16_t* x_sorted, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Stage 3.  Slots of one pass of the active list.
 *   slot_table device int32 [E]
 *   active, n_active  from moe_sort (device)
 *   pass_begin, pass_len  host ints: the pass is active[pass_begin ..
 *              min(pass_begin+pass_len, *n_active))
 *   n_slots    slots in the pool (ids >= n_slots are flagged in dev_err)
 *   slots      device int32 [pass_len]: table[active[i]]
 *   miss       device int32 [pass_len]: experts of the pass with slot -1,
 *              ascending
 *   n_miss     device int32 [1]
 *   dev_err    device int32 [1] (MOE_DEV_ERR_SLOT_RANGE) or NULL */
moe_status moe_slot_lookup(const int32_t* slot_table, const int32_t* active, const int32_t* n_active,
                           int32_t pass_begin, int32_t pass_len, int32_t n_slots, int32_t* slots,
                           int32_t* miss, int32_t* n_miss, int32_t* dev_err, cudaStream_t stream);

/* Stage 3'.  Install n experts: cudaMemcpyAsync of slot_bytes from pinned
 * host_rows[i] to pool + slots[i]*slot_bytes, on the side stream, then
 * records done (if not NULL) on it.  host_rows (pinned) must not change until
 * done has fired (RFC, "Host tier": rows stay reserved until the copy that
 * reads them has run).  slots is a host array; each id must be < n_slots. */
moe_status moe_install_slots(void* pool, size_t slot_bytes, int32_t n_slots, const void* const* host_rows,
                             const int32_t* slots, int32_t n, cudaStream_t side, cudaEvent_t done);

/* Stages 1 + 2 + 3 of one decode token in one launch (the calls above would
 * take three): the routing of moe_route_shared (strength L, n_shared 0..8
 * shared experts of weight shared_w[0], or 1 when shared_w is NULL; with
 * n_shared 0 that is moe_route), the sort of moe_sort without x_sorted, and
 * moe_slot_lookup over the whole active list (pass_begin 0, pass_len
 * E + n_shared) -- the same values in the same buffers, bit for bit.  d is
 * the routed experts' description, as for moe_route_shared; the sort and
 * lookup outputs are those of the widened layer (E + n_shared experts,
 * k + n_shared per token).  T must be 1 (else MOE_ERR_UNSUPPORTED: use the
 * three calls); n_shared outside 0..8 returns MOE_ERR_INVALID, and
 * k + n_shared above 32 MOE_ERR_UNSUPPORTED (as moe_sort on that layer).
 *   slot_table device int32 [E + n_shared] (the first E entries read for
 *   substitution, every active entry for the lookup); n_slots as
 *   moe_slot_lookup; ids, w, offsets, pairs, active, n_active as
 *   moe_route_shared and moe_sort; slots, miss, n_miss, dev_err as
 *   moe_slot_lookup. */
moe_status moe_route_sort_lookup(const float* logits, int32_t T, const moe_layer_desc* d, float L,
                                 const int32_t* slot_table, int32_t n_shared, const float* shared_w,
                                 int32_t n_slots, int32_t* ids, float* w, int32_t* offsets, int32_t* pairs,
                                 int32_t* active, int32_t* n_active, int32_t* slots, int32_t* miss,
                                 int32_t* n_miss, int32_t* dev_err, cudaStream_t stream);

/* Stages 4 + 5 for one pass.
 *   x          device bf16 [T, H]
 *   pool       device base of this layer's size-class pool (slot_bytes stride)
 *   n_slots    slots in the pool
 *   slot_table device int32 [E]
 *   ids, w     from moe_route; offsets, pairs, active, n_active from moe_sort
 *   x_sorted   from moe_sort, or NULL (needed by the tensor-core grouped GEMM,
 *              which runs wherever the fused decode kernel does not
 *              apply when it is given; else unused)
 *   pass_begin, pass_len  which active experts this call runs
 *   y_accum    device fp32 [T, H]; the pass's expert outputs are ADDED:
 *              y_t += sum over the pass's pairs (t, j) of w[t,j] * o_{t,j}.
 *              Zero it before the first pass.  Summation order is fixed
 *              (deterministic run to run).
 *   ws         device workspace, ws_bytes >= moe_workspace_bytes(d, T)
 *   dev_err    device int32 [1]: MOE_DEV_ERR_NOT_RESIDENT / SLOT_RANGE /
 *              TIMEOUT; affected experts are skipped */
moe_status moe_expert_ffn(const uint16_t* x, int32_t T, const moe_layer_desc* d, const void* pool,
                          int32_t n_slots, const int32_t* slot_table, const int32_t* ids, const float* w,
                          const int32_t* offsets, const int32_t* pairs, const int32_t* active,
                          const int32_t* n_active, const uint16_t* x_sorted, int32_t pass_begin,
                          int32_t pass_len, float* y_accum, void* ws, size_t ws_bytes, int32_t* dev_err,
                          cudaStream_t stream);

/* Stages 1-5 of one decode token in one launch, for a layer whose routed
 * experts are resident (RFC "How the prototype works", item "Cache": a fully
 * resident layer never synchronises with the host, so its routing need not
 * leave the device before its FFN).  The fused decode kernel routes the token
 * itself -- the routing of moe_route with strength L over slot_table's
 * residency, bit for bit -- and runs every routed expert, as
 * moe_route_sort_lookup followed by moe_expert_ffn over one pass would.
 *   x        device bf16 [1, H];  logits  device fp32 [1, E]
 *   T        must be 1; E <= 1024; quantized experts only (else
 *            MOE_ERR_UNSUPPORTED: use moe_route_sort_lookup and
 *            moe_expert_ffn)
 *   ids, w, offsets, pairs, active, n_active, slots, miss, n_miss: device
 *            outputs, the values moe_route_sort_lookup writes
 *   y        device fp32 [1, H], OVERWRITTEN with the layer's output
 *   ws       device workspace, ws_bytes >= moe_workspace_bytes(d, 1)
 *   dev_err  as moe_expert_ffn: a routed expert without a slot is flagged
 *            MOE_DEV_ERR_NOT_RESIDENT (and listed in miss) and skipped */
moe_status moe_route_expert_ffn(const uint16_t* x, const float* logits, int32_t T, const moe_layer_desc* d, float L,
                                const void* pool, int32_t n_slots, const int32_t* slot_table, int32_t* ids, float* w,
                                int32_t* offsets, int32_t* pairs, int32_t* active, int32_t* n_active, int32_t* slots,
                                int32_t* miss, int32_t* n_miss, float* y, void* ws, size_t ws_bytes, int32_t* dev_err,
                                cudaStream_t stream);

/* moe_expert_ffn without a caller-supplied workspace.  (The pages have no
 * counterpart; this is an interface convenience.)  For callers that cannot
 * allocate device memory themselves -- e.g. a plugin whose host process owns
 * all device memory through its own allocator, or a serving loop that must
 * not call cudaMalloc (which can synchronise the device) once it is running.
 * The scratch is one fixed device array of moe_noalloc_scratch_bytes() bytes
 * (1 MiB) inside the library, held by every GPU that loads it until the
 * process exits.  Same arguments and results as moe_expert_ffn, except:
 *   - T must be <= 64 and the workspace of a call without x_sorted must fit
 *     1 MiB (moe_workspace_bytes(d, T) less the tensor-core path's per-pair
 *     output buffer, which this call never uses), else MOE_ERR_CAPACITY is
 *     returned
 *     and nothing is launched;
 *   - x_sorted is not taken (the decode kernels do not use it);
 *   - the first call on a device looks up the array's device address (with
 *     that device current); make that first call outside any stream capture;
 *   - every call shares the one array and leaves its contents behind; the
 *     head that moe_workspace_bytes describes as carried over (control block
 *     and tagged h words) is cleared on `stream` (cudaMemsetAsync) before
 *     each call's kernels, the rest needs no initialisation; calls whose
 *     kernels overlap on the GPU (e.g. on two streams at once) race on the
 *     array.
 * Allocates nothing. */
moe_status moe_expert_ffn_noalloc(const uint16_t* x, int32_t T, const moe_layer_desc* d, const void* pool,
                                  int32_t n_slots, const int32_t* slot_table, const int32_t* ids, const float* w,
                                  const int32_t* offsets, const int32_t* pairs, const int32_t* active,
                                  const int32_t* n_active, int32_t pass_begin, int32_t pass_len, float* y_accum,
                                  int32_t* dev_err, cudaStream_t stream);

/* Size of the fixed scratch array used by moe_expert_ffn_noalloc. */
size_t moe_noalloc_scratch_bytes(void);

/* Test/inspection: dequantise slot `slot` of pool through the same code
 * extraction the FFN kernels use.  out_fp32 (device, may be NULL):
 * gate_up [2I, H] then down [H, I], fp32 = fmaf(scale, q, bias); out_bf16
 * (device, may be NULL): the same values rounded to bf16 (RNE). */
moe_status moe_dequant_slot(const void* pool, int32_t slot, const moe_layer_desc* d, float* out_fp32,
                            uint16_t* out_bf16, cudaStream_t stream);

/* Input preparation (the RFC's one-time quantize_experts, on the GPU):
 * quantise rows of fp32 weights w [rows, K] into the slot format:
 * per group scale = bf16((max-min)/(2^b-1)), bias = bf16(min),
 * q = clamp(rint((w - bias)/scale), 0, 2^b-1) (q = 0 if scale = 0); bits = 16
 * writes the weights rounded to bf16 (nearest even).
 *   rows       a multiple of 16
 *   gate_up_I  0: row r of w is storage row r; I > 0: w is a gate/up matrix
 *              [2I, K] (gate rows then up rows) and its rows go to their
 *              storage rows (blocks of 8 gate + 8 up rows)
 *   proj       device, (rows/16) tiles (see the format above), 16-byte
 *              aligned: a slot's gate_up or down projection */
moe_status moe_quantize_rows(const float* w, int32_t rows, int32_t K, int32_t group, int32_t bits,
                             int32_t gate_up_I, uint8_t* proj, cudaStream_t stream);

/* Router projection (the guess input of moe_decode_layer_ahead: a layer's
 * router evaluated on an earlier layer's hidden state; RFC "How the
 * prototype works", item "Reads"):
 *   logits[t][e] = scale * sum_h x[t][h] * W[e][h] + (bias ? bias[e] : 0)
 *   x      device bf16 [T, H], 16-byte aligned; H a multiple of 8
 *   W      device bf16 [E, H] (row e = expert e's router weights), aligned
 *   bias   device fp32 [E] or NULL
 *   logits device fp32 [T, E]
 * fp32 accumulation in a fixed order (deterministic). */
moe_status moe_router_logits(const uint16_t* x, int32_t T, const uint16_t* W, const float* bias, float scale,
                             int32_t E, int32_t H, float* logits, cudaStream_t stream);

/* Test: the fp32 exp used by moe_route, elementwise on n device floats. */
moe_status moe_exp_portable(const float* x, int64_t n, float* out, cudaStream_t stream);

const char* moe_status_string(moe_status s);

/* Which kernels moe_expert_ffn runs on the current device for a call over
 * all E experts of a layer of shape d with T tokens, with (has_x_sorted != 0)
 * or without x_sorted:
 *   MOE_PATH_FUSED_DECODE  one launch: every CTA runs its share of the
 *                          gate/up + SwiGLU tiles, then (the first H/16
 *                          CTAs) a down + combine tile over every expert,
 *                          reading h words tagged with the launch
 *                          (T <= 8, T*k <= 64)
 *   MOE_PATH_GEMV          gate/up + SwiGLU kernel, down kernel (+ combine
 *                          kernel for T > 64): tensor-core GEMV (mma.sync)
 *   MOE_PATH_TC_PREFILL    tcgen05/TMEM grouped GEMM fed by TMA (beyond the
 *                          fused decode kernel's range, x_sorted given, H and
 *                          I multiples of 128): prefill
 *                          chunks and batched decode; a layer with a 16-bit
 *                          (BF16) projection at every T
 * or -1 if d is invalid, T < 1, or a BF16 layer has no path (no x_sorted).
 * Host only; no device work. */
enum { MOE_PATH_FUSED_DECODE = 0, MOE_PATH_GEMV = 1, MOE_PATH_TC_PREFILL = 2 };
int32_t moe_ffn_kernel_path(const moe_layer_desc* d, int32_t T, int32_t has_x_sorted);

/* Test/inspection: the limit, in SM clock cycles, of every bounded device
 * wait (a bulk copy that should land, a pipeline stage that should free up,
 * the single-launch decode FFN's reads of other CTAs' h) in kernels launched afterwards
 * by this process; cycles <= 0 restores the default of 4e9 (about 2 s at the
 * top clock).  A wait that runs out sets MOE_DEV_ERR_TIMEOUT in dev_err and
 * the kernel returns; tests lower the limit to make such a wait run out
 * quickly.  Host only; process-wide. */
void moe_set_wait_limit_cycles(int64_t cycles);

/* Name of the last CUDA error that made a call of this thread return
 * MOE_ERR_CUDA ("no error" if none). */
const char* moe_last_cuda_error(void);

/* ------------------------------------------------------------------------
 * Host slot cache (1bit-MONSTER PR #137: per size class, one LRU per layer,
 * every layer keeps the same share of its experts, empty slots taken first).
 * Host memory only.  Layer l of class c owns slots [base, base + S) of the
 * class pool, base = (index of l among the layers of class c) * S.
 * ---------------------------------------------------------------------- */
typedef struct moe_cache moe_cache;

/* layer_class: host int32 [n_layers] class of each layer (NULL: all 0);
 * slots_per_layer S.  *out receives the object. */
moe_status moe_cache_create(int32_t E, int32_t n_layers, const int32_t* layer_class, int32_t slots_per_layer,
                            moe_cache** out);
void moe_cache_destroy(moe_cache* c);
/* Host expert -> slot table of a layer ([E], -1 = absent), owned by c. */
const int32_t* moe_cache_table(const moe_cache* c, int32_t layer);
int32_t moe_cache_layer_base(const moe_cache* c, int32_t layer);
/* Slots in the pool of class cls (layers of the class * S). */
int32_t moe_cache_class_slots(const moe_cache* c, int32_t cls);
/* Initial residency: experts[i] into slot slots[i] (absolute pool ids inside
 * the layer's range); later entries are more recent. */
moe_status moe_cache_place(moe_cache* c, int32_t layer, const int32_t* experts, const int32_t* slots, int32_t n);
/* One pass: pass_experts (ascending, host) are the experts the pass runs.
 * Hits are touched in order; each miss (ascending) takes the least recently
 * used slot of the layer not used by this pass (never-used slots first),
 * evicting its owner.  Writes the n_out misses and their slots.  Returns
 * MOE_ERR_CAPACITY if a miss found no slot (its out_slot is -1). */
moe_status moe_cache_step(moe_cache* c, int32_t layer, const int32_t* pass_experts, int32_t n_pass,
                          int32_t* out_experts, int32_t* out_slots, int32_t* n_out);
/* Counters since creation: hits, misses, evictions (of a resident expert). */
void moe_cache_stats(const moe_cache* c, int64_t* hits, int64_t* misses, int64_t* evictions);

/* Experts of `layer` that currently have a slot (E means fully resident). */
int32_t moe_cache_resident(const moe_cache* c, int32_t layer);

/* Guessed prefetch (RFC "How the prototype works", item "Reads": the next two
 * layers' experts are guessed and read in the background).  For each of the
 * n experts (host) that is neither resident nor already reserved, take the
 * least recently used slot of the layer that has no copy in flight (empty
 * slots first), evict its owner and reserve the slot for the expert, which
 * stays out of the table until moe_cache_commit.  Writes the n_out reserved
 * (expert, slot) pairs; stops early when every slot has a copy in flight.
 * moe_cache_step never takes a reserved slot. */
moe_status moe_cache_reserve(moe_cache* c, int32_t layer, const int32_t* experts, int32_t n, int32_t* out_experts,
                             int32_t* out_slots, int32_t* n_out);
/* The copy into reserved `slot` has landed: its expert enters the table as
 * the most recent (*entered = 1), or, if the expert was installed elsewhere
 * meanwhile, the slot becomes empty (*entered = 0).  MOE_ERR_INVALID if the
 * slot holds no reservation. */
moe_status moe_cache_commit(moe_cache* c, int32_t layer, int32_t slot, int32_t* entered);

/* ------------------------------------------------------------------------
 * Native driver of one decode layer (the sequence of the calls above).
 * ---------------------------------------------------------------------- */

/* Per-call device buffers, caller-owned, sized for max_tokens tokens (with
 * shared experts, E and k below are those of the widened layer: E + n_shared,
 * k + n_shared). */
typedef struct {
  int32_t* ids;        /* device int32 [max_tokens, k] */
  float* w;            /* device fp32 [max_tokens, k] */
  int32_t* offsets;    /* device int32 [E+1] */
  int32_t* pairs;      /* device int32 [max_tokens*k] */
  int32_t* meta;       /* device int32 [2+2E]: n_active, n_miss, active[E], miss[E] */
  int32_t* meta_host;  /* pinned host int32 [2+2E] (written by the device when it maps it) */
  int32_t* slots;      /* device int32 [E] */
  int32_t* dev_err;    /* device int32 [1] */
  void* ws;            /* device workspace */
  size_t ws_bytes;     /* >= moe_workspace_bytes(desc, max_tokens) */
  int32_t max_tokens;
  uint16_t* x_sorted;  /* device fp16 [max_tokens*k, H], or NULL: beyond the fused range the layer
                          sorts x into it and its FFN runs on the tensor-core grouped GEMM */
} moe_step_buffers;

/* One layer's slot pool and tables. */
typedef struct {
  const moe_layer_desc* desc;
  void* pool;                   /* device base of the layer's size-class pool */
  int32_t n_slots;              /* slots in that pool */
  size_t slot_bytes;            /* moe_slot_bytes(desc) */
  int32_t* table_dev;           /* device int32 [E]: this layer's expert -> slot */
  int32_t* table_stage;         /* pinned host int32 [E]: staging for table uploads */
  const void* const* bank_rows; /* host [E]: pinned host address of each expert's slot bytes */
  int32_t n_shared;             /* always-on shared experts (moe_route_shared), 0..8: their slots
                                   are table_dev[E .. E+n_shared), kept resident by the caller;
                                   table_dev then has E + n_shared entries and the step buffers
                                   are sized for E + n_shared experts, k + n_shared per token */
  const float* shared_w;        /* device fp32 [T] per-token weight of the shared experts, or NULL (1) */
} moe_layer_ctx;

/* One decode layer, T <= 64 tokens (RFC "How the prototype works": each layer
 * copies its routing to the host once; misses cost one host-to-device copy
 * per expert; a fully resident layer never synchronises with the host):
 *   moe_route (L) -> moe_sort (sorting x into b->x_sorted beyond the fused range and
 *   b->x_sorted is given) -> if the layer is not fully resident in `cache`:
 *   moe_slot_lookup, copy n_active/active to meta_host, synchronise `stream`
 *   (for one token without guesses, when the device addresses meta_host at
 *   the same pointer -- page-locked memory from cudaHostAlloc/cudaMallocHost
 *   -- the one-launch routing kernel writes them there itself, then a
 *   sequence word to meta_host[1], and the host waits for that word: bounded,
 *   MOE_ERR_TIMEOUT after 5 s, no copy back and no stream synchronisation),
 *   moe_cache_step, moe_install_slots on `side`, upload the table, record
 *   `installed` on `side` and make `stream` wait on it -> one pass of
 *   moe_expert_ffn over every active expert, writing y.  When experts are
 *   installed, the pass is split: the active list is rewritten as [experts
 *   that were resident..., installed experts...] into b->slots (the LRU step
 *   never evicts an expert of the step, so the resident ones keep their
 *   slots), moe_expert_ffn over the resident ones writes y on `stream` while
 *   the copies run on `side`, and after the wait on `installed` a second
 *   call adds the installed experts' outputs (summation order: resident
 *   experts, then installed, each in expert order; deterministic).
 * y: device fp32 [T, H] (overwritten).  *n_installed (host, may be NULL): the
 * number of experts installed.  Errors as the calls it makes. */
moe_status moe_decode_layer(moe_cache* cache, int32_t layer, const moe_layer_ctx* lc, const moe_step_buffers* b,
                            const uint16_t* x, const float* logits, int32_t T, float L, float* y,
                            cudaStream_t stream, cudaStream_t side, cudaEvent_t installed, int32_t* n_installed);

/* Guessed prefetch state: per layer, the batches of guessed copies in flight. */
typedef struct moe_prefetch moe_prefetch;
moe_status moe_prefetch_create(int32_t n_layers, moe_prefetch** out);
void moe_prefetch_destroy(moe_prefetch* p);
/* Counters: guessed experts (distinct per guess), copies started, guesses
 * entered into a table, copies wasted (the expert was installed normally
 * first), and reservations found still in flight when their layer ran. */
void moe_prefetch_stats(const moe_prefetch* p, int64_t* guessed, int64_t* started, int64_t* entered,
                        int64_t* wasted, int64_t* skipped);

/* One guessed layer: its router evaluated on the current layer's hidden state. */
typedef struct {
  int32_t layer;           /* the guessed layer (not the current one) */
  const moe_layer_ctx* lc; /* its pool and tables */
  const float* logits;     /* device fp32 [T, E] */
  int32_t top;             /* read ahead each token's `top` best guesses (rank order); 0 = all k */
} moe_guess;
/* Buffers of the guessed top-k, caller-owned. */
typedef struct {
  int32_t* ids;      /* device int32 [2 * stride] */
  float* w;          /* device fp32 [2 * stride] */
  int32_t* ids_host; /* pinned host int32 [2 * stride] */
  int32_t stride;    /* >= max_tokens * k of the guessed layers */
} moe_guess_buffers;

/* moe_decode_layer with guessed prefetch (RFC "How the prototype works",
 * item "Reads": the next two layers' experts are guessed by running their
 * routers on the current hidden states and read in the background;
 * PR #50717, commit note: install_ahead skips guessed reads still in flight
 * instead of waiting for them):
 *   1. the guessed copies of `layer` that have landed (event query, no wait)
 *      enter its table, which is uploaded on `stream` if it changed; copies
 *      still in flight are skipped: their experts count as absent now;
 *   2. moe_decode_layer's sequence, with the n_guesses (0..2) guessed
 *      layers' top-k (moe_route, L = 0) launched next to the layer's own
 *      stages and read back on the same synchronisation (one more if the
 *      layer itself is fully resident);
 *   3. after the layer's own misses have their slots, each guessed layer's
 *      absent guesses get reserved slots (moe_cache_reserve) and their
 *      copies start on `ahead` (a stream of their own, so the layer's own
 *      installs never queue behind them), one event per batch.
 * The results (y) are those of moe_decode_layer: the guesses only move
 * installs earlier. */
moe_status moe_decode_layer_ahead(moe_cache* cache, moe_prefetch* pf, int32_t layer, const moe_layer_ctx* lc,
                                  const moe_step_buffers* b, const uint16_t* x, const float* logits, int32_t T,
                                  float L, float* y, cudaStream_t stream, cudaStream_t side, cudaEvent_t installed,
                                  int32_t* n_installed, const moe_guess* guesses, int32_t n_guesses,
                                  const moe_guess_buffers* gb, cudaStream_t ahead);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
