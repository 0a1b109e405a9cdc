/*
 * strata_moe.h -- C interface of the routed int4 expert (mixture-of-experts)
 * layer for one NVIDIA B200 (sm_100a).
 *
 * The layer, for each of n_tokens tokens x[t] (bf16, length hidden):
 *   1. routes the token to its top_k experts: logit[e] = x[t] . Wr[e] + b[e]
 *      (fp32 router weights), softmax over the n_experts logits, the top_k
 *      largest logits (ties: lower expert id first), and the selected
 *      probabilities divided by their sum -> weights w[t][j];
 *   2. finds each selected expert's weights through an expert-id -> slot
 *      table over a fixed-size arena of expert blobs (ro99/strata README,
 *      "Residency": the routed experts of a step are kept in GPU memory
 *      under LRU replacement;
 *      "Strata on a Mac", "What you need": an arena of the most-used experts
 *      with the rest read as tokens need them);
 *   3. runs the expert FFN on 4-bit block-quantised weights with 16-bit
 *      activations (the int4 format of ro99/strata README, model table):
 *      h = silu(Wg x) * (Wu x), y = Wd h, silu(z) = z / (1 + exp(-z));
 *   4. writes out[t] = sum_j w[t][j] * y[t][j] + sum_s y_shared[t][s].
 * The output does not depend on which slot holds which expert, nor on
 * whether experts that are not routed are bound at all (the bit-exact tier of
 * "How these numbers are measured", "Fidelity (paged vs resident output)").
 *
 * Expert blob format (the contract behind every device_ptr; one contiguous
 * blob per expert, as "Strata on a Mac", "What you need", keeps each
 * expert's matrices together so that one request reads an expert).  With
 * H = hidden and I = inter (both multiples of 128):
 *     section  content                                 bytes
 *     GU_q     gate and up int4 weights, I/8 tiles     I*H
 *     D_q      down int4 weights, H/16 tiles           H*I/2
 *     GU_s     gate and up fp16 scales, I/8 tiles      I*H/8
 *     D_s      down fp16 scales, H/16 tiles            H*I/16
 * each starting at the next multiple of 256 bytes; the blob size is rounded
 * up to 256 bytes (strata_moe_expert_bytes).  A tile has 16 rows: gate/up
 * tile t holds rows 8t..8t+7 of Wg as tile rows 0..7 and the same rows of Wu
 * as tile rows 8..15; down tile t holds rows 16t..16t+15 of Wd.  A tile is
 * stored K-group by K-group (128 consecutive K elements): 16 rows x 64 bytes
 * of weights, or 16 rows x 4 fp16 scales (one per block of 32 elements; block
 * b = elements 32b..32b+31 of the group).  In the 64 bytes of one row and
 * group, byte 16w + 4b + m/2 (w, b in 0..3, m in 0..7) holds element
 * 32b + 8w + m, in the low nibble for even m; a nibble is a two's-complement
 * int4 in [-8, 7].  The weight is scale * q.  (Any K range of a tile is one
 * contiguous run of bytes, and the 16 bytes at 16w hold word w of all four
 * blocks of a group.)
 *
 * Ownership: the caller owns every buffer it passes (activations, outputs,
 * routing arrays, router weights, expert blobs); they must stay valid until
 * the stream work that uses them has completed.  The library owns its handle
 * and a device workspace, and never frees caller memory.
 *
 * Ordering: bind and set calls are host-only and synchronous; each forward or
 * route call takes a snapshot of the slot table when it is enqueued, so a
 * later bind affects only later calls.  Rebinding a slot whose blob is still
 * read by enqueued work is the caller's hazard, as for any stream-ordered
 * buffer.  A handle (and an arena) must not be used from several host threads
 * at once.  A route or forward call with more tokens than the workspace holds
 * grows it first (cudaMalloc/cudaFree and a device synchronisation); use
 * strata_moe_reserve to do that up front.
 *
 * Errors: a call that finds a problem on the host returns a status and
 * enqueues nothing.  Problems only the device can see (a routed expert with
 * no slot, an out-of-range expert id given to forward_routed, a kernel wait
 * that timed out) are recorded in a device status word: the affected
 * tokens' outputs are written as zeros, and strata_moe_get_status reports
 * the word.  Nothing traps, and nothing falls back to another computation.
 * n_tokens == 0 returns STRATA_OK and enqueues nothing.
 */
#ifndef STRATA_MOE_H
#define STRATA_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *strata_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef struct strata_moe strata_moe; /* opaque */

typedef enum {
  STRATA_OK = 0,
  STRATA_ERR_INVALID_ARG = 1,      /* bad dimension, index, pointer or alignment */
  STRATA_ERR_UNSUPPORTED = 2,      /* a shape the kernels do not handle */
  STRATA_ERR_NOT_BOUND = 3,        /* a routed expert had no slot (device-detected) */
  STRATA_ERR_SLOT_CONFLICT = 4,    /* the expert is already bound to another slot */
  STRATA_ERR_TOO_MANY_EXPERTS = 5, /* more distinct experts than slots were asked for */
  STRATA_ERR_OOM = 6,              /* workspace allocation failed */
  STRATA_ERR_CUDA = 7,             /* a CUDA runtime call failed */
  STRATA_ERR_DEVICE_STATUS = 8,    /* another device-side error (bad routing, timeout) */
  STRATA_ERR_SCRATCH_LIMIT = 9,    /* too large for strata_moe_forward_noalloc's fixed scratch */
  STRATA_ERR_RANGE = 10            /* a value left the f16 range (device-detected; see forward) */
} strata_status;

/* Create a layer on the current CUDA device.
 * The layer is the routed mixture-of-experts block that the pages put on the
 * hot path of decode and prefill (ro99/strata README, "Residency" and
 * "Kernels"; "Strata on a Mac", "What you need"): n_experts routed experts of
 * which each token uses top_k, plus n_shared always-on experts, all of one
 * SwiGLU shape, over an arena of n_slots expert slots.
 * hidden, inter: H and I, multiples of 128.  n_experts: 1..256.
 * top_k: 1..min(32, n_experts).  n_shared: 0..4 always-on experts of the same
 * shape.  n_slots: arena slots, top_k..n_experts.  On success *out owns a
 * handle (free with strata_moe_destroy).  Errors: INVALID_ARG, OOM, CUDA. */
strata_status strata_moe_create(int hidden, int inter, int n_experts, int top_k, int n_shared,
                                int n_slots, strata_moe **out);

/* Free the handle and its workspace (synchronises the device first). */
void strata_moe_destroy(strata_moe *h);

/* Size in bytes of one expert blob (the format above) for hidden x inter. */
size_t strata_moe_expert_bytes(int hidden, int inter);

/* Weight formats of the expert blobs of a layer.
 * STRATA_FORMAT_INT4 (default): the format described at the top of this file.
 * STRATA_FORMAT_NVFP4 (ro99/strata README, model table: NVFP4 routed experts,
 *   E2M1 weights with E4M3 scales per 16 and an fp32 per-tensor global scale,
 *   run with 16-bit activations): the same sections, tiles and nibble places,
 *   holding 4-bit E2M1 codes (sign, 2-bit exponent with bias 1, 1-bit
 *   mantissa: 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives) instead of
 *   integers; the scale sections hold, per tile row and K group of 128, eight
 *   E4M3 bytes instead of four fp16 values (byte i scales elements
 *   16i..16i+15 of the group); and one more 256-byte-aligned section holds
 *   three fp32 global scales (gate, up, down).  The weight is
 *   (code value * E4M3 scale) * global scale.  The kernels apply the first
 *   product exactly in f16 and the global scale once per dot product.
 * strata_moe_expert_bytes_fmt: blob size in a format (0 for bad arguments).
 * strata_moe_set_format: the format of the layer's blobs; only while no slot
 *   and no shared expert is bound (else INVALID_ARG; also for an unknown
 *   format).  Arenas created afterwards copy blobs of this format's size. */
enum { STRATA_FORMAT_INT4 = 0, STRATA_FORMAT_NVFP4 = 1 };
size_t strata_moe_expert_bytes_fmt(int hidden, int inter, int fmt);
strata_status strata_moe_set_format(strata_moe *h, int fmt);

/* Router weights: W_dev fp32 [n_experts][hidden] row-major (device), bias_dev
 * fp32 [n_experts] (device) or NULL for none.  Pointers must be 16-byte
 * aligned.  Errors: INVALID_ARG. */
strata_status strata_moe_set_router(strata_moe *h, const float *W_dev, const float *bias_dev);

/* Routing function (default: softmax).
 * STRATA_ROUTE_SOFTMAX: the description at the top of this file; corr_dev
 *   must be NULL and routed_scale 1.
 * STRATA_ROUTE_SIGMOID: sigmoid scores, a per-expert correction bias on the
 *   selection and a scale on the routed weights, as ro99/strata README
 *   describes for some models (notes under the model table): score[e] = 1 / (1 + exp(-logit[e])) (evaluated in double, rounded
 *   to fp32); the top_k experts by score[e] + corr[e] (fp32; ties: lower id;
 *   corr_dev: device fp32 [n_experts] or NULL for zeros) in descending order;
 *   weights w[j] = score[j] / (sum of the selected scores, added in that
 *   order) * routed_scale.  Shared experts keep weight 1.
 * corr_dev is read by later calls (caller-owned, must stay valid).
 * Errors: INVALID_ARG (unknown mode, routed_scale not positive and finite,
 * misaligned corr_dev, or corr/scale given with softmax). */
enum { STRATA_ROUTE_SOFTMAX = 0, STRATA_ROUTE_SIGMOID = 1 };
strata_status strata_moe_set_routing(strata_moe *h, int mode, const float *corr_dev,
                                     float routed_scale);

/* Bind shared expert i (0 <= i < n_shared) to the blob at device_ptr
 * (256-byte aligned, strata_moe_expert_bytes long).  Errors: INVALID_ARG. */
strata_status strata_moe_bind_shared(strata_moe *h, int i, const void *device_ptr);

/* The expert-id -> slot table over the arena (ro99/strata README,
 * "Residency": routed experts kept in GPU memory under LRU replacement; "Strata
 * on a Mac", "What you need": a fixed-size arena of the most-used experts).
 * Put expert_id's blob at device_ptr into slot `slot` (0 <= slot < n_slots);
 * expert_id == -1 empties the slot (device_ptr ignored).  device_ptr must be
 * 256-byte aligned.  Errors: INVALID_ARG (range, alignment, NULL),
 * SLOT_CONFLICT (expert_id already sits in another slot). */
strata_status strata_moe_bind_slot(strata_moe *h, int slot, int expert_id, const void *device_ptr);

/* Expert id held by `slot`, or -1 (empty) or -2 (slot out of range). */
int strata_moe_slot_expert(const strata_moe *h, int slot);

/* Grow the device workspace to hold max_tokens tokens now (synchronous), so
 * that later forward/route calls with n_tokens <= max_tokens allocate nothing
 * (for example before capturing them in a CUDA graph).  Errors: OOM, CUDA. */
strata_status strata_moe_reserve(strata_moe *h, int max_tokens);

/* Routing only: step 1 of the description at the top of this file (the
 * router that "Strata on a Mac", "Switches", fuses into one dispatch with its
 * top-k: logits, then the top_k experts and their renormalised weights).
 * x_bf16: device bf16 [n_tokens][hidden].  logits_out: device
 * fp32 [n_tokens][n_experts] or NULL.  idx_out: device int32
 * [n_tokens][top_k], experts in descending logit order (ties: lower id
 * first).  w_out: device fp32 [n_tokens][top_k], the renormalised softmax
 * weights.  Asynchronous on `stream`.  Errors: INVALID_ARG, OOM, CUDA. */
strata_status strata_moe_route(strata_moe *h, const void *x_bf16, int n_tokens, float *logits_out,
                               int32_t *idx_out, float *w_out, strata_stream_t stream);

/* The whole layer: steps 1-4 of the description at the top of this file
 * (ro99/strata README, "Kernels": the W4A16 routed-expert FFN; "How these
 * numbers are measured", "Fidelity (paged vs resident output)": the output
 * does not depend on the slot table).  x_bf16: device bf16
 * [n_tokens][hidden]; out_bf16: device bf16 [n_tokens][hidden] (round to
 * nearest even of the fp32 combine).  Asynchronous on `stream`.
 * Range: the kernels feed the tensor cores f16 operands, so activations and
 * the SwiGLU output h must stay below 65520 in magnitude (larger values round
 * to an f16 infinity), and with more than 64 tokens (the tensor-core path,
 * which dequantises each int4 weight to f16(q * scale)) every fp16 scale of a
 * routed or shared int4 expert must be below 8192 in magnitude (8 * 8192
 * would overflow; NVFP4 weights before the global scale are at most 2688).  A value beyond these limits is detected on the device and
 * reported as STRATA_ERR_RANGE by strata_moe_get_status (the affected outputs
 * are then not meaningful); with up to 64 tokens scales of any finite fp16
 * value are applied exactly in fp32.
 * Host errors: INVALID_ARG (including no router set or a shared expert not
 * bound), OOM, CUDA.  Device errors (see strata_moe_get_status): NOT_BOUND,
 * RANGE, DEVICE_STATUS (a wait that timed out). */
strata_status strata_moe_forward(strata_moe *h, const void *x_bf16, int n_tokens, void *out_bf16,
                                 strata_stream_t stream);

/* The layer with routing given: idx (device int32 [n_tokens][top_k], each in
 * [0, n_experts), distinct within a token) and w (device fp32
 * [n_tokens][top_k]), e.g. from strata_moe_route after the caller has bound
 * the routed experts.  Device errors: NOT_BOUND, DEVICE_STATUS (bad id). */
strata_status strata_moe_forward_routed(strata_moe *h, const void *x_bf16, int n_tokens,
                                        const int32_t *idx, const float *w, void *out_bf16,
                                        strata_stream_t stream);

/* Synchronise `stream`, then read and clear the device status word: STRATA_OK,
 * STRATA_ERR_NOT_BOUND, STRATA_ERR_RANGE, STRATA_ERR_DEVICE_STATUS (in that
 * order of precedence, lowest last), or STRATA_ERR_CUDA if the stream itself
 * failed. */
strata_status strata_moe_get_status(strata_moe *h, strata_stream_t stream);

/* Raw device status bits of the last get_status call (1 = not bound,
 * 2 = bad routing id, 4 = wait timeout, 8 = bounds, 16 = f16 range), for
 * diagnostics. */
int strata_moe_last_device_bits(const strata_moe *h);

/* Limit, in nanoseconds, of every wait of the small-batch (up to 64 tokens)
 * kernel that depends on other multiprocessors or on copies in flight: its
 * grid barriers and its ring stages (default STRATA_DEFAULT_WAIT_NS, 2 s).
 * A wait that runs out sets the device status (STRATA_ERR_DEVICE_STATUS,
 * bit 4) and the kernel winds down: every copy it issued still lands (that
 * wait keeps the default limit) and every grid barrier is still passed, so no
 * other multiprocessor waits on it; that call's outputs are not meaningful,
 * and strata_moe_get_status resets the kernel's counters so that the next
 * call is clean.  0 makes every wait that is not already satisfied give up at
 * once (a way to exercise this path).  The tensor-core (more than 64 tokens)
 * kernels keep the default.  Errors: INVALID_ARG. */
#define STRATA_DEFAULT_WAIT_NS 2000000000ull
strata_status strata_moe_set_wait_limit(strata_moe *h, unsigned long long ns);

/* Per-kernel timing for measurement.  enable != 0 makes every later call
 * record a CUDA event pair around each kernel on the call's stream;
 * strata_moe_profile_read synchronises those events and returns, per phase,
 * the number of launches and their summed milliseconds, then clears them.
 * Phases: 0 router, 1 top-k, 2 bucketing, 3 activation pack, 4 gate/up+SwiGLU,
 * 5 down projection, 6 combine, 7 prefill gather, 8 the whole small-batch
 * layer (one launch).  n_phases <= 9.
 * Errors: INVALID_ARG, CUDA. */
strata_status strata_moe_profile(strata_moe *h, int enable);
strata_status strata_moe_profile_read(strata_moe *h, int n_phases, int *launches, double *ms);

/* ---- Expert arena: least-recently-used residency of routed experts.
 * The paging layer in front of the slot table (ro99/strata README,
 * "Residency": the routed experts of each step kept in GPU memory under LRU
 * replacement and copied in from pinned host memory; "Strata on a Mac",
 * "What you need": a fixed arena of experts, the rest read in as tokens need
 * them).  An arena owns the
 * layer's slot table: it binds slot s to device memory
 * arena_dev + s * strata_moe_expert_bytes(hidden, inter).  Results do not
 * depend on the arena's choices, only copy traffic does. */
typedef struct strata_arena strata_arena; /* opaque */

typedef struct {
  int hits;     /* requested experts that were already resident */
  int misses;   /* requested experts copied in by this call */
  size_t bytes; /* bytes copied host -> device by this call */
} strata_arena_stats;

/* Create an arena for `layer` (which must outlive it).  host_pool: host
 * memory holding all n_experts blobs back to back in expert order
 * (strata_moe_expert_bytes apart), ideally pinned (pageable memory makes the
 * copies synchronous); arena_dev: device memory for n_slots blobs, 256-byte
 * aligned.  Both stay owned by the caller and must outlive the arena.  All
 * slots of the layer are emptied.  Errors: INVALID_ARG, OOM, CUDA. */
strata_status strata_arena_create(strata_moe *layer, const void *host_pool, void *arena_dev,
                                  strata_arena **out);
void strata_arena_destroy(strata_arena *a);

/* Make the experts ids[0..n) (host int32, repeats allowed) resident before the
 * work that `stream` runs next.  Resident ones are hits and become most
 * recently used; each miss is copied (one cudaMemcpyAsync on copy_stream) into
 * the lowest empty slot, else into the least recently used slot not asked for
 * by this call (ties: lowest slot), and bound there.  copy_stream first waits
 * for the work already queued on `stream` (an evicted expert may still be read
 * there); `stream` then waits for the copies.  stats (may be NULL) receives
 * hits, misses and bytes.  Host-side and asynchronous; the layer's slot
 * table changes at once, so enqueue the forward that uses these experts on
 * `stream` after this call.  Errors: INVALID_ARG (an id out of range),
 * TOO_MANY_EXPERTS (more distinct ids than slots; nothing changes), CUDA (a
 * copy could not be enqueued; the slots bound before the failure stay
 * bound, and their copies may still be in flight on copy_stream, while the
 * slot chosen for the failed copy keeps its old expert, in the arena and in
 * the layer's table alike). */
strata_status strata_arena_ensure(strata_arena *a, const int32_t *ids, int n,
                                  strata_stream_t stream, strata_stream_t copy_stream,
                                  strata_arena_stats *stats);

/* Wait for the copies of the last ensure call and return their device time in
 * milliseconds (0 if it copied nothing).  Errors: INVALID_ARG, CUDA. */
strata_status strata_arena_copy_ms(strata_arena *a, float *ms);

/* Slot holding expert_id, -1 if it is not resident, -2 if out of range. */
int strata_arena_slot_of(const strata_arena *a, int expert_id);

/* Prefill through the arena in chunks, for a layer whose experts do not all
 * fit its slots ("Strata on a Mac", "Unsloth's UD-Q4/Q5/Q6_K_XL on the M5
 * Max": prompts stream in chunks of 4096 tokens, and every chunk makes one
 * pass over the experts that are not in the arena; "Switches": the chunk size
 * is a setting).  Every token is routed once; then, chunk by chunk of
 * chunk_tokens tokens, the chunk's distinct experts -- those already
 * resident first -- are made resident in groups of at most n_slots
 * (strata_arena_ensure, LRU), each group's share of the chunk's expert work
 * runs on the tensor cores, and the chunk's output is combined.  Larger
 * chunks re-read fewer experts; each chunk needs one group per n_slots of its
 * distinct experts.  x_bf16 and out_bf16: device bf16 [n_tokens][hidden].
 * The result equals strata_moe_forward's on the same tokens bit for bit when
 * n_tokens > 64 (every chunk, of any size, takes the tensor-core path that
 * the forward takes for more than 64 tokens).  Synchronises `stream` once
 * (to read the routing on the host); may grow the layer's workspace and a
 * pinned host buffer of the arena.  stats (may be NULL): chunks, groups run,
 * experts found resident, copied, and bytes copied.  Errors: INVALID_ARG, OOM,
 * CUDA, and those of strata_arena_ensure; device errors as for forward. */
typedef struct {
  int chunks;   /* chunks of the prompt */
  int passes;   /* expert groups run over all chunks */
  int hits;     /* experts already resident when their group ran */
  int misses;   /* experts copied in */
  size_t bytes; /* bytes copied host -> device */
} strata_prefill_stats;
strata_status strata_arena_prefill(strata_arena *a, const void *x_bf16, int n_tokens,
                                   int chunk_tokens, void *out_bf16, strata_stream_t stream,
                                   strata_stream_t copy_stream, strata_prefill_stats *stats);

/* Size of the fixed device scratch of strata_moe_forward_noalloc, and the
 * most tokens one call of it takes. */
#define STRATA_NOALLOC_SCRATCH_BYTES (16u << 20)
#define STRATA_NOALLOC_MAX_TOKENS 64

/* strata_moe_forward, for callers that must not allocate device memory while
 * they run: code under a memory manager that has carved the whole device into
 * its own pools (a cudaMalloc would fail, or break up those pools), or a
 * decode loop that cannot afford the device-wide synchronisation that
 * cudaMalloc and cudaFree may cause.  The pages describe no such call; it has
 * no counterpart there.
 *
 * Same arguments, result and errors as strata_moe_forward, with these
 * differences.  The workspace is one fixed array of STRATA_NOALLOC_SCRATCH_BYTES
 * bytes of device memory owned by the library (one per device), never the
 * handle's workspace, and the call allocates nothing: no cudaMalloc, cudaFree
 * or other allocating routine.  n_tokens may be at most
 * STRATA_NOALLOC_MAX_TOKENS, and the workspace for n_tokens = T must fit the
 * array: with P = T * (top_k + n_shared), N = n_experts + n_shared and M the
 * device's multiprocessor count, about
 *     4*T*n_experts + 8*T*top_k + 4*(3N + 2) + 12*P + 2*T*hidden
 *       + 2*P*inter + 4*P*hidden + 8*T*max(n_experts, M)
 *       + 4*(2308 + 32*M + hidden/16) + 65536*M  bytes
 * (each term rounded up to 256; the last three terms are the decode
 * kernel's router partial sums, its barrier, cut-item, tile and pair-group
 * counters and its two partial-sum slots per warp and phase, 9.7 MB on 148
 * multiprocessors);
 * a request beyond either limit returns STRATA_ERR_SCRATCH_LIMIT and
 * enqueues nothing.  The current device must be the handle's device
 * (otherwise INVALID_ARG).  The first call on a device looks up the array's
 * address on that device (this can load the library's device code there),
 * so make that first call before any stream capture.  Every call on a device,
 * from any handle, uses the same array, and the array keeps what the last
 * call left in it: the call clears what must start at zero and writes the
 * rest before reading it, but calls whose work overlaps on the GPU (on
 * different streams, without an ordering between them) race on the array and
 * give wrong results.  Per-kernel timing (strata_moe_profile) is not recorded
 * for this call.  The handle must not be used from another host thread
 * during the call. */
strata_status strata_moe_forward_noalloc(strata_moe *h, const void *x_bf16, int n_tokens,
                                         void *out_bf16, strata_stream_t stream);

/* Human-readable name of a status. */
const char *strata_status_str(strata_status s);

#ifdef __cplusplus
}
#endif

#endif /* STRATA_MOE_H */
