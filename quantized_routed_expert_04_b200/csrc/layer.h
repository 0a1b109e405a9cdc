// Internal definitions shared by the host side and the kernels of the routed
// int4 expert layer (not part of the public C interface).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace strata {

constexpr int kMaxExperts = 256;   // routed experts per layer
constexpr int kMaxShared = 4;      // always-on shared experts per layer
constexpr int kMaxIds = kMaxExperts + kMaxShared;
constexpr int kMaxTopK = 32;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per barrier wait

// Device status word bits (OR-ed by kernels, read by strata_moe_get_status).
enum : int {
  STATUS_NOT_BOUND = 1,      // a routed expert had no arena slot
  STATUS_BAD_ROUTING = 2,    // forward_routed got an expert id out of range
  STATUS_TIMEOUT = 4,        // a bounded wait in a kernel gave up
  STATUS_BOUNDS = 8,         // a computed offset fell outside its buffer
  STATUS_RANGE = 16,         // a value left the f16 range of the tensor-core operands
};

// Smallest magnitude that round-to-nearest-even turns into an f16 infinity
// (65504 is the largest finite f16; half-way to the next power step rounds up).
constexpr float kF16Overflow = 65520.0f;

// Weight formats of an expert blob (the values of STRATA_FORMAT_*): 4-bit
// integers with fp16 scales per 32, or NVFP4 (E2M1 codes, E4M3 scales per
// 16, fp32 global scales).
enum : int { kFmtInt4 = 0, kFmtNvfp4 = 1 };

// Byte offsets of the sections of an expert blob: gate+up weights, down
// weights, gate+up scales, down scales, and for NVFP4 the three fp32 global
// scales (see include/strata_moe.h).
struct BlobLayout {
  size_t guq, dq, gus, ds, glob, total;
};

inline BlobLayout blob_layout(int H, int I, int fmt = 0) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  BlobLayout L;
  size_t off = 0;
  L.guq = off; off = up(off + (size_t)I * H);
  L.dq = off;  off = up(off + (size_t)H * I / 2);
  L.gus = off; off = up(off + (size_t)I * H / 8);
  L.ds = off;  off = up(off + (size_t)H * I / 16);
  L.glob = off;
  if (fmt == kFmtNvfp4) off = up(off + 3 * sizeof(float));
  L.total = off;
  return L;
}

// Blob address of every expert id, taken by value at launch time: routed
// experts 0..E-1 (nullptr = not bound to a slot), then shared experts.
struct ExpertTable {
  const uint8_t *ptr[kMaxIds];
};

// Routing workspace (device memory), written by the bucketing kernels.
// Pairs (t, j) -- token t's j-th routed expert (j < k) or shared expert
// j - k -- are sorted by expert id, then by token.
struct Routing {
  int *cnt;        // [E+S] pairs per expert id
  int *off;        // [E+S+1] first sorted position of each id
  int *active;     // [E+S] ids with cnt > 0, ascending
  int *n_active;   // [1]
  int *pair_tok;   // [P] token of sorted pair
  int *pair_j;     // [P] j of sorted pair
  int *inv;        // [T][k+S] sorted position of pair (t, j)
};

}  // namespace strata

struct strata_moe;
// Shape of a layer handle (for the arena, which sees the handle only through
// the public calls): hidden, inter, routed experts, arena slots, device.
void strata_handle_shape(const strata_moe *h, int *hidden, int *inter, int *n_experts,
                         int *n_slots, int *device);
int strata_handle_top_k(const strata_moe *h);
size_t strata_handle_blob_bytes(const strata_moe *h);  // bytes of one blob in the layer's format

// Prefill in chunks over an arena with fewer slots than experts (called by
// the arena): route every token once (idx/w stay in the layer's workspace),
// then per chunk of Tc tokens: pack + bucket + gather, one tensor-core pass
// per group of experts that fit the slots (in_pass[e] marks the group; the
// shared experts run with the first group), and the combine.  Each pair's
// result does not depend on the pass that computes it, so the output equals
// the all-resident forward's.  Chunks always take the tensor-core path.
#include "strata_moe.h"
strata_status strata_layer_route_all(strata_moe *h, const void *x, int T, cudaStream_t stream,
                                     const int32_t **idx, const float **w);
strata_status strata_layer_chunk_prepare(strata_moe *h, const void *x, int Tc, const int32_t *idx,
                                         cudaStream_t stream);
strata_status strata_layer_chunk_pass(strata_moe *h, int Tc, const unsigned char *in_pass,
                                      bool shared, cudaStream_t stream);
strata_status strata_layer_chunk_finish(strata_moe *h, int Tc, const int32_t *idx, const float *w,
                                        void *out, cudaStream_t stream);
