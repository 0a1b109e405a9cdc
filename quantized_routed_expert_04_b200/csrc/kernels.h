// Kernel declarations and launch parameter blocks (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "layer.h"

namespace strata {

// ---- routing (route.cu)
__global__ void router_gemm_kernel(const __nv_bfloat16 *x, const float *W, const float *bias,
                                   int T, int H, int E, float *logits);
// Routing function: softmax (sigmoid = 0) or sigmoid scores with an optional
// correction bias on the selection key and a routed scale on the weights.
struct RouteMode {
  int sigmoid;
  const float *corr;  // [E] or null
  float scale;
};
__global__ void topk_kernel(const float *logits, int T, int E, int k, RouteMode mode,
                            int32_t *idx, float *w);
__global__ void pack_x_kernel(const __nv_bfloat16 *x, int n8, __half *x16, int *status);
__global__ void bucket_count_kernel(const int32_t *idx, int T, int k, int E, int *cnt,
                                    int *status);
__global__ void bucket_fill_kernel(const int32_t *idx, int T, int k, int E, int S, Routing rt);
// Routing of small batches in one launch (see route.cu).
constexpr int kSmallT = 64;
struct SmallRouteParams {
  const __nv_bfloat16 *x;
  const float *W, *bias;
  int T, H, E, k, S;
  float *logits;   // [T][E] written (kRoute)
  int32_t *idx;    // [T][k] written (kRoute) or read
  float *w;        // [T][k] written (kRoute)
  Routing rt;
  __half *x16;
  int *counter;    // last-block counter, zero between launches
  int *status;
  RouteMode mode;
};
template <bool kRoute, bool kBucket>
__global__ void route_small_kernel(SmallRouteParams p);

__global__ void combine_kernel(const float *y, const int32_t *idx, const float *w,
                               const int *inv, ExpertTable table, int T, int H, int k, int S,
                               int E, __nv_bfloat16 *out);

// ---- expert matmuls for small token counts (expert_mma.cu)
//
// One work item = (active expert, group of <= 16 of its pairs, one 16-row
// weight tile of the blob: 8 gate + 8 up rows, or 16 down rows).  Each warp
// of the grid takes an equal contiguous share of the (item, K group)
// sequence; an item cut by a share boundary is finished by its last piece.
constexpr int kMmMaxStages = 8;                     // stages per warp ring
constexpr int kMmWarps = 12;                        // warps per CTA, each with its own ring
constexpr int kMmThreads = 32 * kMmWarps;
constexpr int kMmMaxGroup = 16;                     // pairs per item (two n8 MMA tiles)
constexpr int kMmMaxPairs = 4096;                   // pair tokens staged in shared memory
constexpr int kMmSlotFloats = kMmMaxGroup * 16;     // partial sums of one piece: pairs x rows

struct MmParams {
  ExpertTable table;
  Routing rt;
  int E;
  int K;              // reduction length: H (gate/up) or I (down)
  int kc;             // K elements per stage (multiple of 128, divides K)
  int tiles;          // tiles per expert: I/8 (gate/up) or H/16 (down)
  int group;          // pairs per item: 8 or 16
  int n_ids;          // E + S
  int stages;         // stages per warp ring (<= kMmMaxStages)
  size_t q_off, s_off;  // weight and scale sections (gate+up or down)
  const __half *b_src;  // gate/up: packed x16 [T][H]; down: h16 [P][I]
  int out_ld;         // row length of the output (I for h16, H for y)
  __half *h_out;      // gate/up output, packed like x16
  float *y_out;       // down output
  int *status;
  int stage_bytes;    // kc*8 weight bytes + kc scale bytes, rounded to 128
  float *partial;     // [warps of the grid][kMmSlotFloats] partial sums of cut items
  int *counters;      // [warps of the grid] pieces arrived per cut item (zero between launches)
};

template <bool kGateUp, int NT>   // NT: 8-pair MMA tiles per item (1 or 2)
__global__ void expert_mma_kernel(MmParams p);

size_t mm_smem_bytes(const MmParams &p);

// ---- expert matmuls for many tokens per expert (prefill_tc.cu)
struct TcParams {
  ExpertTable table;
  Routing rt;
  int K;              // H (gate/up) or I (down)
  int row_tiles;      // 128-row weight tiles: I/64 (gate/up) or H/128 (down)
  size_t q_off, s_off;
  int out_ld;         // I (h16) or H (y)
  __half *h_out;
  float *y_out;
  int *status;
};
}  // namespace strata
#include <cuda.h>
namespace strata {
template <bool kGateUp>
__global__ void expert_tc_kernel(TcParams p, const __grid_constant__ CUtensorMap tmap_b64,
                                 const __grid_constant__ CUtensorMap tmap_b256);
__global__ void gather_rows_kernel(const __half *x16, const int *pair_tok, const int *n_pairs_dev,
                                   int H, int P_cap, __half *xp);
size_t tc_smem_bytes();
int tc_threads();
size_t mm_fixed_smem_bytes();

}  // namespace strata
