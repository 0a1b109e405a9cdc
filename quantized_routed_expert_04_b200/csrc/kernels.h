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
__global__ void pack_x_kernel(const __nv_bfloat16 *x, int n8, __half *x16, int fmt,
                              int *status);
__global__ void bucket_count_kernel(const int32_t *idx, int T, int k, int E, int *cnt,
                                    int *status);
__global__ void bucket_fill_kernel(const int32_t *idx, int T, int k, int E, int S, Routing rt);
// Routing only of small batches in one launch (see route.cu).
constexpr int kSmallT = 64;
struct SmallRouteParams {
  const __nv_bfloat16 *x;
  const float *W, *bias;
  int T, H, E, k;
  float *logits;   // [T][E]
  int32_t *idx;    // [T][k]
  float *w;        // [T][k]
  int *counter;    // last-block counter, zero between launches
  RouteMode mode;
};
__global__ void route_small_kernel(SmallRouteParams p);

__global__ void combine_kernel(const float *y, const int32_t *idx, const float *w,
                               const int *inv, ExpertTable table, int check_bound, int T, int H,
                               int k, int S, int E, __nv_bfloat16 *out);

// ---- the whole small-batch layer in one persistent launch (decode_fused.cu)
//
// One work item = (active expert, group of <= 16 of its pairs, one 16-row
// weight tile: 8 gate + 8 up rows, or 16 down rows).
constexpr int kFusedWarps = 16;                     // warps per CTA, each with its own ring
constexpr int kMmMaxStages = 8;                     // stages per warp ring
constexpr int kMmMaxGroup = 16;                     // pairs per item (two n8 MMA tiles)
constexpr int kMmSlotFloats = kMmMaxGroup * 16;     // partial sums of one piece: pairs x rows
struct FusedParams {
  ExpertTable table;
  const __nv_bfloat16 *x;   // [T][H]
  const float *W, *bias;    // router
  RouteMode mode;
  const int32_t *idx_in;    // routing given (forward_routed), else null
  const float *w_in;
  int T, H, I, E, k, S;
  size_t guq, gus, dq, ds;  // blob sections
  size_t glob;              // NVFP4: offset of the three fp32 global scales (gate, up, down)
  int kc;                   // K elements per ring stage (multiple of 128)
  int stages, stage_bytes;  // per-warp ring
  int group;                // pairs per item: 8 or 16
  unsigned long long wait_ns;  // limit of every wait that depends on other warps or copies
  size_t smem_tables;       // offset of the routing tables in dynamic shared memory
  double *rpart;            // router partial sums [max(1, grid / E)][T][E]
  int32_t *idx;             // [T][k] (used when more tokens than warps per CTA)
  float *w;                 // [T][k]
  __half *x16, *h16;        // packed activations [T][H], SwiGLU output [P][I]
  float *y;                 // [P][H]
  float *partial;           // [phase][warps of the grid][2][kMmSlotFloats]
  int *cut_cnt;             // [2][warps of the grid]   } zero between launches
  int *tile_cnt;            // [H/16]                   } (each resets what it
  int *bar;                 // [4] grid barriers, exit  }  used, or the last CTA
  int *grp_done;            // [T*(k+S)] gate/up items done per pair group  }  out resets)
  int *status;
  __nv_bfloat16 *out;       // [T][H]
};
template <int NT, int FMT>   // NT: 8-pair MMA tiles per item (1 or 2); FMT: weight format
__global__ void decode_fused_kernel(FusedParams p);
size_t fused_table_bytes(int T, int k, int S);

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
  int quiet_unbound;  // 1: experts without a blob are left to another pass, not reported
  size_t glob_off;    // NVFP4: offset of the three fp32 global scales in a blob
};
}  // namespace strata
#include <cuda.h>
namespace strata {
template <bool kGateUp, int FMT>
__global__ void expert_tc_kernel(TcParams p, const __grid_constant__ CUtensorMap tmap_b16,
                                 const __grid_constant__ CUtensorMap tmap_b64,
                                 const __grid_constant__ CUtensorMap tmap_b256);
__global__ void gather_rows_kernel(const __half *x16, const int *pair_tok, const int *n_pairs_dev,
                                   int H, int P_cap, __half *xp);
size_t tc_smem_bytes();
int tc_threads();

}  // namespace strata
