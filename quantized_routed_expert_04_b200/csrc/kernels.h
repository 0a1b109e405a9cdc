// Kernel declarations and launch parameter blocks (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "layer.h"

namespace strata {

// ---- routing (route.cu)
__global__ void router_gemv_kernel(const __nv_bfloat16 *x, const float *W, const float *bias,
                                   int T, int H, int E, float *logits);
__global__ void router_gemm_kernel(const __nv_bfloat16 *x, const float *W, const float *bias,
                                   int T, int H, int E, float *logits);
__global__ void topk_kernel(const float *logits, int T, int E, int k, int32_t *idx, float *w);
__global__ void pack_x_kernel(const __nv_bfloat16 *x, int n8, __half *x16);
__global__ void bucket_count_kernel(const int32_t *idx, int T, int k, int E, int *cnt,
                                    int *status);
__global__ void bucket_fill_kernel(const int32_t *idx, int T, int k, int E, int S, Routing rt);
__global__ void combine_kernel(const float *y, const int32_t *idx, const float *w,
                               const int *inv, ExpertTable table, int T, int H, int k, int S,
                               int E, __nv_bfloat16 *out);

// ---- expert matmuls on CUDA cores + legacy tensor cores (expert_mma.cu)
//
// One work item = (active expert, group of <= 16 of its pairs, tile of 32
// weight rows).  For the gate/up pass the 32 rows are 16 rows of Wg and the
// same 16 rows of Wu (so SwiGLU is thread-local); for the down pass they are
// 32 consecutive rows of Wd.
constexpr int kMmStages = 4;
constexpr int kMmGroup = 16;       // pairs per item (two n8 MMA tiles)
constexpr int kMmThreads = 160;    // 1 producer warp + 4 consumer warps

struct MmParams {
  ExpertTable table;
  Routing rt;
  int E;
  int K;              // reduction length: H (gate/up) or I (down)
  int kc;             // K elements per pipeline stage (multiple of 64, divides K)
  int tiles;          // tiles per expert: I/16 (gate/up) or H/32 (down)
  size_t q_off[2];    // packed sections of the two 16-row halves
  size_t s_off[2];    // scale sections
  int row_base_mul;   // first weight row of tile tau = tau * row_base_mul
  int row_half[2];    // extra row offset of each half (0,0) gate/up; (0,16) down
  const __half *b_src;  // gate/up: packed x16 [T][H]; down: h16 [P][I]
  int out_ld;         // row length of the output (I for h16, H for y)
  __half *h_out;      // gate/up output, packed like x16
  float *y_out;       // down output
  int *status;
  // shared-memory layout of one stage
  int wstride, sstride, bstride;
  int w_bytes, s_bytes;  // region offsets: weights at 0, scales at w_bytes, B at w_bytes + s_bytes
  int stage_bytes;
};

template <bool kGateUp>
__global__ void expert_mma_kernel(MmParams p);

size_t mm_smem_bytes(const MmParams &p);

}  // namespace strata
