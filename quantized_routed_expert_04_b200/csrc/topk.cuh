// Top-k selection of one token's experts by one warp (shared by the
// routing kernels of both batch-size paths).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace strata {

// Order-preserving map of an fp32 key to an unsigned integer (larger key,
// larger integer; -0 and +0 equal; NaN below every other key), so that a
// warp's largest key is one hardware warp reduction.
__device__ __forceinline__ uint32_t topk_order_key(float f) {
  if (f != f) return 0u;
  const uint32_t b = f == 0.0f ? 0u : __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One warp per token.  Lane l holds experts l, l+32, ...; k rounds of a warp
// arg-max of the selection key (larger wins, equal keys: lower id wins), each
// round a max-reduction of the keys and a min-reduction of the ids that hold
// it.  Softmax routing: key = logit, weights = exp(l_j - l_0) / sum_j (the
// renormalised softmax of the selected experts).  Sigmoid routing: score =
// 1 / (1 + exp(-l)) in double rounded to fp32, key = score + correction,
// weights = score_j / (sum of the selected scores in selection order) *
// routed scale.  Lane j (< k) returns selection j in sel_e / sel_w.
// kPer: experts per lane (E <= 32 kPer); kShared: the row is in shared
// memory (else global memory written by other CTAs, read from L2).
template <int kPer, bool kShared>
__device__ __forceinline__ void select_topk_warp_t(const float *__restrict__ logit_row, int E,
                                                   int k, const RouteMode &mode, int lane,
                                                   int &sel_e, float &sel_w) {
  uint32_t key[kPer];
  float val[kPer];   // logit (softmax) or score (sigmoid)
  unsigned taken = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    const float l = e < E ? (kShared ? logit_row[e] : __ldcg(logit_row + e)) : 0.0f;
    if (mode.sigmoid && e < E) {
      val[i] = (float)(1.0 / (1.0 + exp(-(double)l)));
      key[i] = topk_order_key(mode.corr ? __fadd_rn(val[i], mode.corr[e]) : val[i]);
    } else {
      val[i] = l;
      key[i] = topk_order_key(l);
    }
    if (e >= E) taken |= 1u << i;
  }
  float v0 = 0.0f, z = 0.0f, my_v = 0.0f;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    // this lane's best untaken key (lowest id among equal keys)
    uint32_t bk = 0u;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (!((taken >> i) & 1u) && (bi < 0 || key[i] > bk)) {
        bk = key[i];
        bi = i;
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bi >= 0 ? bk : 0u);
    const uint32_t cand = bi >= 0 && bk == m ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
    const int be = (int)__reduce_min_sync(0xffffffffu, cand);
    // the winner's logit or score, from the lane that holds it
    float mine = 0.0f;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (i == (be >> 5)) mine = val[i];
    const float bv = __shfl_sync(0xffffffffu, mine, be & 31);
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (mode.sigmoid) {
      z = __fadd_rn(z, bv);
    } else {
      if (j == 0) v0 = bv;
      z += expf(bv - v0);
    }
    if (lane == j) {  // lane j keeps selection j (k <= 32)
      my_v = bv;
      my_e = be;
    }
  }
  sel_e = my_e;
  sel_w = mode.sigmoid ? __fmul_rn(__fdiv_rn(my_v, z), mode.scale) : expf(my_v - v0) / z;
}

__device__ __forceinline__ void select_topk_warp(const float *__restrict__ logit_row, int E, int k,
                                                 const RouteMode &mode, int lane, int &sel_e,
                                                 float &sel_w) {
  select_topk_warp_t<kMaxExperts / 32, false>(logit_row, E, k, mode, lane, sel_e, sel_w);
}

}  // namespace strata
