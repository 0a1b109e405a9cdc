// Top-k selection of one token's experts by one warp (shared by the
// routing kernels of both batch-size paths).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace strata {

// One warp per token.  Lane l holds experts l, l+32, ...; k rounds of a warp
// arg-max of the selection key (larger wins, equal keys: lower id wins).
// Softmax routing: key = logit, weights = exp(l_j - l_0) / sum_j (the
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
  float key[kPer], val[kPer];   // val: logit (softmax) or score (sigmoid)
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    const float l = e < E ? (kShared ? logit_row[e] : __ldcg(logit_row + e)) : -INFINITY;
    if (mode.sigmoid && e < E) {
      val[i] = (float)(1.0 / (1.0 + exp(-(double)l)));
      key[i] = mode.corr ? __fadd_rn(val[i], mode.corr[e]) : val[i];
    } else {
      val[i] = l;
      key[i] = l;
    }
  }
  unsigned taken = 0;
  float v0 = 0.0f, z = 0.0f, my_v = 0.0f;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    float bk = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (be == 0x7fffffff || key[i] > bk)) {
        bk = key[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (oe != 0x7fffffff && (be == 0x7fffffff || ok > bk || (ok == bk && oe < be))) {
        bk = ok;
        be = oe;
      }
    }
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
