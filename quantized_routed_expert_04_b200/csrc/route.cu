// Routing, bucketing, activation packing and the weighted combine.
//
// Router (the fused router dispatch that "Strata on a Mac", "Switches",
// describes among its two opt-ins): logit = x . Wr[e] + b[e] with x bf16 and
// Wr fp32;
// every product is exact in double and the sum is kept in double, then
// rounded once to fp32.  Top-k takes the largest fp32 logits, lower expert id
// first among equal ones; the weights are the softmax probabilities of the
// selected experts divided by their sum, computed directly as
// exp(l_j - l_max) / sum_j exp(l_j - l_max).
//
// Bucketing (large batches) sorts the (token, j) pairs by expert id, then
// token, with no atomics in the ordering (each expert's block walks the pairs
// in order), so the layout -- and every result downstream -- is a pure
// function of the routing, independent of slots and of scheduling.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace strata {

// ---------------------------------------------------------------- router GEMM
// Large batches (prefill): logits of 128 tokens x 64 experts per block on the
// fp64 tensor-core path (mma.m8n8k4, f64 in and out).  The bf16 x fp32
// products are exact in fp64 and every sum is an fp64 sum, rounded once to
// fp32 at the end; the order of the fp64 additions differs from a plain
// ascending loop, which moves a logit by at most about 1e-11 relative before
// that rounding.  8 warps as 4 (tokens) x 2 (experts), each 32 x 32 = 4 x 4
// tiles of 8 x 8; K staged 16 at a time in shared memory (as fp32, exact for
// both operands, widened to fp64 when the fragments are read), two stages so
// that one barrier per slice suffices, the next slice prefetched into
// registers during the MMAs.
constexpr int kRT = 128, kRE = 64, kRK = 16;
constexpr int kRXL = kRT + 8, kRWL = kRE + 8;   // padded rows: conflict-free fragment reads

__device__ __forceinline__ void dmma_8x8x4(double &d0, double &d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(256) router_gemm_kernel(
    const __nv_bfloat16 *__restrict__ x, const float *__restrict__ W,
    const float *__restrict__ bias, int T, int H, int E, float *__restrict__ logits) {
  grid_dependency_wait();
  __shared__ float xs[2][kRK][kRXL];
  __shared__ float ws[2][kRK][kRWL];
  const int t0 = blockIdx.x * kRT, e0 = blockIdx.y * kRE;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wt = (warp & 3) * 32, we = (warp >> 2) * 32;   // warp tile origin in the block
  // global -> register staging: one 16-byte piece of x and of W per thread
  const int xr = tid >> 1, xc = (tid & 1) * 8;              // token row, k offset (8 bf16)
  const int wr = tid >> 2, wc = (tid & 3) * 4;              // expert row, k offset (4 fp32)
  const bool x_ok = t0 + xr < T, w_ok = e0 + wr < E;
  const __nv_bfloat16 *xp = x + (size_t)(x_ok ? t0 + xr : 0) * H + xc;
  const float *wp = W + (size_t)(w_ok ? e0 + wr : 0) * H + wc;
  uint4 xv = make_uint4(0u, 0u, 0u, 0u);
  float4 wv = make_float4(0.f, 0.f, 0.f, 0.f);
  if (x_ok) xv = *reinterpret_cast<const uint4 *>(xp);
  if (w_ok) wv = *reinterpret_cast<const float4 *>(wp);
  auto stage = [&](int b) {
    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&xv);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(h2[q]);
      xs[b][xc + 2 * q][xr] = f.x;
      xs[b][xc + 2 * q + 1][xr] = f.y;
    }
    ws[b][wc + 0][wr] = wv.x;
    ws[b][wc + 1][wr] = wv.y;
    ws[b][wc + 2][wr] = wv.z;
    ws[b][wc + 3][wr] = wv.w;
  };

  double acc[4][4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

  stage(0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < H; k0 += kRK) {
    const bool more = k0 + kRK < H;
    if (more) {
      if (x_ok) xv = *reinterpret_cast<const uint4 *>(xp + k0 + kRK);
      if (w_ok) wv = *reinterpret_cast<const float4 *>(wp + k0 + kRK);
    }
#pragma unroll
    for (int kk = 0; kk < kRK; kk += 4) {
      double a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = (double)xs[buf][kk + (lane & 3)][wt + 8 * i + (lane >> 2)];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = (double)ws[buf][kk + (lane & 3)][we + 8 * j + (lane >> 2)];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma_8x8x4(acc[i][j][0], acc[i][j][1], a[i], b[j]);
    }
    // the other stage was last read before the previous barrier
    if (more) stage(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
  // lane holds rows (lane >> 2) and columns 2 (lane & 3) + {0, 1} of each tile
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + wt + 8 * i + (lane >> 2);
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int e = e0 + we + 8 * j + 2 * (lane & 3) + c;
        if (e >= E) continue;
        double v = acc[i][j][c];
        if (bias) v += (double)bias[e];
        logits[(size_t)t * E + e] = (float)v;
      }
  }
}

// ---------------------------------------------------------------- top-k
__global__ void topk_kernel(const float *__restrict__ logits, int T, int E, int k, RouteMode mode,
                            int32_t *__restrict__ idx, float *__restrict__ w) {
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int e;
  float wt;
  select_topk_warp(logits + (size_t)t * E, E, k, mode, lane, e, wt);
  if (lane < k) {
    idx[(size_t)t * k + lane] = e;
    w[(size_t)t * k + lane] = wt;
  }
}

// ---------------------------------------------------------------- activation pack
// x bf16 -> f16 in the weight format's pair order (pack8_bf16_to_f16); an
// activation beyond the f16 range sets STATUS_RANGE.
__global__ void pack_x_kernel(const __nv_bfloat16 *__restrict__ x, int n8,
                              __half *__restrict__ x16, int fmt, int *status) {
  grid_dependency_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  bool over;
  const uint4 raw = *reinterpret_cast<const uint4 *>(x + (size_t)i * 8);
  const uint4 o = fmt == kFmtInt4 ? pack8_bf16_to_f16<kFmtInt4>(raw, over)
                                  : pack8_bf16_to_f16<kFmtNvfp4>(raw, over);
  if (over) set_status(status, STATUS_RANGE);
  *reinterpret_cast<uint4 *>(x16 + (size_t)i * 8) = o;
}

// ---------------------------------------------------------------- bucketing
// Pair counts per expert id.  Ids outside [0, E) are flagged and skipped.
__global__ void bucket_count_kernel(const int32_t *__restrict__ idx, int T, int k, int E,
                                    int *__restrict__ cnt, int *status) {
  grid_dependency_wait();
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= T * k) return;
  const int e = idx[p];
  if (e < 0 || e >= E) {
    set_status(status, STATUS_BAD_ROUTING);
    return;
  }
  atomicAdd(&cnt[e], 1);
}

// One block per expert id (E routed + S shared).  Computes the id's offset
// and active-list position from the counts, then writes its pairs in token
// order.  cnt of shared ids is T (set here).
__global__ void __launch_bounds__(256) bucket_fill_kernel(const int32_t *__restrict__ idx, int T,
                                                          int k, int E, int S, Routing rt) {
  grid_dependency_wait();
  const int id = blockIdx.x;
  const int nid = E + S;
  const int tid = threadIdx.x;
  __shared__ int s_sum[8], s_act[8];
  __shared__ int s_base;
  // offset = sum of counts of lower ids; active rank = number of lower ids in use
  int part = 0, act = 0;
  for (int i = tid; i < id; i += blockDim.x) {
    const int c = i < E ? rt.cnt[i] : T;
    part += c;
    act += c > 0;
  }
  for (int o = 16; o > 0; o >>= 1) {
    part += __shfl_xor_sync(0xffffffffu, part, o);
    act += __shfl_xor_sync(0xffffffffu, act, o);
  }
  if ((tid & 31) == 0) {
    s_sum[tid >> 5] = part;
    s_act[tid >> 5] = act;
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0, a = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      off += s_sum[i];
      a += s_act[i];
    }
    const int mine = id < E ? rt.cnt[id] : T;
    if (id >= E) rt.cnt[id] = T;
    rt.off[id] = off;
    if (mine > 0) rt.active[a] = id;
    if (id == nid - 1) {
      rt.off[nid] = off + mine;
      *rt.n_active = a + (mine > 0);
    }
    s_base = off;
  }
  __syncthreads();
  const int base = s_base;
  const int kS = k + S;
  if (id >= E) {
    const int j = k + (id - E);
    for (int t = tid; t < T; t += blockDim.x) {
      rt.pair_tok[base + t] = t;
      rt.pair_j[base + t] = j;
      rt.inv[(size_t)t * kS + j] = base + t;
    }
    return;
  }
  // routed: ordered compaction of the pairs p = t*k + j with idx[p] == id
  __shared__ int s_wcnt[8];
  int running = 0;
  const int n = T * k;
  for (int p0 = 0; p0 < n; p0 += blockDim.x) {
    const int p = p0 + tid;
    const bool m = p < n && idx[p] == id;
    const unsigned bal = __ballot_sync(0xffffffffu, m);
    if ((tid & 31) == 0) s_wcnt[tid >> 5] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int wi = 0; wi < (int)(blockDim.x >> 5); ++wi) {
      if (wi < (tid >> 5)) before += s_wcnt[wi];
      total += s_wcnt[wi];
    }
    if (m) {
      const int pos = base + running + before + __popc(bal & ((1u << (tid & 31)) - 1u));
      const int t = p / k, j = p % k;
      rt.pair_tok[pos] = t;
      rt.pair_j[pos] = j;
      rt.inv[(size_t)t * kS + j] = pos;
    }
    running += total;
    __syncthreads();
  }
}

// ---------------------------------------------------------------- combine
// out[t][r] = bf16( sum_j w[t][j] * y[inv[t][j]][r] + sum_s y[inv[t][k+s]][r] )
// in fp32, in that order.  A token with an invalid expert (or, with
// check_bound, an unbound one) gets a zero row.  Each thread handles 4 consecutive r.
__global__ void combine_kernel(const float *__restrict__ y, const int32_t *__restrict__ idx,
                               const float *__restrict__ w, const int *__restrict__ inv,
                               ExpertTable table, int check_bound, int T, int H, int k, int S,
                               int E, __nv_bfloat16 *__restrict__ out) {
  grid_dependency_wait();
  const int t = blockIdx.y;
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (t >= T || r >= H) return;
  const int kS = k + S;
  bool ok = true;
  for (int j = 0; j < k; ++j) {
    const int e = idx[(size_t)t * k + j];
    if (e < 0 || e >= E || (check_bound && !table.ptr[e]) || inv[(size_t)t * kS + j] < 0)
      ok = false;
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (ok) {
    for (int j = 0; j < kS; ++j) {
      const float wj = j < k ? w[(size_t)t * k + j] : 1.0f;
      const float4 v = *reinterpret_cast<const float4 *>(y + (size_t)inv[(size_t)t * kS + j] * H + r);
      if (j < k) {
        acc.x = __fadd_rn(acc.x, __fmul_rn(wj, v.x));
        acc.y = __fadd_rn(acc.y, __fmul_rn(wj, v.y));
        acc.z = __fadd_rn(acc.z, __fmul_rn(wj, v.z));
        acc.w = __fadd_rn(acc.w, __fmul_rn(wj, v.w));
      } else {
        acc.x = __fadd_rn(acc.x, v.x);
        acc.y = __fadd_rn(acc.y, v.y);
        acc.z = __fadd_rn(acc.z, v.z);
        acc.w = __fadd_rn(acc.w, v.w);
      }
    }
  }
  __nv_bfloat162 o0 = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 o1 = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t *>(&o0);
  packed.y = *reinterpret_cast<uint32_t *>(&o1);
  *reinterpret_cast<uint2 *>(out + (size_t)t * H + r) = packed;
}

// ---------------------------------------------------------------- small batches
// Routing only (strata_moe_route) of up to kSmallT tokens in one launch.
// Every block computes the logits of one expert (8 warps split h; per-warp
// double sums added in a fixed order); the last block to finish -- found with
// a device counter, each block's writes released by a fence before its
// counter increment and acquired by the last block with a fence after it --
// takes the top-k of every token and resets the counter for the next launch.
__global__ void __launch_bounds__(256) route_small_kernel(SmallRouteParams p) {
  grid_dependency_wait();
  __shared__ double s_part[8][kSmallT];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = p.T, H = p.H, E = p.E, k = p.k;
  {
    const int e = blockIdx.x;
    const float *wr = p.W + (size_t)e * H;
    const int span = H / 8;
    const int h0 = warp * span;
    for (int t0 = 0; t0 < T; t0 += 8) {
      const int nt = min(8, T - t0);
      double acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0;
#pragma unroll 2
      for (int h = h0 + lane * 4; h < h0 + span; h += 128) {
        const float4 wv = *reinterpret_cast<const float4 *>(wr + h);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (i < nt) {
            const uint2 raw = *reinterpret_cast<const uint2 *>(p.x + (size_t)(t0 + i) * H + h);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
            acc[i] = fma((double)a.x, (double)wv.x, acc[i]);
            acc[i] = fma((double)a.y, (double)wv.y, acc[i]);
            acc[i] = fma((double)b.x, (double)wv.z, acc[i]);
            acc[i] = fma((double)b.y, (double)wv.w, acc[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
      }
      if (lane == 0)
        for (int i = 0; i < nt; ++i) s_part[warp][t0 + i] = acc[i];
    }
    __syncthreads();
    for (int t = tid; t < T; t += blockDim.x) {
      double v = s_part[0][t];
#pragma unroll
      for (int w = 1; w < 8; ++w) v += s_part[w][t];
      if (p.bias) v += (double)p.bias[e];
      p.logits[(size_t)t * E + e] = (float)v;
    }
  }
  // ---- hand over to the last block
  if (gridDim.x > 1) {
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const int prev = atomicAdd(p.counter, 1);
      s_last = prev == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
  }
  for (int t = warp; t < T; t += 8) {
    int e;
    float wt;
    select_topk_warp(p.logits + (size_t)t * E, E, k, p.mode, lane, e, wt);
    if (lane < k) {
      p.idx[(size_t)t * k + lane] = e;
      p.w[(size_t)t * k + lane] = wt;
    }
  }
  if (tid == 0 && gridDim.x > 1) *p.counter = 0;
}

}  // namespace strata
