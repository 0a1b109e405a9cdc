// Expert matmuls for small token counts per expert (decode): int4 weights
// dequantised in registers, contracted on the legacy tensor-core path.
//
// What it computes (the W4A16 expert FFN of ro99/strata README, model table
// and "Kernels"): for every active expert and every pair routed to it,
//   gate/up pass:  h = silu(sum_k sg*qg*x) * (sum_k su*qu*x)   -> h16 (f16)
//   down pass:     y = sum_i sd*qd*h                          -> y (fp32)
// with one fp16 scale per 32 consecutive k.
//
// How:
//  * A persistent grid; CTA b takes a contiguous range of work items
//    (expert, group of <= 16 pairs, 32-row weight tile), so equal numbers of
//    weight bytes land on every SM.
//  * Warp 0 streams each item's K range in chunks of kc through a 4-stage
//    shared-memory ring: 32 packed weight rows as bulk async copies (one per
//    row, rows padded by 16 bytes so the ldmatrix reads below are free of
//    bank conflicts), their fp16 scales as 4-byte async copies, and the
//    activation rows of the item's pairs as bulk copies.  Completion is
//    counted on an mbarrier per stage.
//  * Warps 1-4 split each chunk into 64-element steps.  ldmatrix hands every
//    thread exactly the 32-bit word of nibbles its mma A fragment needs (row
//    g and g+8, word c of a 16-byte quant block); int4x8_to_f16 turns it into
//    exact f16 integers; two m16n8k16 MMAs per quant block give the block's
//    integer-weight dot products in fp32, which are scaled by the block's
//    fp16 scale into fp32 accumulators (so the only rounding of a weight is
//    none at all -- q and the scale are applied exactly, the activation is
//    rounded to f16).
//  * The four warps' partial sums are added in a fixed order; SwiGLU needs
//    no exchange because a thread holds the gate and the up value of the same
//    (row, pair) position.
#include "common.cuh"
#include "kernels.h"

namespace strata {

namespace {

__device__ __forceinline__ void cp_async_4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// lane 0 waits, the result is shared with the warp
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

constexpr int kRedFloats = 4 * 2 * 2 * 32 * 4;  // [warp][m][n-tile][lane][4]

struct Item {
  const uint8_t *blob;
  int id, tau, pi0, ntok;
};

__device__ __forceinline__ Item decode_item(const MmParams &p, const int *item_base, int &a,
                                            int i) {
  while (item_base[a + 1] <= i) ++a;
  Item it;
  it.id = p.rt.active[a];
  const int rem = i - item_base[a];
  const int g = rem / p.tiles;
  it.tau = rem - g * p.tiles;
  const int c = p.rt.cnt[it.id];
  it.pi0 = p.rt.off[it.id] + g * kMmGroup;
  it.ntok = min(kMmGroup, c - g * kMmGroup);
  it.blob = p.table.ptr[it.id];
  return it;
}

}  // namespace

size_t mm_smem_bytes(const MmParams &p) {
  return (size_t)kMmStages * p.stage_bytes + (2 * kMmStages + 2) * sizeof(uint64_t) +
         kRedFloats * sizeof(float) + (kMaxIds + 1) * sizeof(int);
}

template <bool kGateUp>
__global__ void __launch_bounds__(kMmThreads, 1) expert_mma_kernel(MmParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *stages = smem;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kMmStages * p.stage_bytes);
  uint64_t *empty = full + kMmStages;
  uint64_t *red_full = empty + kMmStages;  // partial sums of all 4 consumer warps written
  uint64_t *red_free = red_full + 1;       // consumer warp 0 has read them
  float *red = reinterpret_cast<float *>(red_free + 1);
  int *item_base = reinterpret_cast<int *>(red + kRedFloats);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMmStages; ++s) {
      mbar_init(&full[s], 1 + 32);  // producer's expect_tx arrive + 32 cp.async arrivals
      mbar_init(&empty[s], 4);      // one arrive per consumer warp
    }
    mbar_init(red_full, 4);
    mbar_init(red_free, 1);
    fence_mbar_init();
  }
  grid_dependency_wait();

  // items per active expert -> exclusive prefix (warp 0, 32 ids at a time)
  const int n_active = *p.rt.n_active;
  if (warp == 0) {
    int carry = 0;
    for (int a0 = 0; a0 < n_active; a0 += 32) {
      const int a = a0 + lane;
      int v = 0;
      if (a < n_active) {
        const int c = p.rt.cnt[p.rt.active[a]];
        v = ((c + kMmGroup - 1) / kMmGroup) * p.tiles;
      }
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (a < n_active) item_base[a] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) item_base[n_active] = carry;
  }
  __syncthreads();
  grid_dependency_launch();

  const int n_items = item_base[n_active];
  const int i_begin = (int)((long long)n_items * blockIdx.x / gridDim.x);
  const int i_end = (int)((long long)n_items * (blockIdx.x + 1) / gridDim.x);
  const int n_chunks = p.K / p.kc;
  const int steps = p.kc / 64;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t chunk = 0;
    int a = 0;
    bool alive = true;
    for (int i = i_begin; i < i_end && alive; ++i) {
      const Item it = decode_item(p, item_base, a, i);
      if (!it.blob) {
        if (lane == 0) set_status(p.status, STATUS_NOT_BOUND);
        continue;
      }
      int brow = 0;
      if (lane < it.ntok) brow = kGateUp ? p.rt.pair_tok[it.pi0 + lane] : it.pi0 + lane;
      const int m = lane >> 4;
      const int row = it.tau * p.row_base_mul + p.row_half[m] + (lane & 15);
      const uint8_t *wrow = it.blob + p.q_off[m] + (size_t)row * (p.K / 2);
      const uint8_t *srow = it.blob + p.s_off[m] + (size_t)row * (p.K / 32) * 2;
      const __half *brow_src = p.b_src + (size_t)brow * p.K;
      for (int c = 0; c < n_chunks; ++c, ++chunk) {
        const int s = chunk % kMmStages;
        const uint32_t ph = (chunk / kMmStages) & 1u;
        if (!warp_wait(&empty[s], ph ^ 1u, p.status)) {
          alive = false;
          break;
        }
        uint8_t *st = stages + s * p.stage_bytes;
        const uint8_t *ssrc = srow + (size_t)c * (p.kc / 32) * 2;
        uint8_t *sdst = st + p.w_bytes + lane * p.sstride;
        for (int u = 0; u < steps; ++u) cp_async_4(sdst + 4 * u, ssrc + 4 * u);
        cp_async_mbar_arrive_noinc(&full[s]);
        __syncwarp();
        if (lane == 0)
          mbar_arrive_expect_tx(&full[s], 32u * (p.kc / 2) + (uint32_t)it.ntok * p.kc * 2u);
        __syncwarp();
        bulk_g2s(st + lane * p.wstride, wrow + (size_t)c * (p.kc / 2), p.kc / 2, &full[s]);
        if (lane < it.ntok)
          bulk_g2s(st + p.w_bytes + p.s_bytes + lane * p.bstride, brow_src + (size_t)c * p.kc,
                   p.kc * 2, &full[s]);
      }
    }
    if (!alive) {
      // wind down: let every stage's copies land before the CTA exits
      for (int s = 0; s < kMmStages && s < (int)chunk; ++s) {
        const uint32_t last = chunk - 1 - ((chunk - 1 - s) % kMmStages);
        (void)warp_wait(&full[last % kMmStages], (last / kMmStages) & 1u, p.status);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int g = lane >> 2, cq = lane & 3;
  uint32_t chunk = 0, done = 0;
  int a = 0;
  for (int i = i_begin; i < i_end; ++i) {
    const Item it = decode_item(p, item_base, a, i);
    if (!it.blob) continue;
    const int ntn = (it.ntok + 7) >> 3;
    float acc[2][2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[m][n][v] = 0.0f;

    for (int c = 0; c < n_chunks; ++c, ++chunk) {
      const int s = chunk % kMmStages;
      const uint32_t ph = (chunk / kMmStages) & 1u;
      if (!warp_wait(&full[s], ph, p.status)) return;
      const uint8_t *st = stages + s * p.stage_bytes;
      const uint32_t w_addr = smem_u32(st);
      const uint8_t *sreg = st + p.w_bytes;
      const uint8_t *breg = st + p.w_bytes + p.s_bytes;
      for (int step = cw; step < steps; step += 4) {
        float sc[2][2][2];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const uint32_t v =
                *reinterpret_cast<const uint32_t *>(sreg + (m * 16 + g + 8 * hr) * p.sstride + step * 4);
            const float2 f = __half22float2(bits_h2(v));
            sc[m][hr][0] = f.x;
            sc[m][hr][1] = f.y;
          }
        uint32_t f16w[2][4][4];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          uint32_t q[4];
          const int r = m * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
          ldmatrix_x4(q, w_addr + r * p.wstride + step * 32 + (lane >> 4) * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j) int4x8_to_f16(q[j], f16w[m][j]);
        }
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            if (nt < ntn) {
              const uint4 bv = *reinterpret_cast<const uint4 *>(
                  breg + (nt * 8 + g) * p.bstride + (step * 64 + bb * 32 + cq * 8) * 2);
#pragma unroll
              for (int m = 0; m < 2; ++m) {
                const uint32_t a0[4] = {f16w[m][2 * bb][0], f16w[m][2 * bb + 1][0],
                                        f16w[m][2 * bb][1], f16w[m][2 * bb + 1][1]};
                const uint32_t a1[4] = {f16w[m][2 * bb][2], f16w[m][2 * bb + 1][2],
                                        f16w[m][2 * bb][3], f16w[m][2 * bb + 1][3]};
                const float zero[4] = {0.f, 0.f, 0.f, 0.f};
                float d[4];
                mma_16816(d, a0, bv.x, bv.y, zero);
                mma_16816(d, a1, bv.z, bv.w, d);
                acc[m][nt][0] = fmaf(sc[m][0][bb], d[0], acc[m][nt][0]);
                acc[m][nt][1] = fmaf(sc[m][0][bb], d[1], acc[m][nt][1]);
                acc[m][nt][2] = fmaf(sc[m][1][bb], d[2], acc[m][nt][2]);
                acc[m][nt][3] = fmaf(sc[m][1][bb], d[3], acc[m][nt][3]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ------------------------------------------------------------ epilogue
    // the previous item's partial sums must have been read
    if (!warp_wait(red_free, (done & 1u) ^ 1u, p.status)) return;
    float *mine = red + cw * (2 * 2 * 32 * 4);
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int v = 0; v < 4; ++v) mine[((m * 2 + nt) * 32 + lane) * 4 + v] = acc[m][nt][v];
    __syncwarp();
    if (lane == 0) mbar_arrive(red_full);
    if (cw == 0) {
      if (!warp_wait(red_full, done & 1u, p.status)) return;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        if (nt >= ntn) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int rr = g + 8 * (v >> 1);
          const int n = nt * 8 + 2 * cq + (v & 1);
          if (n >= it.ntok) continue;
          float fin[2];
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const int o = ((m * 2 + nt) * 32 + lane) * 4 + v;
            fin[m] = ((red[o] + red[o + 2 * 2 * 32 * 4]) + red[o + 2 * 2 * 2 * 32 * 4]) +
                     red[o + 3 * 2 * 2 * 32 * 4];
          }
          const size_t prow = (size_t)(it.pi0 + n) * p.out_ld;
          if (kGateUp) {
            const float gv = fin[0], uv = fin[1];
            const float h = gv / (1.0f + expf(-gv)) * uv;
            const int ii = it.tau * 16 + rr;
            // stored like the packed activations: group of 8 in order 0,4,1,5,2,6,3,7
            const int pos = (ii & ~7) | (((ii & 3) << 1) | ((ii >> 2) & 1));
            p.h_out[prow + pos] = __float2half_rn(h);
          } else {
            const int r0 = it.tau * 32 + rr;
            p.y_out[prow + r0] = fin[0];
            p.y_out[prow + r0 + 16] = fin[1];
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(red_free);
    }
    ++done;
  }
}

template __global__ void expert_mma_kernel<true>(MmParams);
template __global__ void expert_mma_kernel<false>(MmParams);

}  // namespace strata
