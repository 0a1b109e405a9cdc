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
//  * Work item = (active expert, group of <= 16 of its pairs, one 16-row
//    weight tile): for gate/up, 8 rows of Wg and the same 8 rows of Wu (so a
//    thread holds gate and up of one (row, pair) and SwiGLU is local); for
//    down, 16 rows of Wd.  The (item, K group) pairs of the pass, laid end to
//    end, are cut into one equal contiguous range per warp of the persistent
//    grid (every warp streams the same number of weight bytes, to within one
//    group).  An item that a cut splits is finished by the last of its
//    pieces, which adds the pieces' partial sums in piece order (fixed, so
//    the result does not depend on timing); all other items are computed
//    whole by one warp, with no cross-warp reduction.
//  * The blob stores a tile K-group by K-group, so any K chunk of a tile is
//    one contiguous run of bytes.  Each warp streams its own items' chunks
//    through a private ring of shared-memory stages: its lane 0 issues one
//    bulk async copy of packed weights and one of scales per stage, a few
//    stages ahead, completion counted in transaction bytes on the stage's
//    mbarrier.  (Many independent rings per SM keep HBM busy; one ring fed by
//    one thread could not.)
//  * For a K group, one 16-byte shared-memory load per row hands thread
//    (g, c) word c of all four quant blocks of rows g and g+8 -- exactly its
//    mma.m16n8k16 A-fragment words -- and int4x8_to_f16 turns each word into
//    exact f16 integers.  Two MMAs per quant block give the block's
//    integer-weight dot products in fp32, scaled by the block's fp16 scale
//    into fp32 accumulators: the weights are applied exactly; the activations
//    are f16.
//  * Activation fragments (x16 or h16 rows of the item's pairs) are read from
//    L2 one group ahead, across item boundaries.
#include "common.cuh"
#include "kernels.h"

namespace strata {

namespace {

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Orders this thread's earlier shared-memory reads before later async-proxy
// (bulk copy) writes to the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Spin (with back-off and a time limit) until *counter reaches `target`;
// acquire ordering for the reads that follow.
__device__ __forceinline__ bool wait_count(const int *counter, int target, int *status) {
  const uint64_t t0 = global_timer_ns();
  unsigned ns = 32;
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
    if (v >= target) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      set_status(status, STATUS_TIMEOUT);
      return false;
    }
    __nanosleep(ns);
    if (ns < 512) ns <<= 1;
  }
}

struct Item {
  const uint8_t *blob;
  int tau, pi0, ntok;
};

// Per active expert, staged in shared memory at kernel start.
struct ActiveTable {
  const uint8_t **blob;
  int *off, *cnt;
};

__device__ __forceinline__ Item decode_item(const MmParams &p, const ActiveTable &at,
                                            const int *item_base, int &a, int i) {
  while (item_base[a + 1] <= i) ++a;
  Item it;
  const int rem = i - item_base[a];
  const int g = rem / p.tiles;
  it.tau = rem - g * p.tiles;
  it.pi0 = at.off[a] + g * p.group;
  it.ntok = min(p.group, at.cnt[a] - g * p.group);
  it.blob = at.blob[a];
  return it;
}

// Activation fragments of one K group for a token row: v[b] = 8 f16 at
// k0 + 32 b + 8 c (stored in the 0,4,1,5,2,6,3,7 order).  For a padding
// column (no token, row == nullptr) the registers keep whatever they hold:
// that column of the MMA result is never read.
__device__ __forceinline__ void load_b(uint4 v[4], const __half *row, int k0, int cq) {
  if (row) {
#pragma unroll
    for (int b = 0; b < 4; ++b) v[b] = ld_nc_v4(row + k0 + 32 * b + 8 * cq);
  }
}

}  // namespace

size_t mm_fixed_smem_bytes() {
  return (size_t)kMmWarps * kMmMaxStages * sizeof(uint64_t) + kMaxIds * sizeof(void *) +
         (3 * kMaxIds + 1) * sizeof(int) + kMmMaxPairs * sizeof(int);
}

size_t mm_smem_bytes(const MmParams &p) {
  return (size_t)kMmWarps * p.stages * p.stage_bytes + mm_fixed_smem_bytes();
}

template <bool kGateUp, int NT>
__global__ void __launch_bounds__(kMmThreads, 1) expert_mma_kernel(MmParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t *ring = smem + (size_t)warp * p.stages * p.stage_bytes;   // this warp's stages
  uint64_t *full_all =
      reinterpret_cast<uint64_t *>(smem + (size_t)kMmWarps * p.stages * p.stage_bytes);
  uint64_t *full = full_all + warp * kMmMaxStages;
  ActiveTable at;
  at.blob = reinterpret_cast<const uint8_t **>(full_all + kMmWarps * kMmMaxStages);
  int *item_base = reinterpret_cast<int *>(at.blob + kMaxIds);
  at.off = item_base + kMaxIds + 1;
  at.cnt = at.off + kMaxIds;
  int *s_ptok = at.cnt + kMaxIds;   // token of each sorted pair (gate/up)

  if (lane == 0)
    for (int s = 0; s < p.stages; ++s) mbar_init(&full[s], 1);
  if (threadIdx.x == 0) fence_mbar_init();
  grid_dependency_wait();

  // active experts: table in shared memory, then items per expert ->
  // exclusive prefix (warp 0, 32 experts at a time)
  const int n_active = *p.rt.n_active;
  const int n_pairs = p.rt.off[p.n_ids];
  for (int a = threadIdx.x; a < n_active; a += blockDim.x) {
    const int id = p.rt.active[a];
    at.blob[a] = p.table.ptr[id];
    at.off[a] = p.rt.off[id];
    at.cnt[a] = p.rt.cnt[id];
  }
  if (kGateUp)
    for (int q = threadIdx.x; q < n_pairs && q < kMmMaxPairs; q += blockDim.x)
      s_ptok[q] = p.rt.pair_tok[q];
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int a0 = 0; a0 < n_active; a0 += 32) {
      const int a = a0 + lane;
      int v = 0;
      if (a < n_active) v = ((at.cnt[a] + p.group - 1) / p.group) * p.tiles;
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
  const int gpc = p.kc / 128;                    // K groups per (full) chunk
  const int groups = p.K / 128;                  // K groups per tile row
  const uint32_t q_stage = (uint32_t)p.kc * 8;   // scale offset inside a stage
  const int g = lane >> 2, cq = lane & 3;

  // This warp's share of the (item, group) sequence: [x_lo, x_hi); the
  // first r = total mod W warps take q + 1 groups, the others q.
  const int W = (int)gridDim.x * kMmWarps;
  const int wg = (int)blockIdx.x * kMmWarps + warp;
  const int total = n_items * groups;
  const int q = total / W, r = total - (total / W) * W;
  auto cut = [&](int w) -> int { return w * q + min(w, r); };
  auto warp_of = [&](int x) -> int {  // the warp whose share holds x
    return x < r * (q + 1) ? x / (q + 1) : r + (x - r * (q + 1)) / q;
  };
  const int x_lo = cut(wg), x_hi = cut(wg + 1);

  // A piece: groups [g0, g1) of item `item`; x is its start in the sequence.
  // Pieces of unbound experts are skipped and flagged.
  struct Piece {
    int item, g0, g1;
  };
  auto piece_at = [&](int x, int &a_hint, Piece &pc) -> bool {
    while (x < x_hi) {
      pc.item = x / groups;
      pc.g0 = x - pc.item * groups;
      pc.g1 = min(groups, pc.g0 + (x_hi - x));
      while (item_base[a_hint + 1] <= pc.item) ++a_hint;
      if (at.blob[a_hint]) return true;
      if (lane == 0) set_status(p.status, STATUS_NOT_BOUND);
      x += pc.g1 - pc.g0;
    }
    return false;
  };

  // ---- copy issue: this warp's pieces in order, gpc groups per stage
  int a_issue = 0;
  Piece pc_issue;
  int x_issue = x_lo;
  bool have_issue = piece_at(x_issue, a_issue, pc_issue);
  int cg_issue = have_issue ? pc_issue.g0 : 0;   // next group to copy
  uint32_t s_issue = 0;
  auto issue_next = [&]() {
    if (!have_issue) return;
    const Item it = decode_item(p, at, item_base, a_issue, pc_issue.item);
    const int slot = (int)(s_issue % p.stages);
    uint8_t *dst = ring + slot * p.stage_bytes;
    const int ng = min(gpc, pc_issue.g1 - cg_issue);
    if (lane == 0) {
      const size_t g0 = (size_t)it.tau * groups + (size_t)cg_issue;
      mbar_arrive_expect_tx(&full[slot], (uint32_t)ng * (1024u + 128u));
      bulk_g2s(dst, it.blob + p.q_off + g0 * 1024, (uint32_t)ng * 1024u, &full[slot]);
      bulk_g2s(dst + q_stage, it.blob + p.s_off + g0 * 128, (uint32_t)ng * 128u, &full[slot]);
    }
    ++s_issue;
    cg_issue += ng;
    if (cg_issue == pc_issue.g1) {
      x_issue += pc_issue.g1 - pc_issue.g0;
      have_issue = piece_at(x_issue, a_issue, pc_issue);
      if (have_issue) cg_issue = pc_issue.g0;
    }
  };
  for (int s = 0; s < p.stages; ++s) issue_next();

  // ---- compute
  auto act_row = [&](const Item &it, int nt) -> const __half * {
    const int n = nt * 8 + g;
    if (n >= it.ntok) return nullptr;
    int src;
    if (kGateUp) {
      const int q = it.pi0 + n;
      src = q < kMmMaxPairs ? s_ptok[q] : p.rt.pair_tok[q];
    } else {
      src = it.pi0 + n;
    }
    return p.b_src + (size_t)src * p.K;
  };
  // Output of one (pair n, row g / g + 8) element pair of an item.
  auto emit = [&](const Item &it, int n, float lo, float hi) {
    const size_t prow = (size_t)(it.pi0 + n) * p.out_ld;
    if (kGateUp) {
      // lo: gate row i, hi: up row i, i = 8 tau + g
      const float h = lo / (1.0f + expf(-lo)) * hi;
      const int ii = it.tau * 8 + g;
      // stored like the packed activations: group of 8 in order 0,4,1,5,2,6,3,7
      const int pos = (ii & ~7) | (((ii & 3) << 1) | ((ii >> 2) & 1));
      if (fabsf(h) >= kF16Overflow) set_status(p.status, STATUS_RANGE);
      p.h_out[prow + pos] = __float2half_rn(h);
    } else {
      const int r0 = it.tau * 16 + g;
      p.y_out[prow + r0] = lo;
      p.y_out[prow + r0 + 8] = hi;
    }
  };
  uint4 bb0[NT][4], bb1[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int b = 0; b < 4; ++b) bb0[nt][b] = bb1[nt][b] = make_uint4(0u, 0u, 0u, 0u);
  int pb = 0;  // buffer holding the current group's fragments
  int a = 0;
  Piece pc;
  int x = x_lo;
  bool have = piece_at(x, a, pc);
  if (have) {
    int a_tmp = a;
    const Item it0 = decode_item(p, at, item_base, a_tmp, pc.item);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) load_b(bb0[nt], act_row(it0, nt), pc.g0 * 128, cq);
  }
  uint32_t s_use = 0;
  while (have) {
    const Item it = decode_item(p, at, item_base, a, pc.item);
    const int ntn = (it.ntok + 7) >> 3;
    int a_nx = a;
    Piece pc_nx;
    const bool have_nx = piece_at(x + (pc.g1 - pc.g0), a_nx, pc_nx);
    const __half *row_cur[NT], *row_nx[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      row_cur[nt] = act_row(it, nt);
      row_nx[nt] = nullptr;
    }
    if (have_nx) {
      int a_tmp = a_nx;
      const Item it_nx = decode_item(p, at, item_base, a_tmp, pc_nx.item);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) row_nx[nt] = act_row(it_nx, nt);
    }
    // acc[nt][0] = (row g: pair 2c, 2c + 1), acc[nt][1] = (row g + 8: same pairs)
    float2 acc[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = make_float2(0.0f, 0.0f);

    for (int cg = pc.g0; cg < pc.g1; ++s_use) {
      const int slot = (int)(s_use % p.stages);
      if (!warp_wait(&full[slot], (s_use / p.stages) & 1u, p.status)) return;
      const uint8_t *stq = ring + slot * p.stage_bytes;
      const uint8_t *sts = stq + q_stage;
      const int ng = min(gpc, pc.g1 - cg);
#pragma unroll 4
      for (int j = 0; j < ng; ++j) {
        // fragments of the next group: this piece, else the next piece
        {
          const int G_next = cg + j + 1;
          const bool same = G_next < pc.g1;
          if (same || have_nx) {
            const int k0 = (same ? G_next : pc_nx.g0) * 128;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const __half *r = same ? row_cur[nt] : row_nx[nt];
              if (pb == 0) load_b(bb1[nt], r, k0, cq);
              else load_b(bb0[nt], r, k0, cq);
            }
          }
        }
        // weights and scales of rows g and g + 8
        const uint4 w0 = *reinterpret_cast<const uint4 *>(stq + j * 1024 + g * 64 + cq * 16);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(stq + j * 1024 + (g + 8) * 64 + cq * 16);
        const uint2 s0 = *reinterpret_cast<const uint2 *>(sts + j * 128 + g * 8);
        const uint2 s1 = *reinterpret_cast<const uint2 *>(sts + j * 128 + (g + 8) * 8);
        const uint32_t wr0[4] = {w0.x, w0.y, w0.z, w0.w};  // word c of blocks 0..3, row g
        const uint32_t wr1[4] = {w1.x, w1.y, w1.z, w1.w};  // row g + 8
        uint32_t f0[4][4], f1[4][4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          int4x8_to_f16(wr0[b], f0[b]);
          int4x8_to_f16(wr1[b], f1[b]);
        }
        float sc0[4], sc1[4];
        {
          float2 f;
          f = __half22float2(bits_h2(s0.x)); sc0[0] = f.x; sc0[1] = f.y;
          f = __half22float2(bits_h2(s0.y)); sc0[2] = f.x; sc0[3] = f.y;
          f = __half22float2(bits_h2(s1.x)); sc1[0] = f.x; sc1[1] = f.y;
          f = __half22float2(bits_h2(s1.y)); sc1[2] = f.x; sc1[3] = f.y;
        }
        auto mma_group = [&](const uint4 (&bv)[NT][4]) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (NT == 1 || nt < ntn) {
              float d[4][4];
              const float zero[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const uint32_t a0[4] = {f0[b][0], f1[b][0], f0[b][1], f1[b][1]};
                mma_16816(d[b], a0, bv[nt][b].x, bv[nt][b].y, zero);
              }
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const uint32_t a1[4] = {f0[b][2], f1[b][2], f0[b][3], f1[b][3]};
                mma_16816(d[b], a1, bv[nt][b].z, bv[nt][b].w, d[b]);
              }
#pragma unroll
              for (int b = 0; b < 4; ++b) {  // paired fp32 FMAs (same rounding as two fmaf)
                acc[nt][0] = __ffma2_rn(make_float2(sc0[b], sc0[b]), make_float2(d[b][0], d[b][1]),
                                        acc[nt][0]);
                acc[nt][1] = __ffma2_rn(make_float2(sc1[b], sc1[b]), make_float2(d[b][2], d[b][3]),
                                        acc[nt][1]);
              }
            }
          }
        };
        if (pb == 0) mma_group(bb0); else mma_group(bb1);
        pb ^= 1;
      }
      cg += ng;
      // the stage's bytes are in registers now: refill it
      fence_proxy_async_smem();
      __syncwarp();
      issue_next();
    }

    // ---- epilogue
    if (pc.g0 == 0 && pc.g1 == groups) {
      // the whole item: this warp holds its complete sums
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const int n = nt * 8 + 2 * cq + v;
          if (nt < ntn && n < it.ntok) emit(it, n, (v ? acc[nt][0].y : acc[nt][0].x), (v ? acc[nt][1].y : acc[nt][1].x));
        }
    } else {
      // one piece of an item cut by warp shares.  Its pieces belong to the
      // warps w_first .. w_last with non-empty shares; w_first's piece comes
      // at the end of its share, the others at the start of theirs.  Each
      // other piece stores its partial sums in its warp's slot and counts
      // itself on w_first's counter (release: fence before the increment);
      // w_first waits for them (acquire), adds the slots in warp order to
      // its own sums and emits.
      const int x_item = pc.item * groups;
      const int w_first = warp_of(x_item), w_last = warp_of(x_item + groups - 1);
      if (pc.g0 > 0) {
        float *mine = p.partial + (size_t)wg * kMmSlotFloats;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int n = nt * 8 + 2 * cq + v;
            if (nt < ntn && n < it.ntok) {
              mine[n * 16 + g] = v ? acc[nt][0].y : acc[nt][0].x;
              mine[n * 16 + g + 8] = v ? acc[nt][1].y : acc[nt][1].x;
            }
          }
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          atomicAdd(&p.counters[w_first], 1);
        }
      } else {
        int others = 0;
        for (int w = w_first + 1; w <= w_last; ++w) others += cut(w + 1) > cut(w);
        int ok = 1;
        if (lane == 0) ok = wait_count(&p.counters[w_first], others, p.status) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) return;
        __threadfence();
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int n = nt * 8 + 2 * cq + v;
            if (nt < ntn && n < it.ntok) {
              float lo = v ? acc[nt][0].y : acc[nt][0].x;
              float hi = v ? acc[nt][1].y : acc[nt][1].x;
              for (int w = w_first + 1; w <= w_last; ++w) {
                if (cut(w + 1) == cut(w)) continue;  // empty share: no piece
                const float *src = p.partial + (size_t)w * kMmSlotFloats;
                lo += __ldcg(src + n * 16 + g);
                hi += __ldcg(src + n * 16 + g + 8);
              }
              emit(it, n, lo, hi);
            }
          }
        __syncwarp();
        if (lane == 0) p.counters[w_first] = 0;  // ready for the next launch
      }
    }
    x += pc.g1 - pc.g0;
    pc = pc_nx;
    have = have_nx;
    a = a_nx;
  }
}

template __global__ void expert_mma_kernel<true, 1>(MmParams);
template __global__ void expert_mma_kernel<false, 1>(MmParams);
template __global__ void expert_mma_kernel<true, 2>(MmParams);
template __global__ void expert_mma_kernel<false, 2>(MmParams);

}  // namespace strata
