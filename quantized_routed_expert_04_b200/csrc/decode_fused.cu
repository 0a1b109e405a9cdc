// The whole layer for small batches (decode, up to 64 tokens) in one
// persistent, cooperative launch: router, top-k, bucketing, gate/up + SwiGLU,
// down projection and the weighted combine.
//
// What it computes (the layer of ro99/strata README, "Kernels": the W4A16
// routed-expert FFN; the fused router + top-k dispatch of "Strata on a Mac",
// "Switches"): logits = x . Wr[e] + b[e] (double sums, one rounding to fp32),
// the top_k experts and their weights, h = silu(Wg x) * (Wu x) per routed and
// shared expert, y = Wd h, and out = sum_j w_j y_j + sum_s y_s (fp32 in that
// order, one rounding to bf16).
//
// Why one launch: at decode sizes the expert weights take tens of
// microseconds to stream, while each extra launch costs a few microseconds of
// launch, prologue and tail.  Here the grid is one CTA per multiprocessor,
// all resident at once (cooperative launch), and the phases are separated by
// grid barriers: device counters, each CTA's writes released by a release
// reduction on the counter and acquired by the waiter's acquire loads (the
// relaxed-only hand-off of the fused Metal router in "Strata on a Mac",
// "Switches", is the failure this ordering avoids).  Every wait is bounded;
// a wait that gives up sets STATUS_TIMEOUT and the CTA winds down, still
// passing every barrier so that no other CTA waits on it.
//
// Phases:
//  R  every CTA packs a slice of x to f16 (range-checked); the router's
//     dot products are cut into units (expert, range of H) spread over every
//     CTA, each storing double partial sums.  Barrier.
//  K  logits = the units' partial sums added in a fixed order + bias, one
//     rounding to fp32; top-k: for up to 16 tokens every CTA selects all
//     tokens itself (one warp per token, the same inputs and code, so the
//     same result everywhere); for more tokens CTA c selects token c and a
//     second barrier publishes the choices.
//  B  every CTA buckets the (token, j) pairs in shared memory: counts,
//     offsets, the active experts, and a stable order by (expert, token), so
//     the layout is a pure function of the routing.
//  G  gate/up + SwiGLU -> h16;  D  down -> y, and the combine.  A down
//     piece starts once every gate/up item of its pair group has counted
//     itself done (a counter per group, release/acquire), not at a grid
//     barrier.
// G and D cut their (item, K group) sequences -- item = (active expert, <= 8
// or 16 of its pairs, one 16-row weight tile) -- into one equal contiguous
// share per warp of the grid, cut at whole ring stages.  Each warp streams
// its shares through its own ring of shared-memory stages filled by bulk
// async copies (lane 0: packed weights and scales, completing as transaction
// bytes on the stage's mbarrier); the ring runs on from the G share into the
// D share, so the first down weights are in flight while the warp waits for
// its first pair group.  The int4 words go from shared memory into
// mma.m16n8k16 A fragments.  int4: int4x8_to_f16 (exact
// integers), two MMAs per quant block, fp32 block-scale FMAs.  NVFP4: each
// code times its E4M3 group scale in f16 (exact: at most six significant
// bits, at most 2688 in magnitude), MMAs chained over the whole piece, and
// the fp32 global scale once at the end.  Either way the weights are applied
// exactly; the activations are f16.
// An item cut by share boundaries is finished by the last of its pieces to
// arrive: every piece stores its partial sums, counts itself on the item's
// counter, and the piece that completes the count adds all pieces' sums in
// warp order (fixed, whoever arrives last) and emits.  Nothing waits on a
// piece.  The combine works the same way: each emitted down item counts
// itself on its 16-row output tile, and the item that completes the tile
// writes that tile of every token's output.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace strata {

namespace {

constexpr int kFW = kFusedWarps;

struct Tables {
  const uint8_t **ptr;   // per expert id: the slot table (null: not bound)
  const uint8_t **blob;  // per active expert (null: not bound)
  int *aoff, *acnt;      // per active expert: first sorted pair, pair count
  int *gbase;            // per active expert: first pair group (prefix), [n_active + 1]
  int *cnt, *off;        // per expert id
  int *misc;             // [0] n_active, [1] pair groups of bound experts, [2] abort
  double *part;          // router partial sums [kFW][8]
  int *idx;              // [T][k] routed expert ids
  float *w;              // [T][k] routed weights
  int *ptok;             // [P] token of each sorted pair
  int *inv;              // [T][k + S] sorted position of pair (t, j), -1 if none
  int *bad;              // [T] token has an unbound or invalid expert
};

struct PhaseInfo {
  int tiles;            // 16-row weight tiles per expert
  int groups;           // K groups of 128 per tile row
  size_t q_off, s_off;  // weight and scale sections
  int x_lo, x_hi;       // this warp's share of the (item, group) sequence
  int q, r;             // share sizes: the first r warps take q + 1 stages
  int unit, total;      // K groups per stage, groups in the phase
};

struct Piece {
  int item, g0, g1;
};

struct Item {
  const uint8_t *blob;
  int tau, pi0, ntok;
};

struct Ring {
  uint8_t *base;
  uint64_t *full;
  int stages, stage_bytes;
  uint32_t issued, used;
};

struct Cursor {  // the copy-issue position, running over the G then the D pieces
  int ph, x, a, cg;
  Piece pc;
  bool have;
  const uint8_t *qsrc, *ssrc;  // the next stage's packed weights and scales
};

__device__ __forceinline__ uint4 ld_v4(const void *ptr) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}

__device__ __forceinline__ int ld_acquire(const int *ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

// Counter increments that publish the writes before them: a release
// reduction (the warp's other lanes' writes are ordered before it by a warp
// barrier), or an acquire-release add whose caller also reads what the
// earlier increments published.
__device__ __forceinline__ void red_release_add(int *ptr, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_acq_rel_add(int *ptr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v)
               : "memory");
  return old;
}

// Ring-stage wait of one warp: every lane tests the phase and the warp votes
// (no divergent branch when the stage is ready, the common case); else lane 0
// polls with the given limit, and once the phase is complete every lane
// observes it itself (acquiring the stage's bytes).
__device__ __forceinline__ bool warp_wait_limit(uint64_t *bar, uint32_t parity, int *status,
                                                unsigned long long limit_ns) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    if (!mbar_try_wait(bar, parity)) {
      const uint64_t t0 = global_timer_ns();
      while (true) {
        if (mbar_try_wait(bar, parity)) break;
        if (global_timer_ns() - t0 > limit_ns) {
          set_status(status, STATUS_TIMEOUT);
          ok = 0;
          break;
        }
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) (void)mbar_try_wait(bar, parity);
  return ok != 0;
}

// Grid barrier: every thread of every CTA calls it the same number of times.
// Thread 0 releases the CTA's writes (fence, then the counter increment) and
// waits, bounded, until every CTA has arrived (acquire).  A CTA that is
// winding down still arrives but does not wait.  Returns false once the CTA
// is winding down.
__device__ bool grid_sync(int *ctr, volatile int *abort_flag, int *status,
                          unsigned long long limit_ns) {
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(ctr) : "memory");
    if (!*abort_flag) {
      const uint64_t t0 = global_timer_ns();
      unsigned ns = 32;
      while (ld_acquire(ctr) < (int)gridDim.x) {
        if (global_timer_ns() - t0 > limit_ns) {
          set_status(status, STATUS_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        __nanosleep(ns);
        if (ns < 64) ns <<= 1;
      }
    }
  }
  __syncthreads();
  return !*abort_flag;
}

// Shares are whole ring stages (ph.unit K groups) of the phase's sequence of
// ph.total groups, so that a piece that starts a share starts a full stage.
__device__ __forceinline__ int share_cut(const PhaseInfo &ph, int w) {
  return min(ph.total, (w * ph.q + min(w, ph.r)) * ph.unit);
}

// The warp whose share holds position x.
__device__ __forceinline__ int share_owner(const PhaseInfo &ph, int x) {
  const int s = x / ph.unit;
  const int big = ph.r * (ph.q + 1);
  return s < big ? s / (ph.q + 1) : ph.r + (s - big) / ph.q;
}

// First piece of a bound expert at or after x in this warp's share.
__device__ __forceinline__ bool piece_at(const Tables &tb, const PhaseInfo &ph, int x, int &a,
                                         Piece &pc) {
  while (x < ph.x_hi) {
    pc.item = x / ph.groups;
    pc.g0 = x - pc.item * ph.groups;
    pc.g1 = min(ph.groups, pc.g0 + (ph.x_hi - x));
    while (tb.gbase[a + 1] * ph.tiles <= pc.item) ++a;
    if (tb.blob[a]) return true;
    x += pc.g1 - pc.g0;
  }
  return false;
}

__device__ __forceinline__ Item item_of(const Tables &tb, const PhaseInfo &ph, int group, int item,
                                        int a) {
  while (tb.gbase[a + 1] * ph.tiles <= item) ++a;
  const int rem = item - tb.gbase[a] * ph.tiles;
  const int g = rem / ph.tiles;
  Item it;
  it.tau = rem - g * ph.tiles;
  it.pi0 = tb.aoff[a] + g * group;
  it.ntok = min(group, tb.acnt[a] - g * group);
  it.blob = tb.blob[a];
  return it;
}

// Move the cursor to the first piece at or after c.x in phase c.ph (and on
// into the D share once the G share is done); caches the piece's sources.
__device__ __forceinline__ void cursor_seek(Cursor &c, const Tables &tb, const PhaseInfo *ph,
                                            int group) {
  while (true) {
    const PhaseInfo &P = ph[c.ph];
    c.have = piece_at(tb, P, c.x, c.a, c.pc);
    if (c.have) {
      const Item it = item_of(tb, P, group, c.pc.item, c.a);
      const size_t g0 = (size_t)it.tau * P.groups + (size_t)c.pc.g0;
      c.qsrc = it.blob + P.q_off + g0 * 1024;
      c.ssrc = it.blob + P.s_off + g0 * 128;
      c.cg = c.pc.g0;
      return;
    }
    if (c.ph == 1) return;
    c.ph = 1;
    c.x = ph[1].x_lo;
    c.a = 0;
  }
}

// Issue the next stage: up to gpc K groups of the current piece (packed
// weights and scales of 16 rows: ng KB and ng x 128 B, each contiguous in the
// blob) as two bulk asynchronous copies by lane 0, completing on the stage's
// barrier as transaction bytes.
__device__ __forceinline__ void issue_next(Cursor &c, Ring &rg, const Tables &tb,
                                           const PhaseInfo *ph, int group, int gpc, int kc,
                                           int lane) {
  if (!c.have) return;
  const int slot = (int)(rg.issued % rg.stages);
  const int ng = min(gpc, c.pc.g1 - c.cg);
  if (lane == 0) {
    uint8_t *dst = rg.base + slot * rg.stage_bytes;
    mbar_arrive_expect_tx(&rg.full[slot], (uint32_t)ng * 1152u);
    bulk_g2s(dst, c.qsrc, (uint32_t)ng * 1024u, &rg.full[slot]);
    bulk_g2s(dst + (size_t)kc * 8, c.ssrc, (uint32_t)ng * 128u, &rg.full[slot]);
  }
  ++rg.issued;
  c.cg += ng;
  c.qsrc += (size_t)ng * 1024;
  c.ssrc += (size_t)ng * 128;
  if (c.cg == c.pc.g1) {
    c.x = c.pc.item * ph[c.ph].groups + c.pc.g1;   // just past this piece (skipped ones included)
    cursor_seek(c, tb, ph, group);
  }
}

// Wait (with a fixed, generous bound) for every copy this warp has issued and
// not consumed, so that no copy is in flight into shared memory when the CTA
// exits.
__device__ __forceinline__ void drain_ring(Ring &rg, int *status) {
  for (uint32_t s = rg.used; s < rg.issued; ++s)
    (void)warp_wait_limit(&rg.full[s % rg.stages], (s / rg.stages) & 1u, status, kWaitLimitNs);
  rg.used = rg.issued;
}

// out[t][16 tau .. 16 tau + 15] for every token: sum_j w_j y_j + sum_s y_s in
// fp32, that order, one rounding to bf16 (zeros for a token with an unbound
// or invalid expert).  Four lanes per token, four rows each.
__device__ void combine_tile(const FusedParams &p, const Tables &tb, int tau, int lane) {
  const int kS = p.k + p.S;
  const int r = 16 * tau + 4 * (lane & 3);
  for (int t = lane >> 2; t < p.T; t += 8) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!tb.bad[t]) {
      for (int j = 0; j < kS; ++j) {
        const float4 v =
            __ldcg(reinterpret_cast<const float4 *>(p.y + (size_t)tb.inv[t * kS + j] * p.H + r));
        if (j < p.k) {
          const float wj = tb.w[t * p.k + j];
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
    const __nv_bfloat162 o0 = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 o1 = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t *>(&o0);
    packed.y = *reinterpret_cast<const uint32_t *>(&o1);
    *reinterpret_cast<uint2 *>(p.out + (size_t)t * p.H + r) = packed;
  }
}

// Bounded wait until *ctr >= target (acquire); false (and STATUS_TIMEOUT) if
// it gives up.  Lane 0 polls; the whole warp returns the result.
__device__ __forceinline__ bool warp_wait_count(const int *ctr, int target, int *status,
                                                unsigned long long limit_ns) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0 && ld_acquire(ctr) < target) {
    const uint64_t t0 = global_timer_ns();
    unsigned ns = 32;
    while (ld_acquire(ctr) < target) {
      if (global_timer_ns() - t0 > limit_ns) {
        set_status(status, STATUS_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(ns);
      if (ns < 256) ns <<= 1;
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// One phase's compute: this warp's pieces in order, consuming the ring
// stages that issue_next filled.  Returns false if a wait gave up (the ring
// is drained first).
template <bool kGateUp, int NT, int FMT>
__device__ bool run_phase(const FusedParams &p, const Tables &tb, const PhaseInfo *ph, int phi,
                          Ring &rg, Cursor &cur, int wg, int lane, int gpc, int kc) {
  const PhaseInfo &P = ph[phi];
  const int G = P.groups;
  const int g = lane >> 2, cq = lane & 3;
  const int K = kGateUp ? p.H : p.I;
  const __half *b_src = kGateUp ? p.x16 : p.h16;
  const int Wtot = (int)gridDim.x * kFW;
  const int kS = p.k + p.S;

  auto act_row = [&](const Item &it, int nt) -> const __half * {
    const int n = nt * 8 + g;
    if (n >= it.ntok) return nullptr;
    const int src = kGateUp ? tb.ptok[it.pi0 + n] : it.pi0 + n;
    return b_src + (size_t)src * K;
  };
  auto load_b = [&](uint4 v[4], const __half *row, int k0) {
    if (row) {
#pragma unroll
      for (int b = 0; b < 4; ++b) v[b] = ld_v4(row + k0 + 32 * b + 8 * cq);
    }
  };
  bool any_big = false;
  // NVFP4: the global scales (gate, up, down) of an item's expert multiply
  // its sums once at the end
  auto globals = [&](const Item &it, float &s_lo, float &s_hi) {
    if (FMT == kFmtNvfp4) {
      const float *gs = reinterpret_cast<const float *>(it.blob + p.glob);
      s_lo = kGateUp ? gs[0] : gs[2];
      s_hi = kGateUp ? gs[1] : gs[2];
    } else {
      s_lo = s_hi = 1.0f;
    }
  };
  // Output of one (pair n, row g / g + 8) element pair of an item.
  auto emit = [&](const Item &it, int n, float lo, float hi) {
    const size_t prow = (size_t)(it.pi0 + n);
    if (FMT == kFmtNvfp4) {
      float s_lo, s_hi;
      globals(it, s_lo, s_hi);
      lo *= s_lo;
      hi *= s_hi;
    }
    if (kGateUp) {
      // lo: gate row i, hi: up row i, i = 8 tau + g; stored like the packed
      // activations (the format's pair order)
      const float h = lo / (1.0f + expf(-lo)) * hi;
      const int pos = packed_pos<FMT>(it.tau * 8 + g);
      any_big |= fabsf(h) >= kF16Overflow;
      p.h16[prow * p.I + pos] = __float2half_rn(h);
    } else {
      const int r0 = it.tau * 16 + g;
      p.y[prow * p.H + r0] = lo;
      p.y[prow * p.H + r0 + 8] = hi;
    }
  };
  // Gate/up: after an item's h rows are stored, count it on its pair group
  // (active expert a, group of its pairs); the down pass reads a group's h
  // rows once all I/8 gate/up items of the group have counted themselves.
  // The count is a release, which waits until the stores before it are
  // performed; it is issued after the next stage's math (or at the end of
  // the share), when they long are, so that the warp does not stall on it.
  int pending_grp = -1;
  auto flush_group = [&]() {
    if (lane == 0 && pending_grp >= 0) red_release_add(&p.grp_done[pending_grp], 1);
    pending_grp = -1;
  };
  auto group_done = [&](const Item &it, int a_item) {
    __syncwarp();
    flush_group();
    pending_grp = tb.gbase[a_item] + (it.pi0 - tb.aoff[a_item]) / p.group;
  };
  // After a down item's rows are stored: count it on its output tile; the
  // item that completes the tile combines it.
  auto tile_done = [&](int tau) {
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atom_acq_rel_add(&p.tile_cnt[tau], 1) == tb.misc[1] - 1;
    if (__shfl_sync(0xffffffffu, last, 0)) {
      __syncwarp();
      combine_tile(p, tb, tau, lane);
      __syncwarp();
      if (lane == 0) p.tile_cnt[tau] = 0;  // ready for the next launch
    }
  };

  uint4 bb[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int b = 0; b < 4; ++b) bb[nt][b] = make_uint4(0u, 0u, 0u, 0u);
  int a = 0;
  Piece pc;
  bool have = piece_at(tb, P, P.x_lo, a, pc);
  bool ok = true;
  int ready_group = -1;   // down: the last pair group seen complete
  while (have && ok) {
    const Item it = item_of(tb, P, p.group, pc.item, a);
    int a_item = a;       // the active expert of this piece
    while (tb.gbase[a_item + 1] * P.tiles <= pc.item) ++a_item;
    if (!kGateUp) {
      const int grp = tb.gbase[a_item] + (it.pi0 - tb.aoff[a_item]) / p.group;
      if (grp != ready_group) {
        if (!warp_wait_count(p.grp_done + grp, p.I / 8, p.status, p.wait_ns)) {
          ok = false;
          break;
        }
        ready_group = grp;
      }
    }
    const int ntn = (it.ntok + 7) >> 3;
    const int x = pc.item * G + pc.g0;   // this piece's place in the sequence
    int a_nx = a;
    Piece pc_nx;
    const bool have_nx = piece_at(tb, P, x + (pc.g1 - pc.g0), a_nx, pc_nx);
    const __half *row_cur[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) row_cur[nt] = act_row(it, nt);
    float2 acc[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = make_float2(0.0f, 0.0f);
    // NVFP4: two chained MMA accumulators per n-tile (even and odd blocks)
    float acc4[NT][2][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc4[n][h][i] = 0.0f;

    for (int cg = pc.g0; cg < pc.g1; ++rg.used) {
      const int slot = (int)(rg.used % rg.stages);
      if (!warp_wait_limit(&rg.full[slot], (rg.used / rg.stages) & 1u, p.status, p.wait_ns)) {
        ok = false;
        break;
      }
      const uint8_t *stq = rg.base + slot * rg.stage_bytes;
      const uint8_t *sts = stq + (size_t)kc * 8;
      const int ng = min(gpc, pc.g1 - cg);
#pragma unroll(NT == 1 ? 2 : 1)
      for (int j = 0; j < ng; ++j) {
        // this group's activation fragments (L1-resident rows), loaded ahead
        // of the weight conversion that hides their latency
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) load_b(bb[nt], row_cur[nt], (cg + j) * 128);
        const uint4 w0 = *reinterpret_cast<const uint4 *>(stq + j * 1024 + g * 64 + cq * 16);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(stq + j * 1024 + (g + 8) * 64 + cq * 16);
        const uint2 s0 = *reinterpret_cast<const uint2 *>(sts + j * 128 + g * 8);
        const uint2 s1 = *reinterpret_cast<const uint2 *>(sts + j * 128 + (g + 8) * 8);
        const uint32_t wr0[4] = {w0.x, w0.y, w0.z, w0.w};
        const uint32_t wr1[4] = {w1.x, w1.y, w1.z, w1.w};
        uint32_t f0[4][4], f1[4][4];
        float sc0[4], sc1[4];
        if (FMT == kFmtInt4) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            int4x8_to_f16(wr0[b], f0[b]);
            int4x8_to_f16(wr1[b], f1[b]);
          }
          float2 f;
          f = __half22float2(bits_h2(s0.x)); sc0[0] = f.x; sc0[1] = f.y;
          f = __half22float2(bits_h2(s0.y)); sc0[2] = f.x; sc0[3] = f.y;
          f = __half22float2(bits_h2(s1.x)); sc1[0] = f.x; sc1[1] = f.y;
          f = __half22float2(bits_h2(s1.y)); sc1[2] = f.x; sc1[3] = f.y;
        } else {
          // word cq of block b holds elements 32 b + 8 cq .. + 7: scale group
          // 2 b + cq / 2 (byte of the row's eight); code x scale is exact in f16
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int sel = 2 * b + (cq >> 1);
            const uint32_t b0 = (sel < 4 ? s0.x : s0.y) >> (8 * (sel & 3));
            const uint32_t b1 = (sel < 4 ? s1.x : s1.y) >> (8 * (sel & 3));
            const __half2 z0 = bits_h2(e4m3_to_f16x2_dup(b0));
            const __half2 z1 = bits_h2(e4m3_to_f16x2_dup(b1));
            e2m1x8_to_f16(wr0[b], f0[b]);
            e2m1x8_to_f16(wr1[b], f1[b]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              f0[b][i] = h2_bits(__hmul2(bits_h2(f0[b][i]), z0));
              f1[b][i] = h2_bits(__hmul2(bits_h2(f1[b][i]), z1));
            }
          }
        }
        auto mma_group = [&](const uint4 (&bv)[NT][4]) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (NT == 1 || nt < ntn) {
              if (FMT == kFmtInt4) {
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
                for (int b = 0; b < 4; ++b) {
                  acc[nt][0] = __ffma2_rn(make_float2(sc0[b], sc0[b]),
                                          make_float2(d[b][0], d[b][1]), acc[nt][0]);
                  acc[nt][1] = __ffma2_rn(make_float2(sc1[b], sc1[b]),
                                          make_float2(d[b][2], d[b][3]), acc[nt][1]);
                }
              } else {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                  const uint32_t a0[4] = {f0[b][0], f1[b][0], f0[b][1], f1[b][1]};
                  const uint32_t a1[4] = {f0[b][2], f1[b][2], f0[b][3], f1[b][3]};
                  mma_16816(acc4[nt][b & 1], a0, bv[nt][b].x, bv[nt][b].y, acc4[nt][b & 1]);
                  mma_16816(acc4[nt][b & 1], a1, bv[nt][b].z, bv[nt][b].w, acc4[nt][b & 1]);
                }
              }
            }
          }
        };
        mma_group(bb);
      }
      cg += ng;
      // the stage's bytes are in registers now: refill it
      __syncwarp();
      if (kGateUp) flush_group();
      issue_next(cur, rg, tb, ph, p.group, gpc, kc, lane);
    }
    if (!ok) break;
    if (FMT == kFmtNvfp4) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[nt][0] = make_float2(acc4[nt][0][0] + acc4[nt][1][0], acc4[nt][0][1] + acc4[nt][1][1]);
        acc[nt][1] = make_float2(acc4[nt][0][2] + acc4[nt][1][2], acc4[nt][0][3] + acc4[nt][1][3]);
      }
    }

    // ---- epilogue
    if (pc.g0 == 0 && pc.g1 == G) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const int n = nt * 8 + 2 * cq + v;
          if (nt < ntn && n < it.ntok)
            emit(it, n, v ? acc[nt][0].y : acc[nt][0].x, v ? acc[nt][1].y : acc[nt][1].x);
        }
      if (kGateUp) group_done(it, a_item);
      else tile_done(it.tau);
    } else {
      // a piece of an item cut by share boundaries: store the partial sums,
      // count the piece; the last piece to arrive adds all of them in warp
      // order and emits
      const int x_item = pc.item * G;
      const int w_first = share_owner(P, x_item), w_last = share_owner(P, x_item + G - 1);
      const int my_slot = x == P.x_lo ? 0 : 1;
      float *mine = p.partial + (((size_t)phi * Wtot + wg) * 2 + my_slot) * kMmSlotFloats;
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
      int n_pieces = 0;
      for (int w = w_first; w <= w_last; ++w) n_pieces += share_cut(P, w + 1) > share_cut(P, w);
      int *ctr = p.cut_cnt + (size_t)phi * Wtot + w_first;
      __syncwarp();
      int last = 0;
      if (lane == 0) last = atom_acq_rel_add(ctr, 1) == n_pieces - 1;
      if (__shfl_sync(0xffffffffu, last, 0)) {
        __syncwarp();
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int n = nt * 8 + 2 * cq + v;
            if (nt < ntn && n < it.ntok) {
              float lo = 0.0f, hi = 0.0f;
              for (int w = w_first; w <= w_last; ++w) {
                if (share_cut(P, w + 1) == share_cut(P, w)) continue;  // empty share
                const int slot = (w == w_first && share_cut(P, w) != x_item) ? 1 : 0;
                const float *src = p.partial + (((size_t)phi * Wtot + w) * 2 + slot) * kMmSlotFloats;
                lo += __ldcg(src + n * 16 + g);
                hi += __ldcg(src + n * 16 + g + 8);
              }
              emit(it, n, lo, hi);
            }
          }
        __syncwarp();
        if (lane == 0) *ctr = 0;  // ready for the next launch
        if (kGateUp) group_done(it, a_item);
        else tile_done(it.tau);
      }
    }
    pc = pc_nx;
    have = have_nx;
    a = a_nx;
  }
  if (kGateUp) {
    __syncwarp();
    flush_group();
  }
  if (kGateUp && __any_sync(0xffffffffu, any_big) && lane == 0) set_status(p.status, STATUS_RANGE);
  if (!ok) drain_ring(rg, p.status);
  return ok;
}

}  // namespace

size_t fused_table_bytes(int T, int k, int S) {
  const size_t P = (size_t)T * (k + S);
  size_t b = 0;
  b += 2 * kMaxIds * sizeof(void *);        // ptr, blob
  b += 2 * kMaxIds * sizeof(int);           // aoff, acnt
  b += (kMaxIds + 2) * sizeof(int);         // gbase
  b += kMaxIds * sizeof(int);               // cnt
  b += (kMaxIds + 2) * sizeof(int);         // off
  b += 16 * sizeof(int);                    // misc
  b += kFW * 8 * sizeof(double);            // router partials
  b += 2 * (size_t)T * k * sizeof(int);     // idx, w
  b += P * sizeof(int) + (size_t)T * (k + S) * sizeof(int) + (size_t)T * sizeof(int);
  return (b + 127) / 128 * 128 + 128;
}

template <int NT, int FMT>
__global__ void __launch_bounds__(kFW * 32, 1) decode_fused_kernel(FusedParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int T = p.T, H = p.H, E = p.E, k = p.k, S = p.S, kS = k + S;
  const int nid = E + S;
  (void)kS;

  // ---- shared memory: rings, stage barriers, tables
  Ring rg;
  rg.stages = p.stages;
  rg.stage_bytes = p.stage_bytes;
  rg.base = smem + (size_t)warp * p.stages * p.stage_bytes;
  rg.full = reinterpret_cast<uint64_t *>(smem + (size_t)kFW * p.stages * p.stage_bytes) +
            warp * kMmMaxStages;
  rg.issued = rg.used = 0;
  Tables tb;
  {
    uint8_t *q = smem + p.smem_tables;
    tb.ptr = reinterpret_cast<const uint8_t **>(q); q += kMaxIds * sizeof(void *);
    tb.blob = reinterpret_cast<const uint8_t **>(q); q += kMaxIds * sizeof(void *);
    tb.aoff = reinterpret_cast<int *>(q); q += kMaxIds * sizeof(int);
    tb.acnt = reinterpret_cast<int *>(q); q += kMaxIds * sizeof(int);
    tb.gbase = reinterpret_cast<int *>(q); q += (kMaxIds + 2) * sizeof(int);
    tb.cnt = reinterpret_cast<int *>(q); q += kMaxIds * sizeof(int);
    tb.off = reinterpret_cast<int *>(q); q += (kMaxIds + 2) * sizeof(int);
    tb.misc = reinterpret_cast<int *>(q); q += 16 * sizeof(int);
    tb.part = reinterpret_cast<double *>(q); q += kFW * 8 * sizeof(double);
    tb.idx = reinterpret_cast<int *>(q); q += (size_t)T * k * sizeof(int);
    tb.w = reinterpret_cast<float *>(q); q += (size_t)T * k * sizeof(float);
    tb.ptok = reinterpret_cast<int *>(q); q += (size_t)T * kS * sizeof(int);
    tb.inv = reinterpret_cast<int *>(q); q += (size_t)T * kS * sizeof(int);
    tb.bad = reinterpret_cast<int *>(q);
  }
  volatile int *abort_flag = tb.misc + 2;
  // the slot table, read with per-lane indices below, into shared memory
  for (int i = tid; i < nid; i += blockDim.x) tb.ptr[i] = p.table.ptr[i];
  if (lane == 0)
    for (int s = 0; s < p.stages; ++s) mbar_init(&rg.full[s], 1);
  if (tid == 0) {
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // ---- phase R: pack the activations; router logits
  {
    const int n8 = T * H / 8;
    bool over = false;
    for (int i = blockIdx.x * blockDim.x + tid; i < n8; i += gridDim.x * blockDim.x) {
      bool o;
      const uint4 v =
          pack8_bf16_to_f16<FMT>(*reinterpret_cast<const uint4 *>(p.x + (size_t)i * 8), o);
      over |= o;
      *reinterpret_cast<uint4 *>(p.x16 + (size_t)i * 8) = v;
    }
    if (over) set_status(p.status, STATUS_RANGE);
  }
  const bool routed_given = p.idx_in != nullptr;
  // Router: unit = (expert e, split sp), sp covering a range of the H/128
  // chunks; splits = grid / E (at least 1) so that small E still uses every
  // CTA.  A unit's warps (the CTA's) take its chunks round-robin, each lane 4
  // consecutive elements; per token a lane's products are summed in double
  // in chunk order, the 32 lanes reduced by one transpose-reduction, the
  // warps added in warp order, and the unit's partial sum stored.
  const int splits = max(1, (int)gridDim.x / E);
  if (!routed_given) {
    const int C = H / 128;
    for (int u = blockIdx.x; u < E * splits; u += gridDim.x) {
      const int e = u / splits, sp = u - (u / splits) * splits;
      const int c0 = sp * C / splits, c1 = (sp + 1) * C / splits;
      const float *wr = p.W + (size_t)e * H;
      for (int t0 = 0; t0 < T; t0 += 8) {
        const int nt = min(8, T - t0);
        double acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0;
        for (int c = c0 + warp; c < c1; c += kFW) {
          const int h = c * 128 + lane * 4;
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
        // transpose-reduction: 8 values per lane -> lane l holds the sum for
        // token 4 (l >> 4 & 1) + 2 (l >> 3 & 1) + (l >> 2 & 1)
        {
          const bool hi16 = lane & 16, hi8 = lane & 8, hi4 = lane & 4;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const double send = hi16 ? acc[i] : acc[i + 4];
            const double keep = hi16 ? acc[i + 4] : acc[i];
            acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
          }
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const double send = hi8 ? acc[i] : acc[i + 2];
            const double keep = hi8 ? acc[i + 2] : acc[i];
            acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
          }
          {
            const double send = hi4 ? acc[0] : acc[1];
            const double keep = hi4 ? acc[1] : acc[0];
            acc[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
          }
          acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 2);
          acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
          const int tok = (hi16 ? 4 : 0) + (hi8 ? 2 : 0) + (hi4 ? 1 : 0);
          if ((lane & 3) == 0) tb.part[warp * 8 + tok] = acc[0];
        }
        __syncthreads();
        if (tid < nt) {
          double v = tb.part[tid];
          for (int w = 1; w < kFW; ++w) v += tb.part[w * 8 + tid];
          p.rpart[((size_t)sp * T + t0 + tid) * E + e] = v;
        }
        __syncthreads();
      }
    }
  }
  bool live = grid_sync(p.bar + 0, abort_flag, p.status, p.wait_ns);

  // ---- phase K: logits (the units' partial sums added in split order, plus
  // the bias, rounded once to fp32) and top-k, from shared memory (the ring
  // space, unused until the weight copies start)
  float *s_logit = reinterpret_cast<float *>(smem);
  const bool redundant = T <= kFW;
  auto logit_of = [&](int t, int e) -> float {
    double v = __ldcg(p.rpart + (size_t)t * E + e);
    for (int sp = 1; sp < splits; ++sp) v += __ldcg(p.rpart + ((size_t)sp * T + t) * E + e);
    if (p.bias) v += (double)p.bias[e];
    return (float)v;
  };
  auto topk_row = [&](const float *row, int &e, float &wt) {
    if (E <= 64) select_topk_warp_t<2, true>(row, E, k, p.mode, lane, e, wt);
    else select_topk_warp_t<kMaxExperts / 32, true>(row, E, k, p.mode, lane, e, wt);
  };
  if (live && !routed_given) {
    if (redundant) {
      for (int q = tid; q < T * E; q += blockDim.x) s_logit[q] = logit_of(q / E, q - (q / E) * E);
      __syncthreads();
      if (warp < T) {
        int e;
        float wt;
        topk_row(s_logit + warp * E, e, wt);
        if (lane < k) {
          tb.idx[warp * k + lane] = e;
          tb.w[warp * k + lane] = wt;
        }
      }
    } else {
      for (int t = blockIdx.x; t < T; t += gridDim.x) {
        for (int e = tid; e < E; e += blockDim.x) s_logit[e] = logit_of(t, e);
        __syncthreads();
        if (warp == 0) {
          int e;
          float wt;
          topk_row(s_logit, e, wt);
          if (lane < k) {
            p.idx[(size_t)t * k + lane] = e;
            p.w[(size_t)t * k + lane] = wt;
          }
        }
        __syncthreads();
      }
    }
  }
  if (!routed_given && !redundant) live = grid_sync(p.bar + 1, abort_flag, p.status, p.wait_ns) && live;
  if (live) {
    if (routed_given) {
      for (int q = tid; q < T * k; q += blockDim.x) {
        tb.idx[q] = p.idx_in[q];
        tb.w[q] = p.w_in[q];
      }
    } else if (!redundant) {
      for (int q = tid; q < T * k; q += blockDim.x) {
        tb.idx[q] = __ldcg(p.idx + q);
        tb.w[q] = __ldcg(p.w + q);
      }
    }
  }
  __syncthreads();

  // ---- phase B: bucketing (every CTA, in shared memory)
  if (live) {
    for (int i = tid; i < nid; i += blockDim.x) tb.cnt[i] = i < E ? 0 : T;
    for (int t = tid; t < T; t += blockDim.x) tb.bad[t] = 0;
    __syncthreads();
    for (int q = tid; q < T * k; q += blockDim.x) {
      const int e = tb.idx[q];
      if (e >= 0 && e < E) {
        atomicAdd(&tb.cnt[e], 1);
        if (!tb.ptr[e]) tb.bad[q / k] = 1;
      } else {
        tb.bad[q / k] = 1;
        if (blockIdx.x == 0) set_status(p.status, STATUS_BAD_ROUTING);
      }
    }
    __syncthreads();
    if (warp == 0) {
      // offsets by id, the active list and the pair groups per active
      // expert: each lane scans a contiguous run of ids, one warp scan joins
      // the runs
      const int per = (nid + 31) >> 5;
      const int i0 = min(nid, lane * per), i1 = min(nid, i0 + per);
      int sc = 0, sf = 0, sg = 0, sb = 0;
      for (int i = i0; i < i1; ++i) {
        const int c = tb.cnt[i];
        const int ng = (c + p.group - 1) / p.group;
        sc += c;
        sf += c > 0;
        sg += ng;
        sb += tb.ptr[i] ? ng : 0;
      }
      int ec = sc, ef = sf, eg = sg, eb = sb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v1 = __shfl_up_sync(0xffffffffu, ec, o);
        const int v2 = __shfl_up_sync(0xffffffffu, ef, o);
        const int v3 = __shfl_up_sync(0xffffffffu, eg, o);
        const int v4 = __shfl_up_sync(0xffffffffu, eb, o);
        if (lane >= o) {
          ec += v1;
          ef += v2;
          eg += v3;
          eb += v4;
        }
      }
      const int carry = __shfl_sync(0xffffffffu, ec, 31);
      const int acarry = __shfl_sync(0xffffffffu, ef, 31);
      const int gcarry = __shfl_sync(0xffffffffu, eg, 31);
      const int gbound = __shfl_sync(0xffffffffu, eb, 31);
      ec -= sc;
      ef -= sf;
      eg -= sg;
      for (int i = i0; i < i1; ++i) {
        const int c = tb.cnt[i];
        const int ng = (c + p.group - 1) / p.group;
        const uint8_t *bp = tb.ptr[i];
        tb.off[i] = ec;
        if (c > 0) {
          tb.blob[ef] = bp;
          tb.aoff[ef] = ec;
          tb.acnt[ef] = c;
          tb.gbase[ef] = eg;
          if (!bp && blockIdx.x == 0) set_status(p.status, STATUS_NOT_BOUND);
          ++ef;
        }
        ec += c;
        eg += ng;
      }
      if (lane == 0) {
        tb.off[nid] = carry;
        tb.gbase[acarry] = gcarry;
        tb.misc[0] = acarry;
        tb.misc[1] = gbound;
      }
      // stable positions of the routed pairs, 32 pairs at a time in order:
      // equal experts within a chunk are ranked by lane, the running cursor
      // (in cnt, reused) moved on by the chunk's count
      __syncwarp();
      for (int i = lane; i < E; i += 32) tb.cnt[i] = tb.off[i];
      __syncwarp();
      const unsigned lt = (1u << lane) - 1u;
      for (int q0 = 0; q0 < T * k; q0 += 32) {
        const int q = q0 + lane;
        const bool in = q < T * k;
        const int e = in ? tb.idx[q] : -1;
        const bool valid = in && e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        const int rank = __popc(peers & lt);
        int pos = -1;
        if (valid) pos = tb.cnt[e] + rank;
        __syncwarp();
        if (valid && rank == __popc(peers) - 1) tb.cnt[e] = pos + 1;
        __syncwarp();
        if (in) {
          const int t = q / k, j = q - (q / k) * k;
          tb.inv[t * kS + j] = pos;
          if (valid) tb.ptok[pos] = t;
        }
      }
      for (int q = lane; q < T * S; q += 32) {
        const int s = q / T, t = q - (q / T) * T;
        const int pos = tb.off[E + s] + t;
        tb.ptok[pos] = t;
        tb.inv[t * kS + k + s] = pos;
      }
    }
    __syncthreads();
  }

  // ---- phases G and D
  const int Wtot = (int)gridDim.x * kFW;
  const int wg = (int)blockIdx.x * kFW + warp;
  const int gpc = p.kc / 128;
  PhaseInfo ph[2];
  Cursor cur;
  cur.ph = 0;
  cur.have = false;
  if (live) {
    const int n_groups = tb.gbase[tb.misc[0]];
    for (int phi = 0; phi < 2; ++phi) {
      PhaseInfo &P = ph[phi];
      P.tiles = phi == 0 ? p.I / 8 : H / 16;
      P.groups = (phi == 0 ? H : p.I) / 128;
      P.q_off = phi == 0 ? p.guq : p.dq;
      P.s_off = phi == 0 ? p.gus : p.ds;
      const int total = n_groups * P.tiles * P.groups;
      const int slots = (total + gpc - 1) / gpc;
      P.unit = gpc;
      P.total = total;
      P.q = slots / Wtot;
      P.r = slots - P.q * Wtot;
      P.x_lo = share_cut(P, wg);
      P.x_hi = share_cut(P, wg + 1);
    }
    cur.x = ph[0].x_lo;
    cur.a = 0;
    cursor_seek(cur, tb, ph, p.group);
    for (int s = 0; s < rg.stages; ++s) issue_next(cur, rg, tb, ph, p.group, gpc, p.kc, lane);
    if (!run_phase<true, NT, FMT>(p, tb, ph, 0, rg, cur, wg, lane, gpc, p.kc)) *abort_flag = 1;
  }
  // the down pass waits per pair group for the gate/up items it reads (no
  // grid barrier); a warp that gave up in the gate/up pass does not start it
  if (live && !*abort_flag) {
    if (!run_phase<false, NT, FMT>(p, tb, ph, 1, rg, cur, wg, lane, gpc, p.kc)) *abort_flag = 1;
    // no combine happens if no expert item ran at all: every token is then
    // one with an unbound expert, and its output row is zero
    if (blockIdx.x == 0 && tb.misc[1] == 0)
      for (int i = tid; i < T * H / 4; i += blockDim.x)
        reinterpret_cast<uint2 *>(p.out)[i] = make_uint2(0u, 0u);
  }
  // copies issued for a phase that did not run (a wait gave up) still land
  // before the CTA exits
  drain_ring(rg, p.status);

  // ---- exit: the last CTA out resets the barrier and pair-group counters
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    tb.misc[3] = atomicAdd(p.bar + 3, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (tb.misc[3]) {
    for (int i = tid; i < T * kS; i += blockDim.x) p.grp_done[i] = 0;
    if (tid == 0) p.bar[0] = p.bar[1] = p.bar[2] = 0;
    __threadfence();
    __syncthreads();
    if (tid == 0) p.bar[3] = 0;
  }
}

template __global__ void decode_fused_kernel<1, kFmtInt4>(FusedParams);
template __global__ void decode_fused_kernel<2, kFmtInt4>(FusedParams);
template __global__ void decode_fused_kernel<1, kFmtNvfp4>(FusedParams);
template __global__ void decode_fused_kernel<2, kFmtNvfp4>(FusedParams);

}  // namespace strata
