// Expert matmuls for many tokens per expert (prefill): a grouped GEMM on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// What it computes (the W4A16 expert FFN of ro99/strata README, model table
// and "Kernels"; the prompt-time expert GEMMs of "Strata on a Mac",
// "Switches"): for every active expert e and the pairs routed to it,
//   gate/up pass:  h = silu(Wg x) * (Wu x)  -> h16 [P][I] (f16)
//   down pass:     y = Wd h                -> y   [P][H] (fp32)
//
// Unit = (expert, block of <= 512 of its pairs, 128 weight rows).  For
// gate/up the 128 rows are 8 blob tiles, i.e. 64 gate rows and the same 64 up
// rows interleaved by 8 (TMEM lane l holds gate if l % 16 < 8, else up; its
// partner is lane l ^ 8, in the same warp).  For down they are 128
// consecutive rows of Wd.  A unit's pairs form one or two chunks of <= 256
// (one MMA N each); every dequantised weight atom feeds both chunks, so an
// expert with many pairs pays the dequantisation once per 512 pairs.
//
// Swapped unit = (expert whose last block has <= 128 pairs, 256 weight rows),
// for int4 blobs whose 128-row tiles pair up: the operands trade places.  The
// block's activations are the MMA's A (M = 128 rows; rows past the pairs are
// ignored) and 256 dequantised weight rows its B (N = 256): one MMA covers
// 256 weight rows where the other form needs two M = 128 MMAs whose cost
// hardly depends on N (M = 64 when the block has <= 64 pairs).  The
// accumulator then holds one pair per TMEM lane and one weight row per
// column.  Each output element is the same K-ordered sum of the same products
// in every form, and comes out bit for bit the same.
// Every CTA runs its plain units first, then its swapped ones (phase 2), in
// which the two rings' shared memory trades roles: activations in the
// three 16 KB stages, weights in the five 32 KB ones (a swapped atom's 256
// rows need a stage that size, and the weight ring's depth is what limits
// these units).  Each ring has one producer role in each phase (a ring
// filled by two roles that skip each other's positions would let one run
// two laps ahead, which a phase-parity wait cannot tell apart); phase 2 has
// barriers of its own, and its producers start once every MMA of phase 1
// has completed.
//
// Warp roles (one CTA per SM, persistent; units interleaved over CTAs; the
// warp ids of each role are in tc_warp below):
//   activation producer: per 64 K elements (one swizzle atom) and chunk, the
//               activation rows (f16, 128-byte swizzle; x_perm or h16) in one
//               256-row TMA box, or in 64-row and 16-row boxes for shorter
//               chunks;
//   MMA: allocates all 512 TMEM columns (two 256-column accumulators), and
//               one thread issues 4 tcgen05.mma (M=128, N=chunk pairs rounded
//               up to 16, K=16) per atom and chunk (swapped: M=64 or 128
//               pairs, N=256 weight rows), commits to the operand stages and,
//               at the end of a unit, to the accumulators it used;
//   8 dequant warps: load their rows' packed weights and scales straight
//               from global memory, one K group ahead (an L2 prefetch of the
//               units ahead only evicted lines before their loads),
//               int4 -> exact f16 integers -> times the fp16 scale (one f16
//               rounding), or NVFP4 E2M1 codes times their E4M3 group scale
//               (exact in f16; the fp32 global scale multiplies the
//               accumulator in the epilogue) -> the K-major 128-byte-swizzled
//               layout, 16 rows each of a 128-row atom (swapped: 32 rows,
//               two blob tiles, of a 256-row atom);
//   8 epilogue warps: two per TMEM lane quarter, each taking alternate
//               32-column blocks: tcgen05.ld, SwiGLU (gate/up; the gate lane
//               and its up partner each compute one column of every pair) or
//               plain (down), transposed through shared memory, stored (a
//               swapped unit: each lane holds one pair's row and stores it);
//   one more warp has no role (it kept a ring of packed weights in shared
//               memory, which now goes to the activation ring).  One thread
//               issues all MMAs: a variant with a second issuing thread (one
//               per accumulator) faulted once and is not used.
// In phase 1 the A operand (16 KB per atom) and the B operand (32 KB per atom
// and chunk) have rings of their own (three and five stages) with one "full"
// and one "empty" mbarrier per stage: the kernel is bound by the hand-offs
// between its roles, and the depth of the activation ring, in stages, is what
// counts most.  Warps therefore test a barrier on every lane and vote before
// the bounded single-lane wait, and arrive through an elect.sync-predicated
// instruction rather than a divergent branch.  A unit of two chunks uses both accumulators; a unit of one
// chunk uses the next one in turn, so the epilogue of a unit overlaps the MMAs
// of the next.
// Every wait is bounded; on a timeout the status word is set and the roles
// wind down (the producers let their issued copies land; the allocating warp
// still frees the tensor memory).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace strata {

namespace {

constexpr int kTcM = 128;          // weight rows per unit
constexpr int kTcN = 256;          // pairs per chunk (max MMA N used)
constexpr int kUnitPairs = 2 * kTcN;
constexpr int kSwapPairs = kTcM;   // swapped unit: at most this many pairs (MMA M) ...
constexpr int kSwapRows = kTcN;    // ... and this many weight rows (MMA N)
constexpr int kAStages = 3;        // A ring: one 64-wide dequantised atom each
constexpr int kBStages = 5;        // B ring: one 64-wide activation atom of one chunk each
constexpr int kDqWarps = 8;
constexpr int kDqRows = kTcM / kDqWarps;    // weight rows per dequant warp
static_assert(kDqRows % 8 == 0, "dequant warps cover whole 8-row groups");
constexpr int kEpiWarps = 8;                // two per TMEM lane quarter
constexpr int kTcWarps = 3 + kDqWarps + kEpiWarps;
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kAccCols = 256;      // TMEM columns per accumulator
constexpr uint32_t kTmemCols = 512;

constexpr int kAStageBytes = kTcM * 128;               // one 64-wide atom
constexpr int kBStageBytes = kTcN * 128;
constexpr int kEpiBytes = kEpiWarps * 1024;            // per epilogue warp: 1 KB

constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kAStages * kAStageBytes;
constexpr int kOffEpi = kOffB + kBStages * kBStageBytes;
constexpr int kOffBar = kOffEpi + kEpiBytes;
constexpr int kNumBars = 2 * (2 * kAStages + 2 * kBStages) + 5;
constexpr int kOffTab = kOffBar + kNumBars * 8 + 16;   // + TMEM address slot
constexpr int kTabBytes = kMaxIds * 8 + (4 * kMaxIds + 2) * 4;
constexpr int kTcSmem = kOffTab + kTabBytes + 1024;    // + alignment slack

// A warp's wait for a barrier phase: one test by every lane and a vote (no
// divergent branch when the phase is already complete, the common case),
// else lane 0 waits with the time limit and tells the others.
__device__ __forceinline__ bool wwait(uint64_t *bar, uint32_t parity, int *status) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// One arrival for the whole (converged) warp, made by the lane elect.sync
// picks as a predicated instruction rather than under a divergent branch.
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// Warp roles.  A warp issues from the scheduler of warp id % 4; the single
// thread that issues every MMA gets scheduler 1 with only warps that mostly
// sleep (two epilogue warps, the producer, the warp with no role), while the dequant warps, the
// busiest, share schedulers 0, 2 and 3 with the other epilogue warps.  An
// epilogue warp may only read its own TMEM lane quarter (warp id % 4).
enum TcRole : int { kRoleAct, kRoleMma, kRoleDq, kRoleEpi, kRoleIdle };
struct TcWarp {
  int role, idx;  // idx: dequant warp 0..7, or epilogue warp 0..7 (= 2 quarter + half)
};
__device__ __forceinline__ TcWarp tc_warp(int warp) {
  switch (warp) {
    case 1: return {kRoleMma, 0};
    case 13: return {kRoleIdle, 0};
    case 17: return {kRoleAct, 0};
    case 0: return {kRoleDq, 0};
    case 4: return {kRoleDq, 1};
    case 8: return {kRoleDq, 2};
    case 2: return {kRoleDq, 3};
    case 6: return {kRoleDq, 4};
    case 10: return {kRoleDq, 5};
    case 3: return {kRoleDq, 6};
    case 7: return {kRoleDq, 7};
    case 12: return {kRoleEpi, 0};
    case 16: return {kRoleEpi, 1};
    case 5: return {kRoleEpi, 2};
    case 9: return {kRoleEpi, 3};
    case 14: return {kRoleEpi, 4};
    case 18: return {kRoleEpi, 5};
    case 11: return {kRoleEpi, 6};
    default: return {kRoleEpi, 7};  // 15
  }
}
static_assert(kTcWarps == 19 && kDqWarps == 8 && kEpiWarps == 8, "role table");

// A compile-time int passed as an argument (selects the instance of a
// generic lambda).
template <int N>
struct IntTag {
  static constexpr int value = N;
};

struct Unit {
  const uint8_t *blob;
  int pi0, n, rt;  // rt: 128-row tile, or 256-row tile of a swapped unit
  bool sw;
  __device__ __forceinline__ int chunks() const { return n > kTcN ? 2 : 1; }
  __device__ __forceinline__ int chunk_n(int c) const { return c == 0 ? min(n, kTcN) : n - kTcN; }
};

// A ring position (stage and phase parity), advanced in the same order by
// the roles that share the ring.
struct RingPos {
  uint32_t st = 0, ph = 0;
  __device__ __forceinline__ void next(uint32_t stages) {
    if (++st == stages) {
      st = 0;
      ph ^= 1u;
    }
  }
};

// Accumulator use: a two-chunk unit uses accumulators 0 and 1; a one-chunk
// unit uses the one after the last it used.  Both the MMA thread and the
// epilogue walk the units in the same order, so they agree on every
// accumulator's use count (and so on the barrier phases).
struct AccTrack {
  uint32_t uses[2] = {0u, 0u};
  int next_single = 0;
  __device__ __forceinline__ int buf_of(int nchunks, int c) const {
    return nchunks == 2 ? c : next_single;
  }
  __device__ __forceinline__ void done_unit(int nchunks) {
    if (nchunks == 2) {
      uses[0]++;
      uses[1]++;
      next_single = 0;
    } else {
      uses[next_single]++;
      next_single ^= 1;
    }
  }
};

}  // namespace

size_t tc_smem_bytes() { return kTcSmem; }
int tc_threads() { return kTcThreads; }
static_assert(kTcSmem <= 232448, "shared memory budget");

template <bool kGateUp, int FMT>
__global__ void __launch_bounds__(kTcThreads, 1)
    expert_tc_kernel(TcParams p, const __grid_constant__ CUtensorMap tmap_b16,
                     const __grid_constant__ CUtensorMap tmap_b64,
                     const __grid_constant__ CUtensorMap tmap_b256) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  // phase 1 (plain units): fullA[s]: the dequant warps' arrivals; fullB[s]:
  // the activation TMA bytes; emptyA/emptyB[s]: the MMAs that read stage s
  // have completed.  Phase 2 (swapped units), on the same shared memory:
  // fullX/emptyX for the activations in the A stages, fullW/emptyW for the
  // weights in the B stages.  p1_done: every MMA of phase 1 has completed.
  uint64_t *fullA = bars, *emptyA = fullA + kAStages;
  uint64_t *fullB = emptyA + kAStages, *emptyB = fullB + kBStages;
  uint64_t *fullX = emptyB + kBStages, *emptyX = fullX + kAStages;
  uint64_t *fullW = emptyX + kAStages, *emptyW = fullW + kBStages;
  uint64_t *acc_full = emptyW + kBStages, *acc_empty = acc_full + 2;
  uint64_t *p1_done = acc_empty + 2;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + kNumBars);
  const uint8_t **t_blob = reinterpret_cast<const uint8_t **>(smem + kOffTab);
  int *t_off = reinterpret_cast<int *>(t_blob + kMaxIds);
  int *t_cnt = t_off + kMaxIds;
  int *unit_base = t_cnt + kMaxIds;        // plain units, prefix over experts
  int *swap_base = unit_base + kMaxIds + 1;  // swapped units, prefix

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TcWarp role = tc_warp(warp);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&fullA[s], kDqWarps);
      mbar_init(&emptyA[s], 1);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&fullB[s], 1);
      mbar_init(&emptyB[s], 1);
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&fullX[s], 1);
      mbar_init(&emptyX[s], 1);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&fullW[s], kDqWarps);
      mbar_init(&emptyW[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kEpiWarps);
    }
    mbar_init(p1_done, 1);
    fence_mbar_init();
    prefetch_tmap(&tmap_b16);
    prefetch_tmap(&tmap_b64);
    prefetch_tmap(&tmap_b256);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  grid_dependency_wait();

  // active experts and units per expert (prefix), in shared memory; an
  // active expert without a blob gets no units (and is reported, unless the
  // call runs one expert pass of several)
  const int n_active = *p.rt.n_active;
  for (int a = threadIdx.x; a < n_active; a += blockDim.x) {
    const int id = p.rt.active[a];
    t_blob[a] = p.table.ptr[id];
    t_off[a] = p.rt.off[id];
    t_cnt[a] = p.rt.cnt[id];
    if (!t_blob[a] && !p.quiet_unbound && blockIdx.x == 0) set_status(p.status, STATUS_NOT_BOUND);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  // swapped units need the 128-row tiles to pair up; they are used for int4
  // blobs (the NVFP4 dequant of two tiles per warp would not fit in the
  // registers this block size leaves)
  constexpr bool kSwapFmt = FMT == kFmtInt4;
  const bool can_swap = kSwapFmt && (p.row_tiles & 1) == 0;
  // an expert's last block of pairs goes to swapped units if it is that short
  auto last_swapped = [&](int cnt) {
    return can_swap && cnt - ((cnt - 1) / kUnitPairs) * kUnitPairs <= kSwapPairs;
  };
  if (warp < 2) {
    // warp 0: plain units per expert (row_tiles per block of 512 pairs but a
    // swapped last block); warp 1: swapped units (row_tiles / 2 or none)
    int *base = warp == 0 ? unit_base : swap_base;
    int carry = 0;
    for (int a0 = 0; a0 < n_active; a0 += 32) {
      const int a = a0 + lane;
      int v = 0;
      if (a < n_active && t_blob[a] && t_cnt[a] > 0) {
        const int nb = (t_cnt[a] + kUnitPairs - 1) / kUnitPairs;
        const bool sl = last_swapped(t_cnt[a]);
        v = warp == 0 ? (nb - (sl ? 1 : 0)) * p.row_tiles : (sl ? p.row_tiles / 2 : 0);
      }
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int nb = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nb;
      }
      if (a < n_active) base[a] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) base[n_active] = carry;
  }
  __syncthreads();
  grid_dependency_launch();

  // units 0 .. n_plain - 1 are plain, the rest swapped
  const int n_plain = unit_base[n_active];
  const int n_units = n_plain + swap_base[n_active];
  const int G = p.K / 128;  // K groups
  // one cursor per phase over the active experts (units are walked in order)
  struct Cursor {
    int a = 0, b = 0;
  };
  auto decode = [&](int u, Cursor &cur) -> Unit {
    Unit un;
    int a, ub;
    if (!kSwapFmt || u < n_plain) {
      while (unit_base[cur.a + 1] <= u) ++cur.a;
      a = cur.a;
      const int rem = u - unit_base[a];
      ub = rem / p.row_tiles;
      un.rt = rem - ub * p.row_tiles;
      un.sw = false;
    } else {
      const int v = u - n_plain;
      while (swap_base[cur.b + 1] <= v) ++cur.b;
      a = cur.b;
      ub = (t_cnt[a] - 1) / kUnitPairs;  // the last block
      un.rt = v - swap_base[a];
      un.sw = true;
    }
    un.pi0 = t_off[a] + ub * kUnitPairs;
    un.n = min(kUnitPairs, t_cnt[a] - ub * kUnitPairs);
    un.blob = t_blob[a];
    return un;
  };

  if (role.role == kRoleAct) {
    // -------------------------------------------------------- activation producer
    uint32_t issued_b = 0, issued_x = 0;  // copies into the B stages, the A stages
    RingPos rb, rx;
    bool ok = true, phase2 = false;
    Cursor cur;
    // a unit's activation rows, per 64 K elements (one swizzle atom) and
    // chunk: one 256-row box, else 64-row boxes and 16-row boxes for the rest
    // (rows land at 128 bytes each whatever the box, so the swizzled layout
    // is the same)
    auto produce = [&](const Unit &un, uint64_t *full, uint64_t *empty, RingPos &r, uint32_t stages,
                       uint8_t *ring, int stage_bytes, uint32_t &issued) {
      const int nc = un.chunks();
      for (int at = 0; at < 2 * G && ok; ++at) {
        for (int c = 0; c < nc; ++c) {
          if (!wwait(&empty[r.st], r.ph ^ 1u, p.status)) { ok = false; break; }
          const int cn = un.chunk_n(c), row0 = un.pi0 + c * kTcN;
          const bool wide = cn > 192;
          const int n64 = wide ? 0 : cn / 64;
          const int n16 = wide ? 0 : (cn - 64 * n64 + 15) / 16;
          const uint32_t tx = wide ? 32768u : n64 * 8192u + n16 * 2048u;
          uint8_t *dst = ring + r.st * stage_bytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[r.st], tx);
            if (wide) {
              tma_load_2d(dst, &tmap_b256, at * 64, row0, &full[r.st]);
            } else {
              for (int q = 0; q < n64; ++q)
                tma_load_2d(dst + q * 8192, &tmap_b64, at * 64, row0 + q * 64, &full[r.st]);
              for (int q = 0; q < n16; ++q)
                tma_load_2d(dst + n64 * 8192 + q * 2048, &tmap_b16, at * 64, row0 + 64 * n64 + 16 * q,
                            &full[r.st]);
            }
          }
          __syncwarp();
          ++issued;
          r.next(stages);
        }
      }
    };
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit un = decode(u, cur);
      if (!un.sw) {
        produce(un, fullB, emptyB, rb, kBStages, smem + kOffB, kBStageBytes, issued_b);
        continue;
      }
      // swapped (<= 128 rows, one chunk) into the A stages, once the weights
      // that phase 1 kept there have been read
      if (!phase2) {
        phase2 = true;
        if (!wwait(p1_done, 0u, p.status)) { ok = false; break; }
      }
      produce(un, fullX, emptyX, rx, kAStages, smem + kOffA, kAStageBytes, issued_x);
    }
    if (!ok) {
      // let issued copies land before the CTA exits (bounded waits)
      for (uint32_t m = issued_b > kBStages ? issued_b - kBStages : 0; m < issued_b; ++m)
        (void)wwait(&fullB[m % kBStages], (m / kBStages) & 1u, p.status);
      for (uint32_t m = issued_x > kAStages ? issued_x - kAStages : 0; m < issued_x; ++m)
        (void)wwait(&fullX[m % kAStages], (m / kAStages) & 1u, p.status);
    }
  } else if (role.role == kRoleIdle) {
    // -------------------------------------------------------- (no role)
  } else if (role.role == kRoleMma) {
    // -------------------------------------------------------- MMA issue
    // One thread does it all: per atom one wait for A, per chunk one wait for
    // B, four MMAs and one commit, so the tensor pipe's queue never runs dry
    // behind warp-level overheads.
    if (lane == 0) {
      RingPos ra, rb, rx, rw;
      AccTrack acc;
      bool ok = true, phase2 = false;
      Cursor cur;
      // stage 0's descriptors; a stage adds its offset / 16 to the address
      // field, a 16-element K step (32 bytes) adds 2
      const uint64_t a_desc0 = umma_desc_sw128(smem_u32(smem + kOffA));
      const uint64_t b_desc0 = umma_desc_sw128(smem_u32(smem + kOffB));
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit un = decode(u, cur);
        if (un.sw) {
          if (!phase2) {
            // the producers of phase 2 reuse the stages once these complete
            phase2 = true;
            umma_commit(p1_done);
          }
          // A: the block's activations (A stages), B: 256 weight rows (B stages)
          const int buf = acc.buf_of(1, 0);
          const uint32_t id = umma_idesc_f16(un.n <= 64 ? 64 : kSwapPairs, kSwapRows);
          const uint32_t dt = tmem_base + buf * kAccCols;
          if (!mbar_wait(&acc_empty[buf], (acc.uses[buf] & 1u) ^ 1u, p.status)) { ok = false; break; }
          tc_fence_after();
          for (int at = 0; at < 2 * G; ++at) {
            if (!mbar_wait(&fullW[rw.st], rw.ph, p.status) ||
                !mbar_wait(&fullX[rx.st], rx.ph, p.status)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = a_desc0 + (uint64_t)((rx.st * kAStageBytes) >> 4);
            const uint64_t bd = b_desc0 + (uint64_t)((rw.st * kBStageBytes) >> 4);
            umma_f16(dt, ad, bd, id, at > 0 ? 1u : 0u);
            umma_f16(dt, ad + 2, bd + 2, id, 1u);
            umma_f16(dt, ad + 4, bd + 4, id, 1u);
            umma_f16(dt, ad + 6, bd + 6, id, 1u);
            umma_commit(&emptyX[rx.st]);
            umma_commit(&emptyW[rw.st]);
            rx.next(kAStages);
            rw.next(kBStages);
          }
          if (!ok) break;
          umma_commit(&acc_full[buf]);
          acc.done_unit(1);
          continue;
        }
        // a plain unit of NC chunks (a compile-time count keeps the chunks'
        // descriptors in registers)
        auto plain = [&](auto nc_tag) {
          constexpr int NC = decltype(nc_tag)::value;
          uint32_t idesc[NC], d_tmem[NC];
          int bufs[NC];
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            bufs[c] = acc.buf_of(NC, c);
            idesc[c] = umma_idesc_f16(kTcM, (un.chunk_n(c) + 15) & ~15);
            d_tmem[c] = tmem_base + bufs[c] * kAccCols;
          }
          for (int at = 0; at < 2 * G && ok; ++at) {
            if (!mbar_wait(&fullA[ra.st], ra.ph, p.status)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = a_desc0 + (uint64_t)((ra.st * kAStageBytes) >> 4);
#pragma unroll
            for (int c = 0; c < NC; ++c) {
              if (at == 0) {
                // the accumulator must have been drained by the epilogue
                const int b = bufs[c];
                if (!mbar_wait(&acc_empty[b], (acc.uses[b] & 1u) ^ 1u, p.status)) { ok = false; break; }
                tc_fence_after();
              }
              if (!mbar_wait(&fullB[rb.st], rb.ph, p.status)) { ok = false; break; }
              tc_fence_after();
              const uint64_t bd = b_desc0 + (uint64_t)((rb.st * kBStageBytes) >> 4);
              umma_f16(d_tmem[c], ad, bd, idesc[c], at > 0 ? 1u : 0u);
              umma_f16(d_tmem[c], ad + 2, bd + 2, idesc[c], 1u);
              umma_f16(d_tmem[c], ad + 4, bd + 4, idesc[c], 1u);
              umma_f16(d_tmem[c], ad + 6, bd + 6, idesc[c], 1u);
              umma_commit(&emptyB[rb.st]);
              rb.next(kBStages);
            }
            if (!ok) break;
            umma_commit(&emptyA[ra.st]);
            ra.next(kAStages);
          }
          if (!ok) return;
#pragma unroll
          for (int c = 0; c < NC; ++c) umma_commit(&acc_full[bufs[c]]);
          acc.done_unit(NC);
        };
        if (un.chunks() == 2)
          plain(IntTag<2>{});
        else
          plain(IntTag<1>{});
      }
    }
    __syncwarp();
  } else if (role.role == kRoleDq) {
    // -------------------------------------------------------- dequant
    const int dw = role.idx;
    const int w = lane & 3;
    const int q = lane >> 2;
    const int row_in_8 = (q & 1) * 4 + (q >> 1);  // lanes 8p..8p+7 -> rows p and p + 4
    RingPos ra, rw;
    bool ok = true, big_scale = false, phase2 = false;
    Cursor cur;
    // One unit into one ring: per 64 K, an atom of 128 rows (NA = 1) or of
    // 256 (NA = 2, a swapped unit: row tiles 2 rt and 2 rt + 1, one below the
    // other).  This warp's 16 rows of half j are blob tile tile0 + 8 j; per K
    // group, tile row tr holds 64 bytes of packed weights (word w of each
    // 32-element block: bytes 16 w .. 16 w + 15 for the group's four blocks)
    // and 8 bytes of scales.
    auto dq_unit = [&](const Unit &un, auto na_tag, uint64_t *full, uint64_t *empty, RingPos &r,
                       uint32_t stages, uint8_t *ring, int stage_bytes) {
      constexpr int NA = decltype(na_tag)::value;
      constexpr int NM = NA * (kDqRows / 8);  // groups of 8 rows; half m / 2
      const int tile0 = un.rt * 8 * NA + dw;
      const uint8_t *gq = un.blob + p.q_off + (size_t)tile0 * G * 1024;
      const uint8_t *gs = un.blob + p.s_off + (size_t)tile0 * G * 128;
      auto q_at = [&](int m, int g) {
        return gq + ((size_t)(m >> 1) * 8 * G + g) * 1024 + (8 * (m & 1) + row_in_8) * 64 + w * 16;
      };
      auto s_at = [&](int m, int g) {
        return gs + ((size_t)(m >> 1) * 8 * G + g) * 128 + (8 * (m & 1) + row_in_8) * 8;
      };
      uint4 qn[NM];
      uint2 sn[NM];
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        qn[m] = ldg_nc_v4(q_at(m, 0));
        sn[m] = ldg_nc_v2(s_at(m, 0));
      }
      for (int g = 0; g < G && ok; ++g) {
        uint4 qc[NM];
        uint2 scur[NM];
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          qc[m] = qn[m];
          scur[m] = sn[m];
        }
        if (g + 1 < G) {
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            qn[m] = ldg_nc_v4(q_at(m, g + 1));
            sn[m] = ldg_nc_v2(s_at(m, g + 1));
          }
        }
        if (FMT == kFmtInt4) {
          // |scale| >= 8192 (or not finite): q * scale can overflow f16
#pragma unroll
          for (int m = 0; m < NM; ++m)
            big_scale |= (__vcmpgeu2(scur[m].x & 0x7FFF7FFFu, 0x70007000u) |
                          __vcmpgeu2(scur[m].y & 0x7FFF7FFFu, 0x70007000u)) != 0u;
        }
#pragma unroll
        for (int atom = 0; atom < 2 && ok; ++atom) {
          if (!wwait(&empty[r.st], r.ph ^ 1u, p.status)) { ok = false; break; }
          uint8_t *ad = ring + r.st * stage_bytes;
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            // row of the operand: half m / 2, this warp's 16 rows of it
            const int rr = kTcM * (m >> 1) + kDqRows * dw + 8 * (m & 1) + row_in_8;
            // blocks 2 atom and 2 atom + 1 of this row: word w of each
            const uint32_t words[2] = {atom ? qc[m].z : qc[m].x, atom ? qc[m].w : qc[m].y};
            const uint32_t sv = atom ? scur[m].y : scur[m].x;
            if (FMT == kFmtInt4) {
              const __half2 sc[2] = {__half2half2(__low2half(bits_h2(sv))),
                                     __half2half2(__high2half(bits_h2(sv)))};
#pragma unroll
              for (int b = 0; b < 2; ++b) {
                uint32_t f[4];
                int4x8_to_f16(words[b], f);
                uint4 o;
                o.x = h2_bits(__hmul2(bits_h2(f[0]), sc[b]));
                o.y = h2_bits(__hmul2(bits_h2(f[1]), sc[b]));
                o.z = h2_bits(__hmul2(bits_h2(f[2]), sc[b]));
                o.w = h2_bits(__hmul2(bits_h2(f[3]), sc[b]));
                const int chunk = (b * 4 + w) ^ (rr & 7);
                *reinterpret_cast<uint4 *>(ad + rr * 128 + chunk * 16) = o;
              }
            } else {
              // NVFP4: word w of block 2 atom + b is scale group 4 atom + 2 b
              // + w / 2 (byte 2 b + w / 2 of the four loaded); code x E4M3
              // scale is exact in f16
#pragma unroll
              for (int b = 0; b < 2; ++b) {
                const __half2 z = bits_h2(e4m3_to_f16x2_dup(sv >> (8 * (2 * b + (w >> 1)))));
                uint32_t f[4];
                e2m1x8_to_f16(words[b], f);
                uint4 o;
                o.x = h2_bits(__hmul2(bits_h2(f[0]), z));
                o.y = h2_bits(__hmul2(bits_h2(f[1]), z));
                o.z = h2_bits(__hmul2(bits_h2(f[2]), z));
                o.w = h2_bits(__hmul2(bits_h2(f[3]), z));
                const int chunk = (b * 4 + w) ^ (rr & 7);
                *reinterpret_cast<uint4 *>(ad + rr * 128 + chunk * 16) = o;
              }
            }
          }
          fence_async_smem();
          __syncwarp();
          warp_arrive(&full[r.st]);
          r.next(stages);
        }
      }
    };
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit un = decode(u, cur);
      if (!un.sw) {
        dq_unit(un, IntTag<1>{}, fullA, emptyA, ra, kAStages, smem + kOffA, kAStageBytes);
        continue;
      }
      // swapped: 256 rows into the B stages, once phase 1's activations
      // there have been read
      if (!phase2) {
        phase2 = true;
        if (!wwait(p1_done, 0u, p.status)) { ok = false; break; }
      }
      dq_unit(un, IntTag<2>{}, fullW, emptyW, rw, kBStages, smem + kOffB, kBStageBytes);
    }
    if (__any_sync(0xffffffffu, big_scale) && lane == 0) set_status(p.status, STATUS_RANGE);
  } else {
    // -------------------------------------------------------- epilogue
    const int ew = role.idx;                  // 0 .. kEpiWarps - 1
    const int qd = warp & 3;                  // TMEM lane quarter of this warp
    const int cpar = ew & 1;                  // which alternate 32-column blocks
    float *stage = reinterpret_cast<float *>(smem + kOffEpi + ew * 1024);
    AccTrack acc;
    bool ok = true, big_h = false;
    Cursor cur;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit un = decode(u, cur);
      if (un.sw) {
        // lane L of quarter qd: pair 32 qd + L of the block (M = 128); column c: weight
        // row c of the unit's 256, i.e. blob tile 16 rt + c / 16, tile row
        // c % 16 (for gate/up: gate if < 8, its up partner at c + 8)
        const int buf = acc.buf_of(1, 0);
        if (!wwait(&acc_full[buf], acc.uses[buf] & 1u, p.status)) { ok = false; break; }
        tc_fence_after();
        // M = 64: rows 16 qd .. 16 qd + 15 in lanes 0..15 of quarter qd
        const bool m64 = un.n <= 64;
        const int row = m64 ? 16 * qd + (lane & 15) : 32 * qd + lane;
        const bool mine = row < un.n && (!m64 || lane < 16);
        for (int col0 = 32 * cpar; col0 < kSwapRows && (m64 ? 16 : 32) * qd < un.n; col0 += 64) {
          float v[32];
          tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * qd) << 16) + buf * kAccCols + col0, v);
          if (kGateUp) {
            // blob tiles 16 rt + col0 / 16 + b: h columns 8 x that tile + the
            // packed position of the tile row
            __half hh[16];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float gv = v[16 * b + i], uv = v[16 * b + 8 + i];
                const float hv = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
                big_h |= mine && fabsf(hv) >= kF16Overflow;
                hh[8 * b + packed_pos<FMT>(i)] = __float2half_rn(hv);
              }
            }
            if (mine) {
              uint32_t hw[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) hw[k] = h2_bits(__halves2half2(hh[2 * k], hh[2 * k + 1]));
              uint4 *dst = reinterpret_cast<uint4 *>(p.h_out + (size_t)(un.pi0 + row) * p.out_ld +
                                                     kTcM * un.rt + col0 / 2);
              dst[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              dst[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
            }
          } else if (mine) {
            float4 *dst = reinterpret_cast<float4 *>(p.y_out + (size_t)(un.pi0 + row) * p.out_ld +
                                                     kSwapRows * un.rt + col0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          }
        }
        tc_fence_before();
        __syncwarp();
        warp_arrive(&acc_empty[buf]);
        acc.done_unit(1);
        continue;
      }
      const int nc = un.chunks();
      // NVFP4: this lane's row's global scale (gate, up or down)
      float gsc = 1.0f;
      if (FMT == kFmtNvfp4) {
        const float *gs = reinterpret_cast<const float *>(un.blob + p.glob_off);
        gsc = kGateUp ? gs[(lane & 15) < 8 ? 0 : 1] : gs[2];
      }
      for (int c = 0; c < nc && ok; ++c) {
        const int buf = acc.buf_of(nc, c);
        const int cn = un.chunk_n(c), pi0 = un.pi0 + c * kTcN;
        if (!wwait(&acc_full[buf], acc.uses[buf] & 1u, p.status)) { ok = false; break; }
        tc_fence_after();
        for (int col0 = 32 * cpar; col0 < cn; col0 += 64) {
          float v[32];
          tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * qd) << 16) + buf * kAccCols + col0, v);
          if (FMT == kFmtNvfp4) {
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] *= gsc;
          }
          if (kGateUp) {
            // lane L: blob tile 2 qd + L / 16, tile row L % 16 (gate if < 8);
            // of each column pair the gate lane computes the even column and
            // its up partner (L ^ 8) the odd one: each sends the partner the
            // value of the partner's column (one shuffle per pair, no branch)
            __half *hs = reinterpret_cast<__half *>(stage);  // [32 pairs][16]
            const bool is_up = (lane & 15) >= 8;
            const int pos16 = 8 * (lane >> 4) + packed_pos<FMT>(lane & 7);
#pragma unroll
            for (int t = 0; t < 32; t += 2) {
              const float mine = is_up ? v[t + 1] : v[t];
              const float other = __shfl_xor_sync(0xffffffffu, is_up ? v[t] : v[t + 1], 8);
              const float gv = is_up ? other : mine;
              const float uv = is_up ? mine : other;
              const float hv = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
              const int c = t + (is_up ? 1 : 0);
              // (columns past the chunk's pairs hold stale accumulators)
              big_h |= col0 + c < cn && fabsf(hv) >= kF16Overflow;
              hs[c * 16 + pos16] = __float2half_rn(hv);
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int piece = lane + 32 * k;  // 64 pieces of 16 bytes
              const int t = piece >> 1, half = piece & 1;
              if (col0 + t < cn) {
                const uint4 val = *reinterpret_cast<const uint4 *>(hs + t * 16 + half * 8);
                __half *dst = p.h_out + (size_t)(pi0 + col0 + t) * p.out_ld + 64 * un.rt +
                              16 * qd + 8 * half;
                *reinterpret_cast<uint4 *>(dst) = val;
              }
            }
            __syncwarp();
          } else {
            // 8 pairs at a time through a 1 KB stage: [8 pairs][32 rows] fp32
#pragma unroll
            for (int t8 = 0; t8 < 32; t8 += 8) {
#pragma unroll
              for (int t = 0; t < 8; ++t) stage[t * 32 + lane] = v[t8 + t];
              __syncwarp();
#pragma unroll
              for (int k = 0; k < 2; ++k) {
                const int piece = lane + 32 * k;  // 64 pieces of 16 bytes
                const int t = piece >> 3, seg = piece & 7;
                if (col0 + t8 + t < cn) {
                  const float4 val = *reinterpret_cast<const float4 *>(stage + t * 32 + seg * 4);
                  float *dst = p.y_out + (size_t)(pi0 + col0 + t8 + t) * p.out_ld + 128 * un.rt +
                               32 * qd + 4 * seg;
                  *reinterpret_cast<float4 *>(dst) = val;
                }
              }
              __syncwarp();
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        warp_arrive(&acc_empty[buf]);
      }
      acc.done_unit(nc);
    }
    if (__any_sync(0xffffffffu, big_h) && lane == 0) set_status(p.status, STATUS_RANGE);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template __global__ void expert_tc_kernel<true, kFmtInt4>(TcParams,
                                                         const __grid_constant__ CUtensorMap,
                                                         const __grid_constant__ CUtensorMap,
                                                         const __grid_constant__ CUtensorMap);
template __global__ void expert_tc_kernel<false, kFmtInt4>(TcParams,
                                                          const __grid_constant__ CUtensorMap,
                                                          const __grid_constant__ CUtensorMap,
                                                          const __grid_constant__ CUtensorMap);
template __global__ void expert_tc_kernel<true, kFmtNvfp4>(TcParams,
                                                          const __grid_constant__ CUtensorMap,
                                                          const __grid_constant__ CUtensorMap,
                                                          const __grid_constant__ CUtensorMap);
template __global__ void expert_tc_kernel<false, kFmtNvfp4>(TcParams,
                                                           const __grid_constant__ CUtensorMap,
                                                           const __grid_constant__ CUtensorMap,
                                                           const __grid_constant__ CUtensorMap);

// x_perm[pair] = x16[token of pair], 16 bytes per thread.
__global__ void gather_rows_kernel(const __half *__restrict__ x16, const int *__restrict__ pair_tok,
                                   const int *__restrict__ n_pairs_dev, int H, int P_cap,
                                   __half *__restrict__ xp) {
  grid_dependency_wait();
  const int n_pairs = min(*n_pairs_dev, P_cap);
  const int per_row = H / 8;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (long long)n_pairs * per_row;
       i += (long long)gridDim.x * blockDim.x) {
    const int pr = (int)(i / per_row), c = (int)(i - (long long)pr * per_row);
    const uint4 v = *reinterpret_cast<const uint4 *>(x16 + (size_t)pair_tok[pr] * H + c * 8);
    *reinterpret_cast<uint4 *>(xp + (size_t)pr * H + c * 8) = v;
  }
}

}  // namespace strata
