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
// Warp roles (one CTA per SM, persistent; units interleaved over CTAs; the
// warp ids of each role are in tc_warp below):
//   activation producer: per 64 K elements (one swizzle atom) and chunk, the
//               activation rows (f16, 128-byte swizzle; x_perm or h16) in one
//               256-row TMA box, or in 64-row and 16-row boxes for shorter
//               chunks;
//   MMA: allocates all 512 TMEM columns (two 256-column accumulators), and
//               one thread issues 4 tcgen05.mma (M=128, N=chunk pairs rounded
//               up to 16, K=16) per atom and chunk, commits to the operand
//               stages and, at the end of a unit, to the accumulators it used;
//   8 dequant warps: load their rows' packed weights and scales straight
//               from global memory (one K group ahead; dequant warp 0 brings
//               the weights of the units ahead into L2 by bulk prefetches),
//               int4 -> exact f16 integers -> times the fp16 scale (one f16
//               rounding), or NVFP4 E2M1 codes times their E4M3 group scale
//               (exact in f16; the fp32 global scale multiplies the
//               accumulator in the epilogue) -> the K-major 128-byte-swizzled
//               A layout, 16 rows each;
//   8 epilogue warps: two per TMEM lane quarter, each taking alternate
//               32-column blocks: tcgen05.ld, SwiGLU (gate/up; the gate lane
//               and its up partner each compute one column of every pair) or
//               plain (down), transposed through shared memory, stored;
//   one more warp has no role (it kept a ring of packed weights in shared
//               memory, which now goes to the activation ring).  One thread
//               issues all MMAs: a variant with a second issuing thread (one
//               per accumulator) faulted once and is not used.
// The A operand (16 KB per atom) and the B operand (32 KB per atom and
// chunk) have rings of their own (three and five stages) with one "full" and
// one "empty" mbarrier per stage: the kernel is bound by the hand-offs
// between its roles, and the depth of the activation ring, in stages, is what
// counts most.  A unit of two chunks uses both accumulators; a unit of one
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
constexpr int kPfUnits = 2;        // units whose weights are prefetched into L2 ahead
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
constexpr int kNumBars = 2 * kAStages + 2 * kBStages + 4;
constexpr int kOffTab = kOffBar + kNumBars * 8 + 16;   // + TMEM address slot
constexpr int kTabBytes = kMaxIds * 8 + (3 * kMaxIds + 1) * 4;
constexpr int kTcSmem = kOffTab + kTabBytes + 1024;    // + alignment slack

__device__ __forceinline__ bool wwait(uint64_t *bar, uint32_t parity, int *status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
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

struct Unit {
  const uint8_t *blob;
  int pi0, n, rt;
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
  // fullA[s]: the dequant warps' arrivals; fullB[s]: the activation TMA bytes;
  // emptyA/emptyB[s]: the MMAs that read stage s have completed
  uint64_t *fullA = bars, *emptyA = fullA + kAStages;
  uint64_t *fullB = emptyA + kAStages, *emptyB = fullB + kBStages;
  uint64_t *acc_full = emptyB + kBStages, *acc_empty = acc_full + 2;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + kNumBars);
  const uint8_t **t_blob = reinterpret_cast<const uint8_t **>(smem + kOffTab);
  int *t_off = reinterpret_cast<int *>(t_blob + kMaxIds);
  int *t_cnt = t_off + kMaxIds;
  int *unit_base = t_cnt + kMaxIds;

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
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kEpiWarps);
    }
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
  if (warp == 0) {
    int carry = 0;
    for (int a0 = 0; a0 < n_active; a0 += 32) {
      const int a = a0 + lane;
      const int v = a < n_active && t_blob[a]
                        ? ((t_cnt[a] + kUnitPairs - 1) / kUnitPairs) * p.row_tiles : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int nb = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nb;
      }
      if (a < n_active) unit_base[a] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) unit_base[n_active] = carry;
  }
  __syncthreads();
  grid_dependency_launch();

  const int n_units = unit_base[n_active];
  const int G = p.K / 128;  // K groups
  auto decode = [&](int u, int &a) -> Unit {
    while (unit_base[a + 1] <= u) ++a;
    const int rem = u - unit_base[a];
    const int ub = rem / p.row_tiles;
    Unit un;
    un.rt = rem - ub * p.row_tiles;
    un.pi0 = t_off[a] + ub * kUnitPairs;
    un.n = min(kUnitPairs, t_cnt[a] - ub * kUnitPairs);
    un.blob = t_blob[a];
    return un;
  };

  if (role.role == kRoleAct) {
    // -------------------------------------------------------- activation producer
    uint32_t issued = 0;
    RingPos rb;
    bool ok = true;
    int a = 0;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit un = decode(u, a);
      const int nc = un.chunks();
      for (int at = 0; at < 2 * G && ok; ++at) {
        for (int c = 0; c < nc; ++c) {
          if (!wwait(&emptyB[rb.st], rb.ph ^ 1u, p.status)) { ok = false; break; }
          const int cn = un.chunk_n(c), row0 = un.pi0 + c * kTcN;
          // one 256-row box, else 64-row boxes and 16-row boxes for the rest
          // (rows land at 128 bytes each whatever the box, so the swizzled
          // layout is the same)
          const bool wide = cn > 192;
          const int n64 = wide ? 0 : cn / 64;
          const int n16 = wide ? 0 : (cn - 64 * n64 + 15) / 16;
          const uint32_t tx = wide ? 32768u : n64 * 8192u + n16 * 2048u;
          uint8_t *dst = smem + kOffB + rb.st * kBStageBytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(&fullB[rb.st], tx);
            if (wide) {
              tma_load_2d(dst, &tmap_b256, at * 64, row0, &fullB[rb.st]);
            } else {
              for (int q = 0; q < n64; ++q)
                tma_load_2d(dst + q * 8192, &tmap_b64, at * 64, row0 + q * 64, &fullB[rb.st]);
              for (int q = 0; q < n16; ++q)
                tma_load_2d(dst + n64 * 8192 + q * 2048, &tmap_b16, at * 64, row0 + 64 * n64 + 16 * q,
                            &fullB[rb.st]);
            }
          }
          __syncwarp();
          ++issued;
          rb.next(kBStages);
        }
      }
    }
    if (!ok) {
      // let issued copies land before the CTA exits (bounded waits)
      for (uint32_t m = issued > kBStages ? issued - kBStages : 0; m < issued; ++m)
        (void)wwait(&fullB[m % kBStages], (m / kBStages) & 1u, p.status);
    }
  } else if (role.role == kRoleIdle) {
    // -------------------------------------------------------- (no role)
  } else if (role.role == kRoleMma) {
    // -------------------------------------------------------- MMA issue
    // One thread does it all: per atom one wait for A, per chunk one wait for
    // B, four MMAs and one commit, so the tensor pipe's queue never runs dry
    // behind warp-level overheads.
    if (lane == 0) {
      RingPos ra, rb;
      AccTrack acc;
      bool ok = true;
      int a = 0;
      // stage 0's descriptors; a stage adds its offset / 16 to the address
      // field, a 16-element K step (32 bytes) adds 2
      const uint64_t a_desc0 = umma_desc_sw128(smem_u32(smem + kOffA));
      const uint64_t b_desc0 = umma_desc_sw128(smem_u32(smem + kOffB));
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit un = decode(u, a);
        const int nc = un.chunks();
        uint32_t idesc[2], d_tmem[2];
        int bufs[2];
        for (int c = 0; c < nc; ++c) {
          bufs[c] = acc.buf_of(nc, c);
          idesc[c] = umma_idesc_f16(kTcM, (un.chunk_n(c) + 15) & ~15);
          d_tmem[c] = tmem_base + bufs[c] * kAccCols;
        }
        for (int at = 0; at < 2 * G && ok; ++at) {
          if (!mbar_wait(&fullA[ra.st], ra.ph, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = a_desc0 + (uint64_t)((ra.st * kAStageBytes) >> 4);
          for (int c = 0; c < nc; ++c) {
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
        if (!ok) break;
        for (int c = 0; c < nc; ++c) umma_commit(&acc_full[bufs[c]]);
        acc.done_unit(nc);
      }
    }
    __syncwarp();
  } else if (role.role == kRoleDq) {
    // -------------------------------------------------------- dequant
    const int dw = role.idx;
    const int w = lane & 3;
    const int q = lane >> 2;
    const int row_in_8 = (q & 1) * 4 + (q >> 1);  // lanes 8p..8p+7 -> rows p and p + 4
    RingPos ra;
    bool ok = true, big_scale = false;
    int a = 0, a_pf = 0;
    // warp 0 of the dequant role brings the weights of the units ahead into
    // L2 (one bulk prefetch per blob tile and section)
    auto prefetch_unit = [&](int v) {
      if (dw != 0 || v >= n_units || lane >= 8) return;
      const Unit nx = decode(v, a_pf);
      const int tile = nx.rt * 8 + lane;
      bulk_prefetch_l2(nx.blob + p.q_off + (size_t)tile * G * 1024, (uint32_t)G * 1024u);
      bulk_prefetch_l2(nx.blob + p.s_off + (size_t)tile * G * 128, (uint32_t)G * 128u);
    };
    for (int i = 0; i < kPfUnits; ++i) prefetch_unit(blockIdx.x + i * gridDim.x);
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit un = decode(u, a);
      prefetch_unit(u + kPfUnits * gridDim.x);
      // this warp's 16 rows are blob tile 8 rt + dw; per K group, row tr holds
      // 64 bytes of packed weights (word w of each 32-element block: bytes
      // 16 w .. 16 w + 15 for the group's four blocks) and 8 bytes of scales
      const uint8_t *gq = un.blob + p.q_off + (size_t)(un.rt * 8 + dw) * G * 1024;
      const uint8_t *gs = un.blob + p.s_off + (size_t)(un.rt * 8 + dw) * G * 128;
      uint4 qn[kDqRows / 8];
      uint2 sn[kDqRows / 8];
#pragma unroll
      for (int m = 0; m < kDqRows / 8; ++m) {
        const int tr = 8 * m + row_in_8;
        qn[m] = ldg_nc_v4(gq + tr * 64 + w * 16);
        sn[m] = ldg_nc_v2(gs + tr * 8);
      }
      for (int g = 0; g < G && ok; ++g) {
        uint4 qc[kDqRows / 8];
        uint2 scur[kDqRows / 8];
#pragma unroll
        for (int m = 0; m < kDqRows / 8; ++m) {
          qc[m] = qn[m];
          scur[m] = sn[m];
        }
        if (g + 1 < G) {
#pragma unroll
          for (int m = 0; m < kDqRows / 8; ++m) {
            const int tr = 8 * m + row_in_8;
            qn[m] = ldg_nc_v4(gq + (size_t)(g + 1) * 1024 + tr * 64 + w * 16);
            sn[m] = ldg_nc_v2(gs + (size_t)(g + 1) * 128 + tr * 8);
          }
        }
        for (int atom = 0; atom < 2 && ok; ++atom) {
          if (!wwait(&emptyA[ra.st], ra.ph ^ 1u, p.status)) { ok = false; break; }
          uint8_t *ad = smem + kOffA + ra.st * kAStageBytes;
#pragma unroll
          for (int m = 0; m < kDqRows / 8; ++m) {
            const int r = kDqRows * dw + 8 * m + row_in_8;
            // blocks 2 atom and 2 atom + 1 of this row: word w of each
            const uint32_t words[2] = {atom ? qc[m].z : qc[m].x, atom ? qc[m].w : qc[m].y};
            const uint32_t sv = atom ? scur[m].y : scur[m].x;
            if (FMT == kFmtInt4) {
              // |scale| >= 8192 (or not finite): q * scale can overflow f16
              big_scale |= __vcmpgeu2(sv & 0x7FFF7FFFu, 0x70007000u) != 0u;
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
                const int chunk = (b * 4 + w) ^ (r & 7);
                *reinterpret_cast<uint4 *>(ad + r * 128 + chunk * 16) = o;
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
                const int chunk = (b * 4 + w) ^ (r & 7);
                *reinterpret_cast<uint4 *>(ad + r * 128 + chunk * 16) = o;
              }
            }
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&fullA[ra.st]);
          ra.next(kAStages);
        }
        if (!ok) break;
      }
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
    int a = 0;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit un = decode(u, a);
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
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
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
