// Host side of the C interface in include/strata_moe.h: the handle, argument
// checks, the expert-id -> slot table, the device workspace, the kernel
// sequence of a forward call, the device status word and optional per-kernel
// timing.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "kernels.h"
#include "strata_moe.h"

using namespace strata;

namespace {

constexpr int kPhases = 9;
enum Phase {
  PH_ROUTER = 0, PH_TOPK, PH_BUCKET, PH_PACK, PH_GATEUP, PH_DOWN, PH_COMBINE, PH_GATHER, PH_FUSED
};

struct EventPair {
  int phase;
  cudaEvent_t a, b;
};

}  // namespace

struct strata_moe {
  int H, I, E, k, S, n_slots;
  int device = 0, num_sms = 0;
  int fmt = kFmtInt4;       // weight format of every blob of the layer
  BlobLayout layout{};

  std::vector<int> slot_expert;            // per slot: expert id or -1
  std::vector<const void *> slot_ptr;      // per slot: blob
  std::vector<int> expert_slot;            // per expert: slot or -1
  std::vector<const void *> shared_ptr;    // per shared expert
  const float *router_W = nullptr;
  const float *router_b = nullptr;
  RouteMode mode{0, nullptr, 1.0f};

  // workspace
  int cap_tokens = 0;
  void *ws = nullptr;
  size_t ws_bytes = 0;
  float *logits = nullptr;
  int32_t *idx = nullptr;
  float *w = nullptr;
  int *meta = nullptr;      // cnt | off | active | n_active
  Routing rt{};
  __half *x16 = nullptr;
  __half *h16 = nullptr;
  float *y = nullptr;
  __half *xp = nullptr;     // activations gathered in sorted pair order (large batches)
  double *rpart = nullptr;  // decode kernel: router partial sums
  float *partial = nullptr; // decode kernel: partial sums of items cut between warps
  int *counters = nullptr;  // decode kernel: barrier, cut-item and tile counters (zero between launches)
  size_t counters_bytes = 0;
  unsigned long long wait_ns = STRATA_DEFAULT_WAIT_NS;  // limit of the decode kernel's waits
  int *status = nullptr;    // device status word (own allocation)
  int *counter = nullptr;   // last-block counter of the small-batch routing kernel
  int last_bits = 0;

  // per-kernel timing
  bool profiling = false;
  std::vector<EventPair> events;
  std::vector<cudaEvent_t> event_pool;
  int prof_launches[kPhases] = {};
  double prof_ms[kPhases] = {};
};

namespace {

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

strata_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return STRATA_OK;
  if (e == cudaErrorMemoryAllocation) return STRATA_ERR_OOM;
  return STRATA_ERR_CUDA;
}

cudaEvent_t take_event(strata_moe *h) {
  if (!h->event_pool.empty()) {
    cudaEvent_t e = h->event_pool.back();
    h->event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Launch `kern` on `stream`; pdl lets it start while the previous kernel in
// the stream drains (every kernel here begins with griddepcontrol.wait
// before it reads anything the previous kernels wrote).
template <typename... Exp, typename... Act>
cudaError_t launch(strata_moe *h, int phase, void (*kern)(Exp...), dim3 grid, dim3 block,
                   size_t smem, cudaStream_t stream, bool pdl, Act &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (pdl && !h->profiling) ? 1 : 0;
  EventPair ev{phase, nullptr, nullptr};
  if (h->profiling) {
    ev.a = take_event(h);
    ev.b = take_event(h);
    cudaEventRecord(ev.a, stream);
  }
  cudaError_t err = cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
  if (h->profiling) {
    cudaEventRecord(ev.b, stream);
    h->events.push_back(ev);
  }
  return err;
}

// Decode kernel workspace: two partial-sum slots per warp of the grid and
// phase (a warp may start its down-projection pieces while the last piece of
// one of its cut gate/up items has yet to read its slot); the counters: 4
// barrier/exit counters, one cut-item counter per warp and phase, one tile
// counter per 16 output rows, one readiness counter per pair group.
size_t fused_partial_bytes(const strata_moe *h) {
  return sizeof(float) * 2 * 2 * (size_t)kFusedWarps * h->num_sms * kMmSlotFloats;
}
size_t fused_counter_bytes(const strata_moe *h) {
  return sizeof(int) * (4 + 2 * (size_t)kFusedWarps * h->num_sms + (size_t)h->H / 16 +
                        (size_t)kSmallT * (kMaxTopK + kMaxShared));
}

strata_status grow_workspace(strata_moe *h, int T) {
  if (T <= h->cap_tokens) return STRATA_OK;
  const int cap = std::max(T, 2 * h->cap_tokens);
  const int kS = h->k + h->S;
  const size_t P = (size_t)cap * kS;
  const int nid = h->E + h->S;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t o_logits = take(sizeof(float) * cap * h->E);
  const size_t o_idx = take(sizeof(int32_t) * cap * h->k);
  const size_t o_w = take(sizeof(float) * cap * h->k);
  const size_t o_meta = take(sizeof(int) * (3 * nid + 2));
  const size_t o_ptok = take(sizeof(int) * P);
  const size_t o_pj = take(sizeof(int) * P);
  const size_t o_inv = take(sizeof(int) * P);
  const size_t o_x16 = take(sizeof(__half) * cap * h->H);
  const size_t o_h16 = take(sizeof(__half) * P * h->I);
  const size_t o_y = take(sizeof(float) * P * h->H);
  const size_t o_xp = cap > kSmallT ? take(sizeof(__half) * P * h->H) : 0;
  const size_t o_rpart = take(sizeof(double) * std::max(h->E, h->num_sms) * (size_t)cap);
  const size_t o_partial = take(fused_partial_bytes(h));
  const size_t o_counters = take(fused_counter_bytes(h));
  void *mem = nullptr;
  cudaError_t e = cudaMalloc(&mem, off);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_status(e);
  }
  if (h->ws) cudaFree(h->ws);
  h->ws = mem;
  h->ws_bytes = off;
  h->cap_tokens = cap;
  char *b = static_cast<char *>(mem);
  h->logits = reinterpret_cast<float *>(b + o_logits);
  h->idx = reinterpret_cast<int32_t *>(b + o_idx);
  h->w = reinterpret_cast<float *>(b + o_w);
  h->meta = reinterpret_cast<int *>(b + o_meta);
  h->rt.cnt = h->meta;
  h->rt.off = h->meta + nid;
  h->rt.active = h->meta + 2 * nid + 1;
  h->rt.n_active = h->meta + 3 * nid + 1;
  h->rt.pair_tok = reinterpret_cast<int *>(b + o_ptok);
  h->rt.pair_j = reinterpret_cast<int *>(b + o_pj);
  h->rt.inv = reinterpret_cast<int *>(b + o_inv);
  h->x16 = reinterpret_cast<__half *>(b + o_x16);
  h->h16 = reinterpret_cast<__half *>(b + o_h16);
  h->y = reinterpret_cast<float *>(b + o_y);
  h->xp = cap > kSmallT ? reinterpret_cast<__half *>(b + o_xp) : nullptr;
  h->rpart = reinterpret_cast<double *>(b + o_rpart);
  h->partial = reinterpret_cast<float *>(b + o_partial);
  h->counters = reinterpret_cast<int *>(b + o_counters);
  h->counters_bytes = fused_counter_bytes(h);
  e = cudaMemset(h->counters, 0, h->counters_bytes);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e);
  return STRATA_OK;
}

ExpertTable make_table(const strata_moe *h) {
  ExpertTable t;
  std::memset(&t, 0, sizeof t);
  for (int s = 0; s < h->n_slots; ++s)
    if (h->slot_expert[s] >= 0) t.ptr[h->slot_expert[s]] = static_cast<const uint8_t *>(h->slot_ptr[s]);
  for (int i = 0; i < h->S; ++i) t.ptr[h->E + i] = static_cast<const uint8_t *>(h->shared_ptr[i]);
  return t;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void *ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// Rows of f16 activations [rows][K] as the B operand of the tensor-core
// kernel: boxes of 64 K x box_rows rows, 128-byte swizzle.
bool encode_rows_map(CUtensorMap *m, const __half *base, int K, int rows, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Activations gathered in sorted pair order (large batches).
strata_status run_gather(strata_moe *h, int T, cudaStream_t stream) {
  const int P = T * (h->k + h->S);
  const int per_row = h->H / 8;
  const long long work = (long long)P * per_row;
  const int gblocks = (int)std::min<long long>((work + 255) / 256, 8LL * h->num_sms);
  return cuda_status(launch(h, PH_GATHER, gather_rows_kernel, dim3(gblocks), dim3(256), 0, stream,
                            true, h->x16, h->rt.pair_tok, h->rt.off + (h->E + h->S), h->H, P,
                            h->xp));
}

// The two tensor-core passes over the experts that `table` binds.  quiet: the
// routed experts without a blob belong to another pass of the same batch.
strata_status run_tc_passes(strata_moe *h, int T, const ExpertTable &table, bool quiet,
                            cudaStream_t stream) {
  const int P = T * (h->k + h->S);
  cudaError_t e;
  const size_t smem = tc_smem_bytes();
  for (int pass = 0; pass < 2; ++pass) {
    const bool gu = pass == 0;
    TcParams p;
    std::memset(&p, 0, sizeof p);
    p.table = table;
    p.rt = h->rt;
    p.K = gu ? h->H : h->I;
    p.row_tiles = gu ? h->I / 64 : h->H / 128;
    p.q_off = gu ? h->layout.guq : h->layout.dq;
    p.s_off = gu ? h->layout.gus : h->layout.ds;
    p.out_ld = gu ? h->I : h->H;
    p.h_out = h->h16;
    p.y_out = h->y;
    p.status = h->status;
    p.quiet_unbound = quiet ? 1 : 0;
    p.glob_off = h->layout.glob;
    CUtensorMap m16, m64, m256;
    if (!encode_rows_map(&m16, gu ? h->xp : h->h16, p.K, P, 16) ||
        !encode_rows_map(&m64, gu ? h->xp : h->h16, p.K, P, 64) ||
        !encode_rows_map(&m256, gu ? h->xp : h->h16, p.K, P, 256))
      return STRATA_ERR_CUDA;
    auto kern = h->fmt == kFmtInt4
                    ? (gu ? expert_tc_kernel<true, kFmtInt4> : expert_tc_kernel<false, kFmtInt4>)
                    : (gu ? expert_tc_kernel<true, kFmtNvfp4> : expert_tc_kernel<false, kFmtNvfp4>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = launch(h, gu ? PH_GATEUP : PH_DOWN, kern, dim3(h->num_sms), dim3(tc_threads()), smem,
                 stream, true, p, m16, m64, m256);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return STRATA_OK;
}

strata_status check_common(strata_moe *h, const void *x, int T, cudaStream_t) {
  if (!h || T < 0) return STRATA_ERR_INVALID_ARG;
  if (T > 0 && (!x || (reinterpret_cast<uintptr_t>(x) & 15))) return STRATA_ERR_INVALID_ARG;
  return STRATA_OK;
}

// Activation pack + bucketing of a large batch, given idx in device memory.
strata_status run_prepare(strata_moe *h, const void *x, int T, const int32_t *idx,
                          cudaStream_t stream) {
  const int kS = h->k + h->S;
  const int nid = h->E + h->S;
  cudaError_t e = cudaMemsetAsync(h->rt.cnt, 0, sizeof(int) * nid, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->rt.inv, 0xFF, sizeof(int) * (size_t)T * kS, stream);
  if (e != cudaSuccess) return cuda_status(e);
  const auto *xb = static_cast<const __nv_bfloat16 *>(x);
  const int n8 = T * h->H / 8;
  e = launch(h, PH_PACK, pack_x_kernel, dim3((n8 + 255) / 256), dim3(256), 0, stream, false, xb,
             n8, h->x16, h->fmt, h->status);
  if (e == cudaSuccess)
    e = launch(h, PH_BUCKET, bucket_count_kernel, dim3((T * h->k + 255) / 256), dim3(256), 0,
               stream, true, idx, T, h->k, h->E, h->rt.cnt, h->status);
  if (e == cudaSuccess)
    e = launch(h, PH_BUCKET, bucket_fill_kernel, dim3(nid), dim3(256), 0, stream, true, idx, T,
               h->k, h->E, h->S, h->rt);
  return cuda_status(e);
}

strata_status run_combine(strata_moe *h, int T, const int32_t *idx, const float *w,
                          const ExpertTable &table, bool check_bound, void *out,
                          cudaStream_t stream) {
  dim3 cgrid((h->H / 4 + 127) / 128, T);
  return cuda_status(launch(h, PH_COMBINE, combine_kernel, cgrid, dim3(128), 0, stream, true,
                            h->y, idx, w, h->rt.inv, table, check_bound ? 1 : 0, T, h->H, h->k,
                            h->S, h->E, static_cast<__nv_bfloat16 *>(out)));
}

// Large batches (T > 64): bucketing + the tensor-core expert passes + combine,
// given idx/w in device memory.
strata_status run_experts(strata_moe *h, const void *x, int T, const int32_t *idx, const float *w,
                          void *out, cudaStream_t stream) {
  const ExpertTable table = make_table(h);
  strata_status st = run_prepare(h, x, T, idx, stream);
  if (st == STRATA_OK) st = run_gather(h, T, stream);
  if (st == STRATA_OK) st = run_tc_passes(h, T, table, false, stream);
  if (st == STRATA_OK) st = run_combine(h, T, idx, w, table, true, out, stream);
  return st;
}

SmallRouteParams small_params(strata_moe *h, const void *x, int T, float *logits, int32_t *idx,
                              float *w) {
  SmallRouteParams p;
  p.x = static_cast<const __nv_bfloat16 *>(x);
  p.W = h->router_W;
  p.bias = h->router_b;
  p.T = T;
  p.H = h->H;
  p.E = h->E;
  p.k = h->k;
  p.logits = logits;
  p.idx = idx;
  p.w = w;
  p.counter = h->counter;
  p.mode = h->mode;
  return p;
}

// Router + top-k.
strata_status run_router(strata_moe *h, const void *x, int T, float *logits, int32_t *idx,
                         float *w, cudaStream_t stream) {
  const auto *xb = static_cast<const __nv_bfloat16 *>(x);
  cudaError_t e;
  if (T <= kSmallT) {
    const SmallRouteParams p = small_params(h, x, T, logits, idx, w);
    e = launch(h, PH_ROUTER, route_small_kernel, dim3(h->E), dim3(256), 0, stream, false, p);
    return cuda_status(e);
  }
  e = launch(h, PH_ROUTER, router_gemm_kernel, dim3((T + 127) / 128, (h->E + 63) / 64), dim3(256), 0,
             stream, false, xb, h->router_W, h->router_b, T, h->H, h->E, logits);
  if (e == cudaSuccess)
    e = launch(h, PH_TOPK, topk_kernel, dim3((T + 7) / 8), dim3(256), 0, stream, true, logits, T,
               h->E, h->k, h->mode, idx, w);
  return cuda_status(e);
}

// The whole small-batch layer in one cooperative launch (decode_fused.cu).
// idx_in/w_in: the routing, or null to compute it.
strata_status run_fused(strata_moe *h, const void *x, int T, const int32_t *idx_in,
                        const float *w_in, void *out, cudaStream_t stream) {
  FusedParams p;
  std::memset(&p, 0, sizeof p);
  p.table = make_table(h);
  p.x = static_cast<const __nv_bfloat16 *>(x);
  p.W = h->router_W;
  p.bias = h->router_b;
  p.mode = h->mode;
  p.idx_in = idx_in;
  p.w_in = w_in;
  p.T = T;
  p.H = h->H;
  p.I = h->I;
  p.E = h->E;
  p.k = h->k;
  p.S = h->S;
  p.guq = h->layout.guq;
  p.gus = h->layout.gus;
  p.dq = h->layout.dq;
  p.ds = h->layout.ds;
  p.group = T <= 8 ? 8 : kMmMaxGroup;
  p.wait_ns = h->wait_ns;
  // ring stages of 512 K elements (4 KB of packed weights + 512 B of scales
  // per copy pair), as many per warp as fit beside the tables
  p.kc = 512;
  p.stage_bytes = (int)align_up((size_t)p.kc * 9, 128);
  const size_t tables = fused_table_bytes(T, h->k, h->S);
  const size_t bars = (size_t)kFusedWarps * kMmMaxStages * sizeof(uint64_t);
  const size_t avail = 232448 - tables - bars;
  p.stages = (int)std::min<size_t>(kMmMaxStages, avail / ((size_t)kFusedWarps * p.stage_bytes));
  if (p.stages < 2) return STRATA_ERR_UNSUPPORTED;
  p.smem_tables = (size_t)kFusedWarps * p.stages * p.stage_bytes + bars;
  const size_t smem = p.smem_tables + tables;
  p.rpart = h->rpart;
  p.idx = h->idx;
  p.w = h->w;
  p.x16 = h->x16;
  p.h16 = h->h16;
  p.y = h->y;
  p.partial = h->partial;
  p.bar = h->counters;
  p.cut_cnt = h->counters + 4;
  p.tile_cnt = h->counters + 4 + 2 * kFusedWarps * h->num_sms;
  p.grp_done = p.tile_cnt + h->H / 16;
  p.status = h->status;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.glob = h->layout.glob;
  auto kern = h->fmt == kFmtInt4
                  ? (p.group <= 8 ? decode_fused_kernel<1, kFmtInt4> : decode_fused_kernel<2, kFmtInt4>)
                  : (p.group <= 8 ? decode_fused_kernel<1, kFmtNvfp4>
                                  : decode_fused_kernel<2, kFmtNvfp4>);
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_status(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(h->num_sms);
  cfg.blockDim = dim3(32 * kFusedWarps);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // every CTA must be resident at once: the phases meet at grid barriers
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  EventPair ev{PH_FUSED, nullptr, nullptr};
  if (h->profiling) {
    ev.a = take_event(h);
    ev.b = take_event(h);
    cudaEventRecord(ev.a, stream);
  }
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (h->profiling) {
    cudaEventRecord(ev.b, stream);
    h->events.push_back(ev);
  }
  return cuda_status(e);
}

}  // namespace

extern "C" {

const char *strata_status_str(strata_status s) {
  switch (s) {
    case STRATA_OK: return "ok";
    case STRATA_ERR_INVALID_ARG: return "invalid argument";
    case STRATA_ERR_UNSUPPORTED: return "unsupported shape";
    case STRATA_ERR_NOT_BOUND: return "routed expert not bound to a slot";
    case STRATA_ERR_SLOT_CONFLICT: return "expert already bound to another slot";
    case STRATA_ERR_TOO_MANY_EXPERTS: return "more distinct experts than slots";
    case STRATA_ERR_OOM: return "out of device memory";
    case STRATA_ERR_CUDA: return "CUDA error";
    case STRATA_ERR_DEVICE_STATUS: return "device-side error";
    case STRATA_ERR_SCRATCH_LIMIT:
      return "request larger than the fixed scratch of strata_moe_forward_noalloc";
    case STRATA_ERR_RANGE:
      return "a value left the f16 range of the tensor-core operands";
  }
  return "unknown status";
}

size_t strata_moe_expert_bytes(int hidden, int inter) {
  return strata_moe_expert_bytes_fmt(hidden, inter, STRATA_FORMAT_INT4);
}

size_t strata_moe_expert_bytes_fmt(int hidden, int inter, int fmt) {
  if (hidden <= 0 || inter <= 0 || hidden % 128 || inter % 128) return 0;
  if (fmt != STRATA_FORMAT_INT4 && fmt != STRATA_FORMAT_NVFP4) return 0;
  return blob_layout(hidden, inter, fmt).total;
}

strata_status strata_moe_set_format(strata_moe *h, int fmt) {
  if (!h || (fmt != STRATA_FORMAT_INT4 && fmt != STRATA_FORMAT_NVFP4)) return STRATA_ERR_INVALID_ARG;
  for (int s = 0; s < h->n_slots; ++s)
    if (h->slot_expert[s] >= 0) return STRATA_ERR_INVALID_ARG;
  for (int i = 0; i < h->S; ++i)
    if (h->shared_ptr[i]) return STRATA_ERR_INVALID_ARG;
  h->fmt = fmt;
  h->layout = blob_layout(h->H, h->I, fmt);
  return STRATA_OK;
}

strata_status strata_moe_create(int hidden, int inter, int n_experts, int top_k, int n_shared,
                                int n_slots, strata_moe **out) {
  if (!out) return STRATA_ERR_INVALID_ARG;
  *out = nullptr;
  if (hidden <= 0 || inter <= 0 || hidden % 128 || inter % 128) return STRATA_ERR_INVALID_ARG;
  if (n_experts < 1 || n_experts > kMaxExperts) return STRATA_ERR_INVALID_ARG;
  if (top_k < 1 || top_k > n_experts || top_k > kMaxTopK) return STRATA_ERR_INVALID_ARG;
  if (n_shared < 0 || n_shared > kMaxShared) return STRATA_ERR_INVALID_ARG;
  if (n_slots < top_k || n_slots > n_experts) return STRATA_ERR_INVALID_ARG;
  strata_moe *h = new (std::nothrow) strata_moe();
  if (!h) return STRATA_ERR_OOM;
  h->H = hidden;
  h->I = inter;
  h->E = n_experts;
  h->k = top_k;
  h->S = n_shared;
  h->n_slots = n_slots;
  h->layout = blob_layout(hidden, inter);
  h->slot_expert.assign(n_slots, -1);
  h->slot_ptr.assign(n_slots, nullptr);
  h->expert_slot.assign(n_experts, -1);
  h->shared_ptr.assign(n_shared, nullptr);
  cudaError_t e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
  if (e == cudaSuccess) e = cudaMalloc(&h->status, 64);
  if (e == cudaSuccess) e = cudaMemset(h->status, 0, 64);
  h->counter = h->status + 16;
  if (e != cudaSuccess) {
    cudaGetLastError();
    if (h->status) cudaFree(h->status);
    delete h;
    return cuda_status(e);
  }
  *out = h;
  return STRATA_OK;
}

void strata_moe_destroy(strata_moe *h) {
  if (!h) return;
  cudaDeviceSynchronize();
  for (auto &ev : h->events) {
    cudaEventDestroy(ev.a);
    cudaEventDestroy(ev.b);
  }
  for (auto e : h->event_pool) cudaEventDestroy(e);
  if (h->ws) cudaFree(h->ws);
  if (h->status) cudaFree(h->status);
  delete h;
}

strata_status strata_moe_set_router(strata_moe *h, const float *W_dev, const float *bias_dev) {
  if (!h || !W_dev) return STRATA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(W_dev) & 15) || (reinterpret_cast<uintptr_t>(bias_dev) & 3))
    return STRATA_ERR_INVALID_ARG;
  h->router_W = W_dev;
  h->router_b = bias_dev;
  return STRATA_OK;
}

strata_status strata_moe_set_routing(strata_moe *h, int mode, const float *corr_dev,
                                     float routed_scale) {
  if (!h || (mode != STRATA_ROUTE_SOFTMAX && mode != STRATA_ROUTE_SIGMOID))
    return STRATA_ERR_INVALID_ARG;
  if (!(routed_scale > 0.0f) || !(routed_scale < 3.0e38f)) return STRATA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(corr_dev) & 3) return STRATA_ERR_INVALID_ARG;
  if (mode == STRATA_ROUTE_SOFTMAX && (corr_dev || routed_scale != 1.0f))
    return STRATA_ERR_INVALID_ARG;
  h->mode.sigmoid = mode == STRATA_ROUTE_SIGMOID;
  h->mode.corr = corr_dev;
  h->mode.scale = routed_scale;
  return STRATA_OK;
}

strata_status strata_moe_bind_shared(strata_moe *h, int i, const void *device_ptr) {
  if (!h || i < 0 || i >= h->S || !device_ptr) return STRATA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(device_ptr) & 255) return STRATA_ERR_INVALID_ARG;
  h->shared_ptr[i] = device_ptr;
  return STRATA_OK;
}

strata_status strata_moe_bind_slot(strata_moe *h, int slot, int expert_id, const void *device_ptr) {
  if (!h || slot < 0 || slot >= h->n_slots) return STRATA_ERR_INVALID_ARG;
  if (expert_id < -1 || expert_id >= h->E) return STRATA_ERR_INVALID_ARG;
  if (expert_id == -1) {
    const int old = h->slot_expert[slot];
    if (old >= 0) h->expert_slot[old] = -1;
    h->slot_expert[slot] = -1;
    h->slot_ptr[slot] = nullptr;
    return STRATA_OK;
  }
  if (!device_ptr || (reinterpret_cast<uintptr_t>(device_ptr) & 255)) return STRATA_ERR_INVALID_ARG;
  const int cur = h->expert_slot[expert_id];
  if (cur >= 0 && cur != slot) return STRATA_ERR_SLOT_CONFLICT;
  const int old = h->slot_expert[slot];
  if (old >= 0) h->expert_slot[old] = -1;
  h->slot_expert[slot] = expert_id;
  h->slot_ptr[slot] = device_ptr;
  h->expert_slot[expert_id] = slot;
  return STRATA_OK;
}

}  // extern "C"

void strata_handle_shape(const strata_moe *h, int *hidden, int *inter, int *n_experts,
                         int *n_slots, int *device) {
  *hidden = h->H;
  *inter = h->I;
  *n_experts = h->E;
  *n_slots = h->n_slots;
  *device = h->device;
}

int strata_handle_top_k(const strata_moe *h) { return h->k; }

size_t strata_handle_blob_bytes(const strata_moe *h) { return h->layout.total; }

strata_status strata_layer_route_all(strata_moe *h, const void *x, int T, cudaStream_t stream,
                                     const int32_t **idx, const float **w) {
  if (!h || !x || T <= 0 || !h->router_W) return STRATA_ERR_INVALID_ARG;
  for (int i = 0; i < h->S; ++i)
    if (!h->shared_ptr[i]) return STRATA_ERR_INVALID_ARG;
  // the chunks take the tensor-core path, whose gathered activations exist
  // only in a workspace for more than kSmallT tokens
  strata_status st = grow_workspace(h, std::max(T, kSmallT + 1));
  if (st == STRATA_OK) st = run_router(h, x, T, h->logits, h->idx, h->w, stream);
  *idx = h->idx;
  *w = h->w;
  return st;
}

strata_status strata_layer_chunk_prepare(strata_moe *h, const void *x, int Tc, const int32_t *idx,
                                         cudaStream_t stream) {
  strata_status st = run_prepare(h, x, Tc, idx, stream);
  if (st == STRATA_OK) st = run_gather(h, Tc, stream);
  return st;
}

strata_status strata_layer_chunk_pass(strata_moe *h, int Tc, const unsigned char *in_pass,
                                      bool shared, cudaStream_t stream) {
  ExpertTable t = make_table(h);
  for (int e = 0; e < h->E; ++e)
    if (!in_pass[e]) t.ptr[e] = nullptr;
  if (!shared)
    for (int i = 0; i < h->S; ++i) t.ptr[h->E + i] = nullptr;
  return run_tc_passes(h, Tc, t, true, stream);
}

strata_status strata_layer_chunk_finish(strata_moe *h, int Tc, const int32_t *idx, const float *w,
                                        void *out, cudaStream_t stream) {
  return run_combine(h, Tc, idx, w, make_table(h), false, out, stream);
}

extern "C" {

int strata_moe_slot_expert(const strata_moe *h, int slot) {
  if (!h || slot < 0 || slot >= h->n_slots) return -2;
  return h->slot_expert[slot];
}

strata_status strata_moe_reserve(strata_moe *h, int max_tokens) {
  if (!h || max_tokens < 0) return STRATA_ERR_INVALID_ARG;
  return grow_workspace(h, max_tokens);
}

strata_status strata_moe_route(strata_moe *h, const void *x_bf16, int n_tokens, float *logits_out,
                               int32_t *idx_out, float *w_out, strata_stream_t stream) {
  strata_status st = check_common(h, x_bf16, n_tokens, stream);
  if (st != STRATA_OK) return st;
  if (!h->router_W) return STRATA_ERR_INVALID_ARG;
  if (n_tokens == 0) return STRATA_OK;
  if (!idx_out || !w_out) return STRATA_ERR_INVALID_ARG;
  st = grow_workspace(h, n_tokens);
  if (st != STRATA_OK) return st;
  return run_router(h, x_bf16, n_tokens, logits_out ? logits_out : h->logits, idx_out, w_out,
                    stream);
}

strata_status strata_moe_forward(strata_moe *h, const void *x_bf16, int n_tokens, void *out_bf16,
                                 strata_stream_t stream) {
  strata_status st = check_common(h, x_bf16, n_tokens, stream);
  if (st != STRATA_OK) return st;
  if (!h->router_W) return STRATA_ERR_INVALID_ARG;
  for (int i = 0; i < h->S; ++i)
    if (!h->shared_ptr[i]) return STRATA_ERR_INVALID_ARG;
  if (n_tokens == 0) return STRATA_OK;
  if (!out_bf16 || (reinterpret_cast<uintptr_t>(out_bf16) & 15)) return STRATA_ERR_INVALID_ARG;
  st = grow_workspace(h, n_tokens);
  if (st != STRATA_OK) return st;
  if (n_tokens <= kSmallT) return run_fused(h, x_bf16, n_tokens, nullptr, nullptr, out_bf16, stream);
  st = run_router(h, x_bf16, n_tokens, h->logits, h->idx, h->w, stream);
  if (st != STRATA_OK) return st;
  return run_experts(h, x_bf16, n_tokens, h->idx, h->w, out_bf16, stream);
}

strata_status strata_moe_forward_routed(strata_moe *h, const void *x_bf16, int n_tokens,
                                        const int32_t *idx, const float *w, void *out_bf16,
                                        strata_stream_t stream) {
  strata_status st = check_common(h, x_bf16, n_tokens, stream);
  if (st != STRATA_OK) return st;
  for (int i = 0; i < h->S; ++i)
    if (!h->shared_ptr[i]) return STRATA_ERR_INVALID_ARG;
  if (n_tokens == 0) return STRATA_OK;
  if (!idx || !w || !out_bf16 || (reinterpret_cast<uintptr_t>(out_bf16) & 15))
    return STRATA_ERR_INVALID_ARG;
  st = grow_workspace(h, n_tokens);
  if (st != STRATA_OK) return st;
  if (n_tokens <= kSmallT) return run_fused(h, x_bf16, n_tokens, idx, w, out_bf16, stream);
  return run_experts(h, x_bf16, n_tokens, idx, w, out_bf16, stream);
}

strata_status strata_moe_get_status(strata_moe *h, strata_stream_t stream) {
  if (!h) return STRATA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return STRATA_ERR_CUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return STRATA_ERR_CUDA;
  if (cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return STRATA_ERR_CUDA;
  h->last_bits = bits;
  if ((bits & STATUS_TIMEOUT) && h->counters &&
      cudaMemset(h->counters, 0, h->counters_bytes) != cudaSuccess)
    return STRATA_ERR_CUDA;
  if (bits & (STATUS_BAD_ROUTING | STATUS_TIMEOUT | STATUS_BOUNDS)) return STRATA_ERR_DEVICE_STATUS;
  if (bits & STATUS_RANGE) return STRATA_ERR_RANGE;
  if (bits & STATUS_NOT_BOUND) return STRATA_ERR_NOT_BOUND;
  return STRATA_OK;
}

int strata_moe_last_device_bits(const strata_moe *h) { return h ? h->last_bits : 0; }

strata_status strata_moe_set_wait_limit(strata_moe *h, unsigned long long ns) {
  if (!h) return STRATA_ERR_INVALID_ARG;
  h->wait_ns = ns;
  return STRATA_OK;
}

strata_status strata_moe_profile(strata_moe *h, int enable) {
  if (!h) return STRATA_ERR_INVALID_ARG;
  h->profiling = enable != 0;
  return STRATA_OK;
}

strata_status strata_moe_profile_read(strata_moe *h, int n_phases, int *launches, double *ms) {
  if (!h || n_phases < 0 || n_phases > kPhases) return STRATA_ERR_INVALID_ARG;
  for (auto &ev : h->events) {
    float t = 0.f;
    if (cudaEventSynchronize(ev.b) != cudaSuccess) return STRATA_ERR_CUDA;
    if (cudaEventElapsedTime(&t, ev.a, ev.b) != cudaSuccess) return STRATA_ERR_CUDA;
    h->prof_launches[ev.phase] += 1;
    h->prof_ms[ev.phase] += t;
    h->event_pool.push_back(ev.a);
    h->event_pool.push_back(ev.b);
  }
  h->events.clear();
  for (int i = 0; i < n_phases; ++i) {
    if (launches) launches[i] = h->prof_launches[i];
    if (ms) ms[i] = h->prof_ms[i];
  }
  for (int i = 0; i < kPhases; ++i) {
    h->prof_launches[i] = 0;
    h->prof_ms[i] = 0.0;
  }
  return STRATA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// strata_moe_forward_noalloc: the small-batch forward with its workspace in a
// fixed device array of this file instead of the handle's growable
// allocation.  It is for callers that may not allocate device memory at the
// time of the call -- code running under a memory manager that owns the
// whole device (every byte of HBM carved into pools at start-up, where a
// cudaMalloc would fail or fragment them), or latency-bound decode loops that
// cannot take the device-wide synchronisation cudaMalloc and cudaFree may
// imply.  The array is shared by every handle on a device and keeps what the
// last call left in it.

static __device__ __align__(256) unsigned char noalloc_scratch[STRATA_NOALLOC_SCRATCH_BYTES];
static_assert(STRATA_NOALLOC_MAX_TOKENS == kSmallT, "the no-allocation forward covers the small-batch path only");

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex noalloc_mutex;
void *noalloc_base[kNoAllocMaxDevices];  // device address of the array, per device

// Device address of the array on `device`, which must be the current device.
// The first call on a device asks the runtime for it (this may load this
// file's device code onto the device); later calls read the cached pointer.
strata_status noalloc_scratch_on(int device, unsigned char **out) {
  if (device < 0 || device >= kNoAllocMaxDevices) return STRATA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(noalloc_mutex);
  if (!noalloc_base[device]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return STRATA_ERR_CUDA;
    }
    noalloc_base[device] = p;
  }
  *out = static_cast<unsigned char *>(noalloc_base[device]);
  return STRATA_OK;
}

// Byte offsets in the array for T tokens: the regions of the small-batch
// workspace (the counters are the only ones that must be zero when a call
// starts).
struct NoAllocLayout {
  size_t logits, idx, w, meta, ptok, pj, inv, x16, h16, y, rpart, counters, partial, total;
};

NoAllocLayout noalloc_layout(const strata_moe *h, int T) {
  const size_t P = (size_t)T * (h->k + h->S);
  const int nid = h->E + h->S;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  NoAllocLayout L;
  L.logits = take(sizeof(float) * T * h->E);
  L.idx = take(sizeof(int32_t) * T * h->k);
  L.w = take(sizeof(float) * T * h->k);
  L.meta = take(sizeof(int) * (3 * nid + 2));
  L.ptok = take(sizeof(int) * P);
  L.pj = take(sizeof(int) * P);
  L.inv = take(sizeof(int) * P);
  L.x16 = take(sizeof(__half) * T * h->H);
  L.h16 = take(sizeof(__half) * P * h->I);
  L.y = take(sizeof(float) * P * h->H);
  L.rpart = take(sizeof(double) * std::max(h->E, h->num_sms) * (size_t)T);
  L.counters = take(fused_counter_bytes(h));
  L.partial = take(fused_partial_bytes(h));
  L.total = off;
  return L;
}

// For the lifetime of the object the handle's workspace pointers name regions
// of the array; the handle's own come back when it goes out of scope (kernel
// arguments are copied at launch, so enqueued work keeps the array's
// addresses).  Per-kernel timing is off meanwhile: recording it creates
// events and grows a host list.
class NoAllocWorkspace {
 public:
  NoAllocWorkspace(strata_moe *h, unsigned char *base, const NoAllocLayout &L)
      : h_(h), logits_(h->logits), idx_(h->idx), w_(h->w), meta_(h->meta), rt_(h->rt),
        x16_(h->x16), h16_(h->h16), y_(h->y), xp_(h->xp),
        rpart_(h->rpart), partial_(h->partial), counters_(h->counters),
        profiling_(h->profiling) {
    const int nid = h->E + h->S;
    h->logits = reinterpret_cast<float *>(base + L.logits);
    h->idx = reinterpret_cast<int32_t *>(base + L.idx);
    h->w = reinterpret_cast<float *>(base + L.w);
    h->meta = reinterpret_cast<int *>(base + L.meta);
    h->rt.cnt = h->meta;
    h->rt.off = h->meta + nid;
    h->rt.active = h->meta + 2 * nid + 1;
    h->rt.n_active = h->meta + 3 * nid + 1;
    h->rt.pair_tok = reinterpret_cast<int *>(base + L.ptok);
    h->rt.pair_j = reinterpret_cast<int *>(base + L.pj);
    h->rt.inv = reinterpret_cast<int *>(base + L.inv);
    h->x16 = reinterpret_cast<__half *>(base + L.x16);
    h->h16 = reinterpret_cast<__half *>(base + L.h16);
    h->y = reinterpret_cast<float *>(base + L.y);
    h->xp = nullptr;
    h->counters = reinterpret_cast<int *>(base + L.counters);
    h->rpart = reinterpret_cast<double *>(base + L.rpart);
    h->partial = reinterpret_cast<float *>(base + L.partial);
    h->profiling = false;
  }
  ~NoAllocWorkspace() {
    h_->logits = logits_;
    h_->idx = idx_;
    h_->w = w_;
    h_->meta = meta_;
    h_->rt = rt_;
    h_->x16 = x16_;
    h_->h16 = h16_;
    h_->y = y_;
    h_->xp = xp_;
    h_->rpart = rpart_;
    h_->partial = partial_;
    h_->counters = counters_;
    h_->profiling = profiling_;
  }
  NoAllocWorkspace(const NoAllocWorkspace &) = delete;
  NoAllocWorkspace &operator=(const NoAllocWorkspace &) = delete;

 private:
  strata_moe *h_;
  float *logits_;
  int32_t *idx_;
  float *w_;
  int *meta_;
  Routing rt_;
  __half *x16_, *h16_;
  float *y_;
  __half *xp_;
  double *rpart_;
  float *partial_;
  int *counters_;
  bool profiling_;
};

}  // namespace

extern "C" strata_status strata_moe_forward_noalloc(strata_moe *h, const void *x_bf16,
                                                    int n_tokens, void *out_bf16,
                                                    strata_stream_t stream) {
  strata_status st = check_common(h, x_bf16, n_tokens, stream);
  if (st != STRATA_OK) return st;
  if (!h->router_W) return STRATA_ERR_INVALID_ARG;
  for (int i = 0; i < h->S; ++i)
    if (!h->shared_ptr[i]) return STRATA_ERR_INVALID_ARG;
  if (n_tokens == 0) return STRATA_OK;
  if (!out_bf16 || (reinterpret_cast<uintptr_t>(out_bf16) & 15)) return STRATA_ERR_INVALID_ARG;
  if (n_tokens > STRATA_NOALLOC_MAX_TOKENS) return STRATA_ERR_SCRATCH_LIMIT;
  const NoAllocLayout L = noalloc_layout(h, n_tokens);
  if (L.total > STRATA_NOALLOC_SCRATCH_BYTES) return STRATA_ERR_SCRATCH_LIMIT;
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess) return STRATA_ERR_CUDA;
  if (device != h->device) return STRATA_ERR_INVALID_ARG;
  unsigned char *base = nullptr;
  st = noalloc_scratch_on(device, &base);
  if (st != STRATA_OK) return st;
  // The decode kernel's barrier, cut-item and tile counters must start at
  // zero (a call that timed out may have left them otherwise).  Everything
  // else is written before it is read.
  cudaError_t e = cudaMemsetAsync(base + L.counters, 0, fused_counter_bytes(h), stream);
  if (e != cudaSuccess) return cuda_status(e);
  NoAllocWorkspace ws(h, base, L);
  return run_fused(h, x_bf16, n_tokens, nullptr, nullptr, out_bf16, stream);
}
