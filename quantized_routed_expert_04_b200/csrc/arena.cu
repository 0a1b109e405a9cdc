// Expert arena with least-recently-used residency: the paging layer that
// decides which experts occupy the layer's slots and copies missing blobs in
// from a host pool.
//
// What it follows: ro99/strata README, "Residency" (the routed experts of
// each decode step are kept in GPU memory under LRU replacement and copied
// in from pinned host memory);
// "Strata on a Mac", "What you need" (a fixed arena of the most-used experts,
// the rest read in as tokens need them).  The layer's output does not depend
// on which slot holds an expert, so the policy only changes copy traffic,
// never results ("How these numbers are measured", "Fidelity").
//
// Policy (deterministic): the experts a call asks for that are resident are
// hits and become most recent; each miss goes to the lowest empty slot, else
// to the slot whose expert was used least recently (ties: lowest slot) among
// slots that hold nothing the call asks for.  One cudaMemcpyAsync per miss,
// host pool -> slot, on the copy stream; the copy stream first waits for the
// work already queued on the compute stream (an evicted blob may still be in
// use there), and the compute stream then waits for the copies.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <new>
#include <vector>

#include "layer.h"
#include "strata_moe.h"

struct strata_arena {
  strata_moe *layer = nullptr;
  const uint8_t *pool = nullptr;   // host: n_experts blobs, blob_bytes apart
  uint8_t *arena = nullptr;        // device: n_slots blobs, blob_bytes apart
  size_t blob_bytes = 0;
  int E = 0, n_slots = 0;
  std::vector<int> slot_of;        // per expert: slot or -1
  std::vector<int> expert_in;      // per slot: expert or -1
  std::vector<uint64_t> last_use;  // per slot: tick of its last request
  uint64_t tick = 0;
  std::vector<char> wanted;        // scratch, per expert
  std::vector<int> ids;            // scratch: distinct requested ids
  int32_t *idx_host = nullptr;     // pinned: routing of a chunked prefill
  size_t idx_host_count = 0;
  cudaEvent_t ready = nullptr, copy_start = nullptr, copy_end = nullptr;
  bool copies_recorded = false;
};

namespace {

strata_status cuda_err(cudaError_t e) {
  if (e == cudaSuccess) return STRATA_OK;
  cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? STRATA_ERR_OOM : STRATA_ERR_CUDA;
}

}  // namespace

extern "C" {

strata_status strata_arena_create(strata_moe *layer, const void *host_pool, void *arena_dev,
                                  strata_arena **out) {
  if (!out) return STRATA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!layer || !host_pool || !arena_dev || (reinterpret_cast<uintptr_t>(arena_dev) & 255))
    return STRATA_ERR_INVALID_ARG;
  int H, I, E, n_slots, device;
  strata_handle_shape(layer, &H, &I, &E, &n_slots, &device);
  strata_arena *a = new (std::nothrow) strata_arena();
  if (!a) return STRATA_ERR_OOM;
  a->layer = layer;
  a->pool = static_cast<const uint8_t *>(host_pool);
  a->arena = static_cast<uint8_t *>(arena_dev);
  a->blob_bytes = strata_handle_blob_bytes(layer);
  a->E = E;
  a->n_slots = n_slots;
  a->slot_of.assign(E, -1);
  a->expert_in.assign(n_slots, -1);
  a->last_use.assign(n_slots, 0);
  a->wanted.assign(E, 0);
  cudaError_t e = cudaEventCreate(&a->ready, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreate(&a->copy_start);
  if (e == cudaSuccess) e = cudaEventCreate(&a->copy_end);
  // the arena starts empty: unbind every slot of the layer
  for (int s = 0; s < n_slots && e == cudaSuccess; ++s) strata_moe_bind_slot(layer, s, -1, nullptr);
  if (e != cudaSuccess) {
    strata_arena_destroy(a);
    return cuda_err(e);
  }
  *out = a;
  return STRATA_OK;
}

void strata_arena_destroy(strata_arena *a) {
  if (!a) return;
  if (a->idx_host) cudaFreeHost(a->idx_host);
  if (a->ready) cudaEventDestroy(a->ready);
  if (a->copy_start) cudaEventDestroy(a->copy_start);
  if (a->copy_end) cudaEventDestroy(a->copy_end);
  delete a;
}

strata_status strata_arena_ensure(strata_arena *a, const int32_t *ids, int n,
                                  strata_stream_t stream, strata_stream_t copy_stream,
                                  strata_arena_stats *stats) {
  if (!a || n < 0 || (n > 0 && !ids)) return STRATA_ERR_INVALID_ARG;
  // distinct, validated request
  a->ids.clear();
  for (int i = 0; i < n; ++i) {
    const int e = ids[i];
    if (e < 0 || e >= a->E) {
      for (int d : a->ids) a->wanted[d] = 0;
      return STRATA_ERR_INVALID_ARG;
    }
    if (!a->wanted[e]) {
      a->wanted[e] = 1;
      a->ids.push_back(e);
    }
  }
  auto clear_wanted = [&]() {
    for (int d : a->ids) a->wanted[d] = 0;
  };
  if ((int)a->ids.size() > a->n_slots) {
    clear_wanted();
    return STRATA_ERR_TOO_MANY_EXPERTS;
  }
  ++a->tick;
  int hits = 0, misses = 0;
  for (int e : a->ids)
    if (a->slot_of[e] >= 0) {
      a->last_use[a->slot_of[e]] = a->tick;
      ++hits;
    }
  // copies: after the work queued so far on `stream`
  cudaError_t err = cudaEventRecord(a->ready, stream);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(copy_stream, a->ready, 0);
  if (err == cudaSuccess) err = cudaEventRecord(a->copy_start, copy_stream);
  for (int e : a->ids) {
    if (err != cudaSuccess) break;
    if (a->slot_of[e] >= 0) continue;
    // victim: lowest empty slot, else least recently used slot not wanted now
    int victim = -1;
    for (int s = 0; s < a->n_slots; ++s) {
      const int held = a->expert_in[s];
      if (held < 0) {
        victim = s;
        break;
      }
      if (a->wanted[held] && a->last_use[s] == a->tick) continue;
      if (victim < 0 || a->last_use[s] < a->last_use[victim]) victim = s;
    }
    // the victim's bookkeeping changes only once its copy is enqueued: a copy
    // that cannot be enqueued leaves the victim bound to its old expert
    uint8_t *dst = a->arena + (size_t)victim * a->blob_bytes;
    err = cudaMemcpyAsync(dst, a->pool + (size_t)e * a->blob_bytes, a->blob_bytes,
                          cudaMemcpyHostToDevice, copy_stream);
    if (err != cudaSuccess) break;
    const int old = a->expert_in[victim];
    if (old >= 0) a->slot_of[old] = -1;
    const strata_status st = strata_moe_bind_slot(a->layer, victim, e, dst);
    if (st != STRATA_OK) {
      clear_wanted();
      return st;
    }
    a->expert_in[victim] = e;
    a->slot_of[e] = victim;
    a->last_use[victim] = a->tick;
    ++misses;
  }
  if (err == cudaSuccess) err = cudaEventRecord(a->copy_end, copy_stream);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(stream, a->copy_end, 0);
  a->copies_recorded = err == cudaSuccess;
  clear_wanted();
  if (stats) {
    stats->hits = hits;
    stats->misses = misses;
    stats->bytes = (size_t)misses * a->blob_bytes;
  }
  return cuda_err(err);
}

strata_status strata_arena_copy_ms(strata_arena *a, float *ms) {
  if (!a || !ms) return STRATA_ERR_INVALID_ARG;
  *ms = 0.0f;
  if (!a->copies_recorded) return STRATA_OK;
  cudaError_t e = cudaEventSynchronize(a->copy_end);
  if (e == cudaSuccess) e = cudaEventElapsedTime(ms, a->copy_start, a->copy_end);
  return cuda_err(e);
}

int strata_arena_slot_of(const strata_arena *a, int expert_id) {
  if (!a || expert_id < 0 || expert_id >= a->E) return -2;
  return a->slot_of[expert_id];
}

strata_status strata_arena_prefill(strata_arena *a, const void *x_bf16, int n_tokens,
                                   int chunk_tokens, void *out_bf16, strata_stream_t stream,
                                   strata_stream_t copy_stream, strata_prefill_stats *stats) {
  if (!a || n_tokens < 0 || chunk_tokens < 1) return STRATA_ERR_INVALID_ARG;
  if (stats) *stats = strata_prefill_stats{0, 0, 0, 0, 0};
  if (n_tokens == 0) return STRATA_OK;
  if (!x_bf16 || !out_bf16 || (reinterpret_cast<uintptr_t>(x_bf16) & 15) ||
      (reinterpret_cast<uintptr_t>(out_bf16) & 15))
    return STRATA_ERR_INVALID_ARG;
  int H, I, E, n_slots, device;
  strata_handle_shape(a->layer, &H, &I, &E, &n_slots, &device);
  const int k = strata_handle_top_k(a->layer);
  // 1. every token's routing, read back to the host
  const int32_t *idx_dev = nullptr;
  const float *w_dev = nullptr;
  strata_status st = strata_layer_route_all(a->layer, x_bf16, n_tokens, stream, &idx_dev, &w_dev);
  if (st != STRATA_OK) return st;
  const size_t n_idx = (size_t)n_tokens * k;
  if (a->idx_host_count < n_idx) {
    if (a->idx_host) cudaFreeHost(a->idx_host);
    a->idx_host = nullptr;
    a->idx_host_count = 0;
    cudaError_t e = cudaMallocHost(&a->idx_host, n_idx * sizeof(int32_t));
    if (e != cudaSuccess) return cuda_err(e);
    a->idx_host_count = n_idx;
  }
  cudaError_t e = cudaMemcpyAsync(a->idx_host, idx_dev, n_idx * sizeof(int32_t),
                                  cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_err(e);
  // 2. chunks: the chunk's experts, those already resident first, in groups
  // that fit the slots; one arena request and one tensor-core pass per group
  std::vector<unsigned char> in_pass(E, 0);
  std::vector<int> order, group;
  const char *xb = static_cast<const char *>(x_bf16);
  char *ob = static_cast<char *>(out_bf16);
  for (int t0 = 0; t0 < n_tokens; t0 += chunk_tokens) {
    const int Tc = std::min(chunk_tokens, n_tokens - t0);
    const int32_t *ci = a->idx_host + (size_t)t0 * k;
    order.clear();
    for (int q = 0; q < Tc * k; ++q) {
      const int ex = ci[q];
      if (ex < 0 || ex >= E) return STRATA_ERR_DEVICE_STATUS;
      if (!in_pass[ex]) {
        in_pass[ex] = 1;
        order.push_back(ex);
      }
    }
    for (int ex : order) in_pass[ex] = 0;
    std::stable_sort(order.begin(), order.end(), [&](int p, int q) {
      const bool rp = a->slot_of[p] >= 0, rq = a->slot_of[q] >= 0;
      return rp != rq ? rp : p < q;
    });
    st = strata_layer_chunk_prepare(a->layer, xb + (size_t)t0 * H * 2, Tc, idx_dev + (size_t)t0 * k,
                                    stream);
    if (st != STRATA_OK) return st;
    for (size_t g0 = 0; g0 < order.size() || g0 == 0; g0 += n_slots) {
      group.assign(order.begin() + g0, order.begin() + std::min(order.size(), g0 + n_slots));
      strata_arena_stats as{0, 0, 0};
      st = strata_arena_ensure(a, group.data(), (int)group.size(), stream, copy_stream, &as);
      if (st != STRATA_OK) return st;
      for (int ex : group) in_pass[ex] = 1;
      st = strata_layer_chunk_pass(a->layer, Tc, in_pass.data(), g0 == 0, stream);
      for (int ex : group) in_pass[ex] = 0;
      if (st != STRATA_OK) return st;
      if (stats) {
        stats->passes += 1;
        stats->hits += as.hits;
        stats->misses += as.misses;
        stats->bytes += as.bytes;
      }
      if (order.empty()) break;
    }
    st = strata_layer_chunk_finish(a->layer, Tc, idx_dev + (size_t)t0 * k, w_dev + (size_t)t0 * k,
                                   ob + (size_t)t0 * H * 2, stream);
    if (st != STRATA_OK) return st;
    if (stats) stats->chunks += 1;
  }
  return STRATA_OK;
}

}  // extern "C"
