// Expert streaming from host memory with an HBM expert cache.
//
// Source: "flash-moe-inference", per-layer pipeline ("I/O: parallel pread
// K=4 experts") and the parallel expert loading listing: the routed experts'
// weights live in slower storage, the K experts a token selects are read in
// parallel, and the operating system's page cache keeps the recently read
// ones (LRU).  Here the slower tier is host memory (page-locked for
// asynchronous copies) and the cache is a fixed set of expert slots in HBM,
// least recently used first out.
//
// One step (decode, M tokens): router logits and top-K on the device with
// the layer's own kernels; the selection read back to the host (the one
// synchronisation of the step); every selected expert that is not in a slot
// copied into a slot that the step does not use, taking the least recently
// used; the selection rewritten to slot numbers; the experts, the shared
// expert and the combine run by moeq_expert_ffn on the slot bank.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <new>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "moeq.h"

struct moeq_expert_cache {
  moeq_layer host;          // the caller's layer: routed banks in host memory
  moeq_layer dev;           // the same layer over the slot banks
  int32_t slots = 0;
  int32_t max_m = 0;        // tokens per step the buffers hold
  // slot banks: [slots] experts of gate, up, down (codes, scales, biases)
  void* mem = nullptr;
  size_t mem_bytes = 0;
  // per step: logits [max_m][E], selection and weights [max_m][K], slot
  // selection [max_m][K] (device); the selection and the slot selection on
  // the host (page-locked)
  float* logits = nullptr;
  int32_t* idx = nullptr;
  float* w = nullptr;
  int32_t* slot_idx = nullptr;
  int32_t* h_idx = nullptr;
  int32_t* h_slot = nullptr;
  std::vector<int32_t> slot_expert;   // expert held by each slot (-1: empty)
  std::vector<int32_t> expert_slot;   // slot of each expert (-1: not cached)
  std::vector<uint64_t> last_use;     // step of each slot's last use
  uint64_t step = 0, hits = 0, misses = 0, bytes = 0;
  // the step's experts are copied in parallel ("parallel pread" of the K
  // experts): misses spread over copy streams, joined to the caller's
  // stream by events
  static constexpr int kCopyStreams = 4;
  cudaStream_t cs[kCopyStreams] = {};
  cudaEvent_t ev[kCopyStreams] = {};
};

namespace {

// Bytes of one expert's codes, scales and biases in tensor t.
size_t code_bytes(const moeq_qtensor& t) { return (size_t)t.out_dim * t.in_dim * t.bits / 8; }
size_t sb_entries(const moeq_qtensor& t) { return (size_t)t.out_dim * (t.in_dim / t.group_size); }
size_t entry_bytes(const moeq_qtensor& t) { return t.format == MOEQ_FMT_MXFP4 ? 1 : 2; }

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// Copy expert e of host tensor h into slot s of device tensor d.
cudaError_t copy_expert(const moeq_qtensor& h, const moeq_qtensor& d, int e, int s,
                        cudaStream_t st, uint64_t& bytes) {
  const size_t cb = code_bytes(h), sb = sb_entries(h) * entry_bytes(h);
  cudaError_t r = cudaMemcpyAsync((uint8_t*)d.w + (size_t)s * d.expert_stride_w * 4,
                                  (const uint8_t*)h.w + (size_t)e * h.expert_stride_w * 4, cb,
                                  cudaMemcpyHostToDevice, st);
  if (r != cudaSuccess) return r;
  const size_t eb = entry_bytes(h);
  r = cudaMemcpyAsync((uint8_t*)d.scales + (size_t)s * d.expert_stride_sb * eb,
                      (const uint8_t*)h.scales + (size_t)e * h.expert_stride_sb * eb, sb,
                      cudaMemcpyHostToDevice, st);
  if (r != cudaSuccess) return r;
  bytes += cb + sb;
  if (h.format != MOEQ_FMT_MXFP4) {
    r = cudaMemcpyAsync((uint8_t*)d.biases + (size_t)s * d.expert_stride_sb * 2,
                        (const uint8_t*)h.biases + (size_t)e * h.expert_stride_sb * 2, sb,
                        cudaMemcpyHostToDevice, st);
    if (r != cudaSuccess) return r;
    bytes += sb;
  }
  return cudaSuccess;
}

}  // namespace

#define MOEQ_API extern "C" __attribute__((visibility("default")))

MOEQ_API void moeq_cache_destroy(moeq_expert_cache* c) {
  if (!c) return;
  for (int i = 0; i < moeq_expert_cache::kCopyStreams; ++i) {
    if (c->cs[i]) cudaStreamDestroy(c->cs[i]);
    if (c->ev[i]) cudaEventDestroy(c->ev[i]);
  }
  if (c->mem) cudaFree(c->mem);
  if (c->h_idx) cudaFreeHost(c->h_idx);
  delete c;
}

MOEQ_API moeq_status moeq_cache_create(const moeq_layer* L, int32_t slots, int32_t max_tokens,
                                       moeq_expert_cache** out) {
  if (!out) return MOEQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (!L) return MOEQ_ERR_INVALID_ARG;
  // the layer's shapes, formats and pointers pass the decode checks
  if (moeq_workspace_bytes(L, 1, MOEQ_MODE_DECODE) == 0) return MOEQ_ERR_UNSUPPORTED;
  const int E = L->n_experts, K = L->top_k;
  if (slots < K || slots > E || max_tokens < 1 || max_tokens > 64) return MOEQ_ERR_INVALID_ARG;
  if ((int64_t)max_tokens * K > slots) return MOEQ_ERR_INVALID_ARG;  // a step's experts fit
  moeq_expert_cache* c = new (std::nothrow) moeq_expert_cache;
  if (!c) return MOEQ_ERR_CUDA;
  c->host = *L;
  c->dev = *L;
  c->slots = slots;
  c->max_m = max_tokens;
  // slot banks, then the step buffers, in one device allocation
  const moeq_qtensor* ht[3] = {&L->gate, &L->up, &L->down};
  moeq_qtensor* dt[3] = {&c->dev.gate, &c->dev.up, &c->dev.down};
  size_t off[3][3], total = 0;
  for (int i = 0; i < 3; ++i) {
    const size_t cb = code_bytes(*ht[i]), ne = sb_entries(*ht[i]), eb = entry_bytes(*ht[i]);
    off[i][0] = total;
    total += round256(cb * slots);
    off[i][1] = total;
    total += round256(ne * eb * slots);
    off[i][2] = total;
    if (ht[i]->format != MOEQ_FMT_MXFP4) total += round256(ne * 2 * slots);
  }
  const size_t off_logits = total;
  total += round256((size_t)max_tokens * E * 4);
  const size_t off_idx = total;
  total += round256((size_t)max_tokens * K * 4);
  const size_t off_w = total;
  total += round256((size_t)max_tokens * K * 4);
  const size_t off_slot = total;
  total += round256((size_t)max_tokens * K * 4);
  bool ok = cudaMalloc(&c->mem, total) == cudaSuccess &&
            cudaMallocHost((void**)&c->h_idx, (size_t)2 * max_tokens * K * 4) == cudaSuccess;
  for (int i = 0; ok && i < moeq_expert_cache::kCopyStreams; ++i)
    ok = cudaStreamCreateWithFlags(&c->cs[i], cudaStreamNonBlocking) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->ev[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    moeq_cache_destroy(c);
    return MOEQ_ERR_CUDA;
  }
  c->mem_bytes = total;
  uint8_t* base = (uint8_t*)c->mem;
  for (int i = 0; i < 3; ++i) {
    moeq_qtensor& d = *dt[i];
    d.w = (const uint32_t*)(base + off[i][0]);
    d.scales = (const uint16_t*)(base + off[i][1]);
    d.biases = ht[i]->format == MOEQ_FMT_MXFP4 ? nullptr : (const uint16_t*)(base + off[i][2]);
    d.expert_stride_w = (int64_t)(code_bytes(*ht[i]) / 4);
    d.expert_stride_sb = (int64_t)sb_entries(*ht[i]);
  }
  // the slot bank is a layer of `slots` experts; its router descriptor has
  // one row per slot (moeq_expert_ffn never reads the router)
  c->dev.n_experts = slots;
  c->dev.router.out_dim = slots;
  c->logits = (float*)(base + off_logits);
  c->idx = (int32_t*)(base + off_idx);
  c->w = (float*)(base + off_w);
  c->slot_idx = (int32_t*)(base + off_slot);
  c->h_slot = c->h_idx + (size_t)max_tokens * K;
  c->slot_expert.assign(slots, -1);
  c->expert_slot.assign(E, -1);
  c->last_use.assign(slots, 0);
  *out = c;
  return MOEQ_OK;
}

MOEQ_API size_t moeq_cache_workspace_bytes(const moeq_expert_cache* c, int32_t M) {
  if (!c || M < 1 || M > c->max_m) return 0;
  return moeq_workspace_bytes(&c->dev, M, MOEQ_MODE_DECODE);
}

MOEQ_API moeq_status moeq_cache_forward(moeq_expert_cache* c, const uint16_t* x, int32_t M,
                                        float* y, const float* residual, int32_t* idx_out,
                                        float* w_out, void* ws, size_t ws_bytes, void* stream) {
  if (!c || !x || !y || M < 1 || M > c->max_m) return MOEQ_ERR_INVALID_ARG;
  if (ws_bytes < moeq_workspace_bytes(&c->dev, M, MOEQ_MODE_DECODE) || !ws)
    return MOEQ_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  const moeq_layer& L = c->host;
  const int E = L.n_experts, K = L.top_k, n = M * K;
  // 1. routing on the device (router qmv, softmax / top-K / renormalisation)
  moeq_status s = moeq_qmv(&L.router, 0, x, M, c->logits, stream);
  if (s != MOEQ_OK) return s;
  s = moeq_route_topk(c->logits, M, E, K, L.renorm, L.router_scale, c->idx, c->w, stream);
  if (s != MOEQ_OK) return s;
  // 2. the selection on the host (every earlier use of the slots has ended
  //    once this returns: the stream is in order)
  if (cudaMemcpyAsync(c->h_idx, c->idx, (size_t)n * 4, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return MOEQ_ERR_CUDA;
  // 3. hits keep their slot; a miss takes an empty slot, else the least
  //    recently used slot the step does not use, and its expert is copied in
  //    (misses round-robin over the copy streams; nothing reads the slots
  //    being filled: the stream was synchronised above)
  ++c->step;
  int n_miss = 0;
  for (int i = 0; i < n; ++i) {
    const int e = c->h_idx[i];
    if (e < 0 || e >= E) return MOEQ_ERR_INVALID_ARG;
    int sl = c->expert_slot[e];
    if (sl >= 0) {
      if (c->last_use[sl] != c->step) ++c->hits;
    } else {
      int v = -1;
      for (int q = 0; q < c->slots; ++q) {
        if (c->last_use[q] == c->step) continue;
        if (c->slot_expert[q] < 0) {
          v = q;
          break;
        }
        if (v < 0 || c->last_use[q] < c->last_use[v]) v = q;
      }
      if (v < 0) return MOEQ_ERR_INVALID_ARG;  // cannot happen: M * K <= slots
      if (c->slot_expert[v] >= 0) c->expert_slot[c->slot_expert[v]] = -1;
      c->slot_expert[v] = e;
      c->expert_slot[e] = v;
      ++c->misses;
      const moeq_qtensor* ht[3] = {&L.gate, &L.up, &L.down};
      const moeq_qtensor* dt[3] = {&c->dev.gate, &c->dev.up, &c->dev.down};
      cudaStream_t cst = c->cs[n_miss % moeq_expert_cache::kCopyStreams];
      ++n_miss;
      for (int t = 0; t < 3; ++t)
        if (copy_expert(*ht[t], *dt[t], e, v, cst, c->bytes) != cudaSuccess) return MOEQ_ERR_CUDA;
      sl = v;
    }
    c->last_use[sl] = c->step;
    c->h_slot[i] = sl;
  }
  for (int q = 0; q < moeq_expert_cache::kCopyStreams && q < n_miss; ++q)
    if (cudaEventRecord(c->ev[q], c->cs[q]) != cudaSuccess ||
        cudaStreamWaitEvent(st, c->ev[q], 0) != cudaSuccess)
      return MOEQ_ERR_CUDA;
  // 4. the selection by slot, then experts, shared expert and combine
  if (cudaMemcpyAsync(c->slot_idx, c->h_slot, (size_t)n * 4, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return MOEQ_ERR_CUDA;
  s = moeq_expert_ffn(&c->dev, x, M, c->slot_idx, c->w, residual, y, ws, ws_bytes,
                      MOEQ_MODE_DECODE, stream);
  if (s != MOEQ_OK) return s;
  if (idx_out && cudaMemcpyAsync(idx_out, c->idx, (size_t)n * 4, cudaMemcpyDeviceToDevice, st) !=
                     cudaSuccess)
    return MOEQ_ERR_CUDA;
  if (w_out && cudaMemcpyAsync(w_out, c->w, (size_t)n * 4, cudaMemcpyDeviceToDevice, st) !=
                   cudaSuccess)
    return MOEQ_ERR_CUDA;
  return MOEQ_OK;
}

MOEQ_API moeq_status moeq_cache_stats(const moeq_expert_cache* c, uint64_t* hits,
                                      uint64_t* misses, uint64_t* bytes_copied) {
  if (!c) return MOEQ_ERR_INVALID_ARG;
  if (hits) *hits = c->hits;
  if (misses) *misses = c->misses;
  if (bytes_copied) *bytes_copied = c->bytes;
  return MOEQ_OK;
}
