// Host-memory expert tier (libfmoe.so): an HBM cache of expert records, least recently
// used evicted, in front of records kept in host memory.  Built on the layer entry
// points of fmoe.h: the routing pass of a layer over the full router, and the expert
// pass of a second layer handle whose records are the cache slots.
//
// The Flash-MoE pages stream the selected experts from SSD for every token and found
// that the OS page cache beat their own caches (hotdry.top, "SSD流式加载"); on B200 the
// slow tier is host memory behind the host link, and the cache is explicit, in HBM.
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/fmoe.h"

namespace {

size_t al256(size_t n) { return (n + 255) / 256 * 256; }

struct TierLayout {
  size_t cache, ws_route, ws_cache, idx, w, sig, sidx, size;
};

fmoe_config cache_config(const fmoe_config& c, int slots) {
  fmoe_config k = c;
  k.n_experts = slots;
  k.has_router_bias = 0;  // the bias only enters the routing, which the full layer does
  return k;
}

bool tier_layout(const fmoe_config* cfg, int slots, int max_tokens, TierLayout* t) {
  if (!cfg || slots < 1 || max_tokens < 1) return false;
  const size_t rb = fmoe_record_bytes(cfg->hidden, cfg->inter, cfg->bits);
  if (rb == 0 || slots > cfg->n_experts) return false;
  const fmoe_config kc = cache_config(*cfg, slots);
  const size_t wr = fmoe_workspace_bytes(cfg), wc = fmoe_workspace_bytes(&kc);
  if (wr == 0 || wc == 0) return false;
  const size_t tk = (size_t)max_tokens * cfg->top_k;
  size_t o = 0;
  t->cache = o;
  o = al256(o + (size_t)(slots + cfg->has_shared) * rb);
  t->ws_route = o;
  o = al256(o + wr);
  t->ws_cache = o;
  o = al256(o + wc);
  t->idx = o;
  o = al256(o + tk * 4);
  t->w = o;
  o = al256(o + tk * 4);
  t->sig = o;
  o = al256(o + (size_t)max_tokens * 4);
  t->sidx = o;
  o = al256(o + tk * 4);
  t->size = o;
  return true;
}

}  // namespace

struct fmoe_tier {
  fmoe_config cfg;
  int slots, max_tokens;
  size_t rb;
  const uint8_t* host;     // E routed records in host memory
  uint8_t* buf;            // the caller's device buffer
  TierLayout lay;
  fmoe_layer_t route;      // full layer: routing only
  fmoe_layer_t cached;     // layer over the cache slots: experts only
  std::vector<int> slot_expert;   // expert held by each slot, -1 if free
  std::vector<uint64_t> slot_use; // last use of each slot (a counter)
  std::vector<uint64_t> slot_call;// last call that placed or used the slot
  std::vector<int> expert_slot;   // slot of each expert, -1 if not cached
  std::vector<int32_t> h_idx, h_sidx;
  uint64_t clock, calls, hits, misses, bytes;
};

extern "C" {

size_t fmoe_tier_buffer_bytes(const fmoe_config* cfg, int slots, int max_tokens) {
  TierLayout t;
  return tier_layout(cfg, slots, max_tokens, &t) ? t.size : 0;
}

fmoe_status fmoe_tier_create(const fmoe_config* cfg, const void* host_experts, const void* shared_record,
                             const float* router, const float* router_bias, const float* shared_gate,
                             void* dev_buf, size_t buf_bytes, int slots, int max_tokens, fmoe_tier_t* out) {
  if (!out) return FMOE_ERR_INVALID_ARG;
  *out = nullptr;
  TierLayout lay;
  if (!tier_layout(cfg, slots, max_tokens, &lay) || !host_experts || !dev_buf) return FMOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dev_buf) % 256 != 0) return FMOE_ERR_INVALID_ARG;
  if (buf_bytes < lay.size) return FMOE_ERR_NO_WORKSPACE;
  if (cfg->has_shared && !shared_record) return FMOE_ERR_INVALID_ARG;
  // every expert a call touches must have a slot of its own during the call
  if ((long long)slots < (long long)cfg->top_k * max_tokens && slots < cfg->n_experts) return FMOE_ERR_UNSUPPORTED;
  fmoe_tier* T = new (std::nothrow) fmoe_tier();
  if (!T) return FMOE_ERR_INVALID_ARG;
  T->cfg = *cfg;
  T->slots = slots;
  T->max_tokens = max_tokens;
  T->rb = fmoe_record_bytes(cfg->hidden, cfg->inter, cfg->bits);
  T->host = static_cast<const uint8_t*>(host_experts);
  T->buf = static_cast<uint8_t*>(dev_buf);
  T->lay = lay;
  uint8_t* cache = T->buf + lay.cache;
  // the routing layer reads only the router (its records are never touched in a
  // routing pass: the cache stands in for them)
  fmoe_weights wr{cache, router, router_bias, shared_gate};
  fmoe_status st = fmoe_layer_create(cfg, &wr, &T->route);
  if (st == FMOE_OK) st = fmoe_layer_set_workspace(T->route, T->buf + lay.ws_route, lay.ws_cache - lay.ws_route);
  const fmoe_config kc = cache_config(*cfg, slots);
  // the expert pass takes its routing from the caller: the cache layer's router and
  // shared gate are never read (the full layer's are passed to satisfy the checks)
  fmoe_weights wc{cache, router, nullptr, shared_gate};
  if (st == FMOE_OK) st = fmoe_layer_create(&kc, &wc, &T->cached);
  if (st == FMOE_OK) st = fmoe_layer_set_workspace(T->cached, T->buf + lay.ws_cache, lay.idx - lay.ws_cache);
  if (st == FMOE_OK && cfg->has_shared &&
      cudaMemcpy(cache + (size_t)slots * T->rb, shared_record, T->rb, cudaMemcpyDefault) != cudaSuccess)
    st = FMOE_ERR_CUDA;
  if (st != FMOE_OK) {
    fmoe_layer_destroy(T->route);
    fmoe_layer_destroy(T->cached);
    delete T;
    return st;
  }
  T->slot_expert.assign(slots, -1);
  T->slot_use.assign(slots, 0);
  T->slot_call.assign(slots, 0);
  T->expert_slot.assign(cfg->n_experts, -1);
  T->h_idx.resize((size_t)max_tokens * cfg->top_k);
  T->h_sidx.resize((size_t)max_tokens * cfg->top_k);
  T->clock = T->calls = T->hits = T->misses = T->bytes = 0;
  *out = T;
  return FMOE_OK;
}

fmoe_status fmoe_tier_forward(fmoe_tier_t T, const uint16_t* x, const uint16_t* resid, int Tn, uint16_t* y,
                              void* stream) {
  if (!T || Tn < 0 || Tn > T->max_tokens) return FMOE_ERR_INVALID_ARG;
  if (Tn == 0) return FMOE_OK;
  const int K = T->cfg.top_k;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* d_idx = reinterpret_cast<int32_t*>(T->buf + T->lay.idx);
  float* d_w = reinterpret_cast<float*>(T->buf + T->lay.w);
  float* d_sig = reinterpret_cast<float*>(T->buf + T->lay.sig);
  int32_t* d_sidx = reinterpret_cast<int32_t*>(T->buf + T->lay.sidx);
  fmoe_status st = fmoe_route(T->route, x, Tn, d_idx, d_w, T->cfg.has_shared ? d_sig : nullptr, stream);
  if (st != FMOE_OK) return st;
  const size_t nk = (size_t)Tn * K;
  if (cudaMemcpyAsync(T->h_idx.data(), d_idx, nk * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return FMOE_ERR_CUDA;
  const uint64_t call = ++T->calls;
  uint8_t* cache = T->buf + T->lay.cache;
  for (size_t i = 0; i < nk; ++i) {
    const int e = T->h_idx[i];
    if (e < 0 || e >= T->cfg.n_experts) return FMOE_ERR_DEVICE;  // the routing pass failed
    int sl = T->expert_slot[e];
    if (sl >= 0) {
      ++T->hits;
    } else {
      // a free slot, else the least recently used one not needed by this call
      int victim = -1;
      for (int j = 0; j < T->slots && victim < 0; ++j)
        if (T->slot_expert[j] < 0) victim = j;
      if (victim < 0) {
        uint64_t best = UINT64_MAX;
        for (int j = 0; j < T->slots; ++j)
          if (T->slot_call[j] != call && T->slot_use[j] < best) {
            best = T->slot_use[j];
            victim = j;
          }
      }
      if (victim < 0) return FMOE_ERR_UNSUPPORTED;  // more distinct experts than slots
      if (T->slot_expert[victim] >= 0) T->expert_slot[T->slot_expert[victim]] = -1;
      if (cudaMemcpyAsync(cache + (size_t)victim * T->rb, T->host + (size_t)e * T->rb, T->rb, cudaMemcpyHostToDevice,
                          s) != cudaSuccess)
        return FMOE_ERR_CUDA;
      T->slot_expert[victim] = e;
      T->expert_slot[e] = victim;
      sl = victim;
      ++T->misses;
      T->bytes += T->rb;
    }
    T->slot_use[sl] = ++T->clock;
    T->slot_call[sl] = call;
    T->h_sidx[i] = sl;
  }
  if (cudaMemcpyAsync(d_sidx, T->h_sidx.data(), nk * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return FMOE_ERR_CUDA;
  // the remapped routing is copied before h_sidx can change: the next call synchronises
  // the stream before it writes h_sidx again
  return fmoe_expert_forward(T->cached, x, resid, Tn, d_sidx, d_w, T->cfg.has_shared ? d_sig : nullptr, y, stream);
}

fmoe_status fmoe_tier_stats(fmoe_tier_t T, uint64_t* hits, uint64_t* misses, uint64_t* bytes_h2d) {
  if (!T) return FMOE_ERR_INVALID_ARG;
  if (hits) *hits = T->hits;
  if (misses) *misses = T->misses;
  if (bytes_h2d) *bytes_h2d = T->bytes;
  return FMOE_OK;
}

fmoe_status fmoe_tier_get_error(fmoe_tier_t T, uint32_t* device_error) {
  if (!T || !device_error) return FMOE_ERR_INVALID_ARG;
  uint32_t a = 0, b = 0;
  const fmoe_status s1 = fmoe_layer_get_error(T->route, &a);
  const fmoe_status s2 = fmoe_layer_get_error(T->cached, &b);
  *device_error = a | b;
  if (s1 == FMOE_ERR_CUDA || s2 == FMOE_ERR_CUDA) return FMOE_ERR_CUDA;
  return (a | b) ? FMOE_ERR_DEVICE : FMOE_OK;
}

fmoe_status fmoe_tier_destroy(fmoe_tier_t T) {
  if (!T) return FMOE_OK;
  fmoe_layer_destroy(T->route);
  fmoe_layer_destroy(T->cached);
  delete T;
  return FMOE_OK;
}

}  // extern "C"
