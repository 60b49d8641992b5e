// Host side of libfmoe.so: validation, the layer handle, workspace layout and
// kernel launches for the C ABI declared in include/fmoe.h.
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/fmoe.h"
#include "fmoe_layer.cuh"

using namespace fmoe;

namespace {

constexpr int kGroup = 64;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
constexpr int kMaxSmem = 232448;  // opt-in maximum dynamic shared memory per block on sm_100

size_t al256(size_t n) { return (n + 255) / 256 * 256; }

struct RecordLayout {
  size_t qh, qi, sh, si, o_gu_sb, o_d_q, o_d_sb, size;
};

bool record_layout(int H, int I, int bits, RecordLayout* L) {
  if (H <= 0 || I <= 0 || H % kGroup || I % kGroup || (bits != 4 && bits != 2)) return false;
  L->qh = (size_t)H * bits / 8;
  L->qi = (size_t)I * bits / 8;
  L->sh = (size_t)(H / kGroup) * 4;
  L->si = (size_t)(I / kGroup) * 4;
  L->o_gu_sb = al256((size_t)I * 2 * L->qh);
  L->o_d_q = al256(L->o_gu_sb + (size_t)I * 2 * L->sh);
  L->o_d_sb = al256(L->o_d_q + (size_t)H * L->qi);
  L->size = al256(L->o_d_sb + (size_t)H * L->si);
  return true;
}

struct WsLayout {
  size_t err, tokens, rflags, hflags, lpart, hbuf, size;
};

int router_splits(int H) {
  int nq = 1;
  for (int n = 2; n <= kMaxSplits; n *= 2)
    if (H % (n * 128) == 0 && H / n >= 1024) nq = n;
  return nq;
}

WsLayout ws_layout(const fmoe_config& c) {
  WsLayout w;
  const int nq = router_splits(c.hidden);
  const size_t flag_bytes = (size_t)kMaxGrid * kFlagStride * sizeof(uint32_t);
  w.err = 0;
  w.tokens = 128;
  w.rflags = 256;
  w.hflags = w.rflags + flag_bytes;
  w.lpart = w.hflags + flag_bytes;
  w.hbuf = al256(w.lpart + 2 * (size_t)(c.n_experts + 1) * nq * sizeof(double));
  w.size = al256(w.hbuf + 2 * (size_t)(c.top_k + 1) * c.inter * sizeof(float));
  return w;
}

bool config_ok(const fmoe_config* c) {
  if (!c) return false;
  RecordLayout L;
  if (!record_layout(c->hidden, c->inter, c->bits, &L)) return false;
  if (c->n_experts < 1 || c->top_k < 1 || c->top_k > c->n_experts) return false;
  if ((c->has_shared != 0 && c->has_shared != 1) || (c->has_router_bias != 0 && c->has_router_bias != 1))
    return false;
  return true;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

struct fmoe_layer {
  fmoe_config cfg;
  fmoe_weights w;
  RecordLayout rec;
  int device;
  int sms;
  int nq, rp, db;
  int smem_bytes;
  int staging_bytes;
  void* ws;
  size_t ws_bytes;
  WsLayout wsl;
  uint64_t wait_ns;
  int hold_cta;
  uint64_t* timeline;
  int timeline_token;
};

namespace {

template <int BITS>
int chunk_cols() {
  return Chunk<BITS>::kCols;
}

// Shared-memory plan: the fixed part plus a staging area that must hold, for the
// worst-case block, the router + shared gate/up burst of P1, one gate/up item, and
// the h vectors plus one down item of P3.
fmoe_status plan(fmoe_layer* L) {
  const fmoe_config& c = L->cfg;
  const int cols = c.bits == 4 ? chunk_cols<4>() : chunk_cols<2>();
  const int nslots = c.top_k + c.has_shared;
  if (c.top_k > kMaxK || c.n_experts + c.has_shared > kMaxExperts || L->sms > kMaxGrid) return FMOE_ERR_UNSUPPORTED;
  L->nq = router_splits(c.hidden);
  int rp = 1;
  while (rp < 8 && (size_t)(rp * 2) * 2 * L->rec.qh <= 8192 && c.inter % (rp * 2) == 0) rp *= 2;
  L->rp = rp;
  Geometry g{c.hidden, c.inter, (int)L->rec.qh, (int)L->rec.qi, (int)L->rec.sh, (int)L->rec.si, rp,
             kMaxDownBlock, nslots, cols};
  const uint32_t fixed = g.fixed_bytes(sizeof(SmemHeader));
  if (fixed >= (uint32_t)kMaxSmem) return FMOE_ERR_UNSUPPORTED;
  const uint32_t staging = (uint32_t)kMaxSmem - fixed;
  const int G = L->sms;
  // P1: x in doubles and the router rows a block touches from the start of the
  // staging area, its shared gate/up rows at the end; top-K's logits and
  // candidates must not reach the shared rows either (they are consumed after it)
  const long long U = (long long)(c.n_experts + c.has_shared) * L->nq;
  const uint32_t rows_touched = (uint32_t)(((U + G - 1) / G + L->nq - 1) / L->nq + 1);
  const int shared_rows = (c.inter + G - 1) / G;
  const uint32_t sc_off = c.has_shared ? ((staging - g.gu_bytes(shared_rows)) & ~127u) : staging;
  const uint64_t p1 = r128((uint32_t)c.hidden * 8u) + (uint64_t)rows_touched * g.router_item();
  const uint32_t p1_items = rows_touched + (c.has_shared ? (uint32_t)g.gu_items(shared_rows) : 0u);
  if (c.has_shared && g.gu_bytes(shared_rows) >= staging) return FMOE_ERR_UNSUPPORTED;
  if (p1 > sc_off || p1_items > (uint32_t)kMaxRoundItems) return FMOE_ERR_UNSUPPORTED;
  // top-K: logits, selection keys, per-warp candidates
  if ((uint64_t)r128((uint32_t)(c.n_experts + 1) * 8u) + (uint64_t)((c.n_experts + 15) & ~15) * 8u +
          (uint64_t)((c.n_experts + 31) / 32) * c.top_k * 12u >
      sc_off)
    return FMOE_ERR_UNSUPPORTED;
  // P2: at least one gate/up row pair per round
  if (g.gu_bytes(1) > staging) return FMOE_ERR_UNSUPPORTED;
  // P3: h of every slot plus one down item; shrink the down item until it fits
  int db = kMaxDownBlock;
  while (db > 1 && (uint64_t)g.h_bytes() + g.dn_item(db) > staging) --db;
  if ((uint64_t)g.h_bytes() + g.dn_item(db) > staging) return FMOE_ERR_UNSUPPORTED;
  L->db = db;
  L->staging_bytes = (int)staging;
  L->smem_bytes = kMaxSmem;
  return FMOE_OK;
}

Params base_params(const fmoe_layer* L, int mode, int T) {
  Params p{};
  const fmoe_config& c = L->cfg;
  p.H = c.hidden;
  p.I = c.inter;
  p.E = c.n_experts;
  p.K = c.top_k;
  p.has_shared = c.has_shared;
  p.has_rbias = c.has_router_bias;
  p.nq = L->nq;
  p.rp = L->rp;
  p.db = L->db;
  p.T = T;
  p.mode = mode;
  p.experts = static_cast<const uint8_t*>(L->w.experts);
  p.rec_bytes = L->rec.size;
  p.o_gu_sb = L->rec.o_gu_sb;
  p.o_d_q = L->rec.o_d_q;
  p.o_d_sb = L->rec.o_d_sb;
  p.qh = (int)L->rec.qh;
  p.qi = (int)L->rec.qi;
  p.sh = (int)L->rec.sh;
  p.si = (int)L->rec.si;
  p.router = L->w.router;
  p.rbias = L->w.router_bias;
  p.sgate = L->w.shared_gate;
  uint8_t* ws = static_cast<uint8_t*>(L->ws);
  p.err = reinterpret_cast<uint32_t*>(ws + L->wsl.err);
  p.tokens = reinterpret_cast<uint32_t*>(ws + L->wsl.tokens);
  p.rflags = reinterpret_cast<uint32_t*>(ws + L->wsl.rflags);
  p.hflags = reinterpret_cast<uint32_t*>(ws + L->wsl.hflags);
  p.lpart = reinterpret_cast<double*>(ws + L->wsl.lpart);
  p.hbuf = reinterpret_cast<float*>(ws + L->wsl.hbuf);
  p.staging_bytes = L->staging_bytes;
  p.wait_ns = L->wait_ns;
  p.hold_cta = L->hold_cta;
  p.timeline = reinterpret_cast<unsigned long long*>(L->timeline);
  p.timeline_token = L->timeline_token;
  return p;
}

fmoe_status launch(const fmoe_layer* L, const Params& p, void* stream) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(L->sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L->smem_bytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (L->cfg.bits == 4)
    e = cudaLaunchKernelEx(&cfg, fmoe_layer_kernel<4>, p);
  else
    e = cudaLaunchKernelEx(&cfg, fmoe_layer_kernel<2>, p);
  return e == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}

fmoe_status ready(const fmoe_layer* L) {
  if (!L) return FMOE_ERR_INVALID_ARG;
  if (!L->ws) return FMOE_ERR_NO_WORKSPACE;
  return FMOE_OK;
}

}  // namespace

extern "C" {

size_t fmoe_record_bytes(int hidden, int inter, int bits) {
  RecordLayout L;
  return record_layout(hidden, inter, bits, &L) ? L.size : 0;
}

size_t fmoe_workspace_bytes(const fmoe_config* cfg) {
  if (!config_ok(cfg)) return 0;
  return ws_layout(*cfg).size;
}

fmoe_status fmoe_layer_create(const fmoe_config* cfg, const fmoe_weights* w, fmoe_layer_t* out) {
  if (!out) return FMOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!config_ok(cfg) || !w) return FMOE_ERR_INVALID_ARG;
  if (!w->experts || !aligned(w->experts, 256)) return FMOE_ERR_INVALID_ARG;
  if (!w->router || !aligned(w->router, 16)) return FMOE_ERR_INVALID_ARG;
  if (cfg->has_shared && (!w->shared_gate || !aligned(w->shared_gate, 16))) return FMOE_ERR_INVALID_ARG;
  if (cfg->has_router_bias && !w->router_bias) return FMOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FMOE_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return FMOE_ERR_CUDA;
  if (prop.major < 10 || !prop.cooperativeLaunch) return FMOE_ERR_CUDA;
  fmoe_layer* L = new (std::nothrow) fmoe_layer();
  if (!L) return FMOE_ERR_INVALID_ARG;
  L->cfg = *cfg;
  L->w = *w;
  if (!cfg->has_shared) L->w.shared_gate = nullptr;
  if (!cfg->has_router_bias) L->w.router_bias = nullptr;
  record_layout(cfg->hidden, cfg->inter, cfg->bits, &L->rec);
  L->device = dev;
  L->sms = prop.multiProcessorCount;
  L->wait_ns = kDefaultWaitNs;
  L->hold_cta = -1;
  L->wsl = ws_layout(*cfg);
  fmoe_status st = plan(L);
  if (st != FMOE_OK) {
    delete L;
    return st;
  }
  if (cudaFuncSetAttribute(fmoe_layer_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, L->smem_bytes) !=
          cudaSuccess ||
      cudaFuncSetAttribute(fmoe_layer_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, L->smem_bytes) !=
          cudaSuccess) {
    delete L;
    return FMOE_ERR_CUDA;
  }
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fmoe_layer_kernel<4>, kThreads, L->smem_bytes) !=
          cudaSuccess ||
      nb < 1) {
    delete L;
    return FMOE_ERR_CUDA;
  }
  *out = L;
  return FMOE_OK;
}

fmoe_status fmoe_layer_destroy(fmoe_layer_t layer) {
  delete layer;
  return FMOE_OK;
}

fmoe_status fmoe_layer_set_workspace(fmoe_layer_t L, void* dev_ptr, size_t bytes) {
  if (!L || !dev_ptr || !aligned(dev_ptr, 256)) return FMOE_ERR_INVALID_ARG;
  if (bytes < L->wsl.size) return FMOE_ERR_NO_WORKSPACE;
  if (cudaMemset(dev_ptr, 0, L->wsl.size) != cudaSuccess) return FMOE_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return FMOE_ERR_CUDA;
  L->ws = dev_ptr;
  L->ws_bytes = bytes;
  return FMOE_OK;
}

fmoe_status fmoe_route(fmoe_layer_t L, const uint16_t* x, int T, int32_t* idx, float* w, float* shared_sigma,
                       void* stream) {
  fmoe_status st = ready(L);
  if (st != FMOE_OK) return st;
  if (T < 0) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!x || !aligned(x, 16) || !idx || !w) return FMOE_ERR_INVALID_ARG;
  Params p = base_params(L, MODE_ROUTE, T);
  p.x = x;
  p.idx_out = idx;
  p.w_out = w;
  p.sig_out = L->cfg.has_shared ? shared_sigma : nullptr;
  return launch(L, p, stream);
}

fmoe_status fmoe_expert_forward(fmoe_layer_t L, const uint16_t* x, const uint16_t* resid, int T,
                                const int32_t* idx, const float* w, const float* shared_sigma, uint16_t* y,
                                void* stream) {
  fmoe_status st = ready(L);
  if (st != FMOE_OK) return st;
  if (T < 0) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!x || !resid || !y || !idx || !w || !aligned(x, 16) || !aligned(resid, 16) || !aligned(y, 16))
    return FMOE_ERR_INVALID_ARG;
  if (L->cfg.has_shared && !shared_sigma) return FMOE_ERR_INVALID_ARG;
  if (y == x) return FMOE_ERR_INVALID_ARG;
  Params p = base_params(L, MODE_EXPERTS, T);
  p.x = x;
  p.resid = resid;
  p.y = y;
  p.idx_in = idx;
  p.w_in = w;
  p.sig_in = shared_sigma;
  return launch(L, p, stream);
}

fmoe_status fmoe_layer_forward(fmoe_layer_t L, const uint16_t* x, const uint16_t* resid, int T, uint16_t* y,
                               void* stream) {
  fmoe_status st = ready(L);
  if (st != FMOE_OK) return st;
  if (T < 0) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!x || !resid || !y || !aligned(x, 16) || !aligned(resid, 16) || !aligned(y, 16)) return FMOE_ERR_INVALID_ARG;
  if (y == x && resid != x) return FMOE_ERR_INVALID_ARG;
  if (y == x) return FMOE_ERR_INVALID_ARG;
  Params p = base_params(L, MODE_FULL, T);
  p.x = x;
  p.resid = resid;
  p.y = y;
  return launch(L, p, stream);
}

fmoe_status fmoe_block_forward(fmoe_layer_t L, const uint16_t* h, int T, double eps, uint16_t* h_out, void* stream) {
  fmoe_status st = ready(L);
  if (st != FMOE_OK) return st;
  if (T < 0 || !(eps >= 0.0)) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!h || !h_out || !aligned(h, 16) || !aligned(h_out, 16)) return FMOE_ERR_INVALID_ARG;
  Params p = base_params(L, MODE_FULL, T);
  p.x = h;
  p.resid = h;
  p.y = h_out;
  p.norm = 1;
  p.norm_eps = eps;
  return launch(L, p, stream);
}

fmoe_status fmoe_rmsnorm(const uint16_t* h, uint16_t* out, int T, int H, double eps, void* stream) {
  if (T < 0 || H <= 0 || !(eps >= 0.0)) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!h || !out) return FMOE_ERR_INVALID_ARG;
  const int threads = H >= 1024 ? 1024 : ((H + 31) / 32) * 32;
  fmoe_rmsnorm_kernel<<<T, threads, 0, static_cast<cudaStream_t>(stream)>>>(h, out, H, eps);
  return cudaGetLastError() == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}

fmoe_status fmoe_layer_get_error(fmoe_layer_t L, uint32_t* device_error) {
  if (!L || !device_error) return FMOE_ERR_INVALID_ARG;
  *device_error = 0;
  if (!L->ws) return FMOE_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) return FMOE_ERR_CUDA;
  uint32_t e = 0;
  uint8_t* ws = static_cast<uint8_t*>(L->ws);
  if (cudaMemcpy(&e, ws + L->wsl.err, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return FMOE_ERR_CUDA;
  *device_error = e;
  if (e == 0) return FMOE_OK;
  // clear the whole workspace: the error word, the tag base and any values an
  // aborted launch left behind
  if (cudaMemset(ws, 0, L->wsl.size) != cudaSuccess) return FMOE_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return FMOE_ERR_CUDA;
  return FMOE_ERR_DEVICE;
}

fmoe_status fmoe_layer_set_wait_limit(fmoe_layer_t L, uint64_t nanoseconds) {
  if (!L || nanoseconds == 0) return FMOE_ERR_INVALID_ARG;
  L->wait_ns = nanoseconds;
  return FMOE_OK;
}

fmoe_status fmoe_layer_debug_hold_block(fmoe_layer_t L, int cta) {
  if (!L || cta < -1 || cta >= L->sms) return FMOE_ERR_INVALID_ARG;
  L->hold_cta = cta;
  return FMOE_OK;
}

fmoe_status fmoe_layer_debug_timeline(fmoe_layer_t L, uint64_t* dev_buf, int token) {
  if (!L || token < 0) return FMOE_ERR_INVALID_ARG;
  L->timeline = dev_buf;
  L->timeline_token = token;
  return FMOE_OK;
}

int fmoe_layer_grid_size(fmoe_layer_t L) { return L ? L->sms : 0; }

const char* fmoe_status_string(fmoe_status s) {
  switch (s) {
    case FMOE_OK: return "ok";
    case FMOE_ERR_INVALID_ARG: return "invalid argument";
    case FMOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case FMOE_ERR_CUDA: return "CUDA error";
    case FMOE_ERR_NO_WORKSPACE: return "workspace missing or too small";
    case FMOE_ERR_DEVICE: return "device-side error";
    case FMOE_ERR_SCRATCH_LIMIT:
      return "the layer needs more scratch than fmoe_layer_forward_noalloc's fixed array (FMOE_NOALLOC_SCRATCH_BYTES)";
  }
  return "unknown status";
}

// ---------------------------------------------------------------------------
// Layer stacks and their CUDA graphs.
}  // extern "C"

struct fmoe_stack {
  std::vector<fmoe_layer*> layers;
  double eps;
  int device;
};

struct fmoe_graph {
  cudaGraphExec_t exec;
};

extern "C" {

fmoe_status fmoe_stack_create(const fmoe_layer_t* layers, int n_layers, double eps, fmoe_stack_t* out) {
  if (!out) return FMOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!layers || n_layers < 1 || !(eps >= 0.0)) return FMOE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    if (!layers[l]) return FMOE_ERR_INVALID_ARG;
    if (!layers[l]->ws) return FMOE_ERR_NO_WORKSPACE;
    if (layers[l]->cfg.hidden != layers[0]->cfg.hidden || layers[l]->device != layers[0]->device)
      return FMOE_ERR_INVALID_ARG;
  }
  fmoe_stack* S = new (std::nothrow) fmoe_stack();
  if (!S) return FMOE_ERR_INVALID_ARG;
  S->layers.assign(layers, layers + n_layers);
  S->eps = eps;
  S->device = layers[0]->device;
  *out = S;
  return FMOE_OK;
}

fmoe_status fmoe_stack_destroy(fmoe_stack_t S) {
  delete S;
  return FMOE_OK;
}

fmoe_status fmoe_stack_forward(fmoe_stack_t S, uint16_t* h, int T, void* stream) {
  if (!S || T < 0) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!h || !aligned(h, 16)) return FMOE_ERR_INVALID_ARG;
  const size_t H = (size_t)S->layers[0]->cfg.hidden;
  for (int t = 0; t < T; ++t)
    for (fmoe_layer* L : S->layers) {
      uint16_t* ht = h + (size_t)t * H;
      const fmoe_status st = fmoe_block_forward(L, ht, 1, S->eps, ht, stream);
      if (st != FMOE_OK) return st;
    }
  return FMOE_OK;
}

fmoe_status fmoe_stack_graph_create(fmoe_stack_t S, uint16_t* h, int T, fmoe_graph_t* out) {
  if (!out) return FMOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!S || T < 1 || !h || !aligned(h, 16)) return FMOE_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FMOE_ERR_CUDA;
  if (dev != S->device) return FMOE_ERR_INVALID_ARG;
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return FMOE_ERR_CUDA;
  fmoe_status st = FMOE_OK;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    st = FMOE_ERR_CUDA;
  } else {
    st = fmoe_stack_forward(S, h, T, cs);
    // end the capture whatever happened, so the stream is usable again
    if (cudaStreamEndCapture(cs, &graph) != cudaSuccess && st == FMOE_OK) st = FMOE_ERR_CUDA;
  }
  if (st == FMOE_OK && cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) st = FMOE_ERR_CUDA;
  if (graph) cudaGraphDestroy(graph);
  cudaStreamDestroy(cs);
  if (st != FMOE_OK) {
    if (exec) cudaGraphExecDestroy(exec);
    return st;
  }
  fmoe_graph* G = new (std::nothrow) fmoe_graph();
  if (!G) {
    cudaGraphExecDestroy(exec);
    return FMOE_ERR_INVALID_ARG;
  }
  G->exec = exec;
  *out = G;
  return FMOE_OK;
}

fmoe_status fmoe_graph_launch(fmoe_graph_t G, void* stream) {
  if (!G) return FMOE_ERR_INVALID_ARG;
  return cudaGraphLaunch(G->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}

fmoe_status fmoe_graph_destroy(fmoe_graph_t G) {
  if (!G) return FMOE_OK;
  const cudaError_t e = cudaGraphExecDestroy(G->exec);
  delete G;
  return e == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// fmoe_layer_forward_noalloc: the same fused kernel with its scratch in a fixed
// file-scope device array instead of a caller-provided workspace.
}  // extern "C"

namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[FMOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the array on device `dev` (current); looked up once per device.
// In host code the array's name is only a host-side handle, never a device address.
fmoe_status noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (dev < 0 || dev >= kMaxDevices) return FMOE_ERR_UNSUPPORTED;
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FMOE_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FMOE_OK;
}

void set_workspace_ptrs(Params& p, const WsLayout& w, uint8_t* ws) {
  p.err = reinterpret_cast<uint32_t*>(ws + w.err);
  p.tokens = reinterpret_cast<uint32_t*>(ws + w.tokens);
  p.rflags = reinterpret_cast<uint32_t*>(ws + w.rflags);
  p.hflags = reinterpret_cast<uint32_t*>(ws + w.hflags);
  p.lpart = reinterpret_cast<double*>(ws + w.lpart);
  p.hbuf = reinterpret_cast<float*>(ws + w.hbuf);
}

}  // namespace

extern "C" {

fmoe_status fmoe_layer_forward_noalloc(fmoe_layer_t L, const uint16_t* x, const uint16_t* resid, int T, uint16_t* y,
                                       void* stream) {
  if (!L || T < 0) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!x || !resid || !y || !aligned(x, 16) || !aligned(resid, 16) || !aligned(y, 16) || y == x)
    return FMOE_ERR_INVALID_ARG;
  if (L->wsl.size > (size_t)FMOE_NOALLOC_SCRATCH_BYTES) return FMOE_ERR_SCRATCH_LIMIT;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FMOE_ERR_CUDA;
  if (dev != L->device) return FMOE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  fmoe_status st = noalloc_scratch(dev, &scratch);
  if (st != FMOE_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  // every call starts from a clean error word, tag base and flags (the values the
  // previous call left there would otherwise be mistaken for this call's)
  if (cudaMemsetAsync(ws, 0, L->wsl.lpart, static_cast<cudaStream_t>(stream)) != cudaSuccess) return FMOE_ERR_CUDA;
  Params p = base_params(L, MODE_FULL, T);
  set_workspace_ptrs(p, L->wsl, ws);
  p.x = x;
  p.resid = resid;
  p.y = y;
  return launch(L, p, stream);
}

}  // extern "C"
