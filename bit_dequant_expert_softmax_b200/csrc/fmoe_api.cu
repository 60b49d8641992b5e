// Host side of libfmoe.so: validation, the layer handle, workspace layout and
// kernel launches for the C ABI declared in include/fmoe.h.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/fmoe.h"
#include "fmoe_gdn.cuh"
#include "fmoe_grouped.cuh"
#include "fmoe_umma.cuh"
#include "fmoe_gemv.cuh"
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

// Workspace of the batched path for up to max_tokens tokens per call.
struct BatchLayout {
  size_t err, ticket, ntiles, ntiles_s, tiles, tcost, tiles_s, tcost_s, tiles_all, pair_token, pidx, idx, w, sig,
      lpart, hbuf, obuf, xn, xg, hg, size;
};

int batch_max_tiles(const fmoe_config& c, int T) { return T * c.top_k + (T + kTileTok - 1) / kTileTok; }

// The tcgen05 path takes whole pieces of every row and units of 128 rows.
bool umma_shape_ok(const fmoe_config& c) {
  const int pc = c.bits == 4 ? UGeom<4>::kPC : UGeom<2>::kPC;
  return c.hidden % pc == 0 && c.inter % pc == 0 && c.hidden % kURows == 0;
}

// 16-pair blocks the activation tiles of one call can need: sum over tiles of
// ceil(n / 16) <= pairs / 16 + tiles, with tiles of up to kUTileTok pairs.
size_t umma_max_blocks16(const fmoe_config& c, int T) {
  const size_t routed = (size_t)T * c.top_k, P = routed + (size_t)T;
  const size_t tiles = std::min(routed, (size_t)c.n_experts) + (routed + kUTileTok - 1) / kUTileTok +
                       (size_t)(T + kUTileTok - 1) / kUTileTok;
  return (P + 15) / 16 + tiles;
}

// The tcgen05 kernels are asked for through FMOE_GROUPED_TCGEN05=1.
bool umma_requested() {
  const char* want = std::getenv("FMOE_GROUPED_TCGEN05");
  return want && want[0] == '1';
}

// umma_tiles: room for the tcgen05 kernels' activation tiles (shapes they take only)
BatchLayout batch_layout(const fmoe_config& c, int T, bool umma_tiles) {
  BatchLayout b;
  const size_t nq = (size_t)router_splits(c.hidden);
  const size_t P = (size_t)T * (c.top_k + 1), mt = (size_t)batch_max_tiles(c, T);
  b.err = 0;
  b.ticket = 128;
  b.ntiles = 256;
  b.ntiles_s = 384;
  size_t o = 512;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = al256(o + bytes);
    return at;
  };
  b.tiles = take(mt * sizeof(GTile));
  b.tcost = take((mt + 1) * sizeof(long long));
  b.tiles_s = take(mt * sizeof(GTile));
  b.tcost_s = take((mt + 1) * sizeof(long long));
  b.tiles_all = take(mt * sizeof(GTile));
  b.pair_token = take(P * 4);
  b.pidx = take(P * 4);
  b.idx = take((size_t)T * c.top_k * 4);
  b.w = take((size_t)T * c.top_k * 4);
  b.sig = take((size_t)T * 4);
  b.lpart = take((size_t)T * (c.n_experts + 1) * nq * 8);
  b.hbuf = take(P * c.inter * 4);
  b.obuf = take(P * c.hidden * 4);
  b.xn = take((size_t)T * c.hidden * 2);
  b.xg = b.hg = 0;
  if (umma_tiles && umma_shape_ok(c)) {
    const size_t nb = umma_max_blocks16(c, T);
    b.xg = take(nb * xg_bytes_per16(c.hidden));
    b.hg = take(nb * hg_bytes_per16(c.inter));
  }
  b.size = o;
  return b;
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
  int used_noalloc;  // fmoe_layer_forward_noalloc has run this layer (its errors land in the fixed array)
  // batched path
  void* bws;
  size_t bws_bytes;
  int max_tokens;
  BatchLayout bl;
  int g_router_smem, g_topk_smem, g_gu_smem, g_dn_smem;
  int small;                  // tiles of <= kSmallTok pairs on the CUDA-core kernels
  int s_gu_smem, s_dn_smem;
  // tcgen05 path of the batched matvecs
  int umma;
  int u_gu_slots, u_dn_slots, u_gu_smem, u_dn_smem;
  uint8_t u_maps[4][sizeof(CUtensorMap)];  // gate/up codes, gate/up words, down codes, down words
};

namespace {

template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// The largest dynamic shared memory a kernel can be given (the per-block maximum less
// its static shared memory).
template <typename K>
bool set_smem_max(K kernel) {
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return false;
  return set_smem(kernel, kMaxSmem - static_cast<int>(a.sharedSizeBytes));
}

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
  // staging area, its shared gate/up rows at the end (both in flight together); the
  // shared rows are consumed while top-K starts, so its logits and candidates must
  // not reach them either
  const long long U = (long long)(c.n_experts + c.has_shared) * L->nq;
  const uint32_t rows_touched = (uint32_t)(((U + G - 1) / G + L->nq - 1) / L->nq + 1);
  const int shared_rows = (c.inter + G - 1) / G;
  const uint32_t sc_off = c.has_shared ? ((staging - g.gu_bytes(shared_rows)) & ~127u) : staging;
  const uint64_t p1 = r128((uint32_t)c.hidden * 8u) + (uint64_t)rows_touched * g.router_item();
  const uint32_t p1_items = rows_touched + (c.has_shared ? (uint32_t)g.gu_items(shared_rows) : 0u);
  if (c.has_shared && g.gu_bytes(shared_rows) >= staging) return FMOE_ERR_UNSUPPORTED;
  if (p1 > sc_off || p1_items > (uint32_t)kMaxRoundItems) return FMOE_ERR_UNSUPPORTED;
  const uint32_t ncand = (uint32_t)((c.n_experts + 31) / 32 * c.top_k);
  if ((uint64_t)2 * r128(ncand * 8u) + (uint64_t)ncand * 4u > sc_off) return FMOE_ERR_UNSUPPORTED;
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

// Pointers of the single-token kernel's scratch words inside a workspace laid out as
// `w` (the caller's workspace, or the fixed array of fmoe_layer_forward_noalloc).
void set_workspace_ptrs(Params& p, const WsLayout& w, uint8_t* ws) {
  p.err = reinterpret_cast<uint32_t*>(ws + w.err);
  p.tokens = reinterpret_cast<uint32_t*>(ws + w.tokens);
  p.rflags = reinterpret_cast<uint32_t*>(ws + w.rflags);
  p.hflags = reinterpret_cast<uint32_t*>(ws + w.hflags);
  p.lpart = reinterpret_cast<double*>(ws + w.lpart);
  p.hbuf = reinterpret_cast<float*>(ws + w.hbuf);
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
  if (L->ws) set_workspace_ptrs(p, L->wsl, static_cast<uint8_t*>(L->ws));
  p.staging_bytes = L->staging_bytes;
  p.wait_ns = L->wait_ns;
  p.hold_cta = L->hold_cta;
  p.timeline = reinterpret_cast<unsigned long long*>(L->timeline);
  p.timeline_token = L->timeline_token;
  return p;
}

// Programmatic dependent launch with the cooperative launch: the next layer call is
// launched while this one runs and its blocks start as SMs free up (each waits for the
// previous grid's completion before touching any data).  Dropped for the rest of the
// process if the runtime refuses the combination.
std::atomic<int> g_pdl_ok{1};

fmoe_status launch(const fmoe_layer* L, const Params& p, void* stream, bool allow_pdl = true) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(L->sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L->smem_bytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  auto go = [&]() {
    if (L->cfg.bits == 4)
      return p.norm ? cudaLaunchKernelEx(&cfg, fmoe_layer_kernel<4, true>, p)
                    : cudaLaunchKernelEx(&cfg, fmoe_layer_kernel<4, false>, p);
    return p.norm ? cudaLaunchKernelEx(&cfg, fmoe_layer_kernel<2, true>, p)
                  : cudaLaunchKernelEx(&cfg, fmoe_layer_kernel<2, false>, p);
  };
  cudaError_t e = cudaErrorNotSupported;
  if (allow_pdl && g_pdl_ok.load(std::memory_order_relaxed)) {
    cfg.numAttrs = 2;
    e = go();
    if (e != cudaSuccess) {
      cudaGetLastError();  // clear the launch error and fall back for good
      g_pdl_ok.store(0, std::memory_order_relaxed);
    }
  }
  if (e != cudaSuccess) {
    cfg.numAttrs = 1;
    e = go();
  }
  return e == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// A 3-D byte tensor over one matrix of every expert record: {row bytes, rows,
// experts}, boxes of `box_bytes` x 128 rows (128B-swizzled for the codes).
bool encode_rows(uint8_t (&out)[sizeof(CUtensorMap)], const uint8_t* base, uint64_t row_bytes, uint64_t rows,
                 uint64_t nexp, uint64_t rec_bytes, uint32_t box_bytes, bool swizzle) {
  const EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  CUtensorMap m;
  const cuuint64_t dims[3] = {row_bytes, rows, nexp};
  const cuuint64_t strides[2] = {row_bytes, rec_bytes};
  const cuuint32_t box[3] = {box_bytes, (cuuint32_t)kURows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  if (fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::memcpy(out, &m, sizeof m);
  return true;
}

// Ring slots and shared memory of the tcgen05 matvecs, and their tensor maps.  The
// tcgen05 kernels run when FMOE_GROUPED_TCGEN05=1 asks for them and the shape fits
// and the maps can be encoded; otherwise the layer keeps the mma.sync kernels (the
// faster of the two on the measured workloads).
template <int BITS>
void plan_umma_bits(fmoe_layer* L, size_t room) {
  const fmoe_config& c = L->cfg;
  int sg = 0, sd = 0;
  for (int s = kUMaxSlots; s >= 2 && !sg; --s)
    if (umma_smem_bytes<BITS, false>(s) <= room) sg = s;
  for (int s = kUMaxSlots; s >= 2 && !sd; --s)
    if (umma_smem_bytes<BITS, true>(s) <= room) sd = s;
  if (sg < 2 || sd < 2) return;  // at least double-buffered
  const uint8_t* e = static_cast<const uint8_t*>(L->w.experts);
  const uint64_t nexp = (uint64_t)c.n_experts + c.has_shared, rb = L->rec.size;
  if (!encode_rows(L->u_maps[0], e, L->rec.qh, 2ull * c.inter, nexp, rb, kUCodeBox, true) ||
      !encode_rows(L->u_maps[1], e + L->rec.o_gu_sb, L->rec.sh, 2ull * c.inter, nexp, rb, UGeom<BITS>::kSbBox, false) ||
      !encode_rows(L->u_maps[2], e + L->rec.o_d_q, L->rec.qi, (uint64_t)c.hidden, nexp, rb, kUCodeBox, true) ||
      !encode_rows(L->u_maps[3], e + L->rec.o_d_sb, L->rec.si, (uint64_t)c.hidden, nexp, rb, UGeom<BITS>::kSbBox,
                   false))
    return;
  L->u_gu_slots = sg;
  L->u_dn_slots = sd;
  // more than half of the SM's shared memory: one block per SM, so that a block's
  // tensor-memory allocation never waits for another block of the same kernel
  L->u_gu_smem = std::max((int)umma_smem_bytes<BITS, false>(sg), kMaxSmem / 2 + 1024);
  L->u_dn_smem = std::max((int)umma_smem_bytes<BITS, true>(sd), kMaxSmem / 2 + 1024);
  L->umma = 1;
}

void plan_umma(fmoe_layer* L, size_t room, bool want) {
  L->umma = 0;
  if (!want || !umma_shape_ok(L->cfg)) return;
  if (L->cfg.bits == 4)
    plan_umma_bits<4>(L, room);
  else
    plan_umma_bits<2>(L, room);
}

// Shared-memory plan of the batched kernels for up to T tokens per call.
fmoe_status plan_batched(fmoe_layer* L, int T, bool want_umma) {
  const fmoe_config& c = L->cfg;
  const int G = L->sms;
  const int rows = c.n_experts + c.has_shared;
  // router: the block's router slices (fp32) plus kRouterTok token rows of the column
  // splits it touches (fp32, exact for bf16)
  const int nq = router_splits(c.hidden), hc = c.hidden / nq;
  const size_t rsm = 128 + r128((uint32_t)(((long long)rows * nq + G - 1) / G) * hc * 4u) +
                     (size_t)kRouterTok * router_splits_touched(rows, nq, G) * hc * 4;
  uint32_t tsm = 0;
  topk_smem(c.n_experts, c.top_k, T, c.has_shared, &tsm);
  auto mv_smem = [&](bool down) {
    const MvGeom g = mv_geom(down, c.hidden, c.inter, c.bits);
    return sizeof(GHeader) + (size_t)g.frag_bytes + (size_t)g.sum_bytes + (size_t)kGWarps * kRing * g.piece_bytes;
  };
  const size_t gsm = mv_smem(false), dsm = mv_smem(true);
  // (less a little for the kernels' static shared words)
  const size_t room = (size_t)kMaxSmem - 1024;
  if (rsm > room || tsm > room || gsm > room || dsm > room) return FMOE_ERR_UNSUPPORTED;
  // segments a block's unit range can touch: its share of the total weight over the
  // lightest tile, plus the partial tiles at both ends
  const long long mt = batch_max_tiles(c, T);
  if (mt * tile_weight(kTileTok) / ((long long)G * tile_weight(1)) + 3 > kMaxSeg) return FMOE_ERR_UNSUPPORTED;
  L->g_router_smem = (int)rsm;
  L->g_topk_smem = (int)tsm;
  L->g_gu_smem = (int)gsm;
  L->g_dn_smem = (int)dsm;
  plan_umma(L, room, want_umma);
  // the small tiles' CUDA-core kernels, on request (FMOE_GROUPED_SMALL=1), beside the
  // mma.sync kernels (slower than the mma.sync kernels alone on the measured workloads)
  const uint32_t sg = c.bits == 4 ? small_smem_bytes<4>(false, c.hidden, c.inter) : small_smem_bytes<2>(false, c.hidden, c.inter);
  const uint32_t sd = c.bits == 4 ? small_smem_bytes<4>(true, c.hidden, c.inter) : small_smem_bytes<2>(true, c.hidden, c.inter);
  const char* want_small = std::getenv("FMOE_GROUPED_SMALL");
  L->small = !L->umma && sg <= room && sd <= room && want_small && want_small[0] == '1';
  L->s_gu_smem = (int)sg;
  L->s_dn_smem = (int)sd;
  return FMOE_OK;
}

GParams batch_params(const fmoe_layer* L, int T) {
  GParams p{};
  const fmoe_config& c = L->cfg;
  p.H = c.hidden;
  p.I = c.inter;
  p.E = c.n_experts;
  p.K = c.top_k;
  p.has_shared = c.has_shared;
  p.has_rbias = c.has_router_bias;
  p.nq = L->nq;
  p.T = T;
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
  uint8_t* ws = static_cast<uint8_t*>(L->bws);
  const BatchLayout& b = L->bl;
  p.err = reinterpret_cast<uint32_t*>(ws + b.err);
  p.ticket = reinterpret_cast<uint32_t*>(ws + b.ticket);
  p.ntiles = reinterpret_cast<int*>(ws + b.ntiles);
  p.tiles = reinterpret_cast<GTile*>(ws + b.tiles);
  p.tcost = reinterpret_cast<long long*>(ws + b.tcost);
  p.ntiles_s = reinterpret_cast<int*>(ws + b.ntiles_s);
  p.tiles_s = reinterpret_cast<GTile*>(ws + b.tiles_s);
  p.tcost_s = reinterpret_cast<long long*>(ws + b.tcost_s);
  p.tiles_all = reinterpret_cast<GTile*>(ws + b.tiles_all);
  p.small_tok = L->small ? kSmallTok : 0;
  p.pair_token = reinterpret_cast<int*>(ws + b.pair_token);
  p.pidx = reinterpret_cast<int*>(ws + b.pidx);
  p.idx = reinterpret_cast<int32_t*>(ws + b.idx);
  p.w = reinterpret_cast<float*>(ws + b.w);
  p.sig = reinterpret_cast<float*>(ws + b.sig);
  p.lpart = reinterpret_cast<double*>(ws + b.lpart);
  p.hbuf = reinterpret_cast<float*>(ws + b.hbuf);
  p.obuf = reinterpret_cast<float*>(ws + b.obuf);
  p.xg = b.xg ? ws + b.xg : nullptr;
  p.hg = b.hg ? ws + b.hg : nullptr;
  p.tile_tok = L->umma ? kUTileTok : kTileTok;
  p.wait_ns = L->wait_ns;
  return p;
}

// One launch, with programmatic stream serialization when the runtime allows it (the
// kernels wait for their predecessor before reading anything).
template <typename P, typename... A>
cudaError_t launch_pdl(void (*kernel)(A...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, const P& p) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_pdl_ok.load(std::memory_order_relaxed) ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, p);
  if (e != cudaSuccess && cfg.numAttrs == 1) {
    cudaGetLastError();
    g_pdl_ok.store(0, std::memory_order_relaxed);
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kernel, p);
  }
  return e;
}

// router and top-K (+ grouping); then, if `experts`, gate/up, down and combine
fmoe_status launch_batched(const fmoe_layer* L, GParams p, bool experts, cudaStream_t s) {
  const int G = L->sms;
  cudaError_t e = launch_pdl(grouped_router_kernel, dim3(G), dim3(kThreads), L->g_router_smem, s, p);
  if (e == cudaSuccess) e = launch_pdl(grouped_topk_kernel, dim3(p.T), dim3(kThreads), L->g_topk_smem, s, p);
  if (experts && e == cudaSuccess && L->umma) {
    const bool b4 = L->cfg.bits == 4;
    e = launch_pdl(b4 ? grouped_stage_x_kernel<4> : grouped_stage_x_kernel<2>, dim3(G), dim3(256), 0, s, p);
    UParams up;
    up.p = p;
    if (e == cudaSuccess) {
      std::memcpy(&up.tm_q, L->u_maps[0], sizeof(CUtensorMap));
      std::memcpy(&up.tm_sb, L->u_maps[1], sizeof(CUtensorMap));
      up.slots = L->u_gu_slots;
      e = launch_pdl(b4 ? grouped_umma_kernel<4, false> : grouped_umma_kernel<2, false>, dim3(G), dim3(kUThreads),
                     L->u_gu_smem, s, up);
    }
    if (e == cudaSuccess) {
      std::memcpy(&up.tm_q, L->u_maps[2], sizeof(CUtensorMap));
      std::memcpy(&up.tm_sb, L->u_maps[3], sizeof(CUtensorMap));
      up.slots = L->u_dn_slots;
      e = launch_pdl(b4 ? grouped_umma_kernel<4, true> : grouped_umma_kernel<2, true>, dim3(G), dim3(kUThreads),
                     L->u_dn_smem, s, up);
    }
  } else {
    const bool b4 = L->cfg.bits == 4;
    if (experts && e == cudaSuccess && L->small)
      e = launch_pdl(b4 ? grouped_small_kernel<4, false> : grouped_small_kernel<2, false>, dim3(G), dim3(kGThreads),
                     L->s_gu_smem, s, p);
    if (experts && e == cudaSuccess)
      e = launch_pdl(b4 ? grouped_matvec_kernel<4, false> : grouped_matvec_kernel<2, false>, dim3(G),
                     dim3(kGThreads), L->g_gu_smem, s, p);
    if (experts && e == cudaSuccess && L->small)
      e = launch_pdl(b4 ? grouped_small_kernel<4, true> : grouped_small_kernel<2, true>, dim3(G), dim3(kGThreads),
                     L->s_dn_smem, s, p);
    if (experts && e == cudaSuccess)
      e = launch_pdl(b4 ? grouped_matvec_kernel<4, true> : grouped_matvec_kernel<2, true>, dim3(G),
                     dim3(kGThreads), L->g_dn_smem, s, p);
  }
  if (experts && e == cudaSuccess)
    e = launch_pdl(grouped_combine_kernel, dim3((p.H + 255) / 256, p.T), dim3(256), 0, s, p);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}

fmoe_status batch_ready(const fmoe_layer* L, int T) {
  if (!L) return FMOE_ERR_INVALID_ARG;
  if (!L->bws) return FMOE_ERR_NO_WORKSPACE;
  if (T > L->max_tokens) return FMOE_ERR_INVALID_ARG;
  return FMOE_OK;
}

int rmsnorm_threads(int H) { return H >= 1024 ? 1024 : ((H + 31) / 32) * 32; }

fmoe_status ready(const fmoe_layer* L) {
  if (!L) return FMOE_ERR_INVALID_ARG;
  if (!L->ws) return FMOE_ERR_NO_WORKSPACE;
  return FMOE_OK;
}

// The fixed scratch array of fmoe_layer_forward_noalloc (one per device that loads the
// library) and its device address per device.
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

// Device error bits of the last fmoe_layer_forward_noalloc call on L's device (they live
// in the fixed array's error word, shared by every layer that uses it); cleared with the
// array's control words when set.  No allocation: the copies go to and from host
// variables through the array's cached device address.
fmoe_status noalloc_get_error(const fmoe_layer* L, uint32_t* device_error) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return FMOE_ERR_CUDA;
  if (cur != L->device) return FMOE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const fmoe_status st = noalloc_scratch(L->device, &scratch);
  if (st != FMOE_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return FMOE_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  uint32_t e = 0;
  if (cudaMemcpy(&e, ws + L->wsl.err, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return FMOE_ERR_CUDA;
  *device_error = e;
  if (e == 0) return FMOE_OK;
  if (cudaMemset(ws, 0, L->wsl.lpart) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return FMOE_ERR_CUDA;
  return FMOE_ERR_DEVICE;
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
  if (!set_smem(fmoe_layer_kernel<4, false>, L->smem_bytes) || !set_smem(fmoe_layer_kernel<2, false>, L->smem_bytes) ||
      !set_smem(fmoe_layer_kernel<4, true>, L->smem_bytes) || !set_smem(fmoe_layer_kernel<2, true>, L->smem_bytes)) {
    delete L;
    return FMOE_ERR_CUDA;
  }
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fmoe_layer_kernel<4, false>, kThreads, L->smem_bytes) !=
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

size_t fmoe_batch_workspace_bytes(const fmoe_config* cfg, int max_tokens) {
  if (!config_ok(cfg) || max_tokens < 1 || max_tokens > kMaxBatch) return 0;
  return batch_layout(*cfg, max_tokens, umma_requested()).size;
}

fmoe_status fmoe_layer_set_batch_workspace(fmoe_layer_t L, void* dev_ptr, size_t bytes, int max_tokens) {
  if (!L || !dev_ptr || !aligned(dev_ptr, 256) || max_tokens < 1 || max_tokens > kMaxBatch)
    return FMOE_ERR_INVALID_ARG;
  // the tcgen05 kernels only when asked for and the workspace has their tiles' room
  bool want_umma = umma_requested() && umma_shape_ok(L->cfg);
  BatchLayout bl = batch_layout(L->cfg, max_tokens, want_umma);
  if (want_umma && bytes < bl.size) {
    want_umma = false;
    bl = batch_layout(L->cfg, max_tokens, false);
  }
  if (bytes < bl.size) return FMOE_ERR_NO_WORKSPACE;
  const fmoe_status st = plan_batched(L, max_tokens, want_umma);
  if (st != FMOE_OK) return st;
  // the attribute is an upper bound shared by every layer using these kernels: set it
  // to the device maximum (a layer-sized value would break larger layers' launches)
  if (!set_smem_max(grouped_router_kernel) || !set_smem_max(grouped_topk_kernel) ||
      !set_smem_max(grouped_matvec_kernel<4, false>) || !set_smem_max(grouped_matvec_kernel<2, false>) ||
      !set_smem_max(grouped_matvec_kernel<4, true>) || !set_smem_max(grouped_matvec_kernel<2, true>) ||
      !set_smem_max(grouped_umma_kernel<4, false>) || !set_smem_max(grouped_umma_kernel<2, false>) ||
      !set_smem_max(grouped_umma_kernel<4, true>) || !set_smem_max(grouped_umma_kernel<2, true>) ||
      !set_smem_max(grouped_small_kernel<4, false>) || !set_smem_max(grouped_small_kernel<2, false>) ||
      !set_smem_max(grouped_small_kernel<4, true>) || !set_smem_max(grouped_small_kernel<2, true>))
    return FMOE_ERR_CUDA;
  if (cudaMemset(dev_ptr, 0, bl.size) != cudaSuccess) return FMOE_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return FMOE_ERR_CUDA;
  L->bws = dev_ptr;
  L->bws_bytes = bytes;
  L->max_tokens = max_tokens;
  L->bl = bl;
  return FMOE_OK;
}

int fmoe_layer_batched_kind(fmoe_layer_t L) {
  if (!L || !L->bws) return 0;
  return L->umma ? 2 : (L->small ? 3 : 1);
}

fmoe_status fmoe_route_batched(fmoe_layer_t L, const uint16_t* x, int T, int32_t* idx, float* w, float* shared_sigma,
                               void* stream) {
  if (T < 0) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return L ? FMOE_OK : FMOE_ERR_INVALID_ARG;
  fmoe_status st = batch_ready(L, T);
  if (st != FMOE_OK) return st;
  if (!x || !aligned(x, 16) || !idx || !w) return FMOE_ERR_INVALID_ARG;
  GParams p = batch_params(L, T);
  p.x = x;
  p.idx_out = idx;
  p.w_out = w;
  p.sig_out = shared_sigma;
  return launch_batched(L, p, false, static_cast<cudaStream_t>(stream));
}

fmoe_status fmoe_layer_forward_batched(fmoe_layer_t L, const uint16_t* x, const uint16_t* resid, int T, uint16_t* y,
                                       void* stream) {
  if (T < 0) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return L ? FMOE_OK : FMOE_ERR_INVALID_ARG;
  fmoe_status st = batch_ready(L, T);
  if (st != FMOE_OK) return st;
  if (!x || !resid || !y || !aligned(x, 16) || !aligned(resid, 16) || !aligned(y, 16)) return FMOE_ERR_INVALID_ARG;
  GParams p = batch_params(L, T);
  p.x = x;
  p.resid = resid;
  p.y = y;
  return launch_batched(L, p, true, static_cast<cudaStream_t>(stream));
}

fmoe_status fmoe_block_forward_batched(fmoe_layer_t L, const uint16_t* h, int T, double eps, uint16_t* h_out,
                                       void* stream) {
  if (T < 0 || !(eps >= 0.0)) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return L ? FMOE_OK : FMOE_ERR_INVALID_ARG;
  fmoe_status st = batch_ready(L, T);
  if (st != FMOE_OK) return st;
  if (!h || !h_out || !aligned(h, 16) || !aligned(h_out, 16)) return FMOE_ERR_INVALID_ARG;
  GParams p = batch_params(L, T);
  uint16_t* xn = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(L->bws) + L->bl.xn);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  fmoe_rmsnorm_kernel<<<T, rmsnorm_threads(L->cfg.hidden), 0, s>>>(h, xn, L->cfg.hidden, eps);
  p.x = xn;
  p.resid = h;
  p.y = h_out;
  return launch_batched(L, p, true, s);
}

fmoe_status fmoe_gdn_step(float* state, const float* q, const float* k, const float* v, const float* alpha,
                          const float* beta, float* o, int heads, int dk, int dv, void* stream) {
  if (heads < 0 || dv < 1 || dk < 4 || dk % 4 != 0 || dk > 128 * kGdnMaxChunks) return FMOE_ERR_INVALID_ARG;
  if (heads == 0) return FMOE_OK;
  if (!state || !q || !k || !v || !alpha || !beta || !o) return FMOE_ERR_INVALID_ARG;
  if (!aligned(state, 16) || !aligned(q, 16) || !aligned(k, 16)) return FMOE_ERR_INVALID_ARG;
  // rows per warp: 8 for dk <= 128, 2 for longer rows (the loads of a warp in flight
  // together, 32 float4 registers either way)
  const bool narrow = dk <= 128;
  const int R = narrow ? 8 : 2;
  const long long warps = (long long)heads * ((dv + R - 1) / R);
  const long long blocks = (warps + kGdnWarps - 1) / kGdnWarps;
  if (blocks > 0x7fffffffLL) return FMOE_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kGdnWarps * 32);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_pdl_ok.load(std::memory_order_relaxed) ? 1 : 0;
  auto kernel = narrow ? gdn_step_kernel<1, 8> : gdn_step_kernel<kGdnMaxChunks, 2>;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, state, q, k, v, alpha, beta, o, heads, dk, dv);
  if (e != cudaSuccess && cfg.numAttrs == 1) {
    cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kernel, state, q, k, v, alpha, beta, o, heads, dk, dv);
  }
  if (e != cudaSuccess) return FMOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}

fmoe_status fmoe_rmsnorm(const uint16_t* h, uint16_t* out, int T, int H, double eps, void* stream) {
  if (T < 0 || H <= 0 || !(eps >= 0.0)) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!h || !out) return FMOE_ERR_INVALID_ARG;
  fmoe_rmsnorm_kernel<<<T, rmsnorm_threads(H), 0, static_cast<cudaStream_t>(stream)>>>(h, out, H, eps);
  return cudaGetLastError() == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}

fmoe_status fmoe_layer_get_error(fmoe_layer_t L, uint32_t* device_error) {
  if (!L || !device_error) return FMOE_ERR_INVALID_ARG;
  *device_error = 0;
  if (!L->ws && !L->bws) return L->used_noalloc ? noalloc_get_error(L, device_error) : FMOE_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) return FMOE_ERR_CUDA;
  uint32_t e = 0, eb = 0;
  uint8_t* ws = static_cast<uint8_t*>(L->ws);
  uint8_t* bws = static_cast<uint8_t*>(L->bws);
  if (ws && cudaMemcpy(&e, ws + L->wsl.err, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return FMOE_ERR_CUDA;
  if (bws && cudaMemcpy(&eb, bws + L->bl.err, sizeof(eb), cudaMemcpyDeviceToHost) != cudaSuccess) return FMOE_ERR_CUDA;
  *device_error = e | eb;
  if ((e | eb) == 0) return FMOE_OK;
  // clear the whole workspaces: the error words, the tag base, the grouping ticket
  // and any values an aborted launch left behind
  if (ws && cudaMemset(ws, 0, L->wsl.size) != cudaSuccess) return FMOE_ERR_CUDA;
  if (bws && cudaMemset(bws, 0, L->bl.size) != cudaSuccess) return FMOE_ERR_CUDA;
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

fmoe_status fmoe_stack_forward(fmoe_stack_t S, uint16_t* h, int T, int batch, void* stream) {
  if (!S || T < 0 || batch < 1) return FMOE_ERR_INVALID_ARG;
  if (T == 0) return FMOE_OK;
  if (!h || !aligned(h, 16)) return FMOE_ERR_INVALID_ARG;
  const size_t H = (size_t)S->layers[0]->cfg.hidden;
  if (batch > 1)
    for (fmoe_layer* L : S->layers)
      if (!L->bws || L->max_tokens < batch) return FMOE_ERR_NO_WORKSPACE;
  for (int t0 = 0; t0 < T; t0 += batch) {
    const int nb = T - t0 < batch ? T - t0 : batch;
    uint16_t* ht = h + (size_t)t0 * H;
    for (fmoe_layer* L : S->layers) {
      const fmoe_status st = batch == 1 ? fmoe_block_forward(L, ht, 1, S->eps, ht, stream)
                                        : fmoe_block_forward_batched(L, ht, nb, S->eps, ht, stream);
      if (st != FMOE_OK) return st;
    }
  }
  return FMOE_OK;
}

fmoe_status fmoe_stack_graph_create(fmoe_stack_t S, uint16_t* h, int T, int batch, fmoe_graph_t* out) {
  if (!out) return FMOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!S || T < 1 || batch < 1 || !h || !aligned(h, 16)) return FMOE_ERR_INVALID_ARG;
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
    st = fmoe_stack_forward(S, h, T, batch, cs);
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
  L->used_noalloc = 1;
  // the memset above precedes the launch: no programmatic overlap with it
  return launch(L, p, stream, false);
}

}  // extern "C"
