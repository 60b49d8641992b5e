// Batched (grouped) routed-expert MoE layer for sm_100a: T decode tokens at once.
//
// The per-token computation is the one of the single-token kernel (same routing,
// same dequantising dot products); what changes is the work order.  The (token,
// slot) pairs are grouped by expert so that every active expert's weights stream
// from HBM once for all of its tokens:
//
//   router   fp64 logits of all T tokens, one pass over the router rows
//   top-K    one block per token (the same rank selection); the last block to
//            finish groups the pairs by expert: a count per expert, offsets, the
//            pairs in (expert, token) order and tiles of <= kTileTok pairs of one
//            expert, each with a work weight
//   gate/up  persistent blocks, each a contiguous, weight-balanced range of
//            (tile, row pair) units: a tile's activations are staged once, every
//            warp streams its own row pairs through a two-slot ring of bulk copies;
//            h = silu(W_g x) * (W_u x) for each pair of the tile
//   down     the same over (tile, output-row block) units, activations = h of the
//            tile's pairs; o = W_d h per pair
//   combine  y = resid + sum_k w_k o_k + sigma o_s per token, in slot order, rounded
//            once to bf16
//
// There are no grid-wide waits: the kernel boundaries order the phases.
#pragma once

#include "fmoe_device.cuh"
#include "fmoe_layer.cuh"
#include "fmoe_topk.cuh"

namespace fmoe {

constexpr int kTileTok = 4;    // pairs whose activations are staged together
constexpr int kRouterTok = 8;  // tokens per pass of the batched router
constexpr int kMaxBatch = 64;  // tokens one batched call may have
constexpr int kMaxSeg = 64;    // tiles one block's unit range may touch
constexpr int kRing = 2;       // bulk copies in flight per warp

struct GTile {
  int expert, p0, n, pad;
};

// Work weight of one unit of a tile of n pairs (relative): the bytes of a unit are
// the same for every tile; the dot-product work grows with n.
__host__ __device__ constexpr int tile_weight(int n) { return 11 + 9 * n > 24 ? 11 + 9 * n : 24; }

struct GParams {
  int H, I, E, K, has_shared, has_rbias, nq, T;
  const uint8_t* experts;
  unsigned long long rec_bytes, o_gu_sb, o_d_q, o_d_sb;
  int qh, qi, sh, si;
  int db;      // output rows per down unit
  int ru;      // bytes of one ring slot
  const float* router;
  const float* rbias;
  const float* sgate;
  const uint16_t* x;      // [T][H] layer input (the normalised block input for blocks)
  const uint16_t* resid;  // [T][H]
  uint16_t* y;            // [T][H]
  int32_t* idx_out;       // optional copies of the routing
  float* w_out;
  float* sig_out;
  uint32_t* err;
  uint32_t* ticket;  // top-K blocks finished (the last one groups)
  int* ntiles;
  GTile* tiles;
  long long* tcost;  // [ntiles + 1] prefix sums of tile weights
  int* pair_token;   // [P] token of each pair
  int* pidx;         // [T][K + 1] pair of (token, slot)
  int32_t* idx;      // [T][K]
  float* w;          // [T][K]
  float* sig;        // [T]
  double* lpart;     // [T][(E + 1) * nq]
  float* hbuf;       // [P][I]
  float* obuf;       // [P][H]
  unsigned long long wait_ns;
};

// ---------------------------------------------------------------- router
// Block b: router rows [r0, r1) (the shared gate vector is row E), staged whole by
// bulk copies; x of kRouterTok tokens at a time as floats.  Unit (row, split q) is a
// warp; every lane accumulates its columns of each token in the single-token
// kernel's order, so the logits are bit-identical to that path.
__global__ void __launch_bounds__(kThreads, 1) grouped_router_kernel(const __grid_constant__ GParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  if (ld_relaxed_u32(p.err) != 0) return;
  const int rows = p.E + (p.has_shared ? 1 : 0);
  const int G = gridDim.x, b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = static_cast<int>(static_cast<long long>(rows) * b / G);
  const int r1 = static_cast<int>(static_cast<long long>(rows) * (b + 1) / G);
  const int nr = r1 - r0;
  const int H = p.H, hc = H / p.nq;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  float* wr = reinterpret_cast<float*>(smem + 128);
  float* xt = wr + static_cast<size_t>(nr) * H;
  __shared__ int fail;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init_fence();
    fail = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0 && nr > 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nr) * H * 4u);
    for (int r = r0; r < r1; ++r)
      bulk_g2s(wr + static_cast<size_t>(r - r0) * H, r < p.E ? p.router + static_cast<size_t>(r) * H : p.sgate,
               static_cast<uint32_t>(H) * 4u, bar);
    if (!mbar_wait_bounded(bar, 0, p.wait_ns, p.err)) fail = 1;
  }
  __syncthreads();
  if (fail) return;
  const int n4 = H / 4;
  for (int tg = 0; tg < p.T; tg += kRouterTok) {
    const int nt = min(kRouterTok, p.T - tg);
    for (int i = threadIdx.x; i < nt * n4; i += kThreads) {
      const int t = i / n4, q = i % n4;
      const uint2 u = reinterpret_cast<const uint2*>(p.x + static_cast<size_t>(tg + t) * H)[q];
      reinterpret_cast<float4*>(xt + static_cast<size_t>(t) * H)[q] =
          make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                      __uint_as_float(u.y & 0xFFFF0000u));
    }
    __syncthreads();
    for (int u = warp; u < nr * p.nq; u += kWarps) {
      const int rl = u / p.nq, qq = u % p.nq;
      const float4* wrow = reinterpret_cast<const float4*>(wr + static_cast<size_t>(rl) * H) + qq * (hc / 4);
      double acc0[kRouterTok], acc1[kRouterTok];
#pragma unroll
      for (int t = 0; t < kRouterTok; ++t) acc0[t] = acc1[t] = 0.0;
      for (int k = lane; k < hc / 4; k += 32) {
        const float4 wv = wrow[k];
#pragma unroll
        for (int t = 0; t < kRouterTok; ++t) {
          if (t < nt) {
            const float4 xv = reinterpret_cast<const float4*>(xt + static_cast<size_t>(t) * H)[qq * (hc / 4) + k];
            acc0[t] = fma(static_cast<double>(wv.x), static_cast<double>(xv.x), acc0[t]);
            acc1[t] = fma(static_cast<double>(wv.y), static_cast<double>(xv.y), acc1[t]);
            acc0[t] = fma(static_cast<double>(wv.z), static_cast<double>(xv.z), acc0[t]);
            acc1[t] = fma(static_cast<double>(wv.w), static_cast<double>(xv.w), acc1[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kRouterTok; ++t) {
        if (t < nt) {
          const double l = warp_sum_d(acc0[t] + acc1[t]);
          if (lane == 0) p.lpart[(static_cast<size_t>(tg + t) * rows + r0 + rl) * p.nq + qq] = l;
        }
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- block scan
// Exclusive prefix sum of one value per thread over the block; *total gets the sum.
// wsum: kWarps + 1 long longs of shared memory.  Every thread calls it.
__device__ __forceinline__ long long block_scan_excl(long long v, long long* wsum, long long* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long s = lane < kWarps ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) wsum[lane] = s;  // inclusive per warp
  }
  __syncthreads();
  const long long base = warp > 0 ? wsum[warp - 1] : 0;
  *total = wsum[kWarps - 1];
  __syncthreads();
  return base + x - v;
}

// ---------------------------------------------------------------- top-K + grouping
struct TopkSmem {
  // byte offsets inside the dynamic shared memory
  uint32_t slog, skey, ckey, cidx, sel, sidx, cnt, tn, wsum, misc;
};

__host__ __device__ inline TopkSmem topk_smem(int E, int K, int T, int has_shared, uint32_t* total) {
  TopkSmem s;
  const int rows = E + has_shared;
  const int ngroups = (E + 31) / 32;
  const int max_tiles = T * K + (T + kTileTok - 1) / kTileTok;
  uint32_t o = 0;
  s.slog = o; o = r128(o + rows * 8u);
  s.skey = o; o = r128(o + E * 8u);
  s.ckey = o; o = r128(o + ngroups * K * 8u);
  s.cidx = o; o = r128(o + ngroups * K * 4u);
  s.sel = o; o = r128(o + (kMaxK + 1) * 4u);
  s.sidx = o; o = r128(o + T * K * 4u);
  s.cnt = o; o = r128(o + E * 4u);
  s.tn = o; o = r128(o + max_tiles * 4u);
  s.wsum = o; o = r128(o + (kWarps + 1) * 8u);
  s.misc = o; o = r128(o + 64u);
  *total = o;
  return s;
}

// The last block: pairs grouped by expert (experts ascending, tokens ascending within
// an expert, then the shared expert's pair of every token), tiles of <= kTileTok
// pairs and the prefix sums of their work weights.
__device__ void build_groups(const GParams& p, uint8_t* smem, const TopkSmem& L) {
  const int E = p.E, K = p.K, T = p.T;
  int* sidx = reinterpret_cast<int*>(smem + L.sidx);
  int* cnt = reinterpret_cast<int*>(smem + L.cnt);
  int* tn = reinterpret_cast<int*>(smem + L.tn);
  long long* wsum = reinterpret_cast<long long*>(smem + L.wsum);
  for (int i = threadIdx.x; i < T * K; i += kThreads) sidx[i] = __ldcg(p.idx + i);
  __syncthreads();
  // per-thread experts: a contiguous run of ceil(E / kThreads)
  const int per = (E + kThreads - 1) / kThreads;
  const int e0 = min(E, static_cast<int>(threadIdx.x) * per), e1 = min(E, e0 + per);
  long long npairs = 0, ntl = 0;
  for (int e = e0; e < e1; ++e) {
    int c = 0;
    for (int i = 0; i < T * K; ++i) c += sidx[i] == e;
    cnt[e] = c;
    npairs += c;
    ntl += (c + kTileTok - 1) / kTileTok;
  }
  long long tot_pairs, tot_tiles;
  const long long poff = block_scan_excl(npairs, wsum, &tot_pairs);
  const long long toff0 = block_scan_excl(ntl, wsum, &tot_tiles);
  {
    long long po = poff, to = toff0;
    for (int e = e0; e < e1; ++e) {
      const int c = cnt[e];
      // the pairs of expert e, tokens ascending
      int j = 0;
      for (int i = 0; i < T * K && j < c; ++i) {
        if (sidx[i] == e) {
          const int t = i / K, k = i % K;
          const int pr = static_cast<int>(po) + j;
          p.pair_token[pr] = t;
          p.pidx[t * (K + 1) + k] = pr;
          ++j;
        }
      }
      for (int i = 0; i * kTileTok < c; ++i) {
        const int n = min(kTileTok, c - i * kTileTok);
        p.tiles[to + i] = GTile{e, static_cast<int>(po) + i * kTileTok, n, 0};
        tn[to + i] = n;
      }
      po += c;
      to += (c + kTileTok - 1) / kTileTok;
    }
  }
  const int routed_tiles = static_cast<int>(tot_tiles);
  const int PR = T * K;  // the shared expert's pairs follow the routed ones
  int ntiles = routed_tiles;
  if (p.has_shared) {
    for (int t = threadIdx.x; t < T; t += kThreads) {
      p.pair_token[PR + t] = t;
      p.pidx[t * (K + 1) + K] = PR + t;
    }
    const int nts = (T + kTileTok - 1) / kTileTok;
    for (int i = threadIdx.x; i < nts; i += kThreads) {
      const int n = min(kTileTok, T - i * kTileTok);
      p.tiles[routed_tiles + i] = GTile{E, PR + i * kTileTok, n, 0};
      tn[routed_tiles + i] = n;
    }
    ntiles += nts;
  }
  __syncthreads();
  // prefix sums of the tiles' work weights (contiguous runs per thread)
  const int tper = (ntiles + kThreads - 1) / kThreads;
  const int i0 = min(ntiles, static_cast<int>(threadIdx.x) * tper), i1 = min(ntiles, i0 + tper);
  long long wsl = 0;
  for (int i = i0; i < i1; ++i) wsl += tile_weight(tn[i]);
  long long wtot;
  long long c = block_scan_excl(wsl, wsum, &wtot);
  for (int i = i0; i < i1; ++i) {
    p.tcost[i] = c;
    c += tile_weight(tn[i]);
  }
  if (threadIdx.x == 0) {
    p.tcost[ntiles] = wtot;
    *p.ntiles = ntiles;
    *p.ticket = 0;  // ready for the next launch (every block of this one has counted)
  }
}

// One block per token: logits from the router partials, the rank top-K, the
// renormalised weights and the shared gate; then the grouping by the last block.
__global__ void __launch_bounds__(kThreads, 1) grouped_topk_kernel(const __grid_constant__ GParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  if (ld_relaxed_u32(p.err) != 0) return;
  uint32_t total;
  const TopkSmem L = topk_smem(p.E, p.K, p.T, p.has_shared, &total);
  const int t = blockIdx.x;
  const int rows = p.E + (p.has_shared ? 1 : 0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double* slog = reinterpret_cast<double*>(smem + L.slog);
  unsigned long long* skey = reinterpret_cast<unsigned long long*>(smem + L.skey);
  unsigned long long* ckey = reinterpret_cast<unsigned long long*>(smem + L.ckey);
  int* cidx = reinterpret_cast<int*>(smem + L.cidx);
  int* sel = reinterpret_cast<int*>(smem + L.sel);
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  const double* lp = p.lpart + static_cast<size_t>(t) * rows * p.nq;
  for (int e = threadIdx.x; e < rows; e += kThreads) {
    double l = router_logit(lp + static_cast<size_t>(e) * p.nq, p.nq);
    if (e < p.E && p.has_rbias) l += static_cast<double>(__ldg(p.rbias + e));
    slog[e] = l;
    if (e < p.E) skey[e] = dkey(l);
  }
  __syncthreads();
  rank_topk<kThreads>(skey, ckey, cidx, p.E, p.K, sel);
  if (warp == 0) {
    const double wk = topk_weight(slog, sel, p.K, lane);
    if (lane < p.K) {
      const size_t o = static_cast<size_t>(t) * p.K + lane;
      p.idx[o] = sel[lane];
      p.w[o] = static_cast<float>(wk);
      if (p.idx_out) {
        p.idx_out[o] = sel[lane];
        p.w_out[o] = static_cast<float>(wk);
      }
    }
    if (lane == 0) {
      const float sg = p.has_shared ? static_cast<float>(1.0 / (1.0 + exp(-slog[p.E]))) : 0.0f;
      p.sig[t] = sg;
      if (p.sig_out) p.sig_out[t] = sg;
    }
  }
  // the last block to finish groups the pairs of all tokens
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) misc[0] = atomicAdd(p.ticket, 1u) == static_cast<uint32_t>(p.T - 1);
  __syncthreads();
  if (!misc[0]) return;
  __threadfence();
  build_groups(p, smem, L);
}

// ---------------------------------------------------------------- grouped matvecs
// Units of a phase: unit (tile i, row block r) of R row blocks per tile carries the
// tile's work weight; block b takes the units whose position falls in its equal share
// [b, b+1) * total / G of the weighted sequence.
struct alignas(128) GHeader {
  uint64_t bars[kWarps][kRing];
  int seg_tile[kMaxSeg];
  int seg_ra[kMaxSeg];
  int seg_rb[kMaxSeg];
  int nseg;
  int first;
  int abort_flag;
  int tok[kTileTok];
};

template <int BITS, bool DOWN>
struct GroupedKernel {
  using C = Chunk<BITS>;
  const GParams& p;
  GHeader* hdr;
  float* xs;    // [kTileTok][xstride] pre-scaled interleaved activations
  float* xsum;  // [kTileTok][nch] chunk sums
  uint8_t* ring;
  int ncol;     // columns of a row: H (gate/up) or I (down)
  int nch;      // chunks of a row
  uint32_t xstride;
  int R;        // row blocks per tile
  int warp, lane;

  __device__ GroupedKernel(const GParams& pp, uint8_t* smem) : p(pp) {
    warp = threadIdx.x >> 5;
    lane = threadIdx.x & 31;
    ncol = DOWN ? p.I : p.H;
    nch = ncol / C::kCols;
    xstride = static_cast<uint32_t>((nch + 31) / 32) * 32u * C::kCols;
    R = DOWN ? (p.H + p.db - 1) / p.db : p.I;
    hdr = reinterpret_cast<GHeader*>(smem);
    xs = reinterpret_cast<float*>(smem + sizeof(GHeader));
    xsum = xs + kTileTok * xstride;
    ring = smem + sizeof(GHeader) + r128(static_cast<uint32_t>(kTileTok) * (xstride + nch) * 4u);
  }

  // ---- the block's segments: (tile, [ra, rb)) in tile order
  __device__ void plan_segments() {
    const int nt = __ldcg(p.ntiles);
    const long long Ctot = __ldcg(p.tcost + nt);
    const int G = gridDim.x, b = blockIdx.x;
    const long long X0 = Ctot * R * b / G, X1 = Ctot * R * (b + 1) / G;
    if (threadIdx.x == 0) {
      hdr->nseg = 0;
      hdr->first = 0;
      hdr->abort_flag = 0;
    }
    __syncthreads();
    // rows of tile i at positions tcost[i]*R + r*w_i, r in [0, R)
    auto range = [&](int i, int& ra, int& rb) {
      const long long c0 = __ldcg(p.tcost + i) * R;
      const long long wi = __ldcg(p.tcost + i + 1) - __ldcg(p.tcost + i);
      ra = X0 <= c0 ? 0 : static_cast<int>(min(static_cast<long long>(R), (X0 - c0 + wi - 1) / wi));
      rb = X1 <= c0 ? 0 : static_cast<int>(min(static_cast<long long>(R), (X1 - c0 + wi - 1) / wi));
    };
    for (int i = threadIdx.x; i < nt; i += kThreads) {
      int ra, rb;
      range(i, ra, rb);
      if (rb > ra) {
        atomicAdd(&hdr->nseg, 1);
        int pa = 0, pb = 0;
        if (i > 0) range(i - 1, pa, pb);
        if (i == 0 || pb <= pa) hdr->first = i;
      }
    }
    __syncthreads();
    const int first = hdr->first, nseg = hdr->nseg;
    if (nseg > kMaxSeg) {  // ruled out by the host plan
      if (threadIdx.x == 0) {
        atomicOr(p.err, FMOE_DEVERR_PLAN);
        hdr->abort_flag = 1;
      }
      __syncthreads();
      return;
    }
    for (int s = threadIdx.x; s < nseg; s += kThreads) {
      int ra, rb;
      range(first + s, ra, rb);
      hdr->seg_tile[s] = first + s;
      hdr->seg_ra[s] = ra;
      hdr->seg_rb[s] = rb;
    }
    __syncthreads();
  }

  // ---- this warp's units in order: segment s, row blocks ra + warp, ra + warp + kWarps, ...
  struct It {
    int s, r;
  };
  __device__ __forceinline__ It norm(It it) const {
    while (it.s < hdr->nseg && it.r >= hdr->seg_rb[it.s]) {
      ++it.s;
      if (it.s < hdr->nseg) it.r = hdr->seg_ra[it.s] + warp;
    }
    return it;
  }
  __device__ __forceinline__ It first_unit() const {
    return hdr->nseg > 0 ? norm(It{0, hdr->seg_ra[0] + warp}) : It{0, 0};
  }
  __device__ __forceinline__ It next_unit(It it) const { return norm(It{it.s, it.r + kWarps}); }
  __device__ __forceinline__ bool valid(It it) const { return it.s < hdr->nseg; }

  __device__ __forceinline__ uint8_t* slot_ptr(int slot) const {
    return ring + (static_cast<uint32_t>(warp) * kRing + slot) * static_cast<uint32_t>(p.ru);
  }

  // bytes [src, src + n) as the 16-byte-aligned cover; returns the lead offset
  __device__ __forceinline__ uint32_t cover(const uint8_t* base, unsigned long long off, uint32_t n,
                                            const uint8_t** src, uint32_t* bytes) const {
    const unsigned long long a = off & ~15ull;
    const unsigned long long e = (off + n + 15ull) & ~15ull;
    *src = base + a;
    *bytes = static_cast<uint32_t>(e - a);
    return static_cast<uint32_t>(off - a);
  }

  // lane 0: bulk copies of unit `it` into ring slot `slot`
  __device__ void issue(It it, int slot) {
    const GTile tl = p.tiles[hdr->seg_tile[it.s]];
    const uint8_t* rec = p.experts + static_cast<unsigned long long>(tl.expert) * p.rec_bytes;
    uint8_t* dst = slot_ptr(slot);
    uint64_t* bar = &hdr->bars[warp][slot];
    const uint8_t* qsrc;
    const uint8_t* ssrc;
    uint32_t qb, sbb;
    if (DOWN) {
      const int j0 = it.r * p.db, n = min(p.H, j0 + p.db) - j0;
      qsrc = rec + p.o_d_q + static_cast<unsigned long long>(j0) * p.qi;
      qb = static_cast<uint32_t>(n) * p.qi;
      cover(rec, p.o_d_sb + static_cast<unsigned long long>(j0) * p.si, static_cast<uint32_t>(n) * p.si, &ssrc, &sbb);
    } else {
      qsrc = rec + static_cast<unsigned long long>(it.r) * 2u * p.qh;
      qb = 2u * p.qh;
      cover(rec, p.o_gu_sb + static_cast<unsigned long long>(it.r) * 2u * p.sh, 2u * p.sh, &ssrc, &sbb);
    }
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, qb + sbb);
    bulk_g2s(dst, qsrc, qb, bar);
    bulk_g2s(dst + r16(qb), ssrc, sbb, bar);
  }

  // ---- activations of a tile: n rows (x rows of the tile's tokens, or h rows of its
  // pairs), every load of the tile issued before any is used; pre-scaled values
  // scattered into the interleaved layout, chunk sums by shuffles over the threads of
  // a chunk (the single-token kernel's staging pattern)
  __device__ void stage_tile(const GTile& tl) {
    constexpr int TPC = C::kCols / 4;
    constexpr int KU = 8;
    const int n4 = ncol / 4;
    const int total = tl.n * n4;
    for (int base = 0; base < total; base += KU * kThreads) {  // block-uniform trip count
      float4 v[KU];
#pragma unroll
      for (int k = 0; k < KU; ++k) {
        const int i = base + static_cast<int>(threadIdx.x) + k * kThreads;
        v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < total) {
          const int j = i / n4, q = i % n4;
          if (DOWN) {
            v[k] = __ldcg(reinterpret_cast<const float4*>(p.hbuf + static_cast<size_t>(tl.p0 + j) * p.I) + q);
          } else {
            const uint2 u = reinterpret_cast<const uint2*>(p.x + static_cast<size_t>(hdr->tok[j]) * p.H)[q];
            v[k] = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                               __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
          }
        }
      }
#pragma unroll
      for (int k = 0; k < KU; ++k) {
        const int i = base + static_cast<int>(threadIdx.x) + k * kThreads;
        float sum = (v[k].x + v[k].y) + (v[k].z + v[k].w);
#pragma unroll
        for (int o = 1; o < TPC; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (i < total) {
          const int j = i / n4, q = i % n4, c0 = 4 * q;
          float* d = xs + static_cast<size_t>(j) * xstride;
          d[C::phys(c0 + 0)] = v[k].x * prescale_factor(C::shift_of(c0 + 0));
          d[C::phys(c0 + 1)] = v[k].y * prescale_factor(C::shift_of(c0 + 1));
          d[C::phys(c0 + 2)] = v[k].z * prescale_factor(C::shift_of(c0 + 2));
          d[C::phys(c0 + 3)] = v[k].w * prescale_factor(C::shift_of(c0 + 3));
          if (q % TPC == 0) xsum[j * nch + q / TPC] = sum;
        }
      }
    }
  }

  // ---- per-lane partial sums of rows qa (and qb) against the n activation rows
  template <bool TWO>
  __device__ __forceinline__ void dot_tile(const uint8_t* qa, const uint32_t* sa, const uint8_t* qb,
                                           const uint32_t* sb, int n, float (&ra)[kTileTok],
                                           float (&rb)[kTileTok]) const {
#pragma unroll
    for (int j = 0; j < kTileTok; ++j) ra[j] = rb[j] = 0.f;
#pragma unroll 1
    for (int m = lane; m < nch; m += 32) {
      const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(qa + 16 * m);
      ulonglong2 bq = make_ulonglong2(0ull, 0ull);
      if (TWO) bq = *reinterpret_cast<const ulonglong2*>(qb + 16 * m);
      const uint32_t swa = sa[C::sb_index(m)];
      const uint32_t swb = TWO ? sb[C::sb_index(m)] : 0u;
#pragma unroll
      for (int j = 0; j < kTileTok; ++j) {
        if (j < n) {
          const float* vs = xs + static_cast<size_t>(j) * xstride;
          const ulonglong2* xv0 = C::f4(vs, m, 0);
          const ulonglong2* xv1 = C::f4(vs, m, C::kF4PerPair);
          unsigned long long a0 = 0ull, a1 = 0ull, b0 = 0ull, b1 = 0ull;
          C::template word_pair2<TWO>(a.x, bq.x, xv0, a0, b0);
          C::template word_pair2<TWO>(a.y, bq.y, xv1, a1, b1);
          const float vm = xsum[j * nch + m];
          ra[j] = fmaf(sb_scale(swa), (pair_sum(a0) + pair_sum(a1)) * kUnscale, ra[j]);
          ra[j] = fmaf(sb_bias(swa), vm, ra[j]);
          if (TWO) {
            rb[j] = fmaf(sb_scale(swb), (pair_sum(b0) + pair_sum(b1)) * kUnscale, rb[j]);
            rb[j] = fmaf(sb_bias(swb), vm, rb[j]);
          }
        }
      }
    }
  }

  // ---- consume unit `it` from ring slot `slot`
  __device__ void consume(It it, int slot) {
    const GTile tl = p.tiles[hdr->seg_tile[it.s]];
    const uint8_t* sl = slot_ptr(slot);
    float ra[kTileTok], rb[kTileTok];
    if (DOWN) {
      const int j0 = it.r * p.db, nrows = min(p.H, j0 + p.db) - j0;
      const uint32_t qb = static_cast<uint32_t>(nrows) * p.qi;
      const uint32_t lead = static_cast<uint32_t>((p.o_d_sb + static_cast<unsigned long long>(j0) * p.si) & 15ull);
      const uint32_t* sbase = reinterpret_cast<const uint32_t*>(sl + r16(qb) + lead);
      for (int i = 0; i < nrows; i += 2) {
        const bool two = i + 1 < nrows;
        if (two)
          dot_tile<true>(sl + static_cast<uint32_t>(i) * p.qi, sbase + i * (p.si / 4),
                         sl + static_cast<uint32_t>(i + 1) * p.qi, sbase + (i + 1) * (p.si / 4), tl.n, ra, rb);
        else
          dot_tile<false>(sl + static_cast<uint32_t>(i) * p.qi, sbase + i * (p.si / 4), nullptr, nullptr, tl.n, ra,
                          rb);
#pragma unroll
        for (int j = 0; j < kTileTok; ++j) {
          if (j < tl.n) {
            const float oa = warp_sum(ra[j]);
            const float ob = two ? warp_sum(rb[j]) : 0.f;
            if (lane == 0) {
              float* o = p.obuf + static_cast<size_t>(tl.p0 + j) * p.H + j0 + i;
              o[0] = oa;
              if (two) o[1] = ob;
            }
          }
        }
      }
    } else {
      const uint32_t lead =
          static_cast<uint32_t>((p.o_gu_sb + static_cast<unsigned long long>(it.r) * 2u * p.sh) & 15ull);
      const uint32_t* sg = reinterpret_cast<const uint32_t*>(sl + r16(2u * p.qh) + lead);
      dot_tile<true>(sl, sg, sl + p.qh, sg + p.sh / 4, tl.n, ra, rb);
#pragma unroll
      for (int j = 0; j < kTileTok; ++j) {
        if (j < tl.n) {
          const float gv = warp_sum(ra[j]);
          const float uv = warp_sum(rb[j]);
          if (lane == 0) p.hbuf[static_cast<size_t>(tl.p0 + j) * p.I + it.r] = (gv / (1.0f + expf(-gv))) * uv;
        }
      }
    }
  }

  __device__ void run() {
    if (threadIdx.x == 0) {
      for (int w = 0; w < kWarps; ++w)
        for (int s = 0; s < kRing; ++s) mbar_init(&hdr->bars[w][s], 1);
      mbar_init_fence();
    }
    __syncthreads();
    plan_segments();
    if (hdr->abort_flag) return;
    // prologue: the warp's first kRing units in flight
    It pre = first_unit();
    uint32_t issued = 0;  // units this warp has requested
    for (int s = 0; s < kRing; ++s) {
      if (valid(pre)) {
        if (lane == 0) issue(pre, s);
        pre = next_unit(pre);
        ++issued;
      }
    }
    uint32_t k = 0;  // units this warp has consumed
    bool ok = true;
    for (int s = 0; s < hdr->nseg; ++s) {
      const GTile tl = p.tiles[hdr->seg_tile[s]];
      __syncthreads();  // the previous tile's activations are no longer read
      if (!DOWN && threadIdx.x < tl.n) hdr->tok[threadIdx.x] = p.pair_token[tl.p0 + threadIdx.x];
      __syncthreads();
      stage_tile(tl);
      __syncthreads();
      if (!ok) continue;
      for (int r = hdr->seg_ra[s] + warp; r < hdr->seg_rb[s]; r += kWarps) {
        const int slot = static_cast<int>(k % kRing);
        const bool arrived = mbar_wait_bounded(&hdr->bars[warp][slot], (k / kRing) & 1u, p.wait_ns, p.err);
        if (!__all_sync(0xffffffffu, arrived)) {
          ok = false;
          break;
        }
        consume(It{s, r}, slot);
        ++k;
        __syncwarp();
        if (valid(pre)) {
          if (lane == 0) issue(pre, slot);
          pre = next_unit(pre);
          ++issued;
        }
      }
    }
    // a warp that stopped early waits for the copies it still has in flight
    if (!ok && lane == 0) {
      for (uint32_t n = k; n < issued; ++n)
        mbar_wait_bounded(&hdr->bars[warp][n % kRing], (n / kRing) & 1u, p.wait_ns, p.err);
    }
  }
};

template <int BITS, bool DOWN>
__global__ void __launch_bounds__(kThreads, 1) grouped_matvec_kernel(const __grid_constant__ GParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  if (ld_relaxed_u32(p.err) != 0) return;
  GroupedKernel<BITS, DOWN> G(p, smem);
  G.run();
}

// y[t][j] = resid[t][j] + sum_k w[t][k] o[pair(t, k)][j] + sigma_t o[pair(t, shared)][j]
__global__ void grouped_combine_kernel(const __grid_constant__ GParams p) {
  if (ld_relaxed_u32(p.err) != 0) return;
  const int t = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= p.H) return;
  const int* pi = p.pidx + static_cast<size_t>(t) * (p.K + 1);
  float pa = 0.f;
  for (int k = 0; k < p.K; ++k)
    pa = fmaf(__ldcg(p.w + static_cast<size_t>(t) * p.K + k), __ldcg(p.obuf + static_cast<size_t>(__ldcg(pi + k)) * p.H + j),
              pa);
  if (p.has_shared) pa = fmaf(__ldcg(p.sig + t), __ldcg(p.obuf + static_cast<size_t>(__ldcg(pi + p.K)) * p.H + j), pa);
  const size_t o = static_cast<size_t>(t) * p.H + j;
  p.y[o] = f32_to_bf16(bf16_to_f32(p.resid[o]) + pa);
}

}  // namespace fmoe
