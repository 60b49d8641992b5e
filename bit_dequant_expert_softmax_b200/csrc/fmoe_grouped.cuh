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
//            (tile, 8 row pairs) units: a tile's activations are staged once, every
//            warp streams its own units' rows through a one-slot ring of bulk copies
//            and multiplies them on the tensor cores (mma.sync, exact bf16 operands);
//            h = silu(W_g x) * (W_u x) for each pair of the tile
//   down     the same over (tile, 16 output rows) units, activations = h of the
//            tile's pairs (bf16 hi + lo); o = W_d h per pair
//   combine  y = resid + sum_k w_k o_k + sigma o_s per token, in slot order, rounded
//            once to bf16
//
// There are no grid-wide waits: the kernel boundaries order the phases.
//
// The pages decode one token at a time (Flash-MoE); grouping a batch's (token,
// expert) pairs by expert is this library's addition for batched decode, with the
// per-pair arithmetic of the single-token path (hotdry.top, "量化策略" and "Metal
// GPU管线").
#pragma once

#include "fmoe_device.cuh"
#include "fmoe_layer.cuh"
#include "fmoe_topk.cuh"

namespace fmoe {

constexpr int kTileTok = 8;    // pairs of one expert whose activations are staged together (MMA N)
constexpr int kRouterTok = 16;  // tokens per pass of the batched router
constexpr int kMaxBatch = 64;  // tokens one batched call may have
constexpr int kMaxSeg = 64;    // tiles one block's unit range may touch
constexpr int kRing = 1;       // bulk copies in flight per warp (16 warps: latency is hidden across warps)

struct GTile {
  int expert, p0, n;
  int tok16;  // the tile's first 16-pair block in the activation tile buffers (tcgen05 path)
};

// Work weight of one unit of a tile of n pairs (relative).  Every unit moves the same
// bytes and, on the tensor cores, does the same work whatever n is.
__host__ __device__ constexpr int tile_weight(int n) { return n > 0 ? 1 : 0; }

struct GParams {
  int H, I, E, K, has_shared, has_rbias, nq, T;
  const uint8_t* experts;
  unsigned long long rec_bytes, o_gu_sb, o_d_q, o_d_sb;
  int qh, qi, sh, si;
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
  int* ntiles;        // tiles of more than small_tok pairs (the tensor-core kernels)
  GTile* tiles;
  long long* tcost;   // [ntiles + 1] prefix sums of tile weights
  int* ntiles_s;      // tiles of at most small_tok pairs (the CUDA-core kernels)
  GTile* tiles_s;
  long long* tcost_s;
  GTile* tiles_all;   // every tile, before the split
  int small_tok;      // 0: every tile goes to the tensor-core kernels
  int* pair_token;   // [P] token of each pair
  int* pidx;         // [T][K + 1] pair of (token, slot)
  int32_t* idx;      // [T][K]
  float* w;          // [T][K]
  float* sig;        // [T]
  double* lpart;     // [T][(E + 1) * nq]
  float* hbuf;       // [P][I]
  float* obuf;       // [P][H]
  uint8_t* xg;       // tcgen05 path: gate/up activation tiles (x of each tile's pairs)
  uint8_t* hg;       // tcgen05 path: down activation tiles (h of each tile's pairs)
  int tile_tok;      // pairs per tile: kTileTok (mma.sync path) or kUTileTok (tcgen05 path)
  unsigned long long wait_ns;
};

// ---------------------------------------------------------------- router
// Units are (row, column split q) in split-major order (u = q * rows + row; the shared
// gate vector is row E), so a block's contiguous range of units touches at most a
// couple of column splits.  Block b stages its units' router slices by bulk copies and,
// kRouterTok tokens at a time, the activations of those splits as floats (exact for
// bf16; widened to fp64 where they are used; all loads
// in flight); a warp per unit, every lane accumulating each token in the single-token
// kernel's order, so the logits are bit-identical to that path.
__host__ __device__ inline int router_splits_touched(int rows, int nq, int G) {
  const int per = (rows * nq + G - 1) / G;  // units of the largest block
  return min(nq, (per + rows - 1) / rows + 1);
}

__global__ void __launch_bounds__(kThreads, 1) grouped_router_kernel(const __grid_constant__ GParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  grid_launch_dependents();
  grid_dependency_wait();
  if (ld_relaxed_u32(p.err) != 0) return;
  const int rows = p.E + (p.has_shared ? 1 : 0);
  const int G = gridDim.x, b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int U = rows * p.nq;
  const int u0 = static_cast<int>(static_cast<long long>(U) * b / G);
  const int u1 = static_cast<int>(static_cast<long long>(U) * (b + 1) / G);
  const int nu = u1 - u0;
  const int H = p.H, hc = H / p.nq;
  const int q0 = nu > 0 ? u0 / rows : 0;
  const int nqs = nu > 0 ? (u1 - 1) / rows - q0 + 1 : 0;  // splits touched
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  float* wr = reinterpret_cast<float*>(smem + 128);               // [nu][hc]
  float* xd = reinterpret_cast<float*>(smem + 128 + r128(static_cast<uint32_t>(nu) * hc * 4u));
  // xd: [kRouterTok][nqs * hc] floats of the touched splits
  __shared__ int fail;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init_fence();
    fail = 0;
  }
  __syncthreads();
  if (nu == 0) return;
  if (threadIdx.x == 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nu) * hc * 4u);
    for (int u = u0; u < u1; ++u) {
      const int q = u / rows, r = u % rows;
      const float* src = (r < p.E ? p.router + static_cast<size_t>(r) * H : p.sgate) + static_cast<size_t>(q) * hc;
      bulk_g2s(wr + static_cast<size_t>(u - u0) * hc, src, static_cast<uint32_t>(hc) * 4u, bar);
    }
  }
  const int n4 = nqs * hc / 4;  // float2 per staged token row in each of the two arrays
  // xa[t][k] = (x[4k], x[4k+1]), xb[t][k] = (x[4k+2], x[4k+3]) of the touched splits:
  // a warp's 8-byte loads of consecutive k are conflict-free
  float2* xa = reinterpret_cast<float2*>(xd);
  float2* xb = xa + static_cast<size_t>(kRouterTok) * n4;
  constexpr int KU = 8;
  for (int tg = 0; tg < p.T; tg += kRouterTok) {
    const int nt = min(kRouterTok, p.T - tg);
    if (tg > 0) __syncthreads();  // the previous group's activations are no longer read
    for (int base = 0; base < nt * n4; base += KU * kThreads) {
      uint2 v[KU];
#pragma unroll
      for (int k = 0; k < KU; ++k) {
        const int i = base + static_cast<int>(threadIdx.x) + k * kThreads;
        v[k] = make_uint2(0u, 0u);
        if (i < nt * n4) {
          const int t = i / n4, c4 = i % n4;
          v[k] = reinterpret_cast<const uint2*>(p.x + static_cast<size_t>(tg + t) * H + static_cast<size_t>(q0) * hc)[c4];
        }
      }
#pragma unroll
      for (int k = 0; k < KU; ++k) {
        const int i = base + static_cast<int>(threadIdx.x) + k * kThreads;
        if (i < nt * n4) {
          const int t = i / n4, c4 = i % n4;
          xa[static_cast<size_t>(t) * n4 + c4] =
              make_float2(__uint_as_float(v[k].x << 16), __uint_as_float(v[k].x & 0xFFFF0000u));
          xb[static_cast<size_t>(t) * n4 + c4] =
              make_float2(__uint_as_float(v[k].y << 16), __uint_as_float(v[k].y & 0xFFFF0000u));
        }
      }
    }
    if (tg == 0 && threadIdx.x == 0 && !mbar_wait_bounded(bar, 0, p.wait_ns, p.err)) fail = 1;
    __syncthreads();
    if (fail) return;
    // tiles of two units x four tokens, spread over all warps (one activation load
    // serves both rows; enough tiles to keep every warp's loads in flight)
    constexpr int kTT = 4;
    const int nup = (nu + 1) / 2, nth = (nt + kTT - 1) / kTT;
    for (int tile = warp; tile < nup * nth; tile += kWarps) {
      const int u = u0 + 2 * (tile / nth), t0 = kTT * (tile % nth);
      const bool two = u + 1 < u1;
      const int qa = u / rows, ra = u % rows;
      const int ub = two ? u + 1 : u;
      const int qb = ub / rows, rb = ub % rows;
      const float4* wa = reinterpret_cast<const float4*>(wr + static_cast<size_t>(u - u0) * hc);
      const float4* wb = reinterpret_cast<const float4*>(wr + static_cast<size_t>(ub - u0) * hc);
      const int ka = (qa - q0) * (hc / 4), kb = (qb - q0) * (hc / 4);
      double a0[kTT], a1[kTT], b0[kTT], b1[kTT];
#pragma unroll
      for (int t = 0; t < kTT; ++t) a0[t] = a1[t] = b0[t] = b1[t] = 0.0;
      for (int k = lane; k < hc / 4; k += 32) {
        const float4 va = wa[k];
        const float4 vb = wb[k];
        const double wa0 = va.x, wa1 = va.y, wa2 = va.z, wa3 = va.w;
        const double wb0 = vb.x, wb1 = vb.y, wb2 = vb.z, wb3 = vb.w;
#pragma unroll
        for (int t = 0; t < kTT; ++t) {
          if (t0 + t < nt) {
            const size_t xt = static_cast<size_t>(t0 + t) * n4 + k;
            const float2 fa0 = xa[xt + ka], fb0 = xb[xt + ka];
            const double xa0x = fa0.x, xa0y = fa0.y, xb0x = fb0.x, xb0y = fb0.y;
            a0[t] = fma(wa0, xa0x, a0[t]);
            a1[t] = fma(wa1, xa0y, a1[t]);
            a0[t] = fma(wa2, xb0x, a0[t]);
            a1[t] = fma(wa3, xb0y, a1[t]);
            // the second unit usually shares the split (and so the loads)
            double xa1x = xa0x, xa1y = xa0y, xb1x = xb0x, xb1y = xb0y;
            if (kb != ka) {
              const float2 fa1 = xa[xt + kb], fb1 = xb[xt + kb];
              xa1x = fa1.x;
              xa1y = fa1.y;
              xb1x = fb1.x;
              xb1y = fb1.y;
            }
            b0[t] = fma(wb0, xa1x, b0[t]);
            b1[t] = fma(wb1, xa1y, b1[t]);
            b0[t] = fma(wb2, xb1x, b0[t]);
            b1[t] = fma(wb3, xb1y, b1[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kTT; ++t) {
        if (t0 + t < nt) {
          const double la = warp_sum_d(a0[t] + a1[t]);
          const double lb = warp_sum_d(b0[t] + b1[t]);
          if (lane == 0) {
            p.lpart[(static_cast<size_t>(tg + t0 + t) * rows + ra) * p.nq + qa] = la;
            if (two) p.lpart[(static_cast<size_t>(tg + t0 + t) * rows + rb) * p.nq + qb] = lb;
          }
        }
      }
    }
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
  uint32_t slog, skey, ckey, cidx, sel, sidx, mask, off, tn, wsum, misc;
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
  s.mask = o; o = r128(o + E * 8u);
  s.off = o; o = r128(o + E * 4u);
  s.tn = o; o = r128(o + max_tiles * 4u);
  s.wsum = o; o = r128(o + (kWarps + 1) * 8u);
  s.misc = o; o = r128(o + 64u);
  *total = o;
  return s;
}

// The last block: pairs grouped by expert (experts ascending, tokens ascending within
// an expert, then the shared expert's pair of every token), tiles of <= kTileTok
// pairs and the prefix sums of their work weights.  A 64-bit token mask per expert
// gives every pair its place without any serial scan: the pair (t, e) is number
// popcount(mask[e] & ((1 << t) - 1)) of expert e.
__device__ void build_groups(const GParams& p, uint8_t* smem, const TopkSmem& L) {
  const int E = p.E, K = p.K, T = p.T, TT = p.tile_tok;
  int* sidx = reinterpret_cast<int*>(smem + L.sidx);
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(smem + L.mask);
  int* off = reinterpret_cast<int*>(smem + L.off);
  int* tn = reinterpret_cast<int*>(smem + L.tn);
  long long* wsum = reinterpret_cast<long long*>(smem + L.wsum);
  for (int e = threadIdx.x; e < E; e += kThreads) mask[e] = 0ull;
  __syncthreads();
  for (int i = threadIdx.x; i < T * K; i += kThreads) {
    const int e = __ldcg(p.idx + i);
    sidx[i] = e;
    atomicOr(&mask[e], 1ull << (i / K));
  }
  __syncthreads();
  // per-thread runs of ceil(E / kThreads) experts: pair and tile offsets
  const int per = (E + kThreads - 1) / kThreads;
  const int e0 = min(E, static_cast<int>(threadIdx.x) * per), e1 = min(E, e0 + per);
  long long npairs = 0, ntl = 0;
  for (int e = e0; e < e1; ++e) {
    const int c = __popcll(mask[e]);
    npairs += c;
    ntl += (c + TT - 1) / TT;
  }
  long long tot_pairs, tot_tiles;
  const long long poff = block_scan_excl(npairs, wsum, &tot_pairs);
  const long long toff0 = block_scan_excl(ntl, wsum, &tot_tiles);
  {
    long long po = poff, to = toff0;
    for (int e = e0; e < e1; ++e) {
      const int c = __popcll(mask[e]);
      off[e] = static_cast<int>(po);
      for (int i = 0; i * TT < c; ++i) {
        const int n = min(TT, c - i * TT);
        p.tiles_all[to + i] = GTile{e, static_cast<int>(po) + i * TT, n, 0};
        tn[to + i] = n;
      }
      po += c;
      to += (c + TT - 1) / TT;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < T * K; i += kThreads) {
    const int e = sidx[i], t = i / K, k = i % K;
    const int pr = off[e] + __popcll(mask[e] & ((1ull << t) - 1ull));
    p.pair_token[pr] = t;
    p.pidx[t * (K + 1) + k] = pr;
  }
  const int routed_tiles = static_cast<int>(tot_tiles);
  const int PR = T * K;  // the shared expert's pairs follow the routed ones
  int ntiles = routed_tiles;
  if (p.has_shared) {
    for (int t = threadIdx.x; t < T; t += kThreads) {
      p.pair_token[PR + t] = t;
      p.pidx[t * (K + 1) + K] = PR + t;
    }
    const int nts = (T + TT - 1) / TT;
    for (int i = threadIdx.x; i < nts; i += kThreads) {
      const int n = min(TT, T - i * TT);
      p.tiles_all[routed_tiles + i] = GTile{E, PR + i * TT, n, 0};
      tn[routed_tiles + i] = n;
    }
    ntiles += nts;
  }
  __syncthreads();
  // split (stable) into the small tiles (<= small_tok pairs) and the others; prefix
  // sums of each list's work weights and of the large tiles' 16-pair blocks
  // (contiguous runs per thread)
  const int tper = (ntiles + kThreads - 1) / kThreads;
  const int i0 = min(ntiles, static_cast<int>(threadIdx.x) * tper), i1 = min(ntiles, i0 + tper);
  long long nsm = 0, nlg = 0, wsm = 0, wlg = 0, b16 = 0;
  for (int i = i0; i < i1; ++i) {
    if (tn[i] <= p.small_tok) {
      ++nsm;
      wsm += tile_weight(tn[i]);
    } else {
      ++nlg;
      wlg += tile_weight(tn[i]);
      b16 += (tn[i] + 15) / 16;
    }
  }
  long long ns_tot, nl_tot, ws_tot, wl_tot, btot;
  long long so = block_scan_excl(nsm, wsum, &ns_tot);
  long long lo = block_scan_excl(nlg, wsum, &nl_tot);
  long long cs = block_scan_excl(wsm, wsum, &ws_tot);
  long long cl = block_scan_excl(wlg, wsum, &wl_tot);
  long long c16 = block_scan_excl(b16, wsum, &btot);
  for (int i = i0; i < i1; ++i) {
    GTile t = p.tiles_all[i];
    if (tn[i] <= p.small_tok) {
      p.tiles_s[so] = t;
      p.tcost_s[so] = cs;
      ++so;
      cs += tile_weight(tn[i]);
    } else {
      t.tok16 = static_cast<int>(c16);
      p.tiles[lo] = t;
      p.tcost[lo] = cl;
      ++lo;
      cl += tile_weight(tn[i]);
      c16 += (tn[i] + 15) / 16;
    }
  }
  if (threadIdx.x == 0) {
    p.tcost[nl_tot] = wl_tot;
    p.tcost_s[ns_tot] = ws_tot;
    *p.ntiles = static_cast<int>(nl_tot);
    *p.ntiles_s = static_cast<int>(ns_tot);
    *p.ticket = 0;  // ready for the next launch (every block of this one has counted)
  }
}

// One block per token: logits from the router partials, the rank top-K, the
// renormalised weights and the shared gate; then the grouping by the last block.
__global__ void __launch_bounds__(kThreads, 1) grouped_topk_kernel(const __grid_constant__ GParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  grid_launch_dependents();
  grid_dependency_wait();
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
// Tensor-core (mma.sync m16n8k16, bf16 in, fp32 accumulate) dequantising matvecs of a
// tile: M = 16 weight rows, N = 8 pairs of the tile, K = the row's columns.
//
// Exactness.  A code c enters the MMA as the bf16 value 1 + c/2^b' (b' = 4 for 4-bit
// codes, 2 for 2-bit: the code placed in the top mantissa bits by one rotate and one
// LOP3, no conversion), the activations as exact bf16 (x is bf16; h, fp32, is split
// into hi = bf16(h) and lo = bf16(h - hi) and both are multiplied).  Every product is
// exact in fp32.  Per 64-column group g the accumulator D_g = X_g + sum_c c*x_c/2^b'
// (X_g = sum of the group's activations) is folded with the group's scale s and bias
// b:  sum_c (s*c + b) x_c = (2^b' s) D_g + (b - 2^b' s) X_g, both coefficients exact.
//
// The K order inside each 16-column step is permuted (the same way for A and B) so
// that one rotate of a code word yields the pair of codes a fragment register holds:
// 4-bit, step columns c0..c0+15 (words w0 = c0..c0+7, w1 = c0+8..c0+15):
//   k = 2q+j      <-> column c0 + q + 4j         (from w0)
//   k = 8 + 2q+j  <-> column c0 + 8 + q + 4j     (from w1)
// 2-bit, one word w = c0..c0+15:
//   k = 2q+j      <-> column c0 + q + 8j
//   k = 8 + 2q+j  <-> column c0 + q + 4 + 8j
// where q = lane % 4 and j in {0, 1}.
constexpr int kGWarps = 16;  // warps of a grouped matvec block
constexpr int kGThreads = kGWarps * 32;
constexpr int kPieceCols = 1024;  // columns of one staged piece of a unit's 16 rows

__device__ __forceinline__ unsigned long long f32x2(float lo, float hi) {
  return (static_cast<unsigned long long>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The register holding codes (q, q+4) of a 4-bit word (low, high half) as bf16 1+c/16.
__device__ __forceinline__ uint32_t codes4_bf16(uint32_t w, int q) {
  return (__funnelshift_r(w, w, (4 * q - 3) & 31) & 0x00780078u) | 0x3F803F80u;
}
// Codes (q + 4h, q + 4h + 8) of a 2-bit word as bf16 1+c/4 (h = 0 or 1).
__device__ __forceinline__ uint32_t codes2_bf16(uint32_t w, int q, int h) {
  return (__funnelshift_r(w, w, (2 * q + 8 * h - 5) & 31) & 0x00600060u) | 0x3F803F80u;
}

// Shared-memory geometry of one grouped matvec phase (host and device).
struct MvGeom {
  int ncol;         // columns of a weight row
  int kc;           // columns per piece
  int npiece;       // pieces per unit
  int R;            // units per tile
  int code_stride;  // bytes per staged code row (padded: rows fall in different banks)
  int sb_stride;    // bytes per staged (scale,bias) row (padded)
  int piece_bytes;  // 16 rows of codes and (scale,bias)
  int frag_bytes;   // staged activations in fragment order (hi and lo for down)
  int sum_bytes;    // per-group activation sums
};

__host__ __device__ inline MvGeom mv_geom(bool down, int H, int I, int bits) {
  MvGeom g;
  g.ncol = down ? I : H;
  g.kc = g.ncol < kPieceCols ? g.ncol : kPieceCols;
  g.npiece = (g.ncol + g.kc - 1) / g.kc;
  g.R = down ? H / 16 : I / 8;
  g.code_stride = static_cast<int>(r16(static_cast<uint32_t>(g.kc * bits / 8))) + 16;
  g.sb_stride = static_cast<int>(r16(static_cast<uint32_t>(g.kc / 64 * 4))) + 16;
  g.piece_bytes = 16 * (g.code_stride + g.sb_stride);
  g.frag_bytes = (down ? 2 : 1) * (g.ncol / 16) * 32 * 8;
  g.sum_bytes = static_cast<int>(r128(static_cast<uint32_t>(g.ncol / 64 * kTileTok * 4)));
  return g;
}

// Units of a phase: unit (tile i, row block r) of R row blocks per tile carries the
// tile's work weight; block b takes the units whose position falls in its equal share
// [b, b+1) * total / G of the weighted sequence.
struct alignas(128) GHeader {
  uint64_t bars[kGWarps][kRing];
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
  const GParams& p;
  MvGeom G;
  GHeader* hdr;
  uint32_t* frag;  // [ncol/16][32] uint2 (and the lo half after it for down)
  float* xsum;     // [ncol/64][kTileTok]
  uint8_t* ring;
  int warp, lane;

  __device__ GroupedKernel(const GParams& pp, uint8_t* smem) : p(pp) {
    warp = threadIdx.x >> 5;
    lane = threadIdx.x & 31;
    G = mv_geom(DOWN, p.H, p.I, BITS);
    hdr = reinterpret_cast<GHeader*>(smem);
    frag = reinterpret_cast<uint32_t*>(smem + sizeof(GHeader));
    xsum = reinterpret_cast<float*>(smem + sizeof(GHeader) + G.frag_bytes);
    ring = smem + sizeof(GHeader) + G.frag_bytes + G.sum_bytes;
  }

  // ---- the block's segments: (tile, [ra, rb)) in tile order
  __device__ void plan_segments() {
    const int nt = __ldcg(p.ntiles);
    const long long Ctot = __ldcg(p.tcost + nt);
    const int NB = gridDim.x, b = blockIdx.x;
    const long long R = G.R;
    const long long X0 = Ctot * R * b / NB, X1 = Ctot * R * (b + 1) / NB;
    if (threadIdx.x == 0) {
      hdr->nseg = 0;
      hdr->first = 0;
      hdr->abort_flag = 0;
    }
    __syncthreads();
    // units of tile i at positions tcost[i]*R + r*w_i, r in [0, R)
    auto range = [&](int i, int& ra, int& rb) {
      const long long c0 = __ldcg(p.tcost + i) * R;
      const long long wi = __ldcg(p.tcost + i + 1) - __ldcg(p.tcost + i);
      ra = X0 <= c0 ? 0 : static_cast<int>(min(R, (X0 - c0 + wi - 1) / wi));
      rb = X1 <= c0 ? 0 : static_cast<int>(min(R, (X1 - c0 + wi - 1) / wi));
    };
    for (int i = threadIdx.x; i < nt; i += kGThreads) {
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
    for (int s = threadIdx.x; s < nseg; s += kGThreads) {
      int ra, rb;
      range(first + s, ra, rb);
      hdr->seg_tile[s] = first + s;
      hdr->seg_ra[s] = ra;
      hdr->seg_rb[s] = rb;
    }
    __syncthreads();
  }

  // ---- this warp's pieces in order: segment s, units ra + warp, ra + warp + kGWarps, ...,
  // pieces 0 .. npiece-1 of each
  struct It {
    int s, u, pc;
  };
  __device__ __forceinline__ It norm(It it) const {
    while (it.s < hdr->nseg && it.u >= hdr->seg_rb[it.s]) {
      ++it.s;
      if (it.s < hdr->nseg) it.u = hdr->seg_ra[it.s] + warp;
    }
    return it;
  }
  __device__ __forceinline__ It first_piece() const {
    return hdr->nseg > 0 ? norm(It{0, hdr->seg_ra[0] + warp, 0}) : It{0, 0, 0};
  }
  __device__ __forceinline__ It next_piece(It it) const {
    if (it.pc + 1 < G.npiece) return It{it.s, it.u, it.pc + 1};
    return norm(It{it.s, it.u + kGWarps, 0});
  }
  __device__ __forceinline__ bool valid(It it) const { return it.s < hdr->nseg; }

  __device__ __forceinline__ uint8_t* slot_ptr(int slot) const {
    return ring + (static_cast<uint32_t>(warp) * kRing + slot) * static_cast<uint32_t>(G.piece_bytes);
  }

  // staged row i (0..15) of unit u: source offsets of its code row piece and its
  // (scale, bias) row piece inside the expert record
  __device__ __forceinline__ void row_src(int u, int i, int pc, unsigned long long* qoff, unsigned long long* soff,
                                          uint32_t* qbytes, uint32_t* sbytes) const {
    const int c0 = pc * G.kc, cols = min(G.kc, G.ncol - c0);
    *qbytes = static_cast<uint32_t>(cols * BITS / 8);
    *sbytes = static_cast<uint32_t>(cols / 64 * 4);
    if (DOWN) {
      const unsigned long long j = static_cast<unsigned long long>(16 * u + i);
      *qoff = p.o_d_q + j * p.qi + static_cast<unsigned long long>(c0 * BITS / 8);
      *soff = p.o_d_sb + j * p.si + static_cast<unsigned long long>(c0 / 64 * 4);
    } else {  // rows 0..7: gate rows 8u..8u+7, rows 8..15: the up rows of the same r
      const unsigned long long r = static_cast<unsigned long long>(8 * u + (i & 7));
      const unsigned long long up = i >= 8 ? 1ull : 0ull;
      *qoff = r * 2u * p.qh + up * p.qh + static_cast<unsigned long long>(c0 * BITS / 8);
      *soff = p.o_gu_sb + r * 2u * p.sh + up * p.sh + static_cast<unsigned long long>(c0 / 64 * 4);
    }
  }

  // the whole warp: bulk copies of piece `it` into ring slot `slot` (lanes 0..15 the
  // code rows, lanes 16..31 the 16-byte covers of the (scale, bias) rows)
  __device__ void issue(It it, int slot) {
    const GTile tl = p.tiles[hdr->seg_tile[it.s]];
    const uint8_t* rec = p.experts + static_cast<unsigned long long>(tl.expert) * p.rec_bytes;
    uint8_t* dst = slot_ptr(slot);
    uint64_t* bar = &hdr->bars[warp][slot];
    const int i = lane & 15;
    unsigned long long qoff, soff;
    uint32_t qb, sb;
    row_src(it.u, i, it.pc, &qoff, &soff, &qb, &sb);
    const unsigned long long a = soff & ~15ull, e = (soff + sb + 15ull) & ~15ull;
    const uint32_t bytes = lane < 16 ? qb : static_cast<uint32_t>(e - a);
    const uint32_t total = __reduce_add_sync(0xffffffffu, bytes);
    if (lane == 0) mbar_arrive_expect_tx(bar, total);
    __syncwarp();
    fence_proxy_async_smem();  // this lane's earlier reads of the slot before the copy
    if (lane < 16)
      bulk_g2s(dst + i * G.code_stride, rec + qoff, qb, bar);
    else
      bulk_g2s(dst + 16 * G.code_stride + i * G.sb_stride, rec + a, bytes, bar);
  }

  // ---- activations of a tile in fragment order, every load issued before any use:
  // x rows of the tile's tokens (bf16) or h rows of its pairs (fp32, split hi + lo);
  // per-group sums by shuffles over the 16 threads of a 64-column group.  Pairs
  // beyond the tile's count are zeros.
  __device__ __forceinline__ uint32_t frag_half(int c, int n) const {
    // 16-bit index of column c of pair n in the fragment array
    const int ks = c >> 4, cc = c & 15;
    int q, reg, j;
    if (BITS == 4) {
      reg = cc >> 3;
      const int pos = cc & 7;
      q = pos & 3;
      j = pos >> 2;
    } else {
      j = cc >> 3;
      const int r = cc & 7;
      q = r & 3;
      reg = r >> 2;
    }
    return static_cast<uint32_t>((((ks * 32 + 4 * n + q) * 2 + reg) * 2) + j);
  }

  __device__ void stage_tile(const GTile& tl) {
    constexpr int KU = 8;
    const int n4 = G.ncol / 4;
    const int total = kTileTok * n4;
    uint16_t* f16 = reinterpret_cast<uint16_t*>(frag);
    uint16_t* f16lo = f16 + (G.ncol / 16) * 32 * 4;
    for (int base = 0; base < total; base += KU * kGThreads) {  // block-uniform trip count
      float4 v[KU];
#pragma unroll
      for (int k = 0; k < KU; ++k) {
        const int i = base + static_cast<int>(threadIdx.x) + k * kGThreads;
        v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        const int n = i / n4, q4 = i % n4;
        if (i < total && n < tl.n) {
          if (DOWN) {
            v[k] = __ldcg(reinterpret_cast<const float4*>(p.hbuf + static_cast<size_t>(tl.p0 + n) * p.I) + q4);
          } else {
            const uint2 u = reinterpret_cast<const uint2*>(p.x + static_cast<size_t>(hdr->tok[n]) * p.H)[q4];
            v[k] = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                               __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
          }
        }
      }
#pragma unroll
      for (int k = 0; k < KU; ++k) {
        const int i = base + static_cast<int>(threadIdx.x) + k * kGThreads;
        float sum = (v[k].x + v[k].y) + (v[k].z + v[k].w);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (i < total) {
          const int n = i / n4, c = 4 * (i % n4);
          const float vv[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t fi = frag_half(c + e, n);
            const uint16_t hi = f32_to_bf16(vv[e]);
            f16[fi] = hi;
            if (DOWN) f16lo[fi] = f32_to_bf16(vv[e] - bf16_to_f32(hi));
          }
          if ((i & 15) == 0) xsum[(c >> 6) * kTileTok + n] = sum;
        }
      }
    }
  }

  // ---- one piece: 16 rows x the piece's columns against the tile's pairs, folded
  // per group into acc (rows g and g+8 of the unit, pairs 2q and 2q+1)
  // acc: (row g, pairs 2q and 2q + 1) and (row g + 8, same pairs) as packed f32x2
  __device__ __forceinline__ void piece(const uint8_t* sl, int u, int pc, unsigned long long (&acc)[2]) const {
    const int g = lane >> 2, q = lane & 3;
    const int c0 = pc * G.kc, cols = min(G.kc, G.ncol - c0);
    const uint8_t* ra = sl + g * G.code_stride;
    const uint8_t* rb = sl + (g + 8) * G.code_stride;
    unsigned long long qo, so;
    uint32_t qb, sbb;
    row_src(u, g, pc, &qo, &so, &qb, &sbb);
    const uint32_t* sa = reinterpret_cast<const uint32_t*>(sl + 16 * G.code_stride + g * G.sb_stride + (so & 15ull));
    row_src(u, g + 8, pc, &qo, &so, &qb, &sbb);
    const uint32_t* sb = reinterpret_cast<const uint32_t*>(sl + 16 * G.code_stride + (g + 8) * G.sb_stride + (so & 15ull));
    const uint2* fr = reinterpret_cast<const uint2*>(frag);
    const uint2* frlo = fr + (G.ncol / 16) * 32;
    constexpr float kScaleMul = BITS == 4 ? 16.0f : 4.0f;
#pragma unroll 2
    for (int grp = 0; grp < cols / 64; ++grp) {
      // a group is 32 bytes of a 4-bit row (two 16-byte loads) or 16 of a 2-bit row
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      const int ks0 = (c0 >> 4) + grp * 4;
      if (BITS == 4) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4 wa = *reinterpret_cast<const uint4*>(ra + grp * 32 + half * 16);
          const uint4 wb = *reinterpret_cast<const uint4*>(rb + grp * 32 + half * 16);
#pragma unroll
          for (int st = 0; st < 2; ++st) {
            const uint32_t a[4] = {codes4_bf16(st ? wa.z : wa.x, q), codes4_bf16(st ? wb.z : wb.x, q),
                                   codes4_bf16(st ? wa.w : wa.y, q), codes4_bf16(st ? wb.w : wb.y, q)};
            const int ks = ks0 + half * 2 + st;
            const uint2 bh = fr[ks * 32 + lane];
            float(&dd)[4] = (st == 0) ? d : e;
            mma_bf16_16816(dd, a, bh.x, bh.y);
            if (DOWN) {
              const uint2 bl = frlo[ks * 32 + lane];
              mma_bf16_16816(dd, a, bl.x, bl.y);
            }
          }
        }
      } else {
        const uint4 wa = *reinterpret_cast<const uint4*>(ra + grp * 16);
        const uint4 wb = *reinterpret_cast<const uint4*>(rb + grp * 16);
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          const uint32_t xa = st == 0 ? wa.x : st == 1 ? wa.y : st == 2 ? wa.z : wa.w;
          const uint32_t xb = st == 0 ? wb.x : st == 1 ? wb.y : st == 2 ? wb.z : wb.w;
          const uint32_t a[4] = {codes2_bf16(xa, q, 0), codes2_bf16(xb, q, 0), codes2_bf16(xa, q, 1),
                                 codes2_bf16(xb, q, 1)};
          const int ks = ks0 + st;
          const uint2 bh = fr[ks * 32 + lane];
          float(&dd)[4] = (st & 1) ? e : d;
          mma_bf16_16816(dd, a, bh.x, bh.y);
          if (DOWN) {
            const uint2 bl = frlo[ks * 32 + lane];
            mma_bf16_16816(dd, a, bl.x, bl.y);
          }
        }
      }
      const unsigned long long X2 =
          *reinterpret_cast<const unsigned long long*>(xsum + ((c0 >> 6) + grp) * kTileTok + 2 * q);
      const uint32_t wsa = sa[grp], wsb = sb[grp];
      const float s16a = kScaleMul * sb_scale(wsa), s16b = kScaleMul * sb_scale(wsb);
      const float cba = sb_bias(wsa) - s16a, cbb = sb_bias(wsb) - s16b;
      // acc = s16 (d + e) + (cb X + acc), two pairs per packed operation
      fma2(acc[0], f32x2(cba, cba), X2);
      fma2(acc[1], f32x2(cbb, cbb), X2);
      fma2(acc[0], f32x2(s16a, s16a), add2(f32x2(d[0], d[1]), f32x2(e[0], e[1])));
      fma2(acc[1], f32x2(s16b, s16b), add2(f32x2(d[2], d[3]), f32x2(e[2], e[3])));
    }
  }

  __device__ __forceinline__ void epilogue(const GTile& tl, int u, const unsigned long long (&acc2)[2]) const {
    const float acc[4] = {__uint_as_float(static_cast<uint32_t>(acc2[0])), __uint_as_float(static_cast<uint32_t>(acc2[0] >> 32)),
                          __uint_as_float(static_cast<uint32_t>(acc2[1])), __uint_as_float(static_cast<uint32_t>(acc2[1] >> 32))};
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int n = 2 * q + j;
      if (n >= tl.n) continue;
      if (DOWN) {
        float* o = p.obuf + static_cast<size_t>(tl.p0 + n) * p.H + 16 * u + g;
        o[0] = acc[j];
        o[8] = acc[2 + j];
      } else {
        const float gv = acc[j], uv = acc[2 + j];
        p.hbuf[static_cast<size_t>(tl.p0 + n) * p.I + 8 * u + g] = (gv / (1.0f + expf(-gv))) * uv;
      }
    }
  }

  __device__ void run() {
    if (threadIdx.x == 0) {
      for (int w = 0; w < kGWarps; ++w)
        for (int s = 0; s < kRing; ++s) mbar_init(&hdr->bars[w][s], 1);
      mbar_init_fence();
    }
    __syncthreads();
    plan_segments();
    if (hdr->abort_flag) return;
    // prologue: the warp's first kRing pieces in flight
    It pre = first_piece();
    uint32_t issued = 0;  // pieces this warp has requested
    for (int s = 0; s < kRing; ++s) {
      if (valid(pre)) {
        issue(pre, s);
        pre = next_piece(pre);
        ++issued;
      }
    }
    uint32_t k = 0;  // pieces this warp has consumed
    bool ok = true;
    for (int s = 0; s < hdr->nseg; ++s) {
      const GTile tl = p.tiles[hdr->seg_tile[s]];
      __syncthreads();  // the previous tile's activations are no longer read
      if (!DOWN && threadIdx.x < tl.n) hdr->tok[threadIdx.x] = p.pair_token[tl.p0 + threadIdx.x];
      __syncthreads();
      stage_tile(tl);
      __syncthreads();
      if (!ok) continue;
      for (int u = hdr->seg_ra[s] + warp; u < hdr->seg_rb[s] && ok; u += kGWarps) {
        unsigned long long acc[2] = {0ull, 0ull};
        for (int pc = 0; pc < G.npiece; ++pc) {
          const int slot = static_cast<int>(k % kRing);
          const bool arrived = mbar_wait_bounded(&hdr->bars[warp][slot], (k / kRing) & 1u, p.wait_ns, p.err);
          if (!__all_sync(0xffffffffu, arrived)) {
            ok = false;
            break;
          }
          piece(slot_ptr(slot), u, pc, acc);
          ++k;
          __syncwarp();
          if (valid(pre)) {
            issue(pre, slot);
            pre = next_piece(pre);
            ++issued;
          }
        }
        if (ok) epilogue(tl, u, acc);
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
__global__ void __launch_bounds__(kGThreads, 1) grouped_matvec_kernel(const __grid_constant__ GParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  grid_launch_dependents();
  grid_dependency_wait();
  if (ld_relaxed_u32(p.err) != 0) return;
  GroupedKernel<BITS, DOWN> G(p, smem);
  G.run();
}

// y[t][j] = resid[t][j] + sum_k w[t][k] o[pair(t, k)][j] + sigma_t o[pair(t, shared)][j]:
// block (column chunk, token) stages the token's pairs and weights once, then every
// thread's K+1 output loads are independent.
__global__ void grouped_combine_kernel(const __grid_constant__ GParams p) {
  __shared__ int spi[kMaxK + 1];
  __shared__ float sw[kMaxK + 1];
  grid_launch_dependents();
  grid_dependency_wait();
  if (ld_relaxed_u32(p.err) != 0) return;
  const int t = blockIdx.y;
  const int ns = p.K + (p.has_shared ? 1 : 0);
  if (threadIdx.x < ns) {
    spi[threadIdx.x] = __ldcg(p.pidx + static_cast<size_t>(t) * (p.K + 1) + threadIdx.x);
    sw[threadIdx.x] = threadIdx.x < p.K ? __ldcg(p.w + static_cast<size_t>(t) * p.K + threadIdx.x) : __ldcg(p.sig + t);
  }
  __syncthreads();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= p.H) return;
  float o[kMaxK + 1];
#pragma unroll
  for (int s = 0; s <= kMaxK; ++s)
    if (s < ns) o[s] = __ldcg(p.obuf + static_cast<size_t>(spi[s]) * p.H + j);
  float pa = 0.f;
#pragma unroll
  for (int s = 0; s <= kMaxK; ++s)
    if (s < ns) pa = fmaf(sw[s], o[s], pa);
  const size_t oi = static_cast<size_t>(t) * p.H + j;
  p.y[oi] = f32_to_bf16(bf16_to_f32(p.resid[oi]) + pa);
}

}  // namespace fmoe
