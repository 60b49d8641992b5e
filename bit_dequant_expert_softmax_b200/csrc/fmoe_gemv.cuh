// Batched routed-expert matvecs of small tiles on the CUDA cores (sm_100a).
//
// In a batched call most active experts are chosen by one or two of the batch's
// tokens (with 32 tokens and top-10 of 512 experts, about half of the distinct
// experts get a single pair).  The tensor-core kernels pay their code-to-operand
// conversion once per weight whatever the tile's pair count; for one or two pairs the
// single-token path's dequantising dot needs fewer instructions per weight: a code
// masked in place is read as a subnormal float and multiplied by a pre-scaled
// activation with packed f32x2 FMAs, the per-chunk sums rescaled and folded with the
// group's scale and bias once.  This kernel takes the tiles of at most kSmallTok
// pairs, the tensor-core kernels the rest; the arithmetic per (pair, row) is the
// single-token kernel's.  Measured on the 32-token top-10 layer it is slower than the
// mma.sync kernels on the same tiles (a warp reduction per row pair and piece and the
// per-row addressing outweigh the cheaper products), so the layer runs it only on
// request (FMOE_GROUPED_SMALL=1).
//
// Work: persistent blocks of kGWarps warps over a contiguous, weight-balanced range of units
// (tile, 16 rows): gate/up units are the gate rows 8u..8u+7 and the up rows of the same
// r (rows 0-7 and 8-15 of the unit), down units 16 output rows.  Per tile a block
// stages the activations of the tile's pairs (x, or h for down) in the pre-scaled,
// lane-interleaved layout; each warp streams its units' 16 rows x 32 chunks per piece
// through a private ring of bulk copies; lane l takes chunk l of every row of
// the piece (rows i and i + 8 together, sharing the activation loads); each row pair's
// partials are reduced over the warp and lane i keeps row i's sums for the unit.
#pragma once

#include "fmoe_grouped.cuh"

namespace fmoe {

constexpr int kSmallTok = 2;  // pairs a CUDA-core tile may have

// Shared-memory geometry of one small-tile matvec phase (host and device).
struct SvGeom {
  int ncol;         // columns of a weight row
  int nch;          // chunks of a row (16 bytes of codes each)
  int pch;          // chunks per piece (32, or fewer for a short row)
  int npiece;       // pieces per unit
  int R;            // units per tile
  int code_stride;  // bytes per staged code row
  int sb_stride;    // bytes per staged (scale, bias) row (16-byte cover + words)
  int piece_bytes;  // 16 rows of codes and (scale, bias)
  int act_floats;   // floats of one pair's staged activations (32-chunk padded)
};

template <int BITS>
__host__ __device__ inline SvGeom sv_geom(bool down, int H, int I) {
  SvGeom g;
  g.ncol = down ? I : H;
  g.nch = g.ncol / Chunk<BITS>::kCols;
  g.pch = g.nch < 32 ? g.nch : 32;
  g.npiece = (g.nch + g.pch - 1) / g.pch;
  g.R = down ? H / 16 : I / 8;
  g.code_stride = g.pch * 16;
  g.sb_stride = static_cast<int>(r16(static_cast<uint32_t>(Chunk<BITS>::sb_index(g.pch - 1) + 1) * 4u)) + 16;
  g.piece_bytes = 16 * (g.code_stride + g.sb_stride);
  g.act_floats = ((g.nch + 31) / 32) * 32 * Chunk<BITS>::kCols;
  return g;
}

template <int BITS>
__host__ __device__ inline uint32_t small_smem_bytes(bool down, int H, int I) {
  const SvGeom g = sv_geom<BITS>(down, H, I);
  return static_cast<uint32_t>(sizeof(GHeader)) +
         static_cast<uint32_t>(kSmallTok) * (static_cast<uint32_t>(g.act_floats) * 4u +
                                             r128(static_cast<uint32_t>((g.act_floats / Chunk<BITS>::kCols) * 8))) +
         static_cast<uint32_t>(kGWarps * kRing * g.piece_bytes);
}

// One word pair of two rows {a, b} against NT pairs' activation pairs, accumulated per
// row and pair (the single-token kernel's masked-code products).
template <int BITS, int NT>
__device__ __forceinline__ void small_word_pair(unsigned long long Wa, unsigned long long Wb,
                                                const ulonglong2* const (&xv)[NT], unsigned long long (&acc_a)[NT],
                                                unsigned long long (&acc_b)[NT]) {
  using C = Chunk<BITS>;
  const unsigned long long Va = Wa >> 8, Vb = Wb >> 8;
#pragma unroll
  for (int k = 0; k < C::kF4PerPair; ++k) {
    ulonglong2 x[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) x[t] = xv[t][k * 32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int P = 2 * k + h;
      const int s = C::shift_pos(P);
      const unsigned long long m32 = ((1ull << BITS) - 1ull) << s;
      const unsigned long long mask = (m32 << 32) | m32;
      const bool hi = BITS * P + BITS > 24;
      const unsigned long long ca = (hi ? Va : Wa) & mask, cb = (hi ? Vb : Wb) & mask;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        fma2(acc_a[t], ca, h ? x[t].y : x[t].x);
        fma2(acc_b[t], cb, h ? x[t].y : x[t].x);
      }
    }
  }
}

template <int BITS, bool DOWN>
struct SmallKernel {
  using C = Chunk<BITS>;
  const GParams& p;
  SvGeom G;
  GHeader* hdr;
  float* xs;      // [kSmallTok][act_floats] pre-scaled, interleaved
  float2* xsum;   // [kSmallTok][act_floats / kCols] (chunk sum, rescale)
  uint8_t* ring;
  int warp, lane;
  int nsum;       // float2 per pair in xsum

  __device__ SmallKernel(const GParams& pp, uint8_t* smem) : p(pp) {
    warp = threadIdx.x >> 5;
    lane = threadIdx.x & 31;
    G = sv_geom<BITS>(DOWN, p.H, p.I);
    hdr = reinterpret_cast<GHeader*>(smem);
    xs = reinterpret_cast<float*>(smem + sizeof(GHeader));
    nsum = G.act_floats / C::kCols;
    xsum = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(xs) + static_cast<size_t>(kSmallTok) * G.act_floats * 4);
    ring = reinterpret_cast<uint8_t*>(xsum) + kSmallTok * r128(static_cast<uint32_t>(nsum * 8));
  }

  // ---- the block's segments over the small tiles (as the tensor-core kernels plan
  // theirs over the large ones)
  __device__ void plan_segments() {
    const int nt = __ldcg(p.ntiles_s);
    const long long Ctot = __ldcg(p.tcost_s + nt);
    const int NB = gridDim.x, b = blockIdx.x;
    const long long R = G.R;
    const long long X0 = Ctot * R * b / NB, X1 = Ctot * R * (b + 1) / NB;
    if (threadIdx.x == 0) {
      hdr->nseg = 0;
      hdr->first = 0;
      hdr->abort_flag = 0;
    }
    __syncthreads();
    auto range = [&](int i, int& ra, int& rb) {
      const long long c0 = __ldcg(p.tcost_s + i) * R;
      const long long wi = __ldcg(p.tcost_s + i + 1) - __ldcg(p.tcost_s + i);
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

  // record offsets of row i (0..15) of unit u, piece pc: its codes and the 16-byte
  // cover of its (scale, bias) words
  __device__ __forceinline__ void row_src(int u, int i, int pc, unsigned long long* qoff, unsigned long long* soff,
                                          uint32_t* qbytes, uint32_t* sbytes) const {
    const int m0 = pc * G.pch, nchp = min(G.pch, G.nch - m0);
    const int c0 = m0 * C::kCols, cols = nchp * C::kCols;
    *qbytes = static_cast<uint32_t>(nchp * 16);
    *sbytes = static_cast<uint32_t>(cols / 64 * 4);
    if (DOWN) {
      const unsigned long long j = static_cast<unsigned long long>(16 * u + i);
      *qoff = p.o_d_q + j * p.qi + static_cast<unsigned long long>(c0 * BITS / 8);
      *soff = p.o_d_sb + j * p.si + static_cast<unsigned long long>(c0 / 64 * 4);
    } else {
      const unsigned long long r = static_cast<unsigned long long>(8 * u + (i & 7));
      const unsigned long long up = i >= 8 ? 1ull : 0ull;
      *qoff = r * 2u * p.qh + up * p.qh + static_cast<unsigned long long>(c0 * BITS / 8);
      *soff = p.o_gu_sb + r * 2u * p.sh + up * p.sh + static_cast<unsigned long long>(c0 / 64 * 4);
    }
  }

  // the whole warp: bulk copies of piece `it` into ring slot `slot` (lanes 0..15 the
  // code rows, lanes 16..31 the (scale, bias) covers)
  __device__ void issue(It it, int slot) {
    const GTile tl = p.tiles_s[hdr->seg_tile[it.s]];
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
    fence_proxy_async_smem();
    if (lane < 16)
      bulk_g2s(dst + i * G.code_stride, rec + qoff, qb, bar);
    else
      bulk_g2s(dst + 16 * G.code_stride + i * G.sb_stride, rec + a, bytes, bar);
  }

  // ---- the tile's activations: x rows (bf16) of its tokens, or h rows (fp32) of its
  // pairs, pre-scaled per chunk into the interleaved layout with the chunk sums
  __device__ void stage_tile(const GTile& tl) {
    constexpr int TPC = C::kCols / 4;
    const int n4 = G.ncol / 4;
    const int total = kSmallTok * n4;
    for (int base = 0; base < total; base += kGThreads) {  // block-uniform trip count
      const int i = base + static_cast<int>(threadIdx.x);
      const int t = i / n4, q = i % n4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < total && t < tl.n) {
        if (DOWN) {
          v = __ldcg(reinterpret_cast<const float4*>(p.hbuf + static_cast<size_t>(tl.p0 + t) * p.I) + q);
        } else {
          const int tok = __ldcg(p.pair_token + tl.p0 + t);
          const uint2 u = reinterpret_cast<const uint2*>(p.x + static_cast<size_t>(tok) * p.H)[q];
          v = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                          __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
        }
      }
      float sum = (v.x + v.y) + (v.z + v.w);
      uint32_t mx = max_abs_bits(v);
#pragma unroll
      for (int o = 1; o < TPC; o <<= 1) {
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (i < total) {
        const int c0 = 4 * q, pre = chunk_pre(mx);
        float* d = xs + static_cast<size_t>(t) * G.act_floats;
        d[C::phys(c0 + 0)] = v.x * prescale_factor(pre, C::shift_of(c0 + 0));
        d[C::phys(c0 + 1)] = v.y * prescale_factor(pre, C::shift_of(c0 + 1));
        d[C::phys(c0 + 2)] = v.z * prescale_factor(pre, C::shift_of(c0 + 2));
        d[C::phys(c0 + 3)] = v.w * prescale_factor(pre, C::shift_of(c0 + 3));
        if (q % TPC == 0) xsum[t * nsum + q / TPC] = make_float2(sum, chunk_unscale(pre));
      }
    }
  }

  // ---- one piece: for each row pair (i, i + 8), the lanes' partials over their chunk
  // of the piece for NT pairs, reduced over the warp; lane i keeps row i's sums
  template <int NT>
  __device__ __forceinline__ void piece(const uint8_t* sl, int u, int pc, float (&mine)[kSmallTok]) const {
    const int m0 = pc * G.pch, nchp = min(G.pch, G.nch - m0);
    const bool live = lane < nchp;
    const int m = m0 + (live ? lane : 0);  // this lane's chunk of the row
    const ulonglong2* xv0[NT];
    const ulonglong2* xv1[NT];
    float2 vm[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float* base = xs + static_cast<size_t>(t) * G.act_floats;
      xv0[t] = C::f4(base, m, 0);
      xv1[t] = C::f4(base, m, C::kF4PerPair);
      vm[t] = xsum[t * nsum + m];
    }
    const uint8_t* sbb = sl + 16 * G.code_stride;
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
      float ra[NT], rb[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) ra[t] = rb[t] = 0.f;
      if (live) {
        unsigned long long qoa, soa, qob, sob;
        uint32_t qba, sba, qbb, sbb2;
        row_src(u, i, pc, &qoa, &soa, &qba, &sba);
        row_src(u, i + 8, pc, &qob, &sob, &qbb, &sbb2);
        const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(sl + i * G.code_stride + 16 * lane);
        const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(sl + (i + 8) * G.code_stride + 16 * lane);
        const uint32_t* sa = reinterpret_cast<const uint32_t*>(sbb + i * G.sb_stride + (soa & 15ull));
        const uint32_t* sb = reinterpret_cast<const uint32_t*>(sbb + (i + 8) * G.sb_stride + (sob & 15ull));
        unsigned long long a0[NT], a1[NT], b0[NT], b1[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) a0[t] = a1[t] = b0[t] = b1[t] = 0ull;
        small_word_pair<BITS, NT>(a.x, b.x, xv0, a0, b0);
        small_word_pair<BITS, NT>(a.y, b.y, xv1, a1, b1);
        const uint32_t wa = sa[C::sb_index(lane)], wb = sb[C::sb_index(lane)];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          ra[t] = fmaf(sb_bias(wa), vm[t].x, sb_scale(wa) * ((pair_sum(a0[t]) + pair_sum(a1[t])) * vm[t].y));
          rb[t] = fmaf(sb_bias(wb), vm[t].x, sb_scale(wb) * ((pair_sum(b0[t]) + pair_sum(b1[t])) * vm[t].y));
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        ra[t] = warp_sum(ra[t]);
        rb[t] = warp_sum(rb[t]);
        if (lane == i) mine[t] += ra[t];
        if (lane == i + 8) mine[t] += rb[t];
      }
    }
  }

  // h = silu(g) * u per pair (gate/up: lane i < 8 has the gate row, lane i + 8 the up
  // row of the same r) or o per pair (down: lane i < 16 has row i)
  __device__ void epilogue(const GTile& tl, int u, const float (&mine)[kSmallTok]) const {
#pragma unroll
    for (int t = 0; t < kSmallTok; ++t) {
      const float other = __shfl_down_sync(0xffffffffu, mine[t], 8);
      if (t >= tl.n) continue;
      if (DOWN) {
        if (lane < 16) p.obuf[static_cast<size_t>(tl.p0 + t) * p.H + 16 * u + lane] = mine[t];
      } else if (lane < 8) {
        const float gv = mine[t], uv = other;
        p.hbuf[static_cast<size_t>(tl.p0 + t) * p.I + 8 * u + lane] = (gv / (1.0f + expf(-gv))) * uv;
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
    It pre = first_piece();
    uint32_t issued = 0;
    for (int s = 0; s < kRing; ++s) {
      if (valid(pre)) {
        issue(pre, s);
        pre = next_piece(pre);
        ++issued;
      }
    }
    uint32_t k = 0;
    bool ok = true;
    for (int s = 0; s < hdr->nseg; ++s) {
      const GTile tl = p.tiles_s[hdr->seg_tile[s]];
      __syncthreads();  // the previous tile's activations are no longer read
      stage_tile(tl);
      __syncthreads();
      if (!ok) continue;
      for (int u = hdr->seg_ra[s] + warp; u < hdr->seg_rb[s] && ok; u += kGWarps) {
        float mine[kSmallTok];
#pragma unroll
        for (int t = 0; t < kSmallTok; ++t) mine[t] = 0.f;
        for (int pc = 0; pc < G.npiece; ++pc) {
          const int slot = static_cast<int>(k % kRing);
          const bool arrived = mbar_wait_bounded(&hdr->bars[warp][slot], (k / kRing) & 1u, p.wait_ns, p.err);
          if (!__all_sync(0xffffffffu, arrived)) {
            ok = false;
            break;
          }
          if (tl.n == 1)
            piece<1>(slot_ptr(slot), u, pc, mine);
          else
            piece<2>(slot_ptr(slot), u, pc, mine);
          ++k;
          __syncwarp();
          if (valid(pre)) {
            issue(pre, slot);
            pre = next_piece(pre);
            ++issued;
          }
        }
        if (ok) epilogue(tl, u, mine);
      }
    }
    if (!ok && lane == 0) {
      for (uint32_t n = k; n < issued; ++n)
        mbar_wait_bounded(&hdr->bars[warp][n % kRing], (n / kRing) & 1u, p.wait_ns, p.err);
    }
  }
};

template <int BITS, bool DOWN>
__global__ void __launch_bounds__(kGThreads, 1) grouped_small_kernel(const __grid_constant__ GParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  grid_launch_dependents();
  grid_dependency_wait();
  if (ld_relaxed_u32(p.err) != 0) return;
  SmallKernel<BITS, DOWN> K(p, smem);
  K.run();
}

}  // namespace fmoe
