// The fused routed-expert MoE layer kernel for sm_100a.
//
// One persistent thread block per SM (cooperative launch).  Per token:
//
//   P1  router matvec (fp64 accumulation of exact fp32 x bf16 products) over a
//       slice of router rows per block, partials published with a per-block flag;
//       while they travel, warps 1-15 consume the block's slice of the shared
//       expert's gate/up rows (they do not depend on the routing) and warp 0 polls.
//   P2  every block computes top-K from the logits redundantly; thread 0 requests
//       the block's slice of the K routed experts' gate/up row pairs one copy after
//       another, and its down rows (P3's data) once half of those have landed;
//       warps 1-15 compute h = silu(g) * u, warp 0 the renormalised softmax
//       weights; h is published with a per-block flag.
//   P3  every block stages h of all K+1 experts, computes its slice of output
//       rows of the K+1 down matvecs and the combine
//       y = resid + sum_k w_k o_k + sigma o_s, rounded once to bf16.
//
// All weight bytes move HBM -> shared memory through the bulk-copy (TMA) engine
// as contiguous row ranges, completion tracked by mbarriers; every wait (flags,
// mbarriers) is bounded.
//
// What is computed follows the Flash-MoE pages: routing on the GPU (tinai-dev
// README, "Pipeline mỗi lớp"), softmax then top-K on the probabilities
// (intelliparadigm.com, section 2.1 router snippet; the selection is made on the
// fp64 logits, the same order), 4-/2-bit codes dequantised as code * scale + bias
// (hotdry.top, "量化策略"), fused SwiGLU and the fused combine with the residual and
// the sigmoid-gated shared expert (hotdry.top, "Metal GPU管线").  How it is computed
// (one persistent kernel, grid-wide flag exchanges, HBM-resident records) is this
// library's own design for B200.
#pragma once

#include "fmoe_device.cuh"
#include "fmoe_topk.cuh"

namespace fmoe {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxK = 32;
constexpr int kNumBars = 96;
constexpr int kMaxRoundItems = kNumBars / 2;
constexpr int kMaxDownBlock = 2 * kWarps;  // output rows per down item (two per warp)
constexpr int kMaxChunks = 8;              // gate/up chunks per round
constexpr int kMaxExperts = 2048;          // routed experts a layer may have
constexpr int kMaxSplits = 4;              // router column splits
constexpr int kMaxGrid = 256;              // blocks a launch may have (flag words reserved)
constexpr int kFlagStride = 8;             // uint32 per flag (one 32-byte sector each)

enum Mode : int { MODE_ROUTE = 1, MODE_EXPERTS = 2, MODE_FULL = 3 };

struct Params {
  int H, I, E, K, has_shared, has_rbias;
  int nq;  // router column splits (router unit = one row x H/nq columns)
  int rp;  // gate/up row pairs per copy item
  int db;  // output rows per down item (<= kMaxDownBlock)
  int T, mode;
  const uint8_t* experts;
  unsigned long long rec_bytes, o_gu_sb, o_d_q, o_d_sb;
  int qh, qi, sh, si;  // bytes: code row over H, code row over I, sb row over H, sb row over I
  const float* router;
  const float* rbias;
  const float* sgate;
  const uint16_t* x;
  const uint16_t* resid;
  uint16_t* y;
  int32_t* idx_out;
  float* w_out;
  float* sig_out;
  const int32_t* idx_in;
  const float* w_in;
  const float* sig_in;
  uint32_t* err;
  uint32_t* tokens;  // tokens this workspace has seen (tag base)
  uint32_t* rflags;  // [kMaxGrid * kFlagStride] per-block "router partials written" tags
  uint32_t* hflags;  // [kMaxGrid * kFlagStride] per-block "h rows written" tags
  double* lpart;     // [2][(E+1)*nq] router partials
  float* hbuf;       // [2][(K+1)*I]  h values
  int norm;         // 1: the input is a pre-norm block's h (the NORM kernel variant)
  double norm_eps;
  int staging_bytes;
  unsigned long long wait_ns;
  int hold_cta;
  unsigned long long* timeline;  // diagnostic: [grid][16] phase timestamps of one token, or null
  int timeline_token;
};

// Rows [ra, rb) of expert slot `slot`, staged at `off`, copy items from `first`.
struct GuChunk {
  int slot, ra, rb;
  uint32_t off, first;
};

// The block's share of a token's expert work (the same for every token of a launch):
// routed gate/up chunks (item numbers relative to the token's first routed item), the
// down rows, and where the down rows and h are staged.
struct ExpertPlan {
  GuChunk ch[kMaxChunks];
  int nc, gitems, ndown, j0, j1, v0, v1, prefetch;
  uint32_t doff, hoff;
};

// Shared-memory header (activations and the staging area follow it).
struct alignas(128) SmemHeader {
  uint64_t bars[kNumBars];
  double red[kWarps];    // per-warp partial sums (RMS normalisation)
  double selog[kMaxK + 1];  // logits of the selection in rank order; slot K: shared gate
  int sel[kMaxK + 1];    // expert of each slot (slot K = shared expert)
  float wsl[kMaxK + 1];  // weight of each slot (w_k; slot K = sigma)
  int abort_flag;
  int skip_token;
  uint32_t tok_base;
  ExpertPlan plan;
};

__host__ __device__ constexpr uint32_t r16(uint32_t n) { return (n + 15u) & ~15u; }
__host__ __device__ constexpr uint32_t r128(uint32_t n) { return (n + 127u) & ~127u; }

// Byte sizes of staged data; used by the kernel and by the host-side plan check.
struct Geometry {
  int H, I, qh, qi, sh, si, rp, db, nslots, cols;
  // gate/up chunk of n row pairs: code rows, then the 16-byte cover of their sb rows
  __host__ __device__ uint32_t gu_q(int n) const { return r16(static_cast<uint32_t>(n) * 2u * qh); }
  __host__ __device__ uint32_t gu_bytes(int n) const {
    return gu_q(n) + r16(static_cast<uint32_t>(n) * 2u * sh) + 16u;
  }
  __host__ __device__ int gu_items(int n) const { return (n + rp - 1) / rp; }
  // down item of n output rows: per slot, code rows then the cover of their sb rows
  __host__ __device__ uint32_t dn_q(int n) const { return r16(static_cast<uint32_t>(n) * qi); }
  __host__ __device__ uint32_t dn_slot(int n) const { return dn_q(n) + r16(static_cast<uint32_t>(n) * si) + 16u; }
  __host__ __device__ uint32_t dn_item(int n) const { return static_cast<uint32_t>(nslots) * dn_slot(n); }
  // bytes of down items for output rows [j0, j1)
  __host__ __device__ uint32_t dn_total(int rows) const {
    if (rows <= 0) return 0u;
    const int full = rows / db, rest = rows % db;
    return static_cast<uint32_t>(full) * dn_item(db) + (rest ? dn_item(rest) : 0u);
  }
  // floats of the lane-interleaved layout of an n-vector (whole groups of 32 chunks)
  __host__ __device__ uint32_t padded(int n) const {
    return static_cast<uint32_t>((n / cols + 31) / 32) * 32u * static_cast<uint32_t>(cols);
  }
  __host__ __device__ uint32_t h_bytes() const {
    return r128(static_cast<uint32_t>(nslots) * padded(I) * 4u + static_cast<uint32_t>(nslots) * (I / cols) * 8u);
  }
  // header + activations + per-chunk (sum, rescale) pairs, before the staging area
  __host__ __device__ uint32_t fixed_bytes(uint32_t header) const {
    return r128(header + padded(H) * 4u + static_cast<uint32_t>(H / cols) * 8u);
  }
  __host__ __device__ uint32_t router_item() const { return static_cast<uint32_t>(H) * 4u; }
};


// NORM: the input is a pre-norm block's h, RMS-normalised while it is staged.
template <int BITS, bool NORM>
struct LayerKernel {
  using C = Chunk<BITS>;

  const Params& p;
  Geometry g;
  SmemHeader* hdr;
  float* xs;       // pre-scaled, lane-interleaved activations [padded H]
  float2* xsum;    // per chunk: (sum of the unscaled activations, rescale 2^(149 - P)) [H / kCols]
  uint8_t* stage;  // staging area
  uint32_t cap;    // staging bytes
  uint32_t nitem;  // items issued so far (same value in every thread)
  int nslots;
  int tok_;

  __device__ LayerKernel(const Params& pp, uint8_t* smem) : p(pp) {
    nslots = p.K + (p.has_shared ? 1 : 0);
    g = Geometry{p.H, p.I, p.qh, p.qi, p.sh, p.si, p.rp, p.db, nslots, C::kCols};
    hdr = reinterpret_cast<SmemHeader*>(smem);
    xs = reinterpret_cast<float*>(smem + sizeof(SmemHeader));
    xsum = reinterpret_cast<float2*>(xs + g.padded(p.H));
    stage = smem + g.fixed_bytes(sizeof(SmemHeader));
    cap = static_cast<uint32_t>(p.staging_bytes);
    nitem = 0;
    tok_ = -1;
  }

  __device__ __forceinline__ uint64_t* bar_of(uint32_t n) const { return &hdr->bars[n % kNumBars]; }
  __device__ __forceinline__ uint32_t parity_of(uint32_t n) const { return (n / kNumBars) & 1u; }

  __device__ __forceinline__ bool wait_item(uint32_t n) {
    return mbar_wait_bounded(bar_of(n), parity_of(n), p.wait_ns, p.err);
  }

  __device__ __forceinline__ const uint8_t* record(int expert) const {
    return p.experts + static_cast<unsigned long long>(expert) * p.rec_bytes;
  }

  // diagnostic timestamps (token 0 only; off unless a timeline buffer is attached)
  __device__ __forceinline__ void mark(int i) const {
    if (p.timeline != nullptr && tok_ == p.timeline_token && threadIdx.x == 0) {
      p.timeline[static_cast<size_t>(blockIdx.x) * 32 + i] = global_timer_ns();
      p.timeline[static_cast<size_t>(blockIdx.x) * 32 + 16 + i] = static_cast<unsigned long long>(clock64());
    }
  }

  // Waits (bounded) for every copy this block may still have in flight.
  __device__ void drain() {
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t lo = nitem > kNumBars ? nitem - kNumBars : 0;
      for (uint32_t n = lo; n < nitem; ++n) mbar_wait_bounded(bar_of(n), parity_of(n), p.wait_ns, p.err);
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------- exchanges
  // Values every block needs from all others (router partials, h rows) are written
  // with plain stores; then the block publishes the token's tag in its own flag word
  // with a release store.  A reader's warp 0 polls the grid's flags (each lane a few,
  // all of a lane's loads in flight together, relaxed loads, bounded), fences, and
  // the block then reads the values once from L2.  Buffers alternate by token parity;
  // no block can run two tokens ahead of another because each token needs every
  // block's values.
  uint32_t tbase_;
  __device__ __forceinline__ uint32_t tag32(int t) const {
    return (tbase_ + static_cast<uint32_t>(t)) % 0xFFFFFFFFu + 1u;
  }

  __device__ __forceinline__ void publish(uint32_t* flags, int t) {
    __syncthreads();
    if (threadIdx.x == 0) st_release_u32(flags + blockIdx.x * kFlagStride, tag32(t));
  }

  __device__ bool wait_all(const uint32_t* flags, int t) {
    int fail = 0;
    if (threadIdx.x < 32) {
      const int G = gridDim.x, lane = threadIdx.x;
      const uint32_t want = tag32(t);
      constexpr int NF = kMaxGrid / 32;
      uint32_t got[NF];
#pragma unroll
      for (int i = 0; i < NF; ++i) {
        const int b = lane + 32 * i;
        got[i] = b < G ? ld_relaxed_u32(flags + b * kFlagStride) : want;
      }
      uint64_t t0 = 0;
      for (int it = 0;; ++it) {
        bool all = true;
#pragma unroll
        for (int i = 0; i < NF; ++i) all &= got[i] == want;
        if (__all_sync(0xffffffffu, all)) break;
        if ((it & 15) == 15) {
          if (t0 == 0) t0 = global_timer_ns();
          const bool bad =
              (ld_relaxed_u32(p.err) & FMOE_DEVERR_BARRIER_TIMEOUT) || global_timer_ns() - t0 > p.wait_ns;
          if (__any_sync(0xffffffffu, bad)) {
            if (lane == 0) atomicOr(p.err, FMOE_DEVERR_BARRIER_TIMEOUT);
            fail = 1;
            break;
          }
        }
        __nanosleep(32);
#pragma unroll
        for (int i = 0; i < NF; ++i) {
          const int b = lane + 32 * i;
          if (got[i] != want) got[i] = ld_relaxed_u32(flags + b * kFlagStride);
        }
      }
      __threadfence();
    }
    return __syncthreads_or(fail) == 0;
  }

  // ---------------------------------------------------------------- activations
  // Column group q = columns [4q, 4q+4).  Two passes, all loads in flight together:
  //  natural (thread -> consecutive groups): chunk sums by shuffles over the kCols/4
  //    threads of a chunk, and for x the doubles of the router (split in two double2
  //    arrays so the router's loads are conflict-free);
  //  transposed (thread -> consecutive float4 slots of the lane-interleaved layout):
  //    pre-scaled floats, conflict-free 16-byte stores.
  __device__ __forceinline__ float4 bf16x4(uint2 u) const {
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xFFFF0000u));
  }

  // RMS denominator sqrt(mean(h^2) + eps) of a pre-norm block's input, in double
  // (squares of bf16 values are exact).  Every block forms the same partial sums in
  // the same order, so every block derives the same normalised vector.
  __device__ double rms_of(const uint16_t* ht) {
    const uint2* src = reinterpret_cast<const uint2*>(ht);
    double s = 0.0;
    for (int q = threadIdx.x; q < p.H / 4; q += kThreads) {
      const float4 v = bf16x4(src[q]);
      s = fma(static_cast<double>(v.x), static_cast<double>(v.x), s);
      s = fma(static_cast<double>(v.y), static_cast<double>(v.y), s);
      s = fma(static_cast<double>(v.z), static_cast<double>(v.z), s);
      s = fma(static_cast<double>(v.w), static_cast<double>(v.w), s);
    }
    s = warp_sum_d(s);
    if ((threadIdx.x & 31) == 0) hdr->red[threadIdx.x >> 5] = s;
    __syncthreads();
    double tot = 0.0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += hdr->red[w];
    return sqrt(tot / p.H + p.norm_eps);
  }

  // n = bf16(h / r) of four packed bf16 values, divided and rounded once in double
  __device__ __forceinline__ uint2 normed(uint2 u, double r) const {
    const float4 v = bf16x4(u);
    const uint32_t a = f64_to_bf16(static_cast<double>(v.x) / r), b = f64_to_bf16(static_cast<double>(v.y) / r);
    const uint32_t c = f64_to_bf16(static_cast<double>(v.z) / r), d = f64_to_bf16(static_cast<double>(v.w) / r);
    return make_uint2(a | (b << 16), c | (d << 16));
  }

  __device__ void stage_x(const uint16_t* xt, double2* xa, double2* xb) {
    constexpr int TPC = C::kCols / 4;
    const int n4 = p.H / 4;
    const uint2* src = reinterpret_cast<const uint2*>(xt);
    const double rn = NORM ? rms_of(xt) : 1.0;
    for (int base = 0; base < n4; base += 2 * kThreads) {  // block-uniform trip count
      uint2 nat[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int q = base + static_cast<int>(threadIdx.x) + k * kThreads;
        nat[k] = q < n4 ? src[q] : make_uint2(0, 0);
      }
      if (NORM) {
#pragma unroll
        for (int k = 0; k < 2; ++k) nat[k] = normed(nat[k], rn);
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int q = base + static_cast<int>(threadIdx.x) + k * kThreads;
        const float4 v = bf16x4(nat[k]);
        float sum = (v.x + v.y) + (v.z + v.w);
        uint32_t mx = max_abs_bits(v);
#pragma unroll
        for (int o = 1; o < TPC; o <<= 1) {
          sum += __shfl_xor_sync(0xffffffffu, sum, o);
          mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (q < n4) {
          if (xa) {
            xa[q] = make_double2(v.x, v.y);
            xb[q] = make_double2(v.z, v.w);
          }
          const int c0 = 4 * q, pre = chunk_pre(mx);
          xs[phys(c0 + 0)] = v.x * prescale_factor(pre, C::shift_of(c0 + 0));
          xs[phys(c0 + 1)] = v.y * prescale_factor(pre, C::shift_of(c0 + 1));
          xs[phys(c0 + 2)] = v.z * prescale_factor(pre, C::shift_of(c0 + 2));
          xs[phys(c0 + 3)] = v.w * prescale_factor(pre, C::shift_of(c0 + 3));
          if (q % TPC == 0) xsum[q / TPC] = make_float2(sum, chunk_unscale(pre));
        }
      }
    }
  }

  // h of every slot (fp32, written by other blocks, read from L2 once every block
  // has published): coalesced 16-byte loads (thread -> 4 consecutive columns), all of
  // a thread's loads in flight together; chunk sums by shuffles over the kCols/4
  // threads of a chunk; pre-scaled values scattered into the interleaved layout.
  __device__ void stage_h(const float* hb, float* hs, uint32_t hstride, float2* hsum) {
    constexpr int TPC = C::kCols / 4;
    const int per_slot = p.I / 4, nch = p.I / C::kCols;
    const int n4 = nslots * per_slot;
    const float4* src = reinterpret_cast<const float4*>(hb);
    for (int base = 0; base < n4; base += 4 * kThreads) {
      float4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = base + static_cast<int>(threadIdx.x) + k * kThreads;
        v[k] = q < n4 ? __ldcg(src + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = base + static_cast<int>(threadIdx.x) + k * kThreads;
        float sum = (v[k].x + v[k].y) + (v[k].z + v[k].w);
        uint32_t mx = max_abs_bits(v[k]);
#pragma unroll
        for (int o = 1; o < TPC; o <<= 1) {
          sum += __shfl_xor_sync(0xffffffffu, sum, o);
          mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (q < n4) {
          const int slot = q / per_slot, c0 = (q % per_slot) * 4, pre = chunk_pre(mx);
          float* d = hs + static_cast<size_t>(slot) * hstride;
          d[phys(c0 + 0)] = v[k].x * prescale_factor(pre, C::shift_of(c0 + 0));
          d[phys(c0 + 1)] = v[k].y * prescale_factor(pre, C::shift_of(c0 + 1));
          d[phys(c0 + 2)] = v[k].z * prescale_factor(pre, C::shift_of(c0 + 2));
          d[phys(c0 + 3)] = v[k].w * prescale_factor(pre, C::shift_of(c0 + 3));
          if (q % TPC == 0) hsum[slot * nch + c0 / C::kCols] = make_float2(sum, chunk_unscale(pre));
        }
      }
      if (base == 0) mark(14);
    }
    mark(15);
  }

  __device__ __forceinline__ static int phys(int c) { return C::phys(c); }

  // ---------------------------------------------------------------- dot products
  // Lane partial of sum_c W[r][c] v[c] over the lane's chunks, for one or two rows
  // sharing the activation loads (W = scale*code + bias; v pre-scaled, interleaved).
  // The lane takes chunks m0, m0 + mstep, ... (by default its lane index, stride 32).
  template <bool TWO>
  __device__ __forceinline__ void dotn(const uint8_t* q0, const uint32_t* s0, const uint8_t* q1,
                                       const uint32_t* s1, const float* vs, const float2* vsum, int nch, float& r0,
                                       float& r1, int m0 = -1, int mstep = 32) const {
    const int lane = threadIdx.x & 31;
#pragma unroll 2
    for (int m = m0 < 0 ? lane : m0; m < nch; m += mstep) {
      const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(q0 + 16 * m);
      ulonglong2 b = make_ulonglong2(0ull, 0ull);
      if (TWO) b = *reinterpret_cast<const ulonglong2*>(q1 + 16 * m);
      const ulonglong2* xv0 = C::f4(vs, m, 0);
      const ulonglong2* xv1 = C::f4(vs, m, C::kF4PerPair);
      unsigned long long a0 = 0ull, a1 = 0ull, b0 = 0ull, b1 = 0ull;
      C::template word_pair2<TWO>(a.x, b.x, xv0, a0, b0);
      C::template word_pair2<TWO>(a.y, b.y, xv1, a1, b1);
      const float2 vm = vsum[m];  // (sum of the chunk's activations, rescale of its products)
      const uint32_t sa = s0[C::sb_index(m)];
      r0 = fmaf(sb_scale(sa), (pair_sum(a0) + pair_sum(a1)) * vm.y, r0);
      r0 = fmaf(sb_bias(sa), vm.x, r0);
      if (TWO) {
        const uint32_t sbv = s1[C::sb_index(m)];
        r1 = fmaf(sb_scale(sbv), (pair_sum(b0) + pair_sum(b1)) * vm.y, r1);
        r1 = fmaf(sb_bias(sbv), vm.x, r1);
      }
    }
  }

  // ---------------------------------------------------------------- gate/up chunks
  // Item i of chunk c (row pairs [ra + i*rp, ...)); the chunk's (scale,bias) cover
  // rides on item 0.  Called by one lane per item.
  __device__ void issue_gu_item(const GuChunk& c, int i) {
    const uint8_t* rec = record(hdr->sel[c.slot]);
    const int n = c.rb - c.ra;
    const int a = c.ra + i * p.rp, b = min(c.rb, a + p.rp);
    const uint32_t qb = static_cast<uint32_t>(b - a) * 2u * p.qh;
    uint32_t sbb = 0;
    unsigned long long sb_a = 0;
    if (i == 0) {
      const unsigned long long sb_start = p.o_gu_sb + static_cast<unsigned long long>(c.ra) * 2u * p.sh;
      sb_a = sb_start & ~15ull;
      const unsigned long long sb_end =
          (sb_start + static_cast<unsigned long long>(n) * 2u * p.sh + 15ull) & ~15ull;
      sbb = static_cast<uint32_t>(sb_end - sb_a);
    }
    uint64_t* bar = bar_of(c.first + i);
    mbar_arrive_expect_tx(bar, qb + sbb);
    bulk_g2s(stage + c.off + static_cast<uint32_t>(a - c.ra) * 2u * p.qh,
             rec + static_cast<unsigned long long>(a) * 2u * p.qh, qb, bar);
    if (i == 0) bulk_g2s(stage + c.off + g.gu_q(n), rec + sb_a, sbb, bar);
  }

  // Warp 0: issue every item of `nc` chunks, one lane per item.
  // Thread 0: every item of `nc` chunks, one after another in the order the warps
  // consume them (copies requested in one instruction by many lanes are served
  // interleaved and all complete late; requested in sequence, the first ones land
  // first).
  __device__ void issue_gu(const GuChunk* ch, int nc) {
    if (threadIdx.x != 0) return;
    fence_proxy_async_smem();
    for (int k = 0; k < nc; ++k) {
      const int items = g.gu_items(ch[k].rb - ch[k].ra);
      for (int i = 0; i < items; ++i) issue_gu_item(ch[k], i);
    }
  }

  // h of row pair r of the chunk -> hbuf[buf][slot][r]  (one warp)
  __device__ bool gu_unit(const GuChunk& c, int r, int buf) {
    const int n = c.rb - c.ra, i = r - c.ra;
    if (!wait_item(c.first + i / p.rp)) return false;
    if (i >= p.rp && !wait_item(c.first)) return false;  // (scale,bias) rows ride on item 0
    const uint8_t* qg = stage + c.off + static_cast<uint32_t>(i) * 2u * p.qh;
    const uint8_t* qu = qg + p.qh;
    const uint32_t lead =
        static_cast<uint32_t>((p.o_gu_sb + static_cast<unsigned long long>(c.ra) * 2u * p.sh) & 15ull);
    const uint32_t* sg = reinterpret_cast<const uint32_t*>(stage + c.off + g.gu_q(n) + lead) + i * 2 * (p.sh / 4);
    const uint32_t* su = sg + p.sh / 4;
    float gv = 0.f, uv = 0.f;
    dotn<true>(qg, sg, qu, su, xs, xsum, p.H / C::kCols, gv, uv);
    gv = warp_sum(gv);
    uv = warp_sum(uv);
    if ((threadIdx.x & 31) == 0) {
      const float hval = (gv / (1.0f + expf(-gv))) * uv;
      p.hbuf[static_cast<size_t>(buf) * (p.K + 1) * p.I + static_cast<size_t>(c.slot) * p.I + r] = hval;
    }
    return true;
  }

  // Consume every row pair of `nc` chunks, spread over warps w0 .. kWarps-1 (unit u ->
  // warp w0 + u % (kWarps - w0)); w0 = 1 keeps warp 0, which issues the copies and
  // computes the routing weights meanwhile, out of the routed rows.
  __device__ void gu_consume(const GuChunk* ch, int nc, int buf, int w0 = 0) {
    const int warp = threadIdx.x >> 5;
    if (warp < w0) return;
    const int nw = kWarps - w0;
    int base = 0;
    for (int k = 0; k < nc; ++k) {
      const int n = ch[k].rb - ch[k].ra;
      int first = (warp - w0 - base) % nw;
      if (first < 0) first += nw;
      for (int i = first; i < n; i += nw) {
        if (!gu_unit(ch[k], ch[k].ra + i, buf)) {
          hdr->abort_flag = 1;
          return;
        }
      }
      base += n;
    }
  }

  // Gate/up of routed units [v0, v1) (unit = slot*I + r) in rounds that fit the
  // whole staging area (used when the block's share does not fit at once).
  __device__ bool gu_rounds(int v0, int v1, int buf) {
    GuChunk ch[kMaxChunks];
    int nc = 0, items = 0;
    uint32_t used = 0;
    const uint32_t per_row = 2u * p.qh + 2u * p.sh;
    int v = v0;
    while (true) {
      bool flush = (v >= v1);
      int s = 0, r = 0, n = 0;
      if (!flush) {
        s = v / p.I;
        r = v % p.I;
        const int seg = min(v1 - v, p.I - r);
        const uint32_t room = cap > used + 64u ? cap - used - 64u : 0u;
        n = min(seg, static_cast<int>(room / per_row));
        while (n > 0 && g.gu_bytes(n) > cap - used) --n;
        n = min(n, (kMaxRoundItems - items) * p.rp);
        if (n <= 0 || nc == kMaxChunks) flush = true;
      }
      if (flush) {
        if (nc == 0) {  // nothing fits at all (the host plan rules this out)
          if (v >= v1) return true;
          hdr->abort_flag = 1;
          return false;
        }
        issue_gu(ch, nc);
        nitem += static_cast<uint32_t>(items);
        gu_consume(ch, nc, buf);
        __syncthreads();
        if (hdr->abort_flag) return false;
        nc = 0;
        items = 0;
        used = 0;
        if (v >= v1) return true;
        continue;
      }
      ch[nc] = GuChunk{s, r, r + n, used, nitem + static_cast<uint32_t>(items)};
      ++nc;
      items += g.gu_items(n);
      used = r128(used + g.gu_bytes(n));
      v += n;
    }
  }

  // ---------------------------------------------------------------- down items
  __device__ void down_range(int& j0, int& j1) const {
    const int G = gridDim.x, b = blockIdx.x;
    j0 = static_cast<int>(static_cast<long long>(p.H) * b / G);
    j1 = static_cast<int>(static_cast<long long>(p.H) * (b + 1) / G);
  }

  __device__ void issue_down(uint32_t item, uint32_t off, int ja, int n) {
    const uint32_t qb = static_cast<uint32_t>(n) * p.qi;
    const unsigned long long sb_start = p.o_d_sb + static_cast<unsigned long long>(ja) * p.si;
    const unsigned long long sb_a = sb_start & ~15ull;
    const unsigned long long sb_end = (sb_start + static_cast<unsigned long long>(n) * p.si + 15ull) & ~15ull;
    const uint32_t sbb = static_cast<uint32_t>(sb_end - sb_a);
    uint64_t* bar = bar_of(item);
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nslots) * (qb + sbb));
    for (int s = 0; s < nslots; ++s) {
      const uint8_t* rec = record(hdr->sel[s]);
      uint8_t* dst = stage + off + s * g.dn_slot(n);
      bulk_g2s(dst, rec + p.o_d_q + static_cast<unsigned long long>(ja) * p.qi, qb, bar);
      bulk_g2s(dst + g.dn_q(n), rec + sb_a, sbb, bar);
    }
  }

  // Warp 0: items [ka, kb) of the block's rows [j0, j1) from staging offset `base`.
  __device__ void issue_down_items(int j0, int j1, int ka, int kb, uint32_t first, uint32_t base) {
    if (threadIdx.x != 0) return;
    fence_proxy_async_smem();
    for (int k = ka; k < kb; ++k) {
      const int ja = j0 + k * p.db, n = min(j1, ja + p.db) - ja;
      issue_down(first + (k - ka), base + (k - ka) * g.dn_item(p.db), ja, n);
    }
  }

  // Consume a down item (rows [ja, ja+n)): y = resid + sum_s w_s o_s.  In a pre-norm
  // block (NORM) y is the residual buffer itself: the block's residual rows are loaded
  // before the dot products, so that the late loads do not queue behind other warps'
  // stores to the same sectors.
  __device__ bool down_item(uint32_t item, uint32_t off, int ja, int n, const float* hs, const float2* hsum,
                            const uint16_t* resid_t, uint16_t* y_t) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ia = warp, ib = warp + kWarps;
    if (ia >= n) return true;
    const bool two = ib < n;
    float ra = 0.f, rb = 0.f;
    if (NORM && lane == 0) {
      ra = bf16_to_f32(resid_t[ja + ia]);
      if (two) rb = bf16_to_f32(resid_t[ja + ib]);
    }
    if (!wait_item(item)) {
      hdr->abort_flag = 1;
      return false;
    }
    const uint32_t lead = static_cast<uint32_t>((p.o_d_sb + static_cast<unsigned long long>(ja) * p.si) & 15ull);
    const int nch = p.I / C::kCols;
    float pa = 0.f, pb = 0.f;
    if constexpr (BITS == 2) {
      if (nch <= 16) {
        // a row of at most 16 chunks would leave half the lanes idle: each half-warp
        // takes every other slot (lanes 0-15 the even slots, 16-31 the odd ones)
        const int half = lane >> 4;
        for (int s0 = 0; s0 < nslots; s0 += 2) {
          const int s = s0 + half;
          float oa = 0.f, ob = 0.f;
          if (s < nslots) {
            const uint8_t* blk = stage + off + s * g.dn_slot(n);
            const uint32_t* sbase = reinterpret_cast<const uint32_t*>(blk + g.dn_q(n) + lead);
            const float* hsl = hs + static_cast<size_t>(s) * g.padded(p.I);
            const float2* hsm = hsum + static_cast<size_t>(s) * nch;
            if (two)
              dotn<true>(blk + static_cast<uint32_t>(ia) * p.qi, sbase + ia * (p.si / 4),
                         blk + static_cast<uint32_t>(ib) * p.qi, sbase + ib * (p.si / 4), hsl, hsm, nch, oa, ob,
                         lane & 15, 16);
            else
              dotn<false>(blk + static_cast<uint32_t>(ia) * p.qi, sbase + ia * (p.si / 4), nullptr, nullptr, hsl,
                          hsm, nch, oa, ob, lane & 15, 16);
            const float ws = hdr->wsl[s];
            pa = fmaf(ws, oa, pa);
            pb = fmaf(ws, ob, pb);
          }
        }
        pa = warp_sum(pa);
        pb = warp_sum(pb);
        if (lane == 0) {
          if (!NORM) {
            ra = bf16_to_f32(resid_t[ja + ia]);
            if (two) rb = bf16_to_f32(resid_t[ja + ib]);
          }
          y_t[ja + ia] = f32_to_bf16(ra + pa);
          if (two) y_t[ja + ib] = f32_to_bf16(rb + pb);
        }
        return true;
      }
    }
    for (int s = 0; s < nslots; ++s) {
      const uint8_t* blk = stage + off + s * g.dn_slot(n);
      const uint32_t* sbase = reinterpret_cast<const uint32_t*>(blk + g.dn_q(n) + lead);
      float oa = 0.f, ob = 0.f;
      const float* hsl = hs + static_cast<size_t>(s) * g.padded(p.I);
      const float2* hsm = hsum + static_cast<size_t>(s) * nch;
      if (two)
        dotn<true>(blk + static_cast<uint32_t>(ia) * p.qi, sbase + ia * (p.si / 4),
                   blk + static_cast<uint32_t>(ib) * p.qi, sbase + ib * (p.si / 4), hsl, hsm, nch, oa, ob);
      else
        dotn<false>(blk + static_cast<uint32_t>(ia) * p.qi, sbase + ia * (p.si / 4), nullptr, nullptr, hsl, hsm,
                    nch, oa, ob);
      const float ws = hdr->wsl[s];
      pa = fmaf(ws, oa, pa);
      pb = fmaf(ws, ob, pb);
    }
    pa = warp_sum(pa);
    pb = warp_sum(pb);
    if (lane == 0) {
      if (!NORM) {
        ra = bf16_to_f32(resid_t[ja + ia]);
        if (two) rb = bf16_to_f32(resid_t[ja + ib]);
      }
      y_t[ja + ia] = f32_to_bf16(ra + pa);
      if (two) y_t[ja + ib] = f32_to_bf16(rb + pb);
    }
    return true;
  }

  // ---------------------------------------------------------------- P1
  // Router units [u0, u1) over (E + has_shared) rows x nq splits (the shared gate
  // vector is the last row) staged after the router's doubles; the block's slice of
  // the shared expert's gate/up rows staged at the end of the staging area, to be
  // consumed after top-K while the routed rows are in flight.  All copies are issued
  // before the activations are staged (they do not depend on them).
  int u0_, u1_, row0_, row1_;
  uint32_t p1first_, rbase_;
  GuChunk sc_;
  bool has_sc_;

  __device__ void phase1_issue(bool route, bool shared_gu) {
    const int rows = p.E + (p.has_shared ? 1 : 0);
    const int G = gridDim.x, b = blockIdx.x;
    u0_ = u1_ = row0_ = row1_ = 0;
    if (route) {
      const long long U = static_cast<long long>(rows) * p.nq;
      u0_ = static_cast<int>(U * b / G);
      u1_ = static_cast<int>(U * (b + 1) / G);
      row0_ = u0_ / p.nq;
      row1_ = (u1_ + p.nq - 1) / p.nq;
    }
    const int hc = p.H / p.nq;
    const uint32_t rib = g.router_item();
    rbase_ = route ? r128(static_cast<uint32_t>(p.H) * 8u) : 0u;
    const int nrouter = row1_ - row0_;
    p1first_ = nitem;
    sc_ = GuChunk{p.K, 0, 0, 0, p1first_ + static_cast<uint32_t>(nrouter)};
    if (shared_gu) {
      sc_.ra = static_cast<int>(static_cast<long long>(p.I) * b / G);
      sc_.rb = static_cast<int>(static_cast<long long>(p.I) * (b + 1) / G);
    }
    has_sc_ = sc_.rb > sc_.ra;
    const int nsh = has_sc_ ? g.gu_items(sc_.rb - sc_.ra) : 0;
    if (has_sc_) sc_.off = (cap - g.gu_bytes(sc_.rb - sc_.ra)) & ~127u;
    if (threadIdx.x < 32) {
      fence_proxy_async_smem();
      for (int r = row0_ + static_cast<int>(threadIdx.x); r < row1_; r += 32) {
        const int ua = max(u0_, r * p.nq), ub = min(u1_, r * p.nq + p.nq);
        uint64_t* bar = bar_of(p1first_ + (r - row0_));
        const uint32_t bytes = static_cast<uint32_t>(ub - ua) * hc * 4u;
        const float* src = (r < p.E) ? p.router + static_cast<size_t>(r) * p.H : p.sgate;
        src += static_cast<size_t>(ua - r * p.nq) * hc;
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(stage + rbase_ + (r - row0_) * rib + static_cast<uint32_t>(ua - r * p.nq) * hc * 4u, src, bytes,
                 bar);
      }
      for (int i = static_cast<int>(threadIdx.x) - (nrouter % 32); i < nsh; i += 32)
        if (i >= 0) issue_gu_item(sc_, i);
    }
    nitem += static_cast<uint32_t>(nrouter + nsh);
  }

  // Router dot products of this block's units: fp64 sums of exact fp32 x bf16 products.
  __device__ bool phase1_consume(int buf, bool route) {
    if (route) {
      const int rows = p.E + (p.has_shared ? 1 : 0);
      const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
      const int hc = p.H / p.nq;
      const uint32_t rib = g.router_item();
      const double2* xa = reinterpret_cast<const double2*>(stage);
      const double2* xb = xa + p.H / 4;
      double* lpart = p.lpart + static_cast<size_t>(buf) * rows * p.nq;
      for (int u = u0_ + warp; u < u1_; u += kWarps) {
        const int r = u / p.nq, qq = u % p.nq;
        if (!wait_item(p1first_ + (r - row0_))) {
          hdr->abort_flag = 1;
          break;
        }
        const float4* wrow = reinterpret_cast<const float4*>(stage + rbase_ + (r - row0_) * rib) + qq * (hc / 4);
        const int k0 = qq * (hc / 4);
        double acc0 = 0.0, acc1 = 0.0;
#pragma unroll 4
        for (int k = lane; k < hc / 4; k += 32) {
          const float4 wv = wrow[k];
          const double2 a = xa[k0 + k];
          const double2 bb = xb[k0 + k];
          acc0 = fma(static_cast<double>(wv.x), a.x, acc0);
          acc1 = fma(static_cast<double>(wv.y), a.y, acc1);
          acc0 = fma(static_cast<double>(wv.z), bb.x, acc0);
          acc1 = fma(static_cast<double>(wv.w), bb.y, acc1);
        }
        const double acc = warp_sum_d(acc0 + acc1);
        if (lane == 0) lpart[u] = acc;
      }
    }
    __syncthreads();
    return hdr->abort_flag == 0;
  }

  // ---------------------------------------------------------------- routing
  // Every block: logits (all threads, one per expert), top-K by ranks in two levels
  // -- within groups of 32 experts, then among the groups' K best -- ordered by logit
  // descending with ties to the lower index (compared through the order-preserving
  // 64-bit key of each fp64 logit), then the renormalised softmax weights of the K
  // and the shared sigmoid gate.
  __device__ void topk(int buf, int t) {
    mark(3);
    if (!wait_all(p.rflags, t)) {
      if (threadIdx.x == 0) hdr->abort_flag = 1;
      __syncthreads();
      return;
    }
    mark(10);
    const int rows = p.E + (p.has_shared ? 1 : 0);
    const int lane = threadIdx.x & 31;
    const int ngroups = (p.E + 31) >> 5;
    unsigned long long* ckey = reinterpret_cast<unsigned long long*>(stage);
    double* cval = reinterpret_cast<double*>(stage + r128(static_cast<uint32_t>(ngroups * p.K) * 8u));
    int* cidx = reinterpret_cast<int*>(stage + 2 * r128(static_cast<uint32_t>(ngroups * p.K) * 8u));
    const double* lpart = p.lpart + static_cast<size_t>(buf) * rows * p.nq;
    for (int e0 = 0; e0 < rows; e0 += kThreads) {  // block-uniform trip count
      const int e = e0 + static_cast<int>(threadIdx.x);
      double l = 0.0;
      if (e < rows) {
        l = router_logit(lpart + static_cast<size_t>(e) * p.nq, p.nq);
        if (e < p.E && p.has_rbias) l += static_cast<double>(__ldg(p.rbias + e));
        if (e == p.E && p.has_shared) hdr->selog[p.K] = l;
      }
      const unsigned long long key = e < p.E ? dkey(l) : 0ull;
      if (e - static_cast<int>(lane) < p.E) {  // warp-uniform: the group's first expert exists
        int rank = 0;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
          const unsigned long long kj = __shfl_sync(0xffffffffu, key, j);
          rank += static_cast<int>(kj > key) | (static_cast<int>(kj == key) & static_cast<int>(j < lane));
        }
        if (rank < p.K) {
          const int slot = (e >> 5) * p.K + rank;
          ckey[slot] = key;
          cval[slot] = l;
          cidx[slot] = e < p.E ? e : 0x7fffffff;
        }
      }
    }
    __syncthreads();
    mark(11);
    constexpr int kStripe = 8;
    const int ncand = ngroups * p.K;
    for (int base = 0; base < ncand * kStripe; base += kThreads) {  // block-uniform trip count
      const int i = base + static_cast<int>(threadIdx.x);
      const int c = i / kStripe, part = i % kStripe;
      unsigned long long kc = 0;
      int ic = 0, rank = 0;
      if (c < ncand) {
        kc = ckey[c];
        ic = cidx[c];
        for (int j = part; j < ncand; j += kStripe) {
          const unsigned long long kj = ckey[j];
          const int ij = cidx[j];
          rank += static_cast<int>(kj > kc) | (static_cast<int>(kj == kc) & static_cast<int>(ij < ic));
        }
      }
#pragma unroll
      for (int o = 1; o < kStripe; o <<= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
      if (c < ncand && part == 0 && kc != 0 && rank < p.K) {
        hdr->sel[rank] = ic;
        hdr->selog[rank] = cval[c];
      }
    }
    __syncthreads();
    mark(12);
  }

  // Warp 0: the renormalised softmax weights of the selection and the shared sigmoid
  // gate (needed only by the combine, so computed while the selected rows fly).
  __device__ void route_weights(int t) {
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const double wk = topk_weight_sorted(hdr->selog, p.K, lane);
    if (lane < p.K) {
      hdr->wsl[lane] = static_cast<float>(wk);
      if (blockIdx.x == 0 && p.idx_out) {
        p.idx_out[static_cast<size_t>(t) * p.K + lane] = hdr->sel[lane];
        p.w_out[static_cast<size_t>(t) * p.K + lane] = static_cast<float>(wk);
      }
    }
    if (lane == 0 && p.has_shared) {
      const double sig = 1.0 / (1.0 + exp(-hdr->selog[p.K]));
      hdr->wsl[p.K] = static_cast<float>(sig);
      if (blockIdx.x == 0 && p.sig_out) p.sig_out[t] = static_cast<float>(sig);
    }
  }

  // Routing given by the caller (expert-forward entry point).
  __device__ void given_routing(int t) {
    if (threadIdx.x == 0) {
      int bad = 0;
      for (int k = 0; k < p.K; ++k) {
        const int e = p.idx_in[static_cast<size_t>(t) * p.K + k];
        if (e < 0 || e >= p.E) bad = 1;
        hdr->sel[k] = e;
        hdr->wsl[k] = p.w_in[static_cast<size_t>(t) * p.K + k];
      }
      if (p.has_shared) hdr->wsl[p.K] = p.sig_in[t];
      hdr->skip_token = bad;
      if (bad && blockIdx.x == 0) atomicOr(p.err, FMOE_DEVERR_BAD_EXPERT);
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------- P2 + P3
  // The block's expert work plan: the same for every token, computed once per launch.
  __device__ void plan_experts() {
    ExpertPlan& pl = hdr->plan;
    const int G = gridDim.x, b = blockIdx.x;
    pl.v0 = static_cast<int>(static_cast<long long>(p.K) * p.I * b / G);
    pl.v1 = static_cast<int>(static_cast<long long>(p.K) * p.I * (b + 1) / G);
    down_range(pl.j0, pl.j1);
    pl.ndown = (pl.j1 - pl.j0 + p.db - 1) / p.db;
    // routed gate/up chunks from offset 0, down items behind them, h at offset 0 (the
    // whole staging area is free: the shared expert's rows are consumed before top-K)
    int nc = 0, gitems = 0;
    uint32_t gtotal = 0;
    int vend = pl.v0;
    while (vend < pl.v1 && nc < kMaxChunks) {
      const int s = vend / p.I, r = vend % p.I, n = min(pl.v1 - vend, p.I - r);
      pl.ch[nc++] = GuChunk{s, r, r + n, gtotal, static_cast<uint32_t>(gitems)};
      gitems += g.gu_items(n);
      gtotal = r128(gtotal + g.gu_bytes(n));
      vend += n;
    }
    pl.nc = nc;
    pl.gitems = gitems;
    pl.doff = gtotal;
    const uint32_t dtotal = g.dn_total(pl.j1 - pl.j0);
    pl.hoff = g.h_bytes() <= pl.doff ? 0u : r128(pl.doff + dtotal);
    pl.prefetch = (vend >= pl.v1) && (pl.doff + dtotal <= cap) && (pl.hoff + g.h_bytes() <= cap) &&
                  (gitems + pl.ndown <= kMaxRoundItems);
  }

  __device__ bool experts(int buf, bool route, const uint16_t* resid_t, uint16_t* y_t) {
    const ExpertPlan& pl = hdr->plan;
    const int j0 = pl.j0, j1 = pl.j1, ndown = pl.ndown;
    const bool prefetch = pl.prefetch != 0;
    const uint32_t doff = pl.doff, hoff = pl.hoff;
    const uint32_t down_first = nitem + static_cast<uint32_t>(pl.gitems);
    if (prefetch) {
      GuChunk ch[kMaxChunks];
      for (int k = 0; k < pl.nc; ++k) {
        ch[k] = pl.ch[k];
        ch[k].first += nitem;
      }
      issue_gu(ch, pl.nc);
      nitem += static_cast<uint32_t>(pl.gitems + ndown);
      if (route) route_weights(tok_);
      // the down rows are requested once the first half of the gate/up rows has
      // landed (thread 0 consumes none of them): requested together, both streams are
      // served interleaved and the gate/up rows complete late, while the down rows are
      // needed only after the h exchange.  The copies are issued whatever the wait
      // returns.
      if (threadIdx.x == 0) {
        if (pl.gitems > 0) (void)wait_item(down_first - static_cast<uint32_t>(pl.gitems - (pl.gitems - 1) / 2));
        issue_down_items(j0, j1, 0, ndown, down_first, doff);
      }
      gu_consume(ch, pl.nc, buf, 1);
      __syncthreads();
      if (hdr->abort_flag) return false;
    } else {
      if (route) route_weights(tok_);
      if (!gu_rounds(pl.v0, pl.v1, buf)) return false;
    }
    publish(p.hflags, tok_);
    mark(5);
    // ---- P3: stage h of every slot, then the down rows
    const uint32_t hbase = prefetch ? hoff : 0u;
    float* hs = reinterpret_cast<float*>(stage + hbase);
    const uint32_t hstride = g.padded(p.I);
    float2* hsum = reinterpret_cast<float2*>(hs + static_cast<size_t>(nslots) * hstride);
    if (!wait_all(p.hflags, tok_)) {
      if (threadIdx.x == 0) hdr->abort_flag = 1;
      __syncthreads();
      return false;
    }
    mark(6);
    stage_h(p.hbuf + static_cast<size_t>(buf) * (p.K + 1) * p.I, hs, hstride, hsum);
    __syncthreads();
    mark(7);
    if (prefetch) {
      for (int k = 0; k < ndown; ++k) {
        const int ja = j0 + k * p.db, n = min(j1, ja + p.db) - ja;
        if (!down_item(down_first + k, doff + k * g.dn_item(p.db), ja, n, hs, hsum, resid_t, y_t)) break;
      }
      __syncthreads();
      mark(8);
    } else {
      const uint32_t dbase = g.h_bytes();
      const int per_round = max(1, min(static_cast<int>((cap - dbase) / g.dn_item(p.db)), kMaxRoundItems));
      for (int ka = 0; ka < ndown; ka += per_round) {
        const int kb = min(ndown, ka + per_round);
        const uint32_t first = nitem;
        issue_down_items(j0, j1, ka, kb, first, dbase);
        nitem += static_cast<uint32_t>(kb - ka);
        for (int k = ka; k < kb; ++k) {
          const int ja = j0 + k * p.db, n = min(j1, ja + p.db) - ja;
          if (!down_item(first + (k - ka), dbase + (k - ka) * g.dn_item(p.db), ja, n, hs, hsum, resid_t, y_t))
            break;
        }
        __syncthreads();
        if (hdr->abort_flag) break;
      }
    }
    return hdr->abort_flag == 0;
  }

  // ---------------------------------------------------------------- driver
  __device__ void run() {
    if (threadIdx.x < 32) {  // warp 0: barriers; warp 1 meanwhile: the expert plan
      for (int i = static_cast<int>(threadIdx.x); i < kNumBars; i += 32) mbar_init(&hdr->bars[i], 1);
      mbar_init_fence();
      if (threadIdx.x == 0) {
        hdr->abort_flag = 0;
        hdr->skip_token = 0;
        hdr->sel[p.K] = p.E;  // the shared expert's record
      }
    } else if (threadIdx.x == 32 && p.mode != MODE_ROUTE) {
      plan_experts();
    }
    // everything above touches only shared memory and the parameters; from here on
    // the kernel reads what the previous grid may have written
    grid_dependency_wait();
    if (threadIdx.x == 0) hdr->tok_base = ld_relaxed_u32(p.tokens);
    const uint32_t err0 = ld_relaxed_u32(p.err);
    __syncthreads();
    tbase_ = hdr->tok_base;
    if (err0 != 0) return;  // sticky error from an earlier call
    const bool route = p.mode != MODE_EXPERTS;
    const bool do_experts = p.mode != MODE_ROUTE;
    for (int t = 0; t < p.T; ++t) {
      const int buf = t & 1;
      tok_ = t;
      mark(0);
      if (!route) {
        given_routing(t);
        if (hdr->skip_token) continue;
      }
      // weight copies first, activations while they fly
      phase1_issue(route, do_experts && p.has_shared);
      double2* xa = route ? reinterpret_cast<double2*>(stage) : nullptr;
      stage_x(p.x + static_cast<size_t>(t) * p.H, xa, xa ? xa + p.H / 4 : nullptr);
      __syncthreads();
      mark(1);
      if (p.hold_cta == static_cast<int>(blockIdx.x)) {  // test hook: never publish anything
        drain();
        return;
      }
      if (!phase1_consume(buf, route)) break;
      if (route) publish(p.rflags, t);
      mark(2);
      // the shared expert does not depend on the routing: warps 1-15 consume its
      // gate/up rows while warp 0 already polls for the router partials (top-K's
      // scratch and the shared rows occupy disjoint parts of the staging area)
      if (has_sc_) gu_consume(&sc_, 1, buf, 1);
      if (route) {
        topk(buf, t);
        if (hdr->abort_flag) break;
        if (!do_experts) route_weights(t);  // otherwise computed while the rows fly
        mark(4);
      }
      if (do_experts) {
        if (!experts(buf, route, p.resid + static_cast<size_t>(t) * p.H, p.y + static_cast<size_t>(t) * p.H))
          break;
        mark(9);
      }
    }
    if (hdr->abort_flag) {
      drain();
      return;
    }
    // the next call's tags continue after this call's tokens (every block has read
    // the base: block 0 could not have finished without all blocks' values)
    if (blockIdx.x == 0 && threadIdx.x == 0) st_relaxed_u32(p.tokens, tbase_ + static_cast<uint32_t>(p.T));
  }
};

template <int BITS, bool NORM>
__global__ void __launch_bounds__(kThreads, 1) fmoe_layer_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  // launched with programmatic stream serialization: let the next call's launch begin
  // now (a no-op otherwise); the kernel waits for the previous grid before it reads
  // anything that grid may have written
  grid_launch_dependents();
  LayerKernel<BITS, NORM> L(p, smem);
  L.run();
}

// RMS normalisation, one block per token: sum of squares in double (exact products
// of bf16 values), then out = bf16(h / sqrt(mean + eps)) rounded once from double.
__global__ void fmoe_rmsnorm_kernel(const uint16_t* h, uint16_t* out, int H, double eps) {
  __shared__ double part[32];
  grid_launch_dependents();
  grid_dependency_wait();
  const uint16_t* ht = h + static_cast<size_t>(blockIdx.x) * H;
  uint16_t* ot = out + static_cast<size_t>(blockIdx.x) * H;
  double s = 0.0;
  for (int c = threadIdx.x; c < H; c += blockDim.x) {
    const double v = bf16_to_f32(ht[c]);
    s = fma(v, v, s);
  }
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
    v = warp_sum_d(v);
    if (threadIdx.x == 0) part[0] = v;
  }
  __syncthreads();
  const double r = sqrt(part[0] / H + eps);
  __syncthreads();
  for (int c = threadIdx.x; c < H; c += blockDim.x) ot[c] = f64_to_bf16(static_cast<double>(bf16_to_f32(ht[c])) / r);
}

}  // namespace fmoe
