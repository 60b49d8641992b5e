// The fused routed-expert MoE layer kernel for sm_100a.
//
// One persistent thread block per SM (cooperative launch).  Per token:
//
//   P1  router matvec (fp64 accumulation of exact fp32 x bf16 products) over a
//       slice of router rows per block; the shared expert's gate/up rows.
//   B1  grid-wide barrier (bounded wait).
//   P2  every block computes softmax / top-K / renormalisation redundantly from
//       the logits (one warp); then streams its slice of the K routed experts'
//       gate/up row pairs, h = silu(g) * u; the down rows it will need are
//       fetched in the same burst when shared memory allows.
//   B2  grid-wide barrier.
//   P3  every block stages h of all K+1 experts, computes its slice of output
//       rows of the K+1 down matvecs and the combine
//       y = resid + sum_k w_k o_k + sigma o_s, rounded once to bf16.
//
// All weight bytes move HBM -> shared memory through the bulk-copy (TMA) engine
// as contiguous row ranges, completion tracked by mbarriers; a block issues its
// whole share of a phase at once when it fits, so its loads are all in flight.
#pragma once

#include "fmoe_device.cuh"

namespace fmoe {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxK = 32;
constexpr int kNumBars = 96;
constexpr int kMaxRoundItems = kNumBars / 2;
constexpr int kMaxDownBlock = 2 * kWarps;  // output rows per down item (two per warp)
constexpr int kMaxChunks = 8;              // gate/up chunks per round

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
  unsigned long long* bar;
  double* lpart;  // [2][(E+1)*nq]
  float* hbuf;    // [2][(K+1)*I]
  int staging_bytes;
  unsigned long long wait_ns;
  int hold_cta;
};

// Shared-memory header (activations and the staging area follow it).
struct alignas(128) SmemHeader {
  uint64_t bars[kNumBars];
  int sel[kMaxK + 1];    // expert of each slot (slot K = shared expert)
  float wsl[kMaxK + 1];  // weight of each slot (w_k; slot K = sigma)
  int abort_flag;
  int skip_token;
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
    return r128(static_cast<uint32_t>(nslots) * padded(I) * 4u + static_cast<uint32_t>(nslots) * (I / cols) * 4u);
  }
  // header + activations + chunk sums, before the staging area
  __host__ __device__ uint32_t fixed_bytes(uint32_t header) const {
    return r128(header + padded(H) * 4u + static_cast<uint32_t>(H / cols) * 4u);
  }
  __host__ __device__ uint32_t router_item() const { return static_cast<uint32_t>(H) * 4u; }
};

// Rows [ra, rb) of expert slot `slot`, staged at `off`, copy items from `first`.
struct GuChunk {
  int slot, ra, rb;
  uint32_t off, first;
};

template <int BITS>
struct LayerKernel {
  using C = Chunk<BITS>;

  const Params& p;
  Geometry g;
  SmemHeader* hdr;
  float* xs;       // pre-scaled, lane-interleaved activations [H]
  float* xsum;     // per-chunk sums of the unscaled activations [H / kCols]
  uint8_t* stage;  // staging area
  uint32_t nitem;  // items issued so far (same value in every thread)
  int nslots;

  __device__ LayerKernel(const Params& pp, uint8_t* smem) : p(pp) {
    nslots = p.K + (p.has_shared ? 1 : 0);
    g = Geometry{p.H, p.I, p.qh, p.qi, p.sh, p.si, p.rp, p.db, nslots, C::kCols};
    hdr = reinterpret_cast<SmemHeader*>(smem);
    xs = reinterpret_cast<float*>(smem + sizeof(SmemHeader));
    xsum = xs + g.padded(p.H);
    stage = smem + g.fixed_bytes(sizeof(SmemHeader));
    nitem = 0;
  }

  __device__ __forceinline__ uint64_t* bar_of(uint32_t n) const { return &hdr->bars[n % kNumBars]; }
  __device__ __forceinline__ uint32_t parity_of(uint32_t n) const { return (n / kNumBars) & 1u; }

  __device__ __forceinline__ bool wait_item(uint32_t n) {
    return mbar_wait_bounded(bar_of(n), parity_of(n), p.wait_ns, p.err);
  }

  __device__ __forceinline__ const uint8_t* record(int expert) const {
    return p.experts + static_cast<unsigned long long>(expert) * p.rec_bytes;
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

  // ---------------------------------------------------------------- grid barrier
  __device__ bool grid_sync() {
    __syncthreads();
    if (threadIdx.x == 0) {
      int ok = hdr->abort_flag == 0;
      __threadfence();
      const unsigned long long old = atomicAdd(p.bar, 1ull);
      const unsigned long long target = (old / gridDim.x + 1ull) * gridDim.x;
      const uint64_t t0 = global_timer_ns();
      while (ok && ld_acquire_u64(p.bar) < target) {
        if ((ld_relaxed_u32(p.err) & FMOE_DEVERR_BARRIER_TIMEOUT) || global_timer_ns() - t0 > p.wait_ns) {
          atomicOr(p.err, FMOE_DEVERR_BARRIER_TIMEOUT);
          ok = 0;
        }
      }
      __threadfence();
      if (!ok) hdr->abort_flag = 1;
    }
    __syncthreads();
    return hdr->abort_flag == 0;
  }

  // ---------------------------------------------------------------- activations
  __device__ void stage_vec(const float* src_f32, const uint16_t* src_bf16, int n, float* dst, float* dsum) {
    for (int c = threadIdx.x; c < n; c += blockDim.x) {
      const float v = src_bf16 ? bf16_to_f32(src_bf16[c]) : __ldcg(src_f32 + c);
      dst[C::phys(c)] = v * prescale_factor(C::shift_of(c));
    }
    for (int m = threadIdx.x; m < n / C::kCols; m += blockDim.x) {
      float s = 0.f;
      for (int j = 0; j < C::kCols; ++j)
        s += src_bf16 ? bf16_to_f32(src_bf16[m * C::kCols + j]) : __ldcg(src_f32 + m * C::kCols + j);
      dsum[m] = s;
    }
  }

  // ---------------------------------------------------------------- dot products
  // Lane partial of sum_c W[r][c] v[c] over the lane's chunks, for up to two rows
  // sharing the activation loads (W = scale*code + bias; v pre-scaled, interleaved).
  __device__ __forceinline__ void dot2(const uint8_t* q0, const uint32_t* s0, const uint8_t* q1,
                                       const uint32_t* s1, bool two, const float* vs, const float* vsum,
                                       int nch, float& r0, float& r1) const {
    const int lane = threadIdx.x & 31;
    for (int m = lane; m < nch; m += 32) {
      const uint4 a4 = *reinterpret_cast<const uint4*>(q0 + 16 * m);
      uint4 b4 = make_uint4(0, 0, 0, 0);
      if (two) b4 = *reinterpret_cast<const uint4*>(q1 + 16 * m);
      const uint32_t wa[4] = {a4.x, a4.y, a4.z, a4.w};
      const uint32_t wb[4] = {b4.x, b4.y, b4.z, b4.w};
      float2 aa = make_float2(0.f, 0.f), ab = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float4 xv[C::kF4PerWord];
#pragma unroll
        for (int f = 0; f < C::kF4PerWord; ++f) xv[f] = *C::f4(vs, m, j * C::kF4PerWord + f);
        word_fma<BITS>(wa[j], xv, aa);
        if (two) word_fma<BITS>(wb[j], xv, ab);
      }
      const float vm = vsum[m];
      const uint32_t sa = s0[C::sb_index(m)];
      r0 = fmaf(sb_scale(sa), (aa.x + aa.y) * kUnscale, r0);
      r0 = fmaf(sb_bias(sa), vm, r0);
      if (two) {
        const uint32_t sbv = s1[C::sb_index(m)];
        r1 = fmaf(sb_scale(sbv), (ab.x + ab.y) * kUnscale, r1);
        r1 = fmaf(sb_bias(sbv), vm, r1);
      }
    }
  }

  // ---------------------------------------------------------------- gate/up chunks
  __device__ void issue_gu(const GuChunk& c) {
    const uint8_t* rec = record(hdr->sel[c.slot]);
    const int n = c.rb - c.ra;
    const unsigned long long sb_start = p.o_gu_sb + static_cast<unsigned long long>(c.ra) * 2u * p.sh;
    const unsigned long long sb_a = sb_start & ~15ull;
    const unsigned long long sb_end = (sb_start + static_cast<unsigned long long>(n) * 2u * p.sh + 15ull) & ~15ull;
    const uint32_t sbb = static_cast<uint32_t>(sb_end - sb_a);
    const int items = g.gu_items(n);
    for (int i = 0; i < items; ++i) {
      const int a = c.ra + i * p.rp, b = min(c.rb, a + p.rp);
      const uint32_t qb = static_cast<uint32_t>(b - a) * 2u * p.qh;
      uint64_t* bar = bar_of(c.first + i);
      mbar_arrive_expect_tx(bar, qb + (i == 0 ? sbb : 0u));
      bulk_g2s(stage + c.off + static_cast<uint32_t>(a - c.ra) * 2u * p.qh,
               rec + static_cast<unsigned long long>(a) * 2u * p.qh, qb, bar);
      if (i == 0) bulk_g2s(stage + c.off + g.gu_q(n), rec + sb_a, sbb, bar);
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
    dot2(qg, sg, qu, su, true, xs, xsum, p.H / C::kCols, gv, uv);
    gv = warp_sum(gv);
    uv = warp_sum(uv);
    if ((threadIdx.x & 31) == 0) {
      const float hval = (gv / (1.0f + expf(-gv))) * uv;
      p.hbuf[static_cast<size_t>(buf) * (p.K + 1) * p.I + static_cast<size_t>(c.slot) * p.I + r] = hval;
    }
    return true;
  }

  // Consume every row pair of `nc` chunks, spread over the warps.
  __device__ void gu_consume(const GuChunk* ch, int nc, int buf) {
    const int warp = threadIdx.x >> 5;
    int base = 0;
    for (int k = 0; k < nc; ++k) {
      const int n = ch[k].rb - ch[k].ra;
      // unit u of this round goes to warp u % kWarps
      int first = (warp - base) % kWarps;
      if (first < 0) first += kWarps;
      for (int i = first; i < n; i += kWarps) {
        if (!gu_unit(ch[k], ch[k].ra + i, buf)) {
          hdr->abort_flag = 1;
          return;
        }
      }
      base += n;
    }
  }

  // Gate/up of units [v0, v1) of the slot list starting at slot s_lo (unit = s*I + r):
  // chunks per slot, in rounds that fit `cap` bytes from staging offset `base`.
  __device__ bool gu_rounds(int s_lo, int v0, int v1, uint32_t base, uint32_t cap, int buf) {
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
        if (threadIdx.x == 0) {
          fence_proxy_async_smem();
          for (int k = 0; k < nc; ++k) issue_gu(ch[k]);
        }
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
      ch[nc] = GuChunk{s_lo + s, r, r + n, base + used, nitem + static_cast<uint32_t>(items)};
      ++nc;
      items += g.gu_items(n);
      used += g.gu_bytes(n);
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

  // Items [ka, kb) of the block's rows [j0, j1) placed from staging offset `base`.
  __device__ void issue_down_items(int j0, int j1, int ka, int kb, uint32_t first, uint32_t base) {
    if (threadIdx.x == 0) {
      fence_proxy_async_smem();
      for (int k = ka; k < kb; ++k) {
        const int ja = j0 + k * p.db, n = min(j1, ja + p.db) - ja;
        issue_down(first + (k - ka), base + (k - ka) * g.dn_item(p.db), ja, n);
      }
    }
  }

  // Consume a down item (rows [ja, ja+n)): y = resid + sum_s w_s o_s.
  __device__ bool down_item(uint32_t item, uint32_t off, int ja, int n, const float* hs, const float* hsum,
                            const uint16_t* resid_t, uint16_t* y_t) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ia = warp, ib = warp + kWarps;
    if (ia >= n) return true;
    if (!wait_item(item)) {
      hdr->abort_flag = 1;
      return false;
    }
    const bool two = ib < n;
    const uint32_t lead = static_cast<uint32_t>((p.o_d_sb + static_cast<unsigned long long>(ja) * p.si) & 15ull);
    const int nch = p.I / C::kCols;
    float pa = 0.f, pb = 0.f;
    for (int s = 0; s < nslots; ++s) {
      const uint8_t* blk = stage + off + s * g.dn_slot(n);
      const uint32_t* sbase = reinterpret_cast<const uint32_t*>(blk + g.dn_q(n) + lead);
      float oa = 0.f, ob = 0.f;
      dot2(blk + static_cast<uint32_t>(ia) * p.qi, sbase + ia * (p.si / 4), blk + static_cast<uint32_t>(ib) * p.qi,
           sbase + ib * (p.si / 4), two, hs + static_cast<size_t>(s) * g.padded(p.I),
           hsum + static_cast<size_t>(s) * nch, nch, oa, ob);
      const float ws = hdr->wsl[s];
      pa = fmaf(ws, oa, pa);
      pb = fmaf(ws, ob, pb);
    }
    pa = warp_sum(pa);
    pb = warp_sum(pb);
    if (lane == 0) {
      y_t[ja + ia] = f32_to_bf16(bf16_to_f32(resid_t[ja + ia]) + pa);
      if (two) y_t[ja + ib] = f32_to_bf16(bf16_to_f32(resid_t[ja + ib]) + pb);
    }
    return true;
  }

  // ---------------------------------------------------------------- P1
  // Router units [u0, u1) over (E + has_shared) rows x nq splits (the shared gate
  // vector is the last row), plus the block's slice of the shared expert's gate/up.
  __device__ bool phase1(int buf, bool route, bool shared_gu) {
    const int rows = p.E + (p.has_shared ? 1 : 0);
    const int G = gridDim.x, b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int u0 = 0, u1 = 0, row0 = 0, row1 = 0;
    if (route) {
      const long long U = static_cast<long long>(rows) * p.nq;
      u0 = static_cast<int>(U * b / G);
      u1 = static_cast<int>(U * (b + 1) / G);
      row0 = u0 / p.nq;
      row1 = (u1 + p.nq - 1) / p.nq;
    }
    const int hc = p.H / p.nq;
    const uint32_t rib = g.router_item();
    const uint32_t rbase = route ? r128(static_cast<uint32_t>(p.H) * 8u) : 0u;
    const int nrouter = row1 - row0;
    const uint32_t first = nitem;
    GuChunk sc{p.K, 0, 0, rbase + static_cast<uint32_t>(nrouter) * rib, first + static_cast<uint32_t>(nrouter)};
    if (shared_gu) {
      sc.ra = static_cast<int>(static_cast<long long>(p.I) * b / G);
      sc.rb = static_cast<int>(static_cast<long long>(p.I) * (b + 1) / G);
    }
    const int nsh = sc.rb > sc.ra ? g.gu_items(sc.rb - sc.ra) : 0;
    if (threadIdx.x == 0) {
      fence_proxy_async_smem();
      for (int r = row0; r < row1; ++r) {
        const int ua = max(u0, r * p.nq), ub = min(u1, r * p.nq + p.nq);
        uint64_t* bar = bar_of(first + (r - row0));
        const uint32_t bytes = static_cast<uint32_t>(ub - ua) * hc * 4u;
        const float* src = (r < p.E) ? p.router + static_cast<size_t>(r) * p.H : p.sgate;
        src += static_cast<size_t>(ua - r * p.nq) * hc;
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(stage + rbase + (r - row0) * rib + static_cast<uint32_t>(ua - r * p.nq) * hc * 4u, src, bytes, bar);
      }
      if (nsh) issue_gu(sc);
    }
    nitem += static_cast<uint32_t>(nrouter + nsh);
    if (route) {
      const double* x64 = reinterpret_cast<const double*>(stage);
      double* lpart = p.lpart + static_cast<size_t>(buf) * rows * p.nq;
      for (int u = u0 + warp; u < u1; u += kWarps) {
        const int r = u / p.nq, q = u % p.nq;
        if (!wait_item(first + (r - row0))) {
          hdr->abort_flag = 1;
          break;
        }
        const float* wrow = reinterpret_cast<const float*>(stage + rbase + (r - row0) * rib) + q * hc;
        const double* xq = x64 + q * hc;
        double acc = 0.0;
        for (int c = 4 * lane; c < hc; c += 128) {
          const float4 wv = *reinterpret_cast<const float4*>(wrow + c);
          const double2 xa = *reinterpret_cast<const double2*>(xq + c);
          const double2 xb = *reinterpret_cast<const double2*>(xq + c + 2);
          acc = fma(static_cast<double>(wv.x), xa.x, acc);
          acc = fma(static_cast<double>(wv.y), xa.y, acc);
          acc = fma(static_cast<double>(wv.z), xb.x, acc);
          acc = fma(static_cast<double>(wv.w), xb.y, acc);
        }
        acc = warp_sum_d(acc);
        if (lane == 0) lpart[u] = acc;
      }
    }
    if (nsh && hdr->abort_flag == 0) gu_consume(&sc, 1, buf);
    __syncthreads();
    return hdr->abort_flag == 0;
  }

  // ---------------------------------------------------------------- routing
  // Warp 0 of every block: logits, top-K (descending, ties to the lower index),
  // renormalised softmax weights, shared sigmoid gate.
  __device__ void topk(int buf, int t) {
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      const int rows = p.E + (p.has_shared ? 1 : 0);
      double* slog = reinterpret_cast<double*>(stage);
      unsigned long long* skey = reinterpret_cast<unsigned long long*>(stage + r128(static_cast<uint32_t>(rows) * 8u));
      const double* lpart = p.lpart + static_cast<size_t>(buf) * rows * p.nq;
      for (int e = lane; e < rows; e += 32) {
        double l = 0.0;
        for (int q = 0; q < p.nq; ++q) l += __ldcg(lpart + static_cast<size_t>(e) * p.nq + q);
        if (e < p.E && p.has_rbias) l += static_cast<double>(p.rbias[e]);
        slog[e] = l;
        if (e < p.E) skey[e] = dkey(l);
      }
      __syncwarp();
      unsigned long long bk = 0;
      int bi = 0x7fffffff;
      for (int e = lane; e < p.E; e += 32)
        if (skey[e] > bk) {
          bk = skey[e];
          bi = e;
        }
      double l0 = 0.0, den = 0.0;
      for (int k = 0; k < p.K; ++k) {
        const uint32_t hi = static_cast<uint32_t>(bk >> 32);
        const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
        const uint32_t lo = (hi == mhi) ? static_cast<uint32_t>(bk) : 0u;
        const uint32_t mlo = __reduce_max_sync(0xffffffffu, lo);
        const unsigned long long best = (static_cast<unsigned long long>(mhi) << 32) | mlo;
        const uint32_t cand = (bk == best) ? static_cast<uint32_t>(bi) : 0xffffffffu;
        const int win = static_cast<int>(__reduce_min_sync(0xffffffffu, cand));
        const double lw = slog[win];
        if (k == 0) l0 = lw;
        den += exp(lw - l0);
        if (lane == 0) {
          hdr->sel[k] = win;
          hdr->wsl[k] = static_cast<float>(lw);  // logit for now, weight below
        }
        if ((win & 31) == lane) {
          skey[win] = 0;
          bk = 0;
          bi = 0x7fffffff;
          for (int e = lane; e < p.E; e += 32)
            if (skey[e] > bk) {
              bk = skey[e];
              bi = e;
            }
        }
        __syncwarp();
      }
      if (lane == 0) {
        for (int k = 0; k < p.K; ++k) {
          const double wk = exp(slog[hdr->sel[k]] - l0) / den;
          hdr->wsl[k] = static_cast<float>(wk);
          if (blockIdx.x == 0 && p.idx_out) {
            p.idx_out[static_cast<size_t>(t) * p.K + k] = hdr->sel[k];
            p.w_out[static_cast<size_t>(t) * p.K + k] = static_cast<float>(wk);
          }
        }
        if (p.has_shared) {
          const double sig = 1.0 / (1.0 + exp(-slog[p.E]));
          hdr->wsl[p.K] = static_cast<float>(sig);
          if (blockIdx.x == 0 && p.sig_out) p.sig_out[t] = static_cast<float>(sig);
        }
      }
    }
    __syncthreads();
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
  __device__ bool experts(int buf, const uint16_t* resid_t, uint16_t* y_t) {
    const int G = gridDim.x, b = blockIdx.x;
    const int v0 = static_cast<int>(static_cast<long long>(p.K) * p.I * b / G);
    const int v1 = static_cast<int>(static_cast<long long>(p.K) * p.I * (b + 1) / G);
    int j0, j1;
    down_range(j0, j1);
    const int ndown = (j1 - j0 + p.db - 1) / p.db;
    const uint32_t cap = static_cast<uint32_t>(p.staging_bytes);
    // the block's gate/up chunks, one per slot its unit range touches
    GuChunk ch[kMaxChunks];
    int nc = 0, gitems = 0;
    uint32_t gbytes = 0;
    const uint32_t dreg = r128(g.dn_total(j1 - j0));
    int vend = v0;
    while (vend < v1 && nc < kMaxChunks) {
      const int s = vend / p.I, r = vend % p.I, n = min(v1 - vend, p.I - r);
      ch[nc++] = GuChunk{s, r, r + n, dreg + gbytes, nitem + static_cast<uint32_t>(gitems)};
      gitems += g.gu_items(n);
      gbytes += g.gu_bytes(n);
      vend += n;
    }
    const bool prefetch = (vend >= v1) && (dreg + gbytes <= cap) && (dreg + g.h_bytes() <= cap) &&
                          (gitems + ndown <= kMaxRoundItems);
    const uint32_t down_first = nitem + static_cast<uint32_t>(gitems);
    if (prefetch) {
      // gate/up first in issue order, the down rows behind them
      if (threadIdx.x == 0) {
        fence_proxy_async_smem();
        for (int k = 0; k < nc; ++k) issue_gu(ch[k]);
      }
      issue_down_items(j0, j1, 0, ndown, down_first, 0);
      nitem += static_cast<uint32_t>(gitems + ndown);
      gu_consume(ch, nc, buf);
      __syncthreads();
      if (hdr->abort_flag) return false;
    } else {
      if (!gu_rounds(0, v0, v1, 0, cap, buf)) return false;
    }
    if (!grid_sync()) return false;
    // ---- P3: stage h of every slot, then the down rows
    const uint32_t hoff = prefetch ? dreg : 0u;
    float* hs = reinterpret_cast<float*>(stage + hoff);
    const int nchI = p.I / C::kCols;
    const uint32_t hstride = g.padded(p.I);
    float* hsum = hs + static_cast<size_t>(nslots) * hstride;
    const float* hb = p.hbuf + static_cast<size_t>(buf) * (p.K + 1) * p.I;
    for (int s = 0; s < nslots; ++s)
      stage_vec(hb + static_cast<size_t>(s) * p.I, nullptr, p.I, hs + static_cast<size_t>(s) * hstride,
                hsum + static_cast<size_t>(s) * nchI);
    __syncthreads();
    if (prefetch) {
      for (int k = 0; k < ndown; ++k) {
        const int ja = j0 + k * p.db, n = min(j1, ja + p.db) - ja;
        if (!down_item(down_first + k, k * g.dn_item(p.db), ja, n, hs, hsum, resid_t, y_t)) break;
      }
      __syncthreads();
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
    if (threadIdx.x == 0) {
      for (int i = 0; i < kNumBars; ++i) mbar_init(&hdr->bars[i], 1);
      mbar_init_fence();
      hdr->abort_flag = 0;
      hdr->skip_token = 0;
      hdr->sel[p.K] = p.E;  // the shared expert's record
    }
    __syncthreads();
    if (ld_relaxed_u32(p.err) != 0) return;  // sticky error from an earlier call
    for (int t = 0; t < p.T; ++t) {
      const int buf = t & 1;
      const uint16_t* x_t = p.x + static_cast<size_t>(t) * p.H;
      const bool route = p.mode != MODE_EXPERTS;
      const bool do_experts = p.mode != MODE_ROUTE;
      // activations: pre-scaled copy for the dequant dots, doubles for the router
      stage_vec(nullptr, x_t, p.H, xs, xsum);
      if (route) {
        double* x64 = reinterpret_cast<double*>(stage);
        for (int c = threadIdx.x; c < p.H; c += blockDim.x) x64[c] = static_cast<double>(bf16_to_f32(x_t[c]));
      }
      __syncthreads();
      if (!route) {
        given_routing(t);
        if (hdr->skip_token) continue;
      }
      if (!phase1(buf, route, do_experts && p.has_shared)) break;
      if (route) {
        if (p.hold_cta == static_cast<int>(blockIdx.x)) return;  // test hook: never arrive
        if (!grid_sync()) break;
        topk(buf, t);
      }
      if (do_experts) {
        if (!experts(buf, p.resid + static_cast<size_t>(t) * p.H, p.y + static_cast<size_t>(t) * p.H)) break;
      }
    }
    if (hdr->abort_flag) drain();
  }
};

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) fmoe_layer_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  LayerKernel<BITS> L(p, smem);
  L.run();
}

// RMS normalisation, one block per token: sum of squares in double (exact products
// of bf16 values), then out = bf16(h / sqrt(mean + eps)) rounded once from double.
__global__ void fmoe_rmsnorm_kernel(const uint16_t* h, uint16_t* out, int H, double eps) {
  __shared__ double part[32];
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
