// Batched routed-expert matvecs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// The work is the grouped gate/up and down of the batched layer (pairs grouped by
// expert, tiles of up to kUTileTok pairs of one expert), with the arithmetic of the
// mma.sync path: a code c enters the product as the exact bf16 value 1 + c/2^b
// (b = 4 for 4-bit codes, 2 for 2-bit), the activations as exact bf16 (h split into
// hi + lo for down), products are exact and the per-64-column-group accumulator D_g
// is folded as (2^b s) D_g + (bias - 2^b s) X_g, X_g the group's activation sum.
// The dequantised weight is code * scale + bias per 64-column group (hotdry.top,
// "量化策略"); routing the batch's pairs by expert is this library's batched form.
//
// One unit of work is 128 weight rows (the MMA M) of one tile over the whole row:
//   gate/up  the 128 consecutive gate/up rows 2r, 2r+1 (r in [64u, 64u + 64)) -- the
//            record interleaves them, so SwiGLU pairs adjacent accumulator lanes
//   down     output rows [128u, 128u + 128)
// Per CTA (persistent, one per SM, a contiguous weight-balanced range of units):
//   producer warp    per piece (128 bytes of codes of every row: 256 columns of
//                    4-bit, 512 of 2-bit) one TMA tensor load of the codes
//                    (128B-swizzled), one of the (scale, bias) words and one bulk copy
//                    of the tile's activations for those columns into a ring slot
//   converter warps  (4) thread = weight row = TMEM lane: a group's 64 codes become
//                    32 words of bf16 pairs (one rotate and one LOP3 per word) stored
//                    with tcgen05.st as the MMA's A operand in tensor memory
//   MMA warps        (2, even and odd groups) one thread each issues tcgen05.mma (A
//                    from TMEM, B = activations from shared memory, D in TMEM) per 16
//                    columns and commits each group to its own accumulator slot
//   fold warps       (8, even and odd groups) thread = weight row: each group's
//                    accumulator (tcgen05.ld) folded into registers with the group's
//                    scale and bias (packed f32x2 FMAs); at the end of a unit the odd
//                    groups' sums join the even ones' and the even-group warps run the
//                    epilogue (SwiGLU and the h tiles of down, or the down outputs)
// Every hand-off is an mbarrier with one elected arrival per warp.  Shared memory
// traffic per weight is the codes (0.5 or 0.25 B) and the activations' share; A never
// touches shared memory.
//
// The code-to-bf16 rotate places code j and code j + 4 (4-bit; j and j + 8 for
// 2-bit) of a word in one 32-bit TMEM column, so the K order of A is permuted inside
// every 8 (16) columns; the activation tiles are written in the same permuted order
// (kpos_of_col), so every product pairs a code with its own activation.
#pragma once

#include <cuda.h>

#include "fmoe_grouped.cuh"

namespace fmoe {

constexpr int kUTileTok = 32;   // pairs per tile (MMA N = 16 or 32)
// Warps: 0-3 converters (TMEM lane quarter w), 4-11 fold warps (quarter w % 4; even
// groups w < 8, odd groups w >= 8), 12 and 13 MMA issuers (even, odd groups), 14
// producer.
constexpr int kUConvWarps = 4;
constexpr int kUFoldWarp0 = 4;
constexpr int kUMmaWarp = 12;
constexpr int kUProdWarp = 14;
constexpr int kUThreads = 15 * 32;
constexpr int kURows = 128;        // MMA M: weight rows per unit
#ifndef FMOE_UMMA_ASLOTS
#define FMOE_UMMA_ASLOTS 8
#endif
constexpr int kUAslots = FMOE_UMMA_ASLOTS;  // groups in flight in tensor memory (4 or 8)
constexpr int kUTmemCols = kUAslots * 64;   // A: kUAslots x 32 columns, D: kUAslots x 32 columns

static_assert(kUAslots == 4 || kUAslots == 8, "tensor memory holds 4 or 8 group slots");
constexpr int kUCodeBox = 128;     // bytes of codes per row per piece
constexpr int kUMaxSlots = 6;      // ring slots at most
constexpr int kUExPitch = kUTileTok + 1;  // floats per row of the h-sum staging

template <int BITS>
struct UGeom {
  static constexpr int kPC = kUCodeBox * 8 / BITS;  // columns per piece: 256 / 512
  static constexpr int kPG = kPC / 64;              // groups per piece: 4 / 8
  static constexpr int kSbBox = kPG * 4;            // (scale, bias) bytes per row per piece
  static constexpr uint32_t kCodeBytes = kURows * kUCodeBox;
  static constexpr uint32_t kSbBytes = kURows * kSbBox;
  static constexpr float kScaleMul = BITS == 4 ? 16.0f : 4.0f;
};

// Position in the MMA's K order of column c of a row (the rotate's permutation):
// 4-bit, inside each 8 columns: column j -> 2j (j < 4), 2(j - 4) + 1 (j >= 4);
// 2-bit, inside each 16 columns: column j -> 2j (j < 8), 2(j - 8) + 1 (j >= 8).
template <int BITS>
__host__ __device__ constexpr int kpos_of_col(int c) {
  return BITS == 4 ? (c & ~7) + 2 * (c & 3) + ((c >> 2) & 1) : (c & ~15) + 2 * (c & 7) + ((c >> 3) & 1);
}

// Bytes of one piece of a tile's activations, npad pairs (a multiple of 16):
// gate/up  [B: (kPC/8) K-blocks x npad x 16 B][X: kPG x npad floats]
// down     [B hi: same][B lo: same][X: kPG x npad floats]
template <int BITS, bool DOWN>
__host__ __device__ constexpr uint32_t upiece_bytes(int npad) {
  return static_cast<uint32_t>(npad) * ((DOWN ? 4u : 2u) * UGeom<BITS>::kPC + 4u * UGeom<BITS>::kPG);
}
// Bytes of the activation tile buffer per 16 pairs of a tile (all pieces of a row).
__host__ __device__ inline size_t xg_bytes_per16(int H) { return 16ull * (2ull * H + H / 16); }
__host__ __device__ inline size_t hg_bytes_per16(int I) { return 16ull * (4ull * I + I / 16); }

// Shared memory of one ring slot: codes (1024-aligned for the 128B swizzle), the
// (scale, bias) words, the activation piece of the largest tile.
template <int BITS, bool DOWN>
__host__ __device__ constexpr uint32_t uslot_bytes() {
  return (UGeom<BITS>::kCodeBytes + UGeom<BITS>::kSbBytes + upiece_bytes<BITS, DOWN>(kUTileTok) + 1023u) & ~1023u;
}

struct alignas(64) UParams {
  CUtensorMap tm_q;   // codes of the phase's rows: {row bytes, rows, experts}
  CUtensorMap tm_sb;  // (scale, bias) words of the phase's rows: {row bytes, rows, experts}
  GParams p;
  int slots;          // ring slots
};

struct UHeader {
  uint64_t full[kUMaxSlots];   // slot landed (producer's expect_tx + the copies' bytes)
  uint64_t empty[kUMaxSlots];  // slot free: 4 converter + 8 fold warps + 2 MMA commits
  uint64_t afull[kUAslots];    // A of a group in TMEM: the 4 converter warps
  uint64_t dfull[kUAslots];    // the group's MMAs complete (A slot reusable, D readable): commit
  uint64_t dfree[kUAslots];    // D of the group read: its parity's 4 fold warps
  uint64_t drain[2];           // each MMA issuer's last commit
  uint64_t ex_full;            // the odd-group fold warps' sums written to shared memory
  uint64_t ex_empty;           // ... and added by the even-group fold warps
  uint64_t red_full;           // the even-group fold warps' h sums written to shared memory
  uint64_t red_empty;          // ... and summed (the first of them)
  int seg_tile[kMaxSeg];
  int seg_ra[kMaxSeg];
  int seg_rb[kMaxSeg];
  int nseg;
  int first;
  int abort_flag;
  uint32_t tmem;
};
constexpr uint32_t kUHeaderBytes = (sizeof(UHeader) + 1023u) & ~1023u;

// Dynamic shared memory of a phase with `slots` ring slots (+1 KB for the alignment);
// after the ring, the odd-group fold warps' sums of a unit (128 rows x kUExPitch
// floats) and the h values of a gate/up unit (64 rows x kUExPitch floats) for the down
// groups' sums.
template <int BITS, bool DOWN>
__host__ __device__ constexpr uint32_t umma_smem_bytes(int slots) {
  return 1024u + kUHeaderBytes + static_cast<uint32_t>(slots) * uslot_bytes<BITS, DOWN>() +
         static_cast<uint32_t>((kURows + 64) * kUExPitch * 4);
}

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  return (static_cast<unsigned long long>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 3-D tiled TMA load into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&w)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
      "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15]), "r"(w[16]), "r"(w[17]), "r"(w[18]),
      "r"(w[19]), "r"(w[20]), "r"(w[21]), "r"(w[22]), "r"(w[23]), "r"(w[24]), "r"(w[25]), "r"(w[26]), "r"(w[27]),
      "r"(w[28]), "r"(w[29]), "r"(w[30]), "r"(w[31])
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major, no swizzle: core matrices of 8 rows x 16 B
// (rows 16 B apart), `lbo` bytes between the two 8-element K halves, `sbo` bytes
// between 8-row groups; descriptor version 1.
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor: bf16 x bf16 -> f32, A and B K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t umma_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kURows >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The mbarrier tracks the completion of every tcgen05.mma this thread issued so far.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Pair (code q, code q + 4) of a 4-bit word as bf16 1 + c/16 (low, high half).
__device__ __forceinline__ uint32_t ucodes4(uint32_t w, int q) {
  return (__funnelshift_r(w, w, (4 * q - 3) & 31) & 0x00780078u) | 0x3F803F80u;
}
// Pair (code q, code q + 8) of a 2-bit word as bf16 1 + c/4.
__device__ __forceinline__ uint32_t ucodes2(uint32_t w, int q) {
  return (__funnelshift_r(w, w, (2 * q - 5) & 31) & 0x00600060u) | 0x3F803F80u;
}

// ---------------------------------------------------------------- activation tiles
// x of every tile's pairs in the MMA's permuted K order, per piece, plus the per-group
// sums X_g; pairs beyond the tile's count are zeros.  Work items (tile, piece); a
// thread per (pair, 16 columns).
template <int BITS>
__global__ void __launch_bounds__(256) grouped_stage_x_kernel(const __grid_constant__ GParams p) {
  using Gm = UGeom<BITS>;
  grid_launch_dependents();
  grid_dependency_wait();
  if (ld_relaxed_u32(p.err) != 0) return;
  const int nt = __ldcg(p.ntiles);
  const int NP = p.H / Gm::kPC;
  constexpr int per = Gm::kPC / 16;  // 16-column blocks per piece row
  for (int item = blockIdx.x; item < nt * NP; item += gridDim.x) {
    const int ti = item / NP, pc = item % NP;
    const GTile tl = p.tiles[ti];
    const int npad = (tl.n + 15) & ~15;
    uint8_t* base = p.xg + static_cast<size_t>(tl.tok16) * xg_bytes_per16(p.H) +
                    static_cast<size_t>(pc) * upiece_bytes<BITS, false>(npad);
    for (int t = threadIdx.x; t < npad * per; t += blockDim.x) {  // npad * per is a multiple of 256
      const int n = t / per, cb = t % per;
      const int c0 = pc * Gm::kPC + cb * 16;
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
      if (n < tl.n) {
        const int tok = __ldcg(p.pair_token + tl.p0 + n);
        const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(tok) * p.H + c0);
        a = src[0];
        b = src[1];
      }
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint16_t out[16];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint16_t v = static_cast<uint16_t>(w[c >> 1] >> (16 * (c & 1)));
        out[kpos_of_col<BITS>(c)] = v;
        sum += bf16_to_f32(v);
      }
      uint4 o0, o1;
      o0.x = out[0] | (static_cast<uint32_t>(out[1]) << 16);
      o0.y = out[2] | (static_cast<uint32_t>(out[3]) << 16);
      o0.z = out[4] | (static_cast<uint32_t>(out[5]) << 16);
      o0.w = out[6] | (static_cast<uint32_t>(out[7]) << 16);
      o1.x = out[8] | (static_cast<uint32_t>(out[9]) << 16);
      o1.y = out[10] | (static_cast<uint32_t>(out[11]) << 16);
      o1.z = out[12] | (static_cast<uint32_t>(out[13]) << 16);
      o1.w = out[14] | (static_cast<uint32_t>(out[15]) << 16);
      // K-block k of pair n at k * npad * 16 + n * 16
      *reinterpret_cast<uint4*>(base + static_cast<size_t>(2 * cb) * npad * 16 + n * 16) = o0;
      *reinterpret_cast<uint4*>(base + static_cast<size_t>(2 * cb + 1) * npad * 16 + n * 16) = o1;
      // the 64-column group's sum over its 4 threads (consecutive cb of the same pair)
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      if ((cb & 3) == 0) {
        float* X = reinterpret_cast<float*>(base + static_cast<size_t>(Gm::kPC / 8) * npad * 16);
        X[(cb >> 2) * npad + n] = sum;
      }
    }
  }
}

// ---------------------------------------------------------------- the matvec kernel
template <int BITS, bool DOWN>
struct UKernel {
  using Gm = UGeom<BITS>;
  const UParams& up;
  const GParams& p;
  UHeader* hdr;
  uint8_t* ring;
  float* ex;
  int warp, lane;
  int NP;  // pieces per unit
  int S;   // ring slots

  __device__ UKernel(const UParams& u, uint8_t* base) : up(u), p(u.p) {
    warp = threadIdx.x >> 5;
    lane = threadIdx.x & 31;
    hdr = reinterpret_cast<UHeader*>(base);
    ring = base + kUHeaderBytes;
    S = u.slots;
    ex = reinterpret_cast<float*>(ring + static_cast<size_t>(S) * uslot_bytes<BITS, DOWN>());
    NP = (DOWN ? p.I : p.H) / Gm::kPC;
  }

  __device__ __forceinline__ uint8_t* slot_q(uint32_t s) const { return ring + s * uslot_bytes<BITS, DOWN>(); }
  __device__ __forceinline__ uint8_t* slot_sb(uint32_t s) const { return slot_q(s) + Gm::kCodeBytes; }
  __device__ __forceinline__ uint8_t* slot_b(uint32_t s) const { return slot_sb(s) + Gm::kSbBytes; }

  // Pipeline waits: try_wait with a suspend-time hint parks the thread until the phase
  // completes (or the hint passes), so a waiting warp takes no issue slots from the
  // warps on the critical path of its SM sub-partition, and wakes without a sleep's
  // delay; the clock bounds the whole wait.
  __device__ __forceinline__ bool spin(uint64_t* bar, uint32_t parity) const {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
      if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
      if (global_timer_ns() - t0 > p.wait_ns) {
        atomicOr(p.err, FMOE_DEVERR_COPY_TIMEOUT);
        return false;
      }
    }
  }

  __device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) {
    if (spin(bar, parity)) return true;
    hdr->abort_flag = 1;
    return false;
  }
  // converter warps: every lane waits, and the warp goes on only if all lanes saw the
  // phase (the tcgen05 loads and stores that follow are warp-collective)
  __device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity) {
    const bool ok = __all_sync(0xffffffffu, spin(bar, parity));
    if (!ok) hdr->abort_flag = 1;
    return ok;
  }
  __device__ __forceinline__ bool aborted() const {
    return *reinterpret_cast<volatile const int*>(&hdr->abort_flag) != 0;
  }

  // ---- the block's segments: (tile, [ra, rb)) in tile order, units of R row blocks
  __device__ void plan(int R) {
    const int nt = __ldcg(p.ntiles);
    const long long Ctot = __ldcg(p.tcost + nt);
    const int NB = gridDim.x, b = blockIdx.x;
    const long long X0 = Ctot * R * b / NB, X1 = Ctot * R * (b + 1) / NB;
    if (threadIdx.x == 0) {
      hdr->nseg = 0;
      hdr->first = 0;
    }
    __syncthreads();
    auto range = [&](int i, int& ra, int& rb) {
      const long long c0 = __ldcg(p.tcost + i) * R;
      const long long wi = __ldcg(p.tcost + i + 1) - __ldcg(p.tcost + i);
      ra = X0 <= c0 ? 0 : static_cast<int>(min(static_cast<long long>(R), (X0 - c0 + wi - 1) / wi));
      rb = X1 <= c0 ? 0 : static_cast<int>(min(static_cast<long long>(R), (X1 - c0 + wi - 1) / wi));
    };
    for (int i = threadIdx.x; i < nt; i += kUThreads) {
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
        hdr->nseg = 0;
      }
      __syncthreads();
      return;
    }
    for (int s = threadIdx.x; s < nseg; s += kUThreads) {
      int ra, rb;
      range(first + s, ra, rb);
      hdr->seg_tile[s] = first + s;
      hdr->seg_ra[s] = ra;
      hdr->seg_rb[s] = rb;
    }
    __syncthreads();
  }

  // ---- producer: one lane of the producer warp
  __device__ void produce() {
    uint32_t pi = 0;
    const int nseg = hdr->nseg;
    for (int s = 0; s < nseg && !aborted(); ++s) {
      const GTile tl = p.tiles[hdr->seg_tile[s]];
      const int npad = (tl.n + 15) & ~15;
      const uint32_t bpiece = upiece_bytes<BITS, DOWN>(npad);
      const uint8_t* tb = DOWN ? p.hg + static_cast<size_t>(tl.tok16) * hg_bytes_per16(p.I)
                               : p.xg + static_cast<size_t>(tl.tok16) * xg_bytes_per16(p.H);
      for (int u = hdr->seg_ra[s]; u < hdr->seg_rb[s]; ++u) {
        for (int pc = 0; pc < NP; ++pc, ++pi) {
          const uint32_t slot = pi % S;
          if (pi >= static_cast<uint32_t>(S) && !wait(&hdr->empty[slot], ((pi / S) - 1) & 1u)) return;
          if (aborted()) return;
          uint64_t* bar = &hdr->full[slot];
          mbar_arrive_expect_tx(bar, Gm::kCodeBytes + Gm::kSbBytes + bpiece);
          tma_load_3d(slot_q(slot), &up.tm_q, bar, pc * kUCodeBox, u * kURows, tl.expert);
          tma_load_3d(slot_sb(slot), &up.tm_sb, bar, pc * Gm::kSbBox, u * kURows, tl.expert);
          bulk_g2s(slot_b(slot), tb + static_cast<size_t>(pc) * bpiece, bpiece, bar);
          issued_ = pi + 1;
        }
      }
    }
  }
  uint32_t issued_ = 0;

  // the producer's copies still in flight land before the block exits
  __device__ void drain_copies() {
    const uint32_t lo = issued_ > static_cast<uint32_t>(S) ? issued_ - S : 0u;
    for (uint32_t pi = lo; pi < issued_; ++pi) mbar_wait_bounded(&hdr->full[pi % S], (pi / S) & 1u, p.wait_ns, p.err);
  }

  // ---- MMA issuer: one lane of the MMA warp.  Group g uses TMEM slot g % kUAslots
  // (use k = g / kUAslots): it waits for the converters' A (afull phase k) and for the
  // fold warps' read of the slot's previous D (dfree phase k - 1), issues the group's
  // K steps and commits them to dfull; after a piece's last group the commit to the
  // slot's empty barrier says its activations are read.
  __device__ void issue_mmas(uint32_t tmem, int par) {
    uint32_t pi = 0, gi = 0;
    const int nseg = hdr->nseg;
    bool ok = true;
    for (int s = 0; s < nseg && ok; ++s) {
      const GTile tl = p.tiles[hdr->seg_tile[s]];
      const int npad = (tl.n + 15) & ~15;
      const uint32_t idesc = umma_idesc(npad);
      const uint32_t kb_bytes = static_cast<uint32_t>(npad) * 16u;  // one K-block of 8 columns
      for (int u = hdr->seg_ra[s]; u < hdr->seg_rb[s] && ok; ++u) {
        for (int pc = 0; pc < NP && ok; ++pc, ++pi) {
          const uint32_t slot = pi % S;
          if (!wait(&hdr->full[slot], (pi / S) & 1u)) {
            ok = false;
            break;
          }
          // the descriptors of the piece differ only in their start address field
          const uint64_t bd0 = umma_sdesc(smem_u32(slot_b(slot)), kb_bytes, 128);
          const uint64_t lo_off = static_cast<uint64_t>((Gm::kPC / 8) * kb_bytes) >> 4;
          for (int gl = par; gl < Gm::kPG; gl += 2) {
            const uint32_t g = gi + gl, a = g % kUAslots, k = g / kUAslots;
            if (!wait(&hdr->afull[a], k & 1u) || (k > 0 && !wait(&hdr->dfree[a], (k - 1) & 1u))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_t = tmem + kUAslots * 32 + a * 32;
            const uint32_t a_t = tmem + a * 32;
            const uint64_t bg = bd0 + ((static_cast<uint64_t>(8 * gl) * kb_bytes) >> 4);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t bj = bg + ((static_cast<uint64_t>(2 * j) * kb_bytes) >> 4);
              umma_ts(d_t, a_t + 8 * j, bj, idesc, j > 0 ? 1u : 0u);
              if (DOWN) umma_ts(d_t, a_t + 8 * j, bj + lo_off, idesc, 1u);
            }
            umma_commit(&hdr->dfull[a]);
          }
          gi += Gm::kPG;
          if (ok) umma_commit(&hdr->empty[slot]);
        }
      }
    }
    // every MMA issued has completed before the block frees its tensor memory
    umma_commit(&hdr->drain[par]);
    mbar_wait_bounded(&hdr->drain[par], 0u, p.wait_ns, p.err);
  }

  // ---- converter warps 0-3, thread = weight row = TMEM lane.  Group g's A goes to
  // TMEM slot g % kUAslots once the MMAs of the slot's previous group completed (dfull
  // phase k - 1).
  __device__ void convert(uint32_t tmem) {
    const int q = warp & 3, row = 32 * q + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    uint32_t pi = 0, gi = 0;
    const int nseg = hdr->nseg;
    for (int s = 0; s < nseg; ++s) {
      for (int u = hdr->seg_ra[s]; u < hdr->seg_rb[s]; ++u) {
        for (int pc = 0; pc < NP; ++pc, ++pi) {
          const uint32_t slot = pi % S;
          if (!wait_warp(&hdr->full[slot], (pi / S) & 1u)) return;
          const uint8_t* qrow = slot_q(slot) + row * kUCodeBox;
          for (int gl = 0; gl < Gm::kPG; ++gl) {
            const uint32_t g = gi + gl;
            uint32_t w[32];
            if (BITS == 4) {  // 32 bytes: 16-byte chunks 2gl, 2gl+1, 128B-swizzled
              const uint4 c0 = *reinterpret_cast<const uint4*>(qrow + (((2 * gl) ^ (row & 7)) << 4));
              const uint4 c1 = *reinterpret_cast<const uint4*>(qrow + (((2 * gl + 1) ^ (row & 7)) << 4));
              const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
              for (int m = 0; m < 8; ++m)
#pragma unroll
                for (int j = 0; j < 4; ++j) w[4 * m + j] = ucodes4(cw[m], j);
            } else {  // 16 bytes: chunk gl
              const uint4 c0 = *reinterpret_cast<const uint4*>(qrow + ((gl ^ (row & 7)) << 4));
              const uint32_t cw[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
              for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int j = 0; j < 8; ++j) w[8 * m + j] = ucodes2(cw[m], j);
            }
            const uint32_t a = g % kUAslots, k = g / kUAslots;
            if (k > 0 && !wait_warp(&hdr->dfull[a], (k - 1) & 1u)) return;
            tc_fence_after();
            tmem_st32(tmem + lane_base + a * 32, w);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&hdr->afull[a]);
          }
          gi += Gm::kPG;
          __syncwarp();
          if (lane == 0) mbar_arrive(&hdr->empty[slot]);  // the warp's codes of the piece are read
        }
      }
    }
  }

  // ---- fold warps 4-11 (quarter w % 4, groups of parity (w - 4) / 4), thread = weight
  // row: D of each of its groups folded with the group's scale and bias into acc; at
  // the unit's end the odd-group sums are added to the even ones' through shared
  // memory and the even-group warps run the epilogue.
  __device__ void fold_all(uint32_t tmem) {
    const int q = warp & 3, fpar = (warp - kUFoldWarp0) >> 2, row = 32 * q + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    uint32_t pi = 0, gi = 0, ku = 0;
    unsigned long long acc2[kUTileTok / 2];  // pairs of pairs' sums (packed f32x2)
    const int nseg = hdr->nseg;
    for (int s = 0; s < nseg; ++s) {
      const GTile tl = p.tiles[hdr->seg_tile[s]];
      const int npad = (tl.n + 15) & ~15;
      const uint32_t bdata = (DOWN ? 2u : 1u) * (Gm::kPC / 8) * static_cast<uint32_t>(npad) * 16u;
      for (int u = hdr->seg_ra[s]; u < hdr->seg_rb[s]; ++u, ++ku) {
#pragma unroll
        for (int n = 0; n < kUTileTok / 2; ++n) acc2[n] = 0ull;
        for (int pc = 0; pc < NP; ++pc, ++pi) {
          const uint32_t slot = pi % S;
          if (!wait_warp(&hdr->full[slot], (pi / S) & 1u)) return;
          const uint8_t* sbrow = slot_sb(slot) + row * Gm::kSbBox;
          const float* X = reinterpret_cast<const float*>(slot_b(slot) + bdata);
          for (int gl = fpar; gl < Gm::kPG; gl += 2) {
            const uint32_t g = gi + gl, a = g % kUAslots;
            const uint32_t sbw = *reinterpret_cast<const uint32_t*>(sbrow + 4 * gl);
            if (!wait_warp(&hdr->dfull[a], (g / kUAslots) & 1u)) return;
            tc_fence_after();
            uint32_t v[kUTileTok];
            tmem_ld16(tmem + lane_base + kUAslots * 32 + a * 32, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
            if (npad > 16)
              tmem_ld16(tmem + lane_base + kUAslots * 32 + a * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&hdr->dfree[a]);
            const float s16 = Gm::kScaleMul * sb_scale(sbw), cb = sb_bias(sbw) - s16;
            const unsigned long long s2 = pack2(s16, s16), c2 = pack2(cb, cb);
            const ulonglong2* X2 = reinterpret_cast<const ulonglong2*>(X + gl * npad);
#pragma unroll
            for (int c = 0; c < kUTileTok / 4; ++c) {
              if (4 * c < npad) {
                const ulonglong2 x = X2[c];
                fma2(acc2[2 * c], c2, x.x);
                fma2(acc2[2 * c + 1], c2, x.y);
                fma2(acc2[2 * c], s2, (static_cast<unsigned long long>(v[4 * c + 1]) << 32) | v[4 * c]);
                fma2(acc2[2 * c + 1], s2, (static_cast<unsigned long long>(v[4 * c + 3]) << 32) | v[4 * c + 2]);
              }
            }
          }
          gi += Gm::kPG;
          __syncwarp();
          if (lane == 0) mbar_arrive(&hdr->empty[slot]);  // the warp's words and sums of the piece are read
        }
        float acc[kUTileTok];
#pragma unroll
        for (int n = 0; n < kUTileTok / 2; ++n) {
          acc[2 * n] = __uint_as_float(static_cast<uint32_t>(acc2[n]));
          acc[2 * n + 1] = __uint_as_float(static_cast<uint32_t>(acc2[n] >> 32));
        }
        // the odd groups' sums join the even groups' in the even-group warps
        float* exr = ex + row * kUExPitch;
        if (fpar == 1) {
          if (ku > 0 && !wait_warp(&hdr->ex_empty, (ku - 1) & 1u)) return;
#pragma unroll
          for (int n = 0; n < kUTileTok; ++n)
            if (n < npad) exr[n] = acc[n];
          __syncwarp();
          if (lane == 0) mbar_arrive(&hdr->ex_full);
          continue;
        }
        if (!wait_warp(&hdr->ex_full, ku & 1u)) return;
#pragma unroll
        for (int n = 0; n < kUTileTok; ++n)
          if (n < npad) acc[n] += exr[n];
        __syncwarp();
        if (lane == 0) mbar_arrive(&hdr->ex_empty);
        if (!epilogue(tl, npad, u, ku, acc, q, row)) return;
      }
    }
  }

  // The unit's outputs: SwiGLU + the down activation tiles and the down group's sums
  // (gate/up), or o per pair (down).  ku counts this thread's units (the phases of
  // the h-sum barriers).
  __device__ bool epilogue(const GTile& tl, int npad, int u, uint32_t ku, float (&acc)[kUTileTok], int q, int row) {
    if (DOWN) {
      const int j = kURows * u + row;
#pragma unroll
      for (int n = 0; n < kUTileTok; ++n)
        if (n < tl.n) p.obuf[static_cast<size_t>(tl.p0 + n) * p.H + j] = acc[n];
      return true;
    }
    // lanes 2i, 2i+1: gate and up of intermediate row 64u + 16q + i
    const int ir = row >> 1, i = 64 * u + ir;
    const bool gate = (lane & 1) == 0;
    uint8_t* tb = p.hg + static_cast<size_t>(tl.tok16) * hg_bytes_per16(p.I);
    const uint32_t dpiece = upiece_bytes<BITS, true>(npad);
    const uint32_t kb_bytes = static_cast<uint32_t>(npad) * 16u;
    const int pd = i / Gm::kPC, P = kpos_of_col<BITS>(i % Gm::kPC);
    uint8_t* hi = tb + static_cast<size_t>(pd) * dpiece + (P >> 3) * kb_bytes + (P & 7) * 2;
    uint8_t* lo = hi + (Gm::kPC / 8) * kb_bytes;
    float* hs = ex + kURows * kUExPitch;  // [64 intermediate rows][kUExPitch]: hi + lo of each h
    if (ku > 0 && !wait_warp(&hdr->red_empty, (ku - 1) & 1u)) return false;
#pragma unroll
    for (int n = 0; n < kUTileTok; ++n) {
      if (n < npad) {
        const float uv = __shfl_xor_sync(0xffffffffu, acc[n], 1);
        if (gate) {
          const float gv = acc[n];
          const float h = (gv / (1.0f + expf(-gv))) * uv;
          const uint16_t hb = f32_to_bf16(h);
          const uint16_t lb = f32_to_bf16(h - bf16_to_f32(hb));
          *reinterpret_cast<uint16_t*>(hi + n * 16) = hb;
          *reinterpret_cast<uint16_t*>(lo + n * 16) = lb;
          hs[ir * kUExPitch + n] = bf16_to_f32(hb) + bf16_to_f32(lb);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&hdr->red_full);
    if (q == 0) {
      if (!wait_warp(&hdr->red_full, ku & 1u)) return false;
      if (lane < npad) {
        float x = 0.f;
        for (int r = 0; r < 64; ++r) x += hs[r * kUExPitch + lane];
        // X of down group u: piece 64u / kPC, group (64u % kPC) / 64 of that piece
        const int pu = (64 * u) / Gm::kPC, gu = ((64 * u) % Gm::kPC) / 64;
        float* Xd = reinterpret_cast<float*>(tb + static_cast<size_t>(pu) * dpiece + 2 * (Gm::kPC / 8) * kb_bytes);
        Xd[gu * npad + lane] = x;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&hdr->red_empty);
    }
    return true;
  }
};

template <int BITS, bool DOWN>
__global__ void __launch_bounds__(kUThreads, 1) grouped_umma_kernel(const __grid_constant__ UParams up) {
  extern __shared__ __align__(1024) uint8_t usmem[];
  grid_launch_dependents();
  grid_dependency_wait();
  if (ld_relaxed_u32(up.p.err) != 0) return;
  uint8_t* base = usmem + ((1024u - (smem_u32(usmem) & 1023u)) & 1023u);
  UKernel<BITS, DOWN> K(up, base);
  UHeader* hdr = K.hdr;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kUMaxSlots; ++s) {
      mbar_init(&hdr->full[s], 1);
      mbar_init(&hdr->empty[s], kUConvWarps + 8 + 2);
    }
    for (int a = 0; a < kUAslots; ++a) {
      mbar_init(&hdr->afull[a], 4);
      mbar_init(&hdr->dfull[a], 1);
      mbar_init(&hdr->dfree[a], 4);
    }
    mbar_init(&hdr->drain[0], 1);
    mbar_init(&hdr->drain[1], 1);
    mbar_init(&hdr->ex_full, 4);
    mbar_init(&hdr->ex_empty, 4);
    mbar_init(&hdr->red_full, 4);
    mbar_init(&hdr->red_empty, 1);
    hdr->abort_flag = 0;
    mbar_init_fence();
  }
  if (K.warp == kUMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&hdr->tmem)),
                 "r"(kUTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = hdr->tmem;
  K.plan(DOWN ? up.p.H / kURows : up.p.I / 64);
  if (K.warp < kUConvWarps) {
    K.convert(tmem);
  } else if (K.warp < kUMmaWarp) {
    K.fold_all(tmem);
  } else if (K.warp < kUProdWarp) {
    if (K.lane == 0) K.issue_mmas(tmem, K.warp - kUMmaWarp);
  } else if (K.lane == 0) {
    K.produce();
    K.drain_copies();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (K.warp == kUMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUTmemCols) : "memory");
}

}  // namespace fmoe
