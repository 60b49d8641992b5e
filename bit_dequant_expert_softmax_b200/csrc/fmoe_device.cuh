// Device helpers for the fused routed-expert MoE layer kernel (sm_100a):
// mbarrier / bulk-copy (TMA engine) wrappers, bounded waits, a grid-wide
// barrier with a time limit, and the dequantising dot products.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/fmoe.h"

namespace fmoe {

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits until the grid this one depends on (programmatic dependent launch) has
// completed and its memory operations are visible; a no-op without such a dependency.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the grid launched after this one (with programmatic serialization) start its
// launch now; a no-op otherwise.
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bulk copy global -> this CTA's shared memory, completion signalled on `bar`
// (transaction bytes).  dst, src and bytes are multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long atom_add_release_u64(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.add.release.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// 16-byte load of two 64-bit words, each read single-copy atomically, not cached in L1.
__device__ __forceinline__ ulonglong2 ld_volatile_v2_u64(const unsigned long long* p) {
  ulonglong2 v;
  asm volatile("ld.volatile.global.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// try_wait with a suspend-time hint: the warp is parked by the hardware until the
// phase completes (or the hint elapses) instead of spinning on the issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of `bar` to complete, for at most limit_ns.  Between polls
// the warp sleeps, so that waiting warps leave the issue slots to computing ones.
#ifndef FMOE_WAIT_SLEEP_NS
#define FMOE_WAIT_SLEEP_NS 64
#endif
__device__ __noinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                               uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    __nanosleep(FMOE_WAIT_SLEEP_NS);
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      atomicOr(err, FMOE_DEVERR_COPY_TIMEOUT);
      return false;
    }
  }
}

// The dequantised weight is code * scale + bias per 64-column group (hotdry.top,
// "量化策略"); the juejin.cn shader section "Metal 着色器" rewrites the product as
// fma(code, scale*x, bias*x).  Here the same sum is folded once per chunk:
// scale * sum(code * x) + bias * sum(x).
//
// Codes as floats without conversion instructions: a code c masked in place at bit
// offset s (s + bits <= 24) reads, as an IEEE float, exactly c * 2^s * 2^-149 (a
// subnormal or the first normal binade).  The activation multiplying it is stored
// pre-scaled by 2^(P - s), so every product is code * x * 2^(P - 149) exactly, and the
// per-chunk sum is rescaled by 2^(149 - P) once.  P is chosen per chunk from the
// largest exponent e of the chunk's activations, P = 100 - e (e clamped to
// [kMinExp, kMaxExp]): the pre-scaled values stay below 2^101 and the products of the
// chunk's largest activations near 2^-45, far inside the normal range, whatever the
// activations' magnitude (the clamp keeps the factor 2^(P - s) and the rescale
// 2^(149 - P) representable; it leaves |x| < 2^-103 or |x| >= 2^105 outside the exact
// range).
//
// Codes are taken in pairs from two adjacent words {w_a, w_b} of a 16-byte load,
// viewed as one 64-bit register: a 64-bit AND with the same mask in both halves
// yields, in place, the codes of position p of both words -- exactly the packed
// operand of one fma.rn.f32x2.  Codes that sit above bit 23 are read from the pair
// shifted right by 8 (the bits crossing from w_b into w_a's top byte are never
// selected by the masks).  The activations are laid out so that one 64-bit shared
// load gives the matching pair {x(word a, p), x(word b, p)}.
constexpr int kPreExp = 100;
constexpr int kMinExp = -26;
constexpr int kMaxExp = 78;

// Pre-scale exponent P of a chunk whose largest |activation| has the float bit pattern
// `maxbits` (sign cleared).
__device__ __forceinline__ int chunk_pre(uint32_t maxbits) {
  const int e = static_cast<int>(maxbits >> 23) - 127;
  return kPreExp - min(max(e, kMinExp), kMaxExp);
}

// 2^(149 - P): the rescale of a chunk's sum of products.
__device__ __forceinline__ float chunk_unscale(int pre) {
  return __uint_as_float(static_cast<uint32_t>(127 + 149 - pre) << 23);
}

__device__ __forceinline__ void fma2(unsigned long long& acc, unsigned long long c, unsigned long long x) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(c), "l"(x));
}

__device__ __forceinline__ float pair_sum(unsigned long long a) {
  return __uint_as_float(static_cast<uint32_t>(a)) + __uint_as_float(static_cast<uint32_t>(a >> 32));
}

// Chunk geometry: one chunk = 16 bytes of codes = 4 words = 2 word pairs.
template <int BITS>
struct Chunk {
  static constexpr int kCols = 128 / BITS;    // 32 (4-bit) or 64 (2-bit) columns
  static constexpr int kWC = 32 / BITS;       // codes per word: 8 or 16
  static constexpr int kF4 = kCols / 4;       // float4 of activations per chunk: 8 or 16
  static constexpr int kF4PerPair = kWC / 2;  // float4 per word pair: 4 or 8
  // bit offset at which position p of a word is masked (after the 8-bit shift when
  // the code lies above bit 23)
  __host__ __device__ static constexpr int shift_pos(int p) {
    return BITS * p + BITS > 24 ? BITS * p - 8 : BITS * p;
  }
  __device__ __forceinline__ static int shift_of(int c) { return shift_pos(c % kWC); }
  // float4 k of a chunk holds, for a = 2*(k / kF4PerPair), kk = k % kF4PerPair:
  // (word a, pos 2kk), (word a+1, pos 2kk), (word a, pos 2kk+1), (word a+1, pos 2kk+1)
  // lane-interleaved layout: float4 k of chunk m at slot ((m/32)*kF4 + k)*32 + m%32,
  // so a warp's lanes (consecutive chunks) read consecutive 16-byte slots
  __device__ __forceinline__ static const ulonglong2* f4(const float* base, int m, int k) {
    return reinterpret_cast<const ulonglong2*>(base) + ((((m >> 5) * kF4 + k) << 5) + (m & 31));
  }
  // float index of column c in the lane-interleaved layout: float4 k of chunk m holds,
  // for the word pair a = word & ~1 and kk = pos / 2, element (pos & 1) * 2 + (word & 1)
  __device__ __forceinline__ static int phys(int c) {
    const int m = c / kCols, r = c % kCols;
    const int word = r / kWC, pos = r % kWC;
    const int k = (word >> 1) * kF4PerPair + (pos >> 1);
    const int e = ((pos & 1) << 1) | (word & 1);
    return ((((m >> 5) * kF4 + k) << 5) + (m & 31)) * 4 + e;
  }
  // (scale,bias) word index of chunk m within its row
  __host__ __device__ __forceinline__ static int sb_index(int m) { return BITS == 4 ? (m >> 1) : m; }

  // One word pair W = {w_a, w_b} against its activation pairs (kF4PerPair float4 at
  // xv[0], xv[32], ... in the interleaved layout), accumulated into acc.
  template <int P>
  __device__ __forceinline__ static void pos(unsigned long long W, unsigned long long V, unsigned long long x,
                                             unsigned long long& acc) {
    if constexpr (P < kWC) {
      constexpr int s = shift_pos(P);
      constexpr unsigned long long m32 = ((1ull << BITS) - 1ull) << s;
      constexpr unsigned long long mask = (m32 << 32) | m32;
      fma2(acc, ((BITS * P + BITS > 24) ? V : W) & mask, x);
    }
  }

  // Word pairs of one or two rows against shared activation pairs.
  template <bool TWO>
  __device__ __forceinline__ static void word_pair2(unsigned long long Wa, unsigned long long Wb,
                                                    const ulonglong2* xv, unsigned long long& acc_a,
                                                    unsigned long long& acc_b) {
    const unsigned long long Va = Wa >> 8;
    const unsigned long long Vb = TWO ? (Wb >> 8) : 0ull;
#pragma unroll
    for (int k = 0; k < kF4PerPair; ++k) {
      const ulonglong2 x = xv[k * 32];
      // positions 2k (x.x) and 2k+1 (x.y)
      switch (k) {
#define FMOE_POS_CASE(K)                                  \
  case K:                                                 \
    pos<2 * K>(Wa, Va, x.x, acc_a);                       \
    pos<2 * K + 1>(Wa, Va, x.y, acc_a);                   \
    if (TWO) pos<2 * K>(Wb, Vb, x.x, acc_b);              \
    if (TWO) pos<2 * K + 1>(Wb, Vb, x.y, acc_b);          \
    break;
        FMOE_POS_CASE(0)
        FMOE_POS_CASE(1)
        FMOE_POS_CASE(2)
        FMOE_POS_CASE(3)
        FMOE_POS_CASE(4)
        FMOE_POS_CASE(5)
        FMOE_POS_CASE(6)
        FMOE_POS_CASE(7)
#undef FMOE_POS_CASE
      }
    }
  }
};

// 2^(P - shift): the pre-scale of an activation met by codes masked at bit `shift`.
__device__ __forceinline__ float prescale_factor(int pre, int shift) {
  return __uint_as_float(static_cast<uint32_t>(127 + pre - shift) << 23);
}

// Largest |v| bit pattern of four floats (sign bits cleared; NaN-free inputs).
__device__ __forceinline__ uint32_t max_abs_bits(float4 v) {
  const uint32_t a = max(__float_as_uint(v.x) & 0x7FFFFFFFu, __float_as_uint(v.y) & 0x7FFFFFFFu);
  const uint32_t b = max(__float_as_uint(v.z) & 0x7FFFFFFFu, __float_as_uint(v.w) & 0x7FFFFFFFu);
  return max(a, b);
}

// (scale, bias) pair word -> floats
__device__ __forceinline__ float sb_scale(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float sb_bias(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Order-preserving map of a double to an unsigned key (larger double -> larger key);
// -0.0 and +0.0 get the same key (they compare equal, so they tie).
__device__ __forceinline__ unsigned long long dkey(double d) {
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(d));
  if (b == 0x8000000000000000ull) b = 0ull;
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Round-to-nearest-even float -> bf16 bits (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

// Round-to-nearest-even double -> bf16 bits in one step (no double rounding).
__device__ __forceinline__ uint16_t f64_to_bf16(double d) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(d));
  const unsigned long long sign = b & 0x8000000000000000ull;
  const unsigned long long mag = b & 0x7FFFFFFFFFFFFFFFull;
  if (mag == 0) return static_cast<uint16_t>(sign >> 48);
  // keep the top 8 significant bits of the 53: drop 45 mantissa bits with RNE
  const unsigned long long drop = 45;
  const unsigned long long half = 1ull << (drop - 1);
  const unsigned long long low = mag & ((1ull << drop) - 1);
  unsigned long long kept = mag >> drop;
  if (low > half || (low == half && (kept & 1))) kept += 1;
  const unsigned long long r = (kept << drop) | sign;
  const float f = static_cast<float>(__longlong_as_double(static_cast<long long>(r)));  // exact
  return static_cast<uint16_t>(__float_as_uint(f) >> 16);
}

}  // namespace fmoe
