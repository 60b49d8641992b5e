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

// Waits for phase `parity` of `bar` to complete, for at most limit_ns.
__device__ __noinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                               uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      atomicOr(err, FMOE_DEVERR_COPY_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------- packed f32x2 FMA
__device__ __forceinline__ void ffma2(float2& acc, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%0, %1};\n\t"
      "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rc;\n\t}"
      : "+f"(acc.x), "+f"(acc.y)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Codes as floats without conversion instructions: a code c masked in place at bit
// offset s (s + bits <= 24) reads, as an IEEE float, exactly c * 2^s * 2^-149 (a
// subnormal or the first normal binade).  The activation multiplying it is stored
// pre-scaled by 2^(kPreExp - s), so every product is code * x * 2^(kPreExp - 149)
// exactly, and the per-chunk sum is rescaled by 2^(149 - kPreExp) once.
constexpr int kPreExp = 100;
constexpr float kUnscale = 562949953421312.0f;  // 2^(149 - kPreExp) = 2^49

__device__ __forceinline__ float cf(uint32_t v) { return __uint_as_float(v); }

// One 32-bit word of codes against its pre-scaled activations.
//  4-bit: columns 8j..8j+7 of the word: xv[0] = cols 0..3, xv[1] = cols 4..7.
//  2-bit: columns 16j..16j+15: xv[0..3].
template <int BITS>
__device__ __forceinline__ void word_fma(uint32_t w, const float4* xv, float2& acc);

template <>
__device__ __forceinline__ void word_fma<4>(uint32_t w, const float4* xv, float2& acc) {
  const uint32_t h = w >> 16;
  ffma2(acc, cf(w & 0xFu), cf(w & 0xF0u), xv[0].x, xv[0].y);
  ffma2(acc, cf(w & 0xF00u), cf(w & 0xF000u), xv[0].z, xv[0].w);
  ffma2(acc, cf(h & 0xFu), cf(h & 0xF0u), xv[1].x, xv[1].y);
  ffma2(acc, cf(h & 0xF00u), cf(h & 0xF000u), xv[1].z, xv[1].w);
}

template <>
__device__ __forceinline__ void word_fma<2>(uint32_t w, const float4* xv, float2& acc) {
  const uint32_t h = w >> 16;
  ffma2(acc, cf(w & 0x3u), cf(w & 0xCu), xv[0].x, xv[0].y);
  ffma2(acc, cf(w & 0x30u), cf(w & 0xC0u), xv[0].z, xv[0].w);
  ffma2(acc, cf(w & 0x300u), cf(w & 0xC00u), xv[1].x, xv[1].y);
  ffma2(acc, cf(w & 0x3000u), cf(w & 0xC000u), xv[1].z, xv[1].w);
  ffma2(acc, cf(h & 0x3u), cf(h & 0xCu), xv[2].x, xv[2].y);
  ffma2(acc, cf(h & 0x30u), cf(h & 0xC0u), xv[2].z, xv[2].w);
  ffma2(acc, cf(h & 0x300u), cf(h & 0xC00u), xv[3].x, xv[3].y);
  ffma2(acc, cf(h & 0x3000u), cf(h & 0xC000u), xv[3].z, xv[3].w);
}

// Chunk geometry: one chunk = 16 bytes of codes = 4 words.
template <int BITS>
struct Chunk {
  static constexpr int kCols = 128 / BITS;        // 32 (4-bit) or 64 (2-bit) columns
  static constexpr int kF4 = kCols / 4;           // float4 per chunk
  static constexpr int kF4PerWord = kF4 / 4;      // 2 or 4
  static constexpr int kGroupsPerChunkLog = 0;
  // shift applied to column c inside its word (where its code is masked)
  __device__ __forceinline__ static int shift_of(int c) { return BITS == 4 ? 4 * (c & 3) : 2 * (c & 7); }
  // index (in floats) of column c in the lane-interleaved activation layout:
  // chunk m, float4 f of the chunk, lane slot m % 32 -> conflict-free LDS.128
  __device__ __forceinline__ static int phys(int c) {
    const int m = c / kCols, f = (c % kCols) >> 2, e = c & 3;
    return ((((m >> 5) * kF4 + f) << 5) + (m & 31)) * 4 + e;
  }
  __device__ __forceinline__ static const float4* f4(const float* base, int m, int f) {
    return reinterpret_cast<const float4*>(base) + ((((m >> 5) * kF4 + f) << 5) + (m & 31));
  }
  // (scale,bias) word index of chunk m within its row
  __device__ __forceinline__ static int sb_index(int m) { return BITS == 4 ? (m >> 1) : m; }
};

__device__ __forceinline__ float prescale_factor(int shift) {
  return __uint_as_float(static_cast<uint32_t>(127 + kPreExp - shift) << 23);
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

// Order-preserving map of a double to an unsigned key (larger double -> larger key).
__device__ __forceinline__ unsigned long long dkey(double d) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(d));
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
