// GatedDeltaNet step for sm_100a: the state update of the linear-attention layers.
//
// Per head h and token: the state S_h [dv][dk] (fp32, row-major, dk contiguous) is
// scaled by the gate alpha_h, read at the key k_h, moved towards the value v_h by a
// rank-1 update of strength beta_h and read at the query q_h:
//   S <- alpha S;  u = S k;  S <- S + beta (v - u) k^T;  o = S q.
// The pages run this step with BLAS on 64 heads x 128 x 128 (hotdry.top, "Metal
// GPU管线", linear-attention paragraph: a scaling, matrix-vector products and a rank-1
// update); the composition is the gated delta rule of GatedDeltaNet.
//
// Design: the step reads and writes the whole state once (8.4 MB at 64 x 128 x 128, the
// HBM bound) and does ~4 flops per element, so what matters is how many bytes are in
// flight.  A warp owns R consecutive rows of one head (R = 8 for dk <= 128, 2 for dk up
// to 512): it issues the 16-byte loads of all its rows (lane-strided, coalesced) and of
// the head's k and q before any arithmetic, then per row reduces
// u_i = (alpha S_i) . k by shuffles, forms the updated row, reduces o_i = S'_i . q and
// writes the row back in place.  No shared memory, no barriers.  The launch lets the
// next kernel on the stream start (programmatic dependent launch) and waits for its
// predecessor before reading anything.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fmoe {

constexpr int kGdnWarps = 8;                // warps per block
constexpr int kGdnMaxChunks = 4;            // 128-column chunks a row may have (dk <= 512)

// MAXC: 128-column chunks a row has at most; R: rows per warp.
template <int MAXC, int R>
__global__ void __launch_bounds__(kGdnWarps * 32)
    gdn_step_kernel(float* __restrict__ S, const float* __restrict__ q, const float* __restrict__ k,
                    const float* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
                    float* __restrict__ o, int heads, int dk, int dv) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long wid = static_cast<long long>(blockIdx.x) * kGdnWarps + (threadIdx.x >> 5);
  const int per_head = (dv + R - 1) / R;
  const long long h64 = wid / per_head;
  if (h64 >= heads) return;
  const int h = static_cast<int>(h64), i0 = static_cast<int>(wid % per_head) * R;
  const int n4 = dk / 4;
  const float4* kh = reinterpret_cast<const float4*>(k + static_cast<size_t>(h) * dk);
  const float4* qh = reinterpret_cast<const float4*>(q + static_cast<size_t>(h) * dk);
  float4* head = reinterpret_cast<float4*>(S + static_cast<size_t>(h) * dv * dk);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 kv[MAXC], qv[MAXC], sv[R][MAXC];
  // every load of the warp's rows and the head's vectors in flight together
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int j = lane + 32 * c;
    const bool in = j < n4;
    kv[c] = in ? __ldg(kh + j) : z;
    qv[c] = in ? __ldg(qh + j) : z;
#pragma unroll
    for (int r = 0; r < R; ++r) sv[r][c] = (in && i0 + r < dv) ? head[static_cast<size_t>(i0 + r) * n4 + j] : z;
  }
  const float a = __ldg(alpha + h), b = __ldg(beta + h);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (i0 + r >= dv) break;  // warp-uniform
    // S <- alpha S; u_i = S_i . k
    float u = 0.f;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      sv[r][c] = make_float4(a * sv[r][c].x, a * sv[r][c].y, a * sv[r][c].z, a * sv[r][c].w);
      u = fmaf(sv[r][c].x, kv[c].x, u);
      u = fmaf(sv[r][c].y, kv[c].y, u);
      u = fmaf(sv[r][c].z, kv[c].z, u);
      u = fmaf(sv[r][c].w, kv[c].w, u);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
    // S_i <- S_i + beta (v_i - u_i) k; o_i = S_i . q
    const int i = i0 + r;
    const float d = b * (__ldg(v + static_cast<size_t>(h) * dv + i) - u);
    float oi = 0.f;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int j = lane + 32 * c;
      sv[r][c] = make_float4(fmaf(d, kv[c].x, sv[r][c].x), fmaf(d, kv[c].y, sv[r][c].y),
                             fmaf(d, kv[c].z, sv[r][c].z), fmaf(d, kv[c].w, sv[r][c].w));
      oi = fmaf(sv[r][c].x, qv[c].x, oi);
      oi = fmaf(sv[r][c].y, qv[c].y, oi);
      oi = fmaf(sv[r][c].z, qv[c].z, oi);
      oi = fmaf(sv[r][c].w, qv[c].w, oi);
      if (j < n4) head[static_cast<size_t>(i) * n4 + j] = sv[r][c];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) oi += __shfl_xor_sync(0xffffffffu, oi, off);
    if (lane == 0) o[static_cast<size_t>(h) * dv + i] = oi;
  }
}

}  // namespace fmoe
