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
// Design: the step reads and writes the whole state once (8 MB at 64 x 128 x 128, the
// HBM bound) and does ~4 flops per element.  One warp owns a row i of one head: it
// holds the row (16-byte loads, lane-strided, coalesced) and the head's k and q in
// registers, reduces u_i = alpha * (S_i . k) by shuffles, forms the updated row, reduces
// o_i = S'_i . q, and writes the row back in place.  No shared memory, no barriers.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fmoe {

constexpr int kGdnWarps = 8;                // warps (rows) per block
constexpr int kGdnMaxChunks = 4;            // 128-column chunks a row may have (dk <= 512)

__global__ void __launch_bounds__(kGdnWarps * 32)
    gdn_step_kernel(float* __restrict__ S, const float* __restrict__ q, const float* __restrict__ k,
                    const float* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
                    float* __restrict__ o, int heads, int dk, int dv) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kGdnWarps + (threadIdx.x >> 5);
  if (row >= static_cast<long long>(heads) * dv) return;
  const int h = static_cast<int>(row / dv), i = static_cast<int>(row % dv);
  float4* srow = reinterpret_cast<float4*>(S + row * dk);
  const float4* kh = reinterpret_cast<const float4*>(k + static_cast<size_t>(h) * dk);
  const float4* qh = reinterpret_cast<const float4*>(q + static_cast<size_t>(h) * dk);
  const int n4 = dk / 4;
  float4 sv[kGdnMaxChunks], kv[kGdnMaxChunks], qv[kGdnMaxChunks];
  const float a = __ldg(alpha + h), b = __ldg(beta + h);
  // every load of the row and the head's vectors in flight together
#pragma unroll
  for (int c = 0; c < kGdnMaxChunks; ++c) {
    const int j = lane + 32 * c;
    const bool in = j < n4;
    sv[c] = in ? srow[j] : make_float4(0.f, 0.f, 0.f, 0.f);
    kv[c] = in ? __ldg(kh + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    qv[c] = in ? __ldg(qh + j) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // S <- alpha S; u_i = S_i . k
  float u = 0.f;
#pragma unroll
  for (int c = 0; c < kGdnMaxChunks; ++c) {
    sv[c] = make_float4(a * sv[c].x, a * sv[c].y, a * sv[c].z, a * sv[c].w);
    u = fmaf(sv[c].x, kv[c].x, u);
    u = fmaf(sv[c].y, kv[c].y, u);
    u = fmaf(sv[c].z, kv[c].z, u);
    u = fmaf(sv[c].w, kv[c].w, u);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
  // S_i <- S_i + beta (v_i - u_i) k; o_i = S_i . q
  const float d = b * (__ldg(v + static_cast<size_t>(h) * dv + i) - u);
  float oi = 0.f;
#pragma unroll
  for (int c = 0; c < kGdnMaxChunks; ++c) {
    const int j = lane + 32 * c;
    sv[c] = make_float4(fmaf(d, kv[c].x, sv[c].x), fmaf(d, kv[c].y, sv[c].y), fmaf(d, kv[c].z, sv[c].z),
                        fmaf(d, kv[c].w, sv[c].w));
    oi = fmaf(sv[c].x, qv[c].x, oi);
    oi = fmaf(sv[c].y, qv[c].y, oi);
    oi = fmaf(sv[c].z, qv[c].z, oi);
    oi = fmaf(sv[c].w, qv[c].w, oi);
    if (j < n4) srow[j] = sv[c];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) oi += __shfl_xor_sync(0xffffffffu, oi, off);
  if (lane == 0) o[static_cast<size_t>(h) * dv + i] = oi;
}

}  // namespace fmoe
