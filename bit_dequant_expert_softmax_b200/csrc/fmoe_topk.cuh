// Top-K selection by ranks, shared by the single-token and the batched kernels.
//
// The K largest router logits, ordered by logit descending with ties to the lower
// expert index (the selection of the pages' softmax-then-top-K -- intelliparadigm.com,
// section 2.1 router snippet; tinai-dev README, "Pipeline mỗi lớp" -- the softmax is
// monotone, so ranking logits or probabilities picks the same experts), compared
// through the order-preserving 64-bit key of each fp64 logit.  Two levels of ranks,
// no dependent reductions: every expert's rank within its group of 32 consecutive
// experts, then every group's K best ranked among all candidates.
#pragma once

#include "fmoe_device.cuh"

namespace fmoe {

// Router logit of one row from its nq column-split partial sums (written by other
// blocks, read from L2), summed in a fixed order.
__device__ __forceinline__ double router_logit(const double* lp, int nq) {
  if (nq == 4) {
    const double2 a = __ldcg(reinterpret_cast<const double2*>(lp));
    const double2 b = __ldcg(reinterpret_cast<const double2*>(lp + 2));
    return ((a.x + a.y) + b.x) + b.y;
  }
  double l = 0.0;
  for (int q = 0; q < nq; ++q) l += __ldcg(lp + q);
  return l;
}

// skey[e], e < E: keys of the logits.  ckey / cidx: scratch of ceil(E/32)*K entries.
// Writes sel[0..K).  Called by every thread of a block of NTHREADS threads; ends
// synchronised.
template <int NTHREADS>
__device__ __forceinline__ void rank_topk(const unsigned long long* skey, unsigned long long* ckey, int* cidx,
                                          int E, int K, int* sel) {
  for (int e = threadIdx.x; e < E; e += NTHREADS) {
    const unsigned long long ke = skey[e];
    const int b0 = e & ~31;
    const int nb = min(32, E - b0);
    int rank = 0;
    if (nb == 32) {
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const unsigned long long kj = skey[b0 + j];
        rank += static_cast<int>(kj > ke) | (static_cast<int>(kj == ke) & static_cast<int>(b0 + j < e));
      }
    } else {
      for (int j = 0; j < nb; ++j) {
        const unsigned long long kj = skey[b0 + j];
        rank += static_cast<int>(kj > ke) | (static_cast<int>(kj == ke) & static_cast<int>(b0 + j < e));
      }
    }
    if (rank < K) {
      const int slot = (e >> 5) * K + rank;
      ckey[slot] = ke;
      cidx[slot] = e;
    }
  }
  const int ngroups = (E + 31) >> 5;
  for (int c = threadIdx.x; c < ngroups * K; c += NTHREADS) {
    const int gsz = min(32, E - (c / K) * 32);
    if (c % K >= gsz) {  // a short last group has fewer than K members
      ckey[c] = 0;
      cidx[c] = 0x7fffffff;
    }
  }
  __syncthreads();
  // every candidate's rank is counted by kStripe consecutive lanes, each over every
  // kStripe-th candidate, and summed by shuffles
  constexpr int kStripe = 8;
  const int ncand = ngroups * K;
  for (int base = 0; base < ncand * kStripe; base += NTHREADS) {  // block-uniform trip count
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
    if (c < ncand && part == 0 && kc != 0 && rank < K) sel[rank] = ic;
  }
  __syncthreads();
}

// Warp-level renormalised softmax weight of rank `lane` (lanes < K): exp(l_k - l_0)
// over the sum of the K terms, in double.  Every lane of the warp calls it.
__device__ __forceinline__ double topk_weight(const double* slog, const int* sel, int K, int lane) {
  const int mysel = lane < K ? sel[lane] : sel[0];
  const double l0 = slog[sel[0]];
  const double ek = lane < K ? exp(slog[mysel] - l0) : 0.0;
  const double den = warp_sum_d(ek);
  return ek / den;
}

// The same weight from the selection's logits already in rank order (l[0] largest).
__device__ __forceinline__ double topk_weight_sorted(const double* l, int K, int lane) {
  const double ek = lane < K ? exp(l[lane] - l[0]) : 0.0;
  const double den = warp_sum_d(ek);
  return ek / den;
}

}  // namespace fmoe
