// route_impl.cuh -- routing of one token by one warp, shared by the
// prefill route kernel and the decode path's first kernel.
//
// Gemma 4 MoE walkthrough (yeyulingfeng.com/587419.html) section 4: top-k on
// the raw logits, softmax over all E, mask, renormalise; section 5: times
// per_expert_scale[id] after the renormalisation.  Section 4 also shows that
// the renormalised masked softmax equals a softmax over the k selected logits
// alone (the all-E denominator cancels), so that closed form is evaluated:
// it needs no pass over the unselected experts and cannot underflow.
//
// Lane l holds logits e = l, l+32, ... (PER per lane, E <= 32 PER; at most
// 16 for E <= 512).  Each of the k rounds is a warp-wide argmax under
// (larger logit, then lower id), so ids come out in the order of a stable
// descending sort.  The weights are formed in fp64 and rounded once to fp32.
// PER is a template parameter so that a round scans only the entries that
// exist (measured on B200: scanning 16 per lane with E = 128 and k = 8 took
// the prefill route kernel 28 us instead of 22 on 8192 tokens).
#pragma once

#include "internal.cuh"

namespace moe {

// true if (va, ia) precedes (vb, ib): larger value, ties to the lower id.
// NaN never precedes anything, so a NaN logit is chosen only when nothing
// else is left (it still yields a valid id).
__device__ __forceinline__ bool route_precedes(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Routes token row z[0..E) with the calling warp (E <= 32 PER).  Lane j < k
// returns the j-th choice in (*id, *wt); the other lanes return id 0,
// weight 0.
template <int PER = kMaxExperts / 32>
__device__ __forceinline__ void route_token_warp(const float* __restrict__ z,
                                                 const float* __restrict__ scale,
                                                 int E, int k, int* id, float* wt) {
  constexpr int kPerLane = PER;
  const int lane = threadIdx.x & 31;
  float v[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldg(z + e) : -INFINITY;
  }
  uint32_t taken = 0;  // bit i: expert lane+32i already chosen
  float my_v = 0.f;
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u)) {
        if (bi == 0x7fffffff || route_precedes(v[i], e, bv, bi)) {
          bv = v[i];
          bi = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (oi != 0x7fffffff && (bi == 0x7fffffff || route_precedes(ov, oi, bv, bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) {
      my_v = bv;
      my_id = bi;
    }
  }
  const float zmax = __shfl_sync(0xffffffffu, my_v, 0);
  const double ex = (lane < k) ? exp((double)my_v - (double)zmax) : 0.0;
  double den = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  double w = ex / den;
  if (lane < k && scale) w *= (double)__ldg(scale + my_id);
  *id = (lane < k) ? my_id : 0;
  *wt = (lane < k) ? (float)w : 0.f;
}

}  // namespace moe
