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
// descending sort.  The argmax compares order-preserving integer keys of the
// fp32 logits, which rank them exactly as the float comparison does.  The weights are formed in fp64 and rounded once to fp32.
// PER is a template parameter so that a round scans only the entries that
// exist (measured on B200: scanning 16 per lane with E = 128 and k = 8 took
// the prefill route kernel 28 us instead of 22 on 8192 tokens).
#pragma once

#include "internal.cuh"

namespace moe {

// Order-preserving key of a logit: a larger key is a larger value.  -0 is
// keyed as +0 (the two compare equal, so the lower id wins the tie) and NaN
// as 0, below every number: a NaN logit is chosen only when nothing else is
// left (it still yields a valid id).
__device__ __forceinline__ uint32_t route_key(float v) {
  if (v != v) return 0u;
  if (v == 0.0f) v = 0.0f;
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Routing variants of llama-cpp-visual-guide lesson 35 (routing section and
// the expert-group fold): scoring 0 is the softmax over all E logits,
// scoring 1 a sigmoid per expert; with n_group > 1 the experts form n_group
// groups of E / n_group consecutive ids, and a token first keeps its
// topk_group best groups (a group scored by its best expert; ties to the
// lower group id), then picks its k experts among theirs.  Both scores are
// increasing in the logit, so everything is ranked on the fp32 logits.
// (RouteOpt: internal.cuh)

// Routes token row z[0..E) with the calling warp (E <= 32 PER).  Lane j < k
// returns the j-th choice in (*id, *wt); the other lanes return id 0,
// weight 0.
//
// Each round, every lane takes its best untaken entry, and two warp
// reductions (redux.sync) pick the winner: the largest key, then the lowest
// id among the lanes holding it.  The kept groups are picked the same way,
// lane g holding group g's best key.
template <int PER = kMaxExperts / 32>
__device__ __forceinline__ void route_token_warp(const float* __restrict__ z,
                                                 const float* __restrict__ scale,
                                                 int E, int k, int* id, float* wt,
                                                 RouteOpt opt = RouteOpt{0, 1, 1}) {
  constexpr int kPerLane = PER;
  const int lane = threadIdx.x & 31;
  float v[kPerLane];
  uint32_t key[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldg(z + e) : 0.f;
    key[i] = route_key(v[i]);
  }
  // bit i: entry lane + 32 i is not (or no longer) a candidate
  uint32_t gone = 0;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i)
    if (lane + 32 * i >= E) gone |= 1u << i;
  if (opt.n_group > 1) {
    const int gs = E / opt.n_group;
    int grp[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) grp[i] = (lane + 32 * i) / gs;
    // lane g < n_group gets group g's best key
    uint32_t my_g = 0;
    for (int g = 0; g < opt.n_group; ++g) {
      uint32_t part = 0;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i)
        if (!((gone >> i) & 1u) && grp[i] == g && key[i] > part) part = key[i];
      const uint32_t m = __reduce_max_sync(0xffffffffu, part);
      if (lane == g) my_g = m;
    }
    // keep the topk_group best groups (larger key, then lower group id)
    uint32_t keep = 0;
    bool open = lane < opt.n_group;
    for (int r = 0; r < opt.topk_group; ++r) {
      const uint32_t gmax = __reduce_max_sync(0xffffffffu, open ? my_g : 0u);
      const uint32_t cand = (open && my_g == gmax) ? (uint32_t)lane : 0xffffffffu;
      const uint32_t gw = __reduce_min_sync(0xffffffffu, cand);
      keep |= 1u << gw;
      if (lane == (int)gw) open = false;
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i)  // (grp < n_group <= 32 for e < E)
      if (lane + 32 * i < E && !((keep >> grp[i]) & 1u)) gone |= 1u << i;
  }
  float my_v = 0.f;
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    // best untaken entry of this lane: larger key, then lower id (lower i)
    uint32_t bk = 0;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      if (!((gone >> i) & 1u) && (bi < 0 || key[i] > bk)) {
        bk = key[i];
        bi = i;
      }
    }
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, bi >= 0 ? bk : 0u);
    const uint32_t cand = (bi >= 0 && bk == kmax) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
    const int win = (int)__reduce_min_sync(0xffffffffu, cand);
    if ((win & 31) == lane) gone |= 1u << (win >> 5);
    if (lane == j) {
      my_id = win;
      // the winner's value from its key (NaN for key 0)
      my_v = __uint_as_float((kmax & 0x80000000u) ? (kmax & 0x7fffffffu) : ~kmax);
    }
  }
  const float zmax = __shfl_sync(0xffffffffu, my_v, 0);
  // softmax: the closed form over the k chosen logits; sigmoid: each
  // chosen expert's sigmoid, normalised over the k (one exp either way)
  double ex = 0.0;
  if (lane < k) {
    if (opt.scoring == MOE_SCORE_SIGMOID)
      ex = 1.0 / (1.0 + exp(-(double)my_v));
    else
      ex = exp((double)my_v - (double)zmax);
  }
  double den = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  double w = ex / den;
  if (lane < k && scale) w *= (double)__ldg(scale + my_id);
  *id = (lane < k) ? my_id : 0;
  *wt = (lane < k) ? (float)w : 0.f;
}

}  // namespace moe
