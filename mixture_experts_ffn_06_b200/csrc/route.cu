// route.cu -- warp-per-token routing kernel.
//
// Gemma 4 MoE walkthrough (yeyulingfeng.com/587419.html) section 4: top-k on
// the raw logits, softmax over all E, mask, renormalise; section 5: multiply
// by per_expert_scale[id] after the renormalisation.  The same section shows
// that the renormalised masked softmax equals a softmax over the k selected
// logits alone (the all-E denominator cancels), so the kernel evaluates that
// closed form: it needs no pass over the unselected experts and cannot
// underflow the way a softmax over all E can.
//
// One warp owns one token.  Lane l holds logits e = l, l+32, ... in registers
// (E <= 512, so at most 16 per lane).  Each of the k rounds is a warp-wide
// argmax under the order (larger logit first, then lower id), so ids are
// bit-exact with a stable descending sort.  The weights are formed in fp64
// and rounded once to fp32.
#include "internal.cuh"

namespace moe {
namespace {

constexpr int kMaxPerLane = kMaxExperts / 32;

// true if (va, ia) precedes (vb, ib): larger value, ties to the lower id.
// NaN never precedes anything, so a NaN logit is chosen only when nothing
// else is left (it still yields a valid id).
__device__ __forceinline__ bool precedes(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(256)
route_kernel(const float* __restrict__ logits, const float* __restrict__ scale,
             int64_t T, int E, int k, int32_t* __restrict__ ids,
             float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* z = logits + t * E;

  float v[kMaxPerLane];
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldg(z + e) : -INFINITY;
  }
  uint32_t taken = 0;  // bit i: expert lane+32i already chosen

  float my_v = 0.f;  // lane j < k keeps the j-th choice
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u)) {
        if (bi == 0x7fffffff || precedes(v[i], e, bv, bi)) {
          bv = v[i];
          bi = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (oi != 0x7fffffff &&
          (bi == 0x7fffffff || precedes(ov, oi, bv, bi))) {
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

  // closed form over the selected logits, in fp64
  const float zmax = __shfl_sync(0xffffffffu, my_v, 0);
  double ex = (lane < k) ? exp((double)my_v - (double)zmax) : 0.0;
  double den = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    den += __shfl_xor_sync(0xffffffffu, den, off);
  if (lane < k) {
    double wt = ex / den;
    if (scale) wt *= (double)__ldg(scale + my_id);
    ids[t * k + lane] = my_id;
    w[t * k + lane] = (float)wt;
  }
}

}  // namespace

cudaError_t launch_route(const float* logits, const float* scale, int64_t T,
                         int E, int k, int32_t* ids, float* w,
                         cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (T + warps - 1) / warps;
  route_kernel<<<(unsigned)blocks, warps * 32, 0, st>>>(logits, scale, T, E, k,
                                                       ids, w);
  return cudaGetLastError();
}

}  // namespace moe
