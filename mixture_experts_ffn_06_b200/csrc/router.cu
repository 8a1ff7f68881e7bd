// router.cu -- router logits from the residual stream: the step ahead of the
// routing in the Gemma 4 walkthrough (yeyulingfeng.com/587419.html, section
// 3, "Gemma4Router-MoE 的入口") and the Gemma4Router class on the vLLM API
// page.  For each token row r of the residual (bf16):
//   1. RMSNorm without gamma, in fp32, returned in bf16:
//        n_h = bf16(r_h * (1 / sqrt(mean(r^2) + eps)))
//   2. a_h = bf16(n_h * bf16(H^-0.5))
//   3. b_h = bf16(a_h * s_h)          (s: the learned per-dimension scale)
//   4. z_e = sum_h b_h W[e,h] in fp32 (GateLinear: bf16 in, fp32 out).
// mean(r^2) is accumulated in double (a square of a bf16 value is exact in
// it), so its rounding to fp32 gives the same normaliser as the oracle's
// sequential double sum unless the two land on different sides of an fp32
// rounding point, which takes a difference in the 53rd bit; 1/sqrt is the
// IEEE fp32 division and square root, not the approximate reciprocal square
// root.  Steps 2 and 3 multiply two bf16 values, exact in fp32, and round
// once to bf16.  The activations are therefore the oracle's; the logits
// differ from it only by the fp32 accumulation of the projection.
//
// One CTA of 4 warps takes 64 tokens and 128 experts (grid.y covers larger
// E); warp w multiplies its 16 tokens (one 16-row MMA tile of activations)
// by the 128 experts' weight rows (16 n8 tiles) with mma.sync m16n8k16 over
// K = H.  Inside each 32-column chunk of K the column order is permuted so
// that every fragment is one 16-byte load: thread (g, c) takes columns
// [8c, 8c + 8) of token rows g and g + 8 and of expert row g; both operands
// share the order, so the dot products are unchanged.  The activations of a
// chunk are formed in registers from the residual and the scale; the weight
// rows come through L1, which the 4 warps share.
#include <cmath>

#include "internal.cuh"

namespace moe {
namespace {

constexpr int kRtWarps = 4;
constexpr int kRtTokens = 16 * kRtWarps;  // tokens per CTA
constexpr int kRtExperts = 128;           // experts per CTA (16 n8 tiles)

__device__ __forceinline__ void rt_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t bf_round(float f) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Steps 1-3 for one bf16 pair of a token row: bf16(bf16(bf16(x inv) root) s)
__device__ __forceinline__ uint32_t rt_act2(uint32_t x2, uint32_t s2, float inv, float root) {
  uint32_t out = 0;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const float x = half ? bf_hi(x2) : bf_lo(x2);
    const float s = half ? bf_hi(s2) : bf_lo(s2);
    const float n = __uint_as_float(bf_round(__fmul_rn(x, inv)) << 16);
    const float a = __uint_as_float(bf_round(__fmul_rn(n, root)) << 16);
    const uint32_t b = bf_round(__fmul_rn(a, s));
    out |= half ? (b << 16) : b;
  }
  return out;
}

__device__ __forceinline__ uint4 rt_act8(const uint4& x, const uint4& s, float inv, float root) {
  return make_uint4(rt_act2(x.x, s.x, inv, root), rt_act2(x.y, s.y, inv, root),
                    rt_act2(x.z, s.z, inv, root), rt_act2(x.w, s.w, inv, root));
}

__global__ void __launch_bounds__(kRtWarps * 32)
router_logits_kernel(const uint4* __restrict__ x, const uint4* __restrict__ w,
                     const uint4* __restrict__ scale, int64_t T, int H, int E, float eps,
                     float root, float* __restrict__ logits) {
  __shared__ float inv_s[kRtTokens];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, cq = lane & 3;
  const int hv = H >> 3;  // 16-byte vectors per row
  const int64_t t0 = (int64_t)blockIdx.x * kRtTokens;
  const int e0 = blockIdx.y * kRtExperts;
  pdl_wait();
  pdl_trigger();
  // ---- step 1: 1 / sqrt(mean(r^2) + eps) of this warp's 16 tokens
  for (int i = 0; i < 16; ++i) {
    const int64_t t = t0 + warp * 16 + i;
    double ss = 0.0;
    if (t < T) {
      const uint4* row = x + t * hv;
      for (int v = lane; v < hv; v += 32) {
        const uint4 q = __ldg(row + v);
        const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const double lo = bf_lo(wd[j]), hi = bf_hi(wd[j]);
          ss = fma(lo, lo, ss);
          ss = fma(hi, hi, ss);
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) {
      const float var = (float)(ss / (double)H);
      inv_s[warp * 16 + i] = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps)));
    }
  }
  __syncwarp();
  // ---- steps 2-4: this warp's 16 tokens x 128 experts over K = H
  const int64_t ta = t0 + warp * 16 + gq, tb = ta + 8;  // A rows g and g + 8
  const bool va = ta < T, vb = tb < T;
  const float inv_a = inv_s[warp * 16 + gq], inv_b = inv_s[warp * 16 + gq + 8];
  const uint4* xa = x + (va ? ta : 0) * hv;
  const uint4* xb = x + (vb ? tb : 0) * hv;
  float acc[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
  const int nch = (H + 31) >> 5;
  for (int ch = 0; ch < nch; ++ch) {
    const int v = ch * 4 + cq;  // 16-byte column group of this thread
    const bool vc = v < hv;
    const uint4 s = vc ? __ldg(scale + v) : z4;
    const uint4 a0 = va && vc ? rt_act8(__ldg(xa + v), s, inv_a, root) : z4;
    const uint4 a8 = vb && vc ? rt_act8(__ldg(xb + v), s, inv_b, root) : z4;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int e = e0 + j * 8 + gq;  // B column (expert) of this thread
      const uint4 b = (e < E && vc) ? __ldg(w + (int64_t)e * hv + v) : z4;
      rt_mma(acc[j], a0.x, a8.x, a0.y, a8.y, b.x, b.y);
      rt_mma(acc[j], a0.z, a8.z, a0.w, a8.w, b.z, b.w);
    }
  }
  // ---- fragment element e: token row g (+8 for e >= 2), expert 2c + e % 2
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int e = e0 + j * 8 + 2 * cq;
    if (va && e < E) logits[ta * E + e] = acc[j][0];
    if (va && e + 1 < E) logits[ta * E + e + 1] = acc[j][1];
    if (vb && e < E) logits[tb * E + e] = acc[j][2];
    if (vb && e + 1 < E) logits[tb * E + e + 1] = acc[j][3];
  }
}

}  // namespace

float router_root(int H) {
  // bf16(fl(H^-0.5)): the fp32 constant cast to bf16 (round to nearest even)
  const float r = (float)std::pow((double)H, -0.5);
  return __bfloat162float(__float2bfloat16_rn(r));
}

cudaError_t launch_router_logits(const __nv_bfloat16* x, const __nv_bfloat16* w_router,
                                 const __nv_bfloat16* scale, int64_t T, int H, int E,
                                 float eps, float* logits, cudaStream_t st, bool pdl) {
  if (T == 0) return cudaSuccess;
  const dim3 grid((unsigned)((T + kRtTokens - 1) / kRtTokens),
                  (unsigned)((E + kRtExperts - 1) / kRtExperts));
  return launch_ex(router_logits_kernel, grid, dim3(kRtWarps * 32), 0, st, pdl,
                   reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(w_router),
                   reinterpret_cast<const uint4*>(scale), T, H, E, eps, router_root(H),
                   logits);
}

}  // namespace moe
