// combine.cu -- weighted combine of the expert outputs.
//
// Gemma 4 MoE walkthrough (yeyulingfeng.com/587419.html) section 7 step 4:
// each token's k expert outputs are summed weighted by its gate weights (the
// per-expert scale is already folded into them); llama-cpp-visual-guide
// lesson 35 adds always-active shared experts, which enter with weight 1.
// The sum is kept in fp32 and rounded to bf16 once.
//
// combine_kernel (the unfused, deterministic path): one block per token
// (grid-stride over tokens); each thread owns 4 hidden columns at a time and
// sums the k+S fp32 rows of y_perm that slot_row names in a fixed order.
// HBM-bound: reads (k+S)*H*4 bytes, writes H*2.
// finalize_kernel (the fused fast path): the w2 epilogue has already added
// every weighted expert row into an fp32 [T,H] accumulator; this rounds it.
// sum_rows_kernel (the fused deterministic path): the w2 epilogue has stored every
// weighted expert row at its (token, choice) position; this pass adds the
// k+S contiguous rows of each token in order and rounds once.  Both paths
// use the same arithmetic (product rounded, then added, in order j), so
// they give bit-identical outputs.
#include "internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256)
combine_kernel(const float4* __restrict__ y_perm,
               const int32_t* __restrict__ slot_row,
               const float* __restrict__ w, int64_t T, int k, int S, int H,
               uint2* __restrict__ out) {
  __shared__ int64_t rows[kMaxTopK + kMaxShared];
  __shared__ float wts[kMaxTopK + kMaxShared];
  const int chunks = H >> 2;  // 4 fp32 per 16-byte chunk
  const int ks = k + S;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < ks) {
      rows[threadIdx.x] = (int64_t)slot_row[t * ks + threadIdx.x] * chunks;
      wts[threadIdx.x] = threadIdx.x < k ? w[t * k + threadIdx.x] : 1.0f;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      // fixed order: routed choices j = 0..k-1, then the shared experts
      // product rounded, then added (no fma), the same arithmetic as the
      // fused path's weighted epilogue followed by sum_rows_kernel
      for (int j = 0; j < ks; ++j) {
        if (rows[j] < 0) continue;  // a slot moe_permute gave no row
        const float4 v = __ldg(y_perm + rows[j] + c);
        const float wt = wts[j];
        a0 = __fadd_rn(a0, __fmul_rn(wt, v.x));
        a1 = __fadd_rn(a1, __fmul_rn(wt, v.y));
        a2 = __fadd_rn(a2, __fmul_rn(wt, v.z));
        a3 = __fadd_rn(a3, __fmul_rn(wt, v.w));
      }
      const __nv_bfloat162 lo = __floats2bfloat162_rn(a0, a1);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(a2, a3);
      uint2 o;
      o.x = *reinterpret_cast<const uint32_t*>(&lo);
      o.y = *reinterpret_cast<const uint32_t*>(&hi);
      out[t * chunks + c] = o;
    }
  }
}

// Sum of the k+S weighted rows of a token, which the fused w2 epilogue has
// stored contiguously, in order j = 0..k+S-1; one bf16 rounding.  Each thread
// owns 4 columns (one float4) of one token at a time, and requests the rows
// of a batch of 8 before it adds the first, so a token with k + S = 8 waits
// for one round trip instead of eight; the additions stay in order j.
__global__ void __launch_bounds__(256)
sum_rows_kernel(const float4* __restrict__ stage, int64_t T, int ks, int H,
                uint2* __restrict__ out, float4* __restrict__ out_f32) {
  pdl_wait();
  pdl_trigger();
  const int c4 = H >> 2;
  const int64_t n = T * c4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += stride) {
    const int64_t t = i / c4;
    const int c = (int)(i - t * c4);
    const float4* src = stage + (t * ks) * (int64_t)c4 + c;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    auto add = [&](const float4& u) {
      a.x = __fadd_rn(a.x, u.x);
      a.y = __fadd_rn(a.y, u.y);
      a.z = __fadd_rn(a.z, u.z);
      a.w = __fadd_rn(a.w, u.w);
    };
    int j = 0;
    for (; j + 8 <= ks; j += 8) {
      float4 u[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) u[q] = __ldg(src + (int64_t)(j + q) * c4);
#pragma unroll
      for (int q = 0; q < 8; ++q) add(u[q]);
    }
    for (; j < ks; ++j) add(__ldg(src + (int64_t)j * c4));
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y);
    const __nv_bfloat162 p1 = __floats2bfloat162_rn(a.z, a.w);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&p0);
    o.y = *reinterpret_cast<const uint32_t*>(&p1);
    out[i] = o;
    if (out_f32) out_f32[i] = a;
  }
}

// out = bf16 RNE of the fp32 accumulator the w2 epilogue added into (and an
// fp32 copy when asked), 8 values per thread-iteration.
__global__ void __launch_bounds__(256)
finalize_kernel(const float4* __restrict__ acc, int64_t n8, uint4* __restrict__ out,
                float4* __restrict__ out_f32) {
  pdl_wait();
  pdl_trigger();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += stride) {
    const float4 a = __ldg(acc + 2 * i);
    const float4 b = __ldg(acc + 2 * i + 1);
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y);
    const __nv_bfloat162 p1 = __floats2bfloat162_rn(a.z, a.w);
    const __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y);
    const __nv_bfloat162 p3 = __floats2bfloat162_rn(b.z, b.w);
    uint4 o;
    o.x = *reinterpret_cast<const uint32_t*>(&p0);
    o.y = *reinterpret_cast<const uint32_t*>(&p1);
    o.z = *reinterpret_cast<const uint32_t*>(&p2);
    o.w = *reinterpret_cast<const uint32_t*>(&p3);
    out[i] = o;
    if (out_f32) {
      out_f32[2 * i] = a;
      out_f32[2 * i + 1] = b;
    }
  }
}

}  // namespace

cudaError_t launch_finalize(const float* acc, int64_t n, __nv_bfloat16* out,
                            float* out_f32, cudaStream_t st, bool pdl) {
  const int64_t n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  const int64_t want = (n8 + 255) / 256;
  const unsigned blocks = (unsigned)(want < 148 * 8 ? want : 148 * 8);
  return launch_ex(finalize_kernel, dim3(blocks), dim3(256), 0, st, pdl,
                   reinterpret_cast<const float4*>(acc), n8,
                   reinterpret_cast<uint4*>(out), reinterpret_cast<float4*>(out_f32));
}

cudaError_t launch_combine(const float* y_perm, const int32_t* slot_row,
                           const float* w, int64_t T, int k, int S, int H,
                           __nv_bfloat16* out, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int64_t blocks = T < 148 * 64 ? T : 148 * 64;
  const int chunks = H / 4;
  const int threads = chunks >= 256 ? 256 : ((chunks + 31) / 32) * 32;
  return launch_ex(combine_kernel, dim3((unsigned)blocks),
                   dim3(threads < 64 ? 64 : threads), 0, st, false,
                   reinterpret_cast<const float4*>(y_perm), slot_row, w, T, k, S, H,
                   reinterpret_cast<uint2*>(out));
}

cudaError_t launch_sum_rows(const float* stage, int64_t T, int ks, int H,
                            __nv_bfloat16* out, float* out_f32, cudaStream_t st,
                            bool pdl) {
  const int64_t n = T * (H / 4);
  if (n == 0) return cudaSuccess;
  const int64_t want = (n + 255) / 256;
  const unsigned blocks = (unsigned)(want < 148 * 8 ? want : 148 * 8);
  return launch_ex(sum_rows_kernel, dim3(blocks), dim3(256), 0, st, pdl,
                   reinterpret_cast<const float4*>(stage), T, ks, H,
                   reinterpret_cast<uint2*>(out), reinterpret_cast<float4*>(out_f32));
}

}  // namespace moe
