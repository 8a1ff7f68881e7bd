// combine.cu -- weighted combine of the expert outputs.
//
// Gemma 4 MoE walkthrough (yeyulingfeng.com/587419.html) section 7 step 4:
// each token's k expert outputs are summed weighted by its gate weights (the
// per-expert scale is already folded into them); llama-cpp-visual-guide
// lesson 35 adds always-active shared experts, which enter with weight 1.
// The sum is kept in fp32 and rounded to bf16 once.
//
// One block per token (grid-stride over tokens); each thread owns 8 hidden
// columns (one 16-byte vector) at a time and gathers the k+S rows of y_perm
// that slot_row names.  HBM-bound: reads (k+S)*H*2 bytes, writes H*2.
#include "internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4& v,
                                           float wt) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(p[i]);
    acc[2 * i] = fmaf(wt, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(wt, f.y, acc[2 * i + 1]);
  }
}

__global__ void __launch_bounds__(256)
combine_kernel(const uint4* __restrict__ y_perm,
               const int32_t* __restrict__ slot_row,
               const float* __restrict__ w, int64_t T, int k, int S, int H,
               uint4* __restrict__ out) {
  __shared__ int64_t rows[kMaxTopK + kMaxShared];
  __shared__ float wts[kMaxTopK + kMaxShared];
  const int chunks = H >> 3;
  const int ks = k + S;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < ks) {
      rows[threadIdx.x] = (int64_t)slot_row[t * ks + threadIdx.x] * chunks;
      wts[threadIdx.x] = threadIdx.x < k ? w[t * k + threadIdx.x] : 1.0f;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      int j = 0;
      for (; j + 4 <= ks; j += 4) {
        const uint4 v0 = __ldg(y_perm + rows[j] + c);
        const uint4 v1 = __ldg(y_perm + rows[j + 1] + c);
        const uint4 v2 = __ldg(y_perm + rows[j + 2] + c);
        const uint4 v3 = __ldg(y_perm + rows[j + 3] + c);
        acc_bf16x8(acc, v0, wts[j]);
        acc_bf16x8(acc, v1, wts[j + 1]);
        acc_bf16x8(acc, v2, wts[j + 2]);
        acc_bf16x8(acc, v3, wts[j + 3]);
      }
      for (; j < ks; ++j) acc_bf16x8(acc, __ldg(y_perm + rows[j] + c), wts[j]);
      uint4 o;
      __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        op[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      out[t * chunks + c] = o;
    }
  }
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* y_perm, const int32_t* slot_row,
                           const float* w, int64_t T, int k, int S, int H,
                           __nv_bfloat16* out, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int64_t blocks = T < 148 * 64 ? T : 148 * 64;
  const int threads = (H / 8) >= 256 ? 256 : (((H / 8) + 31) / 32) * 32;
  combine_kernel<<<(unsigned)blocks, threads < 64 ? 64 : threads, 0, st>>>(
      reinterpret_cast<const uint4*>(y_perm), slot_row, w, T, k, S, H,
      reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace moe
