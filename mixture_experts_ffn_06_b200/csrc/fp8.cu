// fp8.cu -- the e4m3 side of the layer with FP8 experts.
//
// Per-expert FP8 checkpoints (the sglang PR on Gemma 4 FP8 per-expert
// loading; load_weights on the vLLM API page) store each expert's gate, up
// and down weights with a weight_scale.  Here a weight is an e4m3 code times
// one fp32 scale per output row, and the activations are quantised per row
// when the layer runs ("FP8-Dynamic"):
//   s = fl32(amax / 448) for a row whose largest |value| is amax (1 for an
//   all-zero row), code = e4m3(fl32(v / s)), rounded to the nearest value,
//   ties to even, saturating at +-448 (cvt.rn.satfinite.e4m3x2.f32).
// Every step is an IEEE fp32 operation, so the codes and scales are those of
// any other implementation of the same steps, bit for bit.
//
//   quantize_rows   one warp per bf16 row: the row's amax, then its codes
//                   (16-byte loads, 8-byte stores); rows whose slot is -1
//                   (padding rows of h) are skipped;
//   gather_fp8      the token rows of x's codes into the permuted rows of
//                   the routed experts (a warp per row, 16-byte vectors), and
//                   every row's scale, shared experts' rows included (their
//                   codes are read from x's codes by the GEMM itself).
#include "internal.cuh"

namespace moe {
namespace {

// two fp32 values to two e4m3 codes: lo in the low byte, hi in the high byte
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void bf16x8(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__global__ void __launch_bounds__(256)
quantize_rows_kernel(const uint4* __restrict__ src, int64_t rows, int cols,
                     uint2* __restrict__ codes, float* __restrict__ scales,
                     const int32_t* __restrict__ rows_used,
                     const int32_t* __restrict__ slots) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t n = rows_used ? (int64_t)*rows_used : rows;
  const int vec = cols >> 3;  // 8 values per 16-byte vector
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n;
       r += warps) {
    if (slots && slots[r] < 0) continue;
    const uint4* row = src + r * vec;
    float amax = 0.0f;
    for (int c = lane; c < vec; c += 32) {
      float f[8];
      bf16x8(__ldg(row + c), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    uint2* out = codes + r * vec;
    for (int c = lane; c < vec; c += 32) {
      float f[8];
      bf16x8(__ldg(row + c), f);
      uint2 o;
      o.x = (uint32_t)e4m3x2(f[0] / s, f[1] / s) | ((uint32_t)e4m3x2(f[2] / s, f[3] / s) << 16);
      o.y = (uint32_t)e4m3x2(f[4] / s, f[5] / s) | ((uint32_t)e4m3x2(f[6] / s, f[7] / s) << 16);
      out[c] = o;
    }
    if (lane == 0) scales[r] = s;
  }
}

__global__ void __launch_bounds__(256, 4)
gather_fp8_kernel(const uint4* __restrict__ xq, const float* __restrict__ sx,
                  const int32_t* __restrict__ sorted_slots,
                  const int32_t* __restrict__ offsets, int E, int G, int64_t T, int k,
                  int H, uint4* __restrict__ x_perm, float* __restrict__ a_scale,
                  uint4* __restrict__ acc, int64_t n_acc4) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  pdl_wait();
  pdl_trigger();
  const int64_t rows = offsets[G], routed_rows = offsets[E];
  const int chunks = H >> 4;  // 16 codes per 16-byte chunk
  const int64_t R = T * k;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += warps) {
    const int s = sorted_slots[r];
    if (s < 0) continue;
    const int64_t t = (s < R) ? (int64_t)s / k : ((int64_t)s - R) % T;
    if (lane == 0) a_scale[r] = __ldg(sx + t);
    if (r >= routed_rows) continue;  // a shared expert reads x's codes itself
    const uint4* src = xq + t * chunks;
    uint4* dst = x_perm + r * chunks;
    // up to eight 16-byte loads in flight per lane before the stores
    for (int c0 = 0; c0 < chunks; c0 += 256) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c0 + lane + 32 * j < chunks) v[j] = __ldg(src + c0 + lane + 32 * j);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c0 + lane + 32 * j < chunks) __stcs(dst + c0 + lane + 32 * j, v[j]);
    }
  }
  // zero the fp32 accumulator the w2 epilogue adds into (fast combine)
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_acc4;
       i += stride)
    acc[i] = z;
}

}  // namespace

cudaError_t launch_quantize_rows(const __nv_bfloat16* src, int64_t rows, int cols,
                                 uint8_t* codes, float* scales, const int32_t* rows_used,
                                 const int32_t* slots, cudaStream_t st, bool pdl) {
  const int64_t want = (rows + 7) / 8;
  const unsigned blocks = (unsigned)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
  return launch_ex(quantize_rows_kernel, dim3(blocks), dim3(256), 0, st, pdl,
                   reinterpret_cast<const uint4*>(src), rows, cols,
                   reinterpret_cast<uint2*>(codes), scales, rows_used, slots);
}

cudaError_t launch_gather_fp8(const uint8_t* xq, const float* sx, const int32_t* sorted_slots,
                              const int32_t* offsets, int E, int G, int64_t T, int k, int H,
                              int64_t cap, uint8_t* x_perm, float* a_scale, float* acc,
                              int64_t n_acc, cudaStream_t st, bool pdl) {
  const int64_t want = (cap + 7) / 8;
  const unsigned blocks = (unsigned)(want < 148 * 16 ? want : 148 * 16);
  return launch_ex(gather_fp8_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st, pdl,
                   reinterpret_cast<const uint4*>(xq), sx, sorted_slots, offsets, E, G, T,
                   k, H, reinterpret_cast<uint4*>(x_perm), a_scale,
                   reinterpret_cast<uint4*>(acc), acc ? n_acc / 4 : (int64_t)0);
}

}  // namespace moe
