// gemma_block.cu -- the MoE block of a Gemma 4 decoder layer (Gemma 4
// walkthrough, yeyulingfeng.com/587419.html, section 1: the DecoderLayer
// forward; section 7: the tensor flow).  From the residual x [T,H] bf16:
//   h1  = post_ff_norm_1( mlp( pre_ff_norm(x) ) )        dense GeGLU MLP
//   h2  = post_ff_norm_2( moe( pre_ff_norm_2(x), router(x) ) )
//   out = post_ff_norm( h1 + h2 ) + x                    unweighted sum
// Each norm is the standard RMSNorm with a gamma (section 3), computed in
// fp32 and returned in bf16; every module hands bf16 to the next.
//
// The two branches read the same residual and meet only in the last step,
// so they run side by side (section 1: the dense MLP and the MoE in
// parallel):
//   pre_norm_kernel    one block per token: both input norms from one read
//                      of x (and zeroes the dense MLP's one-expert logits);
//   then, forked onto a second stream of the library's own:
//     moe_forward_ex   the dense MLP as the one-expert, weight-1 case of the
//                      layer (E = 1, k = 1, I = I_dense) -> y1;
//   while the caller's stream runs
//     moe_forward_ex   the router on x, then the MoE on pre_ff_norm_2(x) -> y2;
//   joined back:
//   post_norm_kernel   one block per token: the two output norms, their
//                      bf16 sum, the last norm and the residual add.
// The fork and the join are an event each, so the pattern holds under CUDA
// graph capture as well (the second stream joins the capture).  Each branch
// has its own layer workspace; the MoE branch's sits at offset 0, so its
// error word is the block's, and post_norm moves the dense branch's error
// code (if any) into it.
#include <mutex>

#include "internal.cuh"

namespace moe {
namespace {

constexpr int kNormThreads = 256;

// Sum over the block, in double, in a fixed order (lane tree, then warps).
__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read by the previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
  return s;
}

// 1 / sqrt(mean of squares + eps) in fp32 (IEEE square root and division),
// the mean taken in double and rounded once to fp32.
__device__ __forceinline__ float rms_inv(double ss, int H, float eps) {
  const float var = (float)(ss / (double)H);
  return 1.0f / sqrtf(var + eps);
}

__device__ __forceinline__ float bf(__nv_bfloat16 v) { return __bfloat162float(v); }

// y = bf16( fl( fl(x * inv) * g ) )
__device__ __forceinline__ __nv_bfloat16 norm_elem(float x, float inv, __nv_bfloat16 g) {
  return __float2bfloat16_rn(__fmul_rn(__fmul_rn(x, inv), bf(g)));
}

__global__ void __launch_bounds__(kNormThreads)
pre_norm_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ g1,
                const __nv_bfloat16* __restrict__ g2, int H, float eps,
                __nv_bfloat16* __restrict__ a1, __nv_bfloat16* __restrict__ a2,
                float* __restrict__ zero_logits, uint32_t* __restrict__ dense_err) {
  __shared__ double red[kNormThreads / 32];
  const int64_t t = blockIdx.x;
  const __nv_bfloat16* xr = x + t * H;
  double ss = 0.0;
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const double v = (double)bf(xr[h]);
    ss += v * v;
  }
  const float inv = rms_inv(block_sum(ss, red), H, eps);
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const float v = bf(xr[h]);
    a1[t * H + h] = norm_elem(v, inv, g1[h]);
    a2[t * H + h] = norm_elem(v, inv, g2[h]);
  }
  if (threadIdx.x == 0) zero_logits[t] = 0.0f;
  // the dense branch's error word starts clear (post_norm moved out what
  // the previous call left)
  if (t == 0 && threadIdx.x == 0) *dense_err = 0u;
}

__global__ void __launch_bounds__(kNormThreads)
post_norm_kernel(const __nv_bfloat16* __restrict__ y1, const __nv_bfloat16* __restrict__ y2,
                 const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ g1,
                 const __nv_bfloat16* __restrict__ g2, const __nv_bfloat16* __restrict__ g,
                 int H, float eps, __nv_bfloat16* __restrict__ out,
                 float* __restrict__ out_f32, uint32_t* __restrict__ dense_err,
                 uint32_t* __restrict__ block_err) {
  __shared__ double red[kNormThreads / 32];
  const int64_t t = blockIdx.x;
  if (t == 0 && threadIdx.x == 0) {
    const uint32_t e = atomicExch(dense_err, 0u);
    if (e) atomicCAS(block_err, 0u, e);
  }
  const __nv_bfloat16* r1 = y1 + t * H;
  const __nv_bfloat16* r2 = y2 + t * H;
  double s1 = 0.0, s2 = 0.0;
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const double u = (double)bf(r1[h]), v = (double)bf(r2[h]);
    s1 += u * u;
    s2 += v * v;
  }
  const float inv1 = rms_inv(block_sum(s1, red), H, eps);
  const float inv2 = rms_inv(block_sum(s2, red), H, eps);
  // h = bf16( fl(h1 + h2) ), recomputed in the second pass
  auto hsum = [&](int h) {
    const float a = bf(norm_elem(bf(r1[h]), inv1, g1[h]));
    const float b = bf(norm_elem(bf(r2[h]), inv2, g2[h]));
    return bf(__float2bfloat16_rn(__fadd_rn(a, b)));
  };
  double s3 = 0.0;
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const double v = (double)hsum(h);
    s3 += v * v;
  }
  const float inv3 = rms_inv(block_sum(s3, red), H, eps);
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const float z = bf(norm_elem(hsum(h), inv3, g[h]));
    const float o = __fadd_rn(z, bf(x[t * H + h]));
    out[t * H + h] = __float2bfloat16_rn(o);
    if (out_f32) out_f32[t * H + h] = o;
  }
}

moe_shape dense_shape(const moe_shape& s, int I_dense) {
  moe_shape d = s;
  d.E = 1;
  d.k = 1;
  d.I = I_dense;
  d.n_shared = 0;
  d.I_shared = 0;
  return d;
}

// [MoE layer workspace | a1 | a2 | y1 | y2 | zl | dense layer workspace]
struct BlockWs {
  size_t moe, a1, a2, y1, y2, zl, dense, total;
};

BlockWs block_ws(const moe_shape& s, int I_dense) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  const size_t th = (size_t)s.T * (size_t)s.H * 2;
  const moe_shape d = dense_shape(s, I_dense);
  BlockWs w{};
  size_t o = 0;
  w.moe = o;
  o += up(moe_workspace_size(&s));
  w.a1 = o;
  o += up(th);
  w.a2 = o;
  o += up(th);
  w.y1 = o;
  o += up(th);
  w.y2 = o;
  o += up(th);
  w.zl = o;
  o += up(sizeof(float) * (size_t)s.T + 4);
  w.dense = o;
  o += up(moe_workspace_size(&d));
  w.total = o;
  return w;
}

// The second stream and the fork / join events, one set per device, made on
// the first call and kept for the life of the process.  The mutex covers the
// enqueueing from the fork to the join, so that calls from several host
// threads do not interleave their event records.
struct SideStream {
  std::mutex mu;
  bool ready = false;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

constexpr int kMaxBlockDevices = 64;
SideStream g_side[kMaxBlockDevices];

SideStream* side_stream(int dev) {
  if (dev < 0 || dev >= kMaxBlockDevices) return nullptr;
  return &g_side[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_gemma4_workspace_size(const moe_shape* shape, int32_t I_dense) {
  if (validate_shape(shape) != MOE_OK || shape->n_shared != 0 || I_dense < 8 ||
      I_dense % 8 != 0)
    return 0;
  const moe_shape d = dense_shape(*shape, I_dense);
  if (validate_shape(&d) != MOE_OK) return 0;
  return block_ws(*shape, I_dense).total;
}

moe_status moe_gemma4_block(const moe_shape* shape, const moe_bf16* x,
                            const moe_gemma4_block_params* p, const moe_bf16* w13,
                            const moe_bf16* w2, const float* scale, moe_bf16* out,
                            float* out_f32, void* ws, size_t ws_bytes,
                            cudaStream_t stream) {
  moe_status st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!p) return MOE_ERR_INVALID_ARG;
  if (shape->n_shared != 0) return MOE_ERR_UNSUPPORTED;
  if (p->I_dense < 8 || p->I_dense % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!(p->eps >= 0.0f) || !(p->eps < 1e30f)) return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  const moe_shape d = dense_shape(s, p->I_dense);
  if ((st = validate_shape(&d)) != MOE_OK) return st;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < block_ws(s, p->I_dense).total) return MOE_ERR_WORKSPACE;
  if (s.T == 0) return MOE_OK;
  if (!x || !out || !w13 || !w2 || !p->mlp_w13 || !p->mlp_w2 || !p->router_w ||
      !p->router_scale)
    return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 5; ++i)
    if (!p->norm_w[i] || !aligned16(p->norm_w[i])) return MOE_ERR_INVALID_ARG;
  // what the two layer calls below would refuse, refused before anything is
  // launched: rows and weights read in 16-byte vectors or TMA tiles
  if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(p->mlp_w13) ||
      !aligned16(p->mlp_w2) || !aligned16(p->router_w) || !aligned16(p->router_scale))
    return MOE_ERR_INVALID_ARG;
  const BlockWs m = block_ws(s, p->I_dense);
  uint8_t* base = static_cast<uint8_t*>(ws);
  auto* a1 = reinterpret_cast<__nv_bfloat16*>(base + m.a1);
  auto* a2 = reinterpret_cast<__nv_bfloat16*>(base + m.a2);
  auto* y1 = reinterpret_cast<__nv_bfloat16*>(base + m.y1);
  auto* y2 = reinterpret_cast<__nv_bfloat16*>(base + m.y2);
  auto* zl = reinterpret_cast<float*>(base + m.zl);
  void* ws_moe = base + m.moe;
  void* ws_dense = base + m.dense;
  auto* block_err = reinterpret_cast<uint32_t*>(ws_moe);     // the block's error word
  auto* dense_err = reinterpret_cast<uint32_t*>(ws_dense);
  const size_t moe_bytes = m.a1 - m.moe, dense_bytes = m.total - m.dense;
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  auto nw = [&](int i) { return reinterpret_cast<const __nv_bfloat16*>(p->norm_w[i]); };

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  SideStream* side = side_stream(dev);
  if (!side) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(side->mu);
  if (!side->ready) {
    if (cudaStreamCreateWithFlags(&side->s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&side->fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&side->join, cudaEventDisableTiming) != cudaSuccess)
      return MOE_ERR_CUDA;
    side->ready = true;
  }

  if (launch_ex(pre_norm_kernel, dim3((unsigned)s.T), dim3(kNormThreads), 0, stream, false,
                xb, nw(0), nw(2), s.H, p->eps, a1, a2, zl, dense_err) != cudaSuccess)
    return MOE_ERR_CUDA;
  // fork: the dense MLP (one expert, every token with weight 1) on the
  // second stream, once the input norms are written
  if (cudaEventRecord(side->fork, stream) != cudaSuccess ||
      cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  auto mb = [](void* q) { return reinterpret_cast<moe_bf16*>(q); };
  moe_status sd = moe_forward_ex(&d, mb(a1), zl, p->mlp_w13, p->mlp_w2, nullptr, nullptr,
                                 nullptr, mb(y1), nullptr, nullptr, ws_dense, dense_bytes,
                                 nullptr, side->s);
  // the join is recorded whatever the dense branch returned, so that the
  // caller's stream (or its capture) is never left forked
  if (cudaEventRecord(side->join, side->s) != cudaSuccess) return MOE_ERR_CUDA;
  // the router reads the raw residual, the experts its pre_ff_norm_2
  moe_forward_opts o{};
  o.router_x = x;
  o.router_w = p->router_w;
  o.router_scale = p->router_scale;
  o.router_eps = p->router_eps;
  st = moe_forward_ex(&s, mb(a2), nullptr, w13, w2, scale, nullptr, nullptr, mb(y2),
                      nullptr, nullptr, ws_moe, moe_bytes, &o, stream);
  if (cudaStreamWaitEvent(stream, side->join, 0) != cudaSuccess) return MOE_ERR_CUDA;
  if (sd != MOE_OK) return sd;
  if (st != MOE_OK) return st;
  if (launch_ex(post_norm_kernel, dim3((unsigned)s.T), dim3(kNormThreads), 0, stream, false,
                (const __nv_bfloat16*)y1, (const __nv_bfloat16*)y2, xb, nw(1), nw(3), nw(4),
                s.H, p->eps, reinterpret_cast<__nv_bfloat16*>(out), out_f32, dense_err,
                block_err) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
