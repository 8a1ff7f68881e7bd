// route.cu -- warp-per-token routing kernel (moe_route, moe_route_ex and the
// prefill path of moe_forward).  The per-token arithmetic is route_token_warp
// (route_impl.cuh): optional expert-group selection, top-k on the fp32
// logits, closed-form renormalised softmax (or normalised sigmoids) over the
// chosen k in fp64, times per_expert_scale.
#include "route_impl.cuh"

namespace moe {
namespace {

template <int PER>
__global__ void __launch_bounds__(256)
route_kernel(const float* __restrict__ logits, const float* __restrict__ scale,
             int64_t T, int E, int k, int32_t* __restrict__ ids,
             float* __restrict__ w, RouteOpt opt) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();  // let the layout kernels start launching
  if (t >= T) return;
  int id;
  float wt;
  route_token_warp<PER>(logits + t * E, scale, E, k, &id, &wt, opt);
  if (lane < k) {
    ids[t * k + lane] = id;
    w[t * k + lane] = wt;
  }
}

}  // namespace

cudaError_t launch_route(const float* logits, const float* scale, int64_t T,
                         int E, int k, int32_t* ids, float* w,
                         cudaStream_t st, RouteOpt opt) {
  if (T == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (T + warps - 1) / warps;
  // logits per lane: the fewest that cover E (E <= 512)
  auto kern = E <= 32 ? route_kernel<1> : E <= 64 ? route_kernel<2> : E <= 128 ? route_kernel<4>
              : E <= 256 ? route_kernel<8> : route_kernel<16>;
  return launch_ex(kern, dim3((unsigned)blocks), dim3(warps * 32), 0, st, false, logits, scale,
                   T, E, k, ids, w, opt);
}

}  // namespace moe
