// noalloc.cu -- moe_permute_noalloc: the dispatch permutation with its
// scratch in a fixed device array instead of a caller workspace.
//
// Some callers cannot allocate device memory when they launch the layer:
// code inside a CUDA graph capture, runtimes whose pool is reserved up front,
// plug-in hosts that only pass in/out buffers.  For them the counting sort's
// scratch (per-block histograms, per-block bases, per-slot ranks) lives in
// g_permute_scratch below, a 1 MiB array that every GPU loading this library
// holds until the process exits.  The kernels are the ones moe_permute uses;
// only the scratch pointers differ.
//
// Host code must not hand the symbol itself to a kernel: on the host it is a
// stand-in, not a device address.  The device address is looked up with
// cudaGetSymbolAddress (with that device current) and cached per device,
// together with the id of the context it belongs to; when the context has
// changed (after a device reset) it is looked up again.
#include <mutex>

#include "internal.cuh"

namespace moe {
namespace {

constexpr int64_t kNoAllocMaxSlots = MOE_NOALLOC_MAX_SLOTS;
constexpr int64_t kNoAllocBlocks = kNoAllocMaxSlots / kLayoutTile;  // 128
constexpr int64_t kCountInts = kNoAllocBlocks * kMaxExperts;        // [blocks, E]
constexpr int64_t kScratchInts = 2 * kCountInts + kNoAllocMaxSlots;  // 1 MiB
static_assert(kNoAllocMaxSlots % kLayoutTile == 0, "whole layout blocks");

static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context id of each entry

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current context (0 when there is none or the driver
// cannot say).  A device reset gives the device a new primary context with a
// new id, so an address cached under the old id is never reused.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_permute_scratch on the current device, cached per
// device and context.
cudaError_t scratch_address(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long ctx = current_context_id();
  if (slot && g_scratch_ptr[dev] && ctx != 0 && g_scratch_ctx[dev] == ctx) {
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_permute_scratch);
  if (e != cudaSuccess) return e;
  if (slot) {
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    g_scratch_ctx[dev] = current_context_id();  // the lookup made it current
  }
  *out = static_cast<int32_t*>(p);
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_permute_noalloc(const moe_shape* shape,
                                          const int32_t* ids, int32_t* offsets,
                                          int32_t* sorted_slots,
                                          int32_t* slot_row,
                                          cudaStream_t stream) {
  const moe_status st = validate_shape(shape);
  if (st != MOE_OK) return st;
  const int64_t R = shape->T * shape->k;
  if (R > kNoAllocMaxSlots) return MOE_ERR_UNSUPPORTED;
  if (!offsets || !sorted_slots || (shape->T > 0 && (!ids || !slot_row)))
    return MOE_ERR_INVALID_ARG;
  int32_t* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t* lt_count = base;
  int32_t* lt_base = base + kCountInts;
  int32_t* lt_rank = base + 2 * kCountInts;
  int64_t n_lt = (R + kLayoutTile - 1) / kLayoutTile;
  if (n_lt < 1) n_lt = 1;
  const int64_t cap = workspace_map(*shape).cap;
  const cudaError_t e = launch_layout(*shape, ids, offsets, sorted_slots, slot_row,
                                      cap, lt_count, lt_base, lt_rank, n_lt,
                                      /*err=*/nullptr, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
