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
// stand-in, not a device address.  The device address is looked up once per
// device with cudaGetSymbolAddress (with that device current) and cached.
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

// Device address of g_permute_scratch on the current device (cached).
cudaError_t scratch_address(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  if (dev >= 0 && dev < kMaxDevices && g_scratch_ptr[dev]) {
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_permute_scratch);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices) g_scratch_ptr[dev] = static_cast<int32_t*>(p);
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
                                      cap, lt_count, lt_base, lt_rank, n_lt, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
