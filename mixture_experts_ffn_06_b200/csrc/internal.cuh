// internal.cuh -- shared declarations of the MoE library's translation units:
// the workspace map, launch wrappers, and the device-side wait helpers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kSegPad = 128;       // rows per expert-segment granule (GEMM M tile)
constexpr int kLayoutTile = 1024;  // slots per layout block
constexpr int kMaxExperts = 512;
constexpr int kMaxShared = 8;
constexpr int kMaxTopK = 32;

// Device error word values are moe_status codes.
constexpr uint32_t kErrTimeout = MOE_ERR_TIMEOUT;

// Byte offsets of everything that lives in the caller's workspace.
struct WsMap {
  size_t err;          // uint32 error word (+ padding)
  size_t ids, w;       // [T,k] int32 / fp32 (moe_forward)
  size_t offsets;      // [G+1] int32
  size_t sorted_slots; // [cap] int32
  size_t slot_row;     // [T,k+S] int32
  size_t lt_count;     // [n_lt, E] int32 per-layout-block histograms
  size_t lt_base;      // [n_lt, E] int32 per-layout-block exclusive bases
  size_t lt_rank;      // [T*k] int32 stable rank inside the layout block
  size_t x_perm;       // [cap,H] bf16 gathered activations
  size_t h;            // [cap,I] bf16 gated intermediate
  size_t stage;        // [T,k+S,H] fp32 weighted expert rows (moe_forward)
  size_t acc;          // [T,H] fp32 accumulator (moe_forward, fast combine)
  size_t dec_meta;     // decode path: touched-expert lists
  size_t dt_part;      // decode path, tensor-core form: [2*kDtMaxCtas,128,T] fp32
  size_t dt_cnt;       // decode path, tensor-core form: [2, G*row blocks] int32
  size_t logits;       // [T,E] fp32 router logits (moe_forward_ex with a router)
  size_t total;
  // moe_forward_fp8, after `total` (the permuted codes of x reuse x_perm):
  size_t x_q;          // [T,H] e4m3 codes of the token rows
  size_t s_x;          // [T] their scales
  size_t a_scale;      // [cap] row scales of the w13 product's A rows
  size_t h_q;          // [cap,I] e4m3 codes of h
  size_t s_h;          // [cap] their scales
  size_t total_fp8;
  int64_t cap;
  int64_t n_lt;
};

WsMap workspace_map(const moe_shape& s);

// Shape validation shared by every entry point (MOE_OK or the error status).
moe_status validate_shape(const moe_shape* s);

// cudaEventRecord of a caller's stage event; an event node under capture.
bool record_stage_event(void* ev, cudaStream_t st);

// Routing variant (moe_route_opts, checked): scoring, and with n_group > 1
// the expert groups (route_impl.cuh).
struct RouteOpt {
  int scoring;     // MOE_SCORE_SOFTMAX or MOE_SCORE_SIGMOID
  int n_group;     // <= 1: no groups; else <= MOE_MAX_GROUPS and E % n_group == 0
  int topk_group;  // groups kept per token (1..n_group)
};

// ---- launch wrappers (return cudaGetLastError of the launch) ----
cudaError_t launch_route(const float* logits, const float* scale, int64_t T,
                         int E, int k, int32_t* ids, float* w, cudaStream_t st,
                         RouteOpt opt = RouteOpt{0, 1, 1});

// Router logits [T,E] fp32 from the bf16 residual [T,H], the GateLinear
// weight [E,H] and the per-dimension scale [H] (router.cu).
cudaError_t launch_router_logits(const __nv_bfloat16* x, const __nv_bfloat16* w_router,
                                 const __nv_bfloat16* scale, int64_t T, int H, int E,
                                 float eps, float* logits, cudaStream_t st,
                                 bool pdl = false);

// pdl on any launch function: launch its first kernel as a programmatic
// dependent of the previous kernel on the stream (later kernels of the same
// function always are).
// err (may be null): error word that records MOE_ERR_INVALID_ARG when an id
// lies outside [0,E) (such slots get no row and slot_row -1).
cudaError_t launch_layout(const moe_shape& s, const int32_t* ids,
                          int32_t* offsets, int32_t* sorted_slots,
                          int32_t* slot_row, int64_t cap, int32_t* lt_count,
                          int32_t* lt_base, int32_t* lt_rank, int64_t n_lt,
                          uint32_t* err, cudaStream_t st, bool pdl = false);

// Gathers x rows into x_perm for the rows of groups [0, G) (padding rows are
// left as they are); when acc is given it also zeroes acc[0, n_acc)
// (n_acc % 4 == 0).
cudaError_t launch_gather(const __nv_bfloat16* x, const int32_t* sorted_slots,
                          const int32_t* offsets, int G, int64_t T, int k,
                          int H, int64_t cap, __nv_bfloat16* x_perm, float* acc,
                          int64_t n_acc, cudaStream_t st, bool pdl = false);

// FP8 (fp8.cu).  Per-row dynamic e4m3 quantisation of bf16 rows [rows, cols]
// (cols % 8 == 0): codes [rows, cols] bytes, scales [rows].  rows_used
// (device, or null): only rows below *rows_used; slots (or null): rows whose
// slot is negative are skipped.
cudaError_t launch_quantize_rows(const __nv_bfloat16* src, int64_t rows, int cols,
                                 uint8_t* codes, float* scales, const int32_t* rows_used,
                                 const int32_t* slots, cudaStream_t st, bool pdl = false);
// Codes of x's token rows into the routed experts' permuted rows (H % 16 ==
// 0), the row scale of every row in use (shared experts' too), and zeroes
// acc[0, n_acc) when given.
cudaError_t launch_gather_fp8(const uint8_t* xq, const float* sx, const int32_t* sorted_slots,
                              const int32_t* offsets, int E, int G, int64_t T, int k, int H,
                              int64_t cap, uint8_t* x_perm, float* a_scale, float* acc,
                              int64_t n_acc, cudaStream_t st, bool pdl = false);

// out = bf16(acc) (round to nearest even), out_f32 = acc if given; n % 8 == 0.
cudaError_t launch_finalize(const float* acc, int64_t n, __nv_bfloat16* out,
                            float* out_f32, cudaStream_t st, bool pdl = false);

cudaError_t launch_combine(const float* y_perm, const int32_t* slot_row,
                           const float* w, int64_t T, int k, int S, int H,
                           __nv_bfloat16* out, cudaStream_t st);

// out[t] = bf16(sum_{j < ks} stage[t*ks + j]) summed in order j = 0..ks-1;
// out_f32 (optional) receives the fp32 sum.
// pdl: launch as a programmatic dependent of the previous kernel.
cudaError_t launch_sum_rows(const float* stage, int64_t T, int ks, int H,
                            __nv_bfloat16* out, float* out_f32, cudaStream_t st,
                            bool pdl = false);

// The small-T path (decode.cu).
constexpr int kDecodeMaxT = MOE_DECODE_MAX_T;
constexpr int kDecodeForcedMaxT = 1024;
struct DecodeArgs {
  const __nv_bfloat16* x;
  const float* logits;
  const float* scale;
  const __nv_bfloat16 *w13, *w2, *w13_sh, *w2_sh;
  int T, H, E, k, I, S, act;
  RouteOpt route;
  int32_t* ids;          // [T,k] out
  float* w;              // [T,k] out
  int32_t* meta;         // [decode_meta_ints(E+S)] scratch
  int32_t* slots;        // [T*(k+S)] scratch
  __nv_bfloat16* h_dec;  // [T*(k+S), I] scratch
  float* stage;          // [T*(k+S), H] scratch
  __nv_bfloat16* out;    // [T,H]
  float* out_f32;        // [T,H] or nullptr
  // the tensor-core form (decode_tc.cu), T <= kDecodeTcMaxT
  bool tc;
  float* dt_part;        // [2 * kDtMaxCtas, 128, T] fp32 partial sums
  int32_t* dt_cnt;       // [2, G * dt_row_blocks] arrival counters
  uint32_t* err;         // error word
  // FP8 experts (the tensor-core form only): e4m3 codes with one fp32 scale
  // per output row, x and h quantised per row on the way
  bool f8;
  const uint8_t *w13q, *w2q, *w13q_sh, *w2q_sh;
  const float *w13s, *w2s, *w13s_sh, *w2s_sh;
  uint8_t* xq;           // [T,H] codes of x, scales sx [T]
  float* sx;
  uint8_t* hq;           // [touched * N, I] codes of h, scales sh [touched * N]
  float* sh;
};
size_t decode_meta_ints(int G);

// Tensor-core decode products (decode_tc.cu).
constexpr int kDecodeTcMaxT = 64;
constexpr int kDecodeFewMaxT = 8;   // the skinny kernels' one-B-tile form
constexpr int kDtMaxCtas = 2 * 160;  // persistent CTAs: up to 2 per SM
// row blocks of one group: max(ceil(I / 64), ceil(H / 128))
int dt_row_blocks(int H, int I);
// token columns N of the tensor-core form for T tokens: 16, 32 or 64
int dt_columns(int T);
// kernels of the tensor-core form: w13 (+ act) -> h, w2 (x gate weight) -> stage.
// meta / slots come from decode_route; h_dense [touched groups * N, I] bf16.
cudaError_t launch_decode_tc_w13(const DecodeArgs& a, __nv_bfloat16* h_dense,
                                 cudaStream_t st);
cudaError_t launch_decode_tc_w2(const DecodeArgs& a, const __nv_bfloat16* h_dense,
                                cudaStream_t st);
// ev: nullptr or MOE_NUM_STAGES + 1 events (see moe_forward_ex)
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st, void* const* ev);

// Grouped GEMMs on tcgen05.
//   mode 0: h = Act(A W1^T) (*) (A W3^T), B = packed [G][2N][K] gate/up rows,
//           bf16 out [cap, N];
//   mode 1: y = A W^T, B = [G][N][K], fp32 out [cap, N] (unweighted rows);
//   mode 2: as mode 1, but row r adds w_r * y_r into row t of the fp32
//           accumulator out [T, N] (vector reductions: fast, the order of
//           the additions is not fixed);
//   mode 3: as mode 1, but row r stores w_r * y_r at row t*(k+S) + j of
//           out [T*(k+S), N], the (token, choice) order (un-permute), for a
//           fixed-order sum afterwards.
struct GroupedGemmArgs {
  int mode;
  const __nv_bfloat16* A;       // [cap, K]
  const __nv_bfloat16* A_sh;    // [T, K] A rows of the shared groups (segment row
                                // i is token i), or nullptr: those rows are in A
  const __nv_bfloat16* B;       // routed experts' weights
  const __nv_bfloat16* B_sh;    // shared experts' weights (or nullptr)
  const int32_t* offsets;       // [G+1]
  int G, E;                     // groups, routed groups
  int N, K;                     // output columns, reduction length
  int64_t cap;                  // rows of A / out
  void* out;                    // 0: bf16 [cap,N]; 1: fp32 [cap,N]; 2: fp32 [T,N]; 3: fp32 [T*(k+S),N]
  int act;
  uint32_t* err;
  const int32_t* sorted_slots;  // [cap] row -> slot, -1 on padding rows
  // modes 2, 3
  const float* w;               // [T,k]
  int64_t T;
  int k;
  bool pair;                    // run on CTA pairs (2-SM MMA, M = 256)
  // FP8 operands: A and B hold e4m3 bytes (K % 16 == 0); the product of A
  // row r and B row n is scaled by a_scale[r] * b_scale[group row n]
  // (b_scale_sh for the shared groups) before the epilogue uses it
  bool f8;
  const float* a_scale;         // [cap]
  const float* b_scale;         // [E, rows per group]
  const float* b_scale_sh;      // [S, rows per group] or nullptr
};
cudaError_t launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t st,
                                bool pdl = false);

cudaError_t launch_wait_selftest(uint32_t* err, uint32_t timeout_us,
                                 cudaStream_t st);

// TMA map of a row-major bf16 [outer, inner] tensor: box {64, box_rows},
// 128-byte swizzle, out-of-range elements read as zero (gemm_tc.cu).
cudaError_t make_tma_map_bf16(CUtensorMap* m, const void* ptr, uint64_t inner,
                              uint64_t outer, uint32_t box_rows);
// The same for a row-major tensor of e4m3 bytes: box {128, box_rows}.
cudaError_t make_tma_map_e4m3(CUtensorMap* m, const void* ptr, uint64_t inner,
                              uint64_t outer, uint32_t box_rows);
// SMs of the current device (cached per device).
int device_sm_count();

// ---------------------------------------------------------------- device
#ifdef __CUDACC__

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void record_error(uint32_t* err, uint32_t code) {
  if (err) atomicCAS(err, 0u, code);
}

// Programmatic dependent launch.  A kernel launched with the PDL attribute
// may start while its predecessor on the stream is still running; it must
// call pdl_wait() before touching anything the predecessor writes (the wait
// returns at once when there is no such predecessor).  pdl_trigger() lets the
// next kernel start launching.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// cudaLaunchKernelEx with the programmatic-serialisation attribute when pdl.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

#endif  // __CUDACC__

}  // namespace moe
