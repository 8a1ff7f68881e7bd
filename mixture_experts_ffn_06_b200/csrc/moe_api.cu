// moe_api.cu -- the C entry points declared in include/moe.h: argument
// checks, the workspace map, and the launch sequence of each call.  Every
// argument error is returned before anything is enqueued; nothing here
// allocates, frees or synchronises (moe_read_error excepted, as documented).
#include <cmath>

#include "internal.cuh"

namespace moe {

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static int seg_pad(const moe_shape& s) { return s.pad ? s.pad : kSegPad; }

WsMap workspace_map(const moe_shape& s) {
  WsMap m{};
  const int64_t T = s.T, k = s.k, S = s.n_shared, G = s.E + s.n_shared;
  const int P = seg_pad(s);
  m.cap = T * k + T * S + G * (P - 1);
  m.n_lt = (T * k + kLayoutTile - 1) / kLayoutTile;
  if (m.n_lt < 1) m.n_lt = 1;
  const int64_t Imax = s.I > s.I_shared ? s.I : s.I_shared;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  m.err = take(256);
  m.ids = take(sizeof(int32_t) * T * k);
  m.w = take(sizeof(float) * T * k);
  m.offsets = take(sizeof(int32_t) * (G + 1));
  m.sorted_slots = take(sizeof(int32_t) * m.cap);
  m.slot_row = take(sizeof(int32_t) * T * (k + S));
  m.lt_count = take(sizeof(int32_t) * m.n_lt * s.E);
  m.lt_base = take(sizeof(int32_t) * m.n_lt * s.E);
  m.lt_rank = take(sizeof(int32_t) * T * k);
  m.x_perm = take(2ull * m.cap * s.H);
  m.h = take(2ull * m.cap * Imax);
  m.stage = take(4ull * T * (k + S) * s.H);
  m.acc = take(4ull * T * s.H);
  m.dec_meta = take(sizeof(int32_t) * decode_meta_ints((int)G));
  // the tensor-core decode form: partial sums of split units and counters
  const bool dt = T >= 1 && T <= kDecodeTcMaxT;
  m.dt_part = take(dt ? sizeof(float) * 2 * kDtMaxCtas * 128 * T : 0);
  m.dt_cnt = take(dt ? sizeof(int32_t) * 2 * G * dt_row_blocks(s.H, s.I) : 0);
  m.logits = take(sizeof(float) * T * s.E);
  m.total = o;
  m.x_q = take((size_t)T * s.H);
  m.s_x = take(sizeof(float) * T);
  m.a_scale = take(sizeof(float) * m.cap);
  m.h_q = take((size_t)m.cap * Imax);
  m.s_h = take(sizeof(float) * m.cap);
  m.total_fp8 = o;
  return m;
}

static moe_status check_shape(const moe_shape* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->E <= 0 || s->k <= 0 || s->I <= 0 ||
      s->n_shared < 0 || s->pad < 0)
    return MOE_ERR_INVALID_ARG;
  if (s->k > s->E) return MOE_ERR_INVALID_ARG;
  if (s->act != MOE_ACT_SILU && s->act != MOE_ACT_GELU_TANH)
    return MOE_ERR_INVALID_ARG;
  if (s->E > kMaxExperts || s->k > kMaxTopK || s->n_shared > kMaxShared)
    return MOE_ERR_UNSUPPORTED;
  if (s->H % 8 != 0 || s->I % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (s->n_shared > 0 && s->I_shared != s->I) return MOE_ERR_UNSUPPORTED;
  if (s->pad != 0 && s->pad != kSegPad) return MOE_ERR_UNSUPPORTED;
  if (s->T >= (int64_t(1) << 24)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status validate_shape(const moe_shape* s) { return check_shape(s); }

bool record_stage_event(void* ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return false;
  const unsigned flags =
      cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : 0u;
  return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev), st, flags) ==
         cudaSuccess;
}

static moe_status from_cuda(cudaError_t e) {
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

static moe_status check_ws(const moe_shape& s, const void* ws, size_t ws_bytes) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < workspace_map(s).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <class P>
static uint8_t* at(P* base, size_t off) {
  return reinterpret_cast<uint8_t*>(const_cast<void*>(static_cast<const void*>(base))) + off;
}

// Record stage event i (if the caller asked for stage events).  Under stream
// capture the record becomes an event node of the graph, so the caller can
// time the stages of each replay.
static bool mark(void* const* ev, int i, cudaStream_t st) {
  if (!ev || !ev[i]) return true;
  return record_stage_event(ev[i], st);
}

// gather -> w13 GEMM (+activation) -> w2 GEMM.  The w2 GEMM writes
//   combine 0: unweighted fp32 rows to y_perm in permuted order (moe_expert_ffn);
//   combine 2: adds w * y into the fp32 accumulator y_perm = acc [T, H];
//   combine 3: stores w * y at the row's (token, choice) position of
//              y_perm = stage [T, k+S, H].
static moe_status run_expert_ffn(const moe_shape& s, const __nv_bfloat16* x,
                                 const int32_t* offsets,
                                 const int32_t* sorted_slots,
                                 const __nv_bfloat16* w13, const __nv_bfloat16* w2,
                                 const __nv_bfloat16* w13_sh,
                                 const __nv_bfloat16* w2_sh, float* y_perm,
                                 int combine, const float* w, void* ws,
                                 cudaStream_t st, void* const* ev = nullptr,
                                 bool pdl = false, int cta_pairs = 0) {
  const WsMap m = workspace_map(s);
  const int G = s.E + s.n_shared;
  auto* x_perm = reinterpret_cast<__nv_bfloat16*>(at(ws, m.x_perm));
  auto* h = reinterpret_cast<__nv_bfloat16*>(at(ws, m.h));
  auto* err = reinterpret_cast<uint32_t*>(at(ws, m.err));
  if (!mark(ev, 2, st)) return MOE_ERR_CUDA;
  // the shared experts' segments hold tokens 0..T-1 in order: the w13 GEMM
  // reads their A rows from x itself, so only the routed rows are gathered
  cudaError_t e = launch_gather(x, sorted_slots, offsets, s.E, s.T, s.k, s.H, m.cap,
                                x_perm, combine == 2 ? y_perm : nullptr,
                                s.T * (int64_t)s.H, st, pdl);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(ev, 3, st)) return MOE_ERR_CUDA;
  GroupedGemmArgs a{};
  a.mode = 0;
  a.A = x_perm;
  a.A_sh = x;
  a.B = w13;
  a.B_sh = w13_sh;
  a.offsets = offsets;
  a.G = G;
  a.E = s.E;
  a.N = s.I;
  a.K = s.H;
  a.cap = m.cap;
  a.out = h;
  a.act = s.act;
  a.err = err;
  a.sorted_slots = sorted_slots;  // both GEMMs look up which rows are real
  a.w = w;
  a.T = s.T;
  a.k = s.k;
  // CTA pairs (2-SM MMA) when asked; by default only for the w2 GEMM with
  // a long reduction (I >= 1024) once an expert averages two or more full
  // 128-row m-tiles -- measured on B200, pairs help w2 there and cost the
  // w13 GEMM and short reductions a few percent
  const bool big = s.T * (int64_t)s.k >= 2 * 128 * (int64_t)s.E;
  a.pair = cta_pairs == 2;
  e = launch_grouped_gemm(a, st, true);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(ev, 4, st)) return MOE_ERR_CUDA;
  a.mode = combine == 0 ? 1 : combine;
  a.pair = cta_pairs == 2 || (cta_pairs == 0 && big && s.I >= 1024);
  a.A = h;
  a.A_sh = nullptr;  // h holds the shared groups' rows too
  a.B = w2;
  a.B_sh = w2_sh;
  a.N = s.H;
  a.K = s.I;
  a.out = y_perm;
  return from_cuda(launch_grouped_gemm(a, st));
}

}  // namespace moe

using namespace moe;

extern "C" {

int64_t moe_layout_capacity(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return workspace_map(*shape).cap;
}

size_t moe_workspace_size(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return workspace_map(*shape).total;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool weights_aligned(const moe_shape& s, const void* w13, const void* w2,
                            const void* w13_sh, const void* w2_sh) {
  return aligned16(w13) && aligned16(w2) &&
         (s.n_shared == 0 || (aligned16(w13_sh) && aligned16(w2_sh)));
}

moe_status moe_router_logits(const moe_shape* shape, const moe_bf16* x,
                             const moe_bf16* w_router, const moe_bf16* scale, float eps,
                             float* logits, cudaStream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return MOE_ERR_INVALID_ARG;
  if (shape->T == 0) return MOE_OK;
  if (!x || !w_router || !scale || !logits) return MOE_ERR_INVALID_ARG;
  // the kernel reads 16-byte vectors
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(scale)) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_router_logits(reinterpret_cast<const __nv_bfloat16*>(x),
                                        reinterpret_cast<const __nv_bfloat16*>(w_router),
                                        reinterpret_cast<const __nv_bfloat16*>(scale),
                                        shape->T, shape->H, shape->E, eps, logits, stream));
}

// Checks a routing variant against the shape; NULL is the plain routing.
static moe_status check_route_opts(const moe_shape& s, const moe_route_opts* o,
                                   RouteOpt* out) {
  *out = RouteOpt{MOE_SCORE_SOFTMAX, 1, 1};
  if (!o) return MOE_OK;
  if (o->scoring != MOE_SCORE_SOFTMAX && o->scoring != MOE_SCORE_SIGMOID)
    return MOE_ERR_INVALID_ARG;
  out->scoring = o->scoring;
  if (o->n_group <= 1) {
    if (o->n_group < 0) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
  }
  if (o->n_group > MOE_MAX_GROUPS) return MOE_ERR_UNSUPPORTED;
  if (s.E % o->n_group != 0 || o->topk_group < 1 || o->topk_group > o->n_group ||
      s.k > o->topk_group * (s.E / o->n_group))
    return MOE_ERR_INVALID_ARG;
  out->n_group = o->n_group;
  out->topk_group = o->topk_group;
  return MOE_OK;
}

moe_status moe_route(const moe_shape* shape, const float* logits,
                     const float* scale, int32_t* ids, float* w,
                     cudaStream_t stream) {
  return moe_route_ex(shape, logits, scale, nullptr, ids, w, stream);
}

moe_status moe_route_ex(const moe_shape* shape, const float* logits,
                        const float* scale, const moe_route_opts* opts, int32_t* ids,
                        float* w, cudaStream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  RouteOpt ro;
  if ((st = check_route_opts(*shape, opts, &ro)) != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  if (!logits || !ids || !w) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_route(logits, scale, shape->T, shape->E, shape->k, ids,
                                w, stream, ro));
}

moe_status moe_permute(const moe_shape* shape, const int32_t* ids,
                       int32_t* offsets, int32_t* sorted_slots,
                       int32_t* slot_row, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!offsets || !sorted_slots || (shape->T > 0 && (!ids || !slot_row)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const WsMap m = workspace_map(*shape);
  return from_cuda(launch_layout(
      *shape, ids, offsets, sorted_slots, slot_row, m.cap,
      reinterpret_cast<int32_t*>(at(ws, m.lt_count)),
      reinterpret_cast<int32_t*>(at(ws, m.lt_base)),
      reinterpret_cast<int32_t*>(at(ws, m.lt_rank)), m.n_lt,
      reinterpret_cast<uint32_t*>(at(ws, m.err)), stream));
}

moe_status moe_expert_ffn(const moe_shape* shape, const moe_bf16* x,
                          const int32_t* offsets, const int32_t* sorted_slots,
                          const moe_bf16* w13, const moe_bf16* w2,
                          const moe_bf16* w13_sh, const moe_bf16* w2_sh,
                          float* y_perm, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!offsets || !sorted_slots || !w13 || !w2 || !y_perm ||
      (shape->T > 0 && !x))
    return MOE_ERR_INVALID_ARG;
  if (shape->n_shared > 0 && (!w13_sh || !w2_sh)) return MOE_ERR_INVALID_ARG;
  // y_perm rows are written by 16-byte bulk copies; the weights are TMA
  // tiles and x is read in 16-byte vectors
  if (!aligned16(y_perm) || !weights_aligned(*shape, w13, w2, w13_sh, w2_sh) ||
      (shape->T > 0 && !aligned16(x)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  return run_expert_ffn(*shape, reinterpret_cast<const __nv_bfloat16*>(x), offsets,
                        sorted_slots, reinterpret_cast<const __nv_bfloat16*>(w13),
                        reinterpret_cast<const __nv_bfloat16*>(w2),
                        reinterpret_cast<const __nv_bfloat16*>(w13_sh),
                        reinterpret_cast<const __nv_bfloat16*>(w2_sh), y_perm,
                        0, nullptr, ws, stream);
}

moe_status moe_combine(const moe_shape* shape, const float* y_perm,
                       const int32_t* slot_row, const float* w, moe_bf16* out,
                       cudaStream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  if (!y_perm || !slot_row || !w || !out) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_combine(y_perm, slot_row, w, shape->T, shape->k,
                                  shape->n_shared, shape->H,
                                  reinterpret_cast<__nv_bfloat16*>(out), stream));
}

moe_status moe_forward_ex(const moe_shape* shape, const moe_bf16* x,
                          const float* logits, const moe_bf16* w13,
                          const moe_bf16* w2, const float* scale,
                          const moe_bf16* w13_sh, const moe_bf16* w2_sh,
                          moe_bf16* out, int32_t* ids_out, float* w_out, void* ws,
                          size_t ws_bytes, const moe_forward_opts* opts,
                          cudaStream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  const bool use_router = opts && opts->router_w;
  if (!w13 || !w2 || (shape->T > 0 && (!x || (!logits && !use_router) || !out)))
    return MOE_ERR_INVALID_ARG;
  if (use_router) {
    if (!(opts->router_eps >= 0.0f) || !std::isfinite(opts->router_eps))
      return MOE_ERR_INVALID_ARG;
    if (shape->T > 0 && (!opts->router_x || !opts->router_scale ||
                         !aligned16(opts->router_x) || !aligned16(opts->router_w) ||
                         !aligned16(opts->router_scale)))
      return MOE_ERR_INVALID_ARG;
  }
  if (shape->n_shared > 0 && (!w13_sh || !w2_sh)) return MOE_ERR_INVALID_ARG;
  // the weights are TMA tiles or 16-byte copies, x is read in 16-byte vectors
  if (!weights_aligned(*shape, w13, w2, w13_sh, w2_sh) || (shape->T > 0 && !aligned16(x)))
    return MOE_ERR_INVALID_ARG;
  RouteOpt ro;
  if ((st = check_route_opts(*shape, opts ? opts->route : nullptr, &ro)) != MOE_OK)
    return st;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  void* const* ev = opts ? opts->stage_events : nullptr;
  if (shape->T == 0) {
    for (int i = 0; i <= MOE_NUM_STAGES; ++i)
      if (!mark(ev, i, stream)) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  const moe_shape& s = *shape;
  const WsMap m = workspace_map(s);
  int32_t* ids = ids_out ? ids_out : reinterpret_cast<int32_t*>(at(ws, m.ids));
  float* w = w_out ? w_out : reinterpret_cast<float*>(at(ws, m.w));
  auto* offsets = reinterpret_cast<int32_t*>(at(ws, m.offsets));
  auto* sorted_slots = reinterpret_cast<int32_t*>(at(ws, m.sorted_slots));
  auto* slot_row = reinterpret_cast<int32_t*>(at(ws, m.slot_row));
  auto* stage = reinterpret_cast<float*>(at(ws, m.stage));
  const int path = opts ? opts->path : MOE_PATH_AUTO;
  if (opts && (opts->cta_pairs < 0 || opts->cta_pairs > 2)) return MOE_ERR_INVALID_ARG;
  if (path != MOE_PATH_AUTO && path != MOE_PATH_PREFILL && path != MOE_PATH_DECODE)
    return MOE_ERR_INVALID_ARG;
  if (path == MOE_PATH_DECODE && s.T > kDecodeForcedMaxT) return MOE_ERR_UNSUPPORTED;
  // the router ahead of the routing (moe_router_logits), when given: its
  // logits go to the workspace and the routing reads them there
  if (use_router) logits = reinterpret_cast<float*>(at(ws, m.logits));
  auto run_router = [&]() {
    return !use_router ||
           launch_router_logits(reinterpret_cast<const __nv_bfloat16*>(opts->router_x),
                                reinterpret_cast<const __nv_bfloat16*>(opts->router_w),
                                reinterpret_cast<const __nv_bfloat16*>(opts->router_scale),
                                s.T, s.H, s.E, opts->router_eps,
                                const_cast<float*>(logits), stream) == cudaSuccess;
  };
  if (path == MOE_PATH_DECODE || (path == MOE_PATH_AUTO && s.T <= kDecodeMaxT)) {
    // few tokens: stream only the touched experts (decode.cu)
    DecodeArgs d{};
    d.x = reinterpret_cast<const __nv_bfloat16*>(x);
    d.logits = logits;
    d.scale = scale;
    d.w13 = reinterpret_cast<const __nv_bfloat16*>(w13);
    d.w2 = reinterpret_cast<const __nv_bfloat16*>(w2);
    d.w13_sh = reinterpret_cast<const __nv_bfloat16*>(w13_sh);
    d.w2_sh = reinterpret_cast<const __nv_bfloat16*>(w2_sh);
    d.T = (int)s.T;
    d.H = s.H;
    d.E = s.E;
    d.k = s.k;
    d.I = s.I;
    d.S = s.n_shared;
    d.act = s.act;
    d.route = ro;
    d.ids = ids;
    d.w = w;
    d.meta = reinterpret_cast<int32_t*>(at(ws, m.dec_meta));
    d.slots = sorted_slots;
    d.h_dec = reinterpret_cast<__nv_bfloat16*>(at(ws, m.h));
    d.stage = stage;
    d.out = reinterpret_cast<__nv_bfloat16*>(out);
    d.out_f32 = opts ? opts->out_f32 : nullptr;
    // tensor-core products above the few-token form's 8 tokens (measured on
    // B200: the skinny kernels are faster up to 8 tokens, the tcgen05 form
    // from 16 on)
    d.tc = s.T > kDecodeFewMaxT && s.T <= kDecodeTcMaxT;
    d.dt_part = reinterpret_cast<float*>(at(ws, m.dt_part));
    d.dt_cnt = reinterpret_cast<int32_t*>(at(ws, m.dt_cnt));
    d.err = reinterpret_cast<uint32_t*>(at(ws, m.err));
    if (!use_router) return from_cuda(launch_decode(d, stream, ev));
    // the router counts in the first stage: event 0 goes ahead of it
    void* dev[MOE_NUM_STAGES + 1] = {};
    for (int i = 1; ev && i <= MOE_NUM_STAGES; ++i) dev[i] = ev[i];
    if (!mark(ev, 0, stream)) return MOE_ERR_CUDA;
    if (!run_router()) return MOE_ERR_CUDA;
    return from_cuda(launch_decode(d, stream, ev ? dev : nullptr));
  }
  if (!mark(ev, 0, stream)) return MOE_ERR_CUDA;
  if (!run_router()) return MOE_ERR_CUDA;
  if (launch_route(logits, scale, s.T, s.E, s.k, ids, w, stream, ro) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (!mark(ev, 1, stream)) return MOE_ERR_CUDA;
  if (launch_layout(s, ids, offsets, sorted_slots, slot_row, m.cap,
                    reinterpret_cast<int32_t*>(at(ws, m.lt_count)),
                    reinterpret_cast<int32_t*>(at(ws, m.lt_base)),
                    reinterpret_cast<int32_t*>(at(ws, m.lt_rank)), m.n_lt,
                    reinterpret_cast<uint32_t*>(at(ws, m.err)), stream,
                    /*pdl=*/true) != cudaSuccess)
    return MOE_ERR_CUDA;
  const bool det = opts && opts->deterministic;
  float* acc = reinterpret_cast<float*>(at(ws, m.acc));
  st = run_expert_ffn(s, reinterpret_cast<const __nv_bfloat16*>(x), offsets,
                      sorted_slots, reinterpret_cast<const __nv_bfloat16*>(w13),
                      reinterpret_cast<const __nv_bfloat16*>(w2),
                      reinterpret_cast<const __nv_bfloat16*>(w13_sh),
                      reinterpret_cast<const __nv_bfloat16*>(w2_sh),
                      det ? stage : acc, det ? 3 : 2, w, ws, stream, ev, true,
                      opts ? opts->cta_pairs : 0);
  if (st != MOE_OK) return st;
  if (!mark(ev, 5, stream)) return MOE_ERR_CUDA;
  float* out_f32 = opts ? opts->out_f32 : nullptr;
  const cudaError_t e =
      det ? launch_sum_rows(stage, s.T, s.k + s.n_shared, s.H,
                            reinterpret_cast<__nv_bfloat16*>(out), out_f32, stream,
                            true)
          : launch_finalize(acc, s.T * (int64_t)s.H,
                            reinterpret_cast<__nv_bfloat16*>(out), out_f32, stream,
                            true);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return mark(ev, 6, stream) ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_forward(const moe_shape* shape, const moe_bf16* x,
                       const float* logits, const moe_bf16* w13,
                       const moe_bf16* w2, const float* scale,
                       const moe_bf16* w13_sh, const moe_bf16* w2_sh,
                       moe_bf16* out, int32_t* ids_out, float* w_out, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  return moe_forward_ex(shape, x, logits, w13, w2, scale, w13_sh, w2_sh, out,
                        ids_out, w_out, ws, ws_bytes, nullptr, stream);
}

size_t moe_workspace_size_fp8(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return workspace_map(*shape).total_fp8;
}

moe_status moe_quantize_rows_e4m3(const moe_bf16* src, int64_t rows, int cols,
                                  uint8_t* codes, float* scales, cudaStream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!src || !codes || !scales || !aligned16(src) ||
      (reinterpret_cast<uintptr_t>(codes) & 7u) != 0)
    return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_quantize_rows(reinterpret_cast<const __nv_bfloat16*>(src), rows,
                                        cols, codes, scales, nullptr, nullptr, stream));
}

moe_status moe_forward_fp8(const moe_shape* shape, const moe_bf16* x, const float* logits,
                           const moe_fp8_experts* wq, const float* scale, moe_bf16* out,
                           int32_t* ids_out, float* w_out, void* ws, size_t ws_bytes,
                           const moe_forward_opts* opts, cudaStream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  const moe_shape& s = *shape;
  // e4m3 rows are TMA tiles: their byte strides must be multiples of 16
  if (s.H % 16 != 0 || s.I % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (!wq || !wq->w13 || !wq->w13_scale || !wq->w2 || !wq->w2_scale) return MOE_ERR_INVALID_ARG;
  if (s.n_shared > 0 && (!wq->w13_sh || !wq->w13_sh_scale || !wq->w2_sh ||
                         !wq->w2_sh_scale))
    return MOE_ERR_INVALID_ARG;
  // the codes are TMA tiles and x is read in 16-byte vectors: both need
  // 16-byte aligned bases
  if (!weights_aligned(s, wq->w13, wq->w2, wq->w13_sh, wq->w2_sh)) return MOE_ERR_INVALID_ARG;
  const bool use_router = opts && opts->router_w;
  if (s.T > 0 && (!x || (!logits && !use_router) || !out)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (use_router) {
    if (!(opts->router_eps >= 0.0f) || !std::isfinite(opts->router_eps))
      return MOE_ERR_INVALID_ARG;
    if (s.T > 0 && (!opts->router_x || !opts->router_scale || !aligned16(opts->router_x) ||
                    !aligned16(opts->router_w) || !aligned16(opts->router_scale)))
      return MOE_ERR_INVALID_ARG;
  }
  if (opts && (opts->cta_pairs < 0 || opts->cta_pairs > 2)) return MOE_ERR_INVALID_ARG;
  const int path = opts ? opts->path : MOE_PATH_AUTO;
  if (path != MOE_PATH_AUTO && path != MOE_PATH_PREFILL && path != MOE_PATH_DECODE)
    return MOE_ERR_INVALID_ARG;
  // the decode path takes FP8 experts on its tensor-core form: up to 64 tokens
  if (path == MOE_PATH_DECODE && s.T > kDecodeTcMaxT) return MOE_ERR_UNSUPPORTED;
  RouteOpt ro;
  if ((st = check_route_opts(s, opts ? opts->route : nullptr, &ro)) != MOE_OK) return st;
  if (!ws) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  const WsMap m = workspace_map(s);
  if (ws_bytes < m.total_fp8) return MOE_ERR_WORKSPACE;
  void* const* ev = opts ? opts->stage_events : nullptr;
  if (s.T == 0) {
    for (int i = 0; i <= MOE_NUM_STAGES; ++i)
      if (!mark(ev, i, stream)) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  const int G = s.E + s.n_shared;
  int32_t* ids = ids_out ? ids_out : reinterpret_cast<int32_t*>(at(ws, m.ids));
  float* w = w_out ? w_out : reinterpret_cast<float*>(at(ws, m.w));
  auto* offsets = reinterpret_cast<int32_t*>(at(ws, m.offsets));
  auto* sorted_slots = reinterpret_cast<int32_t*>(at(ws, m.sorted_slots));
  auto* slot_row = reinterpret_cast<int32_t*>(at(ws, m.slot_row));
  auto* err = reinterpret_cast<uint32_t*>(at(ws, m.err));
  auto* xq = reinterpret_cast<uint8_t*>(at(ws, m.x_q));
  auto* sx = reinterpret_cast<float*>(at(ws, m.s_x));
  auto* x_perm = reinterpret_cast<uint8_t*>(at(ws, m.x_perm));
  auto* a_scale = reinterpret_cast<float*>(at(ws, m.a_scale));
  auto* h = reinterpret_cast<__nv_bfloat16*>(at(ws, m.h));
  auto* hq = reinterpret_cast<uint8_t*>(at(ws, m.h_q));
  auto* sh = reinterpret_cast<float*>(at(ws, m.s_h));
  auto* stage = reinterpret_cast<float*>(at(ws, m.stage));
  float* acc = reinterpret_cast<float*>(at(ws, m.acc));
  const bool det = opts && opts->deterministic;
  const int cta_pairs = opts ? opts->cta_pairs : 0;
  if (use_router) logits = reinterpret_cast<float*>(at(ws, m.logits));

  if (path == MOE_PATH_DECODE || (path == MOE_PATH_AUTO && s.T <= kDecodeMaxT)) {
    // few tokens: stream only the touched experts' codes (decode.cu,
    // decode_tc.cu).  Stage 0: router and routing; 2: the codes of x;
    // 3: w13 + activation and the codes of h; 4: w2; 5: the row sum.
    DecodeArgs d{};
    d.x = reinterpret_cast<const __nv_bfloat16*>(x);
    d.logits = logits;
    d.scale = scale;
    d.T = (int)s.T;
    d.H = s.H;
    d.E = s.E;
    d.k = s.k;
    d.I = s.I;
    d.S = s.n_shared;
    d.act = s.act;
    d.route = ro;
    d.ids = ids;
    d.w = w;
    d.meta = reinterpret_cast<int32_t*>(at(ws, m.dec_meta));
    d.slots = sorted_slots;
    d.h_dec = h;
    d.stage = stage;
    d.out = reinterpret_cast<__nv_bfloat16*>(out);
    d.out_f32 = opts ? opts->out_f32 : nullptr;
    d.tc = true;
    d.dt_part = reinterpret_cast<float*>(at(ws, m.dt_part));
    d.dt_cnt = reinterpret_cast<int32_t*>(at(ws, m.dt_cnt));
    d.err = err;
    d.f8 = true;
    d.w13q = wq->w13;
    d.w2q = wq->w2;
    d.w13q_sh = wq->w13_sh;
    d.w2q_sh = wq->w2_sh;
    d.w13s = wq->w13_scale;
    d.w2s = wq->w2_scale;
    d.w13s_sh = wq->w13_sh_scale;
    d.w2s_sh = wq->w2_sh_scale;
    d.xq = xq;
    d.sx = sx;
    d.hq = hq;
    d.sh = sh;
    if (!use_router) return from_cuda(launch_decode(d, stream, ev));
    void* dev[MOE_NUM_STAGES + 1] = {};
    for (int i = 1; ev && i <= MOE_NUM_STAGES; ++i) dev[i] = ev[i];
    if (!mark(ev, 0, stream)) return MOE_ERR_CUDA;
    if (launch_router_logits(reinterpret_cast<const __nv_bfloat16*>(opts->router_x),
                             reinterpret_cast<const __nv_bfloat16*>(opts->router_w),
                             reinterpret_cast<const __nv_bfloat16*>(opts->router_scale),
                             s.T, s.H, s.E, opts->router_eps, const_cast<float*>(logits),
                             stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    return from_cuda(launch_decode(d, stream, ev ? dev : nullptr));
  }

  // stage 0: router (if any) and routing; 1: layout; 2: the codes of x and
  // their gather; 3: w13 + activation; 4: the codes of h and w2 + combine;
  // 5: the rounding
  if (!mark(ev, 0, stream)) return MOE_ERR_CUDA;
  if (use_router &&
      launch_router_logits(reinterpret_cast<const __nv_bfloat16*>(opts->router_x),
                           reinterpret_cast<const __nv_bfloat16*>(opts->router_w),
                           reinterpret_cast<const __nv_bfloat16*>(opts->router_scale), s.T,
                           s.H, s.E, opts->router_eps, const_cast<float*>(logits),
                           stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_route(logits, scale, s.T, s.E, s.k, ids, w, stream, ro) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (!mark(ev, 1, stream)) return MOE_ERR_CUDA;
  if (launch_layout(s, ids, offsets, sorted_slots, slot_row, m.cap,
                    reinterpret_cast<int32_t*>(at(ws, m.lt_count)),
                    reinterpret_cast<int32_t*>(at(ws, m.lt_base)),
                    reinterpret_cast<int32_t*>(at(ws, m.lt_rank)), m.n_lt, err, stream,
                    /*pdl=*/true) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (!mark(ev, 2, stream)) return MOE_ERR_CUDA;
  if (launch_quantize_rows(reinterpret_cast<const __nv_bfloat16*>(x), s.T, s.H, xq, sx,
                           nullptr, nullptr, stream, /*pdl=*/true) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_gather_fp8(xq, sx, sorted_slots, offsets, s.E, G, s.T, s.k, s.H, m.cap, x_perm,
                        a_scale, det ? nullptr : acc, s.T * (int64_t)s.H, stream,
                        /*pdl=*/true) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (!mark(ev, 3, stream)) return MOE_ERR_CUDA;
  GroupedGemmArgs a{};
  a.mode = 0;
  a.A = reinterpret_cast<const __nv_bfloat16*>(x_perm);
  a.A_sh = reinterpret_cast<const __nv_bfloat16*>(xq);
  a.B = reinterpret_cast<const __nv_bfloat16*>(wq->w13);
  a.B_sh = reinterpret_cast<const __nv_bfloat16*>(wq->w13_sh);
  a.offsets = offsets;
  a.G = G;
  a.E = s.E;
  a.N = s.I;
  a.K = s.H;
  a.cap = m.cap;
  a.out = h;
  a.act = s.act;
  a.err = err;
  a.sorted_slots = sorted_slots;
  a.w = w;
  a.T = s.T;
  a.k = s.k;
  a.pair = cta_pairs == 2;
  a.f8 = true;
  a.a_scale = a_scale;
  a.b_scale = wq->w13_scale;
  a.b_scale_sh = wq->w13_sh_scale;
  if (launch_grouped_gemm(a, stream, true) != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(ev, 4, stream)) return MOE_ERR_CUDA;
  // h rows in use: below offsets[G]; padding rows (slot -1) are skipped
  if (launch_quantize_rows(h, m.cap, s.I, hq, sh, offsets + G, sorted_slots, stream,
                           /*pdl=*/true) != cudaSuccess)
    return MOE_ERR_CUDA;
  const bool big = s.T * (int64_t)s.k >= 2 * 128 * (int64_t)s.E;
  a.mode = det ? 3 : 2;
  a.pair = cta_pairs == 2 || (cta_pairs == 0 && big && s.I >= 1024);
  a.A = reinterpret_cast<const __nv_bfloat16*>(hq);
  a.A_sh = nullptr;
  a.B = reinterpret_cast<const __nv_bfloat16*>(wq->w2);
  a.B_sh = reinterpret_cast<const __nv_bfloat16*>(wq->w2_sh);
  a.N = s.H;
  a.K = s.I;
  a.out = det ? stage : acc;
  a.a_scale = sh;
  a.b_scale = wq->w2_scale;
  a.b_scale_sh = wq->w2_sh_scale;
  if (launch_grouped_gemm(a, stream, true) != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(ev, 5, stream)) return MOE_ERR_CUDA;
  float* out_f32 = opts ? opts->out_f32 : nullptr;
  const cudaError_t e =
      det ? launch_sum_rows(stage, s.T, s.k + s.n_shared, s.H,
                            reinterpret_cast<__nv_bfloat16*>(out), out_f32, stream, true)
          : launch_finalize(acc, s.T * (int64_t)s.H, reinterpret_cast<__nv_bfloat16*>(out),
                            out_f32, stream, true);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return mark(ev, 6, stream) ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_read_error(void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!ws || ws_bytes < 256) return MOE_ERR_INVALID_ARG;
  uint32_t word = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&word, ws, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof word) != cudaSuccess) return MOE_ERR_CUDA;
  if (word == 0) return MOE_OK;
  if (word >= 1 && word <= MOE_ERR_TIMEOUT) return static_cast<moe_status>(word);
  return MOE_ERR_CUDA;
}

moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes,
                                     uint32_t timeout_us, cudaStream_t stream) {
  if (!ws || ws_bytes < 256 || timeout_us == 0 || timeout_us > 10000000u)
    return MOE_ERR_INVALID_ARG;
  return from_cuda(
      launch_wait_selftest(reinterpret_cast<uint32_t*>(ws), timeout_us, stream));
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

}  // extern "C"
