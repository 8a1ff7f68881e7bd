/*
 * moe.h -- C ABI of the sparse mixture-of-experts feed-forward layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (Gemma 4 MoE walkthrough, yeyulingfeng.com/587419.html,
 * sections 4-7; vLLM API page vllm.model_executor.models.gemma4, class
 * Gemma4MoE; llama-cpp-visual-guide lesson 35):
 *
 *   route    per token: top-k of the fp32 router logits, softmax over all E,
 *            mask to the chosen k, renormalise, times per_expert_scale[id];
 *   permute  reorder (token, choice) slots into expert-contiguous rows;
 *   expert   per row: h = Act(x W1^T) (*) (x W3^T), y = h W2^T, where
 *            W13 = [W1; W3] packs the gate rows first, then the up rows;
 *   combine  out[t] = sum_j w[t,j] y[t,j] + sum_s y_shared[t,s]  (bf16 out).
 *
 * Around it: the router ahead of the routing (moe_router_logits), routing
 * variants (moe_route_ex: sigmoid scoring, expert groups), the Gemma 4 MoE
 * block with its parallel dense MLP and gamma norms (moe_gemma4_block), the
 * layer with FP8 (e4m3) experts and per-row scales (moe_forward_fp8, with
 * its row quantiser moe_quantize_rows_e4m3), and a permutation that needs
 * no workspace (moe_permute_noalloc).
 *
 * Conventions (every entry point):
 *   - All pointers are DEVICE pointers unless a parameter says otherwise.
 *     The caller owns every buffer.  The library never allocates device
 *     memory, frees or synchronises (except moe_read_error, which says so);
 *     moe_gemma4_block creates one CUDA stream and two events per device on
 *     its first call there and keeps them.
 *   - Buffers are dense, row-major and 16-byte aligned.  The layer entry
 *     points (moe_expert_ffn, moe_forward, moe_forward_ex, moe_forward_fp8,
 *     moe_gemma4_block) check it for the token rows and the weights and
 *     return MOE_ERR_INVALID_ARG otherwise.
 *   - bf16 data is passed as uint16_t bit patterns (moe_bf16).
 *   - Work is enqueued on ``stream`` and runs asynchronously.
 *   - Argument and shape errors are returned before anything is launched.
 *     A launch failure returns MOE_ERR_CUDA.  A device-side wait that runs
 *     past its time limit records MOE_ERR_TIMEOUT in the workspace error
 *     word (its first 4 bytes), which moe_read_error returns and clears.
 *     Zero the first 256 bytes of a workspace once before its first use;
 *     the workspace must be 256-byte aligned.
 *   - Router logits must be finite.  With NaN or infinite logits the ids are
 *     still valid expert indices but their choice is unspecified.
 *   - Limits: 1 <= k <= min(E, 32), E <= 512, H % 8 == 0, I % 8 == 0,
 *     n_shared <= 8 and I_shared == I when n_shared > 0, pad == 128 (or 0
 *     for the default 128), T < 2^24.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

struct CUstream_st;
typedef struct CUstream_st* cudaStream_t;

typedef uint16_t moe_bf16;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* bad pointer, size or shape */
  MOE_ERR_UNSUPPORTED = 2, /* valid but outside the limits above */
  MOE_ERR_WORKSPACE = 3,   /* workspace smaller than moe_workspace_size */
  MOE_ERR_CUDA = 4,        /* a CUDA call or launch failed */
  MOE_ERR_TIMEOUT = 5      /* a device-side wait gave up (see moe_read_error) */
} moe_status;

typedef enum {
  MOE_ACT_SILU = 0,      /* v / (1 + e^-v) */
  MOE_ACT_GELU_TANH = 1  /* 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))) */
} moe_act;

typedef struct {
  int64_t T;        /* tokens */
  int32_t H;        /* hidden size */
  int32_t E;        /* routed experts */
  int32_t k;        /* experts chosen per token */
  int32_t I;        /* routed expert intermediate size */
  int32_t n_shared; /* always-active shared experts S (weight 1) */
  int32_t I_shared; /* shared expert intermediate size (== I when S > 0) */
  int32_t act;      /* moe_act */
  int32_t pad;      /* segment padding P in rows: 128, or 0 for 128 */
} moe_shape;

/* Rows of the permuted buffers: T*k + T*S + (E+S)*(P-1).  0 on a bad shape. */
MOE_API int64_t moe_layout_capacity(const moe_shape* shape);

/* Bytes of scratch every entry point below may use (one size for all). */
MOE_API size_t moe_workspace_size(const moe_shape* shape);

/*
 * moe_router_logits -- the router ahead of the routing (walkthrough section
 * 3, "Gemma4Router-MoE 的入口"; the Gemma4Router class on the vLLM page):
 *   x        [T,H] bf16 residual-stream rows (the router's own input, not
 *            the experts' normalised input)
 *   w_router [E,H] bf16 GateLinear weight
 *   scale    [H] bf16 learned per-dimension scale
 *   eps      RMSNorm epsilon (>= 0)
 *   logits   [T,E] fp32 out: z = GateLinear(bf16(bf16(bf16(RMSNorm(x))
 *            * bf16(H^-0.5)) * scale)); the norm in fp32 with no gamma, the
 *            projection accumulated in fp32.  The activations before the
 *            projection match the oracle exactly; the logits within the
 *            fp32 accumulation error.
 * Uses no workspace.  shape->k, I, n_shared, act are not read.
 */
MOE_API moe_status moe_router_logits(const moe_shape* shape, const moe_bf16* x,
                                     const moe_bf16* w_router, const moe_bf16* scale,
                                     float eps, float* logits, cudaStream_t stream);

/*
 * moe_route -- routing of every token (walkthrough section 4 steps 1-5 and
 * section 5; Gemma4MoE.routing_function on the vLLM page).
 *   logits [T,E] fp32, scale [E] fp32 or NULL (all ones)
 *   ids    [T,k] int32 out: the k largest logits, in descending order, equal
 *          logits to the lower id first (bit-exact with the oracle)
 *   w      [T,k] fp32 out: exp(z_id - z_max) / sum over the chosen k, times
 *          scale[id]; computed in fp64 and rounded once to fp32
 */
MOE_API moe_status moe_route(const moe_shape* shape, const float* logits,
                     const float* scale, int32_t* ids, float* w,
                     cudaStream_t stream);

/*
 * moe_route_ex -- the routing variants of llama-cpp-visual-guide lesson 35
 * (routing section: "some models use sigmoid"; the expert-group fold: pick a
 * group first, then experts within it, as n_expert_groups / n_group_used;
 * the DeepSeek-V3 row of its table: 256 routed experts, top-8).
 *   opts NULL, or:
 *     scoring     MOE_SCORE_SOFTMAX: exactly moe_route;
 *                 MOE_SCORE_SIGMOID: each chosen expert's weight is
 *                 sigmoid(z_id) / (sum of sigmoid over the chosen k), times
 *                 scale[id] (fp64, rounded once to fp32)
 *     n_group     0 or 1: no groups.  Else the E experts form n_group groups
 *                 of E / n_group consecutive ids (E % n_group == 0,
 *                 n_group <= 32); each token keeps its topk_group best
 *                 groups -- a group is scored by its largest logit, equal
 *                 scores to the lower group id -- and picks its k experts
 *                 among the experts of those groups only
 *     topk_group  1..n_group, with k <= topk_group * (E / n_group)
 *   Selection always compares the fp32 logits themselves (both scores are
 *   increasing in the logit), so ids and their order are bit-exact with the
 *   oracle.  Other arguments as moe_route.  Bad options return
 *   MOE_ERR_INVALID_ARG (or MOE_ERR_UNSUPPORTED for n_group > 32) before any
 *   launch.
 */
typedef enum {
  MOE_SCORE_SOFTMAX = 0,
  MOE_SCORE_SIGMOID = 1
} moe_scoring;
#define MOE_MAX_GROUPS 32
typedef struct {
  int32_t scoring;     /* moe_scoring */
  int32_t n_group;
  int32_t topk_group;
} moe_route_opts;

MOE_API moe_status moe_route_ex(const moe_shape* shape, const float* logits,
                                const float* scale, const moe_route_opts* opts,
                                int32_t* ids, float* w, cudaStream_t stream);

/*
 * moe_permute -- the dispatch permutation (walkthrough sections 6-7: the
 * "permutation map" turning token picks into per-expert token lists).
 *   ids          [T,k] int32 in (each in [0,E))
 *   offsets      [E+S+1] int32 out: first row of each expert segment; every
 *                segment is padded to a multiple of P rows; offsets[E+S] is
 *                the number of rows in use
 *   sorted_slots [cap] int32 out, cap = moe_layout_capacity: the slot held by
 *                each row, -1 on padding and past offsets[E+S].  Routed slot
 *                t*k+j; shared expert s holds slot T*k + s*T + t.  Within a
 *                segment slots ascend (a stable sort).
 *   slot_row     [T,k+S] int32 out: the row of (t, j), and of (t, shared s)
 *                at column k+s
 *   ws           workspace of ws_bytes >= moe_workspace_size bytes
 * An id outside [0,E) is a caller error that the kernels catch: its slot is
 * given no row (no segment counts it), its slot_row entry is -1, nothing is
 * written out of bounds, and the workspace error word records
 * MOE_ERR_INVALID_ARG, which moe_read_error returns.
 */
MOE_API moe_status moe_permute(const moe_shape* shape, const int32_t* ids,
                       int32_t* offsets, int32_t* sorted_slots,
                       int32_t* slot_row, void* ws, size_t ws_bytes,
                       cudaStream_t stream);

/*
 * moe_expert_ffn -- the gated expert FFN on every permuted row (walkthrough
 * section 6; "MOE Inference" blog, gated FFN: [y1,y3] = x [w1,w3]).
 *   x         [T,H] bf16
 *   offsets, sorted_slots  from moe_permute
 *   w13       [E,2I,H] bf16: rows [0,I) gate (w1), rows [I,2I) up (w3)
 *   w2        [E,H,I] bf16
 *   w13_sh    [S,2I,H] bf16 or NULL when S == 0;  w2_sh [S,H,I] likewise
 *   y_perm    [cap,H] fp32 out, 16-byte aligned (else MOE_ERR_INVALID_ARG):
 *             unweighted expert output of every row in use; padding rows
 *             get 0, rows past offsets[E+S] are not written
 * h = Act(g) (*) u is rounded to bf16 (the second GEMM's operand); every
 * product accumulates in fp32 on the tensor cores.
 */
MOE_API moe_status moe_expert_ffn(const moe_shape* shape, const moe_bf16* x,
                          const int32_t* offsets, const int32_t* sorted_slots,
                          const moe_bf16* w13, const moe_bf16* w2,
                          const moe_bf16* w13_sh, const moe_bf16* w2_sh,
                          float* y_perm, void* ws, size_t ws_bytes,
                          cudaStream_t stream);

/*
 * moe_combine -- weighted combine (walkthrough section 7 step 4; the weighted
 * sum after ggml_mul_mat_id in lesson 35), with shared experts at weight 1.
 *   y_perm [cap,H] fp32, slot_row [T,k+S] int32, w [T,k] fp32
 *   out    [T,H] bf16 out: w[t,j] * y rounded, then added in fp32 in order
 *          j = 0..k-1, then the shared experts; rounded once to bf16
 * A negative slot_row entry (a slot that moe_permute gave no row) adds
 * nothing.
 */
MOE_API moe_status moe_combine(const moe_shape* shape, const float* y_perm,
                       const int32_t* slot_row, const float* w, moe_bf16* out,
                       cudaStream_t stream);

/*
 * moe_forward -- the whole layer: route, permute, expert FFN and combine on
 * one stream, with every intermediate in the workspace (vLLM FusedMoE as the
 * walkthrough's section 6 describes it).  ids_out [T,k] and w_out [T,k] may
 * be NULL; when given they receive the routing.
 * Here the combine is fused into the w2 GEMM's epilogue: each expert row is
 * multiplied by its gate weight and added into an fp32 [T,H] accumulator
 * with vector reductions, which a last pass rounds once to bf16.  The order
 * of those fp32 additions is not fixed, so two calls may differ in the last
 * bits of the fp32 sum (and rarely by one bf16 ulp).  moe_forward_ex with
 * deterministic = 1 instead stores each weighted row at its (token, choice)
 * position and adds the k + S rows of a token in a fixed order: then the
 * result is reproducible and bit-identical to moe_expert_ffn followed by
 * moe_combine, at the cost of writing and reading T*(k+S)*H*4 more bytes.
 * The decode path is always deterministic.
 */
MOE_API moe_status moe_forward(const moe_shape* shape, const moe_bf16* x,
                       const float* logits, const moe_bf16* w13,
                       const moe_bf16* w2, const float* scale,
                       const moe_bf16* w13_sh, const moe_bf16* w2_sh,
                       moe_bf16* out, int32_t* ids_out, float* w_out,
                       void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * moe_forward_ex -- moe_forward with options (opts may be NULL):
 *   stage_events  NULL or MOE_NUM_STAGES + 1 cudaEvent_t created by the
 *                 caller (a NULL entry records nothing); event i is recorded
 *                 before stage i and event MOE_NUM_STAGES after the last one,
 *                 on ``stream``.  Stages:
 *                 0 route, 1 permute, 2 gather, 3 w13 GEMM + activation,
 *                 4 w2 GEMM + gate weight + combine, 5 bf16 rounding
 *                 (with deterministic = 1: the fixed-order sum over the
 *                 k + S rows of each token, then the rounding).
 *   out_f32       NULL or [T,H] fp32: also receives the layer output before
 *                 its rounding to bf16.
 *   path          which kernels run (moe_path).  The decode path (T small)
 *                 routes in one block and streams each touched expert's
 *                 weights once: for T <= 8 through skinny mma.sync kernels,
 *                 for 8 < T <= 64 through tcgen05 kernels that split the
 *                 weight stream evenly over all SMs, above that through the
 *                 skinny kernels' many-token form.  Its stages 1 and 2 are
 *                 empty (folded into stage 0).  Both paths compute the same
 *                 function; they differ in the order of fp32 additions
 *                 inside the products.
 *   router_w      NULL, or the router ahead of the routing (see
 *                 moe_router_logits): with router_w [E,H], router_x [T,H]
 *                 (the residual rows the router reads) and router_scale [H]
 *                 given, the logits are first computed from them into the
 *                 workspace with RMSNorm epsilon router_eps, and ``logits``
 *                 may be NULL.  On the prefill path this is part of stage 0;
 *                 on the decode path it runs before stage 0.
 *   route         NULL, or the routing variant of moe_route_ex (sigmoid
 *                 scoring, expert groups) used by stage 0 on both paths.
 */
#define MOE_NUM_STAGES 6
typedef enum {
  MOE_PATH_AUTO = 0,     /* decode path when T <= MOE_DECODE_MAX_T */
  MOE_PATH_PREFILL = 1,  /* tcgen05 grouped GEMMs over padded expert segments */
  MOE_PATH_DECODE = 2    /* touched experts streamed by skinny kernels; T <= 1024 */
} moe_path;
#define MOE_DECODE_MAX_T 16
typedef struct {
  void* const* stage_events;
  float* out_f32;
  int32_t path;           /* moe_path */
  int32_t deterministic;  /* prefill path: fixed-order combine (see above) */
  int32_t cta_pairs;      /* prefill GEMMs: 0 auto, 1 one CTA per tile, 2 CTA
                             pairs (2-SM MMA, M = 256); results are identical */
  const moe_bf16* router_x;      /* see router_w above */
  const moe_bf16* router_w;
  const moe_bf16* router_scale;
  float router_eps;
  const moe_route_opts* route;   /* NULL, or the routing variant (moe_route_ex) */
} moe_forward_opts;

MOE_API moe_status moe_forward_ex(
    const moe_shape* shape, const moe_bf16* x, const float* logits,
    const moe_bf16* w13, const moe_bf16* w2, const float* scale,
    const moe_bf16* w13_sh, const moe_bf16* w2_sh, moe_bf16* out,
    int32_t* ids_out, float* w_out, void* ws, size_t ws_bytes,
    const moe_forward_opts* opts, cudaStream_t stream);

/*
 * moe_permute_noalloc -- moe_permute for callers that cannot hand the library
 * a workspace: code that runs while a CUDA graph is being captured (where
 * cudaMalloc is not allowed), runtimes whose memory pool is fully reserved up
 * front, and plug-in hosts that pass only the input and output buffers at
 * launch time.  The pages have no counterpart of this entry point; it is a
 * deployment convenience.
 *
 * Same inputs, outputs and results as moe_permute.  Its scratch (per-block
 * histograms, bases and ranks of the counting sort, 1 MiB) is a fixed array
 * in device memory that the library holds on every GPU it is loaded on
 * until the process exits.  Nothing is allocated or freed by the call.
 *   - Limit: T*k <= MOE_NOALLOC_MAX_SLOTS; larger batches (and every shape
 *     moe_permute rejects) return MOE_ERR_UNSUPPORTED / MOE_ERR_INVALID_ARG
 *     before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture begins.
 *   - All calls share the one array: calls that may run at the same time on
 *     the GPU (other streams, other host threads) race and must not overlap.
 *     Every call writes the scratch it later reads, so nothing in the array
 *     has to start at zero and the previous call's leftovers do no harm.
 *   - An id outside [0,E) gets no row and slot_row -1, as in moe_permute;
 *     with no workspace there is no error word to record it in.
 *   - The cached address is kept with the id of the context it belongs to;
 *     after a device reset (a new primary context) the next call looks it
 *     up again, so that call too should come before any stream capture.
 */
#define MOE_NOALLOC_MAX_SLOTS 131072
MOE_API moe_status moe_permute_noalloc(const moe_shape* shape,
                                       const int32_t* ids, int32_t* offsets,
                                       int32_t* sorted_slots,
                                       int32_t* slot_row, cudaStream_t stream);

/*
 * moe_gemma4_block -- the MoE block of a Gemma 4 decoder layer (Gemma 4
 * walkthrough, yeyulingfeng.com/587419.html, section 1: the DecoderLayer
 * forward; section 7: its tensor flow).  From the residual x [T,H] bf16 (the
 * state after the attention half):
 *   h1  = post_ff_norm_1( mlp( pre_ff_norm(x) ) )      dense GeGLU MLP
 *   h2  = post_ff_norm_2( moe( pre_ff_norm_2(x), router(x) ) )
 *   out = post_ff_norm( h1 + h2 ) + x                  unweighted sum
 * The dense MLP is a gated FFN with the experts' activation (shape->act)
 * and intermediate size I_dense; the router is moe_router_logits on the raw
 * residual; the MoE is moe_forward_ex on the normalised one (no shared
 * experts: shape->n_shared must be 0).  Each norm is the standard RMSNorm
 * with a gamma (section 3), in fp32: y = bf16(fl(fl(x / sqrt(fl(mean x^2) +
 * eps)) * gamma)); every module returns bf16, h1 + h2 is one fp32 add
 * rounded to bf16, and the residual add is fp32, rounded once to bf16.
 *   x        [T,H] bf16; w13 [E,2I,H], w2 [E,H,I] bf16; scale [E] fp32 or NULL
 *   out      [T,H] bf16 out; out_f32 NULL or [T,H] fp32 out: the output
 *            before its final rounding
 *   ws       moe_gemma4_workspace_size(shape, I_dense) bytes, 256-byte
 *            aligned, owned by the caller, first 256 bytes zeroed once (its
 *            error word: moe_read_error covers both branches)
 * The two branches run side by side: after the input norms on ``stream``
 * the dense MLP is forked onto a second stream of the library's own (one per
 * device, made on the first call) and joined back by an event before the
 * output norms, so ``stream`` alone orders the call with the caller's work,
 * and the call can be captured into a CUDA graph (make the first call on a
 * device outside a capture: it creates that stream).  Calls from several
 * host threads are serialised while they enqueue.
 * Bad shapes or arguments return before any launch.
 */
typedef struct {
  int32_t I_dense;                /* dense MLP intermediate size (multiple of 8) */
  const moe_bf16* mlp_w13;        /* [2*I_dense, H], gate rows first */
  const moe_bf16* mlp_w2;         /* [H, I_dense] */
  const moe_bf16* norm_w[5];      /* [H] gammas: pre_ff, post_ff_1, pre_ff_2,
                                     post_ff_2, post_ff (16-byte aligned) */
  float eps;                      /* epsilon of those five norms */
  const moe_bf16* router_w;       /* [E,H] GateLinear weight */
  const moe_bf16* router_scale;   /* [H] */
  float router_eps;
} moe_gemma4_block_params;

MOE_API size_t moe_gemma4_workspace_size(const moe_shape* shape, int32_t I_dense);
MOE_API moe_status moe_gemma4_block(const moe_shape* shape, const moe_bf16* x,
                                    const moe_gemma4_block_params* params,
                                    const moe_bf16* w13, const moe_bf16* w2,
                                    const float* scale, moe_bf16* out, float* out_f32,
                                    void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * FP8 experts.  Per-expert FP8 checkpoints store each expert's gate, up and
 * down weights with a weight_scale, which FusedMoE packs as w13_weight /
 * w2_weight and their _scale parameters (prhub.com.cn, sglang PR #24696,
 * the per-expert FP8 loader fix; vLLM API page, load_weights).  The pages fix
 * neither the format nor the scale granularity; this library reads them as:
 *   - a weight is an e4m3 (E4M3FN) code times one fp32 scale per output row;
 *   - activations are quantised per row when the layer runs: with amax the
 *     row's largest |value|, s = fl32(amax / 448) (1 for an all-zero row) and
 *     code = the nearest e4m3 value of fl32(v / s), ties to even, saturating
 *     at +-448 ("FP8-Dynamic").  The intermediate h is quantised the same
 *     way, per (token, expert) row.
 * The products run on the tensor cores as e4m3 x e4m3 with fp32
 * accumulation (tcgen05 kind::f8f6f4); both scales are applied to the fp32
 * result.
 */
typedef struct {
  const uint8_t* w13;          /* [E,2I,H] e4m3 codes, gate rows first */
  const float* w13_scale;      /* [E,2I] */
  const uint8_t* w2;           /* [E,H,I] */
  const float* w2_scale;       /* [E,H] */
  const uint8_t* w13_sh;       /* [S,2I,H], or NULL when S == 0 */
  const float* w13_sh_scale;   /* [S,2I] */
  const uint8_t* w2_sh;        /* [S,H,I] */
  const float* w2_sh_scale;    /* [S,H] */
} moe_fp8_experts;

/*
 * moe_quantize_rows_e4m3 -- the per-row dynamic quantisation above, of bf16
 * rows src [rows, cols] (cols % 8 == 0, src 16-byte aligned) into codes
 * [rows, cols] (8-byte aligned) and scales [rows].  It turns bf16 expert
 * weights into the FP8 form (rows = output channels) as well.  Each code and
 * scale is fixed by IEEE fp32 arithmetic, so it is reproducible bit for bit.
 * Argument errors return MOE_ERR_INVALID_ARG before any launch.
 */
MOE_API moe_status moe_quantize_rows_e4m3(const moe_bf16* src, int64_t rows, int cols,
                                          uint8_t* codes, float* scales,
                                          cudaStream_t stream);

/* Workspace bytes of moe_forward_fp8 (0 for an invalid shape). */
MOE_API size_t moe_workspace_size_fp8(const moe_shape* shape);

/*
 * moe_forward_fp8 -- the layer of moe_forward_ex with FP8 experts:
 * routing, permutation, x quantised per token and gathered, the w13
 * product (+ activation, h in bf16), h quantised per row, the w2 product
 * with the gate weights and the combine, one bf16 rounding.  Requires
 * H % 16 == 0 and I % 16 == 0 (MOE_ERR_UNSUPPORTED otherwise) and a
 * workspace of moe_workspace_size_fp8 bytes (MOE_ERR_WORKSPACE).  The decode
 * path (MOE_PATH_DECODE, or MOE_PATH_AUTO with T <= MOE_DECODE_MAX_T) runs
 * the decode path's tcgen05 form on the codes of the touched experts (up to
 * 64 tokens: MOE_ERR_UNSUPPORTED beyond) and is deterministic; the prefill
 * path runs the tcgen05 grouped GEMMs.  The other options (stage events,
 * out_f32, deterministic, cta_pairs, router, route) mean what they mean for
 * moe_forward_ex.
 */
MOE_API moe_status moe_forward_fp8(const moe_shape* shape, const moe_bf16* x,
                                   const float* logits, const moe_fp8_experts* weights,
                                   const float* scale, moe_bf16* out, int32_t* ids_out,
                                   float* w_out, void* ws, size_t ws_bytes,
                                   const moe_forward_opts* opts, cudaStream_t stream);

/*
 * moe_read_error -- SYNCHRONISES ``stream``, then returns the status recorded
 * in the workspace error word by earlier calls on it (MOE_OK if none) and
 * clears the word.  ws is the device workspace used by those calls.
 */
MOE_API moe_status moe_read_error(void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * moe_selftest_wait_timeout -- exercises the device-side wait limit: launches
 * one block that waits on a flag nothing ever sets, for at most timeout_us
 * microseconds, then records MOE_ERR_TIMEOUT in the workspace error word and
 * returns.  No GPU fault, trap or hang is involved.
 */
MOE_API moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes,
                                     uint32_t timeout_us, cudaStream_t stream);

/* A static, human-readable name for a status. */
MOE_API const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
