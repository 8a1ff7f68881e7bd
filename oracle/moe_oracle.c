/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle for the sparse MoE
 * feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library; the two meet only in the seeded input generators.
 *
 * What it computes, and where the pages define it:
 *
 *   route   -- yeyulingfeng.com/587419.html, section 4 (routing math): top-k
 *              on the raw fp32 router logits, softmax over ALL E logits, a
 *              0/1 indicator mask of the chosen k, renormalisation of the
 *              masked probabilities with the guard "sum > 0 ? sum : 1", and a
 *              gather to [T,k].  Section 5 (per-expert scale) and the
 *              Gemma4MoE routing_function on the vLLM API page
 *              (vllm.model_executor.models.gemma4) then multiply each weight
 *              by per_expert_scale[id] after the renormalisation.
 *   layout  -- section 7 (tensor flow) of the same walkthrough: "token picks
 *              k experts" is reordered into "expert receives a token list".
 *              The pages leave the permutation unspecified; this oracle
 *              fixes it as a stable counting sort of the flat slot t*k+j by
 *              expert, every expert segment padded to a multiple of P rows
 *              with -1, shared-expert segments after the routed ones.
 *   expert  -- gated FFN of the "MOE Inference" blog (gaohongy.github.io,
 *              "门控(Gated) FFN"): y = (Act(x.w1) (*) (x.w3)) . w2, with the
 *              packed [w1, w3] = w13 (gate rows first, up rows second, as in
 *              section 6 of the walkthrough and load_weights on the vLLM
 *              page).  Act is SiLU, v/(1+e^-v), or the tanh GELU,
 *              0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))) (walkthrough
 *              section 6).
 *   route_ex -- llama-cpp-visual-guide lesson 35: sigmoid scoring and expert
 *              groups (see oracle_route_ex).
 *   gemma4 block -- section 1 of the Gemma 4 walkthrough: the dense MLP and
 *              the MoE in parallel from the same residual, each between its
 *              own gamma RMSNorms, summed unweighted, then a last norm and
 *              the residual add (see oracle_gemma4_block).
 *   combine -- walkthrough section 7 step 4: the k expert outputs of a token
 *              are summed weighted by its (scale-folded) gate weights; shared
 *              experts (llama-cpp-visual-guide lesson 35, "shared expert")
 *              are added with weight 1.
 *
 * All floating point is double; bf16 inputs convert to double exactly.
 * Nothing is blocked, fused or reordered beyond the definitions above.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define OK 0
#define EINVAL_ARG (-1)
#define ENOMEM_ARG (-2)

/* ---------------------------------------------------------------- helpers */

static double bf16_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bf16 value (8 significant bits, ties to
 * even), returned as a double.  Used by the diagnostic "round h" flag and
 * by the FP8 layer's bf16 intermediate. */
static double round_to_bf16(double v) {
  if (v == 0.0 || !isfinite(v)) return v;
  int e;
  double m = frexp(v, &e);          /* v = m * 2^e, 0.5 <= |m| < 1 */
  double r = nearbyint(ldexp(m, 8)); /* default rounding mode: ties to even */
  return ldexp(r, e - 8);
}

int oracle_num_threads(void) {
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

typedef void (*range_fn)(void* ctx, int64_t begin, int64_t end);
typedef struct {
  range_fn fn;
  void* ctx;
  int64_t begin, end;
} range_job;

static void* range_thread(void* p) {
  range_job* j = (range_job*)p;
  j->fn(j->ctx, j->begin, j->end);
  return NULL;
}

/* Run fn over [0,n) split into contiguous chunks, one per thread. */
static void parallel_for(int64_t n, int nthreads, range_fn fn, void* ctx) {
  if (nthreads <= 0) nthreads = oracle_num_threads();
  if (nthreads > n) nthreads = (int)(n > 0 ? n : 1);
  if (nthreads <= 1) {
    fn(ctx, 0, n);
    return;
  }
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
  range_job* jobs = (range_job*)malloc(sizeof(range_job) * nthreads);
  int64_t chunk = (n + nthreads - 1) / nthreads;
  int started = 0;
  for (int i = 0; i < nthreads; ++i) {
    int64_t b = i * chunk, e = b + chunk < n ? b + chunk : n;
    if (b >= e) break;
    jobs[i].fn = fn;
    jobs[i].ctx = ctx;
    jobs[i].begin = b;
    jobs[i].end = e;
    if (pthread_create(&th[i], NULL, range_thread, &jobs[i]) != 0) {
      fn(ctx, b, e); /* could not start a thread: do the chunk inline */
      jobs[i].fn = NULL;
    }
    started = i + 1;
  }
  for (int i = 0; i < started; ++i)
    if (jobs[i].fn) pthread_join(th[i], NULL);
  free(th);
  free(jobs);
}

/* ------------------------------------------------------------ activation */

/* Act(v): 0 = SiLU v/(1+exp(-v)); 1 = tanh GELU
 * 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))). */
static double act_fn(int act, double v) {
  if (act == 0) return v / (1.0 + exp(-v));
  const double c = sqrt(2.0 / M_PI);
  return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

int oracle_act(int act, int64_t n, const double* v, double* out) {
  if (act != 0 && act != 1) return EINVAL_ARG;
  for (int64_t i = 0; i < n; ++i) out[i] = act_fn(act, v[i]);
  return OK;
}

/* ----------------------------------------------------------------- route */

typedef struct {
  float v;
  int id;
} logit_id;

/* Descending logit; equal logits go to the lower expert id first. */
static int cmp_logit_desc(const void* a, const void* b) {
  const logit_id* x = (const logit_id*)a;
  const logit_id* y = (const logit_id*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

/*
 * Routing of every token (walkthrough section 4 steps 1-5, section 5 fold).
 *   logits [T,E] fp32, scale [E] fp32 or NULL (= all ones)
 *   ids    [T,k] int32 out, ordered by descending logit, ties to lower id
 *   w      [T,k] double out (renormalised, then times scale[id])
 *   probs  [T,E] double out or NULL: the softmax over all E (step 2)
 * Returns -1 on a bad size or a non-finite logit.
 */
int oracle_route(int64_t T, int E, int k, const float* logits,
                 const float* scale, int32_t* ids, double* w, double* probs) {
  if (T < 0 || E < 1 || k < 1 || k > E) return EINVAL_ARG;
  logit_id* pairs = (logit_id*)malloc(sizeof(logit_id) * E);
  double* p = (double*)malloc(sizeof(double) * E);
  double* gate = (double*)malloc(sizeof(double) * E);
  if (!pairs || !p || !gate) {
    free(pairs); free(p); free(gate);
    return ENOMEM_ARG;
  }
  int rc = OK;
  for (int64_t t = 0; t < T && rc == OK; ++t) {
    const float* z = logits + t * E;
    for (int e = 0; e < E; ++e) {
      if (!isfinite(z[e])) { rc = EINVAL_ARG; break; }
      pairs[e].v = z[e];
      pairs[e].id = e;
    }
    if (rc != OK) break;
    /* step 1: top-k on the raw logits */
    qsort(pairs, (size_t)E, sizeof(logit_id), cmp_logit_desc);
    /* step 2: softmax over all E (shifted by the max, same value) */
    double zmax = (double)pairs[0].v, den = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp((double)z[e] - zmax);
      den += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= den;
    if (probs) memcpy(probs + t * E, p, sizeof(double) * E);
    /* steps 3-4: indicator of the chosen k times the probabilities */
    for (int e = 0; e < E; ++e) gate[e] = 0.0;
    for (int j = 0; j < k; ++j) gate[pairs[j].id] = p[pairs[j].id];
    /* step 5: renormalise with the guard sum > 0 ? sum : 1 */
    double renorm = 0.0;
    for (int e = 0; e < E; ++e) renorm += gate[e];
    if (!(renorm > 0.0)) renorm = 1.0;
    /* gather to [T,k], then fold per_expert_scale (section 5) */
    for (int j = 0; j < k; ++j) {
      int id = pairs[j].id;
      ids[t * k + j] = id;
      double wt = gate[id] / renorm;
      if (scale) wt *= (double)scale[id];
      w[t * k + j] = wt;
    }
  }
  free(pairs);
  free(p);
  free(gate);
  return rc;
}

/* Descending group score; equal scores go to the lower group id first. */
typedef struct {
  float v;
  int g;
} group_score;

static int cmp_group_desc(const void* a, const void* b) {
  const group_score* x = (const group_score*)a;
  const group_score* y = (const group_score*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->g > y->g) - (x->g < y->g);
}

/*
 * Routing variants of llama-cpp-visual-guide lesson 35 (routing section and
 * the shared-expert / expert-group fold):
 *   scoring 0 -- probabilities are the softmax over all E logits (the
 *                listing's ggml_soft_max), exactly oracle_route;
 *   scoring 1 -- probabilities are sigmoid(logit) per expert (the listing's
 *                "some models use sigmoid");
 *   n_group > 1 -- the E experts form n_group groups of E / n_group
 *                consecutive ids; a token first picks its topk_group best
 *                groups, then its k experts among the experts of those
 *                groups ("pick a group first, then experts within it").
 *                A group's score is the best probability among its experts
 *                (reading: the page does not say how a group is scored).
 * Then, as in the listing: top-k of the probabilities (ties to the lower
 * id), the k probabilities gathered and normalised to sum 1, and (section 5
 * of the Gemma 4 walkthrough) times per_expert_scale[id].  Sigmoid and
 * softmax are increasing in the logit, so the probabilities are ranked by
 * comparing the fp32 logits themselves (exact).
 * Returns -1 on bad sizes (E % n_group, topk_group out of range, fewer than
 * k experts in topk_group groups) or a non-finite logit.
 */
int oracle_route_ex(int64_t T, int E, int k, const float* logits,
                    const float* scale, int scoring, int n_group,
                    int topk_group, int32_t* ids, double* w) {
  if (n_group < 1) n_group = 1;
  if (n_group == 1) topk_group = 1;
  if (T < 0 || E < 1 || k < 1 || k > E || (scoring != 0 && scoring != 1))
    return EINVAL_ARG;
  if (E % n_group != 0 || topk_group < 1 || topk_group > n_group ||
      k > topk_group * (E / n_group))
    return EINVAL_ARG;
  const int gs = E / n_group;
  logit_id* pairs = (logit_id*)malloc(sizeof(logit_id) * E);
  group_score* gsc = (group_score*)malloc(sizeof(group_score) * n_group);
  int* keep = (int*)malloc(sizeof(int) * n_group);
  double* p = (double*)malloc(sizeof(double) * E);
  if (!pairs || !gsc || !keep || !p) {
    free(pairs); free(gsc); free(keep); free(p);
    return ENOMEM_ARG;
  }
  int rc = OK;
  for (int64_t t = 0; t < T && rc == OK; ++t) {
    const float* z = logits + t * E;
    for (int e = 0; e < E; ++e)
      if (!isfinite(z[e])) { rc = EINVAL_ARG; break; }
    if (rc != OK) break;
    /* probabilities of every expert */
    if (scoring == 0) {
      double zmax = (double)z[0], den = 0.0;
      for (int e = 1; e < E; ++e) if ((double)z[e] > zmax) zmax = (double)z[e];
      for (int e = 0; e < E; ++e) { p[e] = exp((double)z[e] - zmax); den += p[e]; }
      for (int e = 0; e < E; ++e) p[e] /= den;
    } else {
      for (int e = 0; e < E; ++e) p[e] = 1.0 / (1.0 + exp(-(double)z[e]));
    }
    /* groups: each scored by its best member, the topk_group best kept */
    for (int g = 0; g < n_group; ++g) {
      float best = z[g * gs];
      for (int i = 1; i < gs; ++i) if (z[g * gs + i] > best) best = z[g * gs + i];
      gsc[g].v = best;
      gsc[g].g = g;
      keep[g] = 0;
    }
    qsort(gsc, (size_t)n_group, sizeof(group_score), cmp_group_desc);
    for (int i = 0; i < topk_group; ++i) keep[gsc[i].g] = 1;
    /* top-k among the experts of the kept groups */
    int n = 0;
    for (int e = 0; e < E; ++e) {
      if (!keep[e / gs]) continue;
      pairs[n].v = z[e];
      pairs[n].id = e;
      ++n;
    }
    qsort(pairs, (size_t)n, sizeof(logit_id), cmp_logit_desc);
    /* gather the k probabilities and normalise them to sum 1 */
    double sum = 0.0;
    for (int j = 0; j < k; ++j) sum += p[pairs[j].id];
    if (!(sum > 0.0)) sum = 1.0;
    for (int j = 0; j < k; ++j) {
      const int id = pairs[j].id;
      double wt = p[id] / sum;
      if (scale) wt *= (double)scale[id];
      ids[t * k + j] = id;
      w[t * k + j] = wt;
    }
  }
  free(pairs); free(gsc); free(keep); free(p);
  return rc;
}

/* ---------------------------------------------------------------- layout */

/* Rows the permuted buffers need in the worst case:
 * T*k + T*S + (E+S)*(P-1). */
int64_t oracle_layout_capacity(int64_t T, int E, int k, int S, int P) {
  return T * k + T * S + (int64_t)(E + S) * (P - 1);
}

/*
 * Stable counting sort of the flat slots s = t*k + j by expert.
 *   offsets      [E+S+1]  start row of each segment, each a multiple of P;
 *                         offsets[E+S] = rows in use
 *   sorted_slots [cap]    slot held by each permuted row, -1 on padding;
 *                         shared expert s holds tokens 0..T-1 as the slots
 *                         T*k + s*T + t
 *   slot_row     [T,k+S]  permuted row of (token t, choice j) and of
 *                         (token t, shared expert s) at column k+s
 */
int oracle_layout(int64_t T, int E, int k, int S, int P, const int32_t* ids,
                  int32_t* offsets, int32_t* sorted_slots, int64_t cap,
                  int32_t* slot_row) {
  if (T < 0 || E < 1 || k < 1 || k > E || S < 0 || P < 1) return EINVAL_ARG;
  int G = E + S;
  int64_t* count = (int64_t*)calloc((size_t)G, sizeof(int64_t));
  int64_t* cursor = (int64_t*)malloc(sizeof(int64_t) * G);
  if (!count || !cursor) {
    free(count); free(cursor);
    return ENOMEM_ARG;
  }
  for (int64_t s = 0; s < T * k; ++s) {
    int e = ids[s];
    if (e < 0 || e >= E) { free(count); free(cursor); return EINVAL_ARG; }
    count[e]++;
  }
  for (int s = 0; s < S; ++s) count[E + s] = T;
  int64_t off = 0;
  for (int g = 0; g < G; ++g) {
    offsets[g] = (int32_t)off;
    cursor[g] = off;
    off += (count[g] + P - 1) / P * P;
  }
  offsets[G] = (int32_t)off;
  if (off > cap) { free(count); free(cursor); return EINVAL_ARG; }
  for (int64_t r = 0; r < cap; ++r) sorted_slots[r] = -1;
  for (int64_t s = 0; s < T * k; ++s) {
    int64_t t = s / k, j = s % k;
    int64_t row = cursor[ids[s]]++;
    sorted_slots[row] = (int32_t)s;
    slot_row[t * (k + S) + j] = (int32_t)row;
  }
  for (int s = 0; s < S; ++s)
    for (int64_t t = 0; t < T; ++t) {
      int64_t row = cursor[E + s]++;
      sorted_slots[row] = (int32_t)(T * k + s * T + t);
      slot_row[t * (k + S) + k + s] = (int32_t)row;
    }
  free(count);
  free(cursor);
  return OK;
}

/* ------------------------------------------------------------ expert FFN */

/* y[H] += weight * W2 (Act(W1 x) (*) W3 x) for one token row, where
 * w13e = [W1; W3] is [2I,H] and w2e is [H,I]. */
static void ffn_row(int H, int I, int act, const uint16_t* x,
                    const uint16_t* w13e, const uint16_t* w2e, int round_h,
                    double weight, double* xd, double* a, double* y) {
  for (int h = 0; h < H; ++h) xd[h] = bf16_to_double(x[h]);
  for (int i = 0; i < I; ++i) {
    const uint16_t* r1 = w13e + (int64_t)i * H;        /* gate row */
    const uint16_t* r3 = w13e + (int64_t)(I + i) * H;  /* up row */
    double g = 0.0, u = 0.0;
    for (int h = 0; h < H; ++h) {
      g += xd[h] * bf16_to_double(r1[h]);
      u += xd[h] * bf16_to_double(r3[h]);
    }
    double v = act_fn(act, g) * u;
    a[i] = round_h ? round_to_bf16(v) : v;
  }
  for (int h = 0; h < H; ++h) {
    const uint16_t* r2 = w2e + (int64_t)h * I;
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += a[i] * bf16_to_double(r2[i]);
    y[h] += weight * acc;
  }
}

typedef struct {
  int H, I, act, round_h;
  const uint16_t* x;
  const uint16_t* w13;
  const uint16_t* w2;
  const int64_t* tok;
  const int32_t* exp_id;
  double* y;
} rows_ctx;

static void rows_worker(void* p, int64_t b, int64_t e) {
  rows_ctx* c = (rows_ctx*)p;
  double* xd = (double*)malloc(sizeof(double) * c->H);
  double* a = (double*)malloc(sizeof(double) * c->I);
  for (int64_t r = b; r < e; ++r) {
    double* y = c->y + r * c->H;
    for (int h = 0; h < c->H; ++h) y[h] = 0.0;
    int64_t ex = c->exp_id[r];
    ffn_row(c->H, c->I, c->act, c->x + c->tok[r] * c->H,
            c->w13 + ex * 2 * (int64_t)c->I * c->H,
            c->w2 + ex * (int64_t)c->H * c->I, c->round_h, 1.0, xd, a, y);
  }
  free(xd);
  free(a);
}

/*
 * Unweighted expert outputs of n (token, expert) pairs:
 *   y[r,:] = W2_e (Act(W1_e x_t) (*) W3_e x_t),  t = tok[r], e = exp_id[r],
 * with w13 [*,2I,H] and w2 [*,H,I] the packed weights of that expert set.
 */
int oracle_expert_rows(int H, int I, int act, const uint16_t* x,
                       const uint16_t* w13, const uint16_t* w2, int64_t n,
                       const int64_t* tok, const int32_t* exp_id, int round_h,
                       int nthreads, double* y) {
  if (H < 1 || I < 1 || (act != 0 && act != 1) || n < 0) return EINVAL_ARG;
  rows_ctx c = {H, I, act, round_h, x, w13, w2, tok, exp_id, y};
  parallel_for(n, nthreads, rows_worker, &c);
  return OK;
}

/* --------------------------------------------------------------- forward */

typedef struct {
  int64_t T;
  int H, E, k, I, act, S, Is, round_h;
  const uint16_t *x, *w13, *w2, *w13_sh, *w2_sh;
  const int32_t* ids;
  const double* w;
  const int64_t* tokens;
  double* out;
} fwd_ctx;

static void fwd_worker(void* p, int64_t b, int64_t e) {
  fwd_ctx* c = (fwd_ctx*)p;
  int Imax = c->I > c->Is ? c->I : c->Is;
  double* xd = (double*)malloc(sizeof(double) * c->H);
  double* a = (double*)malloc(sizeof(double) * Imax);
  for (int64_t r = b; r < e; ++r) {
    int64_t t = c->tokens ? c->tokens[r] : r;
    double* y = c->out + r * c->H;
    for (int h = 0; h < c->H; ++h) y[h] = 0.0;
    const uint16_t* xt = c->x + t * c->H;
    for (int j = 0; j < c->k; ++j) {
      int64_t ex = c->ids[t * c->k + j];
      ffn_row(c->H, c->I, c->act, xt, c->w13 + ex * 2 * (int64_t)c->I * c->H,
              c->w2 + ex * (int64_t)c->H * c->I, c->round_h,
              c->w[t * c->k + j], xd, a, y);
    }
    for (int s = 0; s < c->S; ++s)
      ffn_row(c->H, c->Is, c->act, xt,
              c->w13_sh + (int64_t)s * 2 * c->Is * c->H,
              c->w2_sh + (int64_t)s * c->H * c->Is, c->round_h, 1.0, xd, a, y);
  }
  free(xd);
  free(a);
}

/*
 * The whole layer for the tokens listed in ``tokens`` (NULL = all T):
 *   out[r,:] = sum_j w[t,j] * FFN_{ids[t,j]}(x_t) + sum_s FFN_shared_s(x_t)
 * Routing is done for all T tokens; ids_out/w_out (NULL ok) receive it.
 */
/* oracle_forward with the routing of oracle_route_ex (scoring, expert
 * groups); scoring 0 with one group is oracle_forward itself. */
int oracle_forward_ex(int64_t T, int H, int E, int k, int I, int act, int S,
                      int Is, const uint16_t* x, const float* logits,
                      const float* scale, const uint16_t* w13,
                      const uint16_t* w2, const uint16_t* w13_sh,
                      const uint16_t* w2_sh, const int64_t* tokens,
                      int64_t n_tokens, int round_h, int nthreads, double* out,
                      int32_t* ids_out, double* w_out, int scoring, int n_group,
                      int topk_group) {
  if (T < 0 || H < 1 || I < 1 || S < 0 || (S > 0 && (Is < 1 || !w13_sh || !w2_sh)))
    return EINVAL_ARG;
  int32_t* ids = ids_out ? ids_out : (int32_t*)malloc(sizeof(int32_t) * (T * k + 1));
  double* w = w_out ? w_out : (double*)malloc(sizeof(double) * (T * k + 1));
  if (!ids || !w) return ENOMEM_ARG;
  int rc = (scoring == 0 && n_group <= 1)
               ? oracle_route(T, E, k, logits, scale, ids, w, NULL)
               : oracle_route_ex(T, E, k, logits, scale, scoring, n_group, topk_group,
                                 ids, w);
  if (rc == OK) {
    if (!tokens) n_tokens = T;
    for (int64_t r = 0; tokens && r < n_tokens; ++r)
      if (tokens[r] < 0 || tokens[r] >= T) rc = EINVAL_ARG;
  }
  if (rc == OK) {
    fwd_ctx c = {T, H, E, k, I, act, S, Is, round_h, x, w13, w2, w13_sh,
                 w2_sh, ids, w, tokens, out};
    parallel_for(n_tokens, nthreads, fwd_worker, &c);
  }
  if (!ids_out) free(ids);
  if (!w_out) free(w);
  return rc;
}

int oracle_forward(int64_t T, int H, int E, int k, int I, int act, int S,
                   int Is, const uint16_t* x, const float* logits,
                   const float* scale, const uint16_t* w13,
                   const uint16_t* w2, const uint16_t* w13_sh,
                   const uint16_t* w2_sh, const int64_t* tokens,
                   int64_t n_tokens, int round_h, int nthreads, double* out,
                   int32_t* ids_out, double* w_out) {
  return oracle_forward_ex(T, H, E, k, I, act, S, Is, x, logits, scale, w13, w2,
                           w13_sh, w2_sh, tokens, n_tokens, round_h, nthreads, out,
                           ids_out, w_out, 0, 1, 1);
}

/* ----------------------------------------------------------------- router */

/*
 * router -- the step ahead of the routing: "Gemma4Router-MoE 的入口"
 * (section 3 of the Gemma 4 walkthrough, yeyulingfeng.com/587419.html) and
 * the Gemma4Router class on the vLLM API page.  For every residual row r
 * (bf16, H values):
 *   1. RMSNorm with no gamma, computed in fp32 and returned in the input
 *      dtype: n_h = bf16( fl(r_h * fl(1 / fl(sqrt(fl(v + eps))))) ), where
 *      v = fl(mean_h r_h^2) is taken in double and rounded once to fp32 and
 *      fl() is an fp32 operation (IEEE, round to nearest even);
 *   2. times the constant hidden_size^-0.5, itself cast to bf16 first (the
 *      fp32 buffer .to(x.dtype)): a_h = bf16( n_h * bf16(fl(H^-0.5)) );
 *   3. times the learned per-dimension scale in bf16: b_h = bf16(a_h * s_h);
 *   4. GateLinear: bf16 activations and weights, fp32 output:
 *      z[e] = fl( sum_h b_h * W[e,h] ), the sum in double.
 * Products of two bf16 values are exact in double (and in fp32), so steps 2
 * and 3 round exactly once each, as a bf16 multiply does.
 */
int oracle_router_logits(int64_t T, int H, int E, double eps, const uint16_t* x,
                         const uint16_t* w_router, const uint16_t* scale,
                         float* logits) {
  if (T < 0 || H < 1 || E < 1 || !(eps >= 0.0) || !x || !w_router || !scale || !logits)
    return EINVAL_ARG;
  double* b = (double*)malloc(sizeof(double) * (size_t)H);
  if (!b) return ENOMEM_ARG;
  const double root = round_to_bf16((double)(float)pow((double)H, -0.5));
  for (int64_t t = 0; t < T; ++t) {
    const uint16_t* r = x + t * (int64_t)H;
    double ss = 0.0;
    for (int h = 0; h < H; ++h) {
      const double v = bf16_to_double(r[h]);
      ss += v * v;
    }
    const float var = (float)(ss / (double)H);
    const float den = sqrtf(var + (float)eps);
    const float inv = 1.0f / den;
    for (int h = 0; h < H; ++h) {
      const float n = (float)bf16_to_double(r[h]) * inv;
      const double nb = round_to_bf16((double)n);
      const double a = round_to_bf16(nb * root);
      b[h] = round_to_bf16(a * bf16_to_double(scale[h]));
    }
    for (int e = 0; e < E; ++e) {
      const uint16_t* wr = w_router + (int64_t)e * H;
      double z = 0.0;
      for (int h = 0; h < H; ++h) z += b[h] * bf16_to_double(wr[h]);
      logits[t * (int64_t)E + e] = (float)z;
    }
  }
  free(b);
  return OK;
}

/* ------------------------------------------------------- gemma 4 block */

/*
 * Gamma RMSNorm of one row of bf16 values (walkthrough section 3: the
 * standard RMSNorm is y = x / RMS(x) * gamma; the Gemma 4 norms compute in
 * fp32 and return the activation dtype).  Reading of the fp32 steps, as for
 * the router's norm: v = fp32(mean of the squares, taken in double),
 * inv = 1 / sqrt(v + eps) in fp32, y_h = bf16( fp32( fp32(x_h * inv) * g_h ) ).
 *   x [H] bf16 values held in double, g [H] bf16, y [H] out (bf16 values)
 */
static void gamma_rms_norm_row(const double* x, int H, double eps, const uint16_t* g,
                               double* y) {
  double ss = 0.0;
  for (int h = 0; h < H; ++h) ss += x[h] * x[h];
  const float var = (float)(ss / (double)H);
  const float inv = 1.0f / sqrtf(var + (float)eps);
  for (int h = 0; h < H; ++h) {
    const float n = (float)x[h] * inv;
    const float p = n * (float)bf16_to_double(g[h]);
    y[h] = round_to_bf16((double)p);
  }
}

static uint16_t double_to_bf16_bits(double v) {
  /* v already holds a bf16 value: its float bits' upper half */
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

/*
 * The MoE block of a Gemma 4 decoder layer (walkthrough section 1, the
 * DecoderLayer forward; section 7 for the tensor flow), from the residual x
 * [T,H] bf16 that the attention half hands over:
 *   h1 = post_ff_norm_1( mlp( pre_ff_norm(x) ) )        dense GeGLU MLP
 *   h2 = post_ff_norm_2( moe( pre_ff_norm_2(x), router(x) ) )
 *   out = post_ff_norm( h1 + h2 ) + x                    unweighted sum
 * Every module returns bf16 (the activation dtype): the two norm outputs,
 * the MLP and MoE outputs (each computed in fp64 here, then rounded), h1,
 * h2, their sum (one fp32 add, rounded), and the last norm.  out receives
 * the final residual add in fp32, fl(z + x), before its bf16 rounding.
 * The MLP is the E = 1 case of the expert FFN (oracle_forward with one
 * expert and weight 1); the MoE is oracle_forward on the router's logits
 * (oracle_router_logits) with per_expert_scale.
 */
int oracle_gemma4_block(int64_t T, int H, int E, int k, int I, int act, int I_dense,
                        const uint16_t* x, const uint16_t* g_pre, const uint16_t* g_post1,
                        const uint16_t* g_pre2, const uint16_t* g_post2,
                        const uint16_t* g_post, double eps, const uint16_t* router_w,
                        const uint16_t* router_scale, double router_eps,
                        const uint16_t* w13, const uint16_t* w2, const float* scale,
                        const uint16_t* mlp_w13, const uint16_t* mlp_w2, int nthreads,
                        double* out) {
  if (T < 0 || H < 1 || I_dense < 1 || !(eps >= 0.0) || !x || !g_pre || !g_post1 ||
      !g_pre2 || !g_post2 || !g_post || !mlp_w13 || !mlp_w2 || !out)
    return EINVAL_ARG;
  const size_t TH = (size_t)T * (size_t)H;
  uint16_t* a1 = (uint16_t*)malloc(sizeof(uint16_t) * (TH + 1));
  uint16_t* a2 = (uint16_t*)malloc(sizeof(uint16_t) * (TH + 1));
  double* y1 = (double*)malloc(sizeof(double) * (TH + 1));
  double* y2 = (double*)malloc(sizeof(double) * (TH + 1));
  float* z1 = (float*)calloc((size_t)T + 1, sizeof(float));   /* the MLP's logits */
  float* lg = (float*)malloc(sizeof(float) * ((size_t)T * E + 1));
  double* row = (double*)malloc(sizeof(double) * (size_t)H);
  double* r1 = (double*)malloc(sizeof(double) * (size_t)H);
  double* r2 = (double*)malloc(sizeof(double) * (size_t)H);
  int rc = OK;
  if (!a1 || !a2 || !y1 || !y2 || !z1 || !lg || !row || !r1 || !r2) rc = ENOMEM_ARG;
  /* the two input norms */
  for (int64_t t = 0; t < T && rc == OK; ++t) {
    for (int h = 0; h < H; ++h) row[h] = bf16_to_double(x[t * H + h]);
    gamma_rms_norm_row(row, H, eps, g_pre, r1);
    gamma_rms_norm_row(row, H, eps, g_pre2, r2);
    for (int h = 0; h < H; ++h) {
      a1[t * H + h] = double_to_bf16_bits(r1[h]);
      a2[t * H + h] = double_to_bf16_bits(r2[h]);
    }
  }
  /* dense MLP: one expert, weight 1 */
  if (rc == OK)
    rc = oracle_forward(T, H, 1, 1, I_dense, act, 0, 0, a1, z1, NULL, mlp_w13, mlp_w2,
                        NULL, NULL, NULL, T, 0, nthreads, y1, NULL, NULL);
  /* router on the raw residual, MoE on the normalised one */
  if (rc == OK) rc = oracle_router_logits(T, H, E, router_eps, x, router_w, router_scale, lg);
  if (rc == OK)
    rc = oracle_forward(T, H, E, k, I, act, 0, 0, a2, lg, scale, w13, w2, NULL, NULL,
                        NULL, T, 0, nthreads, y2, NULL, NULL);
  for (int64_t t = 0; t < T && rc == OK; ++t) {
    double* o = out + t * H;
    for (int h = 0; h < H; ++h) row[h] = round_to_bf16(y1[t * H + h]);
    gamma_rms_norm_row(row, H, eps, g_post1, r1);                  /* h1 */
    for (int h = 0; h < H; ++h) row[h] = round_to_bf16(y2[t * H + h]);
    gamma_rms_norm_row(row, H, eps, g_post2, r2);                  /* h2 */
    for (int h = 0; h < H; ++h) row[h] = round_to_bf16((double)(float)(r1[h] + r2[h]));
    gamma_rms_norm_row(row, H, eps, g_post, r1);                   /* z */
    for (int h = 0; h < H; ++h)
      o[h] = (double)(float)(r1[h] + bf16_to_double(x[t * H + h]));  /* fl(z + x) */
  }
  free(a1); free(a2); free(y1); free(y2); free(z1); free(lg); free(row); free(r1); free(r2);
  return rc;
}

/* ------------------------------------------------------------ FP8 experts */

/*
 * FP8 expert weights.  The sglang PR on Gemma 4 (prhub.com.cn, PR #24696,
 * "FP8 per-expert MoE weight-loader fix") loads per-expert FP8 checkpoints
 * whose gate / up / down weights each come with a weight_scale, into
 * FusedMoE's w13_weight / w2_weight and their _scale parameters; the vLLM API
 * page (load_weights) names the same parameters.  The pages fix neither the
 * number format nor the granularity of the scales.  The reading taken here
 * (the checkpoint is an "FP8-Dynamic" one):
 *   - a weight is an e4m3 code (E4M3FN: 1 sign bit, 4 exponent bits with
 *     bias 7, 3 mantissa bits, no infinities, 0x7F / 0xFF are NaN, largest
 *     finite 448) times one fp32 scale per output row;
 *   - activations are quantised per row when the layer runs: with amax the
 *     largest |v| of the row, s = fl32(amax / 448) (an all-zero row gets
 *     s = 1), and code(v) = e4m3(fl32(v / s)), rounded to the nearest e4m3
 *     value (ties to the even code), saturating at +-448;
 *   - the layer on the dequantised values, in fp64: per routed (t, e),
 *       g_i = sum_h x'_h w1'_ih,  u_i = sum_h x'_h w3'_ih,  a_i = Act(g_i) u_i,
 *     x' the quantised token row (code times s_x), w' code times row scale;
 *     the intermediate is a bf16 tensor between the two products, as in the
 *     bf16 layer (FusedMoE's activation output in the activation dtype), so
 *     the row a is rounded to bf16 and that bf16 row quantised the same way
 *     as x; then y_h = sum_i a'_i w2'_hi, and the combine is the one of
 *     oracle_forward.  A code times an fp32 scale is exact in double.
 */

static double e4m3_table[256];
static pthread_once_t e4m3_once = PTHREAD_ONCE_INIT;

/* value of an e4m3 code: (8 + m) 2^(e-10) for e > 0, m 2^-9 for e = 0 */
static void e4m3_init(void) {
  for (int b = 0; b < 256; ++b) {
    const int e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7)
      v = NAN;
    else
      v = e == 0 ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
    e4m3_table[b] = (b & 0x80) ? -v : v;
  }
}

static double e4m3_value(uint8_t b) { return e4m3_table[b]; }

/* nearest e4m3 code of v (ties to the even code), saturating at 448 */
static uint8_t e4m3_code(float v) {
  if (v != v) return 0x7F;
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const double a = fabs((double)v);
  if (a >= 448.0) return sign | 0x7E;
  int lo = 0, hi = 126;  /* largest code whose value is <= a */
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (e4m3_table[mid] <= a) lo = mid; else hi = mid - 1;
  }
  const double below = e4m3_table[lo], above = e4m3_table[lo + 1];
  int c;
  if (a - below < above - a) c = lo;
  else if (a - below > above - a) c = lo + 1;
  else c = (lo & 1) ? lo + 1 : lo;
  return sign | (uint8_t)c;
}

int oracle_e4m3_values(int64_t n, const uint8_t* codes, double* out) {
  pthread_once(&e4m3_once, e4m3_init);
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
  return OK;
}

int oracle_e4m3_codes(int64_t n, const float* v, uint8_t* out) {
  pthread_once(&e4m3_once, e4m3_init);
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_code(v[i]);
  return OK;
}

/* per-row scale and codes of n values held as floats */
static float quantize_row(int n, const float* v, uint8_t* codes) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) {
    const float a = fabsf(v[i]);
    if (a > amax) amax = a;
  }
  const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
  for (int i = 0; i < n; ++i) codes[i] = e4m3_code(v[i] / s);
  return s;
}

/* per-row dynamic quantisation of bf16 rows: codes [rows, cols], scales [rows] */
int oracle_quantize_rows_e4m3(int64_t rows, int cols, const uint16_t* src,
                              uint8_t* codes, float* scales) {
  if (rows < 0 || cols < 1 || !src || !codes || !scales) return EINVAL_ARG;
  pthread_once(&e4m3_once, e4m3_init);
  float* v = (float*)malloc(sizeof(float) * (size_t)cols);
  if (!v) return ENOMEM_ARG;
  for (int64_t r = 0; r < rows; ++r) {
    for (int c = 0; c < cols; ++c) v[c] = (float)bf16_to_double(src[r * cols + c]);
    scales[r] = quantize_row(cols, v, codes + r * cols);
  }
  free(v);
  return OK;
}

/*
 * Validity slack of the FP8 layer.  Quantising the intermediate takes
 * integer decisions (its bf16 rounding, the row's amax and with it the
 * scale, each e4m3 code) from a row that an implementation computes in
 * fp32: a value within that arithmetic's error of a rounding boundary can
 * go either way, and both outcomes are the layer's result.  The decisions
 * taken here are those of the exact row; the slack of an output element is
 * the most the other admissible decisions can move it:
 *   - an fp32 implementation's g (and u) lies within
 *       dg = 2^-20 sum_h |x'_h w1'_ih| + 2^-22 |g|
 *     of the exact value (16 fp32 ulps of the sum of magnitudes for the
 *     accumulation, and the scale products), and its a = Act(g) u within
 *       da = dAct (|u| + du) + |Act(g)| du + 2^-21 |a|,
 *     dAct the largest change of Act over [g - dg, g + dg];
 *   - an element's admissible bf16 values are those of [a - da, a + da];
 *     the row's admissible amax values follow, and with them its scales;
 *   - under each admissible scale, d_i = the most an admissible bf16 value
 *     of element i moves its dequantised value, and the slack of y_h adds
 *     weight * (sum_i d_i |w2'_hi| + the largest |change of y_h| that
 *     another admissible scale makes with the exact row's bf16 values).
 */
typedef struct {
  double* g1;   /* sum of |terms| of g, then da */
  double* u1;   /* sum of |terms| of u */
  double* lo;   /* admissible bf16 values of each element */
  double* hi;
  double* d;    /* largest change of each dequantised element */
} fp8_slack_scratch;

static double act_spread(int act, double g, double dg) {
  const double f = act_fn(act, g);
  const double a = fabs(act_fn(act, g - dg) - f), b = fabs(act_fn(act, g + dg) - f);
  return a > b ? a : b;
}

/* the next bf16 value above v >= 0 (8 significant bits; 2^-133 after 0) */
static double bf16_next_up(double v) {
  if (v <= 0.0) return ldexp(1.0, -133);
  int ex;
  frexp(v, &ex);  /* v in [2^(ex-1), 2^ex) */
  const double ulp = ldexp(1.0, ex - 8 < -133 ? -133 : ex - 8);
  return v + ulp;
}

/* dequantised value of v (a bf16 value held as a float) with scale s */
static double deq(float v, float s) { return e4m3_value(e4m3_code(v / s)) * (double)s; }

static void fp8_row_slack(int H, int I, int act, const double* gv, const double* uv,
                          const double* a_exact, const float* af, float s,
                          const uint8_t* w2c, const float* w2s, double weight,
                          fp8_slack_scratch* sc, double* slack) {
  double amax_lo = 0.0, amax_hi = 0.0;
  for (int i = 0; i < I; ++i) {
    const double dg = ldexp(sc->g1[i], -20) + ldexp(fabs(gv[i]), -22);
    const double du = ldexp(sc->u1[i], -20) + ldexp(fabs(uv[i]), -22);
    const double fa = act_fn(act, gv[i]);
    const double da = act_spread(act, gv[i], dg) * (fabs(uv[i]) + du) + fabs(fa) * du +
                      ldexp(fabs(a_exact[i]), -21);
    const double b0 = round_to_bf16(a_exact[i] - da), b1 = round_to_bf16(a_exact[i] + da);
    sc->lo[i] = b0;
    sc->hi[i] = b1;
    /* |values| the element can take span [min |b|, max |b|] over [b0, b1] */
    const double mn = (b0 <= 0.0 && b1 >= 0.0) ? 0.0 : fmin(fabs(b0), fabs(b1));
    const double mx = fmax(fabs(b0), fabs(b1));
    if (mn > amax_lo) amax_lo = mn;
    if (mx > amax_hi) amax_hi = mx;
  }
  /* admissible scales: every bf16 amax in [amax_lo, amax_hi] (a few values
   * at most; the list is cut at 16) */
  float scales[16];
  int ns = 0;
  for (double m = amax_lo; m <= amax_hi && ns < 16; m = bf16_next_up(m)) {
    const float mf = (float)m;
    scales[ns++] = mf > 0.0f ? mf / 448.0f : 1.0f;
  }
  /* element decisions: for each admissible scale, the most an admissible
   * bf16 value of the element moves its dequantised value (monotone in the
   * bf16 value, so the ends of [lo, hi] bound it) */
  int any = 0;
  for (int i = 0; i < I; ++i) {
    sc->d[i] = 0.0;
    if (sc->lo[i] == sc->hi[i]) continue;
    for (int q = 0; q < ns; ++q) {
      const double mid = deq(af[i], scales[q]);
      const double c0 = fabs(deq((float)sc->lo[i], scales[q]) - mid);
      const double c1 = fabs(deq((float)sc->hi[i], scales[q]) - mid);
      if (c0 > sc->d[i]) sc->d[i] = c0;
      if (c1 > sc->d[i]) sc->d[i] = c1;
    }
    if (sc->d[i] > 0.0) any = 1;
  }
  /* scale decisions: the row's change under every other admissible scale,
   * computed exactly (every element moves with the scale) */
  double* dq = NULL;
  int nalt = 0;
  if (ns > 1) {
    dq = (double*)malloc(sizeof(double) * (size_t)ns * I);
    for (int q = 0; dq && q < ns; ++q) {
      if (scales[q] == s) continue;
      for (int i = 0; i < I; ++i) dq[(size_t)nalt * I + i] = deq(af[i], scales[q]) - deq(af[i], s);
      ++nalt;
    }
  }
  if (!any && nalt == 0) {
    free(dq);
    return;
  }
  for (int h = 0; h < H; ++h) {
    const uint8_t* r2 = w2c + (int64_t)h * I;
    double acc = 0.0, worst = 0.0;
    for (int i = 0; any && i < I; ++i)
      if (sc->d[i] > 0.0) acc += sc->d[i] * fabs(e4m3_value(r2[i]) * (double)w2s[h]);
    for (int q = 0; q < nalt; ++q) {
      double y = 0.0;
      for (int i = 0; i < I; ++i) y += dq[(size_t)q * I + i] * (e4m3_value(r2[i]) * (double)w2s[h]);
      if (fabs(y) > worst) worst = fabs(y);
    }
    slack[h] += fabs(weight) * (acc + worst);
  }
  free(dq);
}

/* one expert (or shared expert) on one quantised token row, added to y
 * with the given weight (and its validity slack to ``slack``, if given) */
static void ffn_row_fp8(int H, int I, int act, const double* xq, const uint8_t* w13c,
                        const float* w13s, const uint8_t* w2c, const float* w2s,
                        double weight, double* a, float* af, uint8_t* ac, double* y,
                        double* gv, double* uv, fp8_slack_scratch* sc, double* slack) {
  for (int i = 0; i < I; ++i) {
    const uint8_t* r1 = w13c + (int64_t)i * H;
    const uint8_t* r3 = w13c + (int64_t)(I + i) * H;
    double g = 0.0, u = 0.0, g1 = 0.0, u1 = 0.0;
    for (int h = 0; h < H; ++h) {
      const double tg = xq[h] * (e4m3_value(r1[h]) * (double)w13s[i]);
      const double tu = xq[h] * (e4m3_value(r3[h]) * (double)w13s[I + i]);
      g += tg;
      u += tu;
      if (slack) {
        g1 += fabs(tg);
        u1 += fabs(tu);
      }
    }
    a[i] = act_fn(act, g) * u;
    if (slack) {
      gv[i] = g;
      uv[i] = u;
      sc->g1[i] = g1;
      sc->u1[i] = u1;
    }
  }
  /* the intermediate row in bf16, quantised by the steps of quantize_row */
  for (int i = 0; i < I; ++i) af[i] = (float)round_to_bf16(a[i]);
  const float s = quantize_row(I, af, ac);
  if (slack) fp8_row_slack(H, I, act, gv, uv, a, af, s, w2c, w2s, weight, sc, slack);
  for (int i = 0; i < I; ++i) a[i] = e4m3_value(ac[i]) * (double)s;
  for (int h = 0; h < H; ++h) {
    const uint8_t* r2 = w2c + (int64_t)h * I;
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += a[i] * (e4m3_value(r2[i]) * (double)w2s[h]);
    y[h] += weight * acc;
  }
}

typedef struct {
  int64_t T;
  int H, E, k, I, act, S;
  const uint16_t* x;
  const uint8_t *w13c, *w2c, *sh13c, *sh2c;
  const float *w13s, *w2s, *sh13s, *sh2s;
  const int32_t* ids;
  const double* w;
  const int64_t* tokens;
  double* out;
  double* slack;
} fwd8_ctx;

static void fwd8_worker(void* p, int64_t b, int64_t e) {
  fwd8_ctx* c = (fwd8_ctx*)p;
  const int H = c->H, I = c->I;
  float* xf = (float*)malloc(sizeof(float) * H);
  uint8_t* xc = (uint8_t*)malloc(H);
  double* xq = (double*)malloc(sizeof(double) * H);
  double* a = (double*)malloc(sizeof(double) * I);
  float* af = (float*)malloc(sizeof(float) * I);
  uint8_t* ac = (uint8_t*)malloc(I);
  double* sbuf = (double*)malloc(sizeof(double) * 7 * I);  /* g, u and the slack scratch */
  fp8_slack_scratch sc = {sbuf + 2 * I, sbuf + 3 * I, sbuf + 4 * I, sbuf + 5 * I,
                          sbuf + 6 * I};
  for (int64_t r = b; r < e; ++r) {
    const int64_t t = c->tokens ? c->tokens[r] : r;
    double* y = c->out + r * H;
    double* sl = c->slack ? c->slack + r * H : NULL;
    for (int h = 0; h < H; ++h) y[h] = 0.0;
    for (int h = 0; sl && h < H; ++h) sl[h] = 0.0;
    /* the token row, quantised once */
    for (int h = 0; h < H; ++h) xf[h] = (float)bf16_to_double(c->x[t * H + h]);
    const float sx = quantize_row(H, xf, xc);
    for (int h = 0; h < H; ++h) xq[h] = e4m3_value(xc[h]) * (double)sx;
    for (int j = 0; j < c->k; ++j) {
      const int64_t ex = c->ids[t * c->k + j];
      ffn_row_fp8(H, I, c->act, xq, c->w13c + ex * 2 * (int64_t)I * H,
                  c->w13s + ex * 2 * (int64_t)I, c->w2c + ex * (int64_t)H * I,
                  c->w2s + ex * (int64_t)H, c->w[t * c->k + j], a, af, ac, y, sbuf,
                  sbuf + I, &sc, sl);
    }
    for (int s = 0; s < c->S; ++s)
      ffn_row_fp8(H, I, c->act, xq, c->sh13c + (int64_t)s * 2 * I * H,
                  c->sh13s + (int64_t)s * 2 * I, c->sh2c + (int64_t)s * H * I,
                  c->sh2s + (int64_t)s * H, 1.0, a, af, ac, y, sbuf, sbuf + I, &sc, sl);
  }
  free(xf); free(xc); free(xq); free(a); free(af); free(ac); free(sbuf);
}

/*
 * The layer with FP8 experts, for the tokens listed in ``tokens`` (NULL =
 * all T): routing as oracle_forward; w13 codes [E,2I,H] with scales [E,2I]
 * (gate rows first), w2 codes [E,H,I] with scales [E,H]; shared experts
 * likewise ([S,...], the same I).  ``slack`` (NULL: not computed) receives
 * the validity slack of every output element (see fp8_row_slack).
 */
int oracle_forward_fp8(int64_t T, int H, int E, int k, int I, int act, int S,
                       const uint16_t* x, const float* logits, const float* scale,
                       const uint8_t* w13c, const float* w13s, const uint8_t* w2c,
                       const float* w2s, const uint8_t* sh13c, const float* sh13s,
                       const uint8_t* sh2c, const float* sh2s, const int64_t* tokens,
                       int64_t n_tokens, int nthreads, double* out, int32_t* ids_out,
                       double* w_out, double* slack) {
  if (T < 0 || H < 1 || I < 1 || S < 0 || !x || !w13c || !w13s || !w2c || !w2s ||
      (S > 0 && (!sh13c || !sh13s || !sh2c || !sh2s)))
    return EINVAL_ARG;
  pthread_once(&e4m3_once, e4m3_init);
  int32_t* ids = ids_out ? ids_out : (int32_t*)malloc(sizeof(int32_t) * (T * k + 1));
  double* w = w_out ? w_out : (double*)malloc(sizeof(double) * (T * k + 1));
  if (!ids || !w) return ENOMEM_ARG;
  int rc = oracle_route(T, E, k, logits, scale, ids, w, NULL);
  if (rc == OK) {
    if (!tokens) n_tokens = T;
    for (int64_t r = 0; tokens && r < n_tokens; ++r)
      if (tokens[r] < 0 || tokens[r] >= T) rc = EINVAL_ARG;
  }
  if (rc == OK) {
    fwd8_ctx c = {T, H, E, k, I, act, S, x, w13c, w2c, sh13c, sh2c,
                  w13s, w2s, sh13s, sh2s, ids, w, tokens, out, slack};
    parallel_for(n_tokens, nthreads, fwd8_worker, &c);
  }
  if (!ids_out) free(ids);
  if (!w_out) free(w);
  return rc;
}
