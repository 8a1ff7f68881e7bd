// decode.cu -- the layer for small token counts, where it is bound by HBM:
// every touched expert's weights must be streamed once, and each weight is
// used by only a few tokens.  llama-cpp-visual-guide lesson 35 (cost
// section) notes that decode moves the bottleneck from compute to moving
// data; the design below streams only the touched experts' weights.
//
// Four kernels on one stream, the last three launched as programmatic
// dependents (PDL) so each one's launch overlaps the previous one's tail:
//   decode_route  one block: routes all T tokens (route_impl.cuh), counts
//                 tokens per expert, lists the touched experts in ascending
//                 id (shared experts last) and, per expert, its slots;
//   decode_w13    one CTA per (touched expert, 16 rows of I): h = Act(x W1^T)
//                 (*) (x W3^T) for the expert's tokens, rounded to bf16;
//   decode_w2     one CTA per (touched expert, 64 rows of H): y = h W2^T,
//                 times the gate weight, stored at the (token, choice) row;
//   sum_rows      (combine.cu) adds each token's k+S rows in order, bf16 out.
// For 8 < T <= 64 the two products run as tcgen05 kernels instead
// (decode_tc.cu); the routing and the row sum stay the same.
//
// The skinny products use mma.sync m16n8k16 (bf16 in, fp32 accumulate) with
// weight rows as the 16-row A operand and up to 8 tokens per B tile.  The K
// order inside each 32-column chunk is permuted so that every thread loads
// its A and B elements as one 16-byte vector: thread (g, c) of the warp reads
// columns [8c, 8c+8) of rows g and g+8, and the same columns of its tokens;
// MMA step s takes the words 2s and 2s+1 of those vectors.  A dot product is
// indifferent to the order of its terms as long as A and B share it.  In
// decode_w13 the 4 warps of a CTA split K (H is long) and add their partial
// sums through shared memory; in decode_w2 each warp owns 16 rows and all of
// K (I is short).
//
// With at most 8 tokens (one B tile) the kernels take their "few" form: the
// weights stream through a per-warp ring of shared-memory slots filled with
// 16-byte cp.async copies several chunks ahead, so a lane keeps 5-7 chunks
// in flight without holding them in registers (the register-prefetch form
// holds one or two and is bound by DRAM latency at this size).  Each lane
// reads back only the bytes it copied itself, so the ring needs no barrier.
// In decode_w13_few the four warps take K chunks round-robin, so a CTA reads
// 256 contiguous bytes of each weight row at a time; decode_w2_few starts its
// ring before it waits for h.
#include <algorithm>

#include "route_impl.cuh"

namespace moe {
namespace {

constexpr int kDecThreads = 128;
constexpr int kDecRows = 16;
constexpr int kDecNT = 8;  // token tiles of 8 per pass (64 tokens) for T > 8

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Asks L2 to fetch [p, p + bytes) (16-byte aligned, multiple of 16 bytes).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes)
               : "memory");
}

// L2 policy for weights that are read once: evict them first, so that what
// is read again (the w2 rows asked for early, the token rows) stays.
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte global -> shared copy that skips L1; when !valid nothing is read
// and the 16 bytes are zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid,
                                           uint64_t pol) {
  asm volatile(
      "cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst),
      "l"(src), "r"(valid ? 16 : 0), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d += A(rows g, g+8; 32 permuted columns) x B(token; same columns)
__device__ __forceinline__ void mma_chunk(float (&d)[4], const uint4& ar0,
                                          const uint4& ar8, const uint4& b) {
  mma16816(d, ar0.x, ar8.x, ar0.y, ar8.y, b.x, b.y);
  mma16816(d, ar0.z, ar8.z, ar0.w, ar8.w, b.z, b.w);
}

__device__ __forceinline__ float dec_act(int act, float g) {
  if (act == MOE_ACT_SILU) return g / (1.0f + expf(-g));
  const float c = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * g * (1.0f + tanhf(c * fmaf(0.044715f * g, g * g, g)));
}

// meta layout (int32): [0] n touched groups; [1 + i] group id of the i-th
// touched group; [1 + G + i] first slot-list entry of group i (i <= n).
//
// One block of 32 * ceil(G / 32) threads (at least one warp per token up to
// 32 warps): thread g owns group g.  One block-wide scan of the packed pair
// (touched ? 1 : 0) << 16 | tokens of g gives both the touched index and
// the first slot-list entry of every group (both sums stay below 2^16:
// G <= 520 groups, T (k + S) <= 1024 * 40 slots).  PER logits per lane
// (route_impl.cuh).
template <int PER>
__global__ void __launch_bounds__(1024)
decode_route_kernel(const float* __restrict__ logits, const float* __restrict__ scale,
                    int T, int E, int k, int S, int32_t* __restrict__ ids,
                    float* __restrict__ w, int32_t* __restrict__ meta,
                    int32_t* __restrict__ slots, RouteOpt opt,
                    int32_t* __restrict__ zero, int n_zero) {
  extern __shared__ int32_t dsm[];
  const int G = E + S, R = T * k;
  int32_t* cnt = dsm;            // [G] tokens, then first slot-list entry
  int32_t* ids_s = cnt + G;      // [R]
  __shared__ uint32_t warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  pdl_trigger();
  // the arrival counters of the tensor-core products start at zero
  for (int i = tid; i < n_zero; i += blockDim.x) zero[i] = 0;
  for (int i = tid; i < G; i += blockDim.x) cnt[i] = (i < E) ? 0 : T;
  __syncthreads();
  for (int t = warp; t < T; t += nwarps) {
    int id;
    float wt;
    route_token_warp<PER>(logits + (int64_t)t * E, scale, E, k, &id, &wt, opt);
    if (lane < k) {
      ids[t * k + lane] = id;
      w[t * k + lane] = wt;
      ids_s[t * k + lane] = id;
    }
  }
  __syncthreads();
  for (int s = tid; s < R; s += blockDim.x) atomicAdd(&cnt[ids_s[s]], 1);
  __syncthreads();
  const int c = (tid < G) ? cnt[tid] : 0;
  const uint32_t v = (c > 0 ? 1u << 16 : 0u) | (uint32_t)c;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t ws = lane < nwarps ? warp_sums[lane] : 0u;
    uint32_t wi = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += o;
    }
    warp_sums[lane] = wi - ws;  // exclusive prefix of the warps before
    if (lane == 31) {
      meta[0] = (int32_t)(wi >> 16);                 // touched groups
      meta[1 + G + (wi >> 16)] = (int32_t)(wi & 0xffffu);  // total slots
    }
  }
  __syncthreads();
  const uint32_t excl = incl - v + warp_sums[warp];
  if (tid < G) {
    const int base = (int)(excl & 0xffffu), idx = (int)(excl >> 16);
    cnt[tid] = base;
    if (c > 0) {
      meta[1 + idx] = tid;
      meta[1 + G + idx] = base;
    }
  }
  __syncthreads();
  // slot lists: routed slots by atomic position (the order inside an expert's
  // list only decides which MMA column a token uses, not its result)
  for (int s = tid; s < R; s += blockDim.x) {
    const int p = atomicAdd(&cnt[ids_s[s]], 1);
    slots[p] = s;
  }
  for (int q = tid; q < T * S; q += blockDim.x) {
    const int sh = q / T, t = q - sh * T;
    slots[cnt[E + sh] + t] = R + q;
  }
}

struct DecGroup {
  int g, base, n;
};

__device__ __forceinline__ bool load_group(const int32_t* meta, int G, int idx,
                                           DecGroup* out) {
  const int n_groups = meta[0];
  if (idx >= n_groups) return false;
  out->g = meta[1 + idx];
  out->base = meta[1 + G + idx];
  out->n = meta[1 + G + idx + 1] - out->base;
  return true;
}

// The many-token form (T > 8): NTMAX token tiles kept in registers per pass
// (up to 64 tokens of a group at once), weights loaded one 32-column chunk
// ahead into registers.
__global__ void __launch_bounds__(kDecThreads, 4)
decode_w13_kernel(const __nv_bfloat16* __restrict__ x,
                  const __nv_bfloat16* __restrict__ w13,
                  const __nv_bfloat16* __restrict__ w13_sh,
                  const int32_t* __restrict__ meta, const int32_t* __restrict__ slots,
                  int T, int H, int I, int E, int k, int S, int act,
                  __nv_bfloat16* __restrict__ h_dec) {
  constexpr int NTMAX = kDecNT;
  constexpr int PASS = NTMAX * 8;
  __shared__ int32_t tok_s[PASS];
  __shared__ int32_t slot_s[PASS];
  __shared__ float red[4][NTMAX][32][8];
  pdl_wait();  // routing (meta, slots) comes from decode_route
  pdl_trigger();
  DecGroup grp;
  if (!load_group(meta, E + S, blockIdx.x, &grp)) return;
  const int R = T * k;
  const __nv_bfloat16* W = grp.g < E ? w13 + (int64_t)grp.g * 2 * I * H
                                     : w13_sh + (int64_t)(grp.g - E) * 2 * I * H;
  const int i0 = blockIdx.y * kDecRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, c = lane & 3;
  const int nch = (H + 31) / 32;
  const int ch0 = warp * nch / 4, ch1 = (warp + 1) * nch / 4;
  const int ra = i0 + gq, rb = i0 + gq + 8;  // gate rows; up rows are +I
  const bool va = ra < I, vb = rb < I;
  const __nv_bfloat16* pga = W + (int64_t)ra * H;
  const __nv_bfloat16* pgb = W + (int64_t)rb * H;
  const __nv_bfloat16* pua = W + (int64_t)(I + ra) * H;
  const __nv_bfloat16* pub = W + (int64_t)(I + rb) * H;
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  struct W4 {
    uint4 ga, gb, ua, ub;
  };
  auto load_w = [&](int ch) -> W4 {
    const int col = ch * 32 + 8 * c;
    const bool vc = ch < ch1 && col < H;
    W4 r;
    r.ga = (va && vc) ? ld_stream(pga + col) : z4;
    r.gb = (vb && vc) ? ld_stream(pgb + col) : z4;
    r.ua = (va && vc) ? ld_stream(pua + col) : z4;
    r.ub = (vb && vc) ? ld_stream(pub + col) : z4;
    return r;
  };

  for (int p0 = 0; p0 < grp.n; p0 += PASS) {
    const int np = min(PASS, grp.n - p0);
    const int NT = (np + 7) >> 3;
    __syncthreads();
    // the next chunk's weights are requested before a chunk is multiplied
    // (the first ones before the token rows are even looked up)
    W4 q0 = load_w(ch0);
    for (int i = threadIdx.x; i < np; i += kDecThreads) {
      const int s = slots[grp.base + p0 + i];
      slot_s[i] = s;
      tok_s[i] = s < R ? s / k : (s - R) % T;
    }
    __syncthreads();
    float ag[NTMAX][4], au[NTMAX][4];
#pragma unroll
    for (int nt = 0; nt < NTMAX; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) ag[nt][e] = au[nt][e] = 0.f;
    for (int ch = ch0; ch < ch1; ++ch) {
      const int col = ch * 32 + 8 * c;
      const bool vc = col < H;
      const W4 cur = q0;
      q0 = load_w(ch + 1);
#pragma unroll
      for (int nt = 0; nt < NTMAX; ++nt) {
        if (nt < NT) {
          const int tk = nt * 8 + gq;
          const uint4 xv =
              (tk < np && vc)
                  ? __ldg(reinterpret_cast<const uint4*>(x + (int64_t)tok_s[tk] * H + col))
                  : z4;
          mma_chunk(ag[nt], cur.ga, cur.gb, xv);
          mma_chunk(au[nt], cur.ua, cur.ub, xv);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NTMAX; ++nt) {
      if (nt < NT) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          red[warp][nt][lane][e] = ag[nt][e];
          red[warp][nt][lane][4 + e] = au[nt][e];
        }
      }
    }
    __syncthreads();
    for (int nt = warp; nt < NT; nt += 4) {
      float g4[4], u4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        g4[e] = red[0][nt][lane][e] + red[1][nt][lane][e] + red[2][nt][lane][e] +
                red[3][nt][lane][e];
        u4[e] = red[0][nt][lane][4 + e] + red[1][nt][lane][4 + e] +
                red[2][nt][lane][4 + e] + red[3][nt][lane][4 + e];
      }
      // fragment element e: row gq (+8 for e >= 2), token 2c + (e & 1)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = i0 + gq + (e >= 2 ? 8 : 0);
        const int tk = nt * 8 + 2 * c + (e & 1);
        if (row < I && tk < np)
          h_dec[(int64_t)slot_s[tk] * I + row] =
              __float2bfloat16_rn(dec_act(act, g4[e]) * u4[e]);
      }
    }
  }
}

// One CTA per (touched expert, 64 rows of H); each warp owns 16 rows and the
// whole of K = I, so no cross-warp reduction is needed.  The weight loads run
// two 32-column chunks ahead of the MMAs.
constexpr int kW2Rows = 64;

__global__ void __launch_bounds__(kDecThreads, 4)
decode_w2_kernel(const __nv_bfloat16* __restrict__ h_dec,
                 const __nv_bfloat16* __restrict__ w2,
                 const __nv_bfloat16* __restrict__ w2_sh,
                 const int32_t* __restrict__ meta, const int32_t* __restrict__ slots,
                 const float* __restrict__ wgt, int T, int H, int I, int E, int k,
                 int S, float* __restrict__ stage) {
  constexpr int NTMAX = kDecNT;
  constexpr int PASS = NTMAX * 8;
  __shared__ int32_t slot_s[PASS];
  // This kernel is launched once every decode_w13 block has passed its own
  // wait for the routing, so the expert lists are final here: the weight rows
  // of this block are pulled into L2 while decode_w13 still streams its own.
  DecGroup grp;
  const bool live = load_group(meta, E + S, blockIdx.x, &grp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16* W = nullptr;
  if (live) {
    W = grp.g < E ? w2 + (int64_t)grp.g * H * I : w2_sh + (int64_t)(grp.g - E) * H * I;
    const int rows = min(kDecRows, H - (int)(blockIdx.y * kW2Rows + warp * kDecRows));
    if (lane == 0 && rows > 0)
      prefetch_l2_bulk(W + (int64_t)(blockIdx.y * kW2Rows + warp * kDecRows) * I,
                       (uint32_t)rows * I * 2);
  }
  pdl_wait();  // h_dec comes from decode_w13
  pdl_trigger();
  if (!live) return;
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  const int R = T * k, ks = k + S;
  const int gq = lane >> 2, c = lane & 3;
  const int r0 = blockIdx.y * kW2Rows + warp * kDecRows;
  const int nch = (I + 31) / 32;
  const int ra = r0 + gq, rb = r0 + gq + 8;
  const bool va = ra < H, vb = rb < H;
  const __nv_bfloat16* pa = W + (int64_t)ra * I;
  const __nv_bfloat16* pb = W + (int64_t)rb * I;
  auto load_w = [&](int ch, uint4& a, uint4& b) {
    const int col = ch * 32 + 8 * c;
    const bool vc = ch < nch && col < I;
    a = (va && vc) ? ld_stream(pa + col) : z4;
    b = (vb && vc) ? ld_stream(pb + col) : z4;
  };

  for (int p0 = 0; p0 < grp.n; p0 += PASS) {
    const int np = min(PASS, grp.n - p0);
    const int NT = (np + 7) >> 3;
    __syncthreads();
    for (int i = threadIdx.x; i < np; i += kDecThreads)
      slot_s[i] = slots[grp.base + p0 + i];
    __syncthreads();
    float acc[NTMAX][4];
#pragma unroll
    for (int nt = 0; nt < NTMAX; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    uint4 qa0, qb0, qa1, qb1;  // chunks ch and ch+1 in flight
    load_w(0, qa0, qb0);
    load_w(1, qa1, qb1);
    for (int ch = 0; ch < nch; ++ch) {
      const int col = ch * 32 + 8 * c;
      const bool vc = col < I;
      const uint4 wa = qa0, wb = qb0;
      qa0 = qa1;
      qb0 = qb1;
      load_w(ch + 2, qa1, qb1);
#pragma unroll
      for (int nt = 0; nt < NTMAX; ++nt) {
        if (nt < NT) {
          const int tk = nt * 8 + gq;
          const uint4 hv =
              (tk < np && vc)
                  ? __ldg(reinterpret_cast<const uint4*>(h_dec + (int64_t)slot_s[tk] * I + col))
                  : z4;
          mma_chunk(acc[nt], wa, wb, hv);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NTMAX; ++nt) {
      if (nt < NT) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = r0 + gq + (e >= 2 ? 8 : 0);
          const int tk = nt * 8 + 2 * c + (e & 1);
          if (row < H && tk < np) {
            const int s = slot_s[tk];
            int64_t dst;
            float wt;
            if (s < R) {
              const int t = s / k;
              dst = (int64_t)t * ks + (s - t * k);
              wt = __ldg(wgt + s);
            } else {
              const int q = s - R, sh = q / T;
              dst = (int64_t)(q - sh * T) * ks + k + sh;
              wt = 1.0f;
            }
            stage[dst * H + row] = __fmul_rn(wt, acc[nt][e]);
          }
        }
      }
    }
  }
}


// ---- the few-token form (T <= 8: one B tile, one pass per group) ----

// ring slots per warp (D - 1 chunks in flight) and the shared memory of each
// kernel: the rings, then the token rows (min(T, 8) rows of x or of h)
constexpr int kW13Ring = 6;
constexpr int kW2Ring = 8;
__host__ __device__ constexpr size_t w13_ring_bytes() { return 4u * kW13Ring * 4 * 512; }
__host__ __device__ constexpr size_t w2_ring_bytes() { return 4u * kW2Ring * 2 * 512; }

// One CTA per (touched group, 16 rows of I), as decode_w13_kernel, with the
// gate and up rows streamed through the warp's ring: slot j holds the four
// 16-byte pieces (gate rows g, g+8; up rows g, g+8) of a lane at
// [(j * 4 + part) * 32 + lane], so a warp's reads of one part are
// contiguous.
template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_w13_few_kernel(const __nv_bfloat16* __restrict__ x,
                      const __nv_bfloat16* __restrict__ w13,
                      const __nv_bfloat16* __restrict__ w13_sh,
                      const int32_t* __restrict__ meta, const int32_t* __restrict__ slots,
                      int T, int H, int I, int E, int k, int S, int act,
                      __nv_bfloat16* __restrict__ h_dec) {
  __shared__ int32_t tok_s[8];
  __shared__ int32_t slot_s[8];
  __shared__ float red[4][32][8];
  extern __shared__ __align__(16) uint4 dyn[];
  pdl_wait();  // routing (meta, slots) comes from decode_route
  pdl_trigger();
  DecGroup grp;
  if (!load_group(meta, E + S, blockIdx.x, &grp)) return;
  const int R = T * k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16* W = grp.g < E ? w13 + (int64_t)grp.g * 2 * I * H
                                     : w13_sh + (int64_t)(grp.g - E) * 2 * I * H;
  const int i0 = blockIdx.y * kDecRows;
  const int gq = lane >> 2, c = lane & 3;
  // warp w takes the 32-column chunks w, w + 4, ...: the four warps read
  // 256 contiguous bytes of each weight row at a time
  const int nch = (H + 31) / 32;
  const int ra = i0 + gq, rb = i0 + gq + 8;  // gate rows; up rows are +I
  const bool va = ra < I, vb = rb < I;
  // rows past I are zero-filled from a valid address (nothing is read)
  const __nv_bfloat16* pga = W + (int64_t)(va ? ra : 0) * H;
  const __nv_bfloat16* pgb = W + (int64_t)(vb ? rb : 0) * H;
  const __nv_bfloat16* pua = W + (int64_t)(I + (va ? ra : 0)) * H;
  const __nv_bfloat16* pub = W + (int64_t)(I + (vb ? rb : 0)) * H;
  const uint64_t pol = evict_first_policy();
  uint4* ring = dyn + warp * (D * 4 * 32);
  const uint32_t ring_s = smem_u32(ring + lane);
  auto issue = [&](int i, int slot) {  // the warp's i-th chunk
    const int ch = warp + 4 * i;
    if (ch < nch) {
      const int col = ch * 32 + 8 * c;
      const bool vc = col < H;
      const int cc = vc ? col : 0;
      const uint32_t d = ring_s + (uint32_t)slot * 4 * 512;
      cp_async16(d, pga + cc, va && vc, pol);
      cp_async16(d + 512, pgb + cc, vb && vc, pol);
      cp_async16(d + 1024, pua + cc, va && vc, pol);
      cp_async16(d + 1536, pub + cc, vb && vc, pol);
    }
    cp_async_commit();  // empty groups past the end keep the count uniform
  };
#pragma unroll
  for (int j = 0; j < D - 1; ++j) issue(j, j);

  const int np = grp.n;  // <= T <= 8
  if (threadIdx.x < np) {
    const int s = slots[grp.base + threadIdx.x];
    slot_s[threadIdx.x] = s;
    tok_s[threadIdx.x] = s < R ? s / k : (s - R) % T;
  }
  __syncthreads();
  const int hv = H >> 3;
  uint4* xs = dyn + 4 * (D * 4 * 32);  // [np][H/8]
  for (int i = threadIdx.x; i < np * hv; i += kDecThreads) {
    const int tk = i / hv, cc = i - tk * hv;
    xs[i] = __ldg(reinterpret_cast<const uint4*>(x) + (int64_t)tok_s[tk] * hv + cc);
  }
  __syncthreads();

  const uint4 z4 = make_uint4(0, 0, 0, 0);
  float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
  int slot = 0;
  for (int i = 0, ch = warp; ch < nch; ++i, ch += 4) {
    cp_async_wait<D - 2>();  // chunk ch has landed (this lane's pieces)
    // refill the slot read in the previous iteration, whose values the MMAs
    // there have already consumed
    issue(i + D - 1, slot == 0 ? D - 1 : slot - 1);
    const uint4* q = ring + slot * 4 * 32;
    const uint4 ga = q[lane], gb = q[32 + lane], ua = q[64 + lane], ub = q[96 + lane];
    const int col = ch * 32 + 8 * c;
    const uint4 xv = (gq < np && col < H) ? xs[gq * hv + (col >> 3)] : z4;
    mma_chunk(ag, ga, gb, xv);
    mma_chunk(au, ua, ub, xv);
    slot = slot == D - 1 ? 0 : slot + 1;
  }
  cp_async_wait<0>();
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    red[warp][lane][e] = ag[e];
    red[warp][lane][4 + e] = au[e];
  }
  __syncthreads();
  if (warp == 0) {
    // fragment element e: row gq (+8 for e >= 2), token 2c + (e & 1)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float g = red[0][lane][e] + red[1][lane][e] + red[2][lane][e] + red[3][lane][e];
      const float u = red[0][lane][4 + e] + red[1][lane][4 + e] + red[2][lane][4 + e] +
                      red[3][lane][4 + e];
      const int row = i0 + gq + (e >= 2 ? 8 : 0);
      const int tk = 2 * c + (e & 1);
      if (row < I && tk < np)
        h_dec[(int64_t)slot_s[tk] * I + row] = __float2bfloat16_rn(dec_act(act, g) * u);
    }
  }
}

// One CTA per (touched group, 64 rows of H), as decode_w2_kernel, with the
// w2 rows streamed through the warp's ring (slot j: [(j * 2 + part) * 32 +
// lane], parts = rows g and g+8).  The weights do not depend on the previous
// kernel, so the ring is started before the wait for h.
template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_w2_few_kernel(const __nv_bfloat16* __restrict__ h_dec,
                     const __nv_bfloat16* __restrict__ w2,
                     const __nv_bfloat16* __restrict__ w2_sh,
                     const int32_t* __restrict__ meta, const int32_t* __restrict__ slots,
                     const float* __restrict__ wgt, int T, int H, int I, int E, int k,
                     int S, float* __restrict__ stage) {
  __shared__ int32_t slot_s[8];
  extern __shared__ __align__(16) uint4 dyn[];
  // Launched once every decode_w13 block has passed its own wait for the
  // routing, so the group lists are final here.
  DecGroup grp;
  const bool live = load_group(meta, E + S, blockIdx.x, &grp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, c = lane & 3;
  const int r0 = blockIdx.y * kW2Rows + warp * kDecRows;
  const int nch = (I + 31) / 32;
  const int ra = r0 + gq, rb = r0 + gq + 8;
  const bool va = ra < H, vb = rb < H;
  const __nv_bfloat16* W = nullptr;
  const __nv_bfloat16 *pa = nullptr, *pb = nullptr;
  uint4* ring = dyn + warp * (D * 2 * 32);
  const uint32_t ring_s = smem_u32(ring + lane);
  const uint64_t pol = evict_first_policy();
  auto issue = [&](int ch, int slot) {
    if (ch < nch) {
      const int col = ch * 32 + 8 * c;
      const bool vc = col < I;
      const int cc = vc ? col : 0;
      const uint32_t d = ring_s + (uint32_t)slot * 2 * 512;
      cp_async16(d, pa + cc, va && vc, pol);
      cp_async16(d + 512, pb + cc, vb && vc, pol);
    }
    cp_async_commit();
  };
  if (live) {
    W = grp.g < E ? w2 + (int64_t)grp.g * H * I : w2_sh + (int64_t)(grp.g - E) * H * I;
    pa = W + (int64_t)(va ? ra : 0) * I;
    pb = W + (int64_t)(vb ? rb : 0) * I;
#pragma unroll
    for (int j = 0; j < D - 1; ++j) issue(j, j);
  }
  pdl_wait();  // h_dec comes from decode_w13
  pdl_trigger();
  if (!live) return;
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  const int R = T * k, ks = k + S;
  const int np = grp.n;  // <= T <= 8
  if (threadIdx.x < np) slot_s[threadIdx.x] = slots[grp.base + threadIdx.x];
  __syncthreads();
  const int iv = I >> 3;
  uint4* hs = dyn + 4 * (D * 2 * 32);  // [np][I/8]
  for (int i = threadIdx.x; i < np * iv; i += kDecThreads) {
    const int tk = i / iv, cc = i - tk * iv;
    hs[i] = __ldg(reinterpret_cast<const uint4*>(h_dec) + (int64_t)slot_s[tk] * iv + cc);
  }
  __syncthreads();
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int slot = 0;
  for (int ch = 0; ch < nch; ++ch) {
    cp_async_wait<D - 2>();
    issue(ch + D - 1, slot == 0 ? D - 1 : slot - 1);
    const uint4* q = ring + slot * 2 * 32;
    const uint4 wa = q[lane], wb = q[32 + lane];
    const int col = ch * 32 + 8 * c;
    const uint4 hv = (gq < np && col < I) ? hs[gq * iv + (col >> 3)] : z4;
    mma_chunk(acc, wa, wb, hv);
    slot = slot == D - 1 ? 0 : slot + 1;
  }
  cp_async_wait<0>();
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int row = r0 + gq + (e >= 2 ? 8 : 0);
    const int tk = 2 * c + (e & 1);
    if (row < H && tk < np) {
      const int s = slot_s[tk];
      int64_t dst;
      float wt;
      if (s < R) {
        const int t = s / k;
        dst = (int64_t)t * ks + (s - t * k);
        wt = __ldg(wgt + s);
      } else {
        const int q = s - R, sh = q / T;
        dst = (int64_t)(q - sh * T) * ks + k + sh;
        wt = 1.0f;
      }
      stage[dst * H + row] = __fmul_rn(wt, acc[e]);
    }
  }
}

}  // namespace

size_t decode_meta_ints(int G) { return 2 + 2 * (size_t)G; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st, void* const* ev) {
  auto mark = [&](int i) -> bool { return !ev || !ev[i] || record_stage_event(ev[i], st); };
  const int G = a.E + a.S, R = a.T * a.k;
  if (!mark(0)) return cudaErrorUnknown;

  const size_t smem = sizeof(int32_t) * ((size_t)G + R);
  const int rthreads = 32 * std::min(32, std::max((G + 31) / 32, std::min(a.T, 32)));
  auto rk = a.E <= 32 ? decode_route_kernel<1> : a.E <= 64 ? decode_route_kernel<2>
            : a.E <= 128 ? decode_route_kernel<4> : a.E <= 256 ? decode_route_kernel<8>
            : decode_route_kernel<16>;
  // the tensor-core form counts its (unit, k-block) iterations in 32 bits
  const int64_t dt_iters = (int64_t)(std::min(R, a.E) + a.S) *
                           dt_row_blocks(a.H, a.I) * ((std::max(a.H, a.I) + 63) / 64);
  const bool tc = a.tc && dt_iters < (int64_t(1) << 30);
  const int n_zero = tc ? 2 * G * dt_row_blocks(a.H, a.I) : 0;
  cudaError_t e = launch_ex(rk, dim3(1), dim3(rthreads), smem, st, false, a.logits, a.scale,
                            a.T, a.E, a.k, a.S, a.ids, a.w, a.meta, a.slots, a.route,
                            tc ? a.dt_cnt : (int32_t*)nullptr, n_zero);
  if (e != cudaSuccess) return e;
  if (a.f8) {
    // FP8 experts, on the tensor-core form only: the codes of x, w13 (+ act)
    // -> h, the codes of each (group, token column) row of h, w2 -> stage
    if (!tc) return cudaErrorInvalidValue;
    if (!mark(1) || !mark(2)) return cudaErrorUnknown;
    if ((e = launch_quantize_rows(a.x, a.T, a.H, a.xq, a.sx, nullptr, nullptr, st,
                                  /*pdl=*/true)) != cudaSuccess)
      return e;
    if (!mark(3)) return cudaErrorUnknown;
    if ((e = launch_decode_tc_w13(a, a.h_dec, st)) != cudaSuccess) return e;
    const int64_t h_rows = (int64_t)(std::min(R, a.E) + a.S) * dt_columns(a.T);
    if ((e = launch_quantize_rows(a.h_dec, h_rows, a.I, a.hq, a.sh, nullptr, nullptr, st,
                                  /*pdl=*/true)) != cudaSuccess)
      return e;
    if (!mark(4)) return cudaErrorUnknown;
    if ((e = launch_decode_tc_w2(a, a.h_dec, st)) != cudaSuccess) return e;
    if (!mark(5)) return cudaErrorUnknown;
    e = launch_sum_rows(a.stage, a.T, a.k + a.S, a.H, a.out, a.out_f32, st,
                        /*pdl=*/true);
    if (e != cudaSuccess) return e;
    return mark(6) ? cudaSuccess : cudaErrorUnknown;
  }
  if (!mark(1) || !mark(2) || !mark(3)) return cudaErrorUnknown;
  if (tc) {
    // tensor-core products (decode_tc.cu): h in [touched, N, I] order
    if ((e = launch_decode_tc_w13(a, a.h_dec, st)) != cudaSuccess) return e;
    if (!mark(4)) return cudaErrorUnknown;
    if ((e = launch_decode_tc_w2(a, a.h_dec, st)) != cudaSuccess) return e;
    if (!mark(5)) return cudaErrorUnknown;
    e = launch_sum_rows(a.stage, a.T, a.k + a.S, a.H, a.out, a.out_f32, st,
                        /*pdl=*/true);
    if (e != cudaSuccess) return e;
    return mark(6) ? cudaSuccess : cudaErrorUnknown;
  }
  const int max_groups = (R < a.E ? R : a.E) + a.S;
  // every expert (and shared expert) has at most T tokens: with T <= 8 one
  // B tile holds them all, and the ring kernels keep those token rows in
  // shared memory next to the rings
  const int nx = a.T < 8 ? a.T : 8;
  const size_t w13_smem = w13_ring_bytes() + (size_t)nx * a.H * 2;
  const size_t w2_smem = w2_ring_bytes() + (size_t)nx * a.I * 2;
  const bool few = a.T <= kDecodeFewMaxT && w13_smem <= 200 * 1024 &&
                   w2_smem <= 200 * 1024;
  if (few) {
    auto w13k = decode_w13_few_kernel<kW13Ring>;
    auto w2k = decode_w2_few_kernel<kW2Ring>;
    // dynamic shared memory above 48 KiB needs the opt-in
    if ((e = cudaFuncSetAttribute(w13k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)w13_smem)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(w2k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)w2_smem)) != cudaSuccess)
      return e;
    e = launch_ex(w13k, dim3(max_groups, (a.I + kDecRows - 1) / kDecRows),
                  dim3(kDecThreads), w13_smem, st, true, a.x, a.w13, a.w13_sh,
                  (const int32_t*)a.meta, (const int32_t*)a.slots, a.T, a.H, a.I, a.E,
                  a.k, a.S, a.act, a.h_dec);
    if (e != cudaSuccess) return e;
    if (!mark(4)) return cudaErrorUnknown;
    e = launch_ex(w2k, dim3(max_groups, (a.H + kW2Rows - 1) / kW2Rows),
                  dim3(kDecThreads), w2_smem, st, true, (const __nv_bfloat16*)a.h_dec,
                  a.w2, a.w2_sh, (const int32_t*)a.meta, (const int32_t*)a.slots,
                  (const float*)a.w, a.T, a.H, a.I, a.E, a.k, a.S, a.stage);
    if (e != cudaSuccess) return e;
  } else {
    e = launch_ex(decode_w13_kernel, dim3(max_groups, (a.I + kDecRows - 1) / kDecRows),
                  dim3(kDecThreads), 0, st, true, a.x, a.w13, a.w13_sh,
                  (const int32_t*)a.meta, (const int32_t*)a.slots, a.T, a.H, a.I, a.E,
                  a.k, a.S, a.act, a.h_dec);
    if (e != cudaSuccess) return e;
    if (!mark(4)) return cudaErrorUnknown;
    e = launch_ex(decode_w2_kernel, dim3(max_groups, (a.H + kW2Rows - 1) / kW2Rows),
                  dim3(kDecThreads), 0, st, true, (const __nv_bfloat16*)a.h_dec, a.w2,
                  a.w2_sh, (const int32_t*)a.meta, (const int32_t*)a.slots,
                  (const float*)a.w, a.T, a.H, a.I, a.E, a.k, a.S, a.stage);
    if (e != cudaSuccess) return e;
  }
  if (!mark(5)) return cudaErrorUnknown;
  e = launch_sum_rows(a.stage, a.T, a.k + a.S, a.H, a.out, a.out_f32, st,
                      /*pdl=*/true);
  if (e != cudaSuccess) return e;
  if (!mark(6)) return cudaErrorUnknown;
  return cudaSuccess;
}

}  // namespace moe
