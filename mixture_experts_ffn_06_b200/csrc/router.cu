// router.cu -- router logits from the residual stream: the step ahead of the
// routing in the Gemma 4 walkthrough (yeyulingfeng.com/587419.html, section
// 3, "Gemma4Router-MoE 的入口") and the Gemma4Router class on the vLLM API
// page.  For each token row r of the residual (bf16):
//   1. RMSNorm without gamma, in fp32, returned in bf16:
//        n_h = bf16(r_h * (1 / sqrt(mean(r^2) + eps)))
//   2. a_h = bf16(n_h * bf16(H^-0.5))
//   3. b_h = bf16(a_h * s_h)          (s: the learned per-dimension scale)
//   4. z_e = sum_h b_h W[e,h] in fp32 (GateLinear: bf16 in, fp32 out).
// mean(r^2) is accumulated in double (a square of a bf16 value is exact in
// it), so its rounding to fp32 gives the same normaliser as the oracle's
// sequential double sum unless the two land on different sides of an fp32
// rounding point, which takes a difference in the 53rd bit; 1/sqrt is the
// IEEE fp32 division and square root, not the approximate reciprocal square
// root.  Step 1 is an fp32 product rounded to bf16; steps 2 and 3 multiply
// two bf16 values, whose product is exact in fp32, so the bf16x2 multiply
// (one rounding of the exact product) gives the same bf16 as the fp32
// product cast to bf16.  The activations are therefore the oracle's; the
// logits differ from it only by the fp32 accumulation of the projection.
//
// One CTA of 8 warps takes 64 tokens and up to 128 experts (grid.y covers
// larger E).  It streams the tokens' rows twice through a ring of shared-
// memory slots: once to sum their squares, then with the experts' weight rows
// and the scale for the projection; the second read of the residual comes
// from L2.  Warp w multiplies token group w % 4 (16 tokens, one 16-row MMA
// tile of activations) by the experts' weight rows (n8 tiles) with mma.sync
// m16n8k16 over half of each staged K-block (w / 4 picks the half); the two
// halves are added through shared memory in a fixed order at the end.
// Inside each 32-column chunk of K the column order is permuted so that
// every fragment is one 16-byte shared-memory load: thread (g, c) takes
// columns [8c, 8c + 8) of token rows g and g + 8 and of expert row g; both
// operands share the order, so the dot products are unchanged.  The
// activations of a chunk are formed in registers from the staged residual
// and scale.
#include <cmath>

#include "internal.cuh"

namespace moe {
namespace {

constexpr int kRtWarps = 8;
constexpr int kRtGroups = 4;                 // 16-token groups per CTA
constexpr int kRtTokens = 16 * kRtGroups;    // tokens per CTA
constexpr int kRtThreads = kRtWarps * 32;

__device__ __forceinline__ void rt_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Steps 1-3 for one bf16 pair of a token row: bf16(bf16(bf16(x inv) root) s),
// root2 = bf16(H^-0.5) in both halves
__device__ __forceinline__ uint32_t rt_act2(uint32_t x2, uint32_t s2, float inv,
                                            uint32_t root2) {
  const float lo = __fmul_rn(bf_lo(x2), inv), hi = __fmul_rn(bf_hi(x2), inv);
  uint32_t n2, a2, b2;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(n2) : "f"(hi), "f"(lo));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(a2) : "r"(n2), "r"(root2));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(b2) : "r"(a2), "r"(s2));
  return b2;
}

__device__ __forceinline__ uint4 rt_act8(const uint4& x, const uint4& s, float inv,
                                         uint32_t root2) {
  return make_uint4(rt_act2(x.x, s.x, inv, root2), rt_act2(x.y, s.y, inv, root2),
                    rt_act2(x.z, s.z, inv, root2), rt_act2(x.w, s.w, inv, root2));
}

// 16-byte asynchronous copy global -> shared; src_bytes 0 fills zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 rt_lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

constexpr int kRtKB = 256;  // K columns per staged block
// Bytes per staged row: 512 + 64, so rows g and g + 1 fall 16 banks apart
// and the 8 lanes of one shared-memory phase -- two rows, four 16-byte
// vectors each -- cover the 32 banks once.
constexpr int kRtPitch = kRtKB * 2 + 64;
constexpr uint32_t kRtRingMax = 224 * 1024;
static_assert(kRtKB / 8 == 32, "one staged row is 32 16-byte vectors");

// Rows of one staged block: 8 NT expert rows of W, the 64 token rows of the
// residual, and the scale.
__host__ __device__ constexpr int rt_rows(int NT) { return 8 * NT + kRtTokens + 1; }
// Ring depth: as many blocks as fit in kRtRingMax bytes, at most 4.
__host__ __device__ constexpr int rt_stages(int NT) {
  return kRtRingMax / ((uint32_t)rt_rows(NT) * kRtPitch) > 4
             ? 4
             : (int)(kRtRingMax / ((uint32_t)rt_rows(NT) * kRtPitch));
}

// Norm-pass ring depth: the same shared memory cut into slots of the 64
// token rows alone, at most 6.
__host__ __device__ constexpr int rt_norm_stages(int NT) {
  return rt_stages(NT) * rt_rows(NT) / kRtTokens > 6 ? 6
                                                       : rt_stages(NT) * rt_rows(NT) / kRtTokens;
}

// NT n8 tiles: the CTA's 8 NT experts (<= 128).  The CTA runs 2 nkb jobs
// through shared memory filled with 16-byte asynchronous copies: the norm
// pass stages K-block j of the token rows into a ring of rt_norm_stages(NT)
// slots, up to Q - 1 blocks ahead, and sums their squares; the projection
// stages K-block kb of the expert rows, the token rows (again, now from L2)
// and the scale into a ring of rt_stages(NT) larger slots over the same
// memory, up to S - 1 blocks ahead.  Only rows that exist are
// copied; columns past H are filled with zeros, so the ragged K tail adds
// nothing.  Rows past T or E of a slot hold stale data: a token row past T
// enters the MMA as zeros, and an expert row past E only feeds its own
// output column, which is not stored.
template <int NT>
__global__ void __launch_bounds__(kRtThreads)
router_logits_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w,
                     const __nv_bfloat16* __restrict__ scale, int64_t T, int H, int E, float eps,
                     uint32_t root2, float* __restrict__ logits) {
  constexpr int EB = 8 * NT;           // experts per CTA
  constexpr int S = rt_stages(NT);
  static_assert(S >= 2, "the ring needs two slots");
  constexpr uint32_t BLK = (uint32_t)rt_rows(NT) * kRtPitch;
  constexpr int XR = EB;               // first token row of a slot
  constexpr int SR = EB + kRtTokens;   // the scale row
  constexpr int Q = rt_norm_stages(NT);
  static_assert(Q >= 2, "the norm ring needs two slots");
  constexpr uint32_t NB = (uint32_t)kRtTokens * kRtPitch;  // one norm slot
  static_assert(kRtGroups * NT * 4 * 32 * 4 <= BLK, "the K-half partial sums fit in a slot");
  extern __shared__ __align__(16) uint8_t ring[];  // [S][rt_rows(NT)][kRtPitch]
  __shared__ float inv_s[kRtTokens];
  __shared__ double part_s[kRtTokens];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, cq = lane & 3;
  const int64_t t0 = (int64_t)blockIdx.x * kRtTokens;
  const int e0 = blockIdx.y * EB;
  const int nt = T - t0 < kRtTokens ? (int)(T - t0) : kRtTokens;  // token rows of the CTA
  const int ne = min(EB, E - e0);                                   // expert rows of the CTA
  const int nkb = (H + kRtKB - 1) / kRtKB;
  const uint32_t ring0 = smem_u32(ring);
  // thread t stages 16-byte vector t % 32 of rows t / 32, t / 32 + 8, ...;
  // a vector past H is a zero fill whose source is the row's start
  const int sv = tid & 31, sr0 = tid >> 5;
  const __nv_bfloat16* const xs = x + (t0 + sr0) * H;
  const __nv_bfloat16* const ws = w + (int64_t)(e0 + sr0) * H;
  const int64_t rstep = (int64_t)kRtWarps * H;
  // token rows of K-block kb into the slot at dst (rows from row0 on)
  auto stage_x = [&](int kb, uint32_t dst, int row0) {
    const bool ok = kb * kRtKB + sv * 8 < H;
    const uint32_t nbytes = ok ? 16u : 0u;
    uint32_t d = dst + (uint32_t)(row0 + sr0) * kRtPitch + (uint32_t)sv * 16;
    const __nv_bfloat16* src = xs + (ok ? kb * kRtKB + sv * 8 : 0);
    for (int r = sr0; r < nt; r += kRtWarps, d += kRtWarps * kRtPitch, src += rstep)
      cp_async16(d, src, nbytes);
  };
  // Norm job j -> norm slot j % Q.  With R = the least power of two >= nt,
  // one job holds m = 64 / R K-blocks: block j m + p in rows [p R, p R + nt).
  // One group per job, empty past the last.
  int R = kRtTokens;
  while (R > 1 && nt <= R / 2) R >>= 1;
  const int m = kRtTokens / R;
  const int nnj = (nkb + m - 1) / m;
  auto stage_n = [&](int j) {
    if (j < nnj)
      for (int p = 0; p < m && j * m + p < nkb; ++p)
        stage_x(j * m + p, ring0 + (uint32_t)(j % Q) * NB, p * R);
    cp_async_commit();
  };
  // projection job kb -> slot kb % S
  auto stage_p = [&](int kb) {
    if (kb < nkb) {
      const uint32_t dst = ring0 + (uint32_t)(kb % S) * BLK;
      stage_x(kb, dst, XR);
      const bool ok = kb * kRtKB + sv * 8 < H;
      const uint32_t nbytes = ok ? 16u : 0u;
      const int cc = ok ? kb * kRtKB + sv * 8 : 0;
      uint32_t d = dst + (uint32_t)sr0 * kRtPitch + (uint32_t)sv * 16;
      const __nv_bfloat16* src = ws + cc;
      for (int r = sr0; r < ne; r += kRtWarps, d += kRtWarps * kRtPitch, src += rstep)
        cp_async16(d, src, nbytes);
      if (sr0 == 0)
        cp_async16(dst + (uint32_t)SR * kRtPitch + (uint32_t)sv * 16, scale + cc, nbytes);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int p = 0; p < Q - 1; ++p) stage_n(p);

  // norm pass: lane l of warp w sums slot row nr = 8w + l / 4 -- token nr % R
  // of the job's block nr / R -- vectors l % 4 + 4i
  const int nr = warp * 8 + (lane >> 2);
  const bool nr_ok = nr % R < nt;
  double ss[8];  // one partial sum per vector slot: eight independent chains
#pragma unroll
  for (int i = 0; i < 8; ++i) ss[i] = 0.0;
  // projection: warp w multiplies token rows 16 (w % 4) + g and + g + 8 over
  // chunks [4 (w / 4), 4 (w / 4) + 4) of each K-block
  const int tg = warp & (kRtGroups - 1), kh = warp / kRtGroups;
  const int ra = tg * 16 + gq, rb = ra + 8;
  const bool va = ra < nt, vb = rb < nt, live = tg * 16 < nt;
  float inv_a = 0.f, inv_b = 0.f;
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);

  // ---- step 1: sum of squares, in double
  for (int j = 0; j < nnj; ++j) {
    stage_n(j + Q - 1);
    cp_async_wait<Q - 1>();  // job j has landed (this thread's copies)
    __syncthreads();         // ... and everyone's
    if (nr_ok && j * m + nr / R < nkb) {
      const uint32_t row = ring0 + (uint32_t)(j % Q) * NB + (uint32_t)nr * kRtPitch +
                           (uint32_t)(lane & 3) * 16;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = rt_lds128(row + i * 64);
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const double lo = bf_lo(wd[u]), hi = bf_hi(wd[u]);
          ss[i] = fma(lo, lo, ss[i]);
          ss[i] = fma(hi, hi, ss[i]);
        }
      }
    }
    __syncthreads();  // norm slot j % Q is refilled by job j + Q
  }
  // the projection's first blocks stream while the normalisers are formed
#pragma unroll
  for (int p = 0; p < S - 1; ++p) stage_p(p);
  {
    double sum = ((ss[0] + ss[1]) + (ss[2] + ss[3])) + ((ss[4] + ss[5]) + (ss[6] + ss[7]));
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    if ((lane & 3) == 0) part_s[nr] = sum;
    __syncthreads();
    // token r: its m partial sums in order of the block
    if (tid < nt) {
      double tot = 0.0;
      for (int p = 0; p < m; ++p) tot += part_s[p * R + tid];
      const float var = (float)(tot / (double)H);
      inv_s[tid] = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps)));
    }
    __syncthreads();
    if (va) inv_a = inv_s[ra];
    if (vb) inv_b = inv_s[rb];
  }
  // ---- steps 2-4: this warp's half of each K-block
  for (int kb = 0; kb < nkb; ++kb) {
    stage_p(kb + S - 1);
    cp_async_wait<S - 1>();
    __syncthreads();
    const uint32_t slot = ring0 + (uint32_t)(kb % S) * BLK;
    if (live) {
      const int ch_end = min(4 * kh + 4, (H - kb * kRtKB + 31) / 32);
      const uint32_t xa = slot + (uint32_t)(XR + ra) * kRtPitch;
      const uint32_t xb = xa + 8 * kRtPitch;
      const uint32_t srow = slot + (uint32_t)SR * kRtPitch;
      for (int ch = 4 * kh; ch < ch_end; ++ch) {
        const uint32_t col_b = (uint32_t)(ch * 32 + 8 * cq) * 2;
        const uint4 cs = rt_lds128(srow + col_b);
        const uint4 a0 = va ? rt_act8(rt_lds128(xa + col_b), cs, inv_a, root2) : z4;
        const uint4 a8 = vb ? rt_act8(rt_lds128(xb + col_b), cs, inv_b, root2) : z4;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint4 bv = rt_lds128(slot + (uint32_t)(n * 8 + gq) * kRtPitch + col_b);
          rt_mma(acc[n], a0.x, a8.x, a0.y, a8.y, bv.x, bv.y);
          rt_mma(acc[n], a0.z, a8.z, a0.w, a8.w, bv.z, bv.w);
        }
      }
    }
    __syncthreads();  // slot kb % S is refilled by block kb + S
  }
  cp_async_wait<0>();
  // ---- the two K-halves: the second half's tiles go through slot 0 (free
  // now), the first half adds them and stores
  float* red = reinterpret_cast<float*>(ring);  // [group][n][e][lane]
  if (kh == 1 && live) {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[((tg * NT + n) * 4 + e) * 32 + lane] = acc[n][e];
  }
  __syncthreads();
  if (kh == 1 || !live) return;
  // fragment element e: token row g (+8 for e >= 2), expert 2c + e % 2
  const int64_t ta = t0 + ra, tb = t0 + rb;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    float o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = acc[n][e] + red[((tg * NT + n) * 4 + e) * 32 + lane];
    const int c = n * 8 + 2 * cq;
    const int e = e0 + c;
    if (va && c < ne) logits[ta * E + e] = o[0];
    if (va && c + 1 < ne) logits[ta * E + e + 1] = o[1];
    if (vb && c < ne) logits[tb * E + e] = o[2];
    if (vb && c + 1 < ne) logits[tb * E + e + 1] = o[3];
  }
}

template <int NT>
cudaError_t launch_router_nt(const __nv_bfloat16* x, const __nv_bfloat16* w,
                             const __nv_bfloat16* scale, int64_t T, int H, int E, float eps,
                             uint32_t root2, float* logits, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)rt_stages(NT) * rt_rows(NT) * kRtPitch;
  const cudaError_t e = cudaFuncSetAttribute(
      router_logits_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((T + kRtTokens - 1) / kRtTokens),
                  (unsigned)((E + 8 * NT - 1) / (8 * NT)));
  return launch_ex(router_logits_kernel<NT>, grid, dim3(kRtThreads), smem, st, pdl, x, w,
                   scale, T, H, E, eps, root2, logits);
}

}  // namespace

float router_root(int H) {
  // bf16(fl(H^-0.5)): the fp32 constant cast to bf16 (round to nearest even)
  const float r = (float)std::pow((double)H, -0.5);
  return __bfloat162float(__float2bfloat16_rn(r));
}

cudaError_t launch_router_logits(const __nv_bfloat16* x, const __nv_bfloat16* w_router,
                                 const __nv_bfloat16* scale, int64_t T, int H, int E,
                                 float eps, float* logits, cudaStream_t st, bool pdl) {
  if (T == 0) return cudaSuccess;
  const uint32_t rb = __bfloat16_as_ushort(__float2bfloat16_rn(router_root(H)));
  const uint32_t root2 = rb | (rb << 16);
  // experts per CTA: the fewest n8 tiles that cover E, at most 16 (grid.y
  // takes the rest); with few token tiles, fewer, so that the weight rows
  // stream through more SMs
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int nt = E <= 8 ? 1 : E <= 16 ? 2 : E <= 32 ? 4 : E <= 64 ? 8 : 16;
  const int64_t tiles_t = (T + kRtTokens - 1) / kRtTokens;
  while (nt > 1 && tiles_t * ((E + 8 * nt - 1) / (8 * nt)) <= sms / 2) nt >>= 1;
  switch (nt) {
    case 1: return launch_router_nt<1>(x, w_router, scale, T, H, E, eps, root2, logits, st, pdl);
    case 2: return launch_router_nt<2>(x, w_router, scale, T, H, E, eps, root2, logits, st, pdl);
    case 4: return launch_router_nt<4>(x, w_router, scale, T, H, E, eps, root2, logits, st, pdl);
    case 8: return launch_router_nt<8>(x, w_router, scale, T, H, E, eps, root2, logits, st, pdl);
    default:
      return launch_router_nt<16>(x, w_router, scale, T, H, E, eps, root2, logits, st, pdl);
  }
}

}  // namespace moe
