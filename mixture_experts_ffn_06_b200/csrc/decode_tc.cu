// decode_tc.cu -- the decode path's expert products on the sm_100a tensor
// cores.
//
// With few tokens the layer is bound by streaming the touched experts'
// weights from HBM (llama-cpp-visual-guide lesson 35, cost section: decode
// moves the bottleneck to data movement).  Here each weight tile is the M
// side of a tcgen05 MMA and the tokens are its N side:
//   w13 (MODE 0): A = 64 gate rows + the matching 64 up rows of one expert
//                 (M = 128), B = all N token rows of x (rows past T read as
//                 zero), D[128, N] in TMEM; the epilogue pairs gate row r with
//                 up row r and writes h = bf16(Act(g) * u) for the tokens the
//                 expert was routed to, into h_dense [touched, N, I];
//   w2  (MODE 1): A = 128 rows of W2 (H rows of one expert), B = the
//                 expert's N rows of h_dense; the epilogue multiplies each
//                 routed token's column by its gate weight and stores it at
//                 the (token, choice) row of stage [T*(k+S), H] (sum_rows then
//                 adds the k+S rows of a token in a fixed order).
// Computing all N token columns for every touched expert costs nothing that
// shows (the MMA is idle most of the time) and needs no gather.
//
// Work split (the weight stream must keep every SM busy even when only 8
// experts are touched): the iteration space is (unit, k-block), a unit being
// (touched group, row block), and CTA c of C takes the contiguous range
// [c * total / C, (c + 1) * total / C).  A unit that lies inside one CTA's
// range is finished from TMEM.  A unit split over several CTAs has each of
// them store its partial sum ([128, T] fp32) and count one arrival on the
// unit's counter; the CTA that brings the last arrival adds the partials in
// CTA order (a fixed order: the result does not depend on timing) and
// finishes the unit.  Nothing waits on another CTA.
//
// Roles: warp 0 issues the TMA loads into a ring of shared-memory stages,
// warp 1 lane 0 issues tcgen05.mma into one of two TMEM accumulators, warps
// 2-5 are the epilogue.  Every mbarrier wait is bounded (tc_ptx.cuh); after
// a timeout the block records MOE_ERR_TIMEOUT, the epilogue keeps walking
// its segments without touching TMEM (so its named barriers stay matched),
// and TMEM is freed.
#include <algorithm>

#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int kDtThreads = 192;
constexpr uint64_t kDtTimeoutNs = 1000000000ull;  // 1 s per wait

template <int N>
struct DtCfg {
  static constexpr int A_STAGE = 128 * 64 * 2;  // 16 KiB of weights
  static constexpr int B_STAGE = N * 64 * 2;    // token rows
  // two CTAs per SM, each with about 90 KiB of weights in flight: two
  // producer / MMA pipelines per SM stream faster than one twice as deep
  static constexpr int STAGES = N == 64 ? 3 : (N == 32 ? 4 : 5);
  static constexpr int AS = N < 32 ? 32 : N;    // TMEM columns per accumulator
  static constexpr uint32_t TMEM_COLS = 2 * AS;
};

struct DtParams {
  const int32_t* meta;   // decode_route: [0] touched groups, [1+i] group id,
                         // [1+G+i] first slot-list entry of group i
  const int32_t* slots;  // per-group slot lists
  const float* wgt;      // [T,k] gate weights (MODE 1)
  int T, k, S, E, G, H, I;
  int KB, RB;            // k-blocks per unit, row blocks per group
  int act;
  __nv_bfloat16* h;      // MODE 0 out: [touched][N][I]
  float* stage;          // MODE 1 out: [T*(k+S)][H]
  float* part;           // [2 * gridDim.x][128][T] partial sums
  int32_t* cnt;          // [touched * RB] arrival counters, zero on entry
  // FP8: weight row scales (routed, shared) and the B rows' scales (x's per
  // token, or h's per group and token column)
  const float* ascale;
  const float* ascale_sh;
  const float* bscale;
  uint32_t* err;
  uint64_t timeout_ns;
};

struct DtCtl {
  uint64_t full[12];
  uint64_t empty[12];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t last;          // the epilogue's "this CTA finishes the unit"
  int32_t cm_dst[64];    // per token column: destination row (or -1)
  float cm_w[64];        // per token column: gate weight
};

// 16 consecutive fp32 columns of this thread's TMEM lane, waited on.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
        "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// The epilogue's own barrier (warps 2-5 only).
__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ float dt_act(int act, float g) {
  if (act == MOE_ACT_SILU) return g / (1.0f + expf(-g));
  const float c = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * g * (1.0f + tanhf(c * fmaf(0.044715f * g, g * g, g)));
}

// First iteration of CTA c, and the CTA whose range holds iteration it.
__device__ __forceinline__ int64_t range_start(int64_t c, int64_t total, int64_t C) {
  return c * total / C;
}
__device__ __forceinline__ int cta_of(int64_t it, int64_t total, int64_t C) {
  return (int)(((it + 1) * C + total - 1) / total - 1);
}

// Release-acquire arrival on a unit's counter (one thread, after the
// epilogue's barrier has ordered every epilogue thread's partial-sum stores
// before it); returns the count before the arrival.
__device__ __forceinline__ int arrive_acq_rel(int32_t* cnt) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
               : "=r"(old)
               : "l"(cnt)
               : "memory");
  return old;
}

// The CTA's share of the (unit, k-block) iterations: with fewer iterations
// than CTAs only the first `total` CTAs take part, so that every
// participating range is non-empty and the CTAs sharing a unit are
// consecutive.  Iterations: at most 520 groups x 128 row blocks x 128
// k-blocks < 2^31 (the host checks).
struct DtRange {
  int total, Cn, s0, s1;
};
__device__ __forceinline__ DtRange dt_range(int n_groups, int RB, int KB) {
  DtRange r;
  r.total = n_groups * RB * KB;
  r.Cn = min((int)gridDim.x, r.total);
  const bool part = (int)blockIdx.x < r.Cn;
  r.s0 = part ? (int)range_start(blockIdx.x, r.total, r.Cn) : 0;
  r.s1 = part ? (int)range_start(blockIdx.x + 1, r.total, r.Cn) : 0;
  return r;
}

template <int N, int MODE, bool F8>
__global__ void __launch_bounds__(kDtThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                 const __grid_constant__ CUtensorMap tmAs,
                 const __grid_constant__ CUtensorMap tmB, const DtParams p) {
  using C = DtCfg<N>;
  constexpr int ST = C::STAGES;
  // a k-block is 128 bytes of each row: 64 bf16 values or 128 e4m3 codes
  constexpr int KBE = F8 ? 128 : 64;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sA = base;
  const uint32_t sB = base + ST * C::A_STAGE;
  float(*xch)[N + 1] = reinterpret_cast<float(*)[N + 1]>(
      gbase + ST * (C::A_STAGE + C::B_STAGE));   // [64][N+1] up-row values
  DtCtl* ctl = reinterpret_cast<DtCtl*>(gbase + ST * (C::A_STAGE + C::B_STAGE) +
                                        64 * (N + 1) * sizeof(float));
  volatile int32_t* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&ctl->tmem_full[a]), 1);
      mbar_init(smem_u32(&ctl->tmem_empty[a]), 4);  // one per epilogue warp
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort_flag = 0;
    mbar_init_fence();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmAs);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(smem_u32(&ctl->tmem_base), C::TMEM_COLS);

  // w2: the weights do not depend on the w13 kernel, so before waiting for
  // it the producer (thread 0, which initialised the barriers) fills the
  // ring with the weight tiles of its first iterations.  The routing lists
  // come from the routing kernel, which had completed before the w13
  // kernel (and so this one) could start; they are read through L2.
  int pre = 0;
  if (MODE == 1 && threadIdx.x == 0) {
    const DtRange r = dt_range(__ldcg(p.meta), p.RB, p.KB);
    pre = min(ST, r.s1 - r.s0);
    for (int j = 0; j < pre; ++j) {
      const int it = r.s0 + j;
      const int u = it / p.KB, kb = it - u * p.KB;
      const int i = u / p.RB, rb = u - i * p.RB;
      const int g = __ldcg(p.meta + 1 + i);
      const bool routed = g < p.E;
      const uint32_t fb = smem_u32(&ctl->full[j]);
      mbar_expect_tx(fb, C::A_STAGE + C::B_STAGE);
      tma_load_2d(sA + j * C::A_STAGE, routed ? &tmA : &tmAs, kb * KBE,
                  (routed ? g : g - p.E) * p.H + rb * 128, fb);
    }
  }
  // the routing (meta, slots) and, for w2, h come from the kernels before
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const DtRange rg = dt_range(__ldg(p.meta), p.RB, p.KB);
  const int total = rg.total, Cn = rg.Cn, s0 = rg.s0, s1 = rg.s1;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int32_t last_fill[ST];
      for (int s = 0; s < ST; ++s) last_fill[s] = -1;
      bool ok = true;
      // walk the range unit by unit: the unit's coordinates are computed
      // once, the k-blocks of a unit need no division
      for (int it = s0; ok && it < s1;) {
        const int u = it / p.KB;
        const int kb0 = it - u * p.KB;
        const int kb1 = min(p.KB, s1 - u * p.KB);
        const int it0 = it;
        it = u * p.KB + kb1;
        const int i = u / p.RB, rb = u - i * p.RB;
        const int g = __ldg(p.meta + 1 + i);
        const bool routed = g < p.E;
        const CUtensorMap* ma = routed ? &tmA : &tmAs;
        const int gl = routed ? g : g - p.E;
        const int32_t ar = MODE == 0 ? gl * 2 * p.I + rb * 64 : gl * p.H + rb * 128;
        const int32_t br = MODE == 0 ? 0 : i * N;
        for (int kb = kb0; kb < kb1; ++kb) {
          const uint32_t fb = smem_u32(&ctl->full[stage]);
          if (it0 + (kb - kb0) - s0 < pre) {
            // weights already requested before the wait: only h is left
            tma_load_2d(sB + stage * C::B_STAGE, &tmB, kb * KBE, br, fb);
          } else {
            if (!mbar_wait(smem_u32(&ctl->empty[stage]), phase ^ 1u, abort_flag,
                           p.timeout_ns, p.err)) {
              ok = false;
              break;
            }
            mbar_expect_tx(fb, C::A_STAGE + C::B_STAGE);
            const uint32_t a_dst = sA + stage * C::A_STAGE;
            tma_load_2d(a_dst, ma, kb * KBE, ar, fb);
            // w13: the up rows matching the gate rows, I rows further on
            if (MODE == 0)
              tma_load_2d(a_dst + C::A_STAGE / 2, ma, kb * KBE, ar + p.I, fb);
            tma_load_2d(sB + stage * C::B_STAGE, &tmB, kb * KBE, br, fb);
          }
          last_fill[stage] = (int32_t)phase;
          if (++stage == ST) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok || pre > s1 - s0) {
        // let the copies already issued land before the block exits
        int32_t none = 0;
        volatile int32_t* never = &none;
        for (int s = 0; s < ST; ++s)
          if (last_fill[s] >= 0)
            mbar_wait(smem_u32(&ctl->full[s]), (uint32_t)last_fill[s], never,
                      p.timeout_ns, p.err);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(128, N) : idesc_bf16_f32(128, N);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int it = s0; ok && it < s1;) {
        const int u = it / p.KB;
        const int kb0 = it - u * p.KB;
        const int kb1 = min(p.KB, s1 - u * p.KB);
        it = u * p.KB + kb1;
        if (!mbar_wait(smem_u32(&ctl->tmem_empty[acc]), acc_phase ^ 1u, abort_flag,
                       p.timeout_ns, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + acc * C::AS;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&ctl->full[stage]), phase, abort_flag, p.timeout_ns,
                         p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(sA + stage * C::A_STAGE);
          const uint64_t bd = sw128_kmajor_desc(sB + stage * C::B_STAGE);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma<F8>(d, ad + 2u * kk, bd + 2u * kk, idesc,
                      (kb != kb0 || kk != 0) ? 1u : 0u);
          umma_commit(smem_u32(&ctl->empty[stage]));
          if (++stage == ST) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(smem_u32(&ctl->tmem_full[acc]));
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok || *abort_flag) {
        // wait for the MMAs already issued before TMEM is released
        int32_t none = 0;
        volatile int32_t* never = &none;
        umma_commit(smem_u32(&ctl->drain));
        mbar_wait(smem_u32(&ctl->drain), 0, never, p.timeout_ns, p.err);
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // Warp w reads TMEM lanes [32 (w % 4), 32 (w % 4) + 32): tile row `row`.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int te = threadIdx.x - 64;  // 0..127
    const int R = p.T * p.k, ks = p.k + p.S;
    uint32_t acc = 0, acc_phase = 0;
    for (int it = s0; it < s1;) {
      const int u = it / p.KB;
      const int u0 = u * p.KB, u1 = u0 + p.KB;
      it = min(s1, u1);
      const int i = u / p.RB, rb = u - i * p.RB;

      // which token columns this group was routed to (built while the
      // segment's MMAs still run)
      const int gbase = __ldg(p.meta + 1 + p.G + i);
      const int gn = __ldg(p.meta + 2 + p.G + i) - gbase;
      if (te < N) ctl->cm_dst[te] = -1;
      epi_bar();
      if (te < gn) {
        const int s = __ldg(p.slots + gbase + te);
        int t, dst;
        float w;
        if (s < R) {
          t = s / p.k;
          dst = t * ks + (s - t * p.k);
          w = MODE == 1 ? __ldg(p.wgt + s) : 1.0f;
        } else {
          const int qq = s - R, sh = qq / p.T;
          t = qq - sh * p.T;
          dst = t * ks + p.k + sh;
          w = 1.0f;
        }
        ctl->cm_dst[t] = dst;
        ctl->cm_w[t] = w;
      }

      // this segment's accumulator (skipped, not waited on, after an abort)
      const bool got = mbar_wait(smem_u32(&ctl->tmem_full[acc]), acc_phase, abort_flag,
                                 p.timeout_ns, p.err);
      const bool live = __all_sync(0xffffffffu, got);
      tc_fence_after();
      float v[N];
      if (live) {
        const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::AS;
        if constexpr (N == 16) {
          uint32_t r[16];
          tmem_ld16(ta, r);
#pragma unroll
          for (int c = 0; c < 16; ++c) v[c] = __uint_as_float(r[c]);
        } else {
#pragma unroll
          for (int c0 = 0; c0 < N; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(ta + c0, r);
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c0 + c] = __uint_as_float(r[c]);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < N; ++c) v[c] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->tmem_empty[acc]));
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;

      // a unit split over several CTAs: partial sums, the last one finishes
      const int cf = cta_of(u0, total, Cn), cl = cta_of(u1 - 1, total, Cn);
      if (cf != cl) {
        const int cme = blockIdx.x;
        const int slot = s0 >= u0 ? 2 * cme : 2 * cme + 1;
        float* pp = p.part + ((int64_t)slot * 128 + row) * p.T;
#pragma unroll
        for (int c = 0; c < N; ++c)
          if (c < p.T) __stcg(pp + c, v[c]);
        epi_bar();  // every epilogue thread's stores come before the arrival
        if (te == 0) {
          const int last = arrive_acq_rel(p.cnt + u) == cl - cf;
          if (last) p.cnt[u] = 0;  // ready for the next call
          ctl->last = last;
        }
        epi_bar();
        const bool last = *reinterpret_cast<volatile int32_t*>(&ctl->last) != 0;
        if (!last) {
          epi_bar();  // the column map is rewritten for the next unit
          continue;
        }
        // the partials of the other CTAs (their order, not arrival order)
#pragma unroll
        for (int c = 0; c < N; ++c) v[c] = 0.f;
        for (int cc = cf; cc <= cl; ++cc) {
          const int sl = range_start(cc, total, Cn) >= u0 ? 2 * cc : 2 * cc + 1;
          const float* src = p.part + ((int64_t)sl * 128 + row) * p.T;
#pragma unroll
          for (int c = 0; c < N; ++c)
            if (c < p.T) v[c] += __ldcg(src + c);
        }
      }

      if (F8) {
        // the accumulator of codes times this row's weight scale and each
        // column's scale (x: per token; h: per group and token column)
        const int g = __ldg(p.meta + 1 + i);
        const bool routed = g < p.E;
        const int gl = routed ? g : g - p.E;
        const float* as = routed ? p.ascale : p.ascale_sh;
        float sa = 0.0f;
        if (MODE == 0) {
          const int r = rb * 64 + (row & 63);  // row of I (gate or up half)
          if (r < p.I) sa = __ldg(as + (int64_t)gl * 2 * p.I + (row >= 64 ? p.I : 0) + r);
        } else {
          const int r = rb * 128 + row;  // row of H
          if (r < p.H) sa = __ldg(as + (int64_t)gl * p.H + r);
        }
#pragma unroll
        for (int c = 0; c < N; ++c) {
          float sb = 0.0f;
          if (MODE == 0) {
            if (c < p.T) sb = __ldg(p.bscale + c);
          } else {
            sb = __ldg(p.bscale + (int64_t)i * N + c);
          }
          v[c] *= sa * sb;
        }
      }
      if (MODE == 0 && row >= 64) {
#pragma unroll
        for (int c = 0; c < N; ++c) xch[row - 64][c] = v[c];
      }
      epi_bar();
      if (MODE == 0) {
        const int r = rb * 64 + row;  // row of I (gate rows are tile rows < 64)
        if (row < 64 && r < p.I) {
#pragma unroll
          for (int c = 0; c < N; ++c)
            if (ctl->cm_dst[c] >= 0)
              p.h[((int64_t)i * N + c) * p.I + r] =
                  __float2bfloat16_rn(dt_act(p.act, v[c]) * xch[row][c]);
        }
      } else {
        const int r = rb * 128 + row;  // row of H
        if (r < p.H) {
#pragma unroll
          for (int c = 0; c < N; ++c) {
            const int dst = ctl->cm_dst[c];
            if (dst >= 0) p.stage[(int64_t)dst * p.H + r] = __fmul_rn(ctl->cm_w[c], v[c]);
          }
        }
      }
      epi_bar();  // the column map and xch are rewritten for the next unit
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int N>
constexpr size_t dt_smem_bytes() {
  return 1024 + (size_t)DtCfg<N>::STAGES * (DtCfg<N>::A_STAGE + DtCfg<N>::B_STAGE) +
         64 * (N + 1) * sizeof(float) + sizeof(DtCtl);
}

template <int N, int MODE, bool F8>
cudaError_t launch_dt(const DecodeArgs& a, const void* b_ptr, void* out,
                      cudaStream_t st) {
  const int G = a.E + a.S;
  const int n_max = std::min(a.T * a.k, a.E) + a.S;  // touched groups, at most
  constexpr int KBE = F8 ? 128 : 64;
  auto map = F8 ? make_tma_map_e4m3 : make_tma_map_bf16;
  const void* wa = MODE == 0 ? (F8 ? (const void*)a.w13q : (const void*)a.w13)
                             : (F8 ? (const void*)a.w2q : (const void*)a.w2);
  const void* wa_sh = MODE == 0 ? (F8 ? (const void*)a.w13q_sh : (const void*)a.w13_sh)
                                : (F8 ? (const void*)a.w2q_sh : (const void*)a.w2_sh);
  CUtensorMap mA, mAs, mB;
  cudaError_t e;
  if (MODE == 0) {
    e = map(&mA, wa, a.H, 2ull * a.I * a.E, 64);
    if (e == cudaSuccess)
      e = a.S ? map(&mAs, wa_sh, a.H, 2ull * a.I * a.S, 64) : (mAs = mA, cudaSuccess);
    if (e == cudaSuccess) e = map(&mB, b_ptr, a.H, a.T, N);
  } else {
    e = map(&mA, wa, a.I, (uint64_t)a.H * a.E, 128);
    if (e == cudaSuccess)
      e = a.S ? map(&mAs, wa_sh, a.I, (uint64_t)a.H * a.S, 128) : (mAs = mA, cudaSuccess);
    if (e == cudaSuccess) e = map(&mB, b_ptr, a.I, (uint64_t)n_max * N, N);
  }
  if (e != cudaSuccess) return e;
  DtParams p;
  p.meta = a.meta;
  p.slots = a.slots;
  p.wgt = a.w;
  p.T = a.T;
  p.k = a.k;
  p.S = a.S;
  p.E = a.E;
  p.G = G;
  p.H = a.H;
  p.I = a.I;
  p.KB = MODE == 0 ? (a.H + KBE - 1) / KBE : (a.I + KBE - 1) / KBE;
  p.RB = MODE == 0 ? (a.I + 63) / 64 : (a.H + 127) / 128;
  p.act = a.act;
  p.h = MODE == 0 ? static_cast<__nv_bfloat16*>(out) : nullptr;
  p.stage = MODE == 1 ? static_cast<float*>(out) : nullptr;
  p.part = a.dt_part;
  p.cnt = a.dt_cnt + (MODE == 0 ? 0 : (size_t)G * dt_row_blocks(a.H, a.I));
  p.err = a.err;
  p.timeout_ns = kDtTimeoutNs;
  p.ascale = F8 ? (MODE == 0 ? a.w13s : a.w2s) : nullptr;
  p.ascale_sh = F8 ? (MODE == 0 ? a.w13s_sh : a.w2s_sh) : nullptr;
  p.bscale = F8 ? (MODE == 0 ? a.sx : a.sh) : nullptr;
  constexpr size_t smem = dt_smem_bytes<N>();
  e = cudaFuncSetAttribute(decode_tc_kernel<N, MODE, F8>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  static_assert(2 * (smem + 1024) <= 228 * 1024, "two CTAs per SM");
  e = cudaFuncSetAttribute(decode_tc_kernel<N, MODE, F8>,
                           cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int grid = std::min(kDtMaxCtas, 2 * device_sm_count());
  return launch_ex(decode_tc_kernel<N, MODE, F8>, dim3(grid), dim3(kDtThreads), smem, st,
                   true, mA, mAs, mB, p);
}

}  // namespace

int dt_row_blocks(int H, int I) { return std::max((I + 63) / 64, (H + 127) / 128); }

int dt_columns(int T) { return T <= 16 ? 16 : T <= 32 ? 32 : 64; }

cudaError_t launch_decode_tc_w13(const DecodeArgs& a, __nv_bfloat16* h_dense,
                                 cudaStream_t st) {
  // B: the token rows of x (bf16), or their e4m3 codes
  if (a.f8) {
    if (a.T <= 16) return launch_dt<16, 0, true>(a, a.xq, h_dense, st);
    if (a.T <= 32) return launch_dt<32, 0, true>(a, a.xq, h_dense, st);
    return launch_dt<64, 0, true>(a, a.xq, h_dense, st);
  }
  if (a.T <= 16) return launch_dt<16, 0, false>(a, a.x, h_dense, st);
  if (a.T <= 32) return launch_dt<32, 0, false>(a, a.x, h_dense, st);
  return launch_dt<64, 0, false>(a, a.x, h_dense, st);
}

cudaError_t launch_decode_tc_w2(const DecodeArgs& a, const __nv_bfloat16* h_dense,
                                cudaStream_t st) {
  // B: h [touched * N, I] (bf16), or its e4m3 codes
  if (a.f8) {
    if (a.T <= 16) return launch_dt<16, 1, true>(a, a.hq, a.stage, st);
    if (a.T <= 32) return launch_dt<32, 1, true>(a, a.hq, a.stage, st);
    return launch_dt<64, 1, true>(a, a.hq, a.stage, st);
  }
  if (a.T <= 16) return launch_dt<16, 1, false>(a, h_dense, a.stage, st);
  if (a.T <= 32) return launch_dt<32, 1, false>(a, h_dense, a.stage, st);
  return launch_dt<64, 1, false>(a, h_dense, a.stage, st);
}

}  // namespace moe
