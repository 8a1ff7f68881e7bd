// gemm_tc.cu -- grouped expert GEMMs on the sm_100a tensor cores.
//
// The expert FFN of the Gemma 4 MoE walkthrough (yeyulingfeng.com/587419.html
// section 6; "MOE Inference" blog, gated FFN) is two grouped GEMMs over the
// expert-contiguous rows built by layout.cu:
//   mode 0 (w13): h[r, n] = Act(x_r . W1_e[n]) * (x_r . W3_e[n]),  n < I
//   mode 1 (w2):  y[r, n] = h_r . W2_e[n],                         n < H
// The pages batch these as FusedMoE's grouped GEMM (walkthrough section 7
// step 3) and ggml_mul_mat_id (llama-cpp-visual-guide lesson 35); their
// Triton / ggml kernels are prior art only.  This kernel is written for
// B200:
//
//   * persistent: one 192-thread CTA per SM walks the tile list
//     (expert-major, then panels of 16 m-tiles, then n-tile, then m-tile,
//     so the CTAs running at once share weight and activation tiles
//     through L2);
//   * warp 0 lane 0 is the TMA producer: 128x64 A tiles and 256x64 B tiles
//     (mode 0: 128 gate rows + the matching 128 up rows) into a 4-stage ring
//     of 128-byte-swizzled shared memory;
//   * warp 1 lane 0 issues tcgen05.mma (M=128, N=256, K=16, bf16 -> fp32)
//     into one of two 256-column TMEM accumulators and releases ring slots
//     and accumulators with tcgen05.commit;
//   * warps 2-5 are the epilogue: tcgen05.ld of their 32 TMEM lanes, the
//     gate activation fused in mode 0 (so g and u never reach HBM) with bf16
//     h stores; in modes 2 and 3 each row is multiplied by its gate weight
//     and either added into its token's fp32 output row (mode 2, vector
//     reductions) or stored at its (token, choice) position for a fixed-order
//     sum (mode 3).  Stores go through a shared-memory transpose so each
//     warp instruction writes whole row segments.  Two accumulators let the
//     epilogue of tile i overlap the MMAs of tile i+1.
// Every wait is bounded (tc_ptx.cuh: mbar_wait); on a timeout the block
// records MOE_ERR_TIMEOUT, drains what it issued and frees its TMEM.
#include <atomic>
#include <mutex>

#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BN_ACC = 256;
constexpr int A_STAGE = BM * BK * 2;  // 16 KiB
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN_ACC;
constexpr uint64_t kTimeoutNs = 1000000000ull;  // 1 s per wait
constexpr int kMaxStages = 6;
constexpr int kPanel = 16;  // m-blocks per panel of the tile order
constexpr int kMaxDevices = 64;  // per-device caches of launch attributes

// CG = CTAs per MMA: 1 (M=128 per CTA, B tile 256 rows per CTA, 4 stages) or
// 2 (a CTA pair computes M=256: each CTA loads its own 128 A rows and half of
// the 256 B rows, so a stage is 32 KiB instead of 48 KiB and 6 fit).
// NH (mode 0, CG = 1): gate rows per tile.  128 gives N = 256; 88 gives
// N = 176 (88 gate + 88 up rows), which tiles I = 704 (the Gemma-4 expert
// width) without the half-empty last n-tile of the 128-row form, and with a
// 38 KiB stage 5 stages fit.
template <int CG, int NH = 128>
struct Cfg {
  static constexpr int B_ROWS = NH == 128 ? BN_ACC / CG : 2 * NH;  // B rows per CTA
  static constexpr int B_STAGE = B_ROWS * BK * 2;
  static constexpr int STAGES = CG == 2 ? 6 : (NH == 128 ? 4 : 5);
  static constexpr int N_MMA = NH == 128 ? BN_ACC : 2 * NH;         // MMA N
};

struct Ctl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

// Vector fp32 reduction into global memory (16-byte aligned destination).
__device__ __forceinline__ void red_add_v4(float* dst, float a, float b, float c,
                                           float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a),
               "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Epilogue scratch: one 32x32 fp32 transpose tile per epilogue warp, and
// the destination row / gate weight of each tile row (modes 2 and 3).  With
// FP8 operands each warp also keeps the tile's 256 column scales (mode 0:
// the gate rows' at [0, 128), the up rows' at [128, 256); 0 past the tile).
// The tile is read and written in 16-byte slots: slot q of row r (columns
// 4q..4q+3) sits at slot q ^ (r mod 8) of the row, so that eight lanes
// writing one slot of eight rows, or reading eight slots of one row, touch
// all 32 banks once.
template <bool F8>
struct EpiSmem {
  float buf[4][32][32];
  int64_t rdst[4][32];
  float rw[4][32];
  float cs[F8 ? 4 : 1][F8 ? 256 : 1];
};

struct KParams {
  const int32_t* offsets;
  int G, E, N, K, NT, KB;
  int32_t b_rows_per_group;  // rows of one expert in the B tensor
  int32_t up_off;            // mode 0: row offset of the up half (= N)
  void* out;
  int act;
  uint32_t* err;
  uint64_t timeout_ns;
  const int32_t* sorted_slots;  // row -> slot (-1: padding row)
  const float* w;               // modes 2, 3
  int64_t T;                    // modes 2, 3
  int k, S;                     // modes 2, 3
  int a_sh_x;                   // shared groups' A rows come from tmAs (x)
  // FP8 operands: the product of row r and column n is scaled by
  // a_scale[r] * b_scale[group row of n] (b_scale_sh for shared groups)
  const float* a_scale;
  const float* b_scale;
  const float* b_scale_sh;
};

// A work unit is (group g, block of CG m-tiles, n-tile); units are ordered
// group-major, then by panels of kPanel m-blocks, then n-tile, then m-block
// inside the panel.  The CTAs running at once share B tiles through L2, and
// a group with many m-tiles (a popular expert, a shared expert) is swept a
// panel at a time, so the A rows they re-read for every n-tile stay in L2
// too (kPanel m-tiles, instead of all of the group's).  ub[g] = units of the
// groups before g.
struct Tile {
  int g;
  int64_t row0;  // first row of this CTA's m-tile
  int n0;
  bool valid;    // this CTA's m-tile lies inside the group's segment
};

template <int MODE, int CG, int NH = 128>
__device__ __forceinline__ Tile map_tile(int64_t i, const int32_t* offs,
                                         const int64_t* ub, int G, int NT,
                                         uint32_t rank) {
  constexpr int BN_OUT = MODE == 0 ? NH : BN_ACC;
  int lo = 0, hi = G - 1;  // last g with ub[g] <= i
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ub[mid] <= i) lo = mid; else hi = mid - 1;
  }
  const int64_t mtg = (offs[lo + 1] - offs[lo]) / BM;
  const int64_t mbg = (mtg + CG - 1) / CG;
  const int64_t local = i - ub[lo];
  const int64_t panel = local / ((int64_t)kPanel * NT);
  const int64_t p0 = panel * kPanel;                          // first m-block
  const int64_t pw = mbg - p0 < kPanel ? mbg - p0 : kPanel;   // m-blocks in it
  const int64_t in = local - panel * kPanel * NT;
  const int64_t nt = in / pw;
  const int64_t mt = (p0 + in - nt * pw) * CG + rank;
  return Tile{lo, offs[lo] + mt * BM, (int)nt * BN_OUT, mt < mtg};
}

// 16-byte slot q of row r of a transpose tile (see EpiSmem)
__device__ __forceinline__ float4* tslot(float (*t)[32], int r, int q) {
  return reinterpret_cast<float4*>(&t[r][4 * (q ^ (r & 7))]);
}

// The gate activation in the sigmoid form: SiLU(g) = g sigma(g), and the
// tanh approximation of GELU, 0.5 g (1 + tanh(v)) with v = sqrt(2/pi) (g +
// 0.044715 g^3), is g sigma(2v) since 0.5 (1 + tanh(v)) = 1 / (1 + e^-2v).
// Both use the fast exponential and division intrinsics (a few ulp; the
// limits g -> +-inf come out as g and 0).
template <int ACT>
__device__ __forceinline__ float act_fast(float g) {
  if (ACT == MOE_ACT_SILU) return __fdividef(g, 1.0f + __expf(-g));
  const float m2v = -1.5957691216057308f * fmaf(0.044715f * g, g * g, g);  // -2 v
  return __fdividef(g, 1.0f + __expf(m2v));
}

// h of 32 columns of row r: Act(g_j) * u_j into the transpose tile
template <int ACT>
__device__ __forceinline__ void act_row(const float (&g)[32], const float (&u)[32],
                                        float (*t)[32], int r) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *tslot(t, r, q) = make_float4(
        act_fast<ACT>(g[4 * q + 0]) * u[4 * q + 0], act_fast<ACT>(g[4 * q + 1]) * u[4 * q + 1],
        act_fast<ACT>(g[4 * q + 2]) * u[4 * q + 2], act_fast<ACT>(g[4 * q + 3]) * u[4 * q + 3]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// F8: e4m3 operands (tcgen05.mma kind::f8f6f4): a k-block is 128 values of
// one byte, so the shared-memory tiles keep their 128-byte rows.
template <int MODE, int CG, int NH = 128, bool F8 = false>
__global__ void __launch_bounds__(THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmAs,
                    const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmBs, const KParams p) {
  static_assert(NH == 128 || (MODE == 0 && CG == 1 && NH % 8 == 0 && NH < 128),
                "narrow gate tiles are a mode-0, single-CTA form");
  using C = Cfg<CG, NH>;
  constexpr int STAGES = C::STAGES;
  constexpr int B_STAGE = C::B_STAGE;
  constexpr int KBE = F8 ? 2 * BK : BK;  // elements of one k-block (128 bytes)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sA = base;
  const uint32_t sB = base + STAGES * A_STAGE;
  using Epi = EpiSmem<F8>;
  Epi* epi = reinterpret_cast<Epi*>(gbase + STAGES * (A_STAGE + B_STAGE));
  Ctl* ctl = reinterpret_cast<Ctl*>(epi + 1);
  int64_t* ub = reinterpret_cast<int64_t*>(ctl + 1);        // [G+1]
  int32_t* offs = reinterpret_cast<int32_t*>(ub + p.G + 1);  // [G+1]
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const int64_t unit0 = CG == 2 ? (int64_t)cluster_id_x() : (int64_t)blockIdx.x;
  const int64_t unit_step = CG == 2 ? (int64_t)nclusters_x() : (int64_t)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&ctl->tmem_full[a]), 1);
      mbar_init(smem_u32(&ctl->tmem_empty[a]), 4 * CG);  // one per epilogue warp
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort_flag = 0;
    mbar_init_fence();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmAs);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmBs);
  }
  if (warp == 1) {
    if (CG == 2)
      tmem_alloc_pair(smem_u32(&ctl->tmem_base), TMEM_COLS);
    else
      tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
  }
  // everything above overlaps the previous kernel when launched with PDL;
  // the expert offsets and the operands are its outputs
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= p.G; i += THREADS) offs[i] = p.offsets[i];
  __syncthreads();
  if (warp == 0) {
    // units before each group: lane l sums a contiguous run of groups
    const int per = (p.G + 31) / 32;
    const int g0 = lane * per, g1 = min(g0 + per, p.G);
    int64_t run = 0;
    for (int g = g0; g < g1; ++g) {
      const int64_t mtg = (offs[g + 1] - offs[g]) / BM;
      run += (mtg + CG - 1) / CG * p.NT;
    }
    int64_t incl = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t n = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += n;
    }
    int64_t acc = incl - run;
    for (int g = g0; g < g1; ++g) {
      ub[g] = acc;
      const int64_t mtg = (offs[g + 1] - offs[g]) / BM;
      acc += (mtg + CG - 1) / CG * p.NT;
    }
    if (lane == 31) ub[p.G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();  // the peer's barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int64_t total = ub[p.G];

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int32_t last_fill[STAGES];
      for (int s = 0; s < STAGES; ++s) last_fill[s] = -1;
      bool ok = true;
      for (int64_t t = unit0; ok && t < total; t += unit_step) {
        const Tile tl = map_tile<MODE, CG, NH>(t, offs, ub, p.G, p.NT, rank);
        const bool routed = tl.g < p.E;
        const CUtensorMap* mb = routed ? &tmB : &tmBs;
        // a shared expert's segment holds tokens 0..T-1 in order: with
        // a_sh_x its A rows are read from the token rows themselves
        const bool ax = !routed && p.a_sh_x;
        const CUtensorMap* ma = ax ? &tmAs : &tmA;
        const int32_t arow = (int32_t)(ax ? tl.row0 - offs[tl.g] : tl.row0);
        const int32_t gl = routed ? tl.g : tl.g - p.E;
        // B rows this CTA loads: mode 0 -- gate rows then up rows (CG = 1),
        // or CTA 0 the gate rows and CTA 1 the up rows (CG = 2); otherwise
        // 256 rows, or CTA r rows [128r, 128r + 128)
        const int32_t brow = gl * p.b_rows_per_group + tl.n0 +
                             (int32_t)rank * (MODE == 0 ? p.up_off : C::B_ROWS);
        for (int kb = 0; kb < p.KB; ++kb) {
          const uint32_t fb = smem_u32(&ctl->full[stage]);
          if (!mbar_wait(smem_u32(&ctl->empty[stage]), phase ^ 1u, abort_flag,
                         p.timeout_ns, p.err)) {
            ok = false;
            break;
          }
          if (CG == 1) {
            mbar_expect_tx(fb, A_STAGE + B_STAGE);
            tma_load_2d(sA + stage * A_STAGE, ma, kb * KBE, arow, fb);
            if (MODE == 0) {
              tma_load_2d(sB + stage * B_STAGE, mb, kb * KBE, brow, fb);
              tma_load_2d(sB + stage * B_STAGE + B_STAGE / 2, mb, kb * KBE,
                          brow + p.up_off, fb);
            } else {
              tma_load_2d(sB + stage * B_STAGE, mb, kb * KBE, brow, fb);
            }
          } else {
            // both CTAs' bytes complete on CTA 0's full barrier
            if (rank == 0) mbar_expect_tx(fb, 2 * (A_STAGE + B_STAGE));
            const uint32_t fb0 = fb & kPeerBitMask;
            tma_load_2d_pair(sA + stage * A_STAGE, ma, kb * KBE, arow, fb0);
            tma_load_2d_pair(sB + stage * B_STAGE, mb, kb * KBE, brow, fb0);
          }
          last_fill[stage] = (int32_t)phase;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && (CG == 1 || rank == 0)) {
        // let the copies already issued land before the block exits
        int32_t none = 0;
        volatile int32_t* never = &none;
        for (int s = 0; s < STAGES; ++s)
          if (last_fill[s] >= 0)
            mbar_wait(smem_u32(&ctl->full[s]), (uint32_t)last_fill[s], never,
                      p.timeout_ns, p.err);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // (CTA 0 of the pair issues for both when CG = 2)
    if (lane == 0 && (CG == 1 || rank == 0)) {
      constexpr uint32_t idesc =
          F8 ? idesc_e4m3_f32(BM * CG, C::N_MMA) : idesc_bf16_f32(BM * CG, C::N_MMA);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t t = unit0; ok && t < total; t += unit_step) {
        const uint32_t eb = smem_u32(&ctl->tmem_empty[acc]);
        const bool got = CG == 2
            ? mbar_wait_cluster(eb, acc_phase ^ 1u, abort_flag, p.timeout_ns, p.err)
            : mbar_wait(eb, acc_phase ^ 1u, abort_flag, p.timeout_ns, p.err);
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN_ACC;
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!mbar_wait(smem_u32(&ctl->full[stage]), phase, abort_flag,
                         p.timeout_ns, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(sA + stage * A_STAGE);
          const uint64_t bd = sw128_kmajor_desc(sB + stage * B_STAGE);
          // four MMAs of 32 bytes of K each (16 bf16 or 32 e4m3 values)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if (CG == 2)
              umma_pair<F8>(d, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
            else
              umma<F8>(d, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          if (CG == 2)
            umma_commit_pair_mc(smem_u32(&ctl->empty[stage]), 0x3);
          else
            umma_commit(smem_u32(&ctl->empty[stage]));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (CG == 2)
          umma_commit_pair_mc(smem_u32(&ctl->tmem_full[acc]), 0x3);
        else
          umma_commit(smem_u32(&ctl->tmem_full[acc]));
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok || *abort_flag) {
        // wait for the MMAs already issued before TMEM is released
        int32_t none = 0;
        volatile int32_t* never = &none;
        if (CG == 2)
          umma_commit_pair(smem_u32(&ctl->drain));
        else
          umma_commit(smem_u32(&ctl->drain));
        mbar_wait(smem_u32(&ctl->drain), 0, never, p.timeout_ns, p.err);
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // Each warp owns TMEM lanes [32q, 32q+32), i.e. 32 rows of this CTA's
    // m-tile.  Per 32-column chunk it loads its rows' accumulators (one row
    // per lane), parks them in a swizzled 32x32 shared tile and writes them out
    // transposed, so that every store (or reduction) instruction of the warp
    // covers whole 64/128-byte row segments instead of 32 scattered rows.
    const int q = warp & 3;
    float(*tbuf)[32] = epi->buf[q];
    float* cs = epi->cs[F8 ? q : 0];
    const uint32_t empty0 = CG == 2 ? mapa_shared(smem_u32(&ctl->tmem_empty[0]), 0) : 0u;
    const uint32_t empty1 = CG == 2 ? mapa_shared(smem_u32(&ctl->tmem_empty[1]), 0) : 0u;
    uint32_t acc = 0, acc_phase = 0;
    for (int64_t t = unit0; t < total; t += unit_step) {
      const Tile tl = map_tile<MODE, CG, NH>(t, offs, ub, p.G, p.NT, rank);
      const int64_t wrow0 = tl.row0 + q * 32;  // first tile row of this warp
      // FP8: this lane's row scale, and the tile's column scales (the B rows
      // of the group; mode 0: gate row n at n, up row n at N + n)
      float sa = 1.0f;
      if (F8) {
        if (tl.valid) sa = __ldg(p.a_scale + wrow0 + lane);
        const bool routed = tl.g < p.E;
        const float* sb = (routed ? p.b_scale : p.b_scale_sh) +
                          (int64_t)(routed ? tl.g : tl.g - p.E) * (MODE == 0 ? 2 * p.N : p.N);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int i = lane + 32 * m;
          float v = 0.0f;
          if (MODE == 0) {
            const int col = tl.n0 + (i & 127);
            if ((i & 127) < NH && col < p.N) v = __ldg(sb + (i < 128 ? col : p.N + col));
          } else {
            const int col = tl.n0 + i;
            if (col < p.N) v = __ldg(sb + col);
          }
          cs[i] = v;
        }
        __syncwarp();  // every lane reads every column's scale
      }
      if (MODE <= 1) {
        // 1: a real row.  Padding rows (only in a segment's last tile) feed
        // nothing: mode 0 leaves them as they are (-1), mode 1 writes zeros
        // there (0) so that the caller's y_perm holds no stale values
        const bool real = tl.row0 + BM < (int64_t)offs[tl.g + 1] ||
                          (tl.valid && p.sorted_slots[tl.row0 + q * 32 + lane] >= 0);
        epi->rdst[q][lane] = real ? 1 : (MODE == 1 ? 0 : -1);
        epi->rw[q][lane] = sa;  // mode 1 with FP8: the row's scale
      } else {
        // destination row and gate weight of this lane's tile row (with
        // FP8, times the row's scale)
        int64_t dst = -1;
        float wt = 1.0f;
        if (tl.valid) {
          const int64_t row = tl.row0 + q * 32 + lane;
          const int32_t slot = p.sorted_slots[row];
          const int64_t R = p.T * p.k;
          if (slot >= 0) {
            int64_t tok, j;
            if (slot < R) {
              tok = slot / p.k;
              j = slot - tok * p.k;
              wt = __ldg(p.w + slot);
            } else {
              const int64_t qq = slot - R, sh = qq / p.T;
              tok = qq - sh * p.T;
              j = p.k + sh;
            }
            dst = MODE == 2 ? tok : tok * (p.k + p.S) + j;
          }
        }
        epi->rdst[q][lane] = dst;
        epi->rw[q][lane] = F8 ? wt * sa : wt;
      }
      const bool got = mbar_wait(smem_u32(&ctl->tmem_full[acc]), acc_phase,
                                 abort_flag, p.timeout_ns, p.err);
      // warp-uniform decision; also reconverges the warp for tcgen05.ld
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN_ACC;
      constexpr int CHUNKS = MODE == 0 ? (NH + 31) / 32 : 8;
#pragma unroll 1
      for (int c = 0; c < CHUNKS; ++c) {
        const int col0 = tl.n0 + c * 32;
        if (col0 >= p.N) break;
        if (MODE == 0) {
          // gate columns [32c, 32c + 32) and the matching up columns (NH + 32c
          // + j: with NH = 128 the chunk at 128 + 32c; with a narrow tile it
          // straddles the 32-column chunks starting at 32 (NH / 32 + c) and
          // 32 (NH / 32 + c + 1), so every TMEM load starts at a multiple of
          // 32 columns, all of them inside this accumulator's 256)
          float g[32], u[32];
          {
            uint32_t gb[32], ub0[32];
            if (NH == 128) {
              tmem_ld32x2(tb + c * 32, tb + BN_ACC / 2 + c * 32, gb, ub0);
#pragma unroll
              for (int j = 0; j < 32; ++j) u[j] = __uint_as_float(ub0[j]);
            } else {
              constexpr int UQ = NH / 32, UR = NH % 32;
              uint32_t ub1[32];
              tmem_ld32x2(tb + c * 32, tb + (UQ + c) * 32, gb, ub0);
              tmem_ld32(tb + (UQ + c + 1) * 32, ub1);
#pragma unroll
              for (int j = 0; j < 32; ++j)
                u[j] = __uint_as_float(j + UR < 32 ? ub0[j + UR] : ub1[j + UR - 32]);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) g[j] = __uint_as_float(gb[j]);
          }
          if (!tl.valid) continue;  // the pair's empty half: nothing to store
          if (F8) {
            // column scales of the chunk (the same for every lane: broadcast
            // reads), times this lane's row scale
            const float4* cg = reinterpret_cast<const float4*>(cs + c * 32);
            const float4* cu = reinterpret_cast<const float4*>(cs + 128 + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 a = cg[i], b = cu[i];
              g[4 * i + 0] *= sa * a.x;
              g[4 * i + 1] *= sa * a.y;
              g[4 * i + 2] *= sa * a.z;
              g[4 * i + 3] *= sa * a.w;
              u[4 * i + 0] *= sa * b.x;
              u[4 * i + 1] *= sa * b.y;
              u[4 * i + 2] *= sa * b.z;
              u[4 * i + 3] *= sa * b.w;
            }
          }
          if (p.act == MOE_ACT_SILU)
            act_row<MOE_ACT_SILU>(g, u, tbuf, lane);
          else
            act_row<MOE_ACT_GELU_TANH>(g, u, tbuf, lane);
        } else {
          uint32_t y[32];
          tmem_ld32(tb + c * 32, y);
          if (!tl.valid) continue;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *tslot(tbuf, lane, j) =
                make_float4(__uint_as_float(y[4 * j]), __uint_as_float(y[4 * j + 1]),
                            __uint_as_float(y[4 * j + 2]), __uint_as_float(y[4 * j + 3]));
        }
        __syncwarp();
        if (MODE == 0) {
          // 8 rows x 64 bytes per instruction
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
          const int cc = (lane & 3) * 8;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = i * 8 + (lane >> 2);
            const int64_t rd = epi->rdst[q][r];
            if (col0 + cc < p.N && c * 32 + cc < NH && rd > 0) {
              const float4 v0 = *tslot(tbuf, r, cc / 4), v1 = *tslot(tbuf, r, cc / 4 + 1);
              uint4 o;
              o.x = pack_bf16x2(v0.x, v0.y);
              o.y = pack_bf16x2(v0.z, v0.w);
              o.z = pack_bf16x2(v1.x, v1.y);
              o.w = pack_bf16x2(v1.z, v1.w);
              *reinterpret_cast<uint4*>(out + (wrow0 + r) * (int64_t)p.N + col0 + cc) = o;
            }
          }
        } else {
          // 4 rows x 128 bytes per instruction
          float* out = static_cast<float*>(p.out);
          const int cc = (lane & 7) * 4;
          // FP8: the scales of this lane's four columns (the row's scale is
          // folded into rw)
          float4 c4 = make_float4(1.f, 1.f, 1.f, 1.f);
          if (F8) c4 = *reinterpret_cast<const float4*>(cs + c * 32 + cc);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = i * 4 + (lane >> 3);
            if (col0 + cc < p.N) {
              const float4 v = *tslot(tbuf, r, lane & 7);
              float a0 = v.x, a1 = v.y, a2 = v.z, a3 = v.w;
              if (F8) {
                a0 *= c4.x;
                a1 *= c4.y;
                a2 *= c4.z;
                a3 *= c4.w;
              }
              if (MODE == 1) {
                const float rs = F8 ? epi->rw[q][r] : 1.0f;
                *reinterpret_cast<float4*>(out + (wrow0 + r) * (int64_t)p.N + col0 + cc) =
                    epi->rdst[q][r] > 0 ? make_float4(a0 * rs, a1 * rs, a2 * rs, a3 * rs)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
              } else {
                const int64_t dst = epi->rdst[q][r];
                const float wt = epi->rw[q][r];
                if (dst >= 0) {
                  float* d = out + dst * (int64_t)p.N + col0 + cc;
                  const float b0 = __fmul_rn(wt, a0), b1 = __fmul_rn(wt, a1);
                  const float b2 = __fmul_rn(wt, a2), b3 = __fmul_rn(wt, a3);
                  if (MODE == 2)
                    red_add_v4(d, b0, b1, b2, b3);
                  else
                    *reinterpret_cast<float4*>(d) = make_float4(b0, b1, b2, b3);
                }
              }
            }
          }
        }
        __syncwarp();
      }
      // this warp is done with the accumulator: one arrival per warp (on
      // CTA 0's barrier when the pair shares the MMA)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2)
          mbar_arrive_cluster(acc ? empty1 : empty0);
        else
          mbar_arrive(smem_u32(&ctl->tmem_empty[acc]));
      }
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();  // no peer still uses this CTA's barriers or TMEM
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if (CG == 2)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                  void*, const cuuint64_t*, const cuuint64_t*,
                                  const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [outer, inner] row-major tensor of bf16 (box {64, box_rows}) or of e4m3
// bytes (f8: box {128, box_rows}); rows of 128 bytes, 128-byte swizzle.
cudaError_t make_map(CUtensorMap* m, const void* ptr, uint64_t inner,
                     uint64_t outer, uint32_t box_rows, bool f8 = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * (f8 ? 1 : 2)};
  const cuuint32_t box[2] = {(cuuint32_t)(f8 ? 2 * BK : BK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                         const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// SMs of the current device (cached per device)
int num_sms() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < kMaxDevices;
  int n = cached ? cache[dev].load() : 0;
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n <= 0)
      n = 148;
    if (cached) cache[dev].store(n);
  }
  return n;
}

template <int MODE, int CG, int NH = 128, bool F8 = false>
cudaError_t launch_mode(const GroupedGemmArgs& a, cudaStream_t st, bool pdl) {
  using C = Cfg<CG, NH>;
  constexpr int BN_OUT = MODE == 0 ? NH : BN_ACC;
  constexpr int KBE = F8 ? 2 * BK : BK;
  CUtensorMap mA, mAs, mB, mBs;
  cudaError_t e = make_map(&mA, a.A, (uint64_t)a.K, (uint64_t)a.cap, BM, F8);
  if (e != cudaSuccess) return e;
  const bool a_sh_x = a.A_sh != nullptr && a.G > a.E && a.T > 0;
  if (a_sh_x) {
    e = make_map(&mAs, a.A_sh, (uint64_t)a.K, (uint64_t)a.T, BM, F8);
    if (e != cudaSuccess) return e;
  } else {
    mAs = mA;
  }
  const uint64_t rows_per_group = MODE == 0 ? 2ull * a.N : (uint64_t)a.N;
  // per-CTA B box: mode 0 loads NH gate (and NH up) rows; the others 256
  // rows, or 128 per CTA of a pair
  const uint32_t box_rows = MODE == 0 ? NH : (uint32_t)C::B_ROWS;
  e = make_map(&mB, a.B, (uint64_t)a.K, rows_per_group * (uint64_t)a.E, box_rows, F8);
  if (e != cudaSuccess) return e;
  if (a.B_sh && a.G > a.E) {
    e = make_map(&mBs, a.B_sh, (uint64_t)a.K,
                 rows_per_group * (uint64_t)(a.G - a.E), box_rows, F8);
    if (e != cudaSuccess) return e;
  } else {
    mBs = mB;
  }
  KParams p;
  p.offsets = a.offsets;
  p.G = a.G;
  p.E = a.E;
  p.N = a.N;
  p.K = a.K;
  p.NT = (a.N + BN_OUT - 1) / BN_OUT;
  p.KB = (a.K + KBE - 1) / KBE;
  p.b_rows_per_group = (int32_t)rows_per_group;
  p.up_off = MODE == 0 ? a.N : 0;
  p.out = a.out;
  p.act = a.act;
  p.err = a.err;
  p.timeout_ns = kTimeoutNs;
  p.sorted_slots = a.sorted_slots;
  p.w = a.w;
  p.T = a.T;
  p.k = a.k;
  p.S = a.G - a.E;
  p.a_sh_x = a_sh_x ? 1 : 0;
  p.a_scale = a.a_scale;
  p.b_scale = a.b_scale;
  p.b_scale_sh = a.b_scale_sh;

  const size_t smem = 1024 + (size_t)C::STAGES * (A_STAGE + C::B_STAGE) +
                      sizeof(EpiSmem<F8>) + sizeof(Ctl) +
                      (sizeof(int64_t) + sizeof(int32_t)) * (size_t)(a.G + 1);
  // the shared-memory opt-in is a per-device attribute: set it once on
  // every device this process launches on
  static std::atomic<bool> attr_set[kMaxDevices];
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices || !attr_set[dev].load()) {
    e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, CG, NH, F8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) attr_set[dev].store(true);
  }
  // units: at most (cap / BM) m-tiles, grouped CG at a time, per n-tile
  const int64_t max_units = ((a.cap / BM) / CG + a.G) * p.NT;
  int64_t groups = num_sms() / CG;  // CTAs (or CTA pairs) resident at once
  if (max_units < groups) groups = max_units > 0 ? max_units : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(groups * CG));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (CG == 2) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<MODE, CG, NH, F8>, mA, mAs, mB, mBs, p);
}

__global__ void wait_selftest_kernel(uint32_t* err, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  // nothing ever arrives on ``bar``: the bounded wait must give up
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, timeout_ns, err);
}

}  // namespace

cudaError_t launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t st, bool pdl) {
  // CTA pairs when the experts' segments are large enough that most m-blocks
  // hold two full m-tiles; single CTAs for few rows per expert (decode-sized)
  const bool pair = a.pair;
  // w13 with I a multiple of 88 but not of 128 (I = 704): 176-row B tiles
  // cover the gate and up halves exactly, so no weight row is streamed for
  // nothing.  Only below the ridge point (under 256 rows per expert, where
  // the product is bound by streaming the weights): measured on B200, an
  // N = 176 MMA costs the tensor-bound many-small batch 10 % on w13, and
  // saves 5-7 % of the step at 16-256 tokens.
  const int64_t rows = a.T * a.k + a.T * (int64_t)(a.G - a.E);
  const bool narrow = a.N % 128 != 0 && a.N % 88 == 0 && rows < 256 * (int64_t)a.G;
  if (a.f8) {
    switch (a.mode) {
      case 0:
        return pair ? launch_mode<0, 2, 128, true>(a, st, pdl)
               : narrow ? launch_mode<0, 1, 88, true>(a, st, pdl)
                        : launch_mode<0, 1, 128, true>(a, st, pdl);
      case 1:
        return pair ? launch_mode<1, 2, 128, true>(a, st, pdl)
                    : launch_mode<1, 1, 128, true>(a, st, pdl);
      case 2:
        return pair ? launch_mode<2, 2, 128, true>(a, st, pdl)
                    : launch_mode<2, 1, 128, true>(a, st, pdl);
      case 3:
        return pair ? launch_mode<3, 2, 128, true>(a, st, pdl)
                    : launch_mode<3, 1, 128, true>(a, st, pdl);
    }
    return cudaErrorInvalidValue;
  }
  switch (a.mode) {
    case 0:
      return pair ? launch_mode<0, 2>(a, st, pdl)
                  : narrow ? launch_mode<0, 1, 88>(a, st, pdl) : launch_mode<0, 1>(a, st, pdl);
    case 1: return pair ? launch_mode<1, 2>(a, st, pdl) : launch_mode<1, 1>(a, st, pdl);
    case 2: return pair ? launch_mode<2, 2>(a, st, pdl) : launch_mode<2, 1>(a, st, pdl);
    case 3: return pair ? launch_mode<3, 2>(a, st, pdl) : launch_mode<3, 1>(a, st, pdl);
  }
  return cudaErrorInvalidValue;
}

cudaError_t make_tma_map_bf16(CUtensorMap* m, const void* ptr, uint64_t inner,
                              uint64_t outer, uint32_t box_rows) {
  return make_map(m, ptr, inner, outer, box_rows);
}

cudaError_t make_tma_map_e4m3(CUtensorMap* m, const void* ptr, uint64_t inner,
                              uint64_t outer, uint32_t box_rows) {
  return make_map(m, ptr, inner, outer, box_rows, /*f8=*/true);
}

int device_sm_count() { return num_sms(); }

cudaError_t launch_wait_selftest(uint32_t* err, uint32_t timeout_us,
                                 cudaStream_t st) {
  return launch_ex(wait_selftest_kernel, dim3(1), dim3(32), 0, st, false, err,
                   (uint64_t)timeout_us * 1000ull);
}

}  // namespace moe
