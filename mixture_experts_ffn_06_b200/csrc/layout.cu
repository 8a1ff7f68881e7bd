// layout.cu -- the dispatch permutation and the activation gather.
//
// The Gemma 4 MoE walkthrough (yeyulingfeng.com/587419.html, sections 6-7)
// describes FusedMoE's dispatch as a "permutation map" that turns
// "each token picked k experts" into "each expert received a token list",
// without moving tokens; the pages leave the map itself open.  Here it is a
// stable counting sort of the flat slots s = t*k + j by expert, each expert
// segment padded to a multiple of 128 rows (the GEMM M tile), with the
// always-active shared experts (llama-cpp-visual-guide lesson 35) appended
// as segments that hold every token.
//
// Three launches, all integer work, coalesced:
//   layout_count   one block per 1024 slots: stable rank of every slot among
//                  the equal-expert slots of its block (warp match + per-warp
//                  counts) and the block histogram;
//   layout_scan    one block: per-expert exclusive scan over blocks, padded
//                  segment sizes and their exclusive scan -> offsets;
//   layout_scatter every slot writes sorted_slots[row] and slot_row;
//   layout_pad     padding rows and rows past the last segment get -1.
// gather_rows then copies x[token] into x_perm[row] with 16-byte vector
// loads, one warp per row, and zeroes the fp32 accumulator of the fast
// combine.  Padding rows are skipped: an MMA row depends on its own A row
// alone, so they only ever feed padding rows of h and y, which are never
// read (with few tokens per expert most rows are padding, and writing zeros
// there cost the decode-sized batches about 9% on B200).
#include "internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(kLayoutTile)
layout_count(const int32_t* __restrict__ ids, int64_t R, int E,
             int32_t* __restrict__ lt_count, int32_t* __restrict__ lt_rank) {
  extern __shared__ int32_t wc[];  // [32 warps][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_trigger();
  for (int i = tid; i < 32 * E; i += blockDim.x) wc[i] = 0;
  __syncthreads();

  const int64_t s = (int64_t)blockIdx.x * kLayoutTile + tid;
  const int e = (s < R) ? __ldg(ids + s) : -1;
  const bool valid = (e >= 0 && e < E);
  const int key = valid ? e : -1;
  const uint32_t peers = __match_any_sync(0xffffffffu, key);
  const uint32_t lower = peers & ((1u << lane) - 1u);
  const int rank_in_warp = __popc(lower);
  if (valid && lower == 0) wc[warp * E + e] = __popc(peers);
  __syncthreads();

  if (valid) {
    int base = 0;
    for (int w2 = 0; w2 < warp; ++w2) base += wc[w2 * E + e];
    lt_rank[s] = base + rank_in_warp;
  }
  for (int x = tid; x < E; x += blockDim.x) {
    int c = 0;
    for (int w2 = 0; w2 < 32; ++w2) c += wc[w2 * E + x];
    lt_count[(int64_t)blockIdx.x * E + x] = c;
  }
}

__global__ void __launch_bounds__(1024)
layout_scan(const int32_t* __restrict__ lt_count, int64_t n_lt, int E, int S,
            int64_t T, int P, int32_t* __restrict__ lt_base,
            int32_t* __restrict__ offsets) {
  __shared__ int32_t seg[kMaxExperts + kMaxShared + 1];
  __shared__ int32_t warp_sum[32];
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const int G = E + S;
  // per-expert running sum over layout blocks; the counts of 8 blocks are
  // requested before the first is added (one round trip per 8 blocks)
  for (int e = tid; e < G; e += blockDim.x) {
    int64_t total = 0;
    if (e < E) {
      int64_t b = 0;
      for (; b + 8 <= n_lt; b += 8) {
        int32_t c[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) c[q] = lt_count[(b + q) * E + e];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          lt_base[(b + q) * E + e] = (int32_t)total;
          total += c[q];
        }
      }
      for (; b < n_lt; ++b) {
        lt_base[b * E + e] = (int32_t)total;
        total += lt_count[b * E + e];
      }
    } else {
      total = T;
    }
    seg[e] = (int32_t)((total + P - 1) / P * P);
  }
  __syncthreads();
  // exclusive scan of seg[0..G) (G <= 520 < 1024: one element per thread)
  const int lane = tid & 31, warp = tid >> 5;
  int v = (tid < G) ? seg[tid] : 0;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += n;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int ws = warp_sum[lane];
    int wincl = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wincl, off);
      if (lane >= off) wincl += n;
    }
    warp_sum[lane] = wincl - ws;  // exclusive
  }
  __syncthreads();
  const int excl = incl - v + warp_sum[warp];
  if (tid < G) offsets[tid] = excl;
  if (tid == G - 1) offsets[G] = excl + v;
}

// Index space: [0,R) routed slots, then [R, R+T*S) shared-expert slots.
// A routed slot whose id lies outside [0,E) (a caller's bad input to
// moe_permute) is given no row: layout_count did not count it, its slot_row
// entry is set to -1, and the error word (when given) records
// MOE_ERR_INVALID_ARG.
__global__ void __launch_bounds__(256)
layout_scatter(const int32_t* __restrict__ ids, int64_t T, int k, int E, int S,
               const int32_t* __restrict__ offsets,
               const int32_t* __restrict__ lt_base,
               const int32_t* __restrict__ lt_rank,
               int32_t* __restrict__ sorted_slots,
               int32_t* __restrict__ slot_row, uint32_t* err) {
  const int64_t R = T * k, RS = T * S;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  pdl_wait();
  pdl_trigger();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < R + RS;
       i += stride) {
    if (i < R) {
      const int e = ids[i];
      if (e < 0 || e >= E) {
        const int64_t t = i / k;
        slot_row[t * (k + S) + (i - t * k)] = -1;
        record_error(err, MOE_ERR_INVALID_ARG);
        continue;
      }
      const int64_t b = i / kLayoutTile;
      const int64_t row = (int64_t)offsets[e] + lt_base[b * E + e] + lt_rank[i];
      sorted_slots[row] = (int32_t)i;
      const int64_t t = i / k, j = i - t * k;
      slot_row[t * (k + S) + j] = (int32_t)row;
    } else {
      const int64_t q = i - R, s = q / T, t = q - s * T;
      const int64_t row = (int64_t)offsets[E + s] + t;
      sorted_slots[row] = (int32_t)(R + q);
      slot_row[t * (k + S) + k + s] = (int32_t)row;
    }
  }
}

// Padding rows: block g < G clears segment g's tail (its slots fill rows
// [offsets[g], offsets[g] + count_g); the rest up to offsets[g+1] get -1);
// the blocks past G clear the rows from offsets[G] to cap.
__global__ void __launch_bounds__(256)
layout_pad(const int32_t* __restrict__ offsets, const int32_t* __restrict__ lt_base,
           const int32_t* __restrict__ lt_count, int64_t n_lt, int E, int S,
           int64_t T, int P, int64_t cap, int32_t* __restrict__ sorted_slots) {
  const int G = E + S;
  const int g = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (g < G) {
    int64_t count;
    if (g < E) {
      count = (n_lt > 0) ? (int64_t)lt_base[(n_lt - 1) * E + g] +
                               lt_count[(n_lt - 1) * E + g]
                         : 0;
    } else {
      count = T;
    }
    const int64_t beg = offsets[g] + count, end = offsets[g + 1];
    for (int64_t r = beg + threadIdx.x; r < end; r += blockDim.x)
      sorted_slots[r] = -1;
  } else {
    // rows past offsets[G]
    const int64_t used = offsets[G];
    const int64_t stride = (int64_t)(gridDim.x - G) * blockDim.x;
    for (int64_t r = used + (int64_t)(g - G) * blockDim.x + threadIdx.x; r < cap;
         r += stride)
      sorted_slots[r] = -1;
  }
}

__global__ void __launch_bounds__(256, 4)
gather_rows(const uint4* __restrict__ x, const int32_t* __restrict__ sorted_slots,
            const int32_t* __restrict__ offsets, int G, int64_t T, int k,
            int H, uint4* __restrict__ x_perm, uint4* __restrict__ acc,
            int64_t n_acc4) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  pdl_wait();
  pdl_trigger();
  const int64_t rows = offsets[G];
  const int chunks = H >> 3;  // 8 bf16 per 16-byte chunk
  const int64_t R = T * k;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += warps) {
    const int s = sorted_slots[r];
    uint4* dst = x_perm + r * chunks;
    if (s < 0) continue;
    const int64_t t = (s < R) ? (int64_t)s / k : ((int64_t)s - R) % T;
    const uint4* src = x + t * chunks;
    // up to eight 16-byte loads in flight per lane before the stores (a
    // 5.6 KB row in two rounds); the copies are written with the streaming
    // hint so they do not push x (read k times) out of L2
    for (int c0 = 0; c0 < chunks; c0 += 256) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c0 + lane + 32 * j < chunks) v[j] = __ldg(src + c0 + lane + 32 * j);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c0 + lane + 32 * j < chunks) __stcs(dst + c0 + lane + 32 * j, v[j]);
    }
  }
  // zero the fp32 accumulator the w2 epilogue adds into (fast combine)
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_acc4;
       i += stride)
    acc[i] = z;
}

}  // namespace

cudaError_t launch_layout(const moe_shape& s, const int32_t* ids,
                          int32_t* offsets, int32_t* sorted_slots,
                          int32_t* slot_row, int64_t cap, int32_t* lt_count,
                          int32_t* lt_base, int32_t* lt_rank, int64_t n_lt,
                          uint32_t* err, cudaStream_t st, bool pdl) {
  const int64_t R = s.T * s.k;
  const int E = s.E, S = s.n_shared, G = E + S;
  const int P = s.pad ? s.pad : kSegPad;
  cudaError_t e;
  bool chained = pdl;  // every launch after the first is a dependent
  if (R > 0) {
    const size_t smem = sizeof(int32_t) * 32 * (size_t)E;
    if (smem > 48 * 1024) {
      e = cudaFuncSetAttribute(layout_count, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e != cudaSuccess) return e;
    }
    e = launch_ex(layout_count, dim3((unsigned)n_lt), dim3(kLayoutTile), smem, st,
                  chained, ids, R, E, lt_count, lt_rank);
    if (e != cudaSuccess) return e;
    chained = true;
  }
  e = launch_ex(layout_scan, dim3(1), dim3(1024), 0, st, chained,
                (const int32_t*)lt_count, R > 0 ? n_lt : (int64_t)0, E, S, s.T, P,
                lt_base, offsets);
  if (e != cudaSuccess) return e;
  const int64_t work = R + s.T * S;
  if (work > 0) {
    const int64_t blocks = (work + 255) / 256;
    e = launch_ex(layout_scatter,
                  dim3((unsigned)(blocks < 65535 * 16 ? blocks : 65535 * 16)),
                  dim3(256), 0, st, true, ids, s.T, s.k, E, S,
                  (const int32_t*)offsets, (const int32_t*)lt_base,
                  (const int32_t*)lt_rank, sorted_slots, slot_row, err);
    if (e != cudaSuccess) return e;
  }
  e = launch_ex(layout_pad, dim3((unsigned)(G + 148)), dim3(256), 0, st, true,
                (const int32_t*)offsets, (const int32_t*)lt_base,
                (const int32_t*)lt_count, R > 0 ? n_lt : (int64_t)0, E, S, s.T, P,
                cap, sorted_slots);
  return e;
}

cudaError_t launch_gather(const __nv_bfloat16* x, const int32_t* sorted_slots,
                          const int32_t* offsets, int G, int64_t T, int k,
                          int H, int64_t cap, __nv_bfloat16* x_perm, float* acc,
                          int64_t n_acc, cudaStream_t st, bool pdl) {
  const int64_t want = (cap + 7) / 8;
  const unsigned blocks = (unsigned)(want < 148 * 16 ? want : 148 * 16);
  return launch_ex(gather_rows, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st, pdl,
                   reinterpret_cast<const uint4*>(x), sorted_slots, offsets, G, T, k,
                   H, reinterpret_cast<uint4*>(x_perm), reinterpret_cast<uint4*>(acc),
                   acc ? n_acc / 4 : (int64_t)0);
}

}  // namespace moe
