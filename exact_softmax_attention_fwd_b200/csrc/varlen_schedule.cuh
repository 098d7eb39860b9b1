// varlen_schedule.cuh -- work list for prefill over a ragged batch.
//
// "Attention Kernel", section "Paged 与 ragged KV": a ragged batch is described
// by cumulative sequence lengths instead of being padded into a rectangle.
// The prefill kernel's work unit is (sequence b, 256-row query block qb, query
// head); this kernel lists the (b, qb) pairs so that the persistent prefill
// kernel can deal them out heaviest first: query blocks in descending qb
// (under a causal mask a block's KV work grows with its index), sequences of
// the same qb in arbitrary order.  The order only affects which CTA computes a
// unit, never its result, so the output stays bitwise deterministic.
//
// One CTA of 1024 threads, a counting sort by qb:
//   cnt[L]  = number of sequences whose last query block is L
//   c[L]    = number of sequences with more than L blocks   (suffix sum of cnt)
//   off[L]  = first list position of level L = sum of c over levels above L
// then each (b, L) takes position off[L] + atomicAdd(cursor[L], 1).
// A sequence whose offsets decrease, leave [0, total] or exceed max_seqlen_q
// is left out and flagged (ATTN_DEVERR_BAD_LENGTH).
#pragma once

#include "sm100_primitives.cuh"

namespace attn_b200 {

constexpr int kVarlenMaxLevels = 8192;  // max_seqlen_q <= 2^21

// Query blocks of sequence b, or 0 (flagged) when its offsets are not valid.
__device__ __forceinline__ int varlen_seq_blocks(const int* cu_q, const int* cu_k, int b,
                                                 int total_q, int total_k, int max_seqlen_q) {
  const int q0 = cu_q[b], q1 = cu_q[b + 1], k0 = cu_k[b], k1 = cu_k[b + 1];
  const bool bad = q0 < 0 || q1 < q0 || q1 > total_q || k0 < 0 || k1 < k0 || k1 > total_k ||
                   q1 - q0 > max_seqlen_q;
  if (bad) {
    flag_device_error(kDevErrBadLength);
    return 0;
  }
  return (q1 - q0 + 255) / 256;
}

// a[0..n) := suffix sums of a (inclusive, or exclusive when `exclusive`),
// computed by all 1024 threads of the block.  `warp_sums` holds 32 ints.
__device__ __forceinline__ void block_suffix_sum(int* a, int n, bool exclusive, int* warp_sums) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int chunk = (n + 1023) / 1024;
  const int lo = min(t * chunk, n), hi = min(lo + chunk, n);
  int local = 0;
  for (int L = lo; L < hi; ++L) local += a[L];
  // inclusive suffix over the lanes of this warp
  int v = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int x = __shfl_down_sync(0xffffffffu, v, off);
    if (lane + off < 32) v += x;
  }
  if (lane == 0) warp_sums[w] = v;  // this warp's total
  __syncthreads();
  if (w == 0) {
    int ws = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int x = __shfl_down_sync(0xffffffffu, ws, off);
      if (lane + off < 32) ws += x;
    }
    warp_sums[lane] = ws;  // suffix over warps, inclusive
  }
  __syncthreads();
  // sum of the chunks of all threads after this one
  int run = v - local + (w + 1 < 32 ? warp_sums[w + 1] : 0);
  __syncthreads();  // warp_sums is reused by the next call
  for (int L = hi - 1; L >= lo; --L) {
    const int x = a[L];
    run += x;
    a[L] = exclusive ? run - x : run;
  }
  __syncthreads();
}

// Writes unit_count and units[0 .. unit_count) (at most max_units entries).
__global__ void __launch_bounds__(1024, 1)
    attn_varlen_schedule_kernel(const int* cu_q, const int* cu_k, int B, int total_q, int total_k,
                                int max_seqlen_q, int2* units, int* unit_count, int max_units) {
  extern __shared__ int sh[];
  const int n_levels = (max_seqlen_q + 255) / 256;
  int* lev = sh;                // cnt, then c, then off / cursors
  int* cnt_copy = sh + n_levels;  // c kept for the total
  int* warp_sums = sh + 2 * n_levels;
  for (int L = threadIdx.x; L < n_levels; L += blockDim.x) lev[L] = 0;
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int nqb = varlen_seq_blocks(cu_q, cu_k, b, total_q, total_k, max_seqlen_q);
    if (nqb > 0) atomicAdd(&lev[nqb - 1], 1);
  }
  __syncthreads();
  block_suffix_sum(lev, n_levels, false, warp_sums);  // lev[L] = c[L]
  for (int L = threadIdx.x; L < n_levels; L += blockDim.x) cnt_copy[L] = lev[L];
  __syncthreads();
  block_suffix_sum(lev, n_levels, true, warp_sums);   // lev[L] = off[L]
  if (threadIdx.x == 0) {
    const long long total = (long long)lev[0] + cnt_copy[0];  // off[0] + c[0]
    if (total > max_units) flag_device_error(kDevErrBadLength);  // overlapping ranges
    *unit_count = (int)(total < max_units ? total : max_units);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int nqb = varlen_seq_blocks(cu_q, cu_k, b, total_q, total_k, max_seqlen_q);
    for (int L = 0; L < nqb; ++L) {
      const int pos = atomicAdd(&lev[L], 1);
      if (pos < max_units) units[pos] = make_int2(b, L);
    }
  }
}

}  // namespace attn_b200
