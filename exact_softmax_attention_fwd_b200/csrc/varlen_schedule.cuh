// varlen_schedule.cuh -- work list for prefill over a ragged batch.
//
// "Attention Kernel", section "Paged 与 ragged KV": a ragged batch is described
// by cumulative sequence lengths instead of being padded into a rectangle.
// The prefill kernel's work unit is (sequence b, 256-row query block qb, query
// head); this kernel lists the (b, qb) pairs so that the persistent prefill
// kernel can deal them out heaviest first.  A unit's weight is the number of
// 128-key tiles its two query tiles visit (the kernel's own visibility rule),
// so that long and short sequences, square prefill and appends to a long
// cache are all ordered by the work they carry.  Units of equal weight come in
// arbitrary order; the order only decides which CTA computes a unit, never its
// result, so the output stays bitwise deterministic.
//
// One CTA of 1024 threads, a counting sort by weight level
// (level = weight >> shift, at most kVarlenMaxLevels levels):
//   cnt[L]  = number of units of level L
//   off[L]  = first list position of level L = number of units above level L
// then each unit takes position off[L] + atomicAdd(cursor[L], 1).
// A sequence whose offsets decrease, leave [0, total] or exceed max_seqlen_q
// (or, over a paged cache, whose key length exceeds the block table) is left
// out and flagged (ATTN_DEVERR_BAD_LENGTH).
#pragma once

#include "prefill_sm100.cuh"
#include "sm100_primitives.cuh"

namespace attn_b200 {

constexpr int kVarlenMaxLevels = 8192;  // counting-sort levels (shared memory: 2 ints each)

// Query rows and keys of sequence b, or false (flagged) when its offsets are
// not valid.
// Keys come either as packed ranges (cu_k) or, for a paged cache, as lengths
// (seq_lens_k, at most max_keys = the block table's capacity).
__device__ __forceinline__ bool varlen_seq_lengths(const int* cu_q, const int* cu_k,
                                                   const int* seq_lens_k, int b, int total_q,
                                                   int total_k, int max_seqlen_q, int max_keys,
                                                   int& len_q, int& len_k) {
  const int q0 = cu_q[b], q1 = cu_q[b + 1];
  bool bad = q0 < 0 || q1 < q0 || q1 > total_q || q1 - q0 > max_seqlen_q;
  if (cu_k != nullptr) {
    const int k0 = cu_k[b], k1 = cu_k[b + 1];
    bad = bad || k0 < 0 || k1 < k0 || k1 > total_k;
    len_k = k1 - k0;
  } else {
    len_k = seq_lens_k[b];
    bad = bad || len_k < 0 || len_k > max_keys;
  }
  len_q = q1 - q0;
  if (bad) flag_device_error(kDevErrBadLength);
  return !bad;
}

// 128-key tiles the two query tiles of block qb visit (prefill_kv_range).
__device__ __forceinline__ int varlen_unit_weight(int qb, int len_q, int len_k, bool causal,
                                                  int window, int prefix) {
  int w = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    int lo, hi;
    prefill_kv_range(qb * 256 + i * 128, len_q, len_k, causal, window, prefix, lo, hi);
    w += hi - lo;
  }
  return w;
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
    attn_varlen_schedule_kernel(const int* cu_q, const int* cu_k, const int* seq_lens_k, int B,
                                int total_q, int total_k, int max_seqlen_q, int max_keys,
                                int causal, int window, int prefix, int level_shift,
                                int n_levels, int2* units,
                                int* unit_count, int max_units) {
  extern __shared__ int sh[];
  int* lev = sh;                  // counts, then first positions / cursors
  int* cnt_copy = sh + n_levels;  // counts kept for the total
  int* warp_sums = sh + 2 * n_levels;
  for (int L = threadIdx.x; L < n_levels; L += blockDim.x) lev[L] = 0;
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    int lq, lk;
    if (!varlen_seq_lengths(cu_q, cu_k, seq_lens_k, b, total_q, total_k, max_seqlen_q, max_keys,
                            lq, lk))
      continue;
    for (int qb = 0; qb * 256 < lq; ++qb) {
      const int L = min(varlen_unit_weight(qb, lq, lk, causal != 0, window, prefix) >> level_shift, n_levels - 1);
      atomicAdd(&lev[L], 1);
    }
  }
  __syncthreads();
  for (int L = threadIdx.x; L < n_levels; L += blockDim.x) cnt_copy[L] = lev[L];
  __syncthreads();
  block_suffix_sum(lev, n_levels, true, warp_sums);  // lev[L] = units above level L
  if (threadIdx.x == 0) {
    const long long total = (long long)lev[0] + cnt_copy[0];
    if (total > max_units) flag_device_error(kDevErrBadLength);  // overlapping ranges
    *unit_count = (int)(total < max_units ? total : max_units);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    int lq, lk;
    if (!varlen_seq_lengths(cu_q, cu_k, seq_lens_k, b, total_q, total_k, max_seqlen_q, max_keys,
                            lq, lk))
      continue;
    for (int qb = 0; qb * 256 < lq; ++qb) {
      const int L = min(varlen_unit_weight(qb, lq, lk, causal != 0, window, prefix) >> level_shift, n_levels - 1);
      const int pos = atomicAdd(&lev[L], 1);
      if (pos < max_units) units[pos] = make_int2(b, qb);
    }
  }
}

// Counting-sort levels for weights up to 2 * ceil(max_keys / 128): the shift
// that keeps them within kVarlenMaxLevels, and the level count.
inline void varlen_levels(long long max_keys, int& shift, int& n_levels) {
  const long long max_weight = 2 * ((max_keys + 127) / 128);
  shift = 0;
  while ((max_weight >> shift) + 1 > kVarlenMaxLevels) ++shift;
  n_levels = (int)(max_weight >> shift) + 1;
}

}  // namespace attn_b200
