// bwd_sm100.cuh -- exact softmax attention backward for sm_100a.
//
// What it computes ("Attention Kernel", section "Backward 与重计算"): the
// forward keeps no probability matrix, so the backward recomputes the local
// probabilities from Q, K, the output O and the saved log-sum-exp, with the
// forward's scale, mask and GQA head mapping:
//     P  = exp(scale * Q K^T + M - LSE)          (row by row)
//     dV = P^T dO          dP = dO V^T           D = rowsum(dO * O)
//     dS = P * (dP - D)    dQ = scale * dS K     dK = scale * dS^T Q
// ("Attention 算子加速史", FAQ Q1: recomputation trades FLOPs for HBM traffic.)
// D = rowsum(dO * O) equals rowsum(P * dP) because O = P V.
//
// Three kernels, each output written by exactly one CTA, so results are
// deterministic and no atomics are used (the contract in "Backward 与重计算"
// asks that accumulation and writes be free of races):
//   * attn_bwd_prep_kernel: per query row, D and -LSE*log2(e) into a workspace
//     padded to whole 128-row tiles (padding rows get -inf and 0, so they
//     recompute P = 0 without a predicate).
//   * attn_bwd_dkdv_kernel: one CTA per (key tile, batch, KV head).  K and V
//     stay in shared memory; Q, dO and their row statistics stream through a
//     ring for every query head of the group and every query tile that sees
//     the key tile.  Per query tile, four tcgen05 MMAs with the key tile as M:
//       S^T = K Q^T, dP^T = V dO^T     (SS: both operands in shared memory)
//       dV += P^T dO, dK += dS^T Q     (TS: P^T / dS^T read from tensor memory)
//     so the transposed products land with keys on the TMEM lanes and need no
//     transpose.  dV and dK accumulate in tensor memory across the whole loop.
//     The S^T columns are released as soon as the recompute warps have read
//     them, and P^T and dS^T both go into the dP^T columns, so the next tile's
//     S^T runs on the tensor cores while this tile's P^T is computed.
//   * attn_bwd_dq_kernel: one CTA per (query tile, batch, query head), K/V
//     tiles streaming: S = Q K^T, dP = dO V^T (SS), dQ += dS K (TS).
// Both compute kernels use the forward's organisation: warp 0 lane 0 issues
// TMA copies (no multicast), warp 1 lane 0 issues the MMAs, and two
// warpgroups (warps 4-7, 8-11) each own 64 of the 128 columns of every score
// tile (thread r owns TMEM lane r).  A warpgroup packs its bf16 operands into
// its own 64-column range (32 columns each: dS, and in the dK/dV kernel P
// after it), so the two warpgroups never write a column the other still has to
// read; the TS MMAs read an operand from the two warpgroups' 32-column runs.
#pragma once

#include "sm100_primitives.cuh"

namespace attn_b200 {

// 1-D bulk copy global -> shared (cp.async.bulk, no tensor map); completion is
// counted in bytes on the mbarrier.  Both addresses 16-byte aligned, size a
// multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

struct BwdParams {
  const uint16_t* o;    // [B, Hq, Sq, d] forward output (bf16)
  const uint16_t* d_o;  // [B, Hq, Sq, d] gradient of the output (bf16)
  const float* lse;     // [B, Hq, Sq] forward log-sum-exp (natural log)
  float* nlse2;         // [B*Hq, Sq_pad] workspace: -LSE*log2(e); -inf for empty and padding rows
  float* dsum;          // [B*Hq, Sq_pad] workspace: rowsum(dO * O); 0 for padding rows
  const int* k_lens;    // [B] or nullptr
  uint16_t* dq;         // [B, Hq, Sq, d]
  uint16_t* dk;         // [B, Hkv, Sk, d]
  uint16_t* dv;         // [B, Hkv, Sk, d]
  int B, Hq, Hkv, Sq, Sk, group, Sq_pad, n_qt, n_kt;
  float scale, scale_log2;
  // ragged batches (VARLEN instantiations): q, o, dO, dQ packed [total_q, Hq, d],
  // k, v, dK, dV packed [total_k, Hkv, d], LSE [Hq, total_q]; Sq / Sk are the
  // largest query / key lengths the call allows (max_seqlen_q / _k)
  const int* cu_q;      // [B + 1]
  const int* cu_k;      // [B + 1]
  int total_q, total_k;
  // programmable masks (MASKS instantiations, fixed-length batches): sliding
  // window / prefix-LM (causal only, 0 = off) and a uint8 block mask
  // [B, mask_heads, n_qt, n_kt] over 128 x 128 blocks (nullable), as the forward's
  int window, prefix;
  const uint8_t* block_mask;
  int mask_heads;
};

// Whether the 128 x 128 block (query tile qt, key tile kt) of query head hq is
// switched on by the block mask (always, without one).
__device__ __forceinline__ bool bwd_block_on(const BwdParams& p, int b, int hq, int qt, int kt) {
  if (p.block_mask == nullptr) return true;
  const size_t h = p.mask_heads == 1 ? 0 : (size_t)hq;
  return __ldg(p.block_mask + (((size_t)b * p.mask_heads + h) * p.n_qt + qt) * p.n_kt + kt) != 0;
}

// Block-sparse backward: the candidate iterations [0, n) whose block is on,
// listed in ascending order by all threads of the CTA (flags first, then one
// warp compacts them with ballots), so that every role walks the same list.
// The caller's next __syncthreads publishes list[0, *count).
template <typename On>
__device__ __forceinline__ void bwd_list_blocks(int n, On on, uint16_t* list, uint8_t* flag,
                                                int* count) {
  for (int c = threadIdx.x; c < n; c += blockDim.x) flag[c] = on(c) ? 1 : 0;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int cnt = 0;
    for (int base = 0; base < n; base += 32) {
      const int c = base + lane;
      const bool keep = c < n && flag[c] != 0;
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) list[cnt + __popc(m & ((1u << lane) - 1u))] = (uint16_t)c;
      cnt += __popc(m);
    }
    if (lane == 0) *count = cnt;
  }
}

// One sequence of a backward call: query rows [q0, q0 + lq) and keys
// [k0, k0 + lk) of the packed tensors (fixed-length batches: q0 = k0 = 0,
// lq = Sq, lk = the clamped key length).  False when a ragged sequence's
// offsets are not valid (decreasing, outside the tensors, or longer than the
// call's maxima): nothing of it is computed or written, and it is flagged.
struct BwdSeq {
  int q0, lq, k0, lk;
};

template <bool VARLEN>
__device__ __forceinline__ bool bwd_sequence(const BwdParams& p, int b, bool report, BwdSeq& s) {
  if (!VARLEN) {
    s.q0 = s.k0 = 0;
    s.lq = p.Sq;
    int kl = p.k_lens == nullptr ? p.Sk : __ldg(p.k_lens + b);
    if (kl < 0 || kl > p.Sk) {
      if (report) flag_device_error(kDevErrBadLength);
      kl = kl < 0 ? 0 : p.Sk;
    }
    s.lk = kl;
    return true;
  }
  const int qa = __ldg(p.cu_q + b), qb = __ldg(p.cu_q + b + 1);
  const int ka = __ldg(p.cu_k + b), kb = __ldg(p.cu_k + b + 1);
  if (qa < 0 || qb < qa || qb > p.total_q || ka < 0 || kb < ka || kb > p.total_k ||
      qb - qa > p.Sq || kb - ka > p.Sk) {
    if (report) flag_device_error(kDevErrBadLength);
    s.q0 = s.lq = s.k0 = s.lk = 0;
    return false;
  }
  s.q0 = qa;
  s.lq = qb - qa;
  s.k0 = ka;
  s.lk = kb - ka;
  return true;
}

template <int D>
struct BwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;  // a 128-row bf16 tile (Q, dO, K or V)
  static constexpr int CB_BYTES = 128 * 128;      // one 64-column block of a tile
  static constexpr int NCB = D / 64;
  static constexpr int STAGES = (D == 64) ? 4 : 2;
  static constexpr int STAT_BYTES = 1024;  // -LSE*log2(e) [128] then D [128] of a query tile
  // ---- dK/dV kernel: K, V resident; Q, dO and statistics in a ring
  static constexpr int KV_OFF_K = 0;
  static constexpr int KV_OFF_V = TILE_BYTES;
  static constexpr int KV_OFF_Q = 2 * TILE_BYTES;
  static constexpr int KV_OFF_DO = KV_OFF_Q + STAGES * TILE_BYTES;
  static constexpr int KV_OFF_ST = KV_OFF_DO + STAGES * TILE_BYTES;
  static constexpr int KV_OFF_BAR = KV_OFF_ST + STAGES * STAT_BYTES;
  static constexpr int KB_KV = 0;                  // K and V landed
  static constexpr int KB_QF = 1;                  // STAGES: Q, dO, statistics landed
  static constexpr int KB_QE = KB_QF + STAGES;     // STAGES: stage free (MMA + 256 threads)
  static constexpr int KB_SF = KB_QE + STAGES;     // S^T in TMEM
  static constexpr int KB_SE = KB_SF + 1;          // S^T read by the recompute warps (256)
  static constexpr int KB_DPF = KB_SE + 1;         // dP^T in TMEM
  static constexpr int KB_PDS = KB_DPF + 1;        // P^T and dS^T written (256 threads)
  static constexpr int KB_ACC = KB_PDS + 1;        // every MMA retired
  static constexpr int KB_NUM = KB_ACC + 1;
  static constexpr int KV_OFF_MISC = KV_OFF_BAR + KB_NUM * 8;
  static constexpr int KV_SMEM = KV_OFF_MISC + 16 + 1024;
  // block masks: the iterations a CTA keeps, listed as uint16 ids, then one
  // flag byte per candidate (masked instantiations only)
  static constexpr int LIST_MAX = 4096;
  static constexpr int KV_OFF_LIST = KV_OFF_MISC + 16;
  static constexpr int KV_SMEM_MASKS = KV_SMEM + 3 * LIST_MAX;
  // ---- dQ kernel: Q, dO resident; K, V in a ring
  static constexpr int Q_OFF_Q = 0;
  static constexpr int Q_OFF_DO = TILE_BYTES;
  static constexpr int Q_OFF_K = 2 * TILE_BYTES;
  static constexpr int Q_OFF_V = Q_OFF_K + STAGES * TILE_BYTES;
  static constexpr int Q_OFF_BAR = Q_OFF_V + STAGES * TILE_BYTES;
  static constexpr int QB_QF = 0;                  // Q and dO landed
  static constexpr int QB_KVF = 1;                 // STAGES: K and V landed
  static constexpr int QB_KVE = QB_KVF + STAGES;   // STAGES: stage free
  static constexpr int QB_SF = QB_KVE + STAGES;    // 2: S in TMEM buffer 0 / 1
  static constexpr int QB_DPF = QB_SF + 2;         // dP in TMEM
  static constexpr int QB_DSF = QB_DPF + 1;        // dS written (256 threads)
  static constexpr int QB_ACC = QB_DSF + 1;
  static constexpr int QB_NUM = QB_ACC + 1;
  static constexpr int Q_OFF_MISC = Q_OFF_BAR + QB_NUM * 8;
  static constexpr int Q_SMEM = Q_OFF_MISC + 16 + 1024;
  static constexpr int Q_OFF_LIST = Q_OFF_MISC + 16;
  static constexpr int Q_SMEM_MASKS = Q_SMEM + 3 * LIST_MAX;
  // ---- tensor memory (512 columns)
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t KV_TM_S = 0;        // S^T
  static constexpr uint32_t KV_TM_DP = 128;     // dP^T, then dS^T and P^T (bf16)
  static constexpr uint32_t KV_TM_DV = 256;
  static constexpr uint32_t KV_TM_DK = 256 + D;
  static constexpr uint32_t Q_TM_S0 = 0, Q_TM_S1 = 128;
  static constexpr uint32_t Q_TM_DP = 256;      // dP, then dS (bf16)
  static constexpr uint32_t Q_TM_DQ = 384;
  static constexpr int NUM_THREADS = 384;
  static constexpr uint32_t REGS_PRODUCER = 88;
  static constexpr uint32_t REGS_SOFTMAX = 192;
  static_assert(128 * (REGS_PRODUCER + 2 * REGS_SOFTMAX) <= NUM_THREADS * 168,
                "register reallocation must fit the launch allocation");
  static_assert(KV_SMEM_MASKS <= 232448 && Q_SMEM_MASKS <= 232448, "shared memory");
  static_assert(D == 64 || D == 128, "head dim");
};

// -inf for a masked element, x otherwise.
__device__ __forceinline__ float bwd_keep(bool visible, float x) {
  return visible ? x : -INFINITY;
}

// D = rowsum(dO * O) and -LSE*log2(e) for every padded query row.  D/8
// threads per row, 8 elements each, reduced by shuffles.
template <int D, bool VARLEN>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const BwdParams p) {
  constexpr int TPR = D / 8;
  const long long n_rows = (long long)p.B * p.Hq * p.Sq_pad;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gt / TPR;
  const int part = (int)(gt % TPR);
  const bool valid = row < n_rows;
  const long long bh = valid ? row / p.Sq_pad : 0;
  const int i = valid ? (int)(row % p.Sq_pad) : 0;
  BwdSeq sq;
  const int b = (int)(bh / p.Hq), h = (int)(bh % p.Hq);
  const bool seq_ok = valid && bwd_sequence<VARLEN>(p, b, false, sq);
  const bool live = seq_ok && i < sq.lq;
  // dense: [B*Hq, Sq] rows; ragged: token q0 + i of head h in [total_q, Hq]
  const size_t row_el = VARLEN ? ((size_t)(sq.q0 + i) * p.Hq + h) : ((size_t)bh * p.Sq + i);
  const size_t lse_at = VARLEN ? ((size_t)h * p.total_q + sq.q0 + i) : ((size_t)bh * p.Sq + i);
  float acc = 0.f;
  if (live) {
    const size_t off = row_el * D + part * 8;
    const uint4 a = ld_stream_v4(p.d_o + off);
    const uint4 b = ld_stream_v4(p.o + off);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(bw[e] << 16), acc);
      acc = fmaf(__uint_as_float(aw[e] & 0xFFFF0000u), __uint_as_float(bw[e] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int w = TPR / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
  if (valid && part == 0) {
    float nl = -INFINITY;
    if (live) {
      const float l = p.lse[lse_at];
      nl = (l == -INFINITY) ? -INFINITY : -l * 1.4426950408889634f;
    }
    p.nlse2[row] = nl;
    p.dsum[row] = live ? acc : 0.f;
  }
}

// SS MMA over the head dimension: D[tm] = A B^T, A and B 128-row K-major tiles.
template <int D>
__device__ __forceinline__ void bwd_mma_ss(uint32_t d_tmem, uint32_t a, uint32_t b) {
  using C = BwdCfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint32_t off = (ks >> 2) * C::CB_BYTES + (ks & 3) * 32;
    umma_ss(d_tmem, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024), idesc,
            ks > 0 ? 1u : 0u);
  }
}

// TS MMA over 128 rows: D[tm] (+)= A B with A [128 x 128] bf16 in TMEM (its
// columns 0-31 and 64-95: the two warpgroups' packed runs) and B a 128-row tile
// used MN-major (its rows are the reduction index).
template <int D>
__device__ __forceinline__ void bwd_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b,
                                           bool accumulate) {
  using C = BwdCfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, true);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    umma_ts(d_tmem, a_tmem + (ks >> 2) * 64 + (ks & 3) * 8,
            smem_desc_sw128(b + ks * 2048, C::CB_BYTES, 1024), idesc,
            (accumulate || ks > 0) ? 1u : 0u);
  }
}

// Writes 32 fp32 values (times mul) as bf16 to a global row segment (16-byte stores).
__device__ __forceinline__ void bwd_store32(uint16_t* dst, const uint32_t (&v)[32], float mul) {
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    uint4 w;
    w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * mul, __uint_as_float(v[8 * q4 + 1]) * mul);
    w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * mul, __uint_as_float(v[8 * q4 + 3]) * mul);
    w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * mul, __uint_as_float(v[8 * q4 + 5]) * mul);
    w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * mul, __uint_as_float(v[8 * q4 + 7]) * mul);
    reinterpret_cast<uint4*>(dst)[q4] = w;
  }
}

// ===========================================================================
// dK, dV: one CTA per (key tile kb, batch b, KV head).  Units are numbered key
// tile major, so under a causal mask the heaviest key tiles (the first ones,
// seen by the most query tiles) start first.
// ===========================================================================
template <int D, bool CAUSAL, bool VARLEN, bool MASKS>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const BwdParams p) {
  using C = BwdCfg<D>;
  // the dQ grid does not read what this grid writes: it may be launched as
  // soon as every CTA here has started, and fill the SMs this grid's tail
  // leaves idle
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sbase_ptr = smem_raw + (sbase - raw_addr);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase_ptr + C::KV_OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase_ptr + C::KV_OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return sbase + C::KV_OFF_BAR + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- the unit and its query-tile range
  const int bh_kv = blockIdx.x % (p.B * p.Hkv);
  const int kb = blockIdx.x / (p.B * p.Hkv);
  const int b = bh_kv / p.Hkv, kvh = bh_kv % p.Hkv;
  BwdSeq sq;
  const bool seq_ok = bwd_sequence<VARLEN>(p, b, threadIdx.x == 0 && kb == 0 && kvh == 0, sq);
  const int klen = seq_ok ? sq.lk : 0;
  const long long koff = (long long)klen - sq.lq;  // key j is visible to row i iff j <= i + koff
  const int key0 = kb * 128;
  const int n_qt = VARLEN ? (sq.lq + 127) / 128 : p.n_qt;  // this sequence's query tiles
  int qt_lo = 0, qt_hi = n_qt;
  if (CAUSAL) {
    const long long first_row = (long long)key0 - koff;  // the first row that sees key0
    qt_lo = first_row <= 0 ? 0 : (int)min(first_row / 128, (long long)n_qt);
  }
  if (MASKS) {
    const long long key1 = min((long long)key0 + 127, (long long)klen - 1);
    // prefix keys are seen by every row; a window hides the tile from rows
    // at or past key1 + window - koff
    if (p.prefix > 0 && key0 < min(p.prefix, klen)) qt_lo = 0;
    if (p.window > 0) {
      const long long row_end = key1 + p.window - koff;
      qt_hi = row_end <= 0 ? 0 : (int)min((row_end + 127) / 128, (long long)n_qt);
    }
  }
  const int nq = (!seq_ok || key0 >= klen || qt_hi <= qt_lo) ? 0 : qt_hi - qt_lo;
  const int N = p.group * nq;  // (query head, query tile) candidates
  // with a block mask, only the candidates whose block is on are walked
  const bool listed = MASKS && p.block_mask != nullptr && N > 0 && N <= C::LIST_MAX;
  const uint16_t* list = reinterpret_cast<const uint16_t*>(sbase_ptr + C::KV_OFF_LIST);
  int* list_count = reinterpret_cast<int*>(sbase_ptr + C::KV_OFF_MISC + 8);
  if (listed)
    bwd_list_blocks(
        N, [&](int c) { return bwd_block_on(p, b, kvh * p.group + c / nq, qt_lo + c % nq, kb); },
        reinterpret_cast<uint16_t*>(sbase_ptr + C::KV_OFF_LIST),
        sbase_ptr + C::KV_OFF_LIST + 2 * C::LIST_MAX, list_count);
  // dK/dV rows this CTA writes: a ragged sequence's own keys only (rows past
  // them belong to the next sequence); fixed-length batches write every key
  // row of the tile (padded keys get zeros)
  const int key_rows = VARLEN ? (seq_ok ? sq.lk : 0) : p.Sk;

  if (threadIdx.x == 0) {
    mbar_init(bar(C::KB_KV), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(C::KB_QF + s), 1);
      mbar_init(bar(C::KB_QE + s), 1 + 256);
    }
    mbar_init(bar(C::KB_SF), 1);
    mbar_init(bar(C::KB_SE), 256);
    mbar_init(bar(C::KB_DPF), 1);
    mbar_init(bar(C::KB_PDS), 256);
    mbar_init(bar(C::KB_ACC), 1);
    *abort_flag = 0;
    mbar_init_fence();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int NI = listed ? *list_count : N;  // iterations walked
  auto cand = [&](int n) { return listed ? (int)list[n] : n; };
  const uint32_t sK = sbase + C::KV_OFF_K, sV = sbase + C::KV_OFF_V;
  auto sQ = [&](int s) { return sbase + C::KV_OFF_Q + (uint32_t)s * C::TILE_BYTES; };
  auto sDO = [&](int s) { return sbase + C::KV_OFF_DO + (uint32_t)s * C::TILE_BYTES; };
  auto sST = [&](int s) { return sbase + C::KV_OFF_ST + (uint32_t)s * C::STAT_BYTES; };

  if (warp < 4) {
    warpgroup_reg_dealloc<C::REGS_PRODUCER>();
    if (warp == 0 && lane == 0 && NI > 0) {
      // ======================= TMA producer =======================
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_do);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      mbar_arrive_expect_tx(bar(C::KB_KV), 2 * C::TILE_BYTES);
      // fixed-length maps are (d, S, B*H); ragged ones (d, H, tokens)
      for (int cb = 0; cb < C::NCB; ++cb) {
        tma_load_3d(sK + cb * C::CB_BYTES, &tm_k, bar(C::KB_KV), 64 * cb, VARLEN ? kvh : key0,
                    VARLEN ? sq.k0 + key0 : bh_kv);
        tma_load_3d(sV + cb * C::CB_BYTES, &tm_v, bar(C::KB_KV), 64 * cb, VARLEN ? kvh : key0,
                    VARLEN ? sq.k0 + key0 : bh_kv);
      }
      int issued = 0;
      bool ok = true;
      for (int n = 0; n < NI; ++n) {
        const int s = n % C::STAGES;
        if (n >= C::STAGES &&
            !(ok = mbar_wait(bar(C::KB_QE + s), ((n / C::STAGES) - 1) & 1u, abort_flag)))
          break;
        const int c = cand(n);
        const int hq = kvh * p.group + c / nq;
        const int qt = qt_lo + c % nq;
        const int bh_q = b * p.Hq + hq;
        mbar_arrive_expect_tx(bar(C::KB_QF + s), 2 * C::TILE_BYTES + C::STAT_BYTES);
        const int qy = VARLEN ? hq : qt * 128, qz = VARLEN ? sq.q0 + qt * 128 : bh_q;
        for (int cb = 0; cb < C::NCB; ++cb) {
          tma_load_3d(sQ(s) + cb * C::CB_BYTES, &tm_q, bar(C::KB_QF + s), 64 * cb, qy, qz);
          tma_load_3d(sDO(s) + cb * C::CB_BYTES, &tm_do, bar(C::KB_QF + s), 64 * cb, qy, qz);
        }
        const size_t srow = (size_t)bh_q * p.Sq_pad + (size_t)qt * 128;
        bulk_load(sST(s), p.nlse2 + srow, 512, bar(C::KB_QF + s));
        bulk_load(sST(s) + 512, p.dsum + srow, 512, bar(C::KB_QF + s));
        ++issued;
      }
      // Drain: no copy may still be landing when the CTA exits.
      mbar_wait(bar(C::KB_KV), 0, nullptr);
      for (int n = (issued > C::STAGES ? issued - C::STAGES : 0); n < issued; ++n)
        mbar_wait(bar(C::KB_QF + n % C::STAGES), (n / C::STAGES) & 1u, nullptr);
    } else if (warp == 1 && lane == 0 && NI > 0) {
      // ======================= tcgen05 MMA issuer =======================
      const uint32_t tS = tmem + C::KV_TM_S, tDP = tmem + C::KV_TM_DP;
      const uint32_t tDV = tmem + C::KV_TM_DV, tDK = tmem + C::KV_TM_DK;
      bool ok = mbar_wait(bar(C::KB_KV), 0, abort_flag) && mbar_wait(bar(C::KB_QF), 0, abort_flag);
      if (ok) {
        tc_fence_after_sync();
        bwd_mma_ss<D>(tS, sK, sQ(0));
        umma_commit(bar(C::KB_SF));
        bwd_mma_ss<D>(tDP, sV, sDO(0));
        umma_commit(bar(C::KB_DPF));
      }
      for (int n = 0; ok && n < NI; ++n) {
        const int s = n % C::STAGES, s1 = (n + 1) % C::STAGES;
        if (n + 1 < NI) {
          // S^T of the next query tile, as soon as this tile's S^T has been read
          if (!(ok = mbar_wait(bar(C::KB_SE), n & 1u, abort_flag))) break;
          if (!(ok = mbar_wait(bar(C::KB_QF + s1), ((n + 1) / C::STAGES) & 1u, abort_flag))) break;
          tc_fence_after_sync();
          bwd_mma_ss<D>(tS, sK, sQ(s1));
          umma_commit(bar(C::KB_SF));
        }
        if (!(ok = mbar_wait(bar(C::KB_PDS), n & 1u, abort_flag))) break;
        tc_fence_after_sync();
        bwd_mma_ts<D>(tDV, tDP + 32, sDO(s), n > 0);  // dV += P^T dO
        bwd_mma_ts<D>(tDK, tDP, sQ(s), n > 0);        // dK += dS^T Q
        umma_commit(bar(C::KB_QE + s));  // Q and dO of stage s read for the last time
        if (n + 1 < NI) {
          // dP^T of the next tile overwrites P^T and dS^T only after the two MMAs
          // above read them (MMAs of one thread run in issue order)
          bwd_mma_ss<D>(tDP, sV, sDO(s1));
          umma_commit(bar(C::KB_DPF));
        }
      }
      // every MMA retires before the epilogue reads TMEM and before TMEM is freed
      umma_commit(bar(C::KB_ACC));
      mbar_wait(bar(C::KB_ACC), 0, nullptr);
    }
    __syncwarp();
  } else {
    warpgroup_reg_alloc<C::REGS_SOFTMAX>();
    // ======================= recompute warpgroups =======================
    const int wg = (warp - 4) >> 2;      // query columns [64*wg, 64*wg + 64) of each tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // key row within the tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int c0 = 64 * wg;
    const uint32_t t_s = tmem + lane_off + C::KV_TM_S + c0;
    const uint32_t t_dp = tmem + lane_off + C::KV_TM_DP + c0;
    const int j = key0 + r;
    const float c2 = p.scale_log2;
    const uint64_t c2x2 = f32x2(c2, c2);
    bool ok = true;
    for (int n = 0; ok && n < NI; ++n) {
      const int s = n % C::STAGES;
      const int cn = cand(n);
      const int qt = qt_lo + cn % nq;
      // columns c >= cmin are visible to this key (c relative to this warpgroup's run)
      long long cm = (j >= klen) ? 64 : (CAUSAL ? (long long)j - koff - qt * 128 - c0 : 0);
      long long cx = 64;  // columns [cmin, cmax) are visible to this key
      if (MASKS) {
        if (p.window > 0 && j < klen) cx = (long long)j + p.window - koff - qt * 128 - c0;
        if (p.prefix > 0 && j < p.prefix && j < klen) {
          cm = 0;
          cx = 64;
        }
        if (!bwd_block_on(p, b, kvh * p.group + cn / nq, qt, kb)) cm = 64;
      }
      const int cmin = (int)(cm < 0 ? 0 : (cm > 64 ? 64 : cm));
      const int cmax = MASKS ? (int)(cx < 0 ? 0 : (cx > 64 ? 64 : cx)) : 64;
      const bool edge = __any_sync(0xffffffffu, cmin > 0 || cmax < 64);
      if (!(ok = mbar_wait_warp(bar(C::KB_SF), n & 1u, abort_flag))) break;
      tc_fence_after_sync();
      float pr[64];
      uint32_t pk_p[32];
      {
        uint32_t a[32], bq[32];
        tmem_ld32(t_s, a);
        tmem_ld32(t_s + 32, bq);
        tmem_ld_wait();
        reg_fence32(a);
        reg_fence32(bq);
        tc_fence_before_sync();
        mbar_arrive(bar(C::KB_SE));  // S^T read: the next tile's S^T may overwrite it
        // the statistics arrived with Q (every thread observes the copy itself)
        const bool st_ok = mbar_wait(bar(C::KB_QF + s), (n / C::STAGES) & 1u, abort_flag);
        if (!(ok = __all_sync(0xffffffffu, st_ok))) break;
        const float4* st = reinterpret_cast<const float4*>(sbase_ptr + C::KV_OFF_ST +
                                                           s * C::STAT_BYTES);
#pragma unroll
        for (int e = 0; e < 16; ++e) {  // columns 4e .. 4e+3
          const float4 nl = st[(c0 >> 2) + e];
          const int c = 4 * e;
          const uint32_t s0 = c < 32 ? a[c] : bq[c - 32];
          const uint32_t s1 = c < 32 ? a[c + 1] : bq[c - 31];
          const uint32_t s2 = c < 32 ? a[c + 2] : bq[c - 30];
          const uint32_t s3 = c < 32 ? a[c + 3] : bq[c - 29];
          float x0, x1, x2, x3;
          split_f32x2(fma_f32x2(f32x2(__uint_as_float(s0), __uint_as_float(s1)), c2x2,
                                f32x2(nl.x, nl.y)), x0, x1);
          split_f32x2(fma_f32x2(f32x2(__uint_as_float(s2), __uint_as_float(s3)), c2x2,
                                f32x2(nl.z, nl.w)), x2, x3);
          if (edge) {
            x0 = bwd_keep(c >= cmin && c < cmax, x0);
            x1 = bwd_keep(c + 1 >= cmin && c + 1 < cmax, x1);
            x2 = bwd_keep(c + 2 >= cmin && c + 2 < cmax, x2);
            x3 = bwd_keep(c + 3 >= cmin && c + 3 < cmax, x3);
          }
          pr[c] = ex2(x0);
          pr[c + 1] = ex2(x1);
          pr[c + 2] = ex2(x2);
          pr[c + 3] = ex2(x3);
          pk_p[2 * e] = pack_bf16x2(pr[c], pr[c + 1]);
          pk_p[2 * e + 1] = pack_bf16x2(pr[c + 2], pr[c + 3]);
        }
      }
      if (!(ok = mbar_wait_warp(bar(C::KB_DPF), n & 1u, abort_flag))) break;
      tc_fence_after_sync();
      {
        const float4* st = reinterpret_cast<const float4*>(sbase_ptr + C::KV_OFF_ST +
                                                           s * C::STAT_BYTES);
        uint32_t pk[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // dP^T columns [32h, 32h + 32) of this warpgroup's run
          uint32_t a[32];
          tmem_ld32(t_dp + 32 * h, a);
          tmem_ld_wait();
          reg_fence32(a);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 dd = st[32 + (c0 >> 2) + 8 * h + e];  // D of columns 32h + 4e ..
            const int c = 32 * h + 4 * e;
            const float d0 = __uint_as_float(a[4 * e]) - dd.x;
            const float d1 = __uint_as_float(a[4 * e + 1]) - dd.y;
            const float d2 = __uint_as_float(a[4 * e + 2]) - dd.z;
            const float d3 = __uint_as_float(a[4 * e + 3]) - dd.w;
            pk[16 * h + 2 * e] = pack_bf16x2(pr[c] * d0, pr[c + 1] * d1);
            pk[16 * h + 2 * e + 1] = pack_bf16x2(pr[c + 2] * d2, pr[c + 3] * d3);
          }
        }
        // dS^T then P^T into this warpgroup's 64 dP^T columns (all read above)
        tmem_st32(t_dp, pk);
        tmem_st32(t_dp + 32, pk_p);
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(bar(C::KB_PDS));
      }
      mbar_arrive(bar(C::KB_QE + s));  // this thread is done with stage s's statistics
    }
    // ---- epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (times scale)
    bool have = NI > 0;
    if (have && ok) {
      ok = mbar_wait_warp(bar(C::KB_ACC), 0, abort_flag);
      tc_fence_after_sync();
    }
    if ((!have || ok) && key0 < key_rows) {
      const uint32_t t_acc = tmem + lane_off + (wg ? C::KV_TM_DK : C::KV_TM_DV);
      const int jj = j < key_rows ? j : 0;
      uint16_t* out = (wg ? p.dk : p.dv) +
                      (VARLEN ? ((size_t)(sq.k0 + jj) * p.Hkv + kvh) : ((size_t)bh_kv * p.Sk + jj)) * D;
      const float mul = wg ? p.scale : 1.f;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t v[32];
        if (have) {
          tmem_ld32_sync(t_acc + c, v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        if (j < key_rows) bwd_store32(out + c, v, mul);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ===========================================================================
// dQ: one CTA per (query tile, batch, query head).  Units are numbered query
// tile major from the last tile down, so under a causal mask the heaviest
// tiles start first.
// ===========================================================================
template <int D, bool CAUSAL, bool VARLEN, bool MASKS>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sbase_ptr = smem_raw + (sbase - raw_addr);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase_ptr + C::Q_OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase_ptr + C::Q_OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return sbase + C::Q_OFF_BAR + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int bh_q = blockIdx.x % (p.B * p.Hq);
  const int qt = p.n_qt - 1 - (int)(blockIdx.x / (p.B * p.Hq));
  const int b = bh_q / p.Hq, hq = bh_q % p.Hq;
  const int kvh = hq / p.group;
  const int bh_kv = b * p.Hkv + kvh;
  BwdSeq sq;
  const bool seq_ok = bwd_sequence<VARLEN>(p, b, threadIdx.x == 0, sq);
  const int klen = seq_ok ? sq.lk : 0;
  const int n_rows = seq_ok ? sq.lq : 0;  // dQ rows of this sequence
  const long long koff = (long long)klen - sq.lq;
  const int row0 = qt * 128;
  const int last_row = min(row0 + 127, n_rows - 1);
  long long max_key = (long long)klen - 1;  // the last key any row of the tile sees
  if (CAUSAL)
    max_key = min(max_key, max((long long)last_row + koff, MASKS ? (long long)p.prefix - 1 : -1LL));
  // the first key tile any row sees (a sliding window starts it past 0)
  int kt_lo = 0;
  if (MASKS && p.window > 0) {
    const long long min_key = (long long)row0 + koff - p.window + 1;
    kt_lo = min_key <= 0 ? 0 : (int)(min_key / 128);
  }
  // key tiles [kt_lo, kt_lo + N); none for a tile past the sequence's rows
  const int kt_end = max_key < 0 ? 0 : (int)(max_key / 128) + 1;
  const int N = (row0 >= n_rows || kt_end <= kt_lo) ? 0 : kt_end - kt_lo;
  // with a block mask, only the key tiles whose block is on are walked
  const bool listed = MASKS && p.block_mask != nullptr && N > 0 && N <= C::LIST_MAX;
  const uint16_t* list = reinterpret_cast<const uint16_t*>(sbase_ptr + C::Q_OFF_LIST);
  int* list_count = reinterpret_cast<int*>(sbase_ptr + C::Q_OFF_MISC + 8);
  if (listed)
    bwd_list_blocks(
        N, [&](int c) { return bwd_block_on(p, b, hq, qt, kt_lo + c); },
        reinterpret_cast<uint16_t*>(sbase_ptr + C::Q_OFF_LIST),
        sbase_ptr + C::Q_OFF_LIST + 2 * C::LIST_MAX, list_count);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::QB_QF), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(C::QB_KVF + s), 1);
      mbar_init(bar(C::QB_KVE + s), 1);
    }
    mbar_init(bar(C::QB_SF), 1);
    mbar_init(bar(C::QB_SF + 1), 1);
    mbar_init(bar(C::QB_DPF), 1);
    mbar_init(bar(C::QB_DSF), 256);
    mbar_init(bar(C::QB_ACC), 1);
    *abort_flag = 0;
    mbar_init_fence();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int NI = listed ? *list_count : N;  // key tiles walked
  auto cand = [&](int n) { return listed ? (int)list[n] : n; };
  const uint32_t sQ = sbase + C::Q_OFF_Q, sDO = sbase + C::Q_OFF_DO;
  auto sK = [&](int s) { return sbase + C::Q_OFF_K + (uint32_t)s * C::TILE_BYTES; };
  auto sV = [&](int s) { return sbase + C::Q_OFF_V + (uint32_t)s * C::TILE_BYTES; };

  if (warp < 4) {
    warpgroup_reg_dealloc<C::REGS_PRODUCER>();
    if (warp == 0 && lane == 0 && NI > 0) {
      // ======================= TMA producer =======================
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_do);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      mbar_arrive_expect_tx(bar(C::QB_QF), 2 * C::TILE_BYTES);
      const int qy = VARLEN ? hq : row0, qz = VARLEN ? sq.q0 + row0 : bh_q;
      for (int cb = 0; cb < C::NCB; ++cb) {
        tma_load_3d(sQ + cb * C::CB_BYTES, &tm_q, bar(C::QB_QF), 64 * cb, qy, qz);
        tma_load_3d(sDO + cb * C::CB_BYTES, &tm_do, bar(C::QB_QF), 64 * cb, qy, qz);
      }
      int issued = 0;
      bool ok = true;
      for (int n = 0; n < NI; ++n) {
        const int s = n % C::STAGES;
        if (n >= C::STAGES &&
            !(ok = mbar_wait(bar(C::QB_KVE + s), ((n / C::STAGES) - 1) & 1u, abort_flag)))
          break;
        mbar_arrive_expect_tx(bar(C::QB_KVF + s), 2 * C::TILE_BYTES);
        const int kt = kt_lo + cand(n);
        const int ky = VARLEN ? kvh : kt * 128, kz = VARLEN ? sq.k0 + kt * 128 : bh_kv;
        for (int cb = 0; cb < C::NCB; ++cb) {
          tma_load_3d(sK(s) + cb * C::CB_BYTES, &tm_k, bar(C::QB_KVF + s), 64 * cb, ky, kz);
          tma_load_3d(sV(s) + cb * C::CB_BYTES, &tm_v, bar(C::QB_KVF + s), 64 * cb, ky, kz);
        }
        ++issued;
      }
      mbar_wait(bar(C::QB_QF), 0, nullptr);
      for (int n = (issued > C::STAGES ? issued - C::STAGES : 0); n < issued; ++n)
        mbar_wait(bar(C::QB_KVF + n % C::STAGES), (n / C::STAGES) & 1u, nullptr);
    } else if (warp == 1 && lane == 0 && NI > 0) {
      // ======================= tcgen05 MMA issuer =======================
      const uint32_t tDP = tmem + C::Q_TM_DP, tDQ = tmem + C::Q_TM_DQ;
      auto tS = [&](int n) { return tmem + ((n & 1) ? C::Q_TM_S1 : C::Q_TM_S0); };
      bool ok = mbar_wait(bar(C::QB_QF), 0, abort_flag) && mbar_wait(bar(C::QB_KVF), 0, abort_flag);
      if (ok) {
        tc_fence_after_sync();
        bwd_mma_ss<D>(tS(0), sQ, sK(0));
        umma_commit(bar(C::QB_SF));
        bwd_mma_ss<D>(tDP, sDO, sV(0));
        umma_commit(bar(C::QB_DPF));
      }
      for (int n = 0; ok && n < NI; ++n) {
        const int s = n % C::STAGES, s1 = (n + 1) % C::STAGES;
        if (n + 1 < NI) {
          if (!(ok = mbar_wait(bar(C::QB_KVF + s1), ((n + 1) / C::STAGES) & 1u, abort_flag))) break;
          tc_fence_after_sync();
          bwd_mma_ss<D>(tS(n + 1), sQ, sK(s1));
          umma_commit(bar(C::QB_SF + ((n + 1) & 1)));
        }
        if (!(ok = mbar_wait(bar(C::QB_DSF), n & 1u, abort_flag))) break;
        tc_fence_after_sync();
        bwd_mma_ts<D>(tDQ, tDP, sK(s), n > 0);  // dQ += dS K
        umma_commit(bar(C::QB_KVE + s));
        if (n + 1 < NI) {
          // dP of the next key tile: overwrites dS only after the MMA above read it
          bwd_mma_ss<D>(tDP, sDO, sV(s1));
          umma_commit(bar(C::QB_DPF));
        }
      }
      umma_commit(bar(C::QB_ACC));
      mbar_wait(bar(C::QB_ACC), 0, nullptr);
    }
    __syncwarp();
  } else {
    warpgroup_reg_alloc<C::REGS_SOFTMAX>();
    // ======================= recompute warpgroups =======================
    const int wg = (warp - 4) >> 2;      // key columns [64*wg, 64*wg + 64) of each tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // query row within the tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int c0 = 64 * wg;
    const uint32_t t_dp = tmem + lane_off + C::Q_TM_DP + c0;
    const int row = row0 + r;
    const size_t srow = (size_t)bh_q * p.Sq_pad + row;
    const float nl = p.nlse2[srow];
    const float dd = p.dsum[srow];
    const uint64_t c2x2 = f32x2(p.scale_log2, p.scale_log2);
    const uint64_t nlx2 = f32x2(nl, nl);
    // keys klo <= j < kend are visible to this row
    long long kend = klen, klo = 0;
    if (CAUSAL)
      kend = min(kend, max((long long)row + koff, MASKS ? (long long)p.prefix - 1 : -1LL) + 1);
    if (MASKS && p.window > 0) klo = max(0LL, (long long)row + koff - p.window + 1);
    bool ok = true;
    for (int n = 0; ok && n < NI; ++n) {
      const int kt = kt_lo + cand(n);
      const long long t0 = (long long)kt * 128 + c0;  // this run's first key
      long long cm = kend - t0;  // visible iff cmin <= c < cmax
      if (MASKS && !bwd_block_on(p, b, hq, qt, kt)) cm = 0;
      const long long cn = MASKS ? klo - t0 : 0;
      const int cmin = (int)(cn < 0 ? 0 : (cn > 64 ? 64 : cn));
      const int cmax = (int)(cm < 0 ? 0 : (cm > 64 ? 64 : cm));
      const bool edge = __any_sync(0xffffffffu, cmax < 64 || cmin > 0);
      if (!(ok = mbar_wait_warp(bar(C::QB_SF + (n & 1)), (n >> 1) & 1u, abort_flag))) break;
      tc_fence_after_sync();
      const uint32_t t_s = tmem + lane_off + ((n & 1) ? C::Q_TM_S1 : C::Q_TM_S0) + c0;
      float pr[64];
      {
        uint32_t a[32], bq[32];
        tmem_ld32(t_s, a);
        tmem_ld32(t_s + 32, bq);
        tmem_ld_wait();
        reg_fence32(a);
        reg_fence32(bq);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const uint32_t s0 = c < 32 ? a[c] : bq[c - 32];
          const uint32_t s1 = c < 32 ? a[c + 1] : bq[c - 31];
          float x0, x1;
          split_f32x2(fma_f32x2(f32x2(__uint_as_float(s0), __uint_as_float(s1)), c2x2, nlx2), x0,
                      x1);
          if (edge) {
            x0 = bwd_keep(c < cmax && c >= cmin, x0);
            x1 = bwd_keep(c + 1 < cmax && c + 1 >= cmin, x1);
          }
          pr[c] = ex2(x0);
          pr[c + 1] = ex2(x1);
        }
      }
      if (!(ok = mbar_wait_warp(bar(C::QB_DPF), n & 1u, abort_flag))) break;
      tc_fence_after_sync();
      {
        uint32_t a[32], bq[32];
        tmem_ld32(t_dp, a);
        tmem_ld32(t_dp + 32, bq);
        tmem_ld_wait();
        reg_fence32(a);
        reg_fence32(bq);
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = 2 * e;
          const float d0 = __uint_as_float(c < 32 ? a[c] : bq[c - 32]) - dd;
          const float d1 = __uint_as_float(c < 32 ? a[c + 1] : bq[c - 31]) - dd;
          pk[e] = pack_bf16x2(pr[c] * d0, pr[c + 1] * d1);
        }
        tmem_st32(t_dp, pk);  // dS into the first 32 columns of this warpgroup's run
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(bar(C::QB_DSF));
      }
    }
    // ---- epilogue: each warpgroup writes half of the dQ row (times scale)
    const bool have = NI > 0;
    if (have && ok) {
      ok = mbar_wait_warp(bar(C::QB_ACC), 0, abort_flag);
      tc_fence_after_sync();
    }
    if ((!have || ok) && row0 < n_rows) {
      constexpr int HALF = D / 2;
      const uint32_t t_acc = tmem + lane_off + C::Q_TM_DQ + wg * HALF;
      const int rr = row < n_rows ? row : 0;
      uint16_t* out = p.dq +
                      (VARLEN ? ((size_t)(sq.q0 + rr) * p.Hq + hq) : ((size_t)bh_q * p.Sq + rr)) * D +
                      wg * HALF;
#pragma unroll
      for (int c = 0; c < HALF; c += 32) {
        uint32_t v[32];
        if (have) {
          tmem_ld32_sync(t_acc + c, v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        if (row < n_rows) bwd_store32(out + c, v, p.scale);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
  // launched as a programmatic dependent of the dK/dV grid: this grid does
  // not complete before that one has, so work after the backward in the
  // stream sees dK and dV as well
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace attn_b200
