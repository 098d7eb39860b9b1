// prefill_sm100.cuh -- exact softmax attention forward (prefill) for sm_100a.
//
// What it computes ("Attention Kernel", section "问题与成本"):
//   O = softmax(Q K^T * scale + M) V,  LSE = ln sum exp(scale * Q K^T + M)
// blockwise with the online (m, l, o) recurrence ("Attention Kernel", section
// "Online softmax"; "Attention 算子加速史", section 1.3), so the S_q x S_k
// score matrix never leaves the chip.
//
// Organisation of one CTA (320 threads, one CTA per SM):
//   * It owns two 128-row query tiles of one (batch, query head): rows
//     [256*qb, 256*qb + 256).  The loop order is query tile outside, KV tiles
//     inside, with the output accumulator resident on chip until one final
//     write ("Attention 算子加速史", section 2.1).
//   * warp 0, lane 0  -- TMA producer: the two Q tiles once, then K_j and V_j
//     128-key tiles into a STAGES-deep ring guarded by full/empty mbarriers
//     ("Attention 算子加速史", section 3.3: producer warp, mbarriers, double
//     buffering; TMA as in section 3.1).  No multicast.
//   * warp 1, lane 0  -- tcgen05 MMA issuer: S_i = Q_i K_j^T (SS form, both
//     operands in shared memory) and O_i += P_i V_j (TS form, P read from
//     tensor memory), ping-ponging between the two query tiles so that the
//     tensor core works on one tile while the other tile's softmax runs.
//   * warps 2-5 and 6-9 -- one softmax warpgroup per query tile; thread r of
//     a warpgroup owns row r (= TMEM lane r).  Per KV tile: load the S row
//     from TMEM, apply the causal / key-length predicate (boundary tiles
//     only; tiles that are wholly masked are never visited -- "Attention
//     Kernel", section "FlashAttention 的稳定基础"), update the running max,
//     write P = 2^(S*scale*log2e - m) as bf16 back into TMEM over the S
//     columns, rescale O in TMEM when the max moved, and hand P to the MMA
//     warp.  The division by l happens once in the epilogue ("Attention
//     算子加速史", section 2.2).
//   * Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 and O_1
//     after them (d columns each); P_i aliases the first 64 columns of S_i.
//
// Rescaling is lazy: the max used as the exponent base only moves when the
// new row max exceeds it by more than 8 (log2 units), so P <= 2^8.  The final
// O = o / l and LSE are unchanged in exact arithmetic because the same base
// enters o and l.
//
// Empty rows (no visible key) get O = 0 and LSE = -inf: the exponent base
// falls back to 0 while the running max is -inf, so P = 2^-inf = 0 and l = 0.
#pragma once

#include "sm100_primitives.cuh"

namespace attn_b200 {

struct PrefillParams {
  float* lse;           // [B, Hq, Sq] or nullptr
  const int* k_lens;    // [B] or nullptr
  int B, Hq, Hkv, Sq, Sk;
  int group;            // Hq / Hkv
  float scale_log2;     // scale * log2(e)
  int n_qblocks;        // ceil(Sq / 256)
};

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;  // query rows per tile (MMA M, TMEM lanes)
  static constexpr int BN = 128;  // keys per KV tile
  static constexpr int STAGES = (D == 64) ? 4 : 2;
  static constexpr int TILE_BYTES = BM * D * 2;  // bf16 128 x D tile (Q, K or V)
  static constexpr int CB_BYTES = 128 * 128;     // one 64-column block of a 128-row tile
  static constexpr int NCB = D / 64;             // 64-column blocks per tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
  // barrier indices
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + STAGES;
  static constexpr int B_VFULL = B_KEMPTY + STAGES;
  static constexpr int B_VEMPTY = B_VFULL + STAGES;
  static constexpr int B_SFULL = B_VEMPTY + STAGES;  // 2
  static constexpr int B_PFULL = B_SFULL + 2;        // 2
  static constexpr int B_OFULL = B_PFULL + 2;        // 2
  static constexpr int B_DRAIN = B_OFULL + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem base, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + runtime 1024-B alignment
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns of S_i (P_i aliases its first 64) and of O_i
  __host__ __device__ static constexpr uint32_t tmem_s(int i) { return i ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t tmem_o(int i) { return i ? 256u + D : 256u; }
  static constexpr int NUM_THREADS = 320;
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Number of 128-key tiles query tile i (rows [row0, row0+127]) must visit, and
// the largest key index visible to its first row (tiles beyond that need the
// per-element predicate).
__device__ __forceinline__ int prefill_num_kv_tiles(int row0, int Sq, int klen, bool causal) {
  if (row0 >= Sq) return 0;
  const int last_row = min(row0 + 127, Sq - 1);
  long long lim = (long long)klen - 1;
  if (causal) lim = min(lim, (long long)last_row + (long long)klen - Sq);
  return lim < 0 ? 0 : (int)(lim / 128) + 1;
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(320, 1)
    attn_prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ CUtensorMap tm_o, const PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sbase_ptr = smem_raw + (sbase - raw_addr);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase_ptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase_ptr + C::OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: heaviest causal blocks first (longest processing time first)
  const int qb = p.n_qblocks - 1 - (int)blockIdx.x;
  const int hq = blockIdx.y;
  const int b = blockIdx.z;
  const int kvh = hq / p.group;
  int klen = p.Sk;
  if (p.k_lens != nullptr) {
    klen = p.k_lens[b];
    if (klen < 0 || klen > p.Sk) {
      if (threadIdx.x == 0) flag_device_error(kDevErrBadLength);
      klen = klen < 0 ? 0 : p.Sk;
    }
  }
  // per query tile i in {0, 1}: first row and number of KV tiles to visit
  const int row0_0 = qb * 256, row0_1 = qb * 256 + 128;
  const int nkv_0 = prefill_num_kv_tiles(row0_0, p.Sq, klen, CAUSAL);
  const int nkv_1 = prefill_num_kv_tiles(row0_1, p.Sq, klen, CAUSAL);
  auto row0 = [&](int i) { return i ? row0_1 : row0_0; };
  auto nkv = [&](int i) { return i ? nkv_1 : nkv_0; };
  const int n_max = max(nkv_0, nkv_1);
  const int q_head_row = b * p.Hq + hq;   // z coordinate in the Q / O maps
  const int kv_head_row = b * p.Hkv + kvh;

  // ---- setup: barriers (thread 0), tensor memory (warp 1)
  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_QFULL), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(C::B_KFULL + s), 1);
      mbar_init(bar(C::B_KEMPTY + s), 1);
      mbar_init(bar(C::B_VFULL + s), 1);
      mbar_init(bar(C::B_VEMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_SFULL + i), 1);
      mbar_init(bar(C::B_PFULL + i), 128);
      mbar_init(bar(C::B_OFULL + i), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
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

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0 && n_max > 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      uint32_t q_bytes = 0;
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (nkv(i) > 0) q_bytes += C::TILE_BYTES;
      mbar_arrive_expect_tx(bar(C::B_QFULL), q_bytes);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (nkv(i) == 0) continue;
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_load_3d(sbase + C::OFF_Q + i * C::TILE_BYTES + cb * C::CB_BYTES, &tm_q,
                      bar(C::B_QFULL), 64 * cb, row0(i), q_head_row);
      }
      int loaded = 0;  // KV tiles whose loads were issued
      for (int j = 0; j < n_max; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (uint32_t)(j / C::STAGES) & 1u;
        if (!mbar_wait(bar(C::B_KEMPTY + s), ph ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::TILE_BYTES);
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_load_3d(sbase + C::OFF_K + s * C::TILE_BYTES + cb * C::CB_BYTES, &tm_k,
                      bar(C::B_KFULL + s), 64 * cb, j * 128, kv_head_row);
        if (!mbar_wait(bar(C::B_VEMPTY + s), ph ^ 1u, abort_flag)) {
          loaded = -(j + 1);  // K_j issued, V_j not
          break;
        }
        mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::TILE_BYTES);
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_load_3d(sbase + C::OFF_V + s * C::TILE_BYTES + cb * C::CB_BYTES, &tm_v,
                      bar(C::B_VFULL + s), 64 * cb, j * 128, kv_head_row);
        loaded = j + 1;
      }
      // Drain: never leave the CTA with copies still landing in shared memory.
      mbar_wait(bar(C::B_QFULL), 0, nullptr);
      const int nk = loaded >= 0 ? loaded : -loaded;
      const int nv = loaded >= 0 ? loaded : -loaded - 1;
      for (int j = (nk > C::STAGES ? nk - C::STAGES : 0); j < nk; ++j)
        mbar_wait(bar(C::B_KFULL + j % C::STAGES), (uint32_t)(j / C::STAGES) & 1u, nullptr);
      for (int j = (nv > C::STAGES ? nv - C::STAGES : 0); j < nv; ++j)
        mbar_wait(bar(C::B_VFULL + j % C::STAGES), (uint32_t)(j / C::STAGES) & 1u, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= tcgen05 MMA issuer =======================
    if (lane == 0 && n_max > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      // S_i = Q_i K^T over d in steps of 16 (32 bytes inside a 128-byte swizzled row,
      // 64-column blocks 16 KB apart).
      auto issue_qk = [&](int i, int stage) {
        const uint32_t qa = sbase + C::OFF_Q + i * C::TILE_BYTES;
        const uint32_t ka = sbase + C::OFF_K + stage * C::TILE_BYTES;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * C::CB_BYTES + (ks & 3) * 32;
          umma_ss(tmem + C::tmem_s(i), smem_desc_sw128(qa + off, 16, 1024),
                  smem_desc_sw128(ka + off, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
        }
      };
      // O_i (+)= P_i V over the 128 keys in steps of 16: P from TMEM (8 columns
      // per step), V as an MN-major operand (16 keys = 2048 bytes per step).
      auto issue_pv = [&](int i, int stage, bool accumulate) {
        const uint32_t va = sbase + C::OFF_V + stage * C::TILE_BYTES;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          umma_ts(tmem + C::tmem_o(i), tmem + C::tmem_s(i) + ks * 8,
                  smem_desc_sw128(va + ks * 2048, C::CB_BYTES, 1024), idesc_pv,
                  (accumulate || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(bar(C::B_QFULL), 0, abort_flag);
      if (ok) ok = mbar_wait(bar(C::B_KFULL + 0), 0, abort_flag);
      if (ok) {
        tc_fence_after_sync();
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          if (nkv(i) == 0) continue;
          issue_qk(i, 0);
          umma_commit(bar(C::B_SFULL + i));
        }
        umma_commit(bar(C::B_KEMPTY + 0));
      }
      for (int j = 0; ok && j < n_max; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (uint32_t)(j / C::STAGES) & 1u;
        const int s1 = (j + 1) % C::STAGES;
        const uint32_t ph1 = (uint32_t)((j + 1) / C::STAGES) & 1u;
        if (!(ok = mbar_wait(bar(C::B_VFULL + s), ph, abort_flag))) break;
        bool k_next = false;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          if (!ok) break;
          if (j >= nkv(i)) continue;
          if (!(ok = mbar_wait(bar(C::B_PFULL + i), (uint32_t)j & 1u, abort_flag))) break;
          tc_fence_after_sync();
          issue_pv(i, s, j > 0);
          if (j + 1 < nkv(i)) {
            if (!k_next) {
              if (!(ok = mbar_wait(bar(C::B_KFULL + s1), ph1, abort_flag))) break;
              tc_fence_after_sync();
              k_next = true;
            }
            issue_qk(i, s1);
            umma_commit(bar(C::B_SFULL + i));
          } else {
            umma_commit(bar(C::B_OFULL + i));
          }
        }
        umma_commit(bar(C::B_VEMPTY + s));
        if (k_next) umma_commit(bar(C::B_KEMPTY + s1));
      }
      // Drain: every MMA issued above has completed before TMEM is released.
      umma_commit(bar(C::B_DRAIN));
      mbar_wait(bar(C::B_DRAIN), 0, nullptr);
    }
    __syncwarp();
  } else {
    // ======================= softmax warpgroups =======================
    const int i = (warp - 2) >> 2;       // query tile of this warpgroup
    const int quarter = warp & 3;        // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;   // row within the tile
    const int row = row0(i) + r;
    const int n = nkv(i);
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + C::tmem_s(i);
    const uint32_t t_o = tmem + lane_off + C::tmem_o(i);
    const long long koff = (long long)klen - p.Sq;
    // largest visible key of this row, and of the tile's first row
    long long lim_row = (long long)klen - 1;
    long long lim_tile = lim_row;
    if (CAUSAL) {
      lim_row = min(lim_row, (long long)row + koff);
      lim_tile = min(lim_tile, (long long)row0(i) + koff);
    }
    float c2 = p.scale_log2;
    const bool scale_pos = c2 > 0.f;
    if (!scale_pos) c2 = 1.f;  // scores are pre-multiplied below instead
    float m_run = -INFINITY;   // exponent base (log2 units)
    float l_run = 0.f;         // sum of P (f32)
    float lr_run = 0.f;        // sum of bf16(P)
    bool ok = true;

    for (int j = 0; j < n; ++j) {
      if (!(ok = mbar_wait_warp(bar(C::B_SFULL + i), (uint32_t)j & 1u, abort_flag))) break;
      tc_fence_after_sync();
      float s[128];
      {
        uint32_t u0[32], u1[32], u2[32], u3[32];
        tmem_ld32(t_s, u0);
        tmem_ld32(t_s + 32, u1);
        tmem_ld32(t_s + 64, u2);
        tmem_ld32(t_s + 96, u3);
        tmem_ld_wait();
        reg_fence32(u0);
        reg_fence32(u1);
        reg_fence32(u2);
        reg_fence32(u3);
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          s[k] = __uint_as_float(u0[k]);
          s[32 + k] = __uint_as_float(u1[k]);
          s[64 + k] = __uint_as_float(u2[k]);
          s[96 + k] = __uint_as_float(u3[k]);
        }
      }
      if ((long long)j * 128 + 127 > lim_tile) {
        // boundary tile: per-element predicate
        const long long lim_local = lim_row - (long long)j * 128;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if ((long long)c > lim_local) s[c] = -INFINITY;
      }
      if (!scale_pos) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          s[c] = (s[c] == -INFINITY) ? -INFINITY : s[c] * p.scale_log2;
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mx0 = fmaxf(mx0, s[c]);
        mx1 = fmaxf(mx1, s[c + 1]);
        mx2 = fmaxf(mx2, s[c + 2]);
        mx3 = fmaxf(mx3, s[c + 3]);
      }
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c2;
      float alpha = 1.f;
      if (m_tile > m_run + 8.f) {  // also true for the first finite max
        alpha = ex2(m_run - m_tile);
        m_run = m_tile;
      }
      const float base = (m_run == -INFINITY) ? 0.f : m_run;
      // Two row sums: l over the f32 P (gives the LSE) and lr over the
      // bf16-rounded P that the PV MMA consumes (normalises O, so that the
      // weights applied to V sum to one exactly as used).
      float l0 = 0.f, l1 = 0.f;
      uint64_t r01 = 0ull, r23 = 0ull;  // f32x2 partial sums of the rounded P
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const int cc = 64 * half + c;
          const float p0 = ex2(fmaf(s[cc], c2, -base));
          const float p1 = ex2(fmaf(s[cc + 1], c2, -base));
          const float p2 = ex2(fmaf(s[cc + 2], c2, -base));
          const float p3 = ex2(fmaf(s[cc + 3], c2, -base));
          l0 += p0 + p1;
          l1 += p2 + p3;
          pk[c / 2] = pack_bf16x2(p0, p1);
          pk[c / 2 + 1] = pack_bf16x2(p2, p3);
          r01 = add_f32x2(r01, bf16x2_to_f32x2(pk[c / 2]));
          r23 = add_f32x2(r23, bf16x2_to_f32x2(pk[c / 2 + 1]));
        }
        tmem_st32(t_s + 32 * half, pk);  // P columns [32*half, 32*half + 32)
      }
      l_run = l_run * alpha + (l0 + l1);
      lr_run = lr_run * alpha + (sum_f32x2(r01) + sum_f32x2(r23));
      // Rescale the accumulator when any row of this warp moved its base.  The
      // MMA that last wrote O_i completed before S_i(j) was signalled.
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t u[32];
          tmem_ld32_sync(t_o + c, u);
#pragma unroll
          for (int k = 0; k < 32; ++k) u[k] = __float_as_uint(__uint_as_float(u[k]) * alpha);
          tmem_st32(t_o + c, u);
        }
      }
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(bar(C::B_PFULL + i));
    }

    // ---- epilogue: O = o / l -> bf16, staged through this tile's Q buffer
    // (free once its last MMA completed) and stored with TMA; LSE per row.
    if (row0(i) < p.Sq) {
      if (n > 0 && ok) ok = mbar_wait_warp(bar(C::B_OFULL + i), 0, abort_flag);
      tc_fence_after_sync();
      const bool has_o = (n > 0) && ok;
      const float inv = (lr_run > 0.f) ? (1.f / lr_run) : 0.f;
      uint8_t* stage = sbase_ptr + C::OFF_Q + i * C::TILE_BYTES;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t u[32];
        if (has_o) {
          tmem_ld32_sync(t_o + c, u);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) u[k] = 0u;
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int dcol = c + 8 * q4;        // first of 8 columns in this 16-byte chunk
          const int cb = dcol >> 6;           // 64-column block
          const int chunk = (dcol & 63) >> 3; // 16-byte chunk within the 128-byte row
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(u[8 * q4 + 0]) * inv, __uint_as_float(u[8 * q4 + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(u[8 * q4 + 2]) * inv, __uint_as_float(u[8 * q4 + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(u[8 * q4 + 4]) * inv, __uint_as_float(u[8 * q4 + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(u[8 * q4 + 6]) * inv, __uint_as_float(u[8 * q4 + 7]) * inv);
          *reinterpret_cast<uint4*>(stage + cb * C::CB_BYTES + r * 128 +
                                    ((chunk ^ (r & 7)) << 4)) = w;
        }
      }
      fence_proxy_async_smem();
      named_barrier_sync(1 + i, 128);
      if (warp == 2 + 4 * i && lane == 0 && !*abort_flag) {
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_store_3d(&tm_o, smem_u32(stage) + cb * C::CB_BYTES, 64 * cb, row0(i), q_head_row);
        tma_store_commit();
        tma_store_wait_read_all();
      }
      if (p.lse != nullptr && row < p.Sq) {
        const float lse = (l_run > 0.f) ? (m_run + lg2(l_run)) * 0.69314718055994531f : -INFINITY;
        p.lse[(size_t)q_head_row * p.Sq + row] = lse;
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace attn_b200
