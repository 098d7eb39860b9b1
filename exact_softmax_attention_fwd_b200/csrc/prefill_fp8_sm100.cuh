// prefill_fp8_sm100.cuh -- exact softmax attention forward (prefill) over
// block-scaled E4M3 Q, K and V, for sm_100a.
//
// What it computes: the prefill of prefill_sm100.cuh on the dequantised
// inputs.  Each tensor arrives as E4M3 codes with one fp32 scale per (batch,
// head, block of 128 consecutive rows) -- the block-level scaling that
// "Attention 算子加速史", section 3.3 pairs with FP8 operands (no block shape
// is given there; 128 rows is the tile this kernel loads) -- and an element
// is scale * e4m3(code).
//
// How (dense layout, d = 128; the bf16 kernel's persistent organisation and
// ping-pong of two 128-row query tiles, see prefill_sm100.cuh):
//   * S = Q K^T runs on the FP8 tensor-core path: tcgen05.mma kind::f8f6f4 on
//     the E4M3 codes of a Q tile and a K tile (32 codes of the head dimension
//     per instruction, fp32 accumulation in tensor memory).  The product of
//     codes is exact in fp32 up to accumulation order; the two block scales
//     are one fp32 factor per (query tile, key tile), folded into the exponent
//     multiplier of the softmax.
//   * P V is an f16 MMA (kind::f16, P from tensor memory), so that the weights
//     keep 11 bits of precision: two warps widen each E4M3 V tile into an f16
//     copy in shared memory (E4M3 values are exact in f16; one conversion per
//     pair of codes) in the layout the MMA reads.  The V tile's scale enters
//     the weights before they are rounded, relative to the largest V scale of
//     the query tile's key range (vmax), which keeps them within f16's range:
//     P' = 2^(x + log2(v_scale / vmax)) <= 2^8.  O accumulates in units of
//     vmax and is normalised by the unrounded row sum of P (f16 rounds P' to
//     2^-11 relative, below the forward's tolerance, and a V block whose scale
//     is far below vmax -- whose weights underflow f16 -- still counts with its
//     full weight): O = vmax * sum f16(P') v_code / sum P.
//   * warp 0: TMA producer (E4M3 Q, K, V tiles; no multicast); warp 1: MMA
//     issuer (elect.sync); warps 2-3: V widening; warps 4-11: two softmax
//     warpgroups, one per query tile, thread = row = TMEM lane.
#pragma once

#include "prefill_sm100.cuh"

namespace attn_b200 {

// Parameters: the dense prefill's, plus the block scales (fp32, [B, Hq,
// n_qt] for Q and [B, Hkv, n_kt] for K and V).
struct PrefillFp8Params {
  PrefillParams p;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
};

struct PrefillFp8Cfg {
  static constexpr int D = 128;
  static constexpr int STAGES = 2;
  static constexpr int T8 = 128 * 128;           // a 128-row E4M3 tile (Q, K or V)
  static constexpr int VB = 128 * D * 2;         // a widened f16 V tile
  static constexpr int CB_BYTES = 128 * 128;     // one 64-column block of the f16 tile
  static constexpr int STG_BYTES = 32 * 128;     // per-warp epilogue staging
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * T8;
  static constexpr int OFF_V8 = OFF_K + STAGES * T8;
  static constexpr int OFF_VB = OFF_V8 + STAGES * T8;
  static constexpr int OFF_STG = OFF_VB + STAGES * VB;
  static constexpr int OFF_BAR = OFF_STG + 8 * STG_BYTES;
  static constexpr int B_QFULL = 0;                  // 2
  static constexpr int B_QFREE = B_QFULL + 2;        // 2
  static constexpr int B_KFULL = B_QFREE + 2;
  static constexpr int B_KEMPTY = B_KFULL + STAGES;
  static constexpr int B_VFULL = B_KEMPTY + STAGES;  // E4M3 V landed
  static constexpr int B_VEMPTY = B_VFULL + STAGES;  // E4M3 V widened (64 arrivals)
  static constexpr int B_CFULL = B_VEMPTY + STAGES;  // f16 V ready (64 arrivals)
  static constexpr int B_CEMPTY = B_CFULL + STAGES;  // f16 V read by its P V
  static constexpr int B_SFULL = B_CEMPTY + STAGES;  // 2
  static constexpr int B_PFULL = B_SFULL + 2;        // 2
  static constexpr int B_OFULL = B_PFULL + 2;        // 2
  static constexpr int B_DRAIN = B_OFULL + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  __host__ __device__ static constexpr uint32_t tmem_s(int i) { return i ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t tmem_o(int i) { return i ? 256u + D : 256u; }
  static constexpr int NUM_THREADS = 384;
  static constexpr uint32_t REGS_PRODUCER = 56;
  static constexpr uint32_t REGS_SOFTMAX = 224;
  static_assert(128 * (REGS_PRODUCER + 2 * REGS_SOFTMAX) <= NUM_THREADS * 168, "registers");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Instruction descriptor for kind::f8f6f4 with E4M3 A and B (format code 0)
// and an fp32 accumulator, both operands K-major: D format f32 = 1 [4,6),
// A format [7,10) = 0, B format [10,13) = 0, N>>3 [17,23), M>>4 [24,29).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem], E4M3 operands.
__device__ __forceinline__ void umma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Four E4M3 codes -> two f16x2 (exact: E4M3 values are f16 values), codes 0-1
// -> lo, 2-3 -> hi.
__device__ __forceinline__ void e4m3x4_to_f16x2x2_v(uint32_t four, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(four));
}

// Two floats -> packed f16x2 (round to nearest even); `lo` lands in bits 0-15.
__device__ __forceinline__ uint32_t pack_f16x2_p(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Instruction descriptor of a kind::f16 MMA on f16 A and B, f32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

template <bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    attn_prefill_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v,
                            const __grid_constant__ CUtensorMap tm_o, const PrefillFp8Params f) {
  using C = PrefillFp8Cfg;
  constexpr int D = C::D;
  const PrefillParams& p = f.p;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sbase_ptr = smem_raw + (sbase - raw_addr);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase_ptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase_ptr + C::OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_QFULL + i), 1);
      mbar_init(bar(C::B_QFREE + i), 1);
      mbar_init(bar(C::B_SFULL + i), 1);
      mbar_init(bar(C::B_PFULL + i), 128);
      mbar_init(bar(C::B_OFULL + i), 1);
    }
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(C::B_KFULL + s), 1);
      mbar_init(bar(C::B_KEMPTY + s), 1);
      mbar_init(bar(C::B_VFULL + s), 1);
      mbar_init(bar(C::B_VEMPTY + s), 64);
      mbar_init(bar(C::B_CFULL + s), 64);
      mbar_init(bar(C::B_CEMPTY + s), 1);
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

  if (warp < 4) {
    warpgroup_reg_dealloc<C::REGS_PRODUCER>();
    if (warp == 0) {
      // ======================= TMA producer =======================
      if (lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
        uint32_t q_loads0 = 0, q_loads1 = 0;
        uint32_t kv = 0;
        bool ok = true;
        auto load_q = [&](const PrefillUnit& u, int i) -> bool {
          uint32_t& n = i ? q_loads1 : q_loads0;
          if (n > 0 && !mbar_wait(bar(C::B_QFREE + i), (n - 1) & 1u, abort_flag)) return false;
          mbar_arrive_expect_tx(bar(C::B_QFULL + i), C::T8);
          tma_load_3d(sbase + C::OFF_Q + i * C::T8, &tm_q, bar(C::B_QFULL + i), 0, u.row0[i],
                      u.b * p.Hq + u.hq);
          ++n;
          return true;
        };
        PrefillUnit u;
        for (int k = 0; ok && prefill_unit<CAUSAL, kLayoutDense, false>(p, k, u); ++k) {
          const bool has0 = u.kv_end[0] > u.kv_begin[0], has1 = u.kv_end[1] > u.kv_begin[1];
          const int kv_row = u.b * p.Hkv + u.hq / p.group;
          if (has0 && !(ok = load_q(u, 0))) break;
          for (int j = u.kv_first; j < u.kv_last; ++j) {
            const int s = kv % C::STAGES;
            const uint32_t ph = (kv / C::STAGES) & 1u;
            if (!(ok = mbar_wait(bar(C::B_KEMPTY + s), ph ^ 1u, abort_flag))) break;
            mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::T8);
            tma_load_3d(sbase + C::OFF_K + s * C::T8, &tm_k, bar(C::B_KFULL + s), 0, j * 128,
                        kv_row);
            if (j == u.kv_first && has1 && !(ok = load_q(u, 1))) {
              ++kv;
              break;
            }
            if (!(ok = mbar_wait(bar(C::B_VEMPTY + s), ph ^ 1u, abort_flag))) {
              ++kv;
              break;
            }
            mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::T8);
            tma_load_3d(sbase + C::OFF_V8 + s * C::T8, &tm_v, bar(C::B_VFULL + s), 0, j * 128,
                        kv_row);
            ++kv;
          }
        }
        // no copy may still be landing at exit (bounded waits)
        if (q_loads0 > 0) mbar_wait(bar(C::B_QFULL + 0), (q_loads0 - 1) & 1u, nullptr);
        if (q_loads1 > 0) mbar_wait(bar(C::B_QFULL + 1), (q_loads1 - 1) & 1u, nullptr);
        for (uint32_t j = (kv > C::STAGES ? kv - C::STAGES : 0); j < kv; ++j) {
          mbar_wait(bar(C::B_KFULL + j % C::STAGES), (j / C::STAGES) & 1u, nullptr);
          if (ok) mbar_wait(bar(C::B_VFULL + j % C::STAGES), (j / C::STAGES) & 1u, nullptr);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ======================= tcgen05 MMA issuer =======================
      constexpr uint32_t idesc_qk = idesc_e4m3_f32(128, 128);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, D, true);
      auto wait = [&](uint32_t b, uint32_t ph) -> bool {
        if (__all_sync(0xffffffffu, mbar_test(b, ph))) return true;
        const bool r = mbar_wait_slow(b, ph, abort_flag);
        return __all_sync(0xffffffffu, r);
      };
      // S_i = Q_i K^T: 128-byte rows (all of d), 32 codes (32 bytes) per step
      auto issue_qk = [&](int i, int stage) {
        const uint64_t qd = smem_desc_sw128(opaque_u32(sbase + C::OFF_Q + i * C::T8), 16, 1024);
        const uint64_t kd = smem_desc_sw128(opaque_u32(sbase + C::OFF_K + stage * C::T8), 16, 1024);
        const uint32_t dt = tmem + C::tmem_s(i);
#pragma unroll
        for (int ks = 0; ks < D / 32; ++ks)
          umma_ss_f8(dt, qd + (uint64_t)((ks * 32) >> 4), kd + (uint64_t)((ks * 32) >> 4), idesc_qk,
                     ks > 0 ? 1u : 0u);
      };
      // O_i (+)= P_i V over the widened f16 V tile
      auto issue_pv = [&](int i, int stage, bool accumulate) {
        const uint64_t vd =
            smem_desc_sw128(opaque_u32(sbase + C::OFF_VB + stage * C::VB), C::CB_BYTES, 1024);
        const uint32_t ts = opaque_u32(tmem + C::tmem_s(i));
        const uint32_t dt = tmem + C::tmem_o(i);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_ts(dt, ts + ks * 8, vd + (uint64_t)((ks * 2048) >> 4), idesc_pv,
                  (accumulate || ks > 0) ? 1u : 0u);
      };
      uint32_t kv = 0;
      uint32_t q_waits0 = 0, q_waits1 = 0, p_waits0 = 0, p_waits1 = 0;
      bool ok = true;
      PrefillUnit u;
      for (int k = 0; ok && prefill_unit<CAUSAL, kLayoutDense, false>(p, k, u); ++k) {
        const int jb = u.kv_first, je = u.kv_last;
        if (je <= jb) continue;
        {
          const int s = kv % C::STAGES;
          if (!(ok = wait(bar(C::B_KFULL + s), (kv / C::STAGES) & 1u))) break;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (!ok) break;
            if (u.kv_begin[i] != jb || u.kv_end[i] <= jb) continue;
            uint32_t& qw = i ? q_waits1 : q_waits0;
            if (!(ok = wait(bar(C::B_QFULL + i), qw & 1u))) break;
            ++qw;
            tc_fence_after_sync();
            if (elect_one()) {
              issue_qk(i, s);
              umma_commit(bar(C::B_SFULL + i));
              if (u.kv_end[i] == jb + 1) umma_commit(bar(C::B_QFREE + i));
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) umma_commit(bar(C::B_KEMPTY + s));
          __syncwarp();
        }
        for (int j = jb; ok && j < je; ++j) {
          const uint32_t idx = kv + (uint32_t)(j - jb);
          const int s = idx % C::STAGES;
          const int s1 = (idx + 1) % C::STAGES;
          // the widened f16 copy of V_j (not the E4M3 tile) feeds P V
          if (!(ok = wait(bar(C::B_CFULL + s), (idx / C::STAGES) & 1u))) break;
          bool k_next = false;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (!ok) break;
            const int b0 = u.kv_begin[i], e0 = u.kv_end[i];
            if (j < b0 || j >= e0) continue;
            uint32_t& pw = i ? p_waits1 : p_waits0;
            if (!(ok = wait(bar(C::B_PFULL + i), pw & 1u))) break;
            ++pw;
            tc_fence_after_sync();
            const bool more = j + 1 < e0;
            if (more && !k_next) {
              if (!(ok = wait(bar(C::B_KFULL + s1), ((idx + 1) / C::STAGES) & 1u))) break;
              tc_fence_after_sync();
              k_next = true;
            }
            if (elect_one()) {
              issue_pv(i, s, j > b0);
              if (more) {
                issue_qk(i, s1);
                umma_commit(bar(C::B_SFULL + i));
                if (j + 2 == e0) umma_commit(bar(C::B_QFREE + i));
              } else {
                umma_commit(bar(C::B_OFULL + i));
              }
            }
            __syncwarp();
          }
          if (elect_one()) {
            umma_commit(bar(C::B_CEMPTY + s));
            if (k_next) umma_commit(bar(C::B_KEMPTY + s1));
          }
          __syncwarp();
        }
        kv += (uint32_t)(je - jb);
      }
      if (elect_one()) umma_commit(bar(C::B_DRAIN));
      __syncwarp();
      mbar_wait(bar(C::B_DRAIN), 0, nullptr);
      __syncwarp();
    } else {
      // ======================= V widening (warps 2-3) =======================
      // Each K/V step's E4M3 V tile (128 keys x 128 bytes, 128-byte swizzled
      // as TMA lands it) becomes an f16 tile in the MN-major layout the P V
      // MMA reads: two 64-column blocks of 128 rows x 128 bytes, 128-byte
      // swizzled.  Thread t handles 16-code chunks t, t + 64, ... (8 chunks
      // per key row).
      const int t = threadIdx.x - 64;
      uint32_t kv = 0;
      bool ok = true;
      PrefillUnit u;
      for (int k = 0; ok && prefill_unit<CAUSAL, kLayoutDense, false>(p, k, u); ++k) {
        for (int j = u.kv_first; ok && j < u.kv_last; ++j, ++kv) {
          const int s = kv % C::STAGES;
          const uint32_t ph = (kv / C::STAGES) & 1u;
          if (!(ok = mbar_wait_warp(bar(C::B_VFULL + s), ph, abort_flag))) break;
          if (!(ok = mbar_wait_warp(bar(C::B_CEMPTY + s), ph ^ 1u, abort_flag))) break;
          const uint32_t src = sbase + C::OFF_V8 + s * C::T8;
          uint8_t* dst = sbase_ptr + C::OFF_VB + s * C::VB;
#pragma unroll 4
          for (int m = 0; m < 16; ++m) {
            const int c = t + 64 * m;
            const int row = c >> 3, cc = c & 7;  // key row, 16-code chunk of its 128 codes
            uint4 x;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                         : "r"(src + row * 128 + (((cc ^ (row & 7)) & 7) << 4)));
            uint4 lo, hi;  // codes 0-7 and 8-15 of the chunk as f16
            e4m3x4_to_f16x2x2_v(x.x, lo.x, lo.y);
            e4m3x4_to_f16x2x2_v(x.y, lo.z, lo.w);
            e4m3x4_to_f16x2x2_v(x.z, hi.x, hi.y);
            e4m3x4_to_f16x2x2_v(x.w, hi.z, hi.w);
            // dims 16cc .. 16cc+15: block cc/4, 16-byte chunks 2(cc%4) and 2(cc%4)+1
            const int blk = cc >> 2, q0 = (cc & 3) * 2;
            uint8_t* rowp = dst + blk * C::CB_BYTES + row * 128;
            *reinterpret_cast<uint4*>(rowp + (((q0) ^ (row & 7)) << 4)) = lo;
            *reinterpret_cast<uint4*>(rowp + (((q0 + 1) ^ (row & 7)) << 4)) = hi;
          }
          fence_proxy_async_smem();  // the MMA (async proxy) reads what was written here
          mbar_arrive(bar(C::B_CFULL + s));
          mbar_arrive(bar(C::B_VEMPTY + s));
        }
      }
      __syncwarp();
    }
  } else {
    warpgroup_reg_alloc<C::REGS_SOFTMAX>();
    // ======================= softmax warpgroups =======================
    const int i = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + C::tmem_s(i);
    const uint32_t t_o = tmem + lane_off + C::tmem_o(i);
    const uint32_t stg = sbase + C::OFF_STG + (warp - 4) * C::STG_BYTES;
    uint8_t* stg_ptr = sbase_ptr + C::OFF_STG + (warp - 4) * C::STG_BYTES;
    uint32_t s_waits = 0, o_waits = 0;
    bool stores_pending = false;
    bool ok = true;
    PrefillUnit u;
    for (int k = 0; ok && prefill_unit<CAUSAL, kLayoutDense, false>(p, k, u); ++k) {
      const int row0 = i ? u.row0[1] : u.row0[0];
      if (row0 >= u.sq) continue;
      const int kb = i ? u.kv_begin[1] : u.kv_begin[0];
      const int ke = i ? u.kv_end[1] : u.kv_end[0];
      const int row = row0 + r;
      const int q_head_row = u.b * p.Hq + u.hq;
      const int kv_head_row = u.b * p.Hkv + u.hq / p.group;
      if (p.k_lens != nullptr && r == 0) {
        const int kl = p.k_lens[u.b];
        if (kl < 0 || kl > p.Sk) flag_device_error(kDevErrBadLength);
      }
      const long long koff = (long long)u.klen - u.sq;
      long long hi_row = (long long)u.klen - 1, hi_tile = hi_row;
      if (CAUSAL) {
        hi_row = min(hi_row, (long long)row + koff);
        hi_tile = min(hi_tile, (long long)row0 + koff);
      }
      // the query tile's block scale (scale_log2 carries the softmax scale)
      const float qsl = p.scale_log2 * __ldg(f.q_scale + (size_t)q_head_row * p.n_qt + row0 / 128);
      // the largest V block scale of this tile's key range: P' = P v_scale / vmax
      // <= 2^8 stays in f16's range, and O accumulates in units of vmax
      float vmax = 1e-30f;
      for (int jj = kb + lane; jj < ke; jj += 32)
        vmax = fmaxf(vmax, __ldg(f.v_scale + (size_t)kv_head_row * p.n_kt + jj));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      if (!(vmax < INFINITY)) vmax = 1e30f;
      float m_run = -INFINITY;
      float l_run = 0.f;   // sum of P (f32): the LSE and the normaliser of O

      for (int j = kb; j < ke; ++j) {
        const float ksc = __ldg(f.k_scale + (size_t)kv_head_row * p.n_kt + j);
        // block scales are positive; a V scale that is not (or is NaN) acts as
        // a vanishing one instead of turning the row into NaN
        const float vsc = fmaxf(__ldg(f.v_scale + (size_t)kv_head_row * p.n_kt + j), 1e-30f);
        float c2 = qsl * ksc;  // exponent multiplier of this (query tile, key tile)
        const bool scale_pos = c2 > 0.f;
        if (!(ok = mbar_wait_warp(bar(C::B_SFULL + i), s_waits & 1u, abort_flag))) break;
        ++s_waits;
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
          for (int e = 0; e < 32; ++e) {
            s[e] = __uint_as_float(u0[e]);
            s[32 + e] = __uint_as_float(u1[e]);
            s[64 + e] = __uint_as_float(u2[e]);
            s[96 + e] = __uint_as_float(u3[e]);
          }
        }
        if ((long long)j * 128 + 127 > hi_tile) {
          const long long hl = hi_row - (long long)j * 128;
          const int hi_local = hl < -1 ? -1 : (hl > 127 ? 127 : (int)hl);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > hi_local) s[c] = -INFINITY;
        }
        if (!scale_pos) {  // a non-positive multiplier: scale the scores first
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = (s[c] == -INFINITY) ? -INFINITY : s[c] * c2;
          c2 = 1.f;
        }
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c < 128; c += 8) {
          mx0 = max3f(mx0, s[c], s[c + 1]);
          mx1 = max3f(mx1, s[c + 2], s[c + 3]);
          mx2 = max3f(mx2, s[c + 4], s[c + 5]);
          mx3 = max3f(mx3, s[c + 6], s[c + 7]);
        }
        const float m_tile = max3f(fmaxf(mx0, mx1), mx2, mx3) * c2;
        float alpha = 1.f;
        if (m_tile > m_run + 8.f) {
          alpha = ex2(m_run - m_tile);
          m_run = m_tile;
        }
        const float base = (m_run == -INFINITY) ? 0.f : m_run;
        // P' = 2^(s*c2 - base + log2(v_scale / vmax)) = P * v_scale / vmax
        const float vrel = fminf(vsc, vmax) / vmax;
        const float nb = lg2(vrel) - base;
        const uint64_t c2x2 = f32x2(c2, c2);
        const uint64_t nbx2 = f32x2(nb, nb);
        uint64_t la = 0ull, lb = 0ull;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int cc = 64 * half + 2 * e;
            float x0, x1, x2, x3;
            split_f32x2(fma_f32x2(f32x2(s[cc], s[cc + 1]), c2x2, nbx2), x0, x1);
            split_f32x2(fma_f32x2(f32x2(s[cc + 2], s[cc + 3]), c2x2, nbx2), x2, x3);
            const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
            pk[e] = pack_f16x2_p(p0, p1);
            pk[e + 1] = pack_f16x2_p(p2, p3);
            la = add_f32x2(la, f32x2(p0, p1));
            lb = add_f32x2(lb, f32x2(p2, p3));
          }
          tmem_st32(t_s + 32 * half, pk);
        }
        const float inv_vs = 1.f / vrel;
        l_run = l_run * alpha + (sum_f32x2(la) + sum_f32x2(lb)) * inv_vs;
        if (j > kb && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t v[32];
            tmem_ld32_sync(t_o + c, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(t_o + c, v);
          }
        }
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(bar(C::B_PFULL + i));
      }
      if (!ok) break;

      // ---- epilogue (as the bf16 kernel): O / l -> bf16 by TMA store, LSE
      const bool has_o = ke > kb;
      if (has_o) {
        if (!(ok = mbar_wait_warp(bar(C::B_OFULL + i), o_waits & 1u, abort_flag))) break;
        ++o_waits;
      }
      tc_fence_after_sync();
      // O in units of vmax, normalised by the unrounded weights: f16 rounds P'
      // to 2^-11 relative, and a V block whose scale is far below vmax (a zero
      // block) still counts with its full weight
      const float o_mul = (l_run > 0.f) ? vmax / l_run : 0.f;
      const bool warp_has_rows = row0 + quarter * 32 < p.Sq;
#pragma unroll 1
      for (int cb = 0; cb < D / 64; ++cb) {
        if (stores_pending) {
          if (lane == 0) tma_store_wait_read_all();
          __syncwarp();
          stores_pending = false;
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          if (has_o) {
            tmem_ld32_sync(t_o + 64 * cb + 32 * half, v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int chunk = 4 * half + q4;
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * o_mul, __uint_as_float(v[8 * q4 + 1]) * o_mul);
            w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * o_mul, __uint_as_float(v[8 * q4 + 3]) * o_mul);
            w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * o_mul, __uint_as_float(v[8 * q4 + 5]) * o_mul);
            w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * o_mul, __uint_as_float(v[8 * q4 + 7]) * o_mul);
            *reinterpret_cast<uint4*>(stg_ptr + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = w;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && warp_has_rows && !*abort_flag) {
          tma_store_3d(&tm_o, stg, 64 * cb, row0 + quarter * 32, q_head_row);
          tma_store_commit();
        }
        stores_pending = true;
      }
      if (p.lse != nullptr && row < p.Sq) {
        const float lse = (l_run > 0.f) ? (m_run + lg2(l_run)) * 0.69314718055994531f : -INFINITY;
        p.lse[(size_t)q_head_row * p.Sq + row] = lse;
      }
    }
    if (lane == 0) tma_store_wait_all();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace attn_b200
