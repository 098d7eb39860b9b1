// decode_sm100.cuh -- single-query attention over a paged KV cache, split
// along the keys, plus the deterministic merge of the splits.
//
// Sources: "Attention Kernel", sections "Paged 与 ragged KV" (logical token t
// lives in block t / page_size at offset t mod page_size; the block table
// gives the physical page) and "Prefill 与 decode 是两种 kernel" (decode is
// bound by KV bandwidth and indirect addressing); "Attention 算子加速史",
// section 4.1-4.2 (split-K decode: each split writes a partial output and its
// log-sum-exp, a light kernel merges them) and "Attention Kernel", section
// "Online softmax" (the merge rule).
//
// Split kernel: one warp (and CTA) per (sequence b, KV head, split of
// kSplitTokens tokens).  The warp serves all Hq/Hkv query heads that share the
// KV head (GQA), 16 tokens at a time, with warp-level MMAs:
//   S (heads x 16 tokens)  = q (16 padded heads x d) . K^T
//   O^T (d x heads)       += V^T (d x 16 tokens) . P^T (16 tokens x heads)
// The contraction index of each MMA may be permuted freely as long as both
// operands use the same permutation.  For K a thread owns a contiguous quarter
// of a row (16-byte loads); V^T's fragments come from transposing fragment
// loads (ldmatrix .trans) of 16-byte pieces of V rows, and for an E4M3 cache
// the token order of the scores is permuted to match the byte order those
// loads deliver.  K and V reach the warp through a ring of shared-memory slots filled by
// tensor-memory-access copies (see attn_decode_split_tma_kernel), so that the
// bytes in flight cost no registers.
//
// FP8 cache ("Attention Kernel", section "正确性契约": the cache quantisation
// schema is part of the contract; "Attention 算子加速史", section 3: FP8
// operands with scale factors): K and V may be stored as E4M3 bytes with one
// fp32 scale per (physical page, KV head).  The kernel then streams half the
// bytes and widens them to f16 right before use (exact: E4M3 has 3 mantissa
// bits and a narrower exponent range).  q K^T is an f16 MMA on q scaled by a
// power of two into f16's range; its fp32 scores are multiplied back and by
// the page's K scale.  P^T V is an f16 MMA that accumulates straight into the
// fp32 accumulator: the 16 tokens of a step always lie in one page, so the
// page's V scale enters as a factor vs / vmax (|.| <= 1, the scale's sign) on
// P before P is rounded to f16 (vmax = the largest V scale magnitude of the
// split's pages), and the accumulator, in units of vmax, is multiplied by vmax
// once at the end.  The normaliser sums the weights as applied to the
// dequantised V, f16(P') * vmax / vs per token (f16(P) on a page whose scale
// is zero).
//
// Rescaling is lazy, as in the prefill kernel: the exponent base of a head
// row moves only when the row max exceeds it by more than 8 (log2 units), so
// P <= 2^8 and the accumulator is rescaled only on the steps where some row
// of the warp moved its base.
//
// Merge kernel: one warp per (b, query head) combines the splits in a fixed
// order: LSE = M + log2 sum_s 2^(lse_s - M), O = sum_s 2^(lse_s - LSE) o_s,
// giving empty splits (lse = -inf) zero weight; no atomics, so the result is
// the same on every run.  Partial log-sum-exps are kept in log2 units inside
// the workspace; the final LSE is converted to the natural log.  It is launched
// as a programmatic dependent of the split kernel, so that its launch overlaps
// the split grid's drain; it waits for the split grid's writes before reading.
#pragma once

#include "sm100_primitives.cuh"

namespace attn_b200 {

constexpr int kSplitTokens = 512;

struct DecodeParams {
  const uint16_t* q;        // [B, Hq, D]
  const int* block_table;   // [B, max_pages]
  const int* seq_lens;      // [B]
  float* o_part;            // [B, Hq, n_split, D]
  float* lse_part;          // [B, Hq, n_split] (log2 units)
  uint16_t* o;              // [B, Hq, D] bf16
  float* lse;               // [B, Hq] or nullptr
  int B, Hq, Hkv, group, page_size, max_pages, num_pages, n_split;
  float scale_log2;
};

// Parameters of the split kernel: the decode parameters plus, for E4M3
// caches, the K and V scales (the cache pointers live in the tensor maps).
struct DecodeFp8Params {
  DecodeParams d;
  const float* k_scale;  // [num_pages, Hkv] (E4M3 caches only)
  const float* v_scale;
};

// Programmatic dependent launch: the merge grid may be launched while the
// split grid drains; it waits here for the split grid's writes.  Outside such
// a launch both instructions do nothing.
__device__ __forceinline__ void decode_wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void decode_allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ int decode_clamped_len(const DecodeParams& p, int b, bool report) {
  int len = p.seq_lens[b];
  const long long cap = (long long)p.max_pages * p.page_size;
  if (len < 0 || (long long)len > cap) {
    if (report) flag_device_error(kDevErrBadLength);
    len = len < 0 ? 0 : (int)cap;
  }
  return len;
}

// Two E4M3 bytes (bits 0-7 and 8-15) -> f16x2 (exact), element order kept.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((unsigned short)(two & 0xFFFFu)));
  return r;
}

// Four E4M3 bytes -> two f16x2 (exact): bytes 0-1 -> lo, bytes 2-3 -> hi.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t four, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(four));
}

__device__ __forceinline__ float f16_to_f32(uint32_t h16) {
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"((unsigned short)(h16 & 0xFFFFu)));
  return f;
}

// Two floats -> packed f16x2 (round to nearest even); `lo` lands in bits 0-15.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void mma_m16n8k16_f16(float (&c)[4], uint32_t a0, uint32_t a1,
                                                 uint32_t a2, uint32_t a3, uint32_t b0,
                                                 uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Split kernel with the K/V stream staged in shared memory by TMA.
//
// One warp (and CTA) per (sequence b, KV head, split of kSplitTokens tokens);
// the grid's x index runs over the KV heads of a split first, so that the
// warps reading the same pages run together.  The K and V rows of each step
// arrive by tensor-memory-access copies (cp.async.bulk.tensor, no multicast)
// into a STAGES-deep ring of shared memory, so the bytes in flight cost no
// registers: all slots are filled up front, and lane 0 refills a slot with
// step i + STAGES as soon as the warp has read step i out of it.  The cache is read by the copies as the token-major
// tensor [num_pages * page_size, Hkv, D] (page p starts at token p *
// page_size).  A step is NH chunks of 16 tokens (one for bf16 caches, two for
// E4M3 caches, whose rows are half as long, so that both move about the same
// bytes per step); a chunk never crosses a page (page sizes are multiples of
// 16), so it is one box of 16 rows x (up to) 128 bytes per 128-byte column
// block, for K and for V.  The boxes land 128-byte swizzled (64-byte for
// 64-byte rows), which keeps the fragment loads from shared memory free of
// bank conflicts.
//
// Each lane reads one block-table entry (and, for E4M3 caches, one pair of
// scales) up front: the split has at most 32 chunks, one per lane, and a
// chunk's page is fetched from its lane by a shuffle.  Tokens past the length
// and chunks on a page id outside the pool contribute exact zeros: their
// scores are set to -inf after the q K^T MMA (a K row only reaches its own
// score column) and their V fragments are zeroed after the shared-memory load,
// so stale or non-finite slot contents never reach the output; bad ids are
// flagged.
// ---------------------------------------------------------------------------
template <int D, bool FP8>
struct DecodeTmaCfg {
  static constexpr int NH = FP8 ? 2 : 1;           // 16-token chunks per step
  // ring depth: the bytes in flight per warp against the warps an SM holds
  // (shared memory per warp grows with the depth).  Measured on paged_decode:
  // 3 slots of 8 KB for bf16 (2 slots: -2%); 2 slots of 8 KB for E4M3, 12
  // warps per SM (3 slots: no gain, 4 slots: -15%)
  static constexpr int STAGES = FP8 ? 2 : 3;
  static constexpr int E = FP8 ? 1 : 2;            // bytes per element
  static constexpr int ROW = D * E;                // bytes per token row of one head
  static constexpr int BOX_BYTES = ROW < 128 ? ROW : 128;  // inner box extent in bytes
  static constexpr int NBOX = ROW / BOX_BYTES;     // column boxes per row
  static constexpr int TILE = 16 * ROW;            // 16 tokens of K (or V)
  static constexpr int CHUNK = 2 * TILE;           // K then V of one chunk
  static constexpr int STAGE = NH * CHUNK;
  static constexpr int SMEM = STAGES * STAGE + 64 + 1024;  // ring, barriers, alignment
  static_assert(kSplitTokens / 16 <= 32, "one block-table entry per lane");
};

// Byte offset inside a K or V tile of byte `byte` of token row `tok`, with the
// swizzle the copies apply (the 16-byte chunk index XOR the row within its
// 1024-byte (128-byte rows) or 512-byte (64-byte rows) atom).
template <int D, bool FP8>
__device__ __forceinline__ uint32_t dec_tile_off(int tok, int byte) {
  using C = DecodeTmaCfg<D, FP8>;
  const uint32_t box = (uint32_t)(byte / C::BOX_BYTES);
  const uint32_t a = (uint32_t)(tok * C::BOX_BYTES + byte % C::BOX_BYTES);
  const uint32_t sw = C::BOX_BYTES == 128 ? (a ^ ((a >> 3) & 0x70u)) : (a ^ ((a >> 3) & 0x30u));
  return box * (16u * C::BOX_BYTES) + sw;
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

__device__ __forceinline__ uint2 lds_u2(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

// Transposing fragment loads from shared memory (16-byte rows, one row
// address per lane).  m8n8.x4.b16: lanes 8i..8i+7 address the rows of matrix
// i; register i of lane t holds row t / 4, elements 2 (t % 4) and 2 (t % 4) + 1
// of the transposed matrix i.  m16n16.x1.b8: lanes 0-15 address rows 0-15;
// lane t receives rows 4 (t % 4) .. 4 (t % 4) + 3 of column t / 4 (register 0)
// and of column t / 4 + 8 (register 1), one byte each, in row order.
__device__ __forceinline__ void ldsm_x4_trans_b16(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_m16n16_trans_b8(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m16n16.x1.trans.shared.b8 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}

template <int D, bool FP8>
__global__ void __launch_bounds__(32, 8) attn_decode_split_tma_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const DecodeFp8Params f) {
  using C = DecodeTmaCfg<D, FP8>;
  constexpr int NH = C::NH;
  constexpr int KW = D * C::E / 16;   // 32-bit words of a thread's K quarter row
  const DecodeParams& p = f.d;
  decode_allow_dependents();  // the merge grid may start filling in as CTAs retire
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  const uint32_t bars = sbase + C::STAGES * C::STAGE;
  const int lane = threadIdx.x;
  const int kvh = (int)(blockIdx.x % (unsigned)p.Hkv);
  const int split = (int)(blockIdx.x / (unsigned)p.Hkv);
  const int b = blockIdx.z;
  const int len = decode_clamped_len(p, b, lane == 0 && split == 0 && kvh == 0);
  const int t_begin = split * kSplitTokens;
  if (t_begin >= len) return;  // the merge kernel never reads splits past the end
  const int t_end = min(t_begin + kSplitTokens, len);
  const int n_chunks = (t_end - t_begin + 15) / 16;
  const int n_steps = (n_chunks + NH - 1) / NH;
  const int g = lane >> 2;   // MMA group id: head row of S / P, d-row block of V^T
  const int tq = lane & 3;   // thread within the group
  const int hq0 = kvh * p.group;

  // q rows first: their loads need no page and overlap the block-table reads
  uint32_t qraw[D / 8];
  if (g < p.group) {
    const uint16_t* src = p.q + ((size_t)b * p.Hq + hq0 + g) * D + (D / 4) * tq;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) {
      const uint4 x = *reinterpret_cast<const uint4*>(src + 8 * w);
      qraw[4 * w + 0] = x.x;
      qraw[4 * w + 1] = x.y;
      qraw[4 * w + 2] = x.z;
      qraw[4 * w + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int w = 0; w < D / 8; ++w) qraw[w] = 0u;
  }

  // this lane's chunk: its page (or -1 when the id is outside the pool, or
  // past the split) and scales
  int my_page = -1;
  float my_ks = 0.f, my_vs = 0.f;
  if (lane < n_chunks) {
    const int t = t_begin + 16 * lane;
    const int pg = p.block_table[(size_t)b * p.max_pages + t / p.page_size];
    if (pg >= 0 && pg < p.num_pages) {
      my_page = pg;
      if (FP8) {
        my_ks = __ldg(f.k_scale + (size_t)pg * p.Hkv + kvh);
        my_vs = __ldg(f.v_scale + (size_t)pg * p.Hkv + kvh);
      }
    } else {
      flag_device_error(kDevErrBadPage);
    }
  }
  if (lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(bars + 8u * s, 1);
    mbar_init_fence();
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
  }
  __syncwarp();
  // Step i's copies into slot i % C::STAGES (lane 0; every lane takes part in
  // the shuffles).  Chunks on a bad page, or past the split, add no bytes.
  auto issue = [&](int i) {
    int pg[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) pg[h] = __shfl_sync(0xffffffffu, my_page, NH * i + h);
    if (lane == 0) {
      const int slot = i % C::STAGES;
      const uint32_t bar = bars + 8u * slot;
      uint32_t bytes = 0;
#pragma unroll
      for (int h = 0; h < NH; ++h) bytes += pg[h] >= 0 ? (uint32_t)C::CHUNK : 0u;
      fence_proxy_async_smem();  // the warp's reads of this slot precede the refill
      mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if (pg[h] < 0) continue;
        const uint32_t dst = sbase + slot * C::STAGE + h * C::CHUNK;
        const int tok = pg[h] * p.page_size + (t_begin + 16 * (NH * i + h)) % p.page_size;
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx) {
          const int col = bx * (C::BOX_BYTES / C::E);
          tma_load_3d(dst + bx * 16 * C::BOX_BYTES, &tm_k, bar, col, kvh, tok);
          tma_load_3d(dst + C::TILE + bx * 16 * C::BOX_BYTES, &tm_v, bar, col, kvh, tok);
        }
      }
    }
  };
  int n_issued = 0;
  for (; n_issued < C::STAGES && n_issued < n_steps; ++n_issued) issue(n_issued);
  // E4M3: the largest V scale magnitude of the split's pages (bad pages hold 0)
  float vmax = FP8 ? fabsf(my_vs) : 1.f;
  if (FP8) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    if (!(vmax > 0.f)) vmax = 1.f;
  }
  const float inv_vmax = FP8 ? 1.f / vmax : 1.f;
  // E4M3: this lane's chunk's factor on P (|.| <= 1) and the factor that takes
  // the applied weights back to weights on the dequantised V (0 marks a zero
  // scale, whose weights count as f16(P))
  const float my_rv = my_vs * inv_vmax;
  const float my_back = (FP8 && my_vs != 0.f) ? vmax / my_vs : 0.f;

  // q as the A operand (rows = heads, padded to 16; layout as the register
  // kernels).  E4M3 caches: f16 q scaled by 2^-qe into f16's range.
  uint32_t qa[D / 16][2];
  float qscale = 1.f;
  {
    const uint32_t (&raw)[D / 8] = qraw;
    if (!FP8) {
#pragma unroll
      for (int w = 0; w < D / 8; ++w) qa[w >> 1][w & 1] = raw[w];
    } else {
      float mxq = 0.f;
#pragma unroll
      for (int w = 0; w < D / 8; ++w)
        mxq = fmaxf(mxq, fmaxf(fabsf(__uint_as_float(raw[w] << 16)),
                               fabsf(__uint_as_float(raw[w] & 0xFFFF0000u))));
      mxq = fmaxf(mxq, __shfl_xor_sync(0xffffffffu, mxq, 1));
      mxq = fmaxf(mxq, __shfl_xor_sync(0xffffffffu, mxq, 2));
      int qe = 0;
      if (mxq >= 16384.f) qe = ilogbf(mxq) - 13;
      qscale = ldexpf(1.f, qe);
      const float qinv = ldexpf(1.f, -qe);
#pragma unroll
      for (int w = 0; w < D / 8; ++w)
        qa[w >> 1][w & 1] = pack_f16x2(__uint_as_float(raw[w] << 16) * qinv,
                                       __uint_as_float(raw[w] & 0xFFFF0000u) * qinv);
    }
  }

  const float my_kq = my_ks * qscale;  // E4M3: K scale times the power of two on q
  float c2 = p.scale_log2;
  const bool scale_pos = c2 > 0.f;
  if (!scale_pos) c2 = 1.f;
  float m_run = -INFINITY;  // exponent base of head row g (log2 units)
  float l_run = 0.f;        // sum of P (f32): the LSE
  float lr_run = 0.f;       // sum of the weights the MMA applies: normalises O
  float acc[D / 16][4];
#pragma unroll
  for (int mc = 0; mc < D / 16; ++mc) acc[mc][0] = acc[mc][1] = acc[mc][2] = acc[mc][3] = 0.f;

  int i = 0;
#pragma unroll 1
  for (; i < n_steps; ++i) {
    const int slot = i % C::STAGES;
    int n_here[NH];
    float kqc[NH], rvc[NH], backc[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const int c = NH * i + h;
      const int pg = __shfl_sync(0xffffffffu, my_page, c);
      n_here[h] = pg >= 0 ? min(16, t_end - (t_begin + 16 * c)) : 0;  // <= 0 past the end
      kqc[h] = FP8 ? __shfl_sync(0xffffffffu, my_kq, c) : 1.f;
      rvc[h] = FP8 ? __shfl_sync(0xffffffffu, my_rv, c) : 1.f;
      backc[h] = FP8 ? __shfl_sync(0xffffffffu, my_back, c) : 1.f;
    }
    const uint32_t st = sbase + slot * C::STAGE;
    const bool landed = mbar_wait(bars + 8u * slot, (uint32_t)(i / C::STAGES) & 1u, nullptr);
    if (!__all_sync(0xffffffffu, landed)) break;  // timed out: flagged, wind down

    // ---- S = q K^T (16 padded head rows x 16 tokens per chunk); two
    // independent accumulation chains (even and odd d-chunks), summed
    float s4[NH][4];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const uint32_t kt = st + h * C::CHUNK;
#pragma unroll
      for (int nc = 0; nc < 2; ++nc) {
        // the token in score column g of this MMA: for an E4M3 cache column 2j +
        // e of MMA nc is token 4j + 2nc + e, so that lane tq ends up with the
        // scores of tokens 4tq .. 4tq + 3, the rows its V fragments hold
        const int tok = FP8 ? 4 * (g >> 1) + 2 * nc + (g & 1) : nc * 8 + g;
        uint32_t kw[KW];
#pragma unroll
        for (int w = 0; w < KW / 4; ++w) {
          const uint4 x = lds_u4(kt + dec_tile_off<D, FP8>(tok, (D * C::E / 4) * tq + 16 * w));
          kw[4 * w + 0] = x.x;
          kw[4 * w + 1] = x.y;
          kw[4 * w + 2] = x.z;
          kw[4 * w + 3] = x.w;
        }
        float sx[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if (!FP8) {
#pragma unroll
          for (int kc = 0; kc < D / 16; ++kc)
            mma_m16n8k16_bf16(sx[kc & 1], qa[kc][0], 0u, qa[kc][1], 0u, kw[2 * kc], kw[2 * kc + 1]);
        } else {
#pragma unroll
          for (int kc = 0; kc < D / 16; ++kc) {
            uint32_t k0, k1;
            e4m3x4_to_f16x2x2(kw[kc], k0, k1);
            mma_m16n8k16_f16(sx[kc & 1], qa[kc][0], 0u, qa[kc][1], 0u, k0, k1);
          }
        }
        // this thread's scores of head row g: tokens 8nc + 2tq and 8nc + 2tq + 1
        const float kq = kqc[h];
        s4[h][2 * nc + 0] = (sx[0][0] + sx[1][0]) * kq;
        s4[h][2 * nc + 1] = (sx[0][1] + sx[1][1]) * kq;
      }
    }

    // ---- online softmax for head row g over this thread's 4 NH tokens
    float mx = -INFINITY;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      if (!scale_pos) {
#pragma unroll
        for (int e = 0; e < 4; ++e) s4[h][e] *= p.scale_log2;
      }
      // tokens past the length or on a bad page: their K rows may hold anything
      // (only their own score columns see them), masked here
      if (n_here[h] < 16) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((FP8 ? 4 * tq + e : (e >> 1) * 8 + 2 * tq + (e & 1)) >= n_here[h])
            s4[h][e] = -INFINITY;
      }
      mx = fmaxf(mx, fmaxf(fmaxf(s4[h][0], s4[h][1]), fmaxf(s4[h][2], s4[h][3])));
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    // lazy base: moves only when the max exceeds it by more than 8 (also true
    // for the first finite max; alpha = 2^-inf = 0 then, nothing accumulated)
    const float m_tile = mx * c2;
    float alpha = 1.f;
    if (m_tile > m_run + 8.f) {
      alpha = ex2(m_run - m_tile);
      m_run = m_tile;
    }
    const float base = (m_run == -INFINITY) ? 0.f : m_run;
    // P^T rows (tokens) 2tq, 2tq+1 and 2tq+8, 2tq+9 of each chunk, column g
    // (head): bf16 for a bf16 cache; for an E4M3 cache f16 of P * vs / vmax
    // (<= 2^8), and the weights on the dequantised V are f16(P') * vmax / vs
    uint32_t pb[NH][2];
    float rs = 0.f, rr = 0.f;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float pr[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pr[e] = ex2(fmaf(s4[h][e], c2, -base));
      rs += (pr[0] + pr[1]) + (pr[2] + pr[3]);
      if (!FP8) {
        pb[h][0] = pack_bf16x2(pr[0], pr[1]);
        pb[h][1] = pack_bf16x2(pr[2], pr[3]);
        rr += sum_f32x2(add_f32x2(bf16x2_to_f32x2(pb[h][0]), bf16x2_to_f32x2(pb[h][1])));
      } else {
        const float rv = rvc[h];  // |rv| <= 1, the sign of the scale
        pb[h][0] = pack_f16x2(pr[0] * rv, pr[1] * rv);
        pb[h][1] = pack_f16x2(pr[2] * rv, pr[3] * rv);
        if (backc[h] != 0.f) {
          rr += ((f16_to_f32(pb[h][0]) + f16_to_f32(pb[h][0] >> 16)) +
                 (f16_to_f32(pb[h][1]) + f16_to_f32(pb[h][1] >> 16))) * backc[h];
        } else {
          // a zero scale: the page's values add nothing, but its weights still
          // count in the normaliser (as f16, the rounding of the other pages)
          const uint32_t w0 = pack_f16x2(pr[0], pr[1]), w1 = pack_f16x2(pr[2], pr[3]);
          rr += (f16_to_f32(w0) + f16_to_f32(w0 >> 16)) + (f16_to_f32(w1) + f16_to_f32(w1 >> 16));
        }
      }
    }
    l_run = l_run * alpha + rs;
    lr_run = lr_run * alpha + rr;

    // ---- O^T += V^T P^T; accumulator columns are heads 2tq and 2tq+1, rows
    // d = 16 mc + g and 16 mc + g + 8.  The V^T fragments come from transposing
    // loads: bf16, the contraction runs over tokens 2tq, 2tq+1 (| +8); E4M3,
    // over tokens 4tq .. 4tq + 3 in the order of the scores above.
    uint32_t vw[NH][D / 16][FP8 ? 2 : 4];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const uint32_t vt = st + h * C::CHUNK + C::TILE;
#pragma unroll
      for (int mc = 0; mc < D / 16; ++mc) {
        if constexpr (FP8) {
          uint32_t r[2];
          ldsm_m16n16_trans_b8(r, vt + dec_tile_off<D, FP8>(lane & 15, 16 * mc));
          vw[h][mc][0] = r[0];
          vw[h][mc][1] = r[1];
        } else {
          uint32_t r[4];
          const int mi = lane >> 3;
          ldsm_x4_trans_b16(r, vt + dec_tile_off<D, FP8>((lane & 7) + 8 * (mi >> 1),
                                                         32 * mc + 16 * (mi & 1)));
          vw[h][mc][0] = r[0];
          vw[h][mc][1] = r[1];
          vw[h][mc][2] = r[2];
          vw[h][mc][3] = r[3];
        }
      }
      if (n_here[h] < 16) {  // masked tokens must not inject NaN
        if constexpr (FP8) {
          const int keep = min(max(n_here[h] - 4 * tq, 0), 4);  // bytes = tokens 4tq + b
          const uint32_t m = keep >= 4 ? 0xFFFFFFFFu : ((1u << (8 * keep)) - 1u);
#pragma unroll
          for (int mc = 0; mc < D / 16; ++mc) {
            vw[h][mc][0] &= m;
            vw[h][mc][1] &= m;
          }
        } else {
          const int t0 = 2 * tq;
          const uint32_t m_lo = (t0 < n_here[h] ? 0xFFFFu : 0u) | (t0 + 1 < n_here[h] ? 0xFFFF0000u : 0u);
          const uint32_t m_hi =
              (t0 + 8 < n_here[h] ? 0xFFFFu : 0u) | (t0 + 9 < n_here[h] ? 0xFFFF0000u : 0u);
#pragma unroll
          for (int mc = 0; mc < D / 16; ++mc) {
            vw[h][mc][0] &= m_lo;
            vw[h][mc][1] &= m_lo;
            vw[h][mc][2] &= m_hi;
            vw[h][mc][3] &= m_hi;
          }
        }
      }
    }
    __syncwarp();  // every lane has read the slot: refill it with step i + C::STAGES
    if (n_issued < n_steps) issue(n_issued++);
    if (__any_sync(0xffffffffu, alpha != 1.f)) {  // some head row moved its base
      const float a_h0 = __shfl_sync(0xffffffffu, alpha, (2 * tq) * 4);
      const float a_h1 = __shfl_sync(0xffffffffu, alpha, (2 * tq + 1) * 4);
#pragma unroll
      for (int mc = 0; mc < D / 16; ++mc) {
        acc[mc][0] *= a_h0;
        acc[mc][1] *= a_h1;
        acc[mc][2] *= a_h0;
        acc[mc][3] *= a_h1;
      }
    }
#pragma unroll
    for (int mc = 0; mc < D / 16; ++mc) {
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if constexpr (!FP8) {
          mma_m16n8k16_bf16(acc[mc], vw[h][mc][0], vw[h][mc][1], vw[h][mc][2], vw[h][mc][3],
                            pb[h][0], pb[h][1]);
        } else {
          uint32_t a0, a1, a2, a3;
          e4m3x4_to_f16x2x2(vw[h][mc][0], a0, a2);
          e4m3x4_to_f16x2x2(vw[h][mc][1], a1, a3);
          mma_m16n8k16_f16(acc[mc], a0, a1, a2, a3, pb[h][0], pb[h][1]);
        }
      }
    }
  }
  // after a timed-out wait: no copy may still be landing when the CTA exits
  // (steps [i, n_issued) were issued but not consumed; bounded waits)
  if (lane == 0)
    for (int j = i; j < n_issued; ++j)
      mbar_wait(bars + 8u * (j % C::STAGES), (uint32_t)(j / C::STAGES) & 1u, nullptr);
  __syncwarp();

  // ---- this split's normalised partial output and its log2-sum-exp (the
  // row sums were kept per lane: every lane of a head row shares its base)
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  lr_run += __shfl_xor_sync(0xffffffffu, lr_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  lr_run += __shfl_xor_sync(0xffffffffu, lr_run, 2);
  const int h0 = 2 * tq, h1 = 2 * tq + 1;
  const float l_h0 = __shfl_sync(0xffffffffu, lr_run, h0 * 4);
  const float l_h1 = __shfl_sync(0xffffffffu, lr_run, h1 * 4);
  const float inv0 = l_h0 > 0.f ? vmax / l_h0 : 0.f;  // vmax = 1 for a bf16 cache
  const float inv1 = l_h1 > 0.f ? vmax / l_h1 : 0.f;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int h = hh ? h1 : h0;
    if (h >= p.group) continue;
    const float inv = hh ? inv1 : inv0;
    float* dst = p.o_part + (((size_t)b * p.Hq + hq0 + h) * p.n_split + split) * D + g;
#pragma unroll
    for (int mc = 0; mc < D / 16; ++mc) {
      dst[16 * mc] = acc[mc][hh] * inv;
      dst[16 * mc + 8] = acc[mc][2 + hh] * inv;
    }
  }
  if (tq == 0 && g < p.group) {
    const float lse2 = l_run > 0.f ? m_run + lg2(l_run) : -INFINITY;
    p.lse_part[((size_t)b * p.Hq + hq0 + g) * p.n_split + split] = lse2;
  }
}

template <int D>
__global__ void __launch_bounds__(128) attn_decode_merge_kernel(const DecodeParams p) {
  constexpr int PER = D / 32;  // output columns per lane
  constexpr int R = 16;        // partial rows whose loads are in flight together
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x * 4 + warp;  // b * Hq + hq
  if (pair >= p.B * p.Hq) return;
  const int b = pair / p.Hq;
  const int len = decode_clamped_len(p, b, false);
  const int ns = (len + kSplitTokens - 1) / kSplitTokens;
  decode_wait_prior_grid();  // the split kernel's partials
  const float* lse_s = p.lse_part + (size_t)pair * p.n_split;
  const float* op = p.o_part + (size_t)pair * p.n_split * D + lane * PER;
  auto load_row = [&](float (&x)[PER], int s) {
    if constexpr (PER == 4) {
      const float4 v = *reinterpret_cast<const float4*>(op + (size_t)s * D);
      x[0] = v.x;
      x[1 % PER] = v.y;
      x[2 % PER] = v.z;
      x[3 % PER] = v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(op + (size_t)s * D);
      x[0] = v.x;
      x[1 % PER] = v.y;
    }
  };
  // the first R rows and the first 32 log-sum-exps in one round trip
  float x0[R][PER];
#pragma unroll
  for (int u = 0; u < R; ++u)
    if (u < ns) load_row(x0[u], u);
  const float l0 = lane < ns ? lse_s[lane] : -INFINITY;
  float mx = l0;
  for (int s = lane + 32; s < ns; s += 32) mx = fmaxf(mx, lse_s[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  if (mx != -INFINITY) {
    // rows in fixed order (split 0, 1, ...): deterministic
    float w_l = ex2(l0 - mx);
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const float w = __shfl_sync(0xffffffffu, w_l, u);
      if (u < ns) {
        wsum += w;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += w * x0[u][e];
      }
    }
    for (int s0 = R; s0 < ns; s0 += R) {
      if (s0 % 32 == 0) w_l = s0 + lane < ns ? ex2(lse_s[s0 + lane] - mx) : 0.f;
      float x[R][PER];
#pragma unroll
      for (int u = 0; u < R; ++u)
        if (s0 + u < ns) load_row(x[u], s0 + u);
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const float w = __shfl_sync(0xffffffffu, w_l, (s0 + u) & 31);
        if (s0 + u < ns) {
          wsum += w;
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] += w * x[u][e];
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint16_t* dst = p.o + (size_t)pair * D + lane * PER;
  if constexpr (PER == 4) {
    uint2 w;
    w.x = pack_bf16x2(acc[0] * inv, acc[1 % PER] * inv);
    w.y = pack_bf16x2(acc[2 % PER] * inv, acc[3 % PER] * inv);
    *reinterpret_cast<uint2*>(dst) = w;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1 % PER] * inv);
  }
  if (p.lse != nullptr && lane == 0)
    p.lse[pair] = wsum > 0.f ? (mx + lg2(wsum)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace attn_b200
