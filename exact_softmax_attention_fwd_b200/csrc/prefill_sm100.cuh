// prefill_sm100.cuh -- exact softmax attention forward (prefill) for sm_100a.
//
// What it computes ("Attention Kernel", section "问题与成本"):
//   O = softmax(Q K^T * scale + M) V,  LSE = ln sum exp(scale * Q K^T + M)
// blockwise with the online (m, l, o) recurrence ("Attention Kernel", section
// "Online softmax"; "Attention 算子加速史", section 1.3), so the S_q x S_k
// score matrix never leaves the chip.
//
// Persistent organisation: one CTA per SM (384 threads) walks a list of work
// units.  A unit is two 128-row query tiles of one (batch, query head): rows
// [256*qb, 256*qb + 256).  With a sliding window or a block mask (and an even
// number of query heads per KV head) a unit is instead one 128-row query
// tile of two query heads that share a KV head, so that both tiles stream the
// same key tiles (measured: +8 to +25 % on windows, +9 to +19 % on sparse
// block masks; on causal masks without them the staggered 256-row units
// overlap one tile's epilogue with the other's last step and stay faster).
// Units are ranked heaviest first (largest causal
// q-block first) and dealt to the CTAs in a back-and-forth ("snake") order so
// that every SM gets about the same number of KV tiles.  Inside a unit the
// loop order is query tile outside, KV tiles inside, with the accumulator
// resident on chip until one final write ("Attention 算子加速史", section 2.1).
//
//   * warp 0, lane 0  -- TMA producer: each unit's two Q tiles, then K_j and
//     V_j 128-key tiles into a STAGES-deep ring guarded by full/empty
//     mbarriers ("Attention 算子加速史", section 3.3: a producer warp,
//     mbarriers and multi-buffering; TMA as in section 3.1).  A Q tile of the
//     next unit is loaded as soon as the last MMA reading the current one
//     retires, and K/V of the next unit stream in while the current unit
//     finishes.  No multicast.
//   * warp 1           -- tcgen05 MMA issuer: S_i = Q_i K_j^T (SS form, both
//     operands in shared memory) and O_i += P_i V_j (TS form, P read from
//     tensor memory), ping-ponging between the two query tiles so that the
//     tensor core works on one tile while the other tile's softmax runs.  The
//     whole warp runs the schedule and the waits in uniform control flow and
//     one lane, picked by elect.sync, issues each group of MMAs: the
//     descriptors then stay in uniform registers, and a tile's MMAs go out
//     several times faster than from a lane-0-only branch.
//   * warps 2-3       -- idle (they complete the first warpgroup).
//   * warps 4-7 and 8-11 -- one softmax warpgroup per query tile; thread r of
//     a warpgroup owns row r (= TMEM lane r).  Per KV tile: load the S row
//     from TMEM, apply the causal / key-length predicate (boundary tiles
//     only; tiles that are wholly masked are never visited -- "Attention
//     Kernel", section "FlashAttention 的稳定基础"), update the running max,
//     write P = 2^(S*scale*log2e - m) as bf16 back into TMEM over the S
//     columns, rescale O in TMEM when the max moved, and hand P to the MMA
//     warp.  The division by l happens once per unit ("Attention 算子加速史",
//     section 2.2): each warp normalises its 32 rows, stages them (64 columns
//     at a time) in its own 4 KB shared-memory buffer and stores them by TMA.
//   * Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 and O_1
//     after them (d columns each); P_i aliases the first 64 columns of S_i.
//   * Registers: the kernel is built for 168 per thread (384 x 168 = 64512);
//     the producer/MMA warpgroup gives 112 of each thread's registers back
//     (setmaxnreg 56) and each softmax warpgroup takes 56 more (224):
//     128 x (56 + 224 + 224) = 64512, so the increase never waits.
//
// Rescaling is lazy: the max used as the exponent base only moves when the
// new row max exceeds it by more than 8 (log2 units), so P <= 2^8.  The final
// O = o / l and LSE are unchanged in exact arithmetic because the same base
// enters o and l.
//
// Empty rows (no visible key) get O = 0 and LSE = -inf: the exponent base
// falls back to 0 while the running max is -inf, so P = 2^-inf = 0 and l = 0.
#pragma once

#include <climits>

#include "sm100_primitives.cuh"

namespace attn_b200 {

struct PrefillParams {
  float* lse;           // [B, Hq, Sq] (ragged: [Hq, total_q]) or nullptr
  const int* k_lens;    // [B] or nullptr (fixed-length batches only)
  int B, Hq, Hkv, Sq, Sk;
  int group;            // Hq / Hkv
  float scale_log2;     // scale * log2(e)
  int n_qblocks;        // ceil(Sq / 256)
  // fixed-length units of 128 query rows x two query heads of one KV head
  // (Hq / Hkv even) instead of 256 rows x one head: both tiles then see the
  // same keys and share every K/V tile
  int head_pairs;
  // programmable masks (causal only; 0 = off): a row at key position p sees
  // keys (p - window, p] (sliding window), or keys below prefix as well (prefix-LM)
  int window, prefix;
  // block-sparse mask (MASKS instantiations; nullable): uint8 [B, mask_heads,
  // n_qt, n_kt] over 128 x 128 (query tile, key tile) blocks, 0 = skipped
  const uint8_t* block_mask;
  int mask_heads, n_qt, n_kt;
  // block masks shared by the heads: the unit rows (sequence, query block) are
  // ranked by their visible blocks in each CTA's prologue; the row count, or 0
  // to keep the causal ranking (see prefill_unit)
  int sched_rows;
  // ragged batches: packed token-major tensors, cumulative sequence lengths
  // and the unit list written by attn_varlen_schedule_kernel
  uint16_t* o;          // [total_q, Hq, d] bf16
  const int* cu_q;      // [B + 1]
  const int* cu_k;      // [B + 1] (ragged K/V) or nullptr (paged K/V)
  // paged K/V: [num_pages, page_size, Hkv, d] caches addressed by a block table
  const int* seq_lens_k;    // [B] keys of each sequence
  const int* block_table;   // [B, max_pages]
  int max_pages, page_size, num_pages;
  const int2* units;    // (sequence, query block), heaviest first
  const int* unit_count;
  int total_q;
};

// Most unit rows (sequence, query block) a block-mask launch ranks in shared
// memory; larger launches keep the causal ranking.
constexpr int kPrefillSchedMax = 768;

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;  // query rows per tile (MMA M, TMEM lanes)
  static constexpr int BN = 128;  // keys per KV tile
  static constexpr int STAGES = (D == 64) ? 4 : 2;
  static constexpr int TILE_BYTES = BM * D * 2;  // bf16 128 x D tile (Q, K or V)
  static constexpr int CB_BYTES = 128 * 128;     // one 64-column block of a 128-row tile
  static constexpr int NCB = D / 64;             // 64-column blocks per tile
  static constexpr int STG_BYTES = 32 * 128;     // per-warp epilogue staging: 32 rows x 64 cols
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_STG = OFF_V + STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_STG + 8 * STG_BYTES;
  // barrier indices
  static constexpr int B_QFULL = 0;                  // 2: Q_i landed
  static constexpr int B_QFREE = B_QFULL + 2;        // 2: last MMA reading Q_i retired
  static constexpr int B_KFULL = B_QFREE + 2;
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
  // masked instantiations: + the ranked block-mask unit rows (uint16)
  static constexpr int OFF_SCHED = OFF_MISC + 16;
  static constexpr int SMEM_BYTES_MASKS = SMEM_BYTES + 2 * kPrefillSchedMax;
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns of S_i (P_i aliases its first 64) and of O_i
  __host__ __device__ static constexpr uint32_t tmem_s(int i) { return i ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t tmem_o(int i) { return i ? 256u + D : 256u; }
  static constexpr int NUM_THREADS = 384;
  static constexpr uint32_t REGS_LAUNCH = 168;  // = 65536 / 384 rounded down to a multiple of 8
  static constexpr uint32_t REGS_PRODUCER = 56;
  static constexpr uint32_t REGS_SOFTMAX = 224;
  static_assert(128 * (REGS_PRODUCER + 2 * REGS_SOFTMAX) <= NUM_THREADS * REGS_LAUNCH,
                "register reallocation must fit the launch allocation");
  static_assert(128 * ((REGS_PRODUCER + 16) + 2 * (REGS_SOFTMAX - 16)) <= NUM_THREADS * REGS_LAUNCH,
                "the masked split must fit too");
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(SMEM_BYTES_MASKS <= 232448, "shared memory");
};

// Tensor layouts of a prefill kernel instantiation: dense [B, H, S, d]; a
// ragged batch of packed token-major [tokens, H, d] tensors; or packed
// queries over a paged K/V cache.
constexpr int kLayoutDense = 0;
constexpr int kLayoutRagged = 1;
constexpr int kLayoutPaged = 2;

// The 128-key tiles [lo, hi) the query tile with first row `row0` must visit
// (lo == hi: none).  A row at key position pos = i + (klen - Sq) (bottom-right
// causal alignment) sees keys [max(0, pos - window + 1), max(pos, prefix - 1)]
// within [0, klen) when causal (window / prefix 0 = off), all of [0, klen)
// otherwise; tiles outside the union over the tile's rows are skipped whole
// ("Attention Kernel", section "可编程 mask": block-level skipping, then an
// element-wise rule inside the tiles left).
__device__ __forceinline__ void prefill_kv_range(int row0, int Sq, int klen, bool causal,
                                                 int window, int prefix, int& lo, int& hi) {
  lo = hi = 0;
  if (row0 >= Sq) return;
  const long long off = (long long)klen - Sq;
  const int last_row = min(row0 + 127, Sq - 1);
  long long top = (long long)klen - 1;  // largest key any row of the tile sees
  long long bot = 0;                    // smallest
  if (causal) {
    top = min(top, max((long long)last_row + off, (long long)prefix - 1));
    if (window > 0) bot = max(0LL, (long long)row0 + off - window + 1);
  }
  if (top < bot) return;
  lo = (int)(bot / 128);
  hi = (int)(top / 128) + 1;
}

// Whether key tile kb is computed for the query tile starting at row0: inside
// the tile's range [kbeg, kend) and, with a block mask, not switched off.
__device__ __forceinline__ bool prefill_block_on(const PrefillParams& p, int b, int hq, int row0,
                                                 int kbeg, int kend, int kb) {
  if (kb < kbeg || kb >= kend) return false;
  if (p.block_mask == nullptr) return true;
  const size_t h = p.mask_heads == 1 ? 0 : (size_t)hq;
  return __ldg(p.block_mask + ((((size_t)b * p.mask_heads + h) * p.n_qt + row0 / 128) * p.n_kt +
                               kb)) != 0;
}

// One work unit: query rows [256*qb, 256*qb + 256) of head hq in sequence b.
struct PrefillUnit {
  int qb, hq, b;
  int hq_t[2];  // query head of each tile (hq, or hq and hq + 1 for head pairs)
  int sq;          // query rows of the sequence
  int klen;        // visible keys of the sequence
  int q_tok0;      // ragged batches: packed index of the sequence's first query
  int k_tok0;      //   and first key token (0 otherwise)
  int row0[2];     // first row of each query tile
  int kv_begin[2];  // KV tiles [kv_begin, kv_end) each query tile visits
  int kv_end[2];
  int kv_first;    // the unit's K/V stream: tiles [kv_first, kv_last)
  int kv_last;
};

// The k-th unit of this CTA, or false when the CTA has no more work.  Ranks
// are ordered heaviest first (q-blocks descending, heads inner) and dealt
// back and forth across the CTAs: rank k*G + c for even k, k*G + G-1-c for odd.
// For a ragged batch the (sequence, q-block) order comes from the unit list;
// for a block mask shared by the heads (p.sched_rows > 0) from `sched`, the
// rows (b, query block) sorted by visible blocks in the prologue, heads inner
// -- the random cost of such rows makes the causal ranking a poor proxy.
// MASKS: the instantiation honours p.window / p.prefix; without it both are
// the constant 0, so every range starts at tile 0 and the extra bounds fold away.
template <bool CAUSAL, int LAYOUT, bool MASKS>
__device__ __forceinline__ bool prefill_unit(const PrefillParams& p, int k, PrefillUnit& u,
                                             const uint16_t* sched = nullptr) {
  constexpr bool VARLEN = LAYOUT != kLayoutDense;
  const long long G = gridDim.x;
  const long long c = blockIdx.x;
  const long long r = (long long)k * G + ((k & 1) ? (G - 1 - c) : c);
  if (VARLEN) {
    if (r >= (long long)__ldg(p.unit_count) * p.Hq) return false;
    const int2 e = __ldg(&p.units[r / p.Hq]);
    u.hq = (int)(r % p.Hq);
    u.b = e.x;
    u.qb = e.y;
    u.q_tok0 = __ldg(p.cu_q + u.b);
    u.sq = __ldg(p.cu_q + u.b + 1) - u.q_tok0;  // listed sequences passed the
    if (LAYOUT == kLayoutPaged) {                  // schedule kernel's checks
      u.k_tok0 = 0;
      u.klen = __ldg(p.seq_lens_k + u.b);
    } else {
      u.k_tok0 = __ldg(p.cu_k + u.b);
      u.klen = __ldg(p.cu_k + u.b + 1) - u.k_tok0;
    }
  } else if (MASKS && p.head_pairs) {
    const int n_hp = p.Hq >> 1;
    const int n_qt = (p.Sq + 127) >> 7;
    if (p.sched_rows > 0) {
      if (r >= (long long)p.sched_rows * n_hp) return false;
      const int row = sched[r / n_hp];
      u.qb = row % n_qt;  // 128-row query tile
      u.b = row / n_qt;
      u.hq = 2 * (int)(r % n_hp);
    } else {
      const long long HB = (long long)n_hp * p.B;
      if (r >= (long long)n_qt * HB) return false;
      u.qb = n_qt - 1 - (int)(r / HB);  // 128-row query tile
      const int rem = (int)(r % HB);
      u.hq = 2 * (rem % n_hp);
      u.b = rem / n_hp;
    }
  } else if (MASKS && p.sched_rows > 0) {
    if (r >= (long long)p.sched_rows * p.Hq) return false;
    const int row = sched[r / p.Hq];
    u.qb = row % p.n_qblocks;
    u.b = row / p.n_qblocks;
    u.hq = (int)(r % p.Hq);
  } else {
    const long long HB = (long long)p.Hq * p.B;
    if (r >= (long long)p.n_qblocks * HB) return false;
    u.qb = p.n_qblocks - 1 - (int)(r / HB);
    const int rem = (int)(r % HB);
    u.hq = rem % p.Hq;
    u.b = rem / p.Hq;
  }
  if (!VARLEN) {
    int klen = p.Sk;
    if (p.k_lens != nullptr) {
      klen = p.k_lens[u.b];
      if (klen < 0 || klen > p.Sk) klen = klen < 0 ? 0 : p.Sk;  // flagged by the softmax warps
    }
    u.klen = klen;
    u.sq = p.Sq;
    u.q_tok0 = 0;
    u.k_tok0 = 0;
  }
  const bool pairs = MASKS && !VARLEN && p.head_pairs;
  u.kv_first = INT_MAX;
  u.kv_last = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    u.hq_t[i] = pairs ? u.hq + i : u.hq;
    u.row0[i] = pairs ? u.qb * 128 : u.qb * 256 + i * 128;
    prefill_kv_range(u.row0[i], u.sq, u.klen, CAUSAL, MASKS ? p.window : 0,
                     MASKS ? p.prefix : 0, u.kv_begin[i], u.kv_end[i]);
    if (MASKS && p.block_mask != nullptr) {
      // tighten the range to its first and last computed block, so that a
      // tile with no block left has an empty range (and no Q load)
      int lo = u.kv_begin[i], hi = u.kv_end[i];
      while (lo < hi && !prefill_block_on(p, u.b, u.hq_t[i], u.row0[i], lo, hi, lo)) ++lo;
      while (hi > lo && !prefill_block_on(p, u.b, u.hq_t[i], u.row0[i], lo, hi, hi - 1)) --hi;
      u.kv_begin[i] = lo < hi ? lo : 0;
      u.kv_end[i] = lo < hi ? hi : 0;
    }
    if (u.kv_end[i] > u.kv_begin[i]) {
      u.kv_first = min(u.kv_first, u.kv_begin[i]);
      u.kv_last = max(u.kv_last, u.kv_end[i]);
    }
  }
  if (u.kv_last == 0) u.kv_first = 0;
  return true;
}

template <int D, bool CAUSAL, int LAYOUT, bool MASKS>
__global__ void __launch_bounds__(384, 1)
    attn_prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ CUtensorMap tm_o, const PrefillParams p) {
  using C = PrefillCfg<D>;
  constexpr bool VARLEN = LAYOUT != kLayoutDense;
  constexpr bool PAGED = LAYOUT == kLayoutPaged;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sbase_ptr = smem_raw + (sbase - raw_addr);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase_ptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase_ptr + C::OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- setup: barriers (thread 0), tensor memory (warp 1)
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
      mbar_init(bar(C::B_VEMPTY + s), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    mbar_init_fence();
    fence_proxy_async_smem();
  }
  if (PAGED) {
    // K/V rows of a tile that no page fills (past the sequence's last page, or
    // a skipped page id) keep what the ring held before: zeros at first, then
    // earlier cache rows -- finite either way, and masked to weight 0.
    uint4* ring = reinterpret_cast<uint4*>(sbase_ptr + C::OFF_K);
    for (int x = threadIdx.x; x < 2 * C::STAGES * C::TILE_BYTES / 16; x += C::NUM_THREADS)
      ring[x] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  uint16_t* sched = reinterpret_cast<uint16_t*>(sbase_ptr + C::OFF_SCHED);
  if (MASKS && !VARLEN && p.sched_rows > 0) {
    // Rank the unit rows of a shared block mask by their computed blocks
    // (the MMA work of the row's query tiles), largest first and by index
    // among equals, so that every CTA derives the same order.  The costs sit
    // in the epilogue staging buffers, which are idle until the first unit ends.
    int* cost = reinterpret_cast<int*>(sbase_ptr + C::OFF_STG);
    const int n_q = p.head_pairs ? p.n_qt : p.n_qblocks;
    for (int t = threadIdx.x; t < p.sched_rows; t += C::NUM_THREADS) {
      const int b = t / n_q, qr = t % n_q;
      int klen = p.Sk;
      if (p.k_lens != nullptr) klen = min(max(__ldg(p.k_lens + b), 0), p.Sk);
      int c = 0;
      for (int i = 0; i < (p.head_pairs ? 1 : 2); ++i) {
        const int row0 = p.head_pairs ? qr * 128 : qr * 256 + i * 128;
        int lo, hi;
        prefill_kv_range(row0, p.Sq, klen, CAUSAL, p.window, p.prefix, lo, hi);
        const uint8_t* m = p.block_mask + ((size_t)b * p.n_qt + row0 / 128) * p.n_kt;
#pragma unroll 16
        for (int j = lo; j < hi; ++j) c += __ldg(m + j) != 0;
      }
      cost[t] = c;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < p.sched_rows; t += C::NUM_THREADS) {
      const int ct = cost[t];
      int rank = 0;
      for (int j = 0; j < p.sched_rows; ++j) {
        const int cj = cost[j];
        rank += (cj > ct) | ((cj == ct) & (j < t));
      }
      sched[rank] = (uint16_t)t;
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // Each register reallocation sits inside the branch of the warpgroup that
  // makes it, so that the compiler sees every role's code reachable only under
  // its own register budget.
  if (warp < 4) {
    // the masked instantiations keep more stream state in the MMA warp
    warpgroup_reg_dealloc<MASKS ? C::REGS_PRODUCER + 16 : C::REGS_PRODUCER>();
    if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      uint32_t q_loads0 = 0, q_loads1 = 0;  // Q tiles loaded so far, per tile slot
      uint32_t kv = 0;                      // K/V tiles issued so far (ring position)
      bool ok = true;
      auto load_q = [&](const PrefillUnit& u, int i) -> bool {
        uint32_t& n = i ? q_loads1 : q_loads0;
        if (n > 0 && !mbar_wait(bar(C::B_QFREE + i), (n - 1) & 1u, abort_flag)) return false;
        mbar_arrive_expect_tx(bar(C::B_QFULL + i), C::TILE_BYTES);
        // fixed-length maps are (d, Sq, B*Hq); ragged ones (d, Hq, total_q)
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_load_3d(sbase + C::OFF_Q + i * C::TILE_BYTES + cb * C::CB_BYTES, &tm_q,
                      bar(C::B_QFULL + i), 64 * cb, VARLEN ? u.hq : u.row0[i],
                      VARLEN ? u.q_tok0 + u.row0[i] : u.b * p.Hq + u.hq_t[i]);
        ++n;
        return true;
      };
      PrefillUnit u;
      for (int k = 0; ok && prefill_unit<CAUSAL, LAYOUT, MASKS>(p, k, u, sched); ++k) {
        const bool has0 = u.kv_end[0] > u.kv_begin[0], has1 = u.kv_end[1] > u.kv_begin[1];
        const int kvh = u.hq / p.group;
        const int kv_row = u.b * p.Hkv + kvh;
        if (PAGED) {  // warp 2 streams paged K/V; this thread only loads Q
          if (has0 && !(ok = load_q(u, 0))) break;
          if (has1 && !(ok = load_q(u, 1))) break;
          continue;
        }
        // Q_0 first (its slot frees first under a causal mask), then the first
        // K tile, then Q_1, so that no wait on Q_1 holds back the K/V stream.
        if (has0 && !(ok = load_q(u, 0))) break;
        for (int j = u.kv_first; j < u.kv_last; ++j) {
          // with a block mask, key tiles no query tile of the unit computes are not streamed
          if (MASKS && p.block_mask != nullptr &&
              !prefill_block_on(p, u.b, u.hq_t[0], u.row0[0], u.kv_begin[0], u.kv_end[0], j) &&
              !prefill_block_on(p, u.b, u.hq_t[1], u.row0[1], u.kv_begin[1], u.kv_end[1], j))
            continue;
          const int s = kv % C::STAGES;
          const uint32_t ph = (kv / C::STAGES) & 1u;
          if (!(ok = mbar_wait(bar(C::B_KEMPTY + s), ph ^ 1u, abort_flag))) break;
          mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::TILE_BYTES);
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_3d(sbase + C::OFF_K + s * C::TILE_BYTES + cb * C::CB_BYTES, &tm_k,
                        bar(C::B_KFULL + s), 64 * cb, VARLEN ? kvh : j * 128,
                        VARLEN ? u.k_tok0 + j * 128 : kv_row);
          if (j == u.kv_first && has1 && !(ok = load_q(u, 1))) {
            ++kv;  // K_0 of this unit was issued
            break;
          }
          if (!(ok = mbar_wait(bar(C::B_VEMPTY + s), ph ^ 1u, abort_flag))) {
            ++kv;
            break;
          }
          mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::TILE_BYTES);
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_3d(sbase + C::OFF_V + s * C::TILE_BYTES + cb * C::CB_BYTES, &tm_v,
                        bar(C::B_VFULL + s), 64 * cb, VARLEN ? kvh : j * 128,
                        VARLEN ? u.k_tok0 + j * 128 : kv_row);
          ++kv;
        }
      }
      // Drain: never leave the CTA with copies still landing in shared memory.
      // (On an abort the last K may lack its V; waiting on a V phase that was
      // never armed would only run into the time limit, so V is skipped then.)
      if (q_loads0 > 0) mbar_wait(bar(C::B_QFULL + 0), (q_loads0 - 1) & 1u, nullptr);
      if (q_loads1 > 0) mbar_wait(bar(C::B_QFULL + 1), (q_loads1 - 1) & 1u, nullptr);
      for (uint32_t j = (kv > C::STAGES ? kv - C::STAGES : 0); j < kv; ++j) {
        mbar_wait(bar(C::B_KFULL + j % C::STAGES), (j / C::STAGES) & 1u, nullptr);
        if (ok) mbar_wait(bar(C::B_VFULL + j % C::STAGES), (j / C::STAGES) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else if (PAGED && warp == 2) {
    // ================ paged K/V loader (all 32 lanes) ================
    // The 128-key tile j is 128 / page_size (<= 8) pages.  Lane t reads the
    // block-table entry of page t and issues that page's TMA boxes (page_size
    // rows of one KV head per 64-column block), so a tile's copies go out in
    // one pass of the warp.  The pool [num_pages, page_size, Hkv, d] is read as
    // the token-major tensor [num_pages * page_size, Hkv, d] (page p starts at
    // token p * page_size).  The barrier's byte count (valid pages, counted by
    // a ballot) is set by lane 0 before any copy is issued.
    constexpr int kNoPage = INT_MIN;  // past the sequence's last page
    uint32_t kv = 0;                  // K/V tiles issued so far (ring position)
    bool ok = true;
    PrefillUnit u;
    for (int k = 0; ok && prefill_unit<CAUSAL, LAYOUT, MASKS>(p, k, u, sched); ++k) {
      const int kvh = u.hq / p.group;
      const int ppt = 128 / p.page_size;
      const int n_lp = (u.klen + p.page_size - 1) / p.page_size;  // <= max_pages
      const int* tbl = p.block_table + (size_t)u.b * p.max_pages;
      const uint32_t row_off = (uint32_t)(lane * p.page_size * 128);
      for (int j = u.kv_first; j < u.kv_last; ++j, ++kv) {
        const int s = kv % C::STAGES;
        const uint32_t ph = (kv / C::STAGES) & 1u;
        const int lp = j * ppt + lane;
        const int phys = (lane < ppt && lp < n_lp) ? __ldg(tbl + lp) : kNoPage;
        const bool valid = phys >= 0 && phys < p.num_pages;
        if (phys != kNoPage && !valid) flag_device_error(kDevErrBadPage);  // skipped: its
        const uint32_t bytes = (uint32_t)__popc(__ballot_sync(0xffffffffu, valid)) *  // keys read
                               (uint32_t)(p.page_size * 128 * C::NCB);  // as earlier finite rows
        if (!(ok = mbar_wait_warp(bar(C::B_KEMPTY + s), ph ^ 1u, abort_flag))) break;
        if (lane == 0) mbar_arrive_expect_tx(bar(C::B_KFULL + s), bytes);
        __syncwarp();
        if (valid)
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_3d(sbase + C::OFF_K + s * C::TILE_BYTES + cb * C::CB_BYTES + row_off, &tm_k,
                        bar(C::B_KFULL + s), 64 * cb, kvh, phys * p.page_size);
        if (!(ok = mbar_wait_warp(bar(C::B_VEMPTY + s), ph ^ 1u, abort_flag))) {
          ++kv;  // K of this tile was issued
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(bar(C::B_VFULL + s), bytes);
        __syncwarp();
        if (valid)
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_3d(sbase + C::OFF_V + s * C::TILE_BYTES + cb * C::CB_BYTES + row_off, &tm_v,
                        bar(C::B_VFULL + s), 64 * cb, kvh, phys * p.page_size);
      }
    }
    // Drain as the producer does: no copy may still be landing at exit.
    if (lane == 0) {
      for (uint32_t j = (kv > C::STAGES ? kv - C::STAGES : 0); j < kv; ++j) {
        mbar_wait(bar(C::B_KFULL + j % C::STAGES), (j / C::STAGES) & 1u, nullptr);
        if (ok) mbar_wait(bar(C::B_VFULL + j % C::STAGES), (j / C::STAGES) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= tcgen05 MMA issuer =======================
    // The whole warp walks the schedule and waits; one elected lane issues
    // each group of MMAs and their commits (warp-uniform control flow keeps
    // the descriptors in uniform registers).
    {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      auto wait = [&](uint32_t b, uint32_t ph) -> bool {
        if (__all_sync(0xffffffffu, mbar_test(b, ph))) return true;
        const bool r = mbar_wait_slow(b, ph, abort_flag);
        return __all_sync(0xffffffffu, r);
      };
      auto issue_qk = [&](int i, int stage) {
        const uint64_t qd = smem_desc_sw128(opaque_u32(sbase + C::OFF_Q + i * C::TILE_BYTES), 16, 1024);
        const uint64_t kd = smem_desc_sw128(opaque_u32(sbase + C::OFF_K + stage * C::TILE_BYTES), 16, 1024);
        const uint32_t dt = tmem + C::tmem_s(i);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = (uint64_t)(((ks >> 2) * C::CB_BYTES + (ks & 3) * 32) >> 4);
          umma_ss(dt, qd + off, kd + off, idesc_qk, ks > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int stage, bool accumulate) {
        const uint64_t vd = smem_desc_sw128(opaque_u32(sbase + C::OFF_V + stage * C::TILE_BYTES), C::CB_BYTES, 1024);
        const uint32_t ts = opaque_u32(tmem + C::tmem_s(i));
        const uint32_t dt = tmem + C::tmem_o(i);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_ts(dt, ts + ks * 8, vd + (uint64_t)((ks * 2048) >> 4), idesc_pv,
                  (accumulate || ks > 0) ? 1u : 0u);
      };
      uint32_t kv = 0;                  // ring position
      uint32_t q_waits0 = 0, q_waits1 = 0;  // Q_FULL phases consumed per tile slot
      uint32_t p_waits0 = 0, p_waits1 = 0;  // P_FULL phases consumed per tile slot
      bool ok = true;
      PrefillUnit u;
      for (int k = 0; ok && prefill_unit<CAUSAL, LAYOUT, MASKS>(p, k, u, sched); ++k) {
        const int jb = u.kv_first, je = u.kv_last;  // the unit's K/V stream
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
        if (MASKS && p.block_mask != nullptr) {
          auto on = [&](int i, int kb) {
            return prefill_block_on(p, u.b, u.hq_t[i], u.row0[i], u.kv_begin[i], u.kv_end[i], kb);
          };
          auto next_pos = [&](int kb) {
            for (int x = kb + 1; x < je; ++x)
              if (on(0, x) || on(1, x)) return x;
            return -1;
          };
          uint32_t pos = 0;
          for (int kb = jb; ok && kb >= 0; ++pos) {
            const int kbn = next_pos(kb);
            const uint32_t idx = kv + pos;
            const int s = idx % C::STAGES;
            const int s1 = (idx + 1) % C::STAGES;
            if (!(ok = wait(bar(C::B_VFULL + s), (idx / C::STAGES) & 1u))) break;
            bool k_next = false;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              if (!ok) break;
              if (on(i, kb)) {
                uint32_t& pw = i ? p_waits1 : p_waits0;
                if (!(ok = wait(bar(C::B_PFULL + i), pw & 1u))) break;
                ++pw;
                tc_fence_after_sync();
                if (elect_one()) {
                  issue_pv(i, s, kb > u.kv_begin[i]);
                  if (kb == u.kv_end[i] - 1) umma_commit(bar(C::B_OFULL + i));
                }
                __syncwarp();
              }
              if (kbn >= 0 && on(i, kbn)) {
                if (!k_next) {
                  if (!(ok = wait(bar(C::B_KFULL + s1), ((idx + 1) / C::STAGES) & 1u))) break;
                  k_next = true;
                }
                if (kbn == u.kv_begin[i]) {
                  uint32_t& qw = i ? q_waits1 : q_waits0;
                  if (!(ok = wait(bar(C::B_QFULL + i), qw & 1u))) break;
                  ++qw;
                }
                tc_fence_after_sync();
                if (elect_one()) {
                  issue_qk(i, s1);
                  umma_commit(bar(C::B_SFULL + i));
                  if (kbn == u.kv_end[i] - 1) umma_commit(bar(C::B_QFREE + i));
                }
                __syncwarp();
              }
            }
            if (elect_one()) {
              umma_commit(bar(C::B_VEMPTY + s));
              if (k_next) umma_commit(bar(C::B_KEMPTY + s1));
            }
            __syncwarp();
            kb = kbn;
          }
          kv += pos;
          continue;
        }
        for (int j = jb; ok && j < je; ++j) {
          const uint32_t idx = kv + (uint32_t)(j - jb);
          const int s = idx % C::STAGES;
          const int s1 = (idx + 1) % C::STAGES;
          if (!(ok = wait(bar(C::B_VFULL + s), (idx / C::STAGES) & 1u))) break;
          bool k_next = false;  // K_(j+1) seen to have landed
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (!ok) break;
            const int b0 = u.kv_begin[i], e0 = u.kv_end[i];
            if (j < b0 || j >= e0) {
              if (MASKS && j + 1 == b0 && b0 < e0) {
                if (!k_next) {
                  if (!(ok = wait(bar(C::B_KFULL + s1), ((idx + 1) / C::STAGES) & 1u))) break;
                  k_next = true;
                }
                uint32_t& qw = i ? q_waits1 : q_waits0;
                if (!(ok = wait(bar(C::B_QFULL + i), qw & 1u))) break;
                ++qw;
                tc_fence_after_sync();
                if (elect_one()) {
                  issue_qk(i, s1);
                  umma_commit(bar(C::B_SFULL + i));
                  if (e0 == b0 + 1) umma_commit(bar(C::B_QFREE + i));
                }
                __syncwarp();
              }
              continue;
            }
            uint32_t& pw = i ? p_waits1 : p_waits0;
            if (!(ok = wait(bar(C::B_PFULL + i), pw & 1u))) break;
            ++pw;
            tc_fence_after_sync();
            const bool more = j + 1 < e0;
            if (more && !k_next) {
              // K_(j+1) is normally in long before P_i(j); wait for it first so
              // that PV and the next QK go out back to back
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
            umma_commit(bar(C::B_VEMPTY + s));
            if (k_next) umma_commit(bar(C::B_KEMPTY + s1));
          }
          __syncwarp();
        }
        kv += (uint32_t)(je - jb);
      }
      // Drain: every MMA issued above has completed before TMEM is released.
      if (elect_one()) umma_commit(bar(C::B_DRAIN));
      __syncwarp();
      mbar_wait(bar(C::B_DRAIN), 0, nullptr);
    }
    __syncwarp();
    }  // warps 2-3: nothing to do
  } else {
    warpgroup_reg_alloc<MASKS ? C::REGS_SOFTMAX - 16 : C::REGS_SOFTMAX>();
    // ======================= softmax warpgroups =======================
    const int i = (warp - 4) >> 2;       // query tile slot of this warpgroup
    const int quarter = warp & 3;        // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;   // row within the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + C::tmem_s(i);
    const uint32_t t_o = tmem + lane_off + C::tmem_o(i);
    const uint32_t stg = sbase + C::OFF_STG + (warp - 4) * C::STG_BYTES;
    uint8_t* stg_ptr = sbase_ptr + C::OFF_STG + (warp - 4) * C::STG_BYTES;
    float c2 = p.scale_log2;
    const bool scale_pos = c2 > 0.f;
    if (!scale_pos) c2 = 1.f;  // scores are pre-multiplied below instead
    uint32_t s_waits = 0, o_waits = 0;
    bool stores_pending = false;
    bool ok = true;
    PrefillUnit u;
    for (int k = 0; ok && prefill_unit<CAUSAL, LAYOUT, MASKS>(p, k, u, sched); ++k) {
      const int row0 = i ? u.row0[1] : u.row0[0];
      if (row0 >= u.sq) continue;  // this tile slot holds no rows in this unit
      const int kb = i ? u.kv_begin[1] : u.kv_begin[0];  // this tile's KV tiles [kb, ke)
      const int ke = i ? u.kv_end[1] : u.kv_end[0];
      const int row = row0 + r;
      const int hq_i = i ? u.hq_t[1] : u.hq_t[0];
      const int q_head_row = u.b * p.Hq + hq_i;
      if (!VARLEN && p.k_lens != nullptr && r == 0) {
        const int kl = p.k_lens[u.b];
        if (kl < 0 || kl > p.Sk) flag_device_error(kDevErrBadLength);
      }
      // visible keys of this row: [lo_row, hi_row]; a tile needs the per-element
      // rule unless every row of it sees all of it (j*128 >= lo_tile and
      // j*128 + 127 <= hi_tile, the tightest bounds over its rows)
      const long long koff = (long long)u.klen - u.sq;
      const int last_row = min(row0 + 127, u.sq - 1);
      long long hi_row = (long long)u.klen - 1, hi_tile = hi_row;
      long long lo_row = 0, lo_tile = 0;
      const int prefix = MASKS ? p.prefix : 0, window = MASKS ? p.window : 0;
      if (CAUSAL) {
        hi_row = min(hi_row, max((long long)row + koff, (long long)prefix - 1));
        hi_tile = min(hi_tile, max((long long)row0 + koff, (long long)prefix - 1));
        if (window > 0) {
          lo_row = max(0LL, (long long)row + koff - window + 1);
          lo_tile = max(0LL, (long long)last_row + koff - window + 1);
        }
      }
      float m_run = -INFINITY;   // exponent base (log2 units)
      float l_run = 0.f;         // sum of P (f32)
      float lr_run = 0.f;        // sum of bf16(P)

      for (int j = kb; j < ke; ++j) {
        if (MASKS && p.block_mask != nullptr && !prefill_block_on(p, u.b, hq_i, row0, kb, ke, j))
          continue;  // a block the mask switches off: no S, no P for it
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
        if ((long long)j * 128 + 127 > hi_tile || (MASKS && (long long)j * 128 < lo_tile)) {
          // boundary tile: per-element predicate, in 32-bit once clamped to the tile
          const long long hl = hi_row - (long long)j * 128;
          const long long ll = lo_row - (long long)j * 128;
          const int hi_local = hl < -1 ? -1 : (hl > 127 ? 127 : (int)hl);
          const int lo_local = ll < 0 ? 0 : (ll > 128 ? 128 : (int)ll);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > hi_local || (MASKS && c < lo_local)) s[c] = -INFINITY;
        }
        if (!scale_pos) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            s[c] = (s[c] == -INFINITY) ? -INFINITY : s[c] * p.scale_log2;
        }
        // row max: four chains of 3-input maxes
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
        if (m_tile > m_run + 8.f) {  // also true for the first finite max
          alpha = ex2(m_run - m_tile);
          m_run = m_tile;
        }
        const float base = (m_run == -INFINITY) ? 0.f : m_run;
        // P = 2^(s*c2 - base) two columns at a time (packed f32x2 FMA), two row
        // sums: l over the f32 P (gives the LSE) and lr over the bf16-rounded P
        // that the PV MMA consumes (normalises O, so the weights applied to V
        // sum to one exactly as used).
        const uint64_t c2x2 = f32x2(c2, c2);
        const uint64_t nbx2 = f32x2(-base, -base);
        uint64_t la = 0ull, lb = 0ull;                 // f32x2 partial sums of P
        float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;  // partial sums of bf16(P)
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
            pk[e] = pack_bf16x2(p0, p1);
            pk[e + 1] = pack_bf16x2(p2, p3);
            la = add_f32x2(la, f32x2(p0, p1));
            lb = add_f32x2(lb, f32x2(p2, p3));
            add_bf16x2_halves(pk[e], r0, r1);
            add_bf16x2_halves(pk[e + 1], r2, r3);
          }
          tmem_st32(t_s + 32 * half, pk);  // P columns [32*half, 32*half + 32)
        }
        l_run = l_run * alpha + (sum_f32x2(la) + sum_f32x2(lb));
        lr_run = lr_run * alpha + ((r0 + r1) + (r2 + r3));
        // Rescale the accumulator when any row of this warp moved its base.  The
        // MMA that last wrote O_i completed before S_i(j) was signalled.
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

      // ---- epilogue: O = o / l -> bf16; each warp stages its 32 rows, 64
      // columns at a time, in its own buffer and stores them by TMA; LSE per row.
      const bool has_o = ke > kb;
      if (has_o) {
        if (!(ok = mbar_wait_warp(bar(C::B_OFULL + i), o_waits & 1u, abort_flag))) break;
        ++o_waits;
      }
      tc_fence_after_sync();
      const float inv = (lr_run > 0.f) ? (1.f / lr_run) : 0.f;
      if constexpr (VARLEN) {
        // A TMA box could reach into the next sequence's rows, so each thread
        // writes its own row: d accumulator columns read from TMEM in one
        // batch, normalised, stored as 2d contiguous bytes in 16-byte pieces.
        uint32_t v[D / 32][32];
        if (has_o) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tmem_ld32(t_o + 32 * c, v[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) reg_fence32(v[c]);
        } else {
#pragma unroll
          for (int c = 0; c < D / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) v[c][e] = 0u;
        }
        if (row < u.sq) {
          const size_t tok = (size_t)u.q_tok0 + row;
          uint4* dst = reinterpret_cast<uint4*>(p.o + (tok * p.Hq + u.hq) * D);
#pragma unroll
          for (int q8 = 0; q8 < D / 8; ++q8) {  // 8 bf16 = 16 bytes per store
            const uint32_t* x = &v[q8 >> 2][(q8 & 3) * 8];
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv);
            dst[q8] = w;
          }
          if (p.lse != nullptr) {
            const float lse = (l_run > 0.f) ? (m_run + lg2(l_run)) * 0.69314718055994531f : -INFINITY;
            p.lse[(size_t)u.hq * p.total_q + tok] = lse;
          }
        }
      } else {
        const bool warp_has_rows = row0 + quarter * 32 < p.Sq;
#pragma unroll 1
        for (int cb = 0; cb < C::NCB; ++cb) {
          if (stores_pending) {  // the previous store must have read the buffer
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
              const int chunk = 4 * half + q4;  // 16-byte chunk within the 128-byte row
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * inv, __uint_as_float(v[8 * q4 + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * inv, __uint_as_float(v[8 * q4 + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * inv, __uint_as_float(v[8 * q4 + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * inv, __uint_as_float(v[8 * q4 + 7]) * inv);
              *reinterpret_cast<uint4*>(stg_ptr + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = w;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && warp_has_rows && !*abort_flag) {  // rows past Sq are clipped by the map
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
    }
    // all of this warp's output stores complete before the CTA exits
    if (lane == 0) tma_store_wait_all();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace attn_b200
