// paged_fp8_sm100.cuh -- the E4M3 pages a paged prefill reads, dequantised
// into a bf16 pool.
//
// "Attention Kernel", section "Paged 与 ragged KV" (key token t of sequence b
// lives at offset t mod page_size of the page block_table[b][t / page_size])
// and section "正确性契约" (the cache's quantisation schema is part of the
// contract): an E4M3 cache holds codes, element (page, r, h, i) being
// scale[page, h] * e4m3(code).  attn_fwd_paged_fp8 runs the bf16 paged
// prefill over the dequantised pages: this kernel writes, for every (sequence
// b, logical page pi) the sequence's length reaches, that page's K and V as
// bf16 (RN of scale * value) into slot b * max_pages + pi of a scratch pool,
// and the block table that maps the sequence onto those slots.  Slots past a
// sequence's last page, and pages whose id lies outside [0, num_pages), get
// table entry -1: the prefill kernel never reads the first and flags the
// second as it does for a bf16 cache.
#pragma once

#include "decode_sm100.cuh"

namespace attn_b200 {

// grid (max_pages, B), 256 threads: one logical page slot per CTA; each thread
// widens 16 consecutive codes (one 16-byte load, two 16-byte stores) at a time.
__global__ void __launch_bounds__(256)
    attn_dequant_pages_kernel(const uint8_t* k8, const uint8_t* v8, const float* k_scale,
                              const float* v_scale, const int* block_table, const int* seq_lens_k,
                              int page_size, int Hkv, int d, int max_pages, int num_pages,
                              uint16_t* k_out, uint16_t* v_out, int* table_out) {
  const int pi = blockIdx.x, b = blockIdx.y;
  const size_t slot = (size_t)b * max_pages + pi;
  int len = seq_lens_k[b];
  const long long cap = (long long)max_pages * page_size;
  if (len < 0) len = 0;
  if ((long long)len > cap) len = (int)cap;
  const int n_pages = (len + page_size - 1) / page_size;
  const int phys = pi < n_pages ? block_table[slot] : -1;
  const bool valid = phys >= 0 && phys < num_pages;
  if (threadIdx.x == 0) table_out[slot] = valid ? (int)slot : -1;
  if (!valid) return;
  const int per_page = page_size * Hkv * d;  // codes of one page, K (or V)
  const size_t src0 = (size_t)phys * per_page, dst0 = slot * per_page;
  for (int c = threadIdx.x * 16; c < 2 * per_page; c += blockDim.x * 16) {
    const bool is_v = c >= per_page;
    const int e = is_v ? c - per_page : c;       // element index within the page
    const int h = (e / d) % Hkv;                  // [page_size, Hkv, d]: 16 codes of one row
    const float sc = is_v ? __ldg(v_scale + (size_t)phys * Hkv + h)
                          : __ldg(k_scale + (size_t)phys * Hkv + h);
    const uint4 x = *reinterpret_cast<const uint4*>((is_v ? v8 : k8) + src0 + e);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = e4m3x2_to_f16x2(w[j]), hi = e4m3x2_to_f16x2(w[j] >> 16);
      o[2 * j] = pack_bf16x2(f16_to_f32(lo) * sc, f16_to_f32(lo >> 16) * sc);
      o[2 * j + 1] = pack_bf16x2(f16_to_f32(hi) * sc, f16_to_f32(hi >> 16) * sc);
    }
    uint4* dst = reinterpret_cast<uint4*>((is_v ? v_out : k_out) + dst0 + e);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace attn_b200
