// attn_api.cu -- the C ABI declared in include/attn.h: argument checks on the
// host (before any CUDA call), TMA descriptor construction, and the launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "attn.h"
#include "bwd_sm100.cuh"
#include "decode_sm100.cuh"
#include "paged_fp8_sm100.cuh"
#include "prefill_fp8_sm100.cuh"
#include "prefill_sm100.cuh"
#include "sm100_primitives.cuh"
#include "varlen_schedule.cuh"

namespace attn_b200 {
namespace {

// Rows with no visible key at all (Sk = 0): O = 0, LSE = -inf.
__global__ void fill_empty_rows_kernel(uint4* o, size_t n_vec16, float* lse, size_t n_rows) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t e = i; e < n_vec16; e += stride) o[e] = make_uint4(0u, 0u, 0u, 0u);
  if (lse != nullptr)
    for (size_t e = i; e < n_rows; e += stride) lse[e] = -INFINITY;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled, looked up once (thread-safe static initialisation).
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// A tensor map is a pure function of (address, sizes, strides, box, layout),
// so encoded maps are kept in a small cache keyed by exactly those: repeated
// calls on the same buffers (a serving loop, a benchmark) skip the encode.
struct MapKey {
  const void* ptr;
  int kind;  // 0: [planes, rows, D] tiles; 1: token-major [tokens, heads, D]; 2, 3: E4M3 forms
  int D;
  long long a, b;  // rows, planes  |  heads, tokens
  unsigned box_rows;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && kind == o.kind && D == o.D && a == o.a && b == o.b &&
           box_rows == o.box_rows;
  }
};

class MapCache {
 public:
  bool find(const MapKey& k, CUtensorMap* out) {
    std::lock_guard<std::mutex> g(mu_);
    for (int i = 0; i < kSize; ++i)
      if (used_[i] && keys_[i] == k) {
        *out = maps_[i];
        return true;
      }
    return false;
  }
  void put(const MapKey& k, const CUtensorMap& m) {
    std::lock_guard<std::mutex> g(mu_);
    const int i = next_;
    next_ = (next_ + 1) % kSize;
    keys_[i] = k;
    maps_[i] = m;
    used_[i] = true;
  }

 private:
  static constexpr int kSize = 64;
  std::mutex mu_;
  MapKey keys_[kSize] = {};
  CUtensorMap maps_[kSize] = {};
  bool used_[kSize] = {};
  int next_ = 0;
};

MapCache& map_cache() {
  static MapCache c;
  return c;
}

bool encode_3d(CUtensorMap* map, const void* ptr, const cuuint64_t dims[3],
               const cuuint64_t strides[2], const cuuint32_t box[3],
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, dtype, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over a contiguous [planes, rows, D] tensor, box = box_rows rows
// x 64 columns, 128-byte swizzle (the layout the tcgen05 descriptors expect).
bool make_tile_map(CUtensorMap* map, const void* ptr, int D, long long rows, long long planes,
                   unsigned box_rows = 128) {
  const MapKey key{ptr, 0, D, rows, planes, box_rows};
  if (map_cache().find(key, map)) return true;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  if (!encode_3d(map, ptr, dims, strides, box)) return false;
  map_cache().put(key, *map);
  return true;
}

// 3-D bf16 map over a packed token-major [tokens, heads, D] tensor, box =
// box_rows tokens of one head x 64 columns, 128-byte swizzle: with 128 rows the
// same shared-memory tile as make_tile_map gives (128 rows of 128 bytes); a
// paged pool [num_pages, page_size, heads, D] is such a tensor with
// num_pages * page_size tokens, read one page (box_rows = page_size) at a time.
bool make_token_map(CUtensorMap* map, const void* ptr, int D, long long heads, long long tokens,
                    unsigned box_rows = 128) {
  const MapKey key{ptr, 1, D, heads, tokens, box_rows};
  if (map_cache().find(key, map)) return true;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  const cuuint32_t box[3] = {64, 1, box_rows};
  if (!encode_3d(map, ptr, dims, strides, box)) return false;
  map_cache().put(key, *map);
  return true;
}

// 3-D map over a paged E4M3 pool read as the token-major byte tensor
// [tokens, heads, D]: box = 16 tokens of one head x all D bytes of the row,
// 128-byte swizzle for 128-byte rows, 64-byte swizzle for 64-byte rows.
bool make_token_map_u8(CUtensorMap* map, const void* ptr, int D, long long heads,
                       long long tokens) {
  const MapKey key{ptr, 2, D, heads, tokens, 16u};
  if (map_cache().find(key, map)) return true;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)heads * D};
  const cuuint32_t box[3] = {(cuuint32_t)D, 1, 16};
  if (!encode_3d(map, ptr, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8,
                 D >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return false;
  map_cache().put(key, *map);
  return true;
}

// 3-D map over a contiguous E4M3 [planes, rows, D] tensor (one byte per
// element): box = 128 rows x all D bytes (D = 128: one 128-byte swizzle span).
bool make_tile_map_u8(CUtensorMap* map, const void* ptr, int D, long long rows,
                      long long planes) {
  const MapKey key{ptr, 3, D, rows, planes, 128u};
  if (map_cache().find(key, map)) return true;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)rows * D};
  const cuuint32_t box[3] = {(cuuint32_t)D, 128, 1};
  if (!encode_3d(map, ptr, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  map_cache().put(key, *map);
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Streaming multiprocessors of the current device (cached per device; the
// slots are atomics, so concurrent first calls at worst query twice).
int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// cudaFuncSetAttribute(kernel, max dynamic shared memory) once per kernel and
// device: `done` holds one bit per device for which it has been set.
template <typename Kernel>
bool set_smem_once(Kernel kern, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  done.fetch_or(bit, std::memory_order_release);
  return true;
}

// The unit-list kernel's shared memory grows with the level count; the limit
// is raised once per device to what the largest level count needs.
bool schedule_smem_ready() {
  static std::atomic<unsigned long long> done{0};
  return set_smem_once(attn_varlen_schedule_kernel, (2 * kVarlenMaxLevels + 32) * (int)sizeof(int),
                       done);
}

template <int D, bool CAUSAL, int LAYOUT = kLayoutDense, bool MASKS = false>
int launch_prefill(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const CUtensorMap& mo, const PrefillParams& prm, cudaStream_t stream,
                   long long max_units = 0) {
  using C = PrefillCfg<D>;
  constexpr bool VARLEN = LAYOUT != kLayoutDense;
  auto kern = attn_prefill_sm100_kernel<D, CAUSAL, LAYOUT, MASKS>;
  constexpr int smem = MASKS ? C::SMEM_BYTES_MASKS : C::SMEM_BYTES;
  static std::atomic<unsigned long long> smem_set{0};
  if (!set_smem_once(kern, smem, smem_set)) return ATTN_ERR_CUDA;
  // persistent: one CTA per SM (or fewer when there are fewer work units)
  const long long units =
      VARLEN ? max_units * prm.Hq
      : prm.head_pairs ? (long long)((prm.Sq + 127) / 128) * (prm.Hq / 2) * prm.B
                       : (long long)prm.n_qblocks * prm.Hq * prm.B;
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  dim3 grid((unsigned)(units < sms ? units : sms));
  kern<<<grid, C::NUM_THREADS, smem, stream>>>(mq, mk, mv, mo, prm);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int check_prefill_args(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int Sq, int Sk, int d, int causal, float scale,
                       const int32_t* k_lens) {
  if (q == nullptr || o == nullptr || (Sk > 0 && (k == nullptr || v == nullptr)))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Sk < 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hq > 65535) return ATTN_ERR_INVALID_ARG;  // grid extents
  if (Sq > (1 << 30) || Sk > (1 << 30)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(o) || (Sk > 0 && (!aligned16(k) || !aligned16(v))))
    return ATTN_ERR_ALIGNMENT;
  if ((lse != nullptr && !aligned4(lse)) || (k_lens != nullptr && !aligned4(k_lens)))
    return ATTN_ERR_ALIGNMENT;
  return ATTN_OK;
}

// Units of a ragged batch: sum over sequences of ceil(len_q / 256) is at most
// total_q / 256 + B for non-overlapping ranges; one more for rounding.
long long varlen_max_units(int B, long long total_q) { return total_q / 256 + B + 1; }

// Dense fixed-length prefill with optional key lengths, sliding window, prefix
// and block mask.
int prefill_dense(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Sq, int Sk, int d, int causal, float scale, const int32_t* k_lens,
                  int window, int prefix, const uint8_t* block_mask, int mask_heads,
                  cudaStream_t stream) {
  const long long rows_q = (long long)B * Hq * Sq;
  if (Sk == 0) {
    const size_t n_vec = (size_t)rows_q * d * 2 / 16;
    const int threads = 256;
    const long long want = ((long long)n_vec + threads - 1) / threads;
    const int blocks = (int)(want < 4096 ? (want > 0 ? want : 1) : 4096);
    fill_empty_rows_kernel<<<blocks, threads, 0, stream>>>(reinterpret_cast<uint4*>(o), n_vec, lse,
                                                           (size_t)rows_q);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  CUtensorMap mq, mk, mv, mo;
  if (!make_tile_map(&mq, q, d, Sq, (long long)B * Hq) ||
      !make_tile_map(&mk, k, d, Sk, (long long)B * Hkv) ||
      !make_tile_map(&mv, v, d, Sk, (long long)B * Hkv) ||
      !make_tile_map(&mo, o, d, Sq, (long long)B * Hq, 32))
    return ATTN_ERR_CUDA;
  PrefillParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.lse = lse;
  prm.k_lens = k_lens;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Sq = Sq;
  prm.Sk = Sk;
  prm.group = Hq / Hkv;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.n_qblocks = (Sq + 255) / 256;
  // windows and block masks: units of 128 rows x two query heads of one KV
  // head (both tiles stream the same key tiles)
  prm.head_pairs = (Hq / Hkv) % 2 == 0 && (window > 0 || block_mask != nullptr) ? 1 : 0;
  prm.window = window;
  prm.prefix = prefix;
  prm.block_mask = block_mask;
  prm.mask_heads = mask_heads;
  prm.n_qt = (Sq + 127) / 128;
  prm.n_kt = (Sk + 127) / 128;
  // a block mask shared by the heads: units ranked by their visible blocks
  const long long sched_rows = (long long)B * (prm.head_pairs ? prm.n_qt : prm.n_qblocks);
  if (block_mask != nullptr && mask_heads == 1 && sched_rows <= kPrefillSchedMax)
    prm.sched_rows = (int)sched_rows;
  if (window > 0 || prefix > 0 || block_mask != nullptr) {  // window / prefix need causal
    if (d == 128)
      return causal ? launch_prefill<128, true, kLayoutDense, true>(mq, mk, mv, mo, prm, stream)
                    : launch_prefill<128, false, kLayoutDense, true>(mq, mk, mv, mo, prm, stream);
    return causal ? launch_prefill<64, true, kLayoutDense, true>(mq, mk, mv, mo, prm, stream)
                  : launch_prefill<64, false, kLayoutDense, true>(mq, mk, mv, mo, prm, stream);
  }
  if (d == 128)
    return causal ? launch_prefill<128, true>(mq, mk, mv, mo, prm, stream)
                  : launch_prefill<128, false>(mq, mk, mv, mo, prm, stream);
  return causal ? launch_prefill<64, true>(mq, mk, mv, mo, prm, stream)
                : launch_prefill<64, false>(mq, mk, mv, mo, prm, stream);
}
// Backward: the row-statistics pass, then dK/dV (one CTA per key tile and KV
// head), then dQ (one CTA per query tile and query head) as a programmatic
// dependent of dK/dV.
template <int D, bool CAUSAL, bool VARLEN = false, bool MASKS = false>
int launch_bwd(const CUtensorMap& mq, const CUtensorMap& mdo, const CUtensorMap& mk,
               const CUtensorMap& mv, const BwdParams& prm, cudaStream_t stream) {
  using C = BwdCfg<D>;
  const long long prep_threads = (long long)prm.B * prm.Hq * prm.Sq_pad * (D / 8);
  const long long prep_blocks = (prep_threads + 255) / 256;
  const long long kv_units = (long long)prm.n_kt * prm.B * prm.Hkv;
  const long long q_units = (long long)prm.n_qt * prm.B * prm.Hq;
  if (prep_blocks > INT_MAX || kv_units > INT_MAX || q_units > INT_MAX) return ATTN_ERR_INVALID_ARG;
  attn_bwd_prep_kernel<D, VARLEN><<<(unsigned)prep_blocks, 256, 0, stream>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  // the masked instantiations keep a list of the blocks they walk in shared memory
  constexpr int kv_smem = MASKS ? C::KV_SMEM_MASKS : C::KV_SMEM;
  constexpr int q_smem = MASKS ? C::Q_SMEM_MASKS : C::Q_SMEM;
  auto kv = attn_bwd_dkdv_kernel<D, CAUSAL, VARLEN, MASKS>;
  static std::atomic<unsigned long long> kv_smem_set{0};
  if (!set_smem_once(kv, kv_smem, kv_smem_set)) return ATTN_ERR_CUDA;
  kv<<<(unsigned)kv_units, C::NUM_THREADS, kv_smem, stream>>>(mq, mdo, mk, mv, prm);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  auto dq = attn_bwd_dq_kernel<D, CAUSAL, VARLEN, MASKS>;
  static std::atomic<unsigned long long> q_smem_set{0};
  if (!set_smem_once(dq, q_smem, q_smem_set)) return ATTN_ERR_CUDA;
  // dQ as a programmatic dependent of dK/dV (it reads only the inputs and the
  // prep kernel's statistics, complete before dK/dV started)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)q_units);
  cfg.blockDim = dim3(C::NUM_THREADS);
  cfg.dynamicSmemBytes = q_smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, dq, mq, mdo, mk, mv, prm) != cudaSuccess) return ATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool FP8>
int launch_decode_split(const CUtensorMap& mk, const CUtensorMap& mv, const DecodeFp8Params& pf,
                        dim3 grid, cudaStream_t stream) {
  using C = DecodeTmaCfg<D, FP8>;
  auto kern = attn_decode_split_tma_kernel<D, FP8>;
  static std::atomic<unsigned long long> smem_set{0};
  if (!set_smem_once(kern, C::SMEM, smem_set)) return ATTN_ERR_CUDA;
  kern<<<grid, 32, C::SMEM, stream>>>(mk, mv, pf);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Paged decode over a bf16 cache, or (fp8) an E4M3 cache with per-(page, KV
// head) scales: validation, then the split kernel and the merge kernel.
int decode_paged_common(bool fp8, const void* q, const void* k_cache, const void* v_cache,
                        const float* k_scale, const float* v_scale, const int32_t* block_table,
                        const int32_t* seq_lens, int page_size, int B, int Hq, int Hkv, int d,
                        int max_pages_per_seq, int num_pages, float scale, void* o, float* lse,
                        void* workspace, size_t workspace_bytes, attn_stream_t stream_) {
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || block_table == nullptr ||
      seq_lens == nullptr || o == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || max_pages_per_seq < 1 || num_pages < 1 ||
      page_size < 1)
    return ATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535 || (long long)max_pages_per_seq * page_size > (1ll << 30) ||
      (long long)num_pages * page_size > 0x7fffffffLL)
    return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (page_size % 16 != 0 || page_size > 256) return ATTN_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      !aligned4(block_table) || !aligned4(seq_lens) || (lse != nullptr && !aligned4(lse)))
    return ATTN_ERR_ALIGNMENT;
  if (fp8 && (!aligned4(k_scale) || !aligned4(v_scale))) return ATTN_ERR_ALIGNMENT;
  // the split kernel's grid x runs over (split, KV head) pairs
  const long long n_split_ll = ((long long)max_pages_per_seq * page_size + kSplitTokens - 1) / kSplitTokens;
  if (n_split_ll * Hkv > INT_MAX) return ATTN_ERR_INVALID_ARG;
  const size_t need = attn_decode_workspace_size(B, Hq, max_pages_per_seq, page_size, d);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGNMENT;

  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const long long tokens = (long long)max_pages_per_seq * page_size;
  DecodeParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.q = static_cast<const uint16_t*>(q);
  prm.block_table = block_table;
  prm.seq_lens = seq_lens;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.page_size = page_size;
  prm.max_pages = max_pages_per_seq;
  prm.num_pages = num_pages;
  prm.n_split = (int)((tokens + kSplitTokens - 1) / kSplitTokens);
  prm.scale_log2 = scale * 1.4426950408889634f;
  const size_t parts = (size_t)B * Hq * prm.n_split;
  prm.o_part = static_cast<float*>(workspace);
  prm.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + parts * d * sizeof(float));
  prm.o = static_cast<uint16_t*>(o);
  prm.lse = lse;

  DecodeFp8Params pf;
  pf.d = prm;
  pf.k_scale = k_scale;
  pf.v_scale = v_scale;
  // K/V reach the split kernel through tensor maps over the pool, read as the
  // token-major tensor [num_pages * page_size, Hkv, d]
  CUtensorMap mk, mv;
  const long long pool_tokens = (long long)num_pages * page_size;
  const bool maps_ok =
      fp8 ? make_token_map_u8(&mk, k_cache, d, Hkv, pool_tokens) &&
                make_token_map_u8(&mv, v_cache, d, Hkv, pool_tokens)
          : make_token_map(&mk, k_cache, d, Hkv, pool_tokens, 16) &&
                make_token_map(&mv, v_cache, d, Hkv, pool_tokens, 16);
  if (!maps_ok) return ATTN_ERR_CUDA;
  dim3 grid_split((unsigned)((long long)prm.n_split * Hkv), 1, B);
  dim3 grid_merge((unsigned)(((long long)B * Hq + 3) / 4));
  int st = ATTN_OK;
  if (d == 128)
    st = fp8 ? launch_decode_split<128, true>(mk, mv, pf, grid_split, stream)
             : launch_decode_split<128, false>(mk, mv, pf, grid_split, stream);
  else
    st = fp8 ? launch_decode_split<64, true>(mk, mv, pf, grid_split, stream)
             : launch_decode_split<64, false>(mk, mv, pf, grid_split, stream);
  if (st != ATTN_OK) return st;
  // the merge kernel as a programmatic dependent of the split kernel: its
  // launch overlaps the split grid's drain, its reads wait for the writes
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid_merge;
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = d == 128 ? cudaLaunchKernelEx(&cfg, attn_decode_merge_kernel<128>, prm)
                                 : cudaLaunchKernelEx(&cfg, attn_decode_merge_kernel<64>, prm);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int check_paged_prefill_args(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_table, const int32_t* cu_seqlens_q,
                             const int32_t* seq_lens_k, int page_size, int B, int Hq, int Hkv,
                             long long total_q, int max_seqlen_q, int max_pages_per_seq,
                             int num_pages, int d, int causal, float scale, void* o, float* lse) {
  if (q == nullptr || o == nullptr || k_cache == nullptr || v_cache == nullptr ||
      block_table == nullptr || cu_seqlens_q == nullptr || seq_lens_k == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
  if (total_q < 0 || total_q > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_q < 1 || max_seqlen_q > kVarlenMaxLevels * 256) return ATTN_ERR_INVALID_ARG;
  if (max_pages_per_seq < 1 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
  if ((long long)max_pages_per_seq * page_size > 0x7fffffffLL ||
      (long long)num_pages * page_size > 0x7fffffffLL)
    return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128)
    return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(o) || !aligned16(k_cache) || !aligned16(v_cache))
    return ATTN_ERR_ALIGNMENT;
  if ((lse != nullptr && !aligned4(lse)) || !aligned4(cu_seqlens_q) || !aligned4(seq_lens_k) ||
      !aligned4(block_table))
    return ATTN_ERR_ALIGNMENT;
  return ATTN_OK;
}

// The paged prefill proper: the unit list in `workspace`, then the prefill
// kernel over a bf16 pool (arguments already checked).
int paged_prefill_run(const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_table, const int32_t* cu_seqlens_q,
                      const int32_t* seq_lens_k, int page_size, int B, int Hq, int Hkv,
                      long long total_q, int max_seqlen_q, int max_pages_per_seq, int num_pages,
                      int d, int causal, float scale, void* o, float* lse, void* workspace,
                      cudaStream_t stream) {
  int* unit_count = static_cast<int*>(workspace);
  int2* units = reinterpret_cast<int2*>(static_cast<char*>(workspace) + 16);
  const long long max_units = varlen_max_units(B, total_q);
  const int max_keys = max_pages_per_seq * page_size;
  int shift, n_levels;
  varlen_levels(max_keys, shift, n_levels);
  const size_t sched_smem = (size_t)(2 * n_levels + 32) * sizeof(int);
  if (!schedule_smem_ready()) return ATTN_ERR_CUDA;
  attn_varlen_schedule_kernel<<<1, 1024, sched_smem, stream>>>(
      cu_seqlens_q, nullptr, seq_lens_k, B, (int)total_q, 0, max_seqlen_q, max_keys, causal,
      0, 0, shift, n_levels, units, unit_count, (int)max_units);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  if (!make_token_map(&mq, q, d, Hq, total_q) ||
      !make_token_map(&mk, k_cache, d, Hkv, (long long)num_pages * page_size, page_size) ||
      !make_token_map(&mv, v_cache, d, Hkv, (long long)num_pages * page_size, page_size))
    return ATTN_ERR_CUDA;
  PrefillParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.lse = lse;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.o = static_cast<uint16_t*>(o);
  prm.cu_q = cu_seqlens_q;
  prm.seq_lens_k = seq_lens_k;
  prm.block_table = block_table;
  prm.max_pages = max_pages_per_seq;
  prm.page_size = page_size;
  prm.num_pages = num_pages;
  prm.units = units;
  prm.unit_count = unit_count;
  prm.total_q = (int)total_q;
  if (d == 128)
    return causal ? launch_prefill<128, true, kLayoutPaged>(mq, mk, mv, mq, prm, stream, max_units)
                  : launch_prefill<128, false, kLayoutPaged>(mq, mk, mv, mq, prm, stream, max_units);
  return causal ? launch_prefill<64, true, kLayoutPaged>(mq, mk, mv, mq, prm, stream, max_units)
                : launch_prefill<64, false, kLayoutPaged>(mq, mk, mv, mq, prm, stream, max_units);
}

// ---------------------------------------------------------------------------
// Prefill from and to host memory: the batch is cut into chunks of whole
// (batch, KV head) pairs -- contiguous in every tensor -- and each chunk's
// host-to-device copies, prefill launch and device-to-host copies run on
// three streams (two copy streams owned by the library, the caller's stream
// for the kernels) through two device buffer sets, so that copies of one
// chunk overlap the kernels of another.
// ---------------------------------------------------------------------------
struct HostPipelineLayout {
  int pairs_per_chunk, n_chunks;
  size_t q_bytes, kv_bytes, lse_bytes;  // per chunk
  size_t q_off[2], k_off[2], v_off[2], o_off[2], lse_off[2], klen_off, total;
};

HostPipelineLayout host_pipeline_layout(int B, int Hq, int Hkv, int Sq, int Sk, int d) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  HostPipelineLayout L;
  const long long pairs = (long long)B * Hkv;
  const int G = Hq / Hkv;
  // about eight chunks: enough to overlap, few enough that each launch is large
  L.pairs_per_chunk = (int)((pairs + 7) / 8);
  L.n_chunks = (int)((pairs + L.pairs_per_chunk - 1) / L.pairs_per_chunk);
  L.q_bytes = (size_t)L.pairs_per_chunk * G * Sq * d * 2;
  L.kv_bytes = (size_t)L.pairs_per_chunk * Sk * d * 2;
  L.lse_bytes = (size_t)L.pairs_per_chunk * G * Sq * 4;
  size_t off = 0;
  for (int sl = 0; sl < 2; ++sl) {
    L.q_off[sl] = off;
    off += up(L.q_bytes);
    L.k_off[sl] = off;
    off += up(L.kv_bytes);
    L.v_off[sl] = off;
    off += up(L.kv_bytes);
    L.o_off[sl] = off;
    off += up(L.q_bytes);
    L.lse_off[sl] = off;
    off += up(L.lse_bytes);
  }
  L.klen_off = off;  // key length of every (batch, KV head) pair
  off += up((size_t)pairs * 4);
  L.total = off;
  return L;
}

// Two copy streams and the events of the two buffer sets, created once per
// device and kept for the life of the process.  A call holds its device's
// mutex while it enqueues, so that calls from several host threads do not
// interleave their event records.
struct HostPipelineRes {
  std::mutex mu;
  cudaStream_t h2d, d2h;
  cudaEvent_t start, h2d_done[2], comp_done[2], d2h_done[2];
  bool ready;
};

constexpr int kMaxPipelineDevices = 64;

// On success the device's mutex is held; the caller releases it.
int host_pipeline_res(HostPipelineRes** out) {
  static HostPipelineRes res[kMaxPipelineDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxPipelineDevices) return ATTN_ERR_CUDA;
  HostPipelineRes& r = res[dev];
  r.mu.lock();
  if (!r.ready) {
    const unsigned fl = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&r.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&r.d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&r.start, fl) != cudaSuccess) {
      r.mu.unlock();
      return ATTN_ERR_CUDA;
    }
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&r.h2d_done[i], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&r.comp_done[i], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&r.d2h_done[i], fl) != cudaSuccess) {
        r.mu.unlock();
        return ATTN_ERR_CUDA;
      }
    r.ready = true;
  }
  *out = &r;
  return ATTN_OK;
}

int host_pipeline_enqueue(HostPipelineRes* R, const HostPipelineLayout& L, const void* q,
                          const void* k, const void* v, void* o, float* lse, int B, int Hq,
                          int Hkv, int Sq, int Sk, int d, int causal, float scale,
                          const int32_t* k_lens, char* ws, cudaStream_t stream) {
  int st = ATTN_OK;
  const int G = Hq / Hkv;
  const long long pairs = (long long)B * Hkv;
  int32_t* klen_dev = reinterpret_cast<int32_t*>(ws + L.klen_off);
  // the copy streams start after the caller's earlier work
  if (cudaEventRecord(R->start, stream) != cudaSuccess ||
      cudaStreamWaitEvent(R->h2d, R->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(R->d2h, R->start, 0) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (k_lens != nullptr) {
    // one key length per (batch, KV head) pair: the chunks are batches of pairs
    std::vector<int32_t> per_pair((size_t)pairs);
    for (long long pr = 0; pr < pairs; ++pr) per_pair[(size_t)pr] = k_lens[pr / Hkv];
    if (cudaMemcpyAsync(klen_dev, per_pair.data(), (size_t)pairs * 4, cudaMemcpyHostToDevice,
                        stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)  // per_pair is freed on return
      return ATTN_ERR_CUDA;
  }
  const char* qh = static_cast<const char*>(q);
  const char* kh = static_cast<const char*>(k);
  const char* vh = static_cast<const char*>(v);
  char* oh = static_cast<char*>(o);
  char* lh = reinterpret_cast<char*>(lse);
  const size_t q_pair = (size_t)G * Sq * d * 2, kv_pair = (size_t)Sk * d * 2,
               l_pair = (size_t)G * Sq * 4;
  for (int c = 0; c < L.n_chunks; ++c) {
    const int sl = c & 1;
    const long long p0 = (long long)c * L.pairs_per_chunk;
    const int np = (int)(p0 + L.pairs_per_chunk <= pairs ? L.pairs_per_chunk : pairs - p0);
    char* qd = ws + L.q_off[sl];
    char* kd = ws + L.k_off[sl];
    char* vd = ws + L.v_off[sl];
    char* od = ws + L.o_off[sl];
    float* ld = reinterpret_cast<float*>(ws + L.lse_off[sl]);
    // inputs into buffer set sl once the kernels of chunk c - 2 are done with it
    if (c >= 2 && cudaStreamWaitEvent(R->h2d, R->comp_done[sl], 0) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaMemcpyAsync(qd, qh + p0 * q_pair, np * q_pair, cudaMemcpyHostToDevice, R->h2d) !=
            cudaSuccess ||
        (Sk > 0 && (cudaMemcpyAsync(kd, kh + p0 * kv_pair, np * kv_pair, cudaMemcpyHostToDevice,
                                    R->h2d) != cudaSuccess ||
                    cudaMemcpyAsync(vd, vh + p0 * kv_pair, np * kv_pair, cudaMemcpyHostToDevice,
                                    R->h2d) != cudaSuccess)) ||
        cudaEventRecord(R->h2d_done[sl], R->h2d) != cudaSuccess)
      return ATTN_ERR_CUDA;
    // the kernels, once the inputs landed and chunk c - 2's outputs left buffer set sl
    if (cudaStreamWaitEvent(stream, R->h2d_done[sl], 0) != cudaSuccess ||
        (c >= 2 && cudaStreamWaitEvent(stream, R->d2h_done[sl], 0) != cudaSuccess))
      return ATTN_ERR_CUDA;
    st = prefill_dense(qd, kd, vd, od, lse != nullptr ? ld : nullptr, np, G, 1, Sq, Sk, d, causal,
                       scale, k_lens != nullptr ? klen_dev + p0 : nullptr, 0, 0, nullptr, 1,
                       stream);
    if (st != ATTN_OK) return st;
    if (cudaEventRecord(R->comp_done[sl], stream) != cudaSuccess) return ATTN_ERR_CUDA;
    // outputs back to the host
    if (cudaStreamWaitEvent(R->d2h, R->comp_done[sl], 0) != cudaSuccess ||
        cudaMemcpyAsync(oh + p0 * q_pair, od, np * q_pair, cudaMemcpyDeviceToHost, R->d2h) !=
            cudaSuccess ||
        (lse != nullptr && cudaMemcpyAsync(lh + p0 * l_pair, ld, np * l_pair,
                                           cudaMemcpyDeviceToHost, R->d2h) != cudaSuccess) ||
        cudaEventRecord(R->d2h_done[sl], R->d2h) != cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  // the call is complete on the caller's stream once the last copies are
  for (int sl = 0; sl < 2 && sl < L.n_chunks; ++sl)
    if (cudaStreamWaitEvent(stream, R->d2h_done[(L.n_chunks - 1 - sl) & 1], 0) != cudaSuccess)
      return ATTN_ERR_CUDA;
  return ATTN_OK;
}

int host_pipeline_run(const HostPipelineLayout& L, const void* q, const void* k, const void* v,
                      void* o, float* lse, int B, int Hq, int Hkv, int Sq, int Sk, int d,
                      int causal, float scale, const int32_t* k_lens, char* ws,
                      cudaStream_t stream) {
  HostPipelineRes* R = nullptr;
  const int st = host_pipeline_res(&R);
  if (st != ATTN_OK) return st;
  std::lock_guard<std::mutex> g(R->mu, std::adopt_lock);
  return host_pipeline_enqueue(R, L, q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens,
                               ws, stream);
}

// Workspace of the E4M3 paged prefill: the unit list, the remapped block
// table [B, max_pages], and bf16 K and V pools of one page slot per
// (sequence, logical page), each part 256-byte aligned.
struct PagedFp8Layout {
  size_t table_off, k_off, v_off, total;
};

PagedFp8Layout paged_fp8_layout(int B, size_t units_bytes, int max_pages, int page_size, int Hkv,
                                int d) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  PagedFp8Layout L;
  L.table_off = up(units_bytes);
  const size_t slots = (size_t)B * max_pages;
  L.k_off = L.table_off + up(slots * sizeof(int32_t));
  const size_t pool = slots * page_size * Hkv * d * 2;
  L.v_off = L.k_off + up(pool);
  L.total = L.v_off + up(pool);
  return L;
}

size_t bwd_workspace_bytes(int B, int Hq, int Sq) {
  const size_t pad = ((size_t)Sq + 127) / 128 * 128;
  return 2 * (size_t)B * Hq * pad * sizeof(float);
}
}  // namespace
}  // namespace attn_b200

using namespace attn_b200;

extern "C" {

size_t attn_bwd_workspace_size(int B, int Hq, int Sq) {
  if (B < 1 || Hq < 1 || Sq < 1) return 0;
  return bwd_workspace_bytes(B, Hq, Sq);
}

}  // extern "C"

namespace attn_b200 {
namespace {
// The fixed-length backward, with the programmable masks of the forward
// (window / prefix: causal only; block mask: nullable).
int bwd_dense(const void* q, const void* k, const void* v, const void* o, const float* lse,
              const void* d_o, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk,
              int d, int causal, float scale, const int32_t* k_lens, int window, int prefix,
              const uint8_t* block_mask, int mask_heads, void* workspace, size_t workspace_bytes,
              attn_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (o == nullptr || lse == nullptr || d_o == nullptr || dq == nullptr || workspace == nullptr ||
      (Sk > 0 && (dk == nullptr || dv == nullptr)))
    return ATTN_ERR_INVALID_ARG;
  int st = check_prefill_args(q, k, v, dq, nullptr, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens);
  if (st != ATTN_OK) return st;
  if (!aligned16(o) || !aligned16(d_o) || !aligned16(workspace) || !aligned4(lse) ||
      (Sk > 0 && (!aligned16(dk) || !aligned16(dv))))
    return ATTN_ERR_ALIGNMENT;
  if (workspace_bytes < bwd_workspace_bytes(B, Hq, Sq)) return ATTN_ERR_WORKSPACE;
  if (Sk == 0) {  // no key: every output row is constant zero, so dQ = 0 (dK, dV are empty)
    const size_t bytes = (size_t)B * Hq * Sq * d * 2;
    return cudaMemsetAsync(dq, 0, bytes, stream) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  CUtensorMap mq, mdo, mk, mv;
  if (!make_tile_map(&mq, q, d, Sq, (long long)B * Hq) ||
      !make_tile_map(&mdo, d_o, d, Sq, (long long)B * Hq) ||
      !make_tile_map(&mk, k, d, Sk, (long long)B * Hkv) ||
      !make_tile_map(&mv, v, d, Sk, (long long)B * Hkv))
    return ATTN_ERR_CUDA;
  BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.o = static_cast<const uint16_t*>(o);
  prm.d_o = static_cast<const uint16_t*>(d_o);
  prm.lse = lse;
  prm.Sq_pad = (Sq + 127) / 128 * 128;
  prm.nlse2 = static_cast<float*>(workspace);
  prm.dsum = prm.nlse2 + (size_t)B * Hq * prm.Sq_pad;
  prm.k_lens = k_lens;
  prm.dq = static_cast<uint16_t*>(dq);
  prm.dk = static_cast<uint16_t*>(dk);
  prm.dv = static_cast<uint16_t*>(dv);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Sq = Sq;
  prm.Sk = Sk;
  prm.group = Hq / Hkv;
  prm.n_qt = prm.Sq_pad / 128;
  prm.n_kt = (Sk + 127) / 128;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.window = window;
  prm.prefix = prefix;
  prm.block_mask = block_mask;
  prm.mask_heads = mask_heads;
  if (window > 0 || prefix > 0 || block_mask != nullptr) {
    if (d == 128)
      return causal ? launch_bwd<128, true, false, true>(mq, mdo, mk, mv, prm, stream)
                    : launch_bwd<128, false, false, true>(mq, mdo, mk, mv, prm, stream);
    return causal ? launch_bwd<64, true, false, true>(mq, mdo, mk, mv, prm, stream)
                  : launch_bwd<64, false, false, true>(mq, mdo, mk, mv, prm, stream);
  }
  if (d == 128)
    return causal ? launch_bwd<128, true>(mq, mdo, mk, mv, prm, stream)
                  : launch_bwd<128, false>(mq, mdo, mk, mv, prm, stream);
  return causal ? launch_bwd<64, true>(mq, mdo, mk, mv, prm, stream)
                : launch_bwd<64, false>(mq, mdo, mk, mv, prm, stream);
}
}  // namespace
}  // namespace attn_b200

extern "C" {

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* d_o, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk,
             int d, int causal, float scale, const int32_t* k_lens, void* workspace,
             size_t workspace_bytes, attn_stream_t stream) {
  return bwd_dense(q, k, v, o, lse, d_o, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens,
                   0, 0, nullptr, 1, workspace, workspace_bytes, stream);
}

int attn_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* d_o, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq,
                    int Sk, int d, float scale, const int32_t* k_lens, int window, int prefix,
                    void* workspace, size_t workspace_bytes, attn_stream_t stream) {
  if (window < 0 || prefix < 0 || (window > 0 && prefix > 0)) return ATTN_ERR_INVALID_ARG;
  return bwd_dense(q, k, v, o, lse, d_o, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d, 1, scale, k_lens,
                   window, prefix, nullptr, 1, workspace, workspace_bytes, stream);
}

int attn_bwd_block_sparse(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* d_o, void* dq, void* dk, void* dv, int B,
                          int Hq, int Hkv, int Sq, int Sk, int d, int causal, float scale,
                          const int32_t* k_lens, const uint8_t* block_mask, int mask_heads,
                          void* workspace, size_t workspace_bytes, attn_stream_t stream) {
  if (block_mask == nullptr || (mask_heads != 1 && mask_heads != Hq)) return ATTN_ERR_INVALID_ARG;
  return bwd_dense(q, k, v, o, lse, d_o, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens,
                   0, 0, block_mask, mask_heads, workspace, workspace_bytes, stream);
}


size_t attn_bwd_varlen_workspace_size(int B, int Hq, int max_seqlen_q) {
  if (B < 1 || Hq < 1 || max_seqlen_q < 1) return 0;
  return bwd_workspace_bytes(B, Hq, max_seqlen_q);
}

int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* d_o, void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_k, int B, int Hq, int Hkv, long long total_q,
                    long long total_k, int max_seqlen_q, int max_seqlen_k, int d, int causal,
                    float scale, void* workspace, size_t workspace_bytes,
                    attn_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (q == nullptr || o == nullptr || lse == nullptr || d_o == nullptr || dq == nullptr ||
      workspace == nullptr || cu_seqlens_q == nullptr || cu_seqlens_k == nullptr ||
      (total_k > 0 && (k == nullptr || v == nullptr || dk == nullptr || dv == nullptr)))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
  if (total_q < 0 || total_k < 0 || total_q > 0x7fffffffLL || total_k > 0x7fffffffLL)
    return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_q < 1 || max_seqlen_k < 1 || max_seqlen_q > (1 << 30) || max_seqlen_k > (1 << 30))
    return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(o) || !aligned16(d_o) || !aligned16(dq) ||
      !aligned16(workspace) || !aligned4(lse) || !aligned4(cu_seqlens_q) ||
      !aligned4(cu_seqlens_k) ||
      (total_k > 0 && (!aligned16(k) || !aligned16(v) || !aligned16(dk) || !aligned16(dv))))
    return ATTN_ERR_ALIGNMENT;
  if (workspace_bytes < bwd_workspace_bytes(B, Hq, max_seqlen_q)) return ATTN_ERR_WORKSPACE;
  const long long n_qt = (max_seqlen_q + 127) / 128, n_kt = (max_seqlen_k + 127) / 128;
  if (n_qt * B * Hq > INT_MAX || n_kt * B * Hkv > INT_MAX) return ATTN_ERR_INVALID_ARG;
  if (total_q == 0) return ATTN_OK;  // no query row: no gradient to form
  if (total_k == 0)  // no key anywhere: every output row is constant zero, so dQ = 0
    return cudaMemsetAsync(dq, 0, (size_t)total_q * Hq * d * 2, stream) == cudaSuccess
               ? ATTN_OK
               : ATTN_ERR_CUDA;
  CUtensorMap mq, mdo, mk, mv;
  if (!make_token_map(&mq, q, d, Hq, total_q) || !make_token_map(&mdo, d_o, d, Hq, total_q) ||
      !make_token_map(&mk, k, d, Hkv, total_k) || !make_token_map(&mv, v, d, Hkv, total_k))
    return ATTN_ERR_CUDA;
  BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.o = static_cast<const uint16_t*>(o);
  prm.d_o = static_cast<const uint16_t*>(d_o);
  prm.lse = lse;
  prm.Sq_pad = (int)(n_qt * 128);
  prm.nlse2 = static_cast<float*>(workspace);
  prm.dsum = prm.nlse2 + (size_t)B * Hq * prm.Sq_pad;
  prm.dq = static_cast<uint16_t*>(dq);
  prm.dk = static_cast<uint16_t*>(dk);
  prm.dv = static_cast<uint16_t*>(dv);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Sq = max_seqlen_q;
  prm.Sk = max_seqlen_k;
  prm.group = Hq / Hkv;
  prm.n_qt = (int)n_qt;
  prm.n_kt = (int)n_kt;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.cu_q = cu_seqlens_q;
  prm.cu_k = cu_seqlens_k;
  prm.total_q = (int)total_q;
  prm.total_k = (int)total_k;
  if (d == 128)
    return causal ? launch_bwd<128, true, true>(mq, mdo, mk, mv, prm, stream)
                  : launch_bwd<128, false, true>(mq, mdo, mk, mv, prm, stream);
  return causal ? launch_bwd<64, true, true>(mq, mdo, mk, mv, prm, stream)
                : launch_bwd<64, false, true>(mq, mdo, mk, mv, prm, stream);
}

const char* attn_strerror(int status) {
  switch (status) {
    case ATTN_OK: return "success";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration (head dim, page size or group size)";
    case ATTN_ERR_ALIGNMENT: return "tensor pointer not 16-byte aligned";
    case ATTN_ERR_WORKSPACE: return "decode workspace missing or too small";
    case ATTN_ERR_CUDA: return "CUDA runtime or driver call failed";
    case ATTN_ERR_DEVICE: return "device error word set (bad page id, bad length or wait timeout)";
    default: return "unknown status";
  }
}

int attn_split_tokens(void) { return kSplitTokens; }

int attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Sq, int Sk, int d, int causal, float scale,
                    const int32_t* k_lens, attn_stream_t stream) {
  const int st = check_prefill_args(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens);
  if (st != ATTN_OK) return st;
  return prefill_dense(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens, 0, 0,
                       nullptr, 1, reinterpret_cast<cudaStream_t>(stream));
}

size_t attn_fwd_host_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int d) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Sq < 1 || Sk < 0 || (d != 64 && d != 128))
    return 0;
  return host_pipeline_layout(B, Hq, Hkv, Sq, Sk, d).total;
}

int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Sq, int Sk, int d, int causal, float scale, const int32_t* k_lens,
                  void* workspace, size_t workspace_bytes, attn_stream_t stream_) {
  int st = check_prefill_args(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, nullptr);
  if (st != ATTN_OK) return st;
  const HostPipelineLayout L = host_pipeline_layout(B, Hq, Hkv, Sq, Sk, d);
  if (workspace == nullptr || workspace_bytes < L.total) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGNMENT;
  if (k_lens != nullptr)
    for (int b = 0; b < B; ++b)  // host array: checked here, as the device path clamps
      if (k_lens[b] < 0 || k_lens[b] > Sk) return ATTN_ERR_INVALID_ARG;
  return host_pipeline_run(L, q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens,
                           static_cast<char*>(workspace), reinterpret_cast<cudaStream_t>(stream_));
}

int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Sq, int Sk, int d, float scale, const int32_t* k_lens,
                    int window, int prefix, attn_stream_t stream) {
  const int st = check_prefill_args(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, 1, scale, k_lens);
  if (st != ATTN_OK) return st;
  if (window < 0 || prefix < 0 || (window > 0 && prefix > 0)) return ATTN_ERR_INVALID_ARG;
  return prefill_dense(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, 1, scale, k_lens, window, prefix,
                       nullptr, 1, reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int Hq, int Hkv, int Sq, int Sk, int d, int causal, float scale,
                          const int32_t* k_lens, const uint8_t* block_mask, int mask_heads,
                          attn_stream_t stream) {
  const int st = check_prefill_args(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens);
  if (st != ATTN_OK) return st;
  if (block_mask == nullptr || (mask_heads != 1 && mask_heads != Hq)) return ATTN_ERR_INVALID_ARG;
  return prefill_dense(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens, 0, 0,
                       block_mask, mask_heads, reinterpret_cast<cudaStream_t>(stream));
}

size_t attn_fwd_varlen_workspace_size(int B, long long total_q, int max_seqlen_q) {
  if (B < 1 || total_q < 0 || total_q > 0x7fffffffLL || max_seqlen_q < 1 ||
      max_seqlen_q > kVarlenMaxLevels * 256)
    return 0;
  return 16 + 8 * (size_t)varlen_max_units(B, total_q);
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int Hq,
                    int Hkv, long long total_q, long long total_k, int max_seqlen_q, int d,
                    int causal, float scale, void* workspace, size_t workspace_bytes,
                    attn_stream_t stream_) {
  if (q == nullptr || o == nullptr || cu_seqlens_q == nullptr || cu_seqlens_k == nullptr ||
      (total_k > 0 && (k == nullptr || v == nullptr)))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
  if (total_q < 0 || total_k < 0 || total_q > 0x7fffffffLL || total_k > 0x7fffffffLL)
    return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_q < 1 || max_seqlen_q > kVarlenMaxLevels * 256) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(o) || (total_k > 0 && (!aligned16(k) || !aligned16(v))))
    return ATTN_ERR_ALIGNMENT;
  if ((lse != nullptr && !aligned4(lse)) || !aligned4(cu_seqlens_q) || !aligned4(cu_seqlens_k))
    return ATTN_ERR_ALIGNMENT;
  const size_t need = attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGNMENT;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (total_q == 0) return ATTN_OK;  // no query token: nothing to write
  if (total_k == 0) {  // no key anywhere: every query row is empty
    const size_t n_vec = (size_t)total_q * Hq * d * 2 / 16;
    const int threads = 256;
    const long long want = ((long long)n_vec + threads - 1) / threads;
    const int blocks = (int)(want < 4096 ? (want > 0 ? want : 1) : 4096);
    fill_empty_rows_kernel<<<blocks, threads, 0, stream>>>(reinterpret_cast<uint4*>(o), n_vec, lse,
                                                           (size_t)total_q * Hq);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  // 1. the unit list (heaviest first) in the workspace
  int* unit_count = static_cast<int*>(workspace);
  int2* units = reinterpret_cast<int2*>(static_cast<char*>(workspace) + 16);
  const long long max_units = varlen_max_units(B, total_q);
  int shift, n_levels;
  varlen_levels(total_k, shift, n_levels);  // total_k bounds every key range
  const size_t sched_smem = (size_t)(2 * n_levels + 32) * sizeof(int);
  if (!schedule_smem_ready()) return ATTN_ERR_CUDA;
  attn_varlen_schedule_kernel<<<1, 1024, sched_smem, stream>>>(
      cu_seqlens_q, cu_seqlens_k, nullptr, B, (int)total_q, (int)total_k, max_seqlen_q, 0, causal,
      0, 0, shift, n_levels, units, unit_count, (int)max_units);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  // 2. the prefill kernel over packed token-major tensors
  CUtensorMap mq, mk, mv;
  if (!make_token_map(&mq, q, d, Hq, total_q) || !make_token_map(&mk, k, d, Hkv, total_k) ||
      !make_token_map(&mv, v, d, Hkv, total_k))
    return ATTN_ERR_CUDA;
  PrefillParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.lse = lse;
  prm.k_lens = nullptr;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.o = static_cast<uint16_t*>(o);
  prm.cu_q = cu_seqlens_q;
  prm.cu_k = cu_seqlens_k;
  prm.units = units;
  prm.unit_count = unit_count;
  prm.total_q = (int)total_q;
  // the output map is unused by the ragged path (rows are stored one by one)
  if (d == 128)
    return causal ? launch_prefill<128, true, kLayoutRagged>(mq, mk, mv, mq, prm, stream, max_units)
                  : launch_prefill<128, false, kLayoutRagged>(mq, mk, mv, mq, prm, stream, max_units);
  return causal ? launch_prefill<64, true, kLayoutRagged>(mq, mk, mv, mq, prm, stream, max_units)
                : launch_prefill<64, false, kLayoutRagged>(mq, mk, mv, mq, prm, stream, max_units);
}

int attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_table, const int32_t* cu_seqlens_q,
                   const int32_t* seq_lens_k, int page_size, int B, int Hq, int Hkv,
                   long long total_q, int max_seqlen_q, int max_pages_per_seq, int num_pages, int d,
                   int causal, float scale, void* o, float* lse, void* workspace,
                   size_t workspace_bytes, attn_stream_t stream_) {
  int st = check_paged_prefill_args(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k,
                                    page_size, B, Hq, Hkv, total_q, max_seqlen_q,
                                    max_pages_per_seq, num_pages, d, causal, scale, o, lse);
  if (st != ATTN_OK) return st;
  const size_t need = attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGNMENT;
  if (total_q == 0) return ATTN_OK;
  return paged_prefill_run(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k, page_size,
                           B, Hq, Hkv, total_q, max_seqlen_q, max_pages_per_seq, num_pages, d,
                           causal, scale, o, lse, workspace,
                           reinterpret_cast<cudaStream_t>(stream_));
}

size_t attn_fwd_paged_fp8_workspace_size(int B, long long total_q, int max_seqlen_q,
                                         int max_pages_per_seq, int page_size, int Hkv, int d) {
  const size_t units = attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q);
  if (units == 0 || max_pages_per_seq < 1 || page_size < 1 || Hkv < 1 || d < 1) return 0;
  return paged_fp8_layout(B, units, max_pages_per_seq, page_size, Hkv, d).total;
}

int attn_fwd_paged_fp8(const void* q, const void* k_cache, const void* v_cache,
                       const float* k_scale, const float* v_scale, const int32_t* block_table,
                       const int32_t* cu_seqlens_q, const int32_t* seq_lens_k, int page_size,
                       int B, int Hq, int Hkv, long long total_q, int max_seqlen_q,
                       int max_pages_per_seq, int num_pages, int d, int causal, float scale,
                       void* o, float* lse, void* workspace, size_t workspace_bytes,
                       attn_stream_t stream_) {
  if (k_scale == nullptr || v_scale == nullptr) return ATTN_ERR_INVALID_ARG;
  int st = check_paged_prefill_args(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k,
                                    page_size, B, Hq, Hkv, total_q, max_seqlen_q,
                                    max_pages_per_seq, num_pages, d, causal, scale, o, lse);
  if (st != ATTN_OK) return st;
  if (!aligned4(k_scale) || !aligned4(v_scale)) return ATTN_ERR_ALIGNMENT;
  const size_t units = attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q);
  const PagedFp8Layout L = paged_fp8_layout(B, units, max_pages_per_seq, page_size, Hkv, d);
  if (workspace == nullptr || workspace_bytes < L.total) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGNMENT;
  if ((long long)B * max_pages_per_seq * page_size > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (total_q == 0) return ATTN_OK;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  char* ws = static_cast<char*>(workspace);
  int32_t* table2 = reinterpret_cast<int32_t*>(ws + L.table_off);
  uint16_t* k2 = reinterpret_cast<uint16_t*>(ws + L.k_off);
  uint16_t* v2 = reinterpret_cast<uint16_t*>(ws + L.v_off);
  // 1. the pages the batch references, dequantised into a bf16 pool of one
  //    slot per (sequence, logical page), with the table that maps onto it
  const int threads = 256;
  attn_dequant_pages_kernel<<<dim3((unsigned)max_pages_per_seq, (unsigned)B), threads, 0, stream>>>(
      static_cast<const uint8_t*>(k_cache), static_cast<const uint8_t*>(v_cache), k_scale,
      v_scale, block_table, seq_lens_k, page_size, Hkv, d, max_pages_per_seq, num_pages, k2, v2,
      table2);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  // 2. the bf16 paged prefill over that pool
  return paged_prefill_run(q, k2, v2, table2, cu_seqlens_q, seq_lens_k, page_size, B, Hq, Hkv,
                           total_q, max_seqlen_q, max_pages_per_seq, B * max_pages_per_seq, d,
                           causal, scale, o, lse, workspace, stream);
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, const float* q_scale,
                 const float* k_scale, const float* v_scale, void* o, float* lse, int B, int Hq,
                 int Hkv, int Sq, int Sk, int d, int causal, float scale, const int32_t* k_lens,
                 attn_stream_t stream_) {
  if (q_scale == nullptr || (Sk > 0 && (k_scale == nullptr || v_scale == nullptr)))
    return ATTN_ERR_INVALID_ARG;
  const int st = check_prefill_args(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens);
  if (st != ATTN_OK) return st;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned4(q_scale) || (Sk > 0 && (!aligned4(k_scale) || !aligned4(v_scale))))
    return ATTN_ERR_ALIGNMENT;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (Sk == 0)  // no key: every row empty
    return prefill_dense(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens, 0, 0,
                         nullptr, 1, stream);
  CUtensorMap mq, mk, mv, mo;
  if (!make_tile_map_u8(&mq, q, d, Sq, (long long)B * Hq) ||
      !make_tile_map_u8(&mk, k, d, Sk, (long long)B * Hkv) ||
      !make_tile_map_u8(&mv, v, d, Sk, (long long)B * Hkv) ||
      !make_tile_map(&mo, o, d, Sq, (long long)B * Hq, 32))
    return ATTN_ERR_CUDA;
  PrefillFp8Params f;
  std::memset(&f, 0, sizeof(f));
  PrefillParams& prm = f.p;
  prm.lse = lse;
  prm.k_lens = k_lens;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Sq = Sq;
  prm.Sk = Sk;
  prm.group = Hq / Hkv;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.n_qblocks = (Sq + 255) / 256;
  prm.mask_heads = 1;
  prm.n_qt = (Sq + 127) / 128;
  prm.n_kt = (Sk + 127) / 128;
  f.q_scale = q_scale;
  f.k_scale = k_scale;
  f.v_scale = v_scale;
  using C = PrefillFp8Cfg;
  const long long units = (long long)prm.n_qblocks * Hq * B;
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  dim3 grid((unsigned)(units < sms ? units : sms));
  if (causal) {
    static std::atomic<unsigned long long> done{0};
    if (!set_smem_once(attn_prefill_fp8_kernel<true>, C::SMEM_BYTES, done)) return ATTN_ERR_CUDA;
    attn_prefill_fp8_kernel<true><<<grid, C::NUM_THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, f);
  } else {
    static std::atomic<unsigned long long> done{0};
    if (!set_smem_once(attn_prefill_fp8_kernel<false>, C::SMEM_BYTES, done)) return ATTN_ERR_CUDA;
    attn_prefill_fp8_kernel<false><<<grid, C::NUM_THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, f);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Sq, int Sk, int d, int causal, float scale, attn_stream_t stream) {
  return attn_fwd_masked(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, causal, scale, nullptr, stream);
}

size_t attn_decode_workspace_size(int B, int Hq, int max_pages_per_seq, int page_size, int d) {
  if (B < 1 || Hq < 1 || max_pages_per_seq < 1 || page_size < 1 || d < 1) return 0;
  const long long tokens = (long long)max_pages_per_seq * page_size;
  const long long n_split = (tokens + kSplitTokens - 1) / kSplitTokens;
  const long long parts = (long long)B * Hq * n_split;
  const size_t o_bytes = (size_t)parts * d * sizeof(float);
  const size_t lse_bytes = (size_t)parts * sizeof(float);
  return o_bytes + ((lse_bytes + 255) / 256) * 256;
}

int attn_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_table, const int32_t* seq_lens, int page_size, int B,
                      int Hq, int Hkv, int d, int max_pages_per_seq, int num_pages, float scale,
                      void* o, float* lse, void* workspace, size_t workspace_bytes,
                      attn_stream_t stream_) {
  return decode_paged_common(false, q, k_cache, v_cache, nullptr, nullptr, block_table, seq_lens,
                             page_size, B, Hq, Hkv, d, max_pages_per_seq, num_pages, scale, o,
                             lse, workspace, workspace_bytes, stream_);
}

int attn_decode_paged_fp8(const void* q, const void* k_cache, const void* v_cache,
                          const float* k_scale, const float* v_scale, const int32_t* block_table,
                          const int32_t* seq_lens, int page_size, int B, int Hq, int Hkv, int d,
                          int max_pages_per_seq, int num_pages, float scale, void* o, float* lse,
                          void* workspace, size_t workspace_bytes, attn_stream_t stream_) {
  if (k_scale == nullptr || v_scale == nullptr) return ATTN_ERR_INVALID_ARG;
  return decode_paged_common(true, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens,
                             page_size, B, Hq, Hkv, d, max_pages_per_seq, num_pages, scale, o,
                             lse, workspace, workspace_bytes, stream_);
}

int attn_get_device_error(attn_stream_t stream_, unsigned int* flags_out) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return ATTN_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (flags_out != nullptr) *flags_out = v;
  return v == 0 ? ATTN_OK : ATTN_ERR_DEVICE;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode for callers that may not allocate device memory (see attn.h): the
// split partials go to a file-scope device array instead of a workspace.
// ---------------------------------------------------------------------------
namespace attn_b200 {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

// In host code `g_noalloc_scratch` names a host-side stand-in, not device
// memory; the kernels must be given the address cudaGetSymbolAddress returns,
// which is looked up once per device (with that device current) and cached.
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_device_ptr[kMaxDevices] = {};

int noalloc_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_device_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return ATTN_ERR_CUDA;
    g_noalloc_device_ptr[dev] = p;
  }
  *out = g_noalloc_device_ptr[dev];
  return ATTN_OK;
}

}  // namespace
}  // namespace attn_b200

extern "C" int attn_decode_paged_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_table, const int32_t* seq_lens,
                                         int page_size, int B, int Hq, int Hkv, int d,
                                         int max_pages_per_seq, int num_pages, float scale,
                                         void* o, float* lse, attn_stream_t stream) {
  // Size check first, on the host: nothing is launched for a problem that
  // does not fit the static scratch area.
  const size_t need = attn_decode_workspace_size(B, Hq, max_pages_per_seq, page_size, d);
  if (need == 0) return ATTN_ERR_INVALID_ARG;
  if (need > (size_t)ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = attn_b200::noalloc_scratch_address(&scratch);
  if (st != ATTN_OK) return st;
  return attn_decode_paged(q, k_cache, v_cache, block_table, seq_lens, page_size, B, Hq, Hkv, d,
                           max_pages_per_seq, num_pages, scale, o, lse, scratch,
                           (size_t)ATTN_NOALLOC_SCRATCH_BYTES, stream);
}
