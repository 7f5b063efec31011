// attention_api.cuh -- host side of decode attention over the quantized or
// FP8 cache: argument checks, the workspace size, the launch of the partial
// and combine kernels, and the entry point with library-owned scratch.
// Included at the end of kvq.cu (one translation unit), after the shared
// launch helpers it uses.
#pragma once

#include "attention.cuh"
#include "attention_tc.cuh"

namespace {

// Which decode-attention kernel runs (kvq_set_attention_path).
std::atomic<int> g_attention_path{KVQ_ATTENTION_AUTO};

// CTAs of the tcgen05 kernel the device holds at once (cached per device, after the
// shared-memory opt-in), 0 on failure.
template <int B, int G>
long long tc_ctas() {
  constexpr int kMaxDevices = 64;
  static std::atomic<bool> opted[kMaxDevices];
  static std::atomic<long long> resident[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 0;
  }
  if (!opted[dev].load()) {
    // all of the SM's unified memory as shared memory: two or three CTAs of 64-80 KB
    if (cudaFuncSetAttribute(kvq::attn_tc_kernel<B, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kvq::tc_smem_bytes<B>()) != cudaSuccess ||
        cudaFuncSetAttribute(kvq::attn_tc_kernel<B, G>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    opted[dev].store(true);
  }
  long long n = resident[dev].load();
  if (n == 0) {
    // CTAs per SM from the shared memory each needs and the launch bounds (three);
    // the occupancy query reports one for this kernel
    int sms = 0, smem_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    long long per_sm = smem_sm / (kvq::tc_smem_bytes<B>() + 1024);
    if (per_sm > 3) per_sm = 3;
    if (per_sm < 1) per_sm = 1;
    n = static_cast<long long>(sms) * per_sm;
    resident[dev].store(n);
  }
  return n;
}

// The tcgen05 partial kernel for `group` query heads per kv head: as many CTAs
// as the device holds at once, never more than there are item slots.
template <int B, int G>
kvq_status launch_tc(const kvq::AttnParams& a, long long items, void* stream) {
  const long long ctas = tc_ctas<B, G>();
  if (ctas < 1) return KVQ_ERR_CUDA;
  return launch_pdl(kvq::attn_tc_kernel<B, G>, dim3(static_cast<unsigned>(items < ctas ? items : ctas)),
                    kvq::kTcThreads, kvq::tc_smem_bytes<B>(), stream, a);
}

// Chunks of `chunk` positions a sequence can have: the longest window the
// cache geometry allows.
long long attn_max_chunks(const kvq_cache_desc* d, int page_size, int chunk) {
  const long long max_len = page_size > 0 ? static_cast<long long>(d->block_table_stride) * page_size
                                          : static_cast<long long>(d->dim1);
  return (max_len + chunk - 1) / chunk;
}

// Dynamic shared memory opt-in, once per device for each partial kernel
// (static plus dynamic shared memory above 48 KB needs it).
template <int B, int D, bool kCompact, bool kSplit, bool kG4>
bool allow_attention_smem() {
  constexpr int kMaxDevices = 64;
  static std::atomic<bool> done[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (done[dev].load()) return true;
  if (cudaFuncSetAttribute(kvq::attn_partial_kernel<B, D, kCompact, kSplit, kG4>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kvq::AttnTile<B, D>::kSmemBytes) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  done[dev].store(true);
  return true;
}

// CTAs of a partial kernel the device holds at once (occupancy cached per
// device), 0 on failure.
template <int B, int D, bool kCompact, bool kSplit, bool kG4>
long long partial_ctas() {
  if (!allow_attention_smem<B, D, kCompact, kSplit, kG4>()) return 0;
  constexpr int kMaxDevices = 64;
  static std::atomic<long long> resident[kMaxDevices];
  return first_wave_ctas(kvq::attn_partial_kernel<B, D, kCompact, kSplit, kG4>, kvq::kAttnThreads,
                         kvq::AttnTile<B, D>::kSmemBytes, resident, kMaxDevices);
}

// Persistent grid of the partial kernel: every (sequence, chunk, kv head) work
// item goes to one warp (to one CTA with kSplit); as many CTAs as the device
// holds at once, never more than there are item slots.
template <int B, int D, bool kCompact, bool kSplit, bool kG4>
kvq_status launch_partial(const kvq::AttnParams& a, long long items, long long ctas_max, void* stream) {
  using T = kvq::AttnTile<B, D>;
  if (ctas_max < 1) return KVQ_ERR_CUDA;
  const long long need = kSplit ? items : (items + kvq::kAttnWarps - 1) / kvq::kAttnWarps;
  const long long grid = need < ctas_max ? need : ctas_max;
  return launch_pdl(kvq::attn_partial_kernel<B, D, kCompact, kSplit, kG4>, dim3(static_cast<unsigned>(grid)),
                    kvq::kAttnThreads, T::kSmemBytes, stream, a);
}

// The partial kernel for every walk: only the items that hold data when the
// batch fits its shared-memory slots and every item count fits an int,
// otherwise every item slot.  When the cache geometry has no more 256-position
// item slots than the device holds CTAs (batches of one or two long sequences;
// head_dim <= 128), the four warps of a CTA share each item (measured: 10%
// faster there, slower from two 256-position items per CTA on).
template <int B, int D, bool kG4>
kvq_status launch_partial_walk(const kvq::AttnParams& a, long long items, bool compact, void* stream) {
  if (!compact) return launch_partial<B, D, false, false, kG4>(a, items, partial_ctas<B, D, false, false, kG4>(), stream);
  const long long ctas = partial_ctas<B, D, true, false, kG4>();
  if (D <= 128 && items * kvq::AttnTile<B, D>::kChunk <= ctas * 256)
    return launch_partial<B, D, true, D <= 128, kG4>(a, items, partial_ctas<B, D, true, D <= 128, kG4>(), stream);
  return launch_partial<B, D, true, false, kG4>(a, items, ctas, stream);
}

// The partial kernel (tcgen05 or mma.sync), then the combine kernel.
template <int B, int D>
kvq_status launch_attention(kvq::AttnParams a, const kvq_cache_desc* desc, void* stream) {
  using T = kvq::AttnTile<B, D>;
  a.chunk = T::kChunk;
  const long long max_chunks = attn_max_chunks(desc, a.page_size, T::kChunk);
  if (max_chunks < 1 || max_chunks > 0x7FFFFFFFLL) return KVQ_ERR_RANGE;
  a.max_chunks = static_cast<int>(max_chunks);
  const long long items = static_cast<long long>(a.batch) * a.max_chunks * a.kv_heads;
  const bool compact = a.batch <= T::kSeqlenSlots && items <= 0x7FFFFFFFLL;
  kvq_status st;
  const int path = g_attention_path.load(std::memory_order_relaxed);
  if constexpr (D == kvq::kTcD) {
    // the tcgen05 kernel: head_dim 128, batches its shared memory stages (<= 256 sequences)
    if (path == KVQ_ATTENTION_TCGEN05 && compact) {
      // kTcItem-position entries: every one of them is written
      a.chunk = kvq::kTcItem;
      a.max_chunks = static_cast<int>(attn_max_chunks(desc, a.page_size, kvq::kTcItem));
      switch (a.group) {
        case 1: st = launch_tc<B, 1>(a, items, stream); break;
        case 2: st = launch_tc<B, 2>(a, items, stream); break;
        case 3: st = launch_tc<B, 3>(a, items, stream); break;
        case 4: st = launch_tc<B, 4>(a, items, stream); break;
        case 5: st = launch_tc<B, 5>(a, items, stream); break;
        case 6: st = launch_tc<B, 6>(a, items, stream); break;
        case 7: st = launch_tc<B, 7>(a, items, stream); break;
        default: st = launch_tc<B, 8>(a, items, stream); break;
      }
      if (st != KVQ_OK) return st;
      return launch_pdl(kvq::attn_combine_kernel<D>, dim3(a.n_heads, a.batch), kvq::kCombineThreads, 0, stream, a);
    }
  }
  st = a.group <= 4 ? launch_partial_walk<B, D, true>(a, items, compact, stream)
                    : launch_partial_walk<B, D, false>(a, items, compact, stream);
  if (st != KVQ_OK) return st;
  return launch_pdl(kvq::attn_combine_kernel<D>, dim3(a.n_heads, a.batch), kvq::kCombineThreads, 0, stream, a);
}

template <int B>
kvq_status launch_attention_b(const kvq::AttnParams& a, const kvq_cache_desc* desc, void* stream) {
  if (desc->head_dim == 64) return launch_attention<B, 64>(a, desc, stream);
  if (desc->head_dim == 128) return launch_attention<B, 128>(a, desc, stream);
  return launch_attention<B, 256>(a, desc, stream);
}

}  // namespace

extern "C" {

size_t kvq_decode_attention_workspace_size(const kvq_cache_desc* desc, int batch_size, int n_heads,
                                           int page_size) {
  if (!desc || batch_size < 0 || n_heads < 0 || page_size < 0 || desc->head_dim < 0 || desc->dim1 < 0 ||
      desc->block_table_stride < 0)
    return 0;
  // one entry per (sequence, query head, 128-position chunk slot); SIZE_MAX when that overflows
  const long long chunks = attn_max_chunks(desc, page_size, kvq::kAttnMinChunk);
  size_t n = static_cast<size_t>(batch_size);
  if (__builtin_mul_overflow(n, static_cast<size_t>(n_heads), &n) ||
      __builtin_mul_overflow(n, static_cast<size_t>(chunks), &n) ||
      __builtin_mul_overflow(n, static_cast<size_t>(desc->head_dim) + 2, &n) ||
      __builtin_mul_overflow(n, sizeof(float), &n))
    return SIZE_MAX;
  return n;
}

}  // extern "C"

namespace {

// Shared argument checks and launch of the decode-attention entry points:
// format 4 / 6 / 8 = Q codes with scales, 0 = E5M2 bytes without scales.
kvq_status decode_attention(const void* q, const void* k_codes, const void* k_scales, const void* v_codes,
                            const void* v_scales, void* out, const kvq_cache_desc* desc, int batch_size, int n_heads,
                            int page_size, const int32_t* cache_seqlens, const int32_t* block_table, int format,
                            float softmax_scale, void* workspace, size_t workspace_bytes, void* stream) {
  const bool scaled = format != 0;
  if (!q || !k_codes || !v_codes || !out || !desc || !cache_seqlens) return KVQ_ERR_NULL;
  if (scaled && (!k_scales || !v_scales)) return KVQ_ERR_NULL;
  if (format != 0 && format != 4 && format != 6 && format != 8) return KVQ_ERR_WBITS;
  kvq_status st = check_desc(desc, scaled ? 32 : 8);
  if (st != KVQ_OK) return st;
  const int D = desc->head_dim;
  if (D != 64 && D != 128 && D != 256) return KVQ_ERR_SHAPE;
  if (n_heads < 1 || n_heads % desc->kv_heads || n_heads / desc->kv_heads > kvq::kAttnMaxGroup) return KVQ_ERR_SHAPE;
  if (batch_size < 0 || batch_size > 65535 || desc->kv_heads > 65535 || n_heads > 0x7FFFFFFF) return KVQ_ERR_RANGE;
  if (page_size < 0) return KVQ_ERR_RANGE;
  if (page_size == 0) {
    if (batch_size > desc->dim0) return KVQ_ERR_RANGE;
  } else {
    if (!block_table) return KVQ_ERR_NULL;
    if (page_size != desc->dim1 || desc->block_table_stride < 1) return KVQ_ERR_RANGE;
  }
  const void* ptrs[7] = {q, k_codes, k_scales, v_codes, v_scales, out, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KVQ_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(cache_seqlens) | reinterpret_cast<uintptr_t>(block_table)) & 3u)
    return KVQ_ERR_ALIGN;
  if (batch_size == 0) return KVQ_OK;
  const long long max_chunks = attn_max_chunks(desc, page_size, kvq::kAttnMinChunk);
  if (max_chunks < 1 || max_chunks > 0x7FFFFFFFLL) return KVQ_ERR_RANGE;
  if (!workspace) return KVQ_ERR_NULL;
  const size_t need = kvq_decode_attention_workspace_size(desc, batch_size, n_heads, page_size);
  if (need == SIZE_MAX || workspace_bytes < need) return KVQ_ERR_RANGE;
  kvq::AttnParams a{};
  a.q = static_cast<const __half*>(q);
  a.k_codes = static_cast<const uint8_t*>(k_codes);
  a.k_scales = static_cast<const __half*>(k_scales);
  a.v_codes = static_cast<const uint8_t*>(v_codes);
  a.v_scales = static_cast<const __half*>(v_scales);
  a.out = static_cast<__half*>(out);
  a.ws = static_cast<float*>(workspace);
  a.seqlens = cache_seqlens;
  a.block_table = block_table;
  a.dim0 = desc->dim0;
  a.dim1 = desc->dim1;
  a.kv_heads = desc->kv_heads;
  a.batch = batch_size;
  a.n_heads = n_heads;
  a.group = n_heads / desc->kv_heads;
  a.page_size = page_size;
  a.bt_stride = desc->block_table_stride;
  a.page_shift = -1;
  for (int sh = 0; sh < 31; ++sh)
    if (page_size == (1 << sh)) a.page_shift = sh;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  if (format == 4) return launch_attention_b<4>(a, desc, stream);
  if (format == 6) return launch_attention_b<6>(a, desc, stream);
  if (format == 8) return launch_attention_b<8>(a, desc, stream);
  return launch_attention_b<0>(a, desc, stream);
}

}  // namespace

extern "C" {

kvq_status kvq_decode_attention_q(const void* q, const void* k_codes, const void* k_scales, const void* v_codes,
                                  const void* v_scales, void* out, const kvq_cache_desc* desc, int batch_size,
                                  int n_heads, int page_size, const int32_t* cache_seqlens,
                                  const int32_t* block_table, int wbits, float softmax_scale, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (wbits != 4 && wbits != 6 && wbits != 8) return KVQ_ERR_WBITS;
  return decode_attention(q, k_codes, k_scales, v_codes, v_scales, out, desc, batch_size, n_heads, page_size,
                          cache_seqlens, block_table, wbits, softmax_scale, workspace, workspace_bytes, stream);
}

kvq_status kvq_decode_attention_fp8(const void* q, const void* k_fp8, const void* v_fp8, void* out,
                                    const kvq_cache_desc* desc, int batch_size, int n_heads, int page_size,
                                    const int32_t* cache_seqlens, const int32_t* block_table, float softmax_scale,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  return decode_attention(q, k_fp8, nullptr, v_fp8, nullptr, out, desc, batch_size, n_heads, page_size,
                          cache_seqlens, block_table, 0, softmax_scale, workspace, workspace_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention with library-owned scratch.
//
// Some callers cannot allocate device memory where they call attention: a
// serving loop whose HBM is all handed to its own KV-page pool up front has
// no allocator to draw a workspace from, and cudaMalloc / cudaFree may
// synchronize the device, which a per-token decode step on a busy stream
// cannot afford.  This entry point takes its split-K workspace from a fixed
// array compiled into the library instead, so it allocates nothing.

static __device__ __align__(256) unsigned char g_attention_scratch[KVQ_ATTENTION_SCRATCH_BYTES];

namespace {

// Device address of the current device's copy of the array, or null on
// failure.  Looked up on every call (a host-side query that enqueues nothing):
// an address kept from an earlier call would dangle once the device's primary
// context has been reset and re-created.
void* attention_scratch() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_attention_scratch) != cudaSuccess || !ptr) {
    cudaGetLastError();
    return nullptr;
  }
  return ptr;
}

}  // namespace

extern "C" {

kvq_status kvq_decode_attention_q_noalloc(const void* q, const void* k_codes, const void* k_scales,
                                          const void* v_codes, const void* v_scales, void* out,
                                          const kvq_cache_desc* desc, int batch_size, int n_heads, int page_size,
                                          const int32_t* cache_seqlens, const int32_t* block_table, int wbits,
                                          float softmax_scale, void* stream) {
  if (!desc) return KVQ_ERR_NULL;
  if (kvq_decode_attention_workspace_size(desc, batch_size, n_heads, page_size) > KVQ_ATTENTION_SCRATCH_BYTES)
    return KVQ_ERR_RANGE;
  void* scratch = attention_scratch();
  if (!scratch) return KVQ_ERR_CUDA;
  return kvq_decode_attention_q(q, k_codes, k_scales, v_codes, v_scales, out, desc, batch_size, n_heads,
                                page_size, cache_seqlens, block_table, wbits, softmax_scale, scratch,
                                KVQ_ATTENTION_SCRATCH_BYTES, stream);
}

}  // extern "C"
