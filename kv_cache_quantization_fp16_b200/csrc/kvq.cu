// kvq.cu -- the C ABI (include/kvq.h) of libkvq.so: host-side validation,
// tiling and launch of the sm_100a conversion kernels.
//
// KV-cache format conversions from the page "Implementation: Turboderp org
// Exllamav2 Ext Cache": fp16_to_fp8 / fp8_to_fp16 (Description, Signature)
// and fp16_to_q_kv / q_to_fp16_kv (Description, Signature, I/O Contract), in
// contiguous and paged mode.
//
// Work decomposition.  A window of one sequence is a run of positions; every
// position is H * D contiguous elements in the FP16 cache (and proportionally
// many bytes in the FP8 / code / scale tensors).  The run is cut into tiles of
// `tile_pos` positions; in paged mode tiles are aligned to multiples of
// tile_pos in logical position space and tile_pos divides page_size, so a tile
// never straddles a page.  Two load engines convert tiles (ldg_engine.cuh:
// one tile per CTA from plain global loads; bulk_engine.cuh: persistent CTAs
// fed by TMA bulk copies through shared memory); both share the per-tile
// bodies in ops.cuh and the arithmetic in codec.cuh.
//
// This is a streaming, HBM-bound path: no tensor cores, no collectives.
// The host side of decode attention over the converted caches lives in
// attention_api.cuh, included at the end of this file.

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/kvq.h"
#include "bulk_engine.cuh"
#include "codec.cuh"
#include "ldg_engine.cuh"
#include "ops.cuh"
#include "tiles.cuh"

namespace kvq {

// ---------------------------------------------------------------------------
// Self-check of the fast code rounding against IEEE division.
// ---------------------------------------------------------------------------

template <int B>
__global__ void selfcheck_rounding_kernel(unsigned long long* mismatches) {
  // blockIdx.x enumerates the scale bit patterns 0..0x7BFF (+0 and every
  // positive finite binary16); threads enumerate x over all 65536 bit patterns,
  // skipping Inf / NaN.  Both forms the kernels use are checked: the clamped
  // one for every pair, the unclamped one (used unless the scale is a nonzero
  // subnormal) for every pair a block can produce.  A block gets the scale s
  // only if absmax / maxq rounds to s, so its elements satisfy
  // |x| <= maxq * (s + ulp(s) / 2); s = +0 comes with x = +-0 only, but the
  // unclamped form is checked there for every finite x.
  const uint32_t s_bits = blockIdx.x;
  const __half s16 = __ushort_as_half(static_cast<unsigned short>(s_bits));
  const BlockScale bs = make_block_scale(s16);
  const bool normal = s_bits >= 0x0400u;
  const int e_field = static_cast<int>(s_bits >> 10);  // binary16 exponent field, 1..30 when normal
  const float half_ulp = normal ? __int_as_float((e_field - 26 + 127) << 23) : 0.0f;
  const float reach = QParams<B>::maxq * (bs.s + half_ulp);  // exact: <= 17 significant bits
  unsigned long long bad = 0;
  for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
    if (((xb >> 10) & 0x1F) == 0x1F) continue;
    const float x = __half2float(__ushort_as_half(static_cast<unsigned short>(xb)));
    const uint32_t ref = quant_code_ieee<B>(x, bs.s);
    const uint32_t clamped = quant_code_bits<B, true>(x, bs) & ((1u << B) - 1);
    bad += (clamped != ref);
    if (s_bits == 0 || (normal && fabsf(x) <= reach)) {
      const uint32_t plain = quant_code_bits<B, false>(x, bs) & ((1u << B) - 1);
      bad += (plain != ref);
    }
  }
  if (bad) atomicAdd(mismatches, bad);
}

}  // namespace kvq

// ===========================================================================
// Host side: validation, tiling and launch.
// ===========================================================================

namespace {

using namespace kvq;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kvq_status check_desc(const kvq_cache_desc* d, int mult) {
  if (!d) return KVQ_ERR_NULL;
  if (d->dim0 < 1 || d->dim1 < 1 || d->kv_heads < 1 || d->head_dim < 1) return KVQ_ERR_SHAPE;
  if (d->head_dim % mult) return KVQ_ERR_SHAPE;
  if (static_cast<long long>(d->kv_heads) * d->head_dim > (1LL << 30)) return KVQ_ERR_SHAPE;
  return KVQ_OK;
}

int floor_pow2(long long x) {
  int r = 1;
  while (static_cast<long long>(r) * 2 <= x && r < (1 << 30)) r *= 2;
  return r;
}

int gcd_int(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// Positions per tile: about `target` elements, a power of two, and a divisor
// of page_size in paged mode.
int pick_tile_pos(long long hd, int page_size, long long target) {
  int t = floor_pow2(target / hd > 0 ? target / hd : 1);
  if (page_size > 0) t = gcd_int(t, page_size);
  return t;
}

kvq_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

// Engine chosen by kvq_set_engine (process-wide).
std::atomic<int> g_engine{KVQ_ENGINE_AUTO};

// What KVQ_ENGINE_AUTO runs: the engine measured faster on B200 for each
// operation.  The plain-load engine with per-sequence tiles wins every
// conversion measured (contiguous and paged, quantize and dequantize): the
// bulk engine and the balanced paged grid stay available.
template <class Op>
struct AutoEngine {
  static int pick(const Params&) { return KVQ_ENGINE_LDG_TILED; }
};

// Launch with programmatic stream serialization (the kernels wait on the
// previous grid themselves).
template <class Kernel, class... Args>
kvq_status launch_pdl(Kernel kernel, dim3 grid, int threads, int smem, void* stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return launch_status();
}

// CTAs of `kernel` that the current device holds at once (SMs x resident
// CTAs per SM), cached per device in `cache`; 0 if it cannot be queried.
template <class Kernel>
long long first_wave_ctas(Kernel kernel, int threads, int smem, std::atomic<long long>* cache, int max_devices) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= max_devices) {
    cudaGetLastError();
    return 0;
  }
  long long n = cache[dev].load();
  if (n == 0) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    n = static_cast<long long>(sms) * per_sm;
    cache[dev].store(n);
  }
  return n;
}

template <class Op, bool kPaged>
kvq_status launch_ldg_mode(Params p, int nkv, void* stream) {
  constexpr int kMaxDevices = 64;
  static std::atomic<long long> wave[kMaxDevices];
  p.prefetch_ctas = first_wave_ctas(convert_kernel<Op, kPaged>, LdgCfg<Op>::kThreads, 0, wave, kMaxDevices);
  // Paged tiles are several CTA rounds long: each CTA pays one block-table
  // lookup before its first data load, and a longer tile amortizes it.  Four
  // rounds when that still leaves at least two waves of CTAs (long windows),
  // two otherwise (short windows such as a 512-position prefill, where more,
  // shorter CTAs keep more loads in flight): measured on B200.
  int rounds = 1;
  if (kPaged) {
    rounds = 4;
    const int tp4 = pick_tile_pos(p.g.hd, p.g.page_size, static_cast<long long>(ldg_tile_elems<Op>()) * 4);
    const long long ctas4 =
        ((static_cast<long long>(p.g.width) + tp4 - 1) / tp4 + 1) * p.g.batch * static_cast<long long>(nkv);
    if (ctas4 < 2 * p.prefetch_ctas) rounds = 2;
  }
  const long long target = static_cast<long long>(ldg_tile_elems<Op>()) * rounds;
  p.g.tile_pos = pick_tile_pos(p.g.hd, p.g.page_size, target);
  const long long tiles = (static_cast<long long>(p.g.width) + p.g.tile_pos - 1) / p.g.tile_pos + (kPaged ? 1 : 0);
  if (tiles > 0x7FFFFFFFLL) return KVQ_ERR_RANGE;
  const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(p.g.batch < 65535 ? p.g.batch : 65535),
                  static_cast<unsigned>(nkv));
  return launch_pdl(convert_kernel<Op, kPaged>, grid, LdgCfg<Op>::kThreads, 0, stream, p);
}

// Paged mode on the balanced grid: one wave of CTAs (never more than there are
// positions to convert), each an equal share of the flattened windows.  Needs
// the batch to fit the kernel's shared-memory staging and the windows' total
// to fit an int (the caller checks).
template <class Op>
kvq_status launch_balanced(Params p, int nkv, void* stream) {
  constexpr int kMaxDevices = 64;
  static std::atomic<long long> wave[kMaxDevices];
  const long long ctas = first_wave_ctas(convert_balanced_kernel<Op>, LdgCfg<Op>::kThreads, 0, wave, kMaxDevices);
  if (ctas < 1) return KVQ_ERR_CUDA;
  const long long most = static_cast<long long>(p.g.batch) * p.g.width * nkv;  // windows are at most `width` long
  const unsigned grid = static_cast<unsigned>(most < ctas ? most : ctas);
  // a unit is two rounds of loads of the operation, in whole positions
  const long long per_round = 2 * ldg_tile_elems<Op>() / p.g.hd;
  const int unit = static_cast<int>(per_round < 1 ? 1 : (per_round > (1 << 20) ? (1 << 20) : per_round));
  return launch_pdl(convert_balanced_kernel<Op>, dim3(grid), LdgCfg<Op>::kThreads, 0, stream, p, nkv, unit);
}

bool balanced_eligible(const Params& p) {
  return p.g.page_size > 0 && p.g.batch <= kBalancedMaxBatch &&
         static_cast<long long>(p.g.batch) * p.g.width < 0x7FFFFFFFLL &&
         static_cast<long long>(p.g.bt_stride) * p.g.page_size < 0xFFFFFFFFLL;
}

template <class Op>
kvq_status launch_ldg(const Params& p, int nkv, void* stream, bool tiled) {
  if (p.g.page_size > 0) {
    if (!tiled && balanced_eligible(p)) return launch_balanced<Op>(p, nkv, stream);
    return launch_ldg_mode<Op, true>(p, nkv, stream);
  }
  return launch_ldg_mode<Op, false>(p, nkv, stream);
}

// The bulk engine needs every tile of the input stream 16-byte aligned and a
// multiple of 16 bytes (one position's bytes a multiple of 16), and one tile
// to fit a shared-memory stage.
template <class Op>
bool bulk_eligible(const Params& p) {
  const long long pos_bytes = p.g.hd * Op::kInNum / Op::kInDen;
  if (pos_bytes % 16 != 0) return false;
  const int tp = pick_tile_pos(p.g.hd, p.g.page_size, kBulkTileElems);
  return static_cast<long long>(tp) * pos_bytes <= kBulkStageBytes;
}

// Persistent grid: as many CTAs as fit on the device at once (cached per
// device), never more than there are tiles.
template <class Op>
kvq_status launch_bulk(Params p, int nkv, void* stream) {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> ctas_per_device[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  int ctas = ctas_per_device[dev].load();
  if (ctas == 0) {
    int sms = 0, per_sm = 0;
    if (cudaFuncSetAttribute(bulk_kernel<Op>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBulkSmemBytes) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bulk_kernel<Op>, kBulkThreads, kBulkSmemBytes) !=
            cudaSuccess) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
    ctas = sms * (per_sm > 0 ? per_sm : 1);
    ctas_per_device[dev].store(ctas);
  }
  p.g.tile_pos = pick_tile_pos(p.g.hd, p.g.page_size, kBulkTileElems);
  const int paged = p.g.page_size > 0;
  const long long tiles_x = (static_cast<long long>(p.g.width) + p.g.tile_pos - 1) / p.g.tile_pos + paged;
  const long long total = tiles_x * p.g.batch * nkv;
  if (tiles_x > 0x7FFFFFFFLL) return KVQ_ERR_RANGE;
  const unsigned grid = static_cast<unsigned>(total < ctas ? total : ctas);
  return launch_pdl(bulk_kernel<Op>, dim3(grid), kBulkThreads, kBulkSmemBytes, stream, p,
                    static_cast<int>(tiles_x), nkv);
}

template <class Op>
kvq_status launch(const Params& p, int nkv, void* stream) {
  int engine = g_engine.load(std::memory_order_relaxed);
  if (engine == KVQ_ENGINE_AUTO) engine = AutoEngine<Op>::pick(p);
  if (engine == KVQ_ENGINE_BULK && bulk_eligible<Op>(p)) return launch_bulk<Op>(p, nkv, stream);
  return launch_ldg<Op>(p, nkv, stream, engine == KVQ_ENGINE_LDG_TILED);
}

Geometry make_geometry(const kvq_cache_desc* d, int batch, int offset, int width, int page_size,
                       const int32_t* seqlens, const int32_t* block_table) {
  Geometry g;
  g.dim0 = d->dim0;
  g.dim1 = d->dim1;
  g.hd = static_cast<long long>(d->kv_heads) * d->head_dim;
  g.bt_stride = d->block_table_stride;
  g.batch = batch;
  g.offset = offset;
  g.width = width;
  g.page_size = page_size;
  g.tile_pos = 1;  // set per kernel at launch
  g.seqlens = seqlens;
  g.block_table = block_table;
  return g;
}

kvq_status check_contiguous_window(const kvq_cache_desc* d, int batch, int offset, int width) {
  if (batch < 0 || width < 0 || offset < 0) return KVQ_ERR_RANGE;
  if (batch > d->dim0) return KVQ_ERR_RANGE;
  if (static_cast<long long>(offset) + width > d->dim1) return KVQ_ERR_RANGE;
  return KVQ_OK;
}

kvq_status fp8_common(const void* in, void* out, const kvq_cache_desc* d, int batch, int offset,
                      int width, void* stream, bool encode) {
  if (!in || !out) return KVQ_ERR_NULL;
  kvq_status st = check_desc(d, 8);
  if (st != KVQ_OK) return st;
  if (!aligned16(in) || !aligned16(out)) return KVQ_ERR_ALIGN;
  st = check_contiguous_window(d, batch, offset, width);
  if (st != KVQ_OK) return st;
  if (batch == 0 || width == 0) return KVQ_OK;
  Params p{};
  p.g = make_geometry(d, batch, offset, width, 0, nullptr, nullptr);
  p.in[0] = in;
  p.out[0] = out;
  return encode ? launch<Fp8Encode>(p, 1, stream) : launch<Fp8Decode>(p, 1, stream);
}

// Window / page checks shared by the K+V conversions.
kvq_status check_kv_window(const kvq_cache_desc* d, int batch, int offset, int width, int page_size,
                           const int32_t* seqlens, const int32_t* block_table) {
  if (page_size < 0) return KVQ_ERR_RANGE;
  if (page_size == 0) return check_contiguous_window(d, batch, offset, width);
  if (!seqlens || !block_table) return KVQ_ERR_NULL;
  if (page_size != d->dim1 || batch < 0 || width < 0) return KVQ_ERR_RANGE;
  if (d->block_table_stride < 1) return KVQ_ERR_RANGE;
  if ((reinterpret_cast<uintptr_t>(seqlens) | reinterpret_cast<uintptr_t>(block_table)) & 3u) return KVQ_ERR_ALIGN;
  return KVQ_OK;
}

kvq_status fp8_kv_common(const void* k_in, void* k_out, const void* v_in, void* v_out, const kvq_cache_desc* d,
                         int batch, int offset, int width, int page_size, const int32_t* seqlens,
                         const int32_t* block_table, void* stream, bool encode) {
  if (!k_in || !k_out || !v_in || !v_out) return KVQ_ERR_NULL;
  kvq_status st = check_desc(d, 8);
  if (st != KVQ_OK) return st;
  const void* ptrs[4] = {k_in, k_out, v_in, v_out};
  for (const void* q : ptrs)
    if (!aligned16(q)) return KVQ_ERR_ALIGN;
  st = check_kv_window(d, batch, offset, width, page_size, seqlens, block_table);
  if (st != KVQ_OK) return st;
  if (batch == 0 || width == 0) return KVQ_OK;
  Params p{};
  p.g = make_geometry(d, batch, offset, width, page_size, seqlens, block_table);
  p.in[0] = k_in;
  p.in[1] = v_in;
  p.out[0] = k_out;
  p.out[1] = v_out;
  return encode ? launch<Fp8Encode>(p, 2, stream) : launch<Fp8Decode>(p, 2, stream);
}

kvq_status q_common(const void* k_in, void* k_out, void* k_scales, const void* v_in, void* v_out,
                    void* v_scales, const kvq_cache_desc* d, int batch, int offset, int width,
                    int page_size, const int32_t* seqlens, const int32_t* block_table, int wbits,
                    void* stream, bool encode) {
  if (!k_in || !k_out || !k_scales || !v_in || !v_out || !v_scales) return KVQ_ERR_NULL;
  kvq_status st = check_desc(d, kBlockElems);
  if (st != KVQ_OK) return st;
  if (wbits != 4 && wbits != 6 && wbits != 8) return KVQ_ERR_WBITS;
  const void* ptrs[6] = {k_in, k_out, k_scales, v_in, v_out, v_scales};
  for (const void* q : ptrs)
    if (!aligned16(q)) return KVQ_ERR_ALIGN;
  st = check_kv_window(d, batch, offset, width, page_size, seqlens, block_table);
  if (st != KVQ_OK) return st;
  if (batch == 0 || width == 0) return KVQ_OK;
  Params p{};
  p.g = make_geometry(d, batch, offset, width, page_size, seqlens, block_table);
  p.in[0] = k_in;
  p.in[1] = v_in;
  p.out[0] = k_out;
  p.out[1] = v_out;
  p.scales[0] = k_scales;
  p.scales[1] = v_scales;
  if (encode) {
    if (wbits == 4) return launch<QEncode<4>>(p, 2, stream);
    if (wbits == 6) return launch<QEncode<6>>(p, 2, stream);
    return launch<QEncode<8>>(p, 2, stream);
  }
  if (wbits == 4) return launch<QDecode<4>>(p, 2, stream);
  if (wbits == 6) return launch<QDecode<6>>(p, 2, stream);
  return launch<QDecode<8>>(p, 2, stream);
}

}  // namespace

extern "C" {

kvq_status kvq_fp16_to_fp8(const void* in, void* out, const kvq_cache_desc* desc, int batch_size,
                           int offset, int width, void* stream) {
  return fp8_common(in, out, desc, batch_size, offset, width, stream, true);
}

kvq_status kvq_fp8_to_fp16(const void* in, void* out, const kvq_cache_desc* desc, int batch_size,
                           int offset, int width, void* stream) {
  return fp8_common(in, out, desc, batch_size, offset, width, stream, false);
}

kvq_status kvq_fp16_to_fp8_kv(const void* k_in, void* k_out, const void* v_in, void* v_out,
                              const kvq_cache_desc* desc, int batch_size, int offset, int width,
                              int page_size, const int32_t* cache_seqlens, const int32_t* block_table,
                              void* stream) {
  return fp8_kv_common(k_in, k_out, v_in, v_out, desc, batch_size, offset, width, page_size, cache_seqlens,
                       block_table, stream, true);
}

kvq_status kvq_fp8_to_fp16_kv(const void* k_in, void* k_out, const void* v_in, void* v_out,
                              const kvq_cache_desc* desc, int batch_size, int offset, int width,
                              int page_size, const int32_t* cache_seqlens, const int32_t* block_table,
                              void* stream) {
  return fp8_kv_common(k_in, k_out, v_in, v_out, desc, batch_size, offset, width, page_size, cache_seqlens,
                       block_table, stream, false);
}

kvq_status kvq_fp16_to_q_kv(const void* k_in, void* k_out, void* k_scales, const void* v_in,
                            void* v_out, void* v_scales, const kvq_cache_desc* desc, int batch_size,
                            int offset, int width, int page_size, const int32_t* cache_seqlens,
                            const int32_t* block_table, int wbits, void* stream) {
  return q_common(k_in, k_out, k_scales, v_in, v_out, v_scales, desc, batch_size, offset, width,
                  page_size, cache_seqlens, block_table, wbits, stream, true);
}

kvq_status kvq_q_to_fp16_kv(const void* k_in, void* k_out, const void* k_scales, const void* v_in,
                            void* v_out, const void* v_scales, const kvq_cache_desc* desc,
                            int batch_size, int offset, int width, int page_size,
                            const int32_t* cache_seqlens, const int32_t* block_table, int wbits,
                            void* stream) {
  return q_common(k_in, k_out, const_cast<void*>(k_scales), v_in, v_out, const_cast<void*>(v_scales),
                  desc, batch_size, offset, width, page_size, cache_seqlens, block_table, wbits,
                  stream, false);
}

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_NULL: return "null pointer";
    case KVQ_ERR_SHAPE: return "bad shape";
    case KVQ_ERR_WBITS: return "wbits must be 4, 6 or 8";
    case KVQ_ERR_RANGE: return "window, batch or page geometry out of range";
    case KVQ_ERR_ALIGN: return "buffer not 16-byte aligned";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    case KVQ_ERR_DEVICE: return "device recorded bad paging metadata";
  }
  return "unknown status";
}

kvq_status kvq_poll_device_error(int32_t* code_out, void* stream) {
  if (!code_out) return KVQ_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&h, kvq::g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return KVQ_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(kvq::g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return KVQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
  *code_out = h;
  return h ? KVQ_ERR_DEVICE : KVQ_OK;
}

}  // extern "C"

// Decode attention over the converted caches: host side.
#include "attention_api.cuh"

extern "C" {

long long kvq_count_match(const int64_t* a, long long a_len, const int64_t* b, long long b_len, long long max_a) {
  long long n = a_len < b_len ? a_len : b_len;
  if (max_a < n) n = max_a;
  if (n <= 0) return 0;
  if (!a || !b) return -1;
  long long i = 0;
  while (i < n && a[i] == b[i]) ++i;
  return i;
}

kvq_status kvq_set_engine(int engine) {
  if (engine != KVQ_ENGINE_AUTO && engine != KVQ_ENGINE_LDG && engine != KVQ_ENGINE_BULK &&
      engine != KVQ_ENGINE_LDG_TILED)
    return KVQ_ERR_RANGE;
  g_engine.store(engine);
  return KVQ_OK;
}

int kvq_get_engine(void) { return g_engine.load(); }

kvq_status kvq_set_attention_path(int path) {
  if (path != KVQ_ATTENTION_AUTO && path != KVQ_ATTENTION_MMA && path != KVQ_ATTENTION_TCGEN05) return KVQ_ERR_RANGE;
  g_attention_path.store(path);
  return KVQ_OK;
}

int kvq_get_attention_path(void) { return g_attention_path.load(); }

kvq_status kvq_selfcheck_code_rounding(int wbits, unsigned long long* mismatches, void* stream) {
  if (!mismatches) return KVQ_ERR_NULL;
  if (wbits != 4 && wbits != 6 && wbits != 8) return KVQ_ERR_WBITS;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(mismatches, 0, sizeof(unsigned long long), s) != cudaSuccess) return KVQ_ERR_CUDA;
  if (wbits == 4)
    kvq::selfcheck_rounding_kernel<4><<<0x7C00, 256, 0, s>>>(mismatches);
  else if (wbits == 6)
    kvq::selfcheck_rounding_kernel<6><<<0x7C00, 256, 0, s>>>(mismatches);
  else
    kvq::selfcheck_rounding_kernel<8><<<0x7C00, 256, 0, s>>>(mismatches);
  return launch_status();
}

}  // extern "C"

// The self-check of the arithmetic the decode-attention error bound rests on.
#include "attention_selfcheck.cuh"
