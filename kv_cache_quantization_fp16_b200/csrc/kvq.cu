// kvq.cu -- sm_100a kernels and the C ABI (include/kvq.h) of libkvq.so.
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
// never straddles a page.  One CTA converts one tile: thread 0 resolves the
// tile (window clipping, the block_table lookup) once and stages the physical
// row in shared memory, then all threads stream the tile's elements as a flat
// array; each op fixes its CTA size and how many independent loads every
// thread has in flight (see the per-op structs).  Grid: x = tiles, y =
// sequences, z = K / V (the fused K+V launch).
//
// This is a streaming, HBM-bound path: no tensor cores, no shared-memory
// staging of the data, no collectives.

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvq.h"
#include "codec.cuh"

namespace kvq {

constexpr int kBlockElems = 32;  // Q scale block along head_dim

// Per-device error word for problems only the device can see.
__device__ int g_device_error;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_error, 0, code); }

struct Geometry {
  int dim0, dim1;
  long long hd;  // kv_heads * head_dim: elements per position
  int bt_stride;
  int batch, offset, width, page_size;
  int tile_pos;
  const int32_t* seqlens;
  const int32_t* block_table;
};

// Tile `tile_x` of sequence `seq` in contiguous mode: first row and number of
// positions, or false when the tile lies past the end of the window.
__device__ __forceinline__ bool contiguous_tile(const Geometry& g, int seq, int tile_x, long long& row0,
                                                int& nrows) {
  const long long p0 = static_cast<long long>(g.offset) + static_cast<long long>(tile_x) * g.tile_pos;
  const long long p1 = min(static_cast<long long>(g.offset) + g.width, p0 + g.tile_pos);
  if (p0 >= p1) return false;
  row0 = static_cast<long long>(seq) * g.dim1 + p0;
  nrows = static_cast<int>(p1 - p0);
  return true;
}

// Paged mode: the window of sequence `seq` is [max(0, seqlen + offset),
// seqlen + offset + width) in logical positions; tile `tile_x` is the x-th
// tile_pos-aligned run of it (tile_pos divides page_size, so the run lies in
// one page).  `bt_row` is the sequence's block-table row staged in shared
// memory (or null: read it from global memory).  Bad metadata is recorded by
// the thread with `report` set and the tile is skipped.
__device__ __forceinline__ bool paged_tile(const Geometry& g, int seq, int tile_x, int seqlen,
                                           const int* bt_row, bool report, long long& row0, int& nrows) {
  const long long start = static_cast<long long>(seqlen) + g.offset;
  const long long lo = start < 0 ? 0 : start;
  const long long hi = start + g.width;
  if (lo >= hi) return false;
  const long long t0 = (lo / g.tile_pos) * g.tile_pos + static_cast<long long>(tile_x) * g.tile_pos;
  const long long p0 = max(lo, t0);
  const long long p1 = min(hi, t0 + g.tile_pos);
  if (p0 >= p1) return false;
  const long long lp = p0 / g.page_size;
  if (lp >= g.bt_stride) {
    if (report) record_error(KVQ_DEV_BAD_PAGE_INDEX);
    return false;
  }
  const int page = bt_row ? bt_row[lp] : g.block_table[static_cast<long long>(seq) * g.bt_stride + lp];
  if (page < 0 || page >= g.dim0) {
    if (report) record_error(KVQ_DEV_BAD_PAGE);
    return false;
  }
  row0 = static_cast<long long>(page) * g.page_size + p0 % g.page_size;
  nrows = static_cast<int>(p1 - p0);
  return true;
}

struct Params {
  Geometry g;
  const void* in[2];
  void* out[2];
  void* scales[2];  // Q encode: written; Q decode: read
};

// ---------------------------------------------------------------------------
// Per-tile bodies
// ---------------------------------------------------------------------------

// FP8: 128-thread CTAs with 8 independent 16-byte loads (or 8-byte loads for
// decode) per thread, so a whole tile is requested at once and enough CTAs
// stay resident (up to 16 per SM) for small windows to run in one wave.
struct Fp8Encode {
  static constexpr int kThreads = 128;
  static constexpr int kUnroll = 8;
  static constexpr int kElemsPerTile = kThreads * kUnroll * 8;
  static constexpr int kMinBlocksPerSM = 8;
  __device__ static void tile(const Params& p, int kv, long long row0, int nrows) {
    const long long e0 = row0 * p.g.hd;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __half*>(p.in[kv]) + e0);
    uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.out[kv]) + e0);
    const int nvec = static_cast<int>(nrows * p.g.hd / 8);
    for (int base = 0; base < nvec; base += kThreads * kUnroll) {
      uint4 x[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = base + u * kThreads + threadIdx.x;
        if (v < nvec) x[u] = __ldg(src + v);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = base + u * kThreads + threadIdx.x;
        if (v < nvec) dst[v] = e5m2_encode_v8(x[u]);
      }
    }
  }
};

struct Fp8Decode {
  static constexpr int kThreads = 128;
  static constexpr int kUnroll = 8;
  static constexpr int kElemsPerTile = kThreads * kUnroll * 8;
  static constexpr int kMinBlocksPerSM = 8;
  __device__ static void tile(const Params& p, int kv, long long row0, int nrows) {
    const long long e0 = row0 * p.g.hd;
    const uint2* src = reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(p.in[kv]) + e0);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.out[kv]) + e0);
    const int nvec = static_cast<int>(nrows * p.g.hd / 8);
    for (int base = 0; base < nvec; base += kThreads * kUnroll) {
      uint2 x[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = base + u * kThreads + threadIdx.x;
        if (v < nvec) x[u] = __ldg(src + v);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = base + u * kThreads + threadIdx.x;
        if (v < nvec) dst[v] = e5m2_decode_v8(x[u]);
      }
    }
  }
};

// Q encode: one thread owns whole 32-element blocks (4 x 16-byte loads), so
// the absmax needs no shuffles, the scale and reciprocal are computed once per
// block, and the packed codes leave as one 16-byte (Q4) or three 8-byte (Q6)
// stores.  Two blocks per thread are loaded before either is encoded.
template <int B>
struct QEncode {
  static constexpr int kThreads = 256;
  static constexpr int kUnrollBlocks = 2;
  static constexpr int kElemsPerTile = kThreads * kBlockElems * kUnrollBlocks;
  static constexpr int kMinBlocksPerSM = 4;

  __device__ static void tile(const Params& p, int kv, long long row0, int nrows) {
    const long long e0 = row0 * p.g.hd;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __half*>(p.in[kv]) + e0);
    uint8_t* codes = static_cast<uint8_t*>(p.out[kv]) + e0 * B / 8;
    __half* scales = static_cast<__half*>(p.scales[kv]) + e0 / kBlockElems;
    const int nblk = static_cast<int>(nrows * p.g.hd / kBlockElems);
    for (int base = 0; base < nblk; base += kThreads * kUnrollBlocks) {
      uint4 x[kUnrollBlocks][4];
#pragma unroll
      for (int u = 0; u < kUnrollBlocks; ++u) {
        const int b = base + u * kThreads + threadIdx.x;
        if (b < nblk) {
#pragma unroll
          for (int k = 0; k < 4; ++k) x[u][k] = __ldg(src + static_cast<long long>(b) * 4 + k);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnrollBlocks; ++u) {
        const int b = base + u * kThreads + threadIdx.x;
        if (b >= nblk) continue;
        const __half s16 = block_scale<B>(absmax_bits_block(x[u]));
        const BlockScale bs = make_block_scale(s16);
        uint32_t w[B];
        if (__half_as_ushort(s16) < 0x0400u)
          encode_block_words<B, true>(x[u], bs, w);
        else
          encode_block_words<B, false>(x[u], bs, w);
        if (B == 4) {
          reinterpret_cast<uint4*>(codes)[b] = make_uint4(w[0], w[1], w[2 % B], w[3 % B]);
        } else {
          uint2* dst = reinterpret_cast<uint2*>(codes + static_cast<long long>(b) * 24);
          dst[0] = make_uint2(w[0], w[1]);
          dst[1] = make_uint2(w[2 % B], w[3 % B]);
          dst[2] = make_uint2(w[4 % B], w[5 % B]);
        }
        scales[b] = s16;
      }
    }
  }
};

template <int B>
struct QDecode {
  static constexpr int kThreads = 256;
  static constexpr int kUnroll = 4;
  static constexpr int kElemsPerTile = kThreads * kUnroll * 8;
  static constexpr int kMinBlocksPerSM = 5;
  __device__ static void tile(const Params& p, int kv, long long row0, int nrows) {
    const long long e0 = row0 * p.g.hd;
    const uint8_t* codes = static_cast<const uint8_t*>(p.in[kv]) + e0 * B / 8;
    const __half* scales = static_cast<const __half*>(p.scales[kv]) + e0 / kBlockElems;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.out[kv]) + e0);
    const int nvec = static_cast<int>(nrows * p.g.hd / 8);
    for (int base = 0; base < nvec; base += kThreads * kUnroll) {
      uint32_t lo[kUnroll], hi[kUnroll];
      __half s[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = base + u * kThreads + threadIdx.x;
        lo[u] = hi[u] = 0;
        s[u] = __ushort_as_half(0);
        if (v < nvec) {
          if (B == 4) {
            lo[u] = __ldg(reinterpret_cast<const uint32_t*>(codes) + v);
          } else {
            // lane pair = one 12-byte group; the even lane needs words 0-1, the
            // odd lane words 1-2 (bits 48..95 of the group)
            const uint32_t* grp = reinterpret_cast<const uint32_t*>(codes + static_cast<long long>(v >> 1) * 12);
            const uint32_t sh = (v & 1) * 16;
            const uint32_t a = __ldg(grp + (v & 1));
            const uint32_t b = __ldg(grp + (v & 1) + 1);
            lo[u] = __funnelshift_r(a, b, sh);
            hi[u] = (b >> sh) & 0xFFFFu;
          }
          s[u] = __ldg(scales + (v >> 2));
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = base + u * kThreads + threadIdx.x;
        if (v >= nvec) continue;
        const __half2 s2 = __halves2half2(s[u], s[u]);
        dst[v] = (B == 4) ? dequant_q4_v8(lo[u], s2) : dequant_q6_v8(lo[u], hi[u], s2);
      }
    }
  }
};

// ---------------------------------------------------------------------------
// The kernel: one tile per CTA; the tile is resolved once and staged in smem.
// ---------------------------------------------------------------------------

template <class Op>
__global__ void __launch_bounds__(Op::kThreads, Op::kMinBlocksPerSM) convert_kernel(const __grid_constant__ Params p) {
  // Programmatic dependent launch: this grid may be launched while the
  // previous kernel on the stream is still running; wait for it to finish (and
  // its writes to become visible) before touching global memory, and let the
  // next kernel start launching as soon as every CTA of this grid has started.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int s_bt[Op::kThreads];
  __shared__ int s_seqlen;
  const int kv = blockIdx.z;
  for (int seq = blockIdx.y; seq < p.g.batch; seq += gridDim.y) {
    long long row0 = 0;
    int nrows = 0;
    bool ok;
    if (p.g.page_size == 0) {
      ok = contiguous_tile(p.g, seq, blockIdx.x, row0, nrows);
    } else {
      // Stage the sequence's block-table row (when it fits) together with its
      // length, so the page lookup costs one memory round trip, not two.
      const bool staged = p.g.bt_stride <= Op::kThreads;
      if (staged && static_cast<int>(threadIdx.x) < p.g.bt_stride)
        s_bt[threadIdx.x] = p.g.block_table[static_cast<long long>(seq) * p.g.bt_stride + threadIdx.x];
      if (threadIdx.x == 0) s_seqlen = p.g.seqlens[seq];
      __syncthreads();
      ok = paged_tile(p.g, seq, blockIdx.x, s_seqlen, staged ? s_bt : nullptr, threadIdx.x == 0, row0, nrows);
      __syncthreads();  // s_bt and s_seqlen are rewritten for the next sequence
    }
    if (ok) Op::tile(p, kv, row0, nrows);
  }
}

// ---------------------------------------------------------------------------
// Self-check of the fast code rounding against IEEE division.
// ---------------------------------------------------------------------------

template <int B>
__global__ void selfcheck_rounding_kernel(unsigned long long* mismatches) {
  // blockIdx.x enumerates s bit patterns 1..0x7BFF; threads enumerate x over
  // all 65536 bit patterns, skipping Inf / NaN.  Both forms the kernels use
  // are checked: the clamped one for every pair, the unclamped one (used when
  // the scale is normal) for every pair a block can produce.  A block gets the
  // scale s only if absmax / maxq rounds to s, so its elements satisfy
  // |x| <= maxq * (s + ulp(s) / 2).
  const uint32_t s_bits = 1 + blockIdx.x;
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
    if (normal && fabsf(x) <= reach) {
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

template <class Op>
kvq_status launch(Params p, int nkv, void* stream) {
  p.g.tile_pos = pick_tile_pos(p.g.hd, p.g.page_size, Op::kElemsPerTile);
  const int paged = p.g.page_size > 0;
  const long long tiles = (static_cast<long long>(p.g.width) + p.g.tile_pos - 1) / p.g.tile_pos + paged;
  if (tiles > 0x7FFFFFFFLL) return KVQ_ERR_RANGE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(p.g.batch < 65535 ? p.g.batch : 65535),
                     static_cast<unsigned>(nkv));
  cfg.blockDim = dim3(Op::kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, convert_kernel<Op>, p) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return launch_status();
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
  g.tile_pos = 1;  // set per kernel by launch()
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

kvq_status q_common(const void* k_in, void* k_out, void* k_scales, const void* v_in, void* v_out,
                    void* v_scales, const kvq_cache_desc* d, int batch, int offset, int width,
                    int page_size, const int32_t* seqlens, const int32_t* block_table, int wbits,
                    void* stream, bool encode) {
  if (!k_in || !k_out || !k_scales || !v_in || !v_out || !v_scales) return KVQ_ERR_NULL;
  kvq_status st = check_desc(d, kBlockElems);
  if (st != KVQ_OK) return st;
  if (wbits != 4 && wbits != 6) return KVQ_ERR_WBITS;
  const void* ptrs[6] = {k_in, k_out, k_scales, v_in, v_out, v_scales};
  for (const void* q : ptrs)
    if (!aligned16(q)) return KVQ_ERR_ALIGN;
  if (page_size < 0) return KVQ_ERR_RANGE;
  if (page_size == 0) {
    st = check_contiguous_window(d, batch, offset, width);
    if (st != KVQ_OK) return st;
  } else {
    if (!seqlens || !block_table) return KVQ_ERR_NULL;
    if (page_size != d->dim1 || batch < 0 || width < 0) return KVQ_ERR_RANGE;
    if (d->block_table_stride < 1) return KVQ_ERR_RANGE;
    if ((reinterpret_cast<uintptr_t>(seqlens) | reinterpret_cast<uintptr_t>(block_table)) & 3u)
      return KVQ_ERR_ALIGN;
  }
  if (batch == 0 || width == 0) return KVQ_OK;
  Params p{};
  p.g = make_geometry(d, batch, offset, width, page_size, seqlens, block_table);
  p.in[0] = k_in;
  p.in[1] = v_in;
  p.out[0] = k_out;
  p.out[1] = v_out;
  p.scales[0] = k_scales;
  p.scales[1] = v_scales;
  if (encode) return wbits == 4 ? launch<QEncode<4>>(p, 2, stream) : launch<QEncode<6>>(p, 2, stream);
  return wbits == 4 ? launch<QDecode<4>>(p, 2, stream) : launch<QDecode<6>>(p, 2, stream);
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
    case KVQ_ERR_WBITS: return "wbits must be 4 or 6";
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

kvq_status kvq_selfcheck_code_rounding(int wbits, unsigned long long* mismatches, void* stream) {
  if (!mismatches) return KVQ_ERR_NULL;
  if (wbits != 4 && wbits != 6) return KVQ_ERR_WBITS;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(mismatches, 0, sizeof(unsigned long long), s) != cudaSuccess) return KVQ_ERR_CUDA;
  if (wbits == 4)
    kvq::selfcheck_rounding_kernel<4><<<0x7BFF, 256, 0, s>>>(mismatches);
  else
    kvq::selfcheck_rounding_kernel<6><<<0x7BFF, 256, 0, s>>>(mismatches);
  return launch_status();
}

}  // extern "C"
