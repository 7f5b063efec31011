// ops.cuh -- per-tile bodies of the four conversions, shared by both load
// engines (plain 16-byte global loads, and TMA bulk copies into shared
// memory).  A tile is `nrows` positions starting at physical row `row0`, a
// flat contiguous run of nrows * H * D elements in every tensor.
//
// The operations are fp16_to_fp8 / fp8_to_fp16 / fp16_to_q_kv / q_to_fp16_kv
// of the page "Implementation: Turboderp org Exllamav2 Ext Cache"
// (Description; I/O Contract); the arithmetic lives in codec.cuh.
//
// Each body is templated on where its main input stream is read from (`Src`:
// global memory through the non-coherent path, or a shared-memory copy of
// the tile), on the number of threads that share the tile (NT), on how many
// independent loads each thread issues before it computes (U: one round of
// loads), and on whether each round asks L2 for the next round's input
// (kPf, for tiles of several rounds read from global memory).
#pragma once

#include "codec.cuh"
#include "tiles.cuh"

namespace kvq {

struct GlobalSrc {
  static constexpr bool kGlobal = true;
  template <class T>
  __device__ __forceinline__ static T load(const T* p) { return __ldg(p); }
};

struct SharedSrc {
  static constexpr bool kGlobal = false;
  template <class T>
  __device__ __forceinline__ static T load(const T* p) { return *p; }
};

// L2 prefetch of `bytes` bytes from `base`: one 128-byte line per thread and
// step (plus the last byte, so a range that starts mid-line is covered).
__device__ __forceinline__ void prefetch_l2_range(const void* base, long long bytes, int tid, int nthreads) {
  if (bytes <= 0) return;
  const char* b = static_cast<const char*>(base);
  for (long long off = static_cast<long long>(tid) * 128; off < bytes; off += static_cast<long long>(nthreads) * 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(b + off));
  if (tid == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(b + bytes - 1));
}

// In a tile of several rounds (paged tiles), ask L2 for the next round's
// input units [next, next + per_round) while this round is converted, so that
// DRAM keeps streaming between the rounds of a CTA.  Units are `unit_bytes`
// apart in the input stream.  A prefetch never changes what a load returns.
template <bool kOn>
__device__ __forceinline__ void prefetch_next_round(const void* in, int unit_bytes, int next, int total,
                                                    int per_round, int tid, int nt) {
  if (!kOn || next >= total) return;
  const int units = min(per_round, total - next);
  prefetch_l2_range(static_cast<const uint8_t*>(in) + static_cast<long long>(next) * unit_bytes,
                    static_cast<long long>(units) * unit_bytes, tid, nt);
}

// FP8 encode: 8 binary16 (16 bytes) in, 8 bytes out per thread step.
struct Fp8Encode {
  static constexpr int kInNum = 2, kInDen = 1;  // input bytes per element
  static constexpr bool kReadsScales = false;
  template <class Src, int NT, int U, bool kPf>
  __device__ static void body(const Params& p, int kv, long long row0, int nrows, const void* in, int tid) {
    const long long e0 = row0 * p.g.hd;
    const uint4* src = static_cast<const uint4*>(in);
    uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.out[kv]) + e0);
    const int nvec = static_cast<int>(nrows * p.g.hd / 8);
    for (int base = 0; base < nvec; base += NT * U) {
      prefetch_next_round<kPf>(in, 16, base + NT * U, nvec, NT * U, tid, NT);
      uint4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = base + u * NT + tid;
        if (v < nvec) x[u] = Src::load(src + v);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = base + u * NT + tid;
        if (v < nvec) dst[v] = e5m2_encode_v8(x[u]);
      }
    }
  }
};

// FP8 decode: 8 bytes in, 8 binary16 out per thread step.
struct Fp8Decode {
  static constexpr int kInNum = 1, kInDen = 1;
  static constexpr bool kReadsScales = false;
  template <class Src, int NT, int U, bool kPf>
  __device__ static void body(const Params& p, int kv, long long row0, int nrows, const void* in, int tid) {
    const long long e0 = row0 * p.g.hd;
    const uint2* src = static_cast<const uint2*>(in);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.out[kv]) + e0);
    const int nvec = static_cast<int>(nrows * p.g.hd / 8);
    for (int base = 0; base < nvec; base += NT * U) {
      prefetch_next_round<kPf>(in, 8, base + NT * U, nvec, NT * U, tid, NT);
      uint2 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = base + u * NT + tid;
        if (v < nvec) x[u] = Src::load(src + v);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = base + u * NT + tid;
        if (v < nvec) dst[v] = e5m2_decode_v8(x[u]);
      }
    }
  }
};

// Q encode: one thread owns whole 32-element blocks (4 x 16-byte loads), so
// the absmax needs no shuffles, the scale and reciprocal are computed once per
// block, and the packed codes leave as one 16-byte (Q4), three 8-byte (Q6) or
// two 16-byte (Q8) stores.  U blocks per thread are loaded before any is encoded.
template <int B>
struct QEncode {
  static constexpr int kInNum = 2, kInDen = 1;
  static constexpr bool kReadsScales = false;
  template <class Src, int NT, int U, bool kPf>
  __device__ static void body(const Params& p, int kv, long long row0, int nrows, const void* in, int tid) {
    const long long e0 = row0 * p.g.hd;
    const uint4* src = static_cast<const uint4*>(in);
    uint8_t* codes = static_cast<uint8_t*>(p.out[kv]) + e0 * B / 8;
    __half* scales = static_cast<__half*>(p.scales[kv]) + e0 / kBlockElems;
    const int nblk = static_cast<int>(nrows * p.g.hd / kBlockElems);
    for (int base = 0; base < nblk; base += NT * U) {
      prefetch_next_round<kPf>(in, 64, base + NT * U, nblk, NT * U, tid, NT);
      uint4 x[U][4];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int b = base + u * NT + tid;
        if (b < nblk) {
#pragma unroll
          for (int k = 0; k < 4; ++k) x[u][k] = Src::load(src + static_cast<long long>(b) * 4 + k);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int b = base + u * NT + tid;
        if (b >= nblk) continue;
        const __half s16 = block_scale<B>(absmax_bits_block(x[u]));
        const BlockScale bs = make_block_scale(s16);
        uint32_t w[B];
        // Only a nonzero subnormal scale needs the clamp; a zero scale (all-zero
        // block) gives rh = rl = 0, hence code z, on the unclamped path too, so
        // zero blocks do not split a warp across both paths.
        if (__half_as_ushort(s16) - 1u < 0x03FFu)
          encode_block_words<B, true>(x[u], bs, w);
        else
          encode_block_words<B, false>(x[u], bs, w);
        if (B == 4) {
          reinterpret_cast<uint4*>(codes)[b] = make_uint4(w[0], w[1], w[2 % B], w[3 % B]);
        } else if (B == 8) {
          uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<long long>(b) * 32);
          dst[0] = make_uint4(w[0], w[1], w[2 % B], w[3 % B]);
          dst[1] = make_uint4(w[4 % B], w[5 % B], w[6 % B], w[7 % B]);
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

// Q decode: a quad of lanes covers one 32-element block, 8 elements (one
// 16-byte FP16 store) per lane, so the stores of a warp are contiguous.
template <int B>
struct QDecode {
  static constexpr int kInNum = B, kInDen = 8;
  static constexpr bool kReadsScales = true;
  template <class Src, int NT, int U, bool kPf>
  __device__ static void body(const Params& p, int kv, long long row0, int nrows, const void* in, int tid) {
    const long long e0 = row0 * p.g.hd;
    const uint8_t* codes = static_cast<const uint8_t*>(in);
    const __half* scales = static_cast<const __half*>(p.scales[kv]) + e0 / kBlockElems;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.out[kv]) + e0);
    const int nvec = static_cast<int>(nrows * p.g.hd / 8);
    for (int base = 0; base < nvec; base += NT * U) {
      prefetch_next_round<kPf>(in, B, base + NT * U, nvec, NT * U, tid, NT);  // codes: B bytes per 8 elements
      prefetch_next_round<kPf>(scales, 2, (base + NT * U) / 4, nvec / 4, NT * U / 4, tid, NT);
      uint32_t lo[U], hi[U];
      __half s[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = base + u * NT + tid;
        lo[u] = hi[u] = 0;
        s[u] = __ushort_as_half(0);
        if (v < nvec) {
          if (B == 4) {
            lo[u] = Src::load(reinterpret_cast<const uint32_t*>(codes) + v);
          } else if (B == 8) {
            const uint2 q = Src::load(reinterpret_cast<const uint2*>(codes) + v);
            lo[u] = q.x;
            hi[u] = q.y;
          } else {
            // lane pair = one 12-byte group; the even lane needs words 0-1, the
            // odd lane words 1-2 (bits 48..95 of the group)
            const uint32_t* grp = reinterpret_cast<const uint32_t*>(codes + static_cast<long long>(v >> 1) * 12);
            const uint32_t sh = (v & 1) * 16;
            const uint32_t a = Src::load(grp + (v & 1));
            const uint32_t b = Src::load(grp + (v & 1) + 1);
            lo[u] = __funnelshift_r(a, b, sh);
            hi[u] = (b >> sh) & 0xFFFFu;
          }
          s[u] = __ldg(scales + (v >> 2));
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = base + u * NT + tid;
        if (v >= nvec) continue;
        const __half2 s2 = __halves2half2(s[u], s[u]);
        dst[v] = (B == 4) ? dequant_q4_v8(lo[u], s2)
                 : (B == 8) ? dequant_q8_v8(lo[u], hi[u], s2)
                            : dequant_q6_v8(lo[u], hi[u], s2);
      }
    }
  }
};

}  // namespace kvq
