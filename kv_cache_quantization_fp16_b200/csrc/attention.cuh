// attention.cuh -- decode attention that reads the quantized KV cache
// directly: the conversions' consumer "during the attention forward pass"
// (page "Implementation: Turboderp org Exllamav2 Ext Cache", Usage), with the
// FP16 cache never written back.
//
// One new query per sequence and head; GQA: `group` query heads share a kv
// head.  Keys and values are the dequantized codes, bit for bit what
// q_to_fp16_kv writes: RN16((code - z) * s), with (code - z) formed exactly
// in binary16 and one rounding in the multiply; or, for an FP8 cache (format
// code 0), the E5M2 bytes decoded exactly as fp8_to_fp16 does.
//
// Split-K flash decoding.  Kernel 1 (attn_partial_kernel) is a persistent
// grid (one wave of CTAs of four warps).  Every (sequence, chunk, kv head)
// that holds data is a work item (128-position chunks for 4- and 6-bit codes,
// 256 for 8-bit codes and E5M2); warps take them from a compact enumeration,
// in contiguous ranges or round-robin depending on the format (AttnWalk).
// (When there are few items, the four warps of a CTA take a quarter of each
// item instead and merge the quarters in shared memory.)  A warp streams its
// items through two shared-memory buffers of 16 or 32 positions (cp.async
// copies of K and V codes, scales and, with an item's first sub-chunk, the
// group's query rows), filling one while it computes on the other, 16
// positions at a time:
//   * S^T = K Q^T on mma.sync m16n8k16 with the cache rows as the A operand
//     (16 positions) and the query heads as the N columns: each lane
//     dequantizes one contiguous span of D/4 elements of each of its two
//     positions (the head_dim order inside the MMA is permuted so that a
//     lane's elements over all k-steps are that span); the query fragments
//     use the same permutation;
//   * online softmax (base 2) per query head with lazy rescaling: the
//     reference maximum only moves when a score exceeds it by more than
//     kAttnRescaleLog2, so the accumulators are rarely touched and every
//     weight stays below 2^kAttnRescaleLog2;
//   * O^T += V^T P^T: the weights, split into a binary16 high part and a
//     binary16 residual (about 22 significant bits), are transposed into the
//     B fragment of P^T with movmatrix; for groups of up to four query heads
//     one MMA carries both parts (columns 0-3 and 4-7); V^T A fragments pair
//     two positions at one head_dim index, built by interleaving the bytes of
//     two rows before the codes are unpacked.
// Code unpacking avoids per-code shifts: `(w & 0x000F000F) | 0x64006400` is
// the binary16 pair (1024 + c0, 1024 + c4) of a Q4 word, and the high-nibble
// pair is 16x that, brought back exactly with an FMA by 1/16.
// When a softmax state ends the warp writes its (max, sum, accumulator) per
// query head to the workspace entry of the state's first chunk.  Kernel 2
// (attn_combine_kernel) merges the entries of each (sequence, head) and writes
// binary16 outputs.
#pragma once

#include <type_traits>

#include "codec.cuh"
#include "tiles.cuh"

namespace kvq {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = 32 * kAttnWarps;
constexpr int kAttnMaxGroup = 8;        // query heads per kv head (one MMA N block of P^T)
constexpr float kAttnRescaleLog2 = 8.0f;  // lazy-rescale threshold (log2 units)

struct AttnParams {
  const __half* q;  // [batch, n_heads, D]
  const uint8_t* k_codes;
  const __half* k_scales;
  const uint8_t* v_codes;
  const __half* v_scales;
  __half* out;  // [batch, n_heads, D]
  float* ws;    // [batch, n_heads, max_chunks, D + 2]: m (log2 domain), l, acc[D]
  const int32_t* seqlens;
  const int32_t* block_table;
  int dim0, dim1, kv_heads, batch, n_heads, group, page_size, bt_stride, max_chunks;
  int page_shift;  // log2(page_size) when it is a power of two, else -1
  int chunk;  // positions per work item (AttnTile<B, D>::kChunk)
  float scale_log2;  // softmax_scale * log2(e)
};

__device__ __forceinline__ void mma_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ __half2 as_h2(uint32_t x) { return *reinterpret_cast<const __half2*>(&x); }
__device__ __forceinline__ uint32_t as_u32(__half2 x) { return *reinterpret_cast<const uint32_t*>(&x); }

// (code - z) of a binary16 pair holding 1024 + code (exact).
template <int Z>
__device__ __forceinline__ uint32_t minus_z(uint32_t h) {
  const __half2 off = __halves2half2(__ushort_as_half(static_cast<unsigned short>(0x6400 + Z)),
                                     __ushort_as_half(static_cast<unsigned short>(0x6400 + Z)));
  return as_u32(__hsub2_rn(as_h2(h), off));
}

// (code - z) of a binary16 pair holding 1024 + 16 * code: h / 16 - (64 + z),
// exact (h / 16 is exact, the difference is a small integer).
template <int Z>
__device__ __forceinline__ uint32_t minus_z_x16(uint32_t h) {
  static_assert(Z == 8, "the 16x form is used for 4-bit codes only");
  // 1/16 = 0x2C00, -(64 + 8) = -72 = 0xD480 in binary16
  const __half2 sixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
  const __half2 off = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));
  return as_u32(__hfma2(as_h2(h), sixteenth, off));
}

// 2^x for the softmax weights: the hardware approximation (relative error
// about 2^-22 over the range used; results below 2^-126 flush to zero, which
// only drops weights that cannot matter next to the reference weight 1).
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t scale_pair(uint32_t d, __half2 s2) { return as_u32(__hmul2_rn(as_h2(d), s2)); }

// ---------------------------------------------------------------------------
// Unpacking of one row's span (same-row pairs) and of two rows' spans
// (cross-row pairs), per code width.  Results are (code - z) in binary16,
// exact; the caller multiplies by the scale.
//
// Same-row pair order (`row_pair_elem`): pair r of a span holds elements
// (e0, e1) = row_pair_elem(r, 0 / 1).  Cross-row order (`xrow_elem`): pair r
// holds element xrow_elem(r) of row 0 (low half) and of row 1 (high half).
// ---------------------------------------------------------------------------

template <int B>
struct AttnCodec;

template <>
struct AttnCodec<4> {
  static constexpr int kZ = 8;
  // pairs per 32-bit word: (0,4), (1,5), (2,6), (3,7)
  __host__ __device__ static constexpr int row_pair_elem(int r, int e) { return 8 * (r >> 2) + (r & 3) + 4 * e; }
  __host__ __device__ static constexpr int xrow_elem(int r) { return r; }
  template <int NW>
  __device__ static void row_pairs(const uint32_t (&w)[NW], uint32_t (&out)[4 * NW]) {
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const uint32_t x = w[i], y = w[i] >> 8;
      out[4 * i + 0] = minus_z<kZ>((x & 0x000F000Fu) | 0x64006400u);
      out[4 * i + 1] = minus_z_x16<kZ>((x & 0x00F000F0u) | 0x64006400u);
      out[4 * i + 2] = minus_z<kZ>((y & 0x000F000Fu) | 0x64006400u);
      out[4 * i + 3] = minus_z_x16<kZ>((y & 0x00F000F0u) | 0x64006400u);
    }
  }
  // rows r0, r1 (NW words each) -> 8 * NW cross-row pairs, element order 0..8NW-1
  template <int NW>
  __device__ static void xrow_pairs(const uint32_t (&w0)[NW], const uint32_t (&w1)[NW], uint32_t (&out)[8 * NW]) {
#pragma unroll
    for (int i = 0; i < NW; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // bytes 2h, 2h+1 of each row: elements 8i + 4h .. 8i + 4h + 3
        const uint32_t x = __byte_perm(w0[i], w1[i], h ? 0x7632 : 0x5410);
        const uint32_t y = x >> 8;
        out[8 * i + 4 * h + 0] = minus_z<kZ>((x & 0x000F000Fu) | 0x64006400u);
        out[8 * i + 4 * h + 1] = minus_z_x16<kZ>((x & 0x00F000F0u) | 0x64006400u);
        out[8 * i + 4 * h + 2] = minus_z<kZ>((y & 0x000F000Fu) | 0x64006400u);
        out[8 * i + 4 * h + 3] = minus_z_x16<kZ>((y & 0x00F000F0u) | 0x64006400u);
      }
    }
  }
};

// FP8 (E5M2; format code 0): the byte is the high byte of the binary16 value,
// so a byte permute against zero decodes two values exactly; no scale.
template <>
struct AttnCodec<0> {
  // pairs per 32-bit word: (0,1), (2,3)
  __host__ __device__ static constexpr int row_pair_elem(int r, int e) { return 2 * r + e; }
  __host__ __device__ static constexpr int xrow_elem(int r) { return r; }
  template <int NW>
  __device__ static void row_pairs(const uint32_t (&w)[NW], uint32_t (&out)[2 * NW]) {
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      out[2 * i + 0] = __byte_perm(w[i], 0u, 0x1404);  // [0, b0, 0, b1]
      out[2 * i + 1] = __byte_perm(w[i], 0u, 0x3424);  // [0, b2, 0, b3]
    }
  }
  // rows r0, r1 (NW words each) -> 4 * NW cross-row pairs, element order 0..4NW-1
  template <int NW>
  __device__ static void xrow_pairs(const uint32_t (&w0)[NW], const uint32_t (&w1)[NW], uint32_t (&out)[4 * NW]) {
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const uint32_t a = w0[i] << 8, b = w1[i] << 8;    // [0, b0, b1, b2] of each row
      const uint32_t c = w0[i] >> 16, d = w1[i] >> 16;  // [b2, b3, 0, 0] of each row
      out[4 * i + 0] = __byte_perm(a, b, 0x5410);
      out[4 * i + 1] = __byte_perm(a, b, 0x6420);
      out[4 * i + 2] = __byte_perm(a, b, 0x7430);
      out[4 * i + 3] = __byte_perm(c, d, 0x5612);
    }
  }
};

template <>
struct AttnCodec<8> {
  static constexpr int kZ = 128;
  // pairs per 32-bit word: (0,1), (2,3)
  __host__ __device__ static constexpr int row_pair_elem(int r, int e) { return 2 * r + e; }
  __host__ __device__ static constexpr int xrow_elem(int r) { return r; }
  template <int NW>
  __device__ static void row_pairs(const uint32_t (&w)[NW], uint32_t (&out)[2 * NW]) {
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      out[2 * i + 0] = minus_z<kZ>(__byte_perm(w[i], 0x64646464u, 0x5140));
      out[2 * i + 1] = minus_z<kZ>(__byte_perm(w[i], 0x64646464u, 0x7362));
    }
  }
  template <int NW>
  __device__ static void xrow_pairs(const uint32_t (&w0)[NW], const uint32_t (&w1)[NW], uint32_t (&out)[4 * NW]) {
#pragma unroll
    for (int i = 0; i < NW; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // t = [r0.c(2h), r0.c(2h+1), r1.c(2h), r1.c(2h+1)]
        const uint32_t t = __byte_perm(w0[i], w1[i], h ? 0x7632 : 0x5410);
        out[4 * i + 2 * h + 0] = minus_z<kZ>(__byte_perm(t, 0x64646464u, 0x4240));
        out[4 * i + 2 * h + 1] = minus_z<kZ>(__byte_perm(t, 0x64646464u, 0x4341));
      }
    }
  }
};

// Q6: a 16-code group is 12 bytes (three little-endian words, code k at bits
// [6k, 6k + 6)).  Eight codes are six bytes B0..B5; pairs (q, q + 4) sit at
// the same bit offsets of (B0..B2) and (B3..B5), so one byte permute puts
// them 16 bits apart: (0,4) = B0 | B3, (1,5) = (B0 B1 | B3 B4) >> 6,
// (2,6) = (B1 B2 | B4 B5) >> 4, (3,7) = (B2 | B5) >> 2.
template <>
struct AttnCodec<6> {
  static constexpr int kZ = 32;
  __host__ __device__ static constexpr int row_pair_elem(int r, int e) { return 8 * (r >> 2) + (r & 3) + 4 * e; }
  __host__ __device__ static constexpr int xrow_elem(int r) { return 8 * (r >> 3) + ((r >> 1) & 3) + 4 * (r & 1); }
  // 8 codes from bytes B0..B5 = bytes o..o+5 of the pair (a, b) (o = 0 or 2):
  // four (1024 + code) pairs (q, q + 4)
  __device__ static void raw8_at(uint32_t a, uint32_t b, uint32_t o, uint32_t (&r)[4]) {
    const uint32_t add = o * 0x1111u;  // every selector nibble moves up by o bytes
    const uint32_t p0 = __byte_perm(a, b, 0x3300u + add);  // B0, B0, B3, B3
    const uint32_t p1 = __byte_perm(a, b, 0x4310u + add);  // B0, B1, B3, B4
    const uint32_t p2 = __byte_perm(a, b, 0x5421u + add);  // B1, B2, B4, B5
    const uint32_t p3 = __byte_perm(a, b, 0x5522u + add);  // B2, B2, B5, B5
    r[0] = (p0 & 0x003F003Fu) | 0x64006400u;
    r[1] = ((p1 >> 6) & 0x003F003Fu) | 0x64006400u;
    r[2] = ((p2 >> 4) & 0x003F003Fu) | 0x64006400u;
    r[3] = ((p3 >> 2) & 0x003F003Fu) | 0x64006400u;
  }
  // NG groups (3 words each) -> 8 * NG same-row pairs
  template <int NG>
  __device__ static void row_pairs_g(const uint32_t (&w)[3 * NG], uint32_t (&out)[8 * NG]) {
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      uint32_t r0[4], r1[4];
      raw8_at(w[3 * g], w[3 * g + 1], 0, r0);
      raw8_at(w[3 * g + 1], w[3 * g + 2], 2, r1);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        out[8 * g + q] = minus_z<kZ>(r0[q]);
        out[8 * g + 4 + q] = minus_z<kZ>(r1[q]);
      }
    }
  }
  // two rows, NG groups each -> 16 * NG cross-row pairs in xrow_elem order
  template <int NG>
  __device__ static void xrow_pairs_g(const uint32_t (&w0)[3 * NG], const uint32_t (&w1)[3 * NG],
                                      uint32_t (&out)[16 * NG]) {
#pragma unroll
    for (int g = 0; g < NG; ++g) {
#pragma unroll
      for (int hg = 0; hg < 2; ++hg) {
        uint32_t a[4], b[4];
        raw8_at(w0[3 * g + hg], w0[3 * g + hg + 1], 2 * hg, a);
        raw8_at(w1[3 * g + hg], w1[3 * g + hg + 1], 2 * hg, b);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          // element q of both rows, then element q + 4 of both rows
          out[16 * g + 8 * hg + 2 * q] = minus_z<kZ>(__byte_perm(a[q], b[q], 0x5410));
          out[16 * g + 8 * hg + 2 * q + 1] = minus_z<kZ>(__byte_perm(a[q], b[q], 0x7632));
        }
      }
    }
  }
};

// Per-warp shared-memory staging.  A work item is one (sequence, kv head,
// kChunk-position chunk): 128 positions for 4- and 6-bit codes, whose walk
// carries one softmax state over pairs of chunks, and 256 for 8-bit codes and
// E5M2 (512 measured 25% slower from load imbalance).  A warp streams it
// through two buffers of kSub positions each (K codes, V codes, K scales, V
// scales), filling one while it computes on the other.  Row strides are padded
// where that removes bank conflicts of the fragment reads (K: one span per
// lane of two rows eight apart; V: four rows per lane, byte-interleaved in
// pairs).
template <int B, int D>
struct AttnTile {
  static constexpr int kBits = B == 0 ? 8 : B;  // bits per cached element (format 0: E5M2 bytes)
  static constexpr int kRowBytes = D * kBits / 8;
  static constexpr int kStrideK = kRowBytes + (kRowBytes % 128 == 0 ? 16 : 0);
  static constexpr int kStrideV = kRowBytes + ((B == 6 && D == 64) ? 0 : 16);
  static constexpr int kScales = B == 0 ? 0 : D / 32;  // binary16 scales per row
  // positions per work item / workspace entry: 128 for the 4- and 6-bit codes
  // (their blocked walk), 256 for 8-bit codes and E5M2 (their round-robin walk)
  static constexpr int kChunk = (B == 4 || B == 6) ? 128 : 256;
  static constexpr int kSub = kRowBytes <= 96 ? 32 : 16;   // positions per staged buffer (measured)
  static constexpr int kBufK = kSub * kStrideK;
  static constexpr int kBufV = kSub * kStrideV;
  static constexpr int kBufS = kSub * kScales * 2;
  static constexpr int kBufBytes = (kBufK + kBufV + 2 * kBufS + 15) / 16 * 16;
  static constexpr int kQBytes = kAttnMaxGroup * D * 2;  // the item's query rows (copied with its first sub-chunk)
  static constexpr int kWarpBytes = 2 * kBufBytes + kQBytes;
  // sequence lengths staged per CTA, with the running count of work items
  // (larger batches read global memory and walk every item slot)
  static constexpr int kSeqlenSlots = 256;
  static constexpr int kSmemBytes = kAttnWarps * kWarpBytes + 2 * kSeqlenSlots * 4 + 16;
  static constexpr int KN = D / 4;   // K elements per lane per position (one contiguous span)
  static constexpr int VN = D / 8;   // V elements per lane per row (one contiguous span)
  static constexpr int KS = D / 16;  // k-steps of Q K^T = m-tiles of V^T P^T
  static constexpr int kKSpanBytes = KN * kBits / 8;
  static constexpr int kVSpanBytes = VN * kBits / 8;
};
constexpr int kAttnMinChunk = 128;  // sizes the workspace: the smallest kChunk of any (B, D)

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n"
               ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_small(void* dst, const void* src) {
  static_assert(N == 4 || N == 8 || N == 16, "cp.async sizes");
  asm volatile("cp.async.ca.shared.global [%0], [%1], %2;\n"
               ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "n"(N)
               : "memory");
}

// NB bytes (a multiple of 4) from shared memory at p, aligned to the widest
// access NB and the offset allow, as 32-bit words.
template <int NB>
__device__ __forceinline__ void lds_words(const uint8_t* p, uint32_t (&w)[NB / 4]) {
  if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int v = 0; v < NB / 16; ++v) {
      const uint4 x = reinterpret_cast<const uint4*>(p)[v];
      w[4 * v] = x.x, w[4 * v + 1] = x.y, w[4 * v + 2] = x.z, w[4 * v + 3] = x.w;
    }
  } else if constexpr (NB % 8 == 0) {
#pragma unroll
    for (int v = 0; v < NB / 8; ++v) {
      const uint2 x = reinterpret_cast<const uint2*>(p)[v];
      w[2 * v] = x.x, w[2 * v + 1] = x.y;
    }
  } else {
#pragma unroll
    for (int v = 0; v < NB / 4; ++v) w[v] = reinterpret_cast<const uint32_t*>(p)[v];
  }
}

// The K span of one lane (KN elements starting at element KN * j of a staged
// row) as (code - z) pairs times the scale: KN / 2 half2 registers in
// row_pair_elem order.
template <int B, int D>
__device__ __forceinline__ void k_span(const uint8_t* row, const __half* srow, int j, uint32_t (&out)[D / 8]) {
  using T = AttnTile<B, D>;
  constexpr int KN = T::KN, NB = T::kKSpanBytes;
  uint32_t w[NB / 4];
  lds_words<NB>(row + j * NB, w);
  if constexpr (B == 6) {
    AttnCodec<6>::row_pairs_g<NB / 12>(w, out);
  } else {
    AttnCodec<B>::template row_pairs<NB / 4>(w, out);
  }
  // scales: one 32-element block per 16 registers (KN <= 32: one block); E5M2 has none
  constexpr int kRegsPerBlock = 16;
#pragma unroll
  for (int b = 0; b < (T::kScales ? (KN + 31) / 32 : 0); ++b) {
    const __half s = srow[(KN * j) / 32 + b];
    const __half2 s2 = __halves2half2(s, s);
#pragma unroll
    for (int r = b * kRegsPerBlock; r < (b + 1) * kRegsPerBlock && r < KN / 2; ++r) out[r] = scale_pair(out[r], s2);
  }
}

// The V spans of one lane for a pair of rows (VN elements starting at element
// VN * g): VN cross-row pairs (row r0 low half, r1 high half) times the two
// rows' scales, in xrow_elem order.
template <int B, int D>
__device__ __forceinline__ void v_span_pair(const uint8_t* r0, const uint8_t* r1, __half s0, __half s1, int g,
                                            uint32_t (&out)[D / 8]) {
  using T = AttnTile<B, D>;
  constexpr int VN = T::VN, NB = T::kVSpanBytes;
  if constexpr (B == 6 && VN == 8) {
    // 6 bytes at byte 6g: the aligned 8 bytes around them, bytes o..o+5 (o = 0 or 2)
    const int base = (6 * g) & ~3;
    const uint32_t o = (6 * g) & 3;
    const uint32_t* const w0 = reinterpret_cast<const uint32_t*>(r0 + base);
    const uint32_t* const w1 = reinterpret_cast<const uint32_t*>(r1 + base);
    const uint32_t a0 = w0[0], b0 = w0[1];
    const uint32_t a1 = w1[0], b1 = w1[1];
    uint32_t x[4], y[4];
    AttnCodec<6>::raw8_at(a0, b0, o, x);
    AttnCodec<6>::raw8_at(a1, b1, o, y);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      out[2 * q] = minus_z<32>(__byte_perm(x[q], y[q], 0x5410));
      out[2 * q + 1] = minus_z<32>(__byte_perm(x[q], y[q], 0x7632));
    }
  } else {
    uint32_t w0[NB / 4], w1[NB / 4];
    lds_words<NB>(r0 + g * NB, w0);
    lds_words<NB>(r1 + g * NB, w1);
    if constexpr (B == 6) {
      AttnCodec<6>::xrow_pairs_g<NB / 12>(w0, w1, out);
    } else {
      AttnCodec<B>::template xrow_pairs<NB / 4>(w0, w1, out);
    }
  }
  if constexpr (T::kScales > 0) {
    const __half2 s2 = __halves2half2(s0, s1);
#pragma unroll
    for (int r = 0; r < VN; ++r) out[r] = scale_pair(out[r], s2);
  }
}


// One sub-chunk of one work item, as a warp walks its items.
template <class I>
struct AttnCursor {
  I item;               // work item index, or -1 past the end
  int seq, chunk, kvh;  // what the item is
  int nch;              // chunks of the sequence (blocked walk)
  int sub;              // sub-chunk within the item
  int n;                // positions of this sub-chunk (<= kSub)
  bool last;            // last sub-chunk of the item
  bool fresh;           // the item starts a new softmax state (otherwise it continues the previous one)
};

// Work items in walk order.  An item is one (sequence, kChunk-position
// chunk, kv head); its workspace entry is (sequence, query head, chunk).
// kCompact: only items that hold data are enumerated.  The CTA stages the
// batch in shared memory: kSeqlenSlots sequence lengths, then kSeqlenSlots
// running item counts (entry i counts the items of sequences 0..i), then the
// total.  The launch guarantees that the batch fits the slots and that every
// count fits an int.  Without kSplit, one of two walks (chosen per format, by
// measurement: streams of launches over the paged pool):
//   Blocked (4- and 6-bit codes, 128-position chunks): items are numbered (kv
//   head, sequence, chunk), chunk fastest, so the running counts count the
//   chunks of one kv head.  Warp w of W takes the contiguous range
//   [w U / W, (w + 1) U / W) of the U items, so the warps' shares differ by at
//   most one small item.  When W is a multiple of the kv heads, the warps of
//   every kv head get the same ranges of (sequence, chunk), so the kv heads of
//   a position are read at about the same time.  Within its range a warp
//   carries one softmax state over the two chunks of each aligned pair (chunks
//   2i, 2i + 1 of one sequence and kv head) and writes it to the entry of the
//   first chunk it took; the entry of the second gets a -inf maximum, which the
//   combine skips.  A state never spans more than 256 positions.  These codes
//   cost the most instructions per byte: the balance pays.
//   Round-robin (8-bit codes and E5M2, 256-position chunks): items are
//   numbered (sequence, chunk, kv head), kv head fastest, and warp w takes
//   items w, w + W, ...: the warps of a round read neighbouring items, so the
//   kv heads of a position, which share DRAM pages, are read together.  These
//   formats come closest to the DRAM limit, where that locality pays.
//   kSplit (for batches too small to give every warp an item): items as in
//   the round-robin walk but always 256 positions long (for 4- and 6-bit codes
//   a pair of chunks, whose second entry gets a -inf maximum); a CTA takes
//   items in turn and each of its four warps
//   a quarter of the item's positions, every warp walking the same kSplitSubs
//   sub-chunks per item (empty ones where its quarter runs past the sequence),
//   so that the CTA can merge the four partial results at the end of each item.
// Otherwise: every (sequence, chunk, kv head) slot up to the cache's capacity
// is visited in turn (kv head fastest) and empty ones are skipped (lengths
// staged when the batch fits); every item has its own state and entry.
template <int B, int D, bool kCompact, bool kSplit = false>
struct AttnWalk {
  static_assert(kCompact || !kSplit, "the split walk enumerates compactly");
  using T = AttnTile<B, D>;
  using Item = typename std::conditional<kCompact, int, long long>::type;
  using Cursor = AttnCursor<Item>;
  static constexpr bool kBlocked = kCompact && !kSplit && (B == 4 || B == 6);
  // chunks per kSplit item: 256 positions (two 128-position chunks for 4- and
  // 6-bit codes, whose second chunk's entry gets a -inf maximum)
  static constexpr int kItemChunks = kSplit ? 256 / T::kChunk : 1;
  static constexpr int kQuarter = kItemChunks * T::kChunk / kAttnWarps;  // positions per warp and item (kSplit)
  static constexpr int kSplitSubs = kQuarter / T::kSub;                   // sub-chunks per warp and item (kSplit)
  static_assert(kSplitSubs >= 1 && kQuarter % T::kSub == 0, "a quarter item is whole sub-chunks");
  const AttnParams& a;
  bool staged;   // the batch's lengths are in shared memory
  Item end = 0;  // kBlocked: one past this warp's last item

  // first position of this warp's part of an item
  __device__ static int offset() { return kSplit ? kQuarter * static_cast<int>(threadIdx.x >> 5) : 0; }
  // positions and last-sub-chunk flag of sub-chunk `sub` of an item of sequence length L
  __device__ void set_sub(Cursor& c, int L, int sub) const {
    c.sub = sub;
    if constexpr (kSplit) {
      const int rest = L - c.chunk * T::kChunk - offset() - sub * T::kSub;
      c.n = max(0, min(rest, T::kSub));
      c.last = sub == kSplitSubs - 1;
    } else {
      const int rest = min(L - c.chunk * T::kChunk, T::kChunk) - sub * T::kSub;
      c.n = min(rest, T::kSub);
      c.last = rest <= T::kSub;
    }
  }

  // the staged block, after the warps' buffers in dynamic shared memory
  __device__ static int* block() {
    extern __shared__ __align__(16) uint8_t smem[];
    return reinterpret_cast<int*>(smem + kAttnWarps * T::kWarpBytes);
  }
  // walkers in the grid: warps, or CTAs with kSplit
  __device__ static Item stride() { return static_cast<Item>(gridDim.x) * (kSplit ? 1 : kAttnWarps); }

  __device__ long long max_len() const {
    return a.page_size == 0 ? static_cast<long long>(a.dim1) : static_cast<long long>(a.max_chunks) * T::kChunk;
  }
  // sequence length, clamped to what the cache (or the launched chunks) can hold
  __device__ int length(int seq) const {
    long long L = staged ? block()[seq] : a.seqlens[seq];
    if (L < 0) L = 0;
    const long long m = max_len();
    return static_cast<int>(L > m ? m : L);
  }
  // first sub-chunk of item `item` (kCompact), or of the first non-empty item slot at or after it
  __device__ Cursor seek(Item item) const {
    Cursor c;
    c.fresh = true;
    if constexpr (kCompact) {
      const int* const s_items = block() + T::kSeqlenSlots;
      if (item >= (kBlocked ? end : s_items[T::kSeqlenSlots])) {
        c.item = -1;
        return c;
      }
      int kvh = 0;
      Item local = item;  // the item among those of its kv head (kBlocked) or of the batch
      if constexpr (kBlocked) {
        const unsigned per_head = static_cast<unsigned>(s_items[T::kSeqlenSlots]);
        kvh = static_cast<int>(static_cast<unsigned>(item) / per_head);
        local = static_cast<Item>(static_cast<unsigned>(item) - static_cast<unsigned>(kvh) * per_head);
      }
      int lo = 0, hi = a.batch - 1;  // the first sequence whose running count exceeds the item
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s_items[mid] > local) hi = mid;
        else lo = mid + 1;
      }
      const int prev = lo ? s_items[lo - 1] : 0;
      const unsigned r = static_cast<unsigned>(local - prev);
      c.seq = lo;
      c.item = item;
      if constexpr (kBlocked) {
        c.kvh = kvh;
        c.chunk = static_cast<int>(r);
        c.nch = s_items[lo] - prev;
      } else {
        const unsigned item_chunk = r / static_cast<unsigned>(a.kv_heads);
        c.chunk = static_cast<int>(item_chunk) * kItemChunks;
        c.kvh = static_cast<int>(r - item_chunk * static_cast<unsigned>(a.kv_heads));
      }
      set_sub(c, length(lo), 0);
      return c;
    } else {
      const long long n_items = static_cast<long long>(a.batch) * a.max_chunks * a.kv_heads;
      for (; item < n_items; item += stride()) {
        if (n_items < (1LL << 31)) {  // 32-bit index arithmetic suffices
          const unsigned it = static_cast<unsigned>(item), t = it / static_cast<unsigned>(a.kv_heads);
          c.kvh = static_cast<int>(it - t * static_cast<unsigned>(a.kv_heads));
          c.seq = static_cast<int>(t / static_cast<unsigned>(a.max_chunks));
          c.chunk = static_cast<int>(t - static_cast<unsigned>(c.seq) * static_cast<unsigned>(a.max_chunks));
        } else {
          const long long t = item / a.kv_heads;
          c.kvh = static_cast<int>(item - t * a.kv_heads);
          c.seq = static_cast<int>(t / a.max_chunks);
          c.chunk = static_cast<int>(t - static_cast<long long>(c.seq) * a.max_chunks);
        }
        const int L = length(c.seq);
        // 64-bit: a slot's chunk can reach max_chunks (up to 2^31 - 1), far past any length
        const long long p0 = static_cast<long long>(c.chunk) * T::kChunk;
        if (p0 < L) {
          c.item = item;
          set_sub(c, L, 0);
          return c;
        }
      }
      c.item = -1;
      return c;
    }
  }
  __device__ Cursor next(const Cursor& c) const {
    if (!c.last) {
      Cursor d = c;
      set_sub(d, length(c.seq), c.sub + 1);
      return d;
    }
    if constexpr (kBlocked) {
      // the next item of this warp's range: the sequence's next chunk, or a seek
      if (c.item + 1 >= end) {
        Cursor d;
        d.item = -1;
        return d;
      }
      if (c.chunk + 1 < c.nch) {
        Cursor d = c;
        d.item = c.item + 1;
        d.chunk = c.chunk + 1;
        d.fresh = (d.chunk & 1) == 0;
        set_sub(d, length(c.seq), 0);
        return d;
      }
      return seek(c.item + 1);
    } else {
      return seek(c.item + stride());
    }
  }
};

// Scales of one sub-chunk (lane i: position i; rows without data get zero
// scales, which dequantize whatever codes the buffer holds to zero), the E5M2
// value rows without data zeroed (a weight of 0 times a stale Inf or NaN byte
// would still poison the sum; key rows are masked by their -inf score), and,
// for the first sub-chunk of an item that starts a softmax state, its query rows.
template <int B, int D, class Cursor>
__device__ __forceinline__ void attn_issue_rest(const AttnParams& a, const Cursor& c, long long hr, uint8_t* buf,
                                                uint8_t* sq, int lane) {
  using T = AttnTile<B, D>;
  constexpr int SC = T::kSub, P = T::kRowBytes / 16;
  uint8_t* const sv = buf + T::kBufK;
  __half* const sks = reinterpret_cast<__half*>(buf + T::kBufK + T::kBufV);
  __half* const svs = sks + SC * T::kScales;
  if constexpr (T::kScales > 0) {
    if (lane < SC) {
      if (hr >= 0) {
        cp_async_small<T::kScales * 2>(sks + lane * T::kScales, a.k_scales + hr * T::kScales);
        cp_async_small<T::kScales * 2>(svs + lane * T::kScales, a.v_scales + hr * T::kScales);
      } else {
#pragma unroll
        for (int e = 0; e < T::kScales; ++e)
          sks[lane * T::kScales + e] = svs[lane * T::kScales + e] = __ushort_as_half(0);
      }
    }
  } else {
    if (lane < SC && hr < 0) {
#pragma unroll
      for (int part = 0; part < P; ++part)
        *reinterpret_cast<uint4*>(sv + lane * T::kStrideV + part * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (c.sub == 0 && c.fresh) {
    const __half* q = a.q + (static_cast<long long>(c.seq) * a.n_heads + static_cast<long long>(c.kvh) * a.group) * D;
    for (int t = lane; t < a.group * D / 8; t += 32) cp_async16(sq + t * 16, q + t * 8);
  }
}

// Issue the copies of one sub-chunk into a warp buffer (and, for the first
// sub-chunk of an item, its query rows into the warp's query area); returns
// the bit mask of its positions that hold data (bit i: position i).
// A sub-chunk starts at a multiple of kSub positions.  When the cache is
// contiguous or its page size is a multiple of kSub, the sub-chunk's rows are
// consecutive cache rows: one block-table lookup for the warp, and every lane
// copies fixed 16-byte parts of rows R apart.  Otherwise every lane resolves
// its own position's row.
template <int B, int D, class Cursor>
__device__ __forceinline__ uint32_t attn_issue(const AttnParams& a, const Cursor& c, int offset, uint8_t* buf,
                                               uint8_t* sq, int lane) {
  using T = AttnTile<B, D>;
  constexpr int SC = T::kSub, P = T::kRowBytes / 16;
  uint8_t* const sk = buf;
  uint8_t* const sv = buf + T::kBufK;
  const int p0 = c.chunk * T::kChunk + offset + c.sub * SC;  // first position of the sub-chunk
  if (a.page_size == 0 || a.page_size % SC == 0) {
    long long row0;
    int n = c.n;
    if (a.page_size == 0) {
      row0 = static_cast<long long>(c.seq) * a.dim1 + p0;
    } else {
      const int lp = a.page_shift >= 0 ? p0 >> a.page_shift : p0 / a.page_size;
      const int page = lp < a.bt_stride ? a.block_table[static_cast<long long>(c.seq) * a.bt_stride + lp] : -1;
      if (page < 0 || page >= a.dim0) {
        if (n > 0 && lane == 0) record_error(KVQ_DEV_BAD_PAGE);
        n = 0;
      }
      row0 = static_cast<long long>(page) * a.page_size + (p0 - lp * a.page_size);
    }
    const long long hr0 = row0 * a.kv_heads + c.kvh;
    // lane = (row rl of each group of R rows, 16-byte part pt); R * P <= 32 lanes busy
    constexpr int R = 32 / P, NPASS = (SC + R - 1) / R;
    const int rl = lane / P, pt = lane - rl * P;
    if (lane < R * P && rl < n) {
      const long long rstride = static_cast<long long>(a.kv_heads) * T::kRowBytes;
      const long long off = (hr0 + static_cast<long long>(rl) * a.kv_heads) * T::kRowBytes + pt * 16;
      const uint8_t* ks = a.k_codes + off;
      const uint8_t* vs = a.v_codes + off;
#pragma unroll
      for (int k = 0; k < NPASS; ++k) {
        const int r = rl + R * k;
        if (r < n) {
          cp_async16(sk + r * T::kStrideK + pt * 16, ks);
          cp_async16(sv + r * T::kStrideV + pt * 16, vs);
        }
        ks += R * rstride;
        vs += R * rstride;
      }
    }
    attn_issue_rest<B, D>(a, c, lane < n ? hr0 + static_cast<long long>(lane) * a.kv_heads : -1, buf, sq, lane);
    return n >= 32 ? 0xFFFFFFFFu : ((1u << n) - 1u);
  }
  // cache row of this lane's position (lanes < n): -1 bad paging metadata, -2 past the window
  long long hr = -2;
  if (lane < c.n) {
    const int p = p0 + lane;
    const int lp = p / a.page_size;
    const int page = lp < a.bt_stride ? a.block_table[static_cast<long long>(c.seq) * a.bt_stride + lp] : -1;
    const long long row =
        (page < 0 || page >= a.dim0) ? -1 : static_cast<long long>(page) * a.page_size + (p - lp * a.page_size);
    if (row < 0) record_error(KVQ_DEV_BAD_PAGE);
    hr = row < 0 ? -1 : row * a.kv_heads + c.kvh;
  }
  const uint32_t mask = __ballot_sync(0xFFFFFFFFu, hr >= 0);
  // codes: task t = (row t / P, 16-byte part t % P), 32 tasks per pass
#pragma unroll
  for (int t0 = 0; t0 < SC * P; t0 += 32) {
    const int t = t0 + lane, r = t / P, part = t - r * P;
    const long long h = __shfl_sync(0xFFFFFFFFu, hr, r);
    if (h >= 0) {
      const long long src = h * T::kRowBytes + part * 16;
      cp_async16(sk + r * T::kStrideK + part * 16, a.k_codes + src);
      cp_async16(sv + r * T::kStrideV + part * 16, a.v_codes + src);
    }
  }
  attn_issue_rest<B, D>(a, c, hr, buf, sq, lane);
  return mask;
}

// Transpose of an 8 x 8 binary16 block held across the warp: lane 4r + c holds
// elements (r, 2c) and (r, 2c + 1) of the block before and of its transpose after.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// kG4 (group <= 4): the query operand repeats the group's heads in columns 4..7,
// so the lanes holding columns 4..7 compute the same weights as those holding
// 0..3 and contribute the residual parts: one V^T P^T product per step carries
// both parts (columns 0..3 high, 4..7 residual), summed when the item ends.
template <int B, int D, bool kCompact, bool kSplit, bool kG4>
__global__ void __launch_bounds__(kAttnThreads, D > 128 ? 2 : 4)
    attn_partial_kernel(const __grid_constant__ AttnParams a) {
  using T = AttnTile<B, D>;
  using Codec = AttnCodec<B>;
  constexpr int KS = T::KS;  // k-steps of K Q^T, m-tiles of V^T P^T
  constexpr int KR = D / 8;  // registers of one K span / one V span pair
  constexpr int SC = T::kSub;

  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, j = lane & 3;
  uint8_t* const wbuf = smem + warp * T::kWarpBytes;
  int* const s_len = reinterpret_cast<int*>(smem + kAttnWarps * T::kWarpBytes);
  using Walk = AttnWalk<B, D, kCompact, kSplit>;
  static_assert(!kSplit || kAttnMaxGroup * (D + 2) * 4 <= T::kBufBytes, "a warp's partial result fits its buffer");

  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const bool staged = kCompact || a.batch <= T::kSeqlenSlots;
  if (staged)
    for (int i = threadIdx.x; i < a.batch; i += kAttnThreads) s_len[i] = a.seqlens[i];
  __syncthreads();
  if (kCompact && warp == 0) {
    // running item counts over the batch (a warp-wide inclusive scan per 32
    // sequences; the launch guarantees that the total fits an int)
    int* const s_items = s_len + T::kSeqlenSlots;
    const Walk w0{a, true};
    int run = 0;
    for (int base = 0; base < a.batch; base += 32) {
      const int i = base + lane;
      constexpr int kItemLen = Walk::kItemChunks * T::kChunk;
      int n = i < a.batch ? (w0.length(i) + kItemLen - 1) / kItemLen * (Walk::kBlocked ? 1 : a.kv_heads) : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, n, o);
        if (lane >= o) n += t;
      }
      n += run;
      if (i < a.batch) s_items[i] = n;
      run = __shfl_sync(0xFFFFFFFFu, n, 31);
    }
    if (lane == 0) s_items[T::kSeqlenSlots] = run;
  }
  __syncthreads();  // the last CTA-wide barrier: from here on every warp walks its own items

  uint8_t* const sq_area = wbuf + 2 * T::kBufBytes;
  const int offset = Walk::offset();
  typename Walk::Item first = kSplit ? static_cast<typename Walk::Item>(blockIdx.x)
                                     : static_cast<typename Walk::Item>(blockIdx.x) * kAttnWarps + warp;
  Walk walk{a, staged};
  if constexpr (Walk::kBlocked) {
    // this warp's contiguous range of the U = (items of one kv head) x kv heads items
    const long long U = static_cast<long long>(s_len[2 * T::kSeqlenSlots]) * a.kv_heads;
    const long long W = static_cast<long long>(gridDim.x) * kAttnWarps;
    const long long w = static_cast<long long>(blockIdx.x) * kAttnWarps + warp;
    first = static_cast<typename Walk::Item>(w * U / W);
    walk.end = static_cast<typename Walk::Item>((w + 1) * U / W);
  }
  typename Walk::Cursor cur = walk.seek(first);
  if (cur.item < 0) return;
  uint32_t mask_cur = attn_issue<B, D>(a, cur, offset, wbuf, sq_area, lane);
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  int b = 0;

  // This lane's score columns are 2j and 2j + 1: query heads 2j + e, or with kG4
  // heads (2j + e) & 3.
  uint32_t qb0[KS], qb1[KS];
  float m_ref[2], l_part[2];
  float acc[KS][4];
  int run_chunk = 0;  // the chunk whose entry receives the current softmax state

  // Per iteration: wait for the current sub-chunk, take the item's query
  // fragments if it starts here, issue the next sub-chunk's copies into the
  // other buffer, then compute on the current one.
  while (true) {
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncwarp();
    if (cur.sub == 0 && !cur.fresh) {
      // an item that continues the state: its own entry is marked empty (-inf maximum)
      if ((!kG4 || j < 2) && g == 0) {
        const long long head0 = static_cast<long long>(cur.seq) * a.n_heads + static_cast<long long>(cur.kvh) * a.group;
        float* const entry = a.ws + (head0 * a.max_chunks + cur.chunk) * (D + 2);
        const long long entry_stride = static_cast<long long>(a.max_chunks) * (D + 2);
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if (2 * j + e < a.group) entry[(2 * j + e) * entry_stride] = -INFINITY;
      }
    }
    if (cur.sub == 0 && cur.fresh) {
      // a new item: query fragments (B operand of K Q^T, column g = head g, or g & 3
      // with kG4; heads past the group zero; head_dim elements in the K span order)
      // and a fresh softmax state
      const __half(*sq)[D] = reinterpret_cast<const __half(*)[D]>(sq_area);
      const int hq = kG4 ? (g & 3) : g;
      const bool live = hq < a.group;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        const int d00 = T::KN * j + Codec::row_pair_elem(2 * s, 0), d01 = T::KN * j + Codec::row_pair_elem(2 * s, 1);
        const int d10 = T::KN * j + Codec::row_pair_elem(2 * s + 1, 0);
        const int d11 = T::KN * j + Codec::row_pair_elem(2 * s + 1, 1);
        const __half* qr = sq[live ? hq : 0];
        qb0[s] = live ? as_u32(__halves2half2(qr[d00], qr[d01])) : 0u;
        qb1[s] = live ? as_u32(__halves2half2(qr[d10], qr[d11])) : 0u;
      }
      m_ref[0] = m_ref[1] = -INFINITY;
      l_part[0] = l_part[1] = 0.0f;
      run_chunk = cur.chunk;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.0f;
      if (cur.chunk == 0 && cur.kvh == 0 && lane == 0) {
        const long long L = a.seqlens[cur.seq];
        if (L > walk.max_len()) record_error(KVQ_DEV_BAD_PAGE_INDEX);  // window longer than the cache
      }
      __syncwarp();  // the query area may be refilled below
    }
    const typename Walk::Cursor nxt = walk.next(cur);
    uint32_t mask_nxt = 0;
    if (nxt.item >= 0) {
      mask_nxt = attn_issue<B, D>(a, nxt, offset, wbuf + (b ^ 1) * T::kBufBytes, sq_area, lane);
      asm volatile("cp.async.commit_group;\n" ::: "memory");
    }

    const uint8_t* const buf = wbuf + b * T::kBufBytes;
    const uint8_t* const sk = buf;
    const uint8_t* const sv = buf + T::kBufK;
    const __half* const sks = reinterpret_cast<const __half*>(buf + T::kBufK + T::kBufV);
    const __half* const svs = sks + SC * T::kScales;

    // one 16-position step; a full buffer of 4-bit codes runs its steps unrolled
    // (measured 2.5% faster: one step's dequantization overlaps the other's latency)
    auto step = [&](const int t0) {
      // ---- S^T = K Q^T for positions t0 + g (rows g) and t0 + 8 + g (rows g + 8):
      // this lane's K spans are the A fragments, the query the B fragment
      float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      {
        uint32_t ka[KR], kb[KR];
        k_span<B, D>(sk + (t0 + g) * T::kStrideK, sks + (t0 + g) * T::kScales, j, ka);
        k_span<B, D>(sk + (t0 + 8 + g) * T::kStrideK, sks + (t0 + 8 + g) * T::kScales, j, kb);
#pragma unroll
        for (int s = 0; s < KS; ++s) mma_16816(sc, ka[2 * s], kb[2 * s], ka[2 * s + 1], kb[2 * s + 1], qb0[s], qb1[s]);
      }
      // x[e], x[2 + e]: scaled scores of column 2j + e at positions t0 + g and
      // t0 + 8 + g; positions without data -inf (only a step with such
      // positions pays for the mask)
      float x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = sc[i] * a.scale_log2;
      const uint32_t live16 = (mask_cur >> t0) & 0xFFFFu;
      const bool full = live16 == 0xFFFFu;  // the same in every lane
      if (!full) {
        if (!((live16 >> g) & 1u)) x[0] = x[1] = -INFINITY;
        if (!((live16 >> (g + 8)) & 1u)) x[2] = x[3] = -INFINITY;
      }
      // lazy rescale: the reference of a head moves only when the step's maximum
      // exceeds it by more than the threshold; each lane tests its own scores and
      // the warp takes the maximum only when one of them does
      const bool grow = fmaxf(x[0], x[2]) > m_ref[0] + kAttnRescaleLog2 ||
                        fmaxf(x[1], x[3]) > m_ref[1] + kAttnRescaleLog2;
      if (__any_sync(0xFFFFFFFFu, grow)) {
        float al[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mx = fmaxf(x[e], x[2 + e]);
          mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
          al[e] = 1.0f;
          if (mx > m_ref[e] + kAttnRescaleLog2) {
            al[e] = (m_ref[e] == -INFINITY) ? 0.0f : exp2_approx(m_ref[e] - mx);
            m_ref[e] = mx;
          }
          l_part[e] *= al[e];
        }
        // accumulator columns 2j, 2j + 1 belong to this lane's heads
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          acc[mt][0] *= al[0];
          acc[mt][1] *= al[1];
          acc[mt][2] *= al[0];
          acc[mt][3] *= al[1];
        }
      }
      float p[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) p[i] = exp2_approx(x[i] - m_ref[i & 1]);
      if (!full) {
        // a head with no data yet has reference -inf: its masked scores weigh 0
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (x[i] == -INFINITY) p[i] = 0.0f;
      }
      l_part[0] += p[0] + p[2];
      l_part[1] += p[1] + p[3];
      // ---- the weights as a binary16 high part and a binary16 residual; rows of
      // the 8 x 8 blocks P[t0 + (0..7)][columns] and P[t0 + 8 + (0..7)][columns],
      // transposed into the B fragments of P^T
      const uint32_t h0 = pack_half2(p[0], p[1]), h1 = pack_half2(p[2], p[3]);
      const float2 f0 = __half22float2(as_h2(h0)), f1 = __half22float2(as_h2(h1));
      const uint32_t r0 = pack_half2(p[0] - f0.x, p[1] - f0.y), r1 = pack_half2(p[2] - f1.x, p[3] - f1.y);

      // ---- O^T += V^T P^T: row pairs (2j, 2j+1) and (2j+8, 2j+9) of the 16 positions
      uint32_t va[KR], vb[KR];
      {
        const int i0 = t0 + 2 * j, i1 = i0 + 8;
        const int sblk = (T::VN * g) / 32;
        const __half zero = __ushort_as_half(0);
        const __half s00 = T::kScales ? svs[i0 * T::kScales + sblk] : zero;
        const __half s01 = T::kScales ? svs[(i0 + 1) * T::kScales + sblk] : zero;
        const __half s10 = T::kScales ? svs[i1 * T::kScales + sblk] : zero;
        const __half s11 = T::kScales ? svs[(i1 + 1) * T::kScales + sblk] : zero;
        v_span_pair<B, D>(sv + i0 * T::kStrideV, sv + (i0 + 1) * T::kStrideV, s00, s01, g, va);
        v_span_pair<B, D>(sv + i1 * T::kStrideV, sv + (i1 + 1) * T::kStrideV, s10, s11, g, vb);
      }
      if constexpr (kG4) {
        // columns 0..3 the high parts, 4..7 (lanes j >= 2) the residuals
        const uint32_t b0 = movmatrix_trans(j >= 2 ? r0 : h0), b1 = movmatrix_trans(j >= 2 ? r1 : h1);
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) mma_16816(acc[mt], va[2 * mt], va[2 * mt + 1], vb[2 * mt], vb[2 * mt + 1], b0, b1);
      } else {
        const uint32_t bh0 = movmatrix_trans(h0), bh1 = movmatrix_trans(h1);
        const uint32_t bl0 = movmatrix_trans(r0), bl1 = movmatrix_trans(r1);
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          mma_16816(acc[mt], va[2 * mt], va[2 * mt + 1], vb[2 * mt], vb[2 * mt + 1], bh0, bh1);
          mma_16816(acc[mt], va[2 * mt], va[2 * mt + 1], vb[2 * mt], vb[2 * mt + 1], bl0, bl1);
        }
      }
        };
    if (B == 4 && !kSplit && cur.n == SC) {
#pragma unroll
      for (int t0 = 0; t0 < SC; t0 += 16) step(t0);
    } else {
      for (int t0 = 0; t0 < cur.n; t0 += 16) step(t0);
    }

    // the state is written when it ends: at the last sub-chunk of an item that the
    // next one does not continue
    if (cur.last && (nxt.item < 0 || nxt.fresh)) {
      // the state's partial result: (max, sum, accumulator) of every head of the group
      float l_sum[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = l_part[e];
        l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
        l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
        l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
        l_sum[e] = l;
      }
      if constexpr (kG4) {
        // high part (lanes j < 2) plus residual (lanes j + 2)
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[mt][i] += __shfl_xor_sync(0xFFFFFFFFu, acc[mt][i], 2);
      }
      const long long head0 = static_cast<long long>(cur.seq) * a.n_heads + static_cast<long long>(cur.kvh) * a.group;
      float* const entry = a.ws + (head0 * a.max_chunks + run_chunk) * (D + 2);
      const long long entry_stride = static_cast<long long>(a.max_chunks) * (D + 2);  // next head, same chunk
      // kSplit: the warp's quarter goes to its own buffer (free now: the next
      // sub-chunk streams into the other one), one (D + 2)-float row per head
      float* const ws = kSplit ? reinterpret_cast<float*>(wbuf + b * T::kBufBytes) : entry;
      const long long hstride = kSplit ? D + 2 : entry_stride;
      if (kSplit) __syncwarp();  // every lane is done reading the buffer
      if (!kG4 || j < 2) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * j + e;
          if (h < a.group) {
            if (g == 0) {
              ws[h * hstride] = m_ref[e];
              ws[h * hstride + 1] = l_sum[e];
            }
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
              ws[h * hstride + 2 + T::VN * g + Codec::xrow_elem(2 * mt)] = acc[mt][e];
              ws[h * hstride + 2 + T::VN * g + Codec::xrow_elem(2 * mt + 1)] = acc[mt][2 + e];
            }
          }
        }
      }
      if constexpr (kSplit) {
        // Merge the four quarters into the item's workspace entry.  Every warp
        // of the CTA walks the same items with the same number of sub-chunks,
        // so all four reach these barriers together and use the same buffer b.
        __syncthreads();
        for (int e = threadIdx.x; e < a.group * D; e += kAttnThreads) {
          const int h = e / D, d = e - h * D;
          const float* part[kAttnWarps];
          float mx = -INFINITY;
#pragma unroll
          for (int w = 0; w < kAttnWarps; ++w) {
            part[w] = reinterpret_cast<const float*>(smem + w * T::kWarpBytes + b * T::kBufBytes) + h * (D + 2);
            mx = fmaxf(mx, part[w][0]);
          }
          float o = 0.0f, l = 0.0f;
#pragma unroll
          for (int w = 0; w < kAttnWarps; ++w) {
            const float f = (part[w][0] == -INFINITY) ? 0.0f : exp2f(part[w][0] - mx);
            o += f * part[w][2 + d];
            l += f * part[w][1];
          }
          entry[h * entry_stride + 2 + d] = o;
          if (d == 0) {
            entry[h * entry_stride] = mx;
            entry[h * entry_stride + 1] = l;
            // the item's second chunk, when it holds data, has no entry of its own
            if (Walk::kItemChunks == 2 && (cur.chunk + 1) * T::kChunk < walk.length(cur.seq))
              entry[h * entry_stride + (D + 2)] = -INFINITY;
          }
        }
        __syncthreads();  // the buffers are refilled from the next iteration on
      }
    }
    __syncwarp();  // every lane is done with this buffer before it is refilled
    if (nxt.item < 0) break;
    cur = nxt;
    mask_cur = mask_nxt;
    b ^= 1;
  }
}

// Merge the chunk entries of every (sequence, head): CTA (head, sequence) of
// four warps.  Warp w takes chunks w, w + 4, ... in batches of kCombineBatch<D>
// whose loads are all issued before any is used (lane l owns head_dim elements
// l, l + 32, ...), and folds each batch into a running (max, sum, accumulator)
// that it rescales when the maximum moves; the four warps' results meet in
// shared memory.
constexpr int kCombineThreads = 128;
template <int D>
constexpr int kCombineBatch = 1024 / D;  // chunks per warp in flight: 32 loaded values per lane

template <int D>
__global__ void __launch_bounds__(kCombineThreads, 8) attn_combine_kernel(const __grid_constant__ AttnParams a) {
  constexpr int kWarps = kCombineThreads / 32, DPL = D / 32, NB = kCombineBatch<D>;
  __shared__ float s_m[kWarps], s_l[kWarps];
  __shared__ float s_o[kWarps][D];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int h = blockIdx.x, seq = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long L = a.seqlens[seq];
  if (L < 0) L = 0;
  if (a.page_size == 0 && L > a.dim1) L = a.dim1;
  long long nch = (L + a.chunk - 1) / a.chunk;
  if (nch > a.max_chunks) nch = a.max_chunks;
  const float* ws = a.ws + (static_cast<long long>(seq) * a.n_heads + h) * a.max_chunks * (D + 2);
  float m_run = -INFINITY, l_run = 0.0f, acc[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) acc[k] = 0.0f;
  for (long long c0 = warp; c0 < nch; c0 += static_cast<long long>(kWarps) * NB) {
    float mc[NB], lc[NB], x[NB][DPL];
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      const long long c = c0 + static_cast<long long>(i) * kWarps;
      const bool in = c < nch;
      const float* e = ws + (in ? c : 0) * (D + 2);
      mc[i] = in ? e[0] : -INFINITY;
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      // an entry with a -inf maximum holds nothing (no data, or merged into an earlier entry)
      const long long c = c0 + static_cast<long long>(i) * kWarps;
      const bool live = mc[i] != -INFINITY;
      const float* e = ws + (live ? c : 0) * (D + 2);
      lc[i] = live ? e[1] : 0.0f;
#pragma unroll
      for (int k = 0; k < DPL; ++k) x[i][k] = live ? e[2 + lane + 32 * k] : 0.0f;
    }
    float mb = m_run;
#pragma unroll
    for (int i = 0; i < NB; ++i) mb = fmaxf(mb, mc[i]);
    const float r = (m_run == -INFINITY) ? 0.0f : exp2f(m_run - mb);
    l_run *= r;
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[k] *= r;
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      const float f = (mc[i] == -INFINITY) ? 0.0f : exp2f(mc[i] - mb);
      l_run += f * lc[i];
#pragma unroll
      for (int k = 0; k < DPL; ++k) acc[k] += f * x[i][k];
    }
    m_run = mb;
  }
  if (lane == 0) {
    s_m[warp] = m_run;
    s_l[warp] = l_run;
  }
#pragma unroll
  for (int k = 0; k < DPL; ++k) s_o[warp][lane + 32 * k] = acc[k];
  __syncthreads();
  float mstar = s_m[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) mstar = fmaxf(mstar, s_m[w]);
  float fw[kWarps], lt = 0.0f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    fw[w] = (s_m[w] == -INFINITY) ? 0.0f : exp2f(s_m[w] - mstar);
    lt += fw[w] * s_l[w];
  }
  for (int d = threadIdx.x; d < D; d += kCombineThreads) {
    float o = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) o += fw[w] * s_o[w][d];
    const float y = (lt > 0.0f) ? o / lt : 0.0f;
    a.out[(static_cast<long long>(seq) * a.n_heads + h) * D + d] = __float2half_rn(y);
  }
}

}  // namespace kvq
