// attention_selfcheck.cuh -- measures, on the device, the three arithmetic
// constants the decode-attention error bound rests on:
//   [0] the largest relative error of ex2.approx.ftz.f32 over every binary32
//       argument in [-126, 8] (the softmax weights 2^(x - m) with x - m <= 8,
//       and the lazy-rescale factors; results below 2^-126 flush to zero and
//       are bounded separately as an absolute error);
//   [1] the largest relative error of exp2f over every binary32 argument in
//       [-126, 0] (the chunk merge factors);
//   [2] the largest accumulation error of mma.sync m16n8k16 (binary16
//       products, binary32 accumulator) on adversarial random inputs, in units
//       of 2^-23 times the largest magnitude among the 16 products and the
//       accumulator.  The bound models one MMA step as exact products, aligned
//       to the largest exponent and truncated, then a truncated normalization:
//       an error below (16 + 2) * 2^-23 * max |term|.
// The references are binary64 (exp2 of a binary32 argument to within one
// binary64 ulp; the 17-term sums exact to within 17 * 2^-53 relative), far
// below what is measured.  Maxima of non-negative doubles are combined with
// atomicMax on their bit patterns, which order the same way.
#pragma once

#include <stdint.h>

namespace kvq {

__device__ __forceinline__ void atomic_max_nonneg(double* dst, double v) {
  atomicMax(reinterpret_cast<unsigned long long*>(dst), static_cast<unsigned long long>(__double_as_longlong(v)));
}

// Warp-wide maximum, then one atomic per warp.
__device__ __forceinline__ void warp_max_to(double* dst, double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  if ((threadIdx.x & 31) == 0 && v > 0.0) atomic_max_nonneg(dst, v);
}

// Every binary32 bit pattern in [lo_bits, hi_bits] (both of one sign, as
// unsigned integers) through f, relative error against exp2 in binary64.
template <bool kApprox>
__global__ void selfcheck_exp2_kernel(uint32_t lo_bits, uint32_t hi_bits, double* result) {
  double worst = 0.0;
  const uint64_t n = static_cast<uint64_t>(hi_bits) - lo_bits + 1;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float x = __uint_as_float(static_cast<uint32_t>(lo_bits + i));
    float y;
    if (kApprox) {
      asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    } else {
      y = exp2f(x);
    }
    const double ref = exp2(static_cast<double>(x));
    worst = fmax(worst, fabs(static_cast<double>(y) - ref) / ref);
  }
  warp_max_to(result, worst);
}

// Counter-based pseudo-random 32-bit words (a 64-bit mix of the counter), so
// that every lane can regenerate any element of a trial's matrices.
__device__ __forceinline__ uint32_t mix32(uint64_t x) {
  x ^= x >> 33;
  x *= 0xFF51AFD7ED558CCDull;
  x ^= x >> 33;
  x *= 0xC4CEB9FE1A85EC53ull;
  x ^= x >> 33;
  return static_cast<uint32_t>(x);
}

// A binary16 with a random sign, a random 10-bit fraction and an exponent in
// [2^-10, 2^10]; about one element in eight is zero, so that some steps have
// few live terms.
__device__ __forceinline__ uint16_t rand_half(uint64_t key) {
  const uint32_t r = mix32(key);
  if ((r & 7u) == 0u) return 0;
  const uint32_t e = 5u + (r >> 3) % 21u;  // biased exponent 5..25
  return static_cast<uint16_t>(((r >> 16) & 0x8000u) | (e << 10) | ((r >> 8) & 0x3FFu));
}

// Element (row, col) of trial t's matrix `which` (0: A 16x16, 1: B 16x8 as
// [k][n]).
__device__ __forceinline__ __half trial_elem(uint64_t t, int which, int row, int col) {
  return __ushort_as_half(rand_half((t * 4 + which) * 4096 + row * 64 + col));
}

// Accumulator: random sign, magnitude 2^e with e in [-30, 30] and a random
// significand, zero in one trial of eight.
__device__ __forceinline__ float trial_acc(uint64_t t, int row, int col) {
  const uint32_t r = mix32((t * 4 + 2) * 4096 + row * 64 + col);
  if ((r & 7u) == 0u) return 0.0f;
  const int e = static_cast<int>((r >> 3) % 61u) - 30;
  const float m = 1.0f + static_cast<float>((r >> 9) & 0x7FFFFFu) * 0x1p-23f;
  return ((r >> 8) & 1u ? -1.0f : 1.0f) * ldexpf(m, e);
}

__global__ void selfcheck_mma_kernel(uint64_t trials_per_warp, double* result) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const uint64_t warp = (static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  double worst = 0.0;
  for (uint64_t it = 0; it < trials_per_warp; ++it) {
    const uint64_t t = warp * trials_per_warp + it;
    auto frag_a = [&](int r, int k) {
      const __half2 h = __halves2half2(trial_elem(t, 0, r, k), trial_elem(t, 0, r, k + 1));
      return *reinterpret_cast<const uint32_t*>(&h);
    };
    auto frag_b = [&](int k, int n) {
      const __half2 h = __halves2half2(trial_elem(t, 1, k, n), trial_elem(t, 1, k + 1, n));
      return *reinterpret_cast<const uint32_t*>(&h);
    };
    // fragments of m16n8k16 (row.col): A rows g, g + 8, columns 2j.., 2j + 8..;
    // B column g, rows 2j.., 2j + 8..; C / D rows g, g + 8, columns 2j, 2j + 1
    const uint32_t a0 = frag_a(g, 2 * j), a1 = frag_a(g + 8, 2 * j), a2 = frag_a(g, 2 * j + 8);
    const uint32_t a3 = frag_a(g + 8, 2 * j + 8);
    const uint32_t b0 = frag_b(2 * j, g), b1 = frag_b(2 * j + 8, g);
    float c[4];
    const int rows[4] = {g, g, g + 8, g + 8}, cols[4] = {2 * j, 2 * j + 1, 2 * j, 2 * j + 1};
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] = trial_acc(t, rows[e], cols[e]);
    float d[4] = {c[0], c[1], c[2], c[3]};
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      double exact = c[e], big = fabs(static_cast<double>(c[e]));
      for (int k = 0; k < 16; ++k) {
        const double p = static_cast<double>(__half2float(trial_elem(t, 0, rows[e], k))) *
                         static_cast<double>(__half2float(trial_elem(t, 1, k, cols[e])));
        exact += p;
        big = fmax(big, fabs(p));
      }
      if (big > 0.0) worst = fmax(worst, fabs(static_cast<double>(d[e]) - exact) / (big * 0x1p-23));
    }
  }
  warp_max_to(result, worst);
}

}  // namespace kvq

extern "C" {

kvq_status kvq_selfcheck_attention_numerics(double* results, void* stream) {
  if (!results) return KVQ_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(results) & 7u) return KVQ_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(results, 0, 3 * sizeof(double), s) != cudaSuccess) return KVQ_ERR_CUDA;
  // binary32 bit patterns: -0 .. -126 (0x80000000 .. 0xC2FC0000) and +0 .. +8 (0 .. 0x41000000)
  kvq::selfcheck_exp2_kernel<true><<<1184, 256, 0, s>>>(0x80000000u, 0xC2FC0000u, results);
  kvq::selfcheck_exp2_kernel<true><<<1184, 256, 0, s>>>(0x00000000u, 0x41000000u, results);
  kvq::selfcheck_exp2_kernel<false><<<1184, 256, 0, s>>>(0x80000000u, 0xC2FC0000u, results + 1);
  // 1184 CTAs x 8 warps x 256 trials x 128 outputs: 310 M accumulations
  kvq::selfcheck_mma_kernel<<<1184, 256, 0, s>>>(256, results + 2);
  return launch_status();
}

}  // extern "C"
