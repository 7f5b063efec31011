// attention.cuh -- decode attention that reads the quantized KV cache
// directly: the conversions' consumer "during the attention forward pass"
// (page "Implementation: Turboderp org Exllamav2 Ext Cache", Usage), with the
// FP16 cache never written back.
//
// One new query per sequence and head; GQA: `group` query heads share a kv
// head.  Keys and values are the dequantized codes, bit for bit what
// q_to_fp16_kv writes (dequantized in registers with the same arithmetic).
//
// Split-K flash decoding.  Kernel 1 (attn_partial_kernel): one CTA per
// (chunk of positions, kv head, sequence), four warps.  The CTA first copies
// its whole chunk of K and V codes and scales into shared memory with
// cp.async (all copies in flight at once, so a CTA keeps tens of KB of
// loads outstanding), then each warp takes 16 positions at a time and
//   * dequantizes K for the 16 positions into mma.sync m16n8k16 A fragments
//     (positions are the M dimension, the query heads of the group the N
//     dimension, padded to 8), multiplies by the preloaded query fragments
//     (fp16 inputs, fp32 accumulation: products are exact);
//   * updates an online softmax (base 2) per query head;
//   * dequantizes V for the 16 positions into A fragments of O^T = V^T P^T
//     (head_dim is the M dimension) and accumulates with P split into a
//     binary16 high part and a binary16 residual (two MMAs), so the weights
//     keep about 22 significant bits.
// The head_dim order inside a fragment is permuted so that every lane's
// slice of a cache row is contiguous (one wide load, one scale); the query
// and the output use the same permutation.  The four warps' states merge
// in shared memory and the chunk's (max, sum, accumulator) goes to the
// workspace.  Kernel 2 (attn_combine_kernel) merges the chunks of each
// (sequence, head) and writes binary16 outputs.
#pragma once

#include "codec.cuh"
#include "tiles.cuh"

namespace kvq {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = 32 * kAttnWarps;
constexpr int kAttnMaxGroup = 8;  // query heads per kv head (one MMA N block)

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
  int chunk;  // positions per CTA (AttnTile<B, D>::kChunk)
  float scale_log2;  // softmax_scale * log2(e)
};

__device__ __forceinline__ void mma_16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Shared-memory staging of one CTA's chunk: K codes, V codes (rows padded
// by 16 bytes so that the fragment reads of neighbouring rows fall in
// different banks), K scales, V scales, then each position's cache row index.
// Rows of up to 64 code bytes take 256-position chunks, longer rows 128.
template <int B, int D>
struct AttnTile {
  static constexpr int kRowBytes = D * B / 8;
  static constexpr int kStride = kRowBytes + 16;
  static constexpr int kScales = D / 32;
  static constexpr int kChunk = kRowBytes <= 64 ? 256 : 128;
  static constexpr int kCodeBytes = kChunk * kStride;
  static constexpr int kScaleBytes = kChunk * kScales * 2;
  static constexpr int kStageBytes = 2 * (kCodeBytes + kScaleBytes);
  static constexpr int kAccBytes = kAttnWarps * D * (kAttnMaxGroup + 1) * 4;  // merge area (aliases the stage)
  static constexpr int kRowIdxOffset = kStageBytes > kAccBytes ? kStageBytes : kAccBytes;
  static constexpr int kSmemBytes = kRowIdxOffset + kChunk * 8;
};
constexpr int kAttnMinChunk = 128;  // smallest chunk any (B, D) uses: sizes the workspace

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_small(void* dst, const void* src) {
  static_assert(N == 4 || N == 8 || N == 16, "cp.async sizes");
  asm volatile("cp.async.ca.shared.global [%0], [%1], %2;\n" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "n"(N)
               : "memory");
}

// Dequantize N consecutive elements [d, d + N) of one staged row (d a
// multiple of N, N a multiple of 8) into N / 2 half2 registers (element
// pairs (d + 2e, d + 2e + 1)).  Every 32-element block inside the span
// starts at a multiple of 32, so 8-element unit u uses scale (d >> 5) + (u >> 2).
template <int B, int N>
__device__ __forceinline__ void dequant_span(const uint8_t* row, const __half* srow, int d, uint32_t out[N / 2]) {
  static_assert(N % 8 == 0, "whole 8-element units");
  constexpr int NB = N * B / 8;  // bytes of the span; the span starts at a multiple of NB
  const uint8_t* p = row + d * B / 8;
  uint32_t w[(NB + 3) / 4 + 1];
  if constexpr (B == 6 && N == 8) {
    // 6 bytes at a 2-byte offset: the two words of the 12-byte group half
    const uint32_t* grp = reinterpret_cast<const uint32_t*>(row + (d >> 4) * 12);
    const int half = (d >> 3) & 1;
    const uint32_t a = grp[half], b = grp[half + 1];
    w[0] = __funnelshift_r(a, b, 16 * half);
    w[1] = (b >> (16 * half)) & 0xFFFFu;
  } else if constexpr (NB % 16 == 0) {
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
#pragma unroll
  for (int u = 0; u < N / 8; ++u) {
    const __half s = srow[(d >> 5) + (u >> 2)];
    const __half2 s2 = __halves2half2(s, s);
    uint4 r;
    if constexpr (B == 4) {
      r = dequant_q4_v8(w[u], s2);
    } else if constexpr (B == 8) {
      r = dequant_q8_v8(w[2 * u], w[2 * u + 1], s2);
    } else if constexpr (N == 8) {
      r = dequant_q6_v8(w[0], w[1], s2);
    } else {
      const int q = u >> 1;  // 16-code group: words 3q .. 3q + 2
      r = (u & 1) ? dequant_q6_v8(__funnelshift_r(w[3 * q + 1], w[3 * q + 2], 16), w[3 * q + 2] >> 16, s2)
                  : dequant_q6_v8(w[3 * q], w[3 * q + 1] & 0xFFFFu, s2);
    }
    out[4 * u + 0] = r.x;
    out[4 * u + 1] = r.y;
    out[4 * u + 2] = r.z;
    out[4 * u + 3] = r.w;
  }
}

// Physical row of logical position p of sequence `seq`, or -1 when the paging
// metadata points outside the cache.
__device__ __forceinline__ long long attn_row(const AttnParams& a, int seq, long long p, const int* bt_chunk,
                                              long long lp0) {
  if (a.page_size == 0) return static_cast<long long>(seq) * a.dim1 + p;
  const long long lp = p / a.page_size;
  if (lp >= a.bt_stride) return -1;
  const int page = bt_chunk[lp - lp0];
  if (page < 0 || page >= a.dim0) return -1;
  return static_cast<long long>(page) * a.page_size + p % a.page_size;
}

template <int B, int D>
__global__ void __launch_bounds__(kAttnThreads) attn_partial_kernel(const __grid_constant__ AttnParams a) {
  using T = AttnTile<B, D>;
  constexpr int KS = D / 16;  // k-steps of Q K^T, m-blocks of V^T P^T
  constexpr int KN = D / 4;   // K elements per lane per position
  constexpr int VN = D / 8;   // V elements per lane per position
  constexpr int C = T::kChunk;

  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* const sk = smem;
  uint8_t* const sv = smem + T::kCodeBytes;
  __half* const sks = reinterpret_cast<__half*>(smem + 2 * T::kCodeBytes);
  __half* const svs = sks + C * T::kScales;
  long long* const s_hr = reinterpret_cast<long long*>(smem + T::kRowIdxOffset);
  float(*const s_acc)[D][kAttnMaxGroup + 1] = reinterpret_cast<float(*)[D][kAttnMaxGroup + 1]>(smem);
  __shared__ int s_bt[C + 1];
  __shared__ float s_p[kAttnWarps][16][kAttnMaxGroup + 1];
  __shared__ float s_m[kAttnWarps][kAttnMaxGroup];
  __shared__ float s_l[kAttnWarps][kAttnMaxGroup];
  __shared__ int s_bad;

  const int chunk = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, j = lane & 3;

  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) s_bad = 0;

  long long L = a.seqlens[seq];
  if (L < 0) L = 0;
  const long long max_len = a.page_size == 0 ? static_cast<long long>(a.dim1)
                                             : static_cast<long long>(a.max_chunks) * C;
  if (L > max_len) {  // longer than the cache (contiguous) or than the launched chunks (paged)
    if (threadIdx.x == 0 && chunk == 0 && kvh == 0) record_error(KVQ_DEV_BAD_PAGE_INDEX);
    L = max_len;
  }
  const long long p0 = static_cast<long long>(chunk) * C;
  if (p0 >= L) return;  // the whole CTA leaves together
  const long long p1 = min(L, p0 + C);
  const int n = static_cast<int>(p1 - p0);

  // block-table entries of the chunk's logical pages, staged once
  long long lp0 = 0;
  if (a.page_size > 0) {
    lp0 = p0 / a.page_size;
    const long long lp1 = (p1 - 1) / a.page_size;
    for (long long lp = lp0 + threadIdx.x; lp <= lp1; lp += kAttnThreads)
      s_bt[lp - lp0] = lp < a.bt_stride ? a.block_table[static_cast<long long>(seq) * a.bt_stride + lp] : -1;
  }
  __syncthreads();

  // cache row of every position of the chunk (-1: bad paging metadata, -2: past the window)
  for (int i = threadIdx.x; i < C; i += kAttnThreads) {
    long long hr = -2;
    if (i < n) {
      const long long row = attn_row(a, seq, p0 + i, s_bt, lp0);
      if (row < 0) s_bad = 1;
      hr = row < 0 ? -1 : row * a.kv_heads + kvh;
    }
    s_hr[i] = hr;
  }
  __syncthreads();

  // issue every copy of the chunk; rows without data get zero scales, which
  // dequantize whatever codes the buffer holds to zero
  {
    constexpr int P = T::kRowBytes / 16;
    for (int t = threadIdx.x; t < C * P; t += kAttnThreads) {
      const int i = t / P, part = t - i * P;
      const long long hr = s_hr[i];
      if (hr >= 0) {
        const long long off = hr * T::kRowBytes + part * 16;
        cp_async16(sk + i * T::kStride + part * 16, a.k_codes + off);
        cp_async16(sv + i * T::kStride + part * 16, a.v_codes + off);
      }
    }
    for (int i = threadIdx.x; i < C; i += kAttnThreads) {
      const long long hr = s_hr[i];
      if (hr >= 0) {
        cp_async_small<T::kScales * 2>(sks + i * T::kScales, a.k_scales + hr * T::kScales);
        cp_async_small<T::kScales * 2>(svs + i * T::kScales, a.v_scales + hr * T::kScales);
      } else {
#pragma unroll
        for (int e = 0; e < T::kScales; ++e) sks[i * T::kScales + e] = svs[i * T::kScales + e] = __ushort_as_half(0);
      }
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  }

  // query fragments (B operand of Q K^T): head g of the group, this lane's
  // permuted head_dim slice d = KN*j + 4s + {0..3}; loaded while the copies fly
  uint32_t qf[KS][2];
  {
    const bool live = g < a.group;
    const __half* qrow = a.q + (static_cast<long long>(seq) * a.n_heads + kvh * a.group + (live ? g : 0)) * D;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const int d0 = KN * j + 4 * s;
      qf[s][0] = live ? __ldg(reinterpret_cast<const uint32_t*>(qrow + d0)) : 0u;
      qf[s][1] = live ? __ldg(reinterpret_cast<const uint32_t*>(qrow + d0 + 2)) : 0u;
    }
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();

  float m_run[2] = {-INFINITY, -INFINITY};  // heads 2j, 2j+1 (log2 domain)
  float l_run[2] = {0.0f, 0.0f};
  float acc[KS][4];
#pragma unroll
  for (int mb = 0; mb < KS; ++mb) acc[mb][0] = acc[mb][1] = acc[mb][2] = acc[mb][3] = 0.0f;

  for (int t0 = 16 * warp; t0 < n; t0 += 16 * kAttnWarps) {
    // ---- K: positions t0 + g and t0 + g + 8, elements [KN*j, KN*j + KN)
    uint32_t kd[2][KN / 2];
    bool kvalid[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = t0 + g + 8 * r;
      kvalid[r] = s_hr[i] >= 0;
      dequant_span<B, KN>(sk + i * T::kStride, sks + i * T::kScales, KN * j, kd[r]);
    }
    float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const uint32_t af[4] = {kd[0][2 * s], kd[1][2 * s], kd[0][2 * s + 1], kd[1][2 * s + 1]};
      mma_16816(sc, af, qf[s][0], qf[s][1]);
    }
    // scores: sc[0] = (pos g, head 2j), sc[1] = (g, 2j+1), sc[2] = (g+8, 2j), sc[3] = (g+8, 2j+1)
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[e] = kvalid[e >> 1] ? sc[e] * a.scale_log2 : -INFINITY;

    // ---- online softmax for heads 2j, 2j+1 over the 16 positions
    float p_[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = fmaxf(sc[h], sc[2 + h]);
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
      const float m_new = fmaxf(m_run[h], mx);
      const float alpha = (m_new == -INFINITY) ? 1.0f : exp2f(m_run[h] - m_new);
      p_[h] = (sc[h] == -INFINITY) ? 0.0f : exp2f(sc[h] - m_new);
      p_[2 + h] = (sc[2 + h] == -INFINITY) ? 0.0f : exp2f(sc[2 + h] - m_new);
      float sum = p_[h] + p_[2 + h];
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 8);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 16);
      l_run[h] = l_run[h] * alpha + sum;
      m_run[h] = m_new;
      if (alpha != 1.0f) {
#pragma unroll
        for (int mb = 0; mb < KS; ++mb) {
          acc[mb][h] *= alpha;
          acc[mb][2 + h] *= alpha;
        }
      }
    }

    // ---- P^T as the B operand: lane needs P[head g][pos 2j, 2j+1, 2j+8, 2j+9]
    s_p[warp][g][2 * j] = p_[0];
    s_p[warp][g][2 * j + 1] = p_[1];
    s_p[warp][g + 8][2 * j] = p_[2];
    s_p[warp][g + 8][2 * j + 1] = p_[3];
    __syncwarp();
    const float b0 = s_p[warp][2 * j][g], b1 = s_p[warp][2 * j + 1][g];
    const float b2 = s_p[warp][2 * j + 8][g], b3 = s_p[warp][2 * j + 9][g];
    __syncwarp();
    const uint32_t bh0 = pack_half2(b0, b1), bh1 = pack_half2(b2, b3);
    const __half2 h0 = *reinterpret_cast<const __half2*>(&bh0), h1 = *reinterpret_cast<const __half2*>(&bh1);
    const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
    const uint32_t bl0 = pack_half2(b0 - f0.x, b1 - f0.y), bl1 = pack_half2(b2 - f1.x, b3 - f1.y);

    // ---- V: positions t0 + {2j, 2j+1, 2j+8, 2j+9}, elements [VN*g, VN*g + VN)
    uint32_t vd[4][VN / 2];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = t0 + 2 * j + (r & 1) + 8 * (r >> 1);
      dequant_span<B, VN>(sv + i * T::kStride, svs + i * T::kScales, VN * g, vd[r]);
    }
#pragma unroll
    for (int mb = 0; mb < KS; ++mb) {
      // rows d = VN*g + 2mb (+1 for rows g+8); columns = positions
      const uint32_t af[4] = {__byte_perm(vd[0][mb], vd[1][mb], 0x5410), __byte_perm(vd[0][mb], vd[1][mb], 0x7632),
                              __byte_perm(vd[2][mb], vd[3][mb], 0x5410), __byte_perm(vd[2][mb], vd[3][mb], 0x7632)};
      mma_16816(acc[mb], af, bh0, bh1);
      mma_16816(acc[mb], af, bl0, bl1);
    }
  }

  // ---- merge the four warps: acc[mb] holds O^T[d][h] for d = VN*g + 2mb (c0, c1: heads 2j, 2j+1)
  // and d + 1 (c2, c3).  The merge area aliases the staged chunk.
  __syncthreads();
  if (g == 0) {
    s_m[warp][2 * j] = m_run[0];
    s_m[warp][2 * j + 1] = m_run[1];
    s_l[warp][2 * j] = l_run[0];
    s_l[warp][2 * j + 1] = l_run[1];
  }
#pragma unroll
  for (int mb = 0; mb < KS; ++mb) {
    const int d = VN * g + 2 * mb;
    s_acc[warp][d][2 * j] = acc[mb][0];
    s_acc[warp][d][2 * j + 1] = acc[mb][1];
    s_acc[warp][d + 1][2 * j] = acc[mb][2];
    s_acc[warp][d + 1][2 * j + 1] = acc[mb][3];
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_bad) record_error(KVQ_DEV_BAD_PAGE);
  const int slots = a.group * (D + 2);
  for (int t = threadIdx.x; t < slots; t += kAttnThreads) {
    const int h = t / (D + 2), col = t % (D + 2);
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) mstar = fmaxf(mstar, s_m[w][h]);
    float v = 0.0f;
    if (col == 0) {
      v = mstar;
    } else {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float f = (s_m[w][h] == -INFINITY) ? 0.0f : exp2f(s_m[w][h] - mstar);
        v += f * (col == 1 ? s_l[w][h] : s_acc[w][col - 2][h]);
      }
    }
    const long long slot = (static_cast<long long>(seq) * a.n_heads + kvh * a.group + h) * a.max_chunks + chunk;
    a.ws[slot * (D + 2) + col] = v;
  }
}

// Merge the chunks of every (sequence, head): thread d of CTA (head, sequence).
template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(const __grid_constant__ AttnParams a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int h = blockIdx.x, seq = blockIdx.y, d = threadIdx.x;
  long long L = a.seqlens[seq];
  if (L < 0) L = 0;
  if (a.page_size == 0 && L > a.dim1) L = a.dim1;
  long long nch = (L + a.chunk - 1) / a.chunk;
  if (nch > a.max_chunks) nch = a.max_chunks;
  const float* ws = a.ws + (static_cast<long long>(seq) * a.n_heads + h) * a.max_chunks * (D + 2);
  float mstar = -INFINITY;
  for (long long c = 0; c < nch; ++c) mstar = fmaxf(mstar, ws[c * (D + 2)]);
  float l = 0.0f, o = 0.0f;
  for (long long c = 0; c < nch; ++c) {
    const float mc = ws[c * (D + 2)];
    const float f = (mc == -INFINITY) ? 0.0f : exp2f(mc - mstar);
    l += f * ws[c * (D + 2) + 1];
    o += f * ws[c * (D + 2) + 2 + d];
  }
  const float y = (l > 0.0f) ? o / l : 0.0f;
  a.out[(static_cast<long long>(seq) * a.n_heads + h) * D + d] = __float2half_rn(y);
}

}  // namespace kvq
