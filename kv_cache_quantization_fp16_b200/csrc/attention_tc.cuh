// attention_tc.cuh -- decode attention over the quantized or FP8 cache on the
// fifth-generation tensor cores (tcgen05.mma, accumulators in tensor memory),
// for head_dim 128.  Same contract and workspace as the mma.sync kernel in
// attention.cuh (page "Implementation: Turboderp org Exllamav2 Ext Cache",
// Usage: conversion "during the attention forward pass"): keys and values are
// bit for bit what q_to_fp16_kv / fp8_to_fp16 write, and every 256-position
// work item leaves (max, sum, accumulator) per query head for the combine
// kernel.
//
// CTA: four warps, one cache position per thread within a 128-position tile
// and one output row per thread; thread 0 also issues every tcgen05.mma (a
// fifth, MMA-only warp made the occupancy calculator round the CTA up to eight
// warps of registers, one CTA per SM).  Per tile:
//   * each math thread copies its position's K and V codes and scales into a
//     shared-memory stage with cp.async (the next tile's K as soon as this
//     tile's K row is read, its V as soon as this tile's V row is read, so each
//     copy has about a tile's time to land), dequantizes the K row and stores
//     it into tensor memory (tcgen05.st: lane = position, the A operand of
//     S^T), and the V row into shared memory (the MN-major A operand of O^T);
//   * S^T [128 positions x 16] = K Q^T: eight kind::f16 MMAs (K = 16 each), A
//     from tensor memory, B = the group's query rows in shared memory (rows
//     >= group zero), accumulated in binary32 in tensor memory;
//   * the math threads read S^T (tcgen05.ld: a thread's lane is its
//     position), and run the online softmax in base 2 with lazy rescaling:
//     the tile's maximum per head comes from a warp reduction and a shared
//     memory exchange, and the reference moves only when it exceeds the
//     current one by more than 2^8; the weights go to shared memory as a
//     binary16 high part and a binary16 residual (the MN-major B operand P^T);
//   * O^T [128 head_dim rows x 16] = V^T P_hi^T + V^T P_lo^T: sixteen MMAs;
//     each math thread folds its row (one head_dim element, all heads) into
//     binary32 accumulators in registers, rescaled when the reference moved.
// The math threads overlap the tensor-core work: the S MMAs run while they
// fold the previous tile's O^T and dequantize V, and the O^T MMAs while they
// dequantize the next tile's K.  Signals run both ways through mbarriers
// whose waits are bounded (1 s, then KVQ_DEV_TIMEOUT and a CTA-wide abort
// flag); an aborted CTA still passes every barrier of its schedule and frees
// its tensor memory.
//
// Element order.  For 4- and 6-bit codes the cheapest unpacking yields, per 8
// consecutive head_dim elements, the pairs (0,4), (1,5), (2,6), (3,7); the
// MMA's reduction dimension and the query rows use that order (perm8), and so
// do the output rows, which the write-out maps back.  8-bit codes and E5M2
// bytes unpack in natural order.
#pragma once

#include "attention.cuh"
#include "bulk_engine.cuh"

namespace kvq {

constexpr int kTcD = 128;
constexpr int kTcTile = 128;                  // positions per tile (the MMA's M for S^T)
constexpr int kTcItem = 256;                  // positions per work item (= workspace chunk)
constexpr int kTcMathThreads = 128;
constexpr int kTcThreads = kTcMathThreads;
constexpr uint32_t kTcTmemCols = 128;         // K tile 64 columns, S^T 2 x 16, O^T 2 x 16
// S^T is accumulated in two independent halves of the reduction (head_dim 0-63
// and 64-127), O^T in one accumulator for the weights' high parts and one for
// their residuals: four chains of four to eight MMAs instead of two of eight
// and sixteen, summed by the threads that read them.
constexpr uint32_t kTcColK = 0, kTcColS0 = 64, kTcColS1 = 80, kTcColOh = 96, kTcColOl = 112;
constexpr int kTcN = 16;                      // MMA N: query heads of the group, zero-padded

// Shared memory of one CTA (dynamic): this struct, then the code stage of
// TcStage<B>::kChunks chunks of 128 x 16 bytes (chunk i of position p at
// i * 2048 + p * 16: a thread's accesses are 16 bytes apart from its
// neighbours', free of bank conflicts).  Every format needs more than 64 KB in
// all, so at most three CTAs share an SM and their tensor memory (3 x 128
// columns) fits the SM's 512.
struct TcShared {
  uint8_t v[kTcD * kTcTile * 2];  // V^T operand: (d/8) * 2048 + p * 16 + (d%8) * 2
  uint8_t p_hi[kTcN * kTcTile * 2];  // P^T operand: (n/8) * 2048 + p * 16 + (n%8) * 2
  uint8_t p_lo[kTcN * kTcTile * 2];
  uint8_t q[kTcN * kTcD * 2];     // Q operand (K-major): (n/8) * 2048 + (k/8) * 128 + (n%8) * 16 + (k%8) * 2
  float wmax[4][kAttnMaxGroup];
  float wsum[4][kAttnMaxGroup];
  uint64_t bar_kv, bar_p, bar_s, bar_o;
  uint32_t tmem;
  volatile int abort;
  int seqlen[256];
  int items[257];                 // running item counts (compact enumeration), then the total
};


// Instruction descriptor of tcgen05.mma kind::f16: binary16 A and B, binary32
// accumulator, M x N, A / B K-major (0) or MN-major (1).
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor, no swizzle: 8 x 16-byte core matrices,
// `lbo` bytes between core matrices along the leading dimension, `sbo` along
// the strided one.
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&f)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(r[i]);
}

// Wait for the phase with the given parity, the thread suspended in hardware
// between checks (up to 2 us at a time) instead of spinning; gives up like
// mbar_wait (abort flag, or 1 s, then KVQ_DEV_TIMEOUT).
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  uint32_t done;
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
    asm volatile(
        "{\n"
        "  .reg .pred p;\n"
        "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        "  selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(2000u)
        : "memory");
    if (done) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      record_error(KVQ_DEV_TIMEOUT);
      return false;
    }
  }
}

// Warp-wide maximum of a binary32 value (order-preserving integer key).
__device__ __forceinline__ float warp_max_f32(float x) {
  const int b = __float_as_int(x);
  int key = b >= 0 ? b : b ^ 0x7FFFFFFF;
  key = __reduce_max_sync(0xFFFFFFFFu, key);
  return __int_as_float(key >= 0 ? key : key ^ 0x7FFFFFFF);
}

// ---------------------------------------------------------------------------
// Per-format unpacking of one 8-element chunk of a row into four binary16
// pairs (code - z) * s, in MMA order.  kPerm: chunk order is perm8.
// ---------------------------------------------------------------------------
template <int B>
struct TcFmt;

template <>
struct TcFmt<4> {
  static constexpr bool kPerm = true;
  static constexpr bool kScaled = true;
  static constexpr int kRowBytes = kTcD / 2;
  __device__ static uint4 chunk(const uint32_t* w, int j, __half2 s2) {
    const uint32_t x = w[j], y = x >> 8;
    uint4 r;
    r.x = scale_pair(minus_z<8>((x & 0x000F000Fu) | 0x64006400u), s2);
    r.y = scale_pair(minus_z_x16<8>((x & 0x00F000F0u) | 0x64006400u), s2);
    r.z = scale_pair(minus_z<8>((y & 0x000F000Fu) | 0x64006400u), s2);
    r.w = scale_pair(minus_z_x16<8>((y & 0x00F000F0u) | 0x64006400u), s2);
    return r;
  }
};

template <>
struct TcFmt<6> {
  static constexpr bool kPerm = true;
  static constexpr bool kScaled = true;
  static constexpr int kRowBytes = kTcD * 6 / 8;
  __device__ static uint4 chunk(const uint32_t* w, int j, __half2 s2) {
    const int g = j >> 1, h = j & 1;
    uint32_t r[4];
    AttnCodec<6>::raw8_at(w[3 * g + h], w[3 * g + h + 1], 2u * h, r);
    return make_uint4(scale_pair(minus_z<32>(r[0]), s2), scale_pair(minus_z<32>(r[1]), s2),
                      scale_pair(minus_z<32>(r[2]), s2), scale_pair(minus_z<32>(r[3]), s2));
  }
};

template <>
struct TcFmt<8> {
  static constexpr bool kPerm = false;
  static constexpr bool kScaled = true;
  static constexpr int kRowBytes = kTcD;
  __device__ static uint4 chunk(const uint32_t* w, int j, __half2 s2) {
    const uint32_t a = w[2 * j], b = w[2 * j + 1];
    return make_uint4(scale_pair(minus_z<128>(__byte_perm(a, 0x64646464u, 0x5140)), s2),
                      scale_pair(minus_z<128>(__byte_perm(a, 0x64646464u, 0x7362)), s2),
                      scale_pair(minus_z<128>(__byte_perm(b, 0x64646464u, 0x5140)), s2),
                      scale_pair(minus_z<128>(__byte_perm(b, 0x64646464u, 0x7362)), s2));
  }
};

template <>
struct TcFmt<0> {  // E5M2 bytes: the high byte of the binary16 value
  static constexpr bool kPerm = false;
  static constexpr bool kScaled = false;
  static constexpr int kRowBytes = kTcD;
  __device__ static uint4 chunk(const uint32_t* w, int j, __half2) {
    const uint32_t a = w[2 * j], b = w[2 * j + 1];
    return make_uint4(__byte_perm(a, 0u, 0x1404), __byte_perm(a, 0u, 0x3424), __byte_perm(b, 0u, 0x1404),
                      __byte_perm(b, 0u, 0x3424));
  }
};

// head_dim element held at position i (0..7) of an 8-element chunk.
template <bool kPerm>
__host__ __device__ constexpr int tc_perm8(int i) {
  return kPerm ? (i >> 1) + 4 * (i & 1) : i;
}

// The code stage: K row chunks, V row chunks, then one chunk with the K
// scales (bytes 0..7) and the V scales (bytes 8..15).
template <int B>
struct TcStage {
  static constexpr int kRowChunks = TcFmt<B>::kRowBytes / 16;
  static constexpr int kK = 0, kV = kRowChunks, kS = 2 * kRowChunks;
  static constexpr int kChunks = 2 * kRowChunks + (TcFmt<B>::kScaled ? 1 : 0);
  static constexpr int kBytes = kChunks * kTcTile * 16;
};

template <int B>
constexpr int tc_smem_bytes() {
  return static_cast<int>((sizeof(TcShared) + 127) / 128 * 128) + TcStage<B>::kBytes;
}

// Copy position p's K row and K scales (or V row and V scales) of cache row hr
// into the stage.
template <int B, bool kValues>
__device__ __forceinline__ void tc_stage_row(const AttnParams& a, long long hr, uint8_t* stage, int p) {
  using S = TcStage<B>;
  const uint8_t* src = (kValues ? a.v_codes : a.k_codes) + hr * TcFmt<B>::kRowBytes;
  uint8_t* dst = stage + (kValues ? S::kV : S::kK) * (kTcTile * 16) + p * 16;
#pragma unroll
  for (int i = 0; i < S::kRowChunks; ++i) cp_async16(dst + i * (kTcTile * 16), src + i * 16);
  if constexpr (TcFmt<B>::kScaled)
    cp_async_small<8>(stage + S::kS * (kTcTile * 16) + p * 16 + (kValues ? 8 : 0),
                      (kValues ? a.v_scales : a.k_scales) + hr * (kTcD / 32));
}

// Position p's K (or V) row words and its four scales from the stage.
template <int B, bool kValues>
__device__ __forceinline__ void tc_read_row(const uint8_t* stage, int p, uint32_t (&w)[TcFmt<B>::kRowBytes / 4],
                                            uint2& sc) {
  using S = TcStage<B>;
  const uint8_t* src = stage + (kValues ? S::kV : S::kK) * (kTcTile * 16) + p * 16;
#pragma unroll
  for (int i = 0; i < S::kRowChunks; ++i) {
    const uint4 x = *reinterpret_cast<const uint4*>(src + i * (kTcTile * 16));
    w[4 * i] = x.x, w[4 * i + 1] = x.y, w[4 * i + 2] = x.z, w[4 * i + 3] = x.w;
  }
  if constexpr (TcFmt<B>::kScaled)
    sc = *reinterpret_cast<const uint2*>(stage + S::kS * (kTcTile * 16) + p * 16 + (kValues ? 8 : 0));
}

__device__ __forceinline__ __half2 tc_scale2(uint2 s, int blk) {
  const uint32_t w = blk < 2 ? s.x : s.y;
  const __half h = __ushort_as_half(static_cast<unsigned short>((blk & 1) ? (w >> 16) : (w & 0xFFFFu)));
  return __halves2half2(h, h);
}

// One tile of one work item, as every role walks them.
struct TcTile {
  int item;   // compact item index, -1 past the end
  int seq, chunk, kvh;
  int t;      // tile within the item (0 or 1)
  int p0;     // first position of the tile in the sequence
  int n;      // positions of the tile that hold data (1..128)
  bool last;  // last tile of its item
};

struct TcWalk {
  const AttnParams& a;
  const TcShared& sh;
  __device__ int length(int seq) const {
    long long L = sh.seqlen[seq];
    if (L < 0) L = 0;
    const long long m =
        a.page_size == 0 ? static_cast<long long>(a.dim1) : static_cast<long long>(a.max_chunks) * kTcItem;
    return static_cast<int>(L > m ? m : L);
  }
  __device__ TcTile first(int item) const {
    TcTile c;
    if (item >= sh.items[a.batch]) {
      c.item = -1;
      return c;
    }
    int lo = 0, hi = a.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sh.items[mid] > item) hi = mid;
      else lo = mid + 1;
    }
    const unsigned r = static_cast<unsigned>(item - (lo ? sh.items[lo - 1] : 0));
    const unsigned ch = r / static_cast<unsigned>(a.kv_heads);
    c.item = item;
    c.seq = lo;
    c.chunk = static_cast<int>(ch);
    c.kvh = static_cast<int>(r - ch * static_cast<unsigned>(a.kv_heads));
    c.t = 0;
    set(c);
    return c;
  }
  __device__ void set(TcTile& c) const {
    const int L = length(c.seq);
    const int in_item = min(L - c.chunk * kTcItem, kTcItem);
    c.p0 = c.chunk * kTcItem + c.t * kTcTile;
    c.n = min(in_item - c.t * kTcTile, kTcTile);
    c.last = in_item <= (c.t + 1) * kTcTile;
  }
  __device__ TcTile next(const TcTile& c) const {
    if (c.last) return first(c.item + static_cast<int>(gridDim.x));
    TcTile d = c;
    d.t += 1;
    set(d);
    return d;
  }
};

// Cache row (position * kv_heads + kv head) of position `pos` of sequence
// `seq`, or -1 (bad paging metadata, recorded).
__device__ __forceinline__ long long tc_cache_row(const AttnParams& a, int seq, int kvh, int pos) {
  long long row;
  if (a.page_size == 0) {
    row = static_cast<long long>(seq) * a.dim1 + pos;
  } else {
    const int lp = pos / a.page_size;
    const int page = lp < a.bt_stride ? a.block_table[static_cast<long long>(seq) * a.bt_stride + lp] : -1;
    if (page < 0 || page >= a.dim0) {
      record_error(KVQ_DEV_BAD_PAGE);
      return -1;
    }
    row = static_cast<long long>(page) * a.page_size + (pos - lp * a.page_size);
  }
  return row * a.kv_heads + kvh;
}

template <int B, int G>
__global__ void __launch_bounds__(kTcThreads, 3) attn_tc_kernel(const __grid_constant__ AttnParams a) {
  using F = TcFmt<B>;
  constexpr bool kPerm = F::kPerm;
  extern __shared__ __align__(16) uint8_t tc_smem_raw[];
  TcShared& sh = *reinterpret_cast<TcShared*>(tc_smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  static_assert(G >= 1 && G <= kAttnMaxGroup, "query heads per kv head");

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sh.tmem)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(&sh.bar_kv, kTcMathThreads);
    mbar_init(&sh.bar_p, kTcMathThreads);
    mbar_init(&sh.bar_s, 1);
    mbar_init(&sh.bar_o, 1);
    sh.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // query rows >= group and the weight rows of heads 8..15 stay zero
  for (int i = tid; i < kTcN * kTcD * 2 / 16; i += kTcThreads) reinterpret_cast<uint4*>(sh.q)[i] = make_uint4(0, 0, 0, 0);
  for (int i = tid; i < kTcN * kTcTile * 2 / 16; i += kTcThreads) {
    reinterpret_cast<uint4*>(sh.p_hi)[i] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(sh.p_lo)[i] = make_uint4(0, 0, 0, 0);
  }

  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the batch's lengths and running item counts (the launch guarantees batch <= 256
  // and an item total that fits an int)
  for (int i = tid; i < a.batch; i += kTcThreads) sh.seqlen[i] = a.seqlens[i];
  __syncthreads();
  const TcWalk walk{a, sh};
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < a.batch; base += 32) {
      const int i = base + lane;
      int n = i < a.batch ? (walk.length(i) + kTcItem - 1) / kTcItem * a.kv_heads : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, n, o);
        if (lane >= o) n += t;
      }
      n += run;
      if (i < a.batch) sh.items[i] = n;
      run = __shfl_sync(0xFFFFFFFFu, n, 31);
    }
    if (lane == 0) sh.items[a.batch] = run;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the zeroed operands
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;
  uint32_t tiles_done = 0;  // tiles this CTA has processed: the phase of all four barriers

  {
    // ---------------- every thread: one position, one output row ----------------
    const int p = tid;  // position within the tile; output row (tensor-memory lane) of O^T
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int d_out = (p & ~7) + tc_perm8<kPerm>(p & 7);  // head_dim element of this thread's O^T row
    float m_ref[kAttnMaxGroup], l_part[kAttnMaxGroup], acc[kAttnMaxGroup], alpha_prev[kAttnMaxGroup];
#pragma unroll
    for (int g = 0; g < kAttnMaxGroup; ++g) m_ref[g] = -INFINITY, l_part[g] = 0.0f, acc[g] = 0.0f, alpha_prev[g] = 1.0f;
    // fold the previous tile's O^T row into the accumulators (after its MMAs completed)
    auto fold_o = [&](bool ok) {
      float o[16], ol[16];
      tc_ld16(tmem + lane_base + kTcColOh, o);
      tc_ld16(tmem + lane_base + kTcColOl, ol);
#pragma unroll
      for (int g = 0; g < kAttnMaxGroup; ++g) o[g] += ol[g];
#pragma unroll
      for (int g = 0; g < kAttnMaxGroup; ++g)
        if (g < G) acc[g] = acc[g] * alpha_prev[g] + (ok ? o[g] : 0.0f);
    };
    // the item's (max, sum, accumulator) per head into its workspace entry, then a fresh state
    auto finish_item = [&](const TcTile& it) {
#pragma unroll
      for (int g = 0; g < kAttnMaxGroup; ++g) {
        if (g >= G) break;
        float x = l_part[g];
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o2);
        if (lane == 0) sh.wsum[warp][g] = x;
      }
      asm volatile("bar.sync 3, %0;" ::"n"(kTcMathThreads) : "memory");
      const long long head0 = static_cast<long long>(it.seq) * a.n_heads + static_cast<long long>(it.kvh) * G;
      const long long stride = static_cast<long long>(a.max_chunks) * (kTcD + 2);
      float* const entry = a.ws + (head0 * a.max_chunks + it.chunk) * (kTcD + 2);
#pragma unroll
      for (int g = 0; g < kAttnMaxGroup; ++g) {
        if (g >= G) break;
        entry[g * stride + 2 + d_out] = acc[g];
        if (p == 0) {
          entry[g * stride] = m_ref[g];
          entry[g * stride + 1] = sh.wsum[0][g] + sh.wsum[1][g] + sh.wsum[2][g] + sh.wsum[3][g];
        }
      }
#pragma unroll
      for (int g = 0; g < kAttnMaxGroup; ++g) m_ref[g] = -INFINITY, l_part[g] = 0.0f, acc[g] = 0.0f;
    };

    uint8_t* const stage = tc_smem_raw + (sizeof(TcShared) + 127) / 128 * 128;
    // the MMAs (thread 0): S^T = K Q^T once every thread's K row is in tensor memory,
    // O^T = V^T P^T once every thread's V row and weights are in shared memory
    const uint32_t idesc_s = tc_idesc(128, kTcN, 0, 0);
    const uint32_t idesc_o = tc_idesc(128, kTcN, 1, 1);
    const uint64_t q_desc = tc_sdesc(smem_addr(sh.q), 128, 2048);
    const uint64_t v_desc = tc_sdesc(smem_addr(sh.v), 128, 2048);
    const uint64_t hi_desc = tc_sdesc(smem_addr(sh.p_hi), 128, 2048);
    const uint64_t lo_desc = tc_sdesc(smem_addr(sh.p_lo), 128, 2048);
    auto issue_s = [&](uint32_t ph) {
      if (tc_wait(&sh.bar_kv, ph, &sh.abort)) {
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < kTcD / 32; ++s) {
          tc_mma_ts(tmem + kTcColS0, tmem + kTcColK + 8 * s, q_desc + 16 * s, idesc_s, s > 0);
          tc_mma_ts(tmem + kTcColS1, tmem + kTcColK + 32 + 8 * s, q_desc + 64 + 16 * s, idesc_s, s > 0);
        }
      }
      tc_commit(&sh.bar_s);  // arrives once the MMAs above (if any) are done
    };
    auto issue_o = [&](uint32_t ph) {
      if (tc_wait(&sh.bar_p, ph, &sh.abort)) {
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < kTcTile / 16; ++s) {
          tc_mma_ss(tmem + kTcColOh, v_desc + 16 * s, hi_desc + 16 * s, idesc_o, s > 0);
          tc_mma_ss(tmem + kTcColOl, v_desc + 16 * s, lo_desc + 16 * s, idesc_o, s > 0);
        }
      }
      tc_commit(&sh.bar_o);
    };
    TcTile cur = walk.first(blockIdx.x);
    TcTile prev;
    prev.item = -1;
    long long hr_cur = -1;
    if (cur.item >= 0 && p < cur.n) hr_cur = tc_cache_row(a, cur.seq, cur.kvh, cur.p0 + p);
    if (hr_cur >= 0) tc_stage_row<B, false>(a, hr_cur, stage, p);
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (hr_cur >= 0) tc_stage_row<B, true>(a, hr_cur, stage, p);
    asm volatile("cp.async.commit_group;" ::: "memory");
    // Copy groups of this thread, oldest first: ..., K(t), V(t), K(t+1), V(t+1).  At
    // the start of tile t the two youngest are K(t), V(t) (or K(t), V(t) of the first
    // tile): waiting for all but one lands K(t).
    for (; cur.item >= 0; ++tiles_done) {
      const uint32_t ph = tiles_done & 1u;
      const TcTile nxt = walk.next(cur);
      long long hr_nxt = -1;
      if (nxt.item >= 0 && p < nxt.n) hr_nxt = tc_cache_row(a, nxt.seq, nxt.kvh, nxt.p0 + p);
      const bool valid = hr_cur >= 0;
      // a new item: its query rows (perm8 order within each 8 elements), rows < group
      if (cur.t == 0) {
        if (cur.chunk == 0 && cur.kvh == 0 && p == 0 &&
            static_cast<long long>(sh.seqlen[cur.seq]) > walk.length(cur.seq))
          record_error(KVQ_DEV_BAD_PAGE_INDEX);  // window longer than the cache
        const int g = p >> 4, j = p & 15;
        if (g < G) {
          const uint4 x = *reinterpret_cast<const uint4*>(
              a.q + (static_cast<long long>(cur.seq) * a.n_heads + static_cast<long long>(cur.kvh) * G + g) * kTcD +
              8 * j);
          const uint4 y = kPerm ? make_uint4(__byte_perm(x.x, x.z, 0x5410), __byte_perm(x.x, x.z, 0x7632),
                                             __byte_perm(x.y, x.w, 0x5410), __byte_perm(x.y, x.w, 0x7632))
                                : x;
          *reinterpret_cast<uint4*>(sh.q + (g >> 3) * 2048 + j * 128 + (g & 7) * 16) = y;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      // K row -> tensor memory (the S MMAs of the previous tile are complete)
      asm volatile("cp.async.wait_group 1;" ::: "memory");
      {
        uint32_t w[F::kRowBytes / 4];
        uint2 sc = make_uint2(0, 0);
        tc_read_row<B, false>(stage, p, w, sc);
#pragma unroll
        for (int blk = 0; blk < kTcD / 32; ++blk) {
          const __half2 s2 = F::kScaled ? tc_scale2(sc, blk) : __half2();
          uint32_t r[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 u = F::chunk(w, 4 * blk + c, s2);
            r[4 * c] = u.x, r[4 * c + 1] = u.y, r[4 * c + 2] = u.z, r[4 * c + 3] = u.w;
          }
          tc_st16(tmem + lane_base + kTcColK + 16 * blk, r);
        }
        // every word of the staged K row has been used: its slots take the next tile's K codes
        if (hr_nxt >= 0) tc_stage_row<B, false>(a, hr_nxt, stage, p);
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&sh.bar_kv);
      if (tid == 0) issue_s(ph);
      // the previous tile's O^T: fold it in, finish its item when it was the last
      if (prev.item >= 0) {
        const bool ok = tc_wait(&sh.bar_o, ph ^ 1u, &sh.abort);
        tc_fence_after();
        fold_o(ok);
        if (prev.last) finish_item(prev);
      }
      // V row -> shared memory (the O^T MMAs of the previous tile are complete)
      asm volatile("cp.async.wait_group 1;" ::: "memory");
      {
        uint32_t w[F::kRowBytes / 4];
        uint2 sc = make_uint2(0, 0);
        tc_read_row<B, true>(stage, p, w, sc);
#pragma unroll
        for (int j = 0; j < kTcD / 8; ++j) {
          const __half2 s2 = F::kScaled ? tc_scale2(sc, j >> 2) : __half2();
          const uint4 u = valid ? F::chunk(w, j, s2) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(sh.v + j * 2048 + p * 16) = u;
        }
        if (hr_nxt >= 0) tc_stage_row<B, true>(a, hr_nxt, stage, p);
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      // scores of this tile
      const bool ok_s = tc_wait(&sh.bar_s, ph, &sh.abort);
      tc_fence_after();
      float s[16], s1[16];
      tc_ld16(tmem + lane_base + kTcColS0, s);
      tc_ld16(tmem + lane_base + kTcColS1, s1);
#pragma unroll
      for (int g = 0; g < kAttnMaxGroup; ++g) s[g] += s1[g];
      float x[kAttnMaxGroup];
#pragma unroll
      for (int g = 0; g < kAttnMaxGroup; ++g) {
        x[g] = (valid && ok_s) ? s[g] * a.scale_log2 : -INFINITY;
        if (g < G) {
          const float wm = warp_max_f32(x[g]);
          if (lane == 0) sh.wmax[warp][g] = wm;
        }
      }
      asm volatile("bar.sync 3, %0;" ::"n"(kTcMathThreads) : "memory");
      uint32_t hi[kAttnMaxGroup / 2], lo[kAttnMaxGroup / 2];
#pragma unroll
      for (int g = 0; g < kAttnMaxGroup; g += 2) {
        float pw[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = g + e;
          pw[e] = 0.0f;
          if (h >= G) continue;  // heads past the group: zero weights
          const float mt = fmaxf(fmaxf(sh.wmax[0][h], sh.wmax[1][h]), fmaxf(sh.wmax[2][h], sh.wmax[3][h]));
          float al = 1.0f;
          if (mt > m_ref[h] + kAttnRescaleLog2) {
            al = (m_ref[h] == -INFINITY) ? 0.0f : exp2_approx(m_ref[h] - mt);
            m_ref[h] = mt;
          }
          alpha_prev[h] = al;
          pw[e] = (x[h] == -INFINITY) ? 0.0f : exp2_approx(x[h] - m_ref[h]);
          l_part[h] = l_part[h] * al + pw[e];
        }
        hi[g / 2] = pack_half2(pw[0], pw[1]);
        const float2 f = __half22float2(as_h2(hi[g / 2]));
        lo[g / 2] = pack_half2(pw[0] - f.x, pw[1] - f.y);
      }
      *reinterpret_cast<uint4*>(sh.p_hi + p * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(sh.p_lo + p * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&sh.bar_p);
      if (tid == 0) issue_o(ph);
      prev = cur;
      cur = nxt;
      hr_cur = hr_nxt;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // the last tile's O^T
    if (prev.item >= 0) {
      const bool ok = tc_wait(&sh.bar_o, (tiles_done & 1u) ^ 1u, &sh.abort);
      tc_fence_after();
      fold_o(ok);
      finish_item(prev);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
  }
}

}  // namespace kvq
