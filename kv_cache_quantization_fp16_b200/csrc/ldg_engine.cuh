// ldg_engine.cuh -- the plain-load engine: one tile per CTA, every thread
// issues its 16-byte (or 8/4-byte) global loads for the whole tile before it
// computes.  Grid: x = tiles of a sequence's window, y = sequences, z = K / V.
#pragma once

#include "ops.cuh"

namespace kvq {

// CTA size, loads in flight per thread, the occupancy the register budget is
// sized for, elements per load unit, and whether the rounds of a paged tile
// prefetch their successor into L2, per operation.
template <class Op>
struct LdgCfg;
template <>
struct LdgCfg<Fp8Encode> {
  static constexpr int kThreads = 128, kUnroll = 8, kMinBlocksPerSM = 8, kUnitElems = 8;
  static constexpr bool kPrefetchRounds = false;  // measured: slower on paged prefill
};
template <>
struct LdgCfg<Fp8Decode> {  // measured: 4 loads x 12 CTAs beat 8 x 8 (headline decode alone 0.84 -> 0.93)
  static constexpr int kThreads = 128, kUnroll = 4, kMinBlocksPerSM = 12, kUnitElems = 8;
  static constexpr bool kPrefetchRounds = false;  // measured: slower on paged prefill
};
template <int B>
struct LdgCfg<QEncode<B>> {
  // measured: 128-thread CTAs, 8 per SM, beat 256 x 4 (paged Q4 prefill quantize 0.77 -> 0.81)
  static constexpr int kThreads = 128, kUnroll = 2, kMinBlocksPerSM = 8, kUnitElems = kBlockElems;
  static constexpr bool kPrefetchRounds = false;  // measured: no gain
};
template <int B>
struct LdgCfg<QDecode<B>> {
  // measured: 128 x 8 loads x 8 CTAs/SM beat 256 x 4 x 5 on the paged Q4 prefill (0.79 -> 0.82)
  static constexpr int kThreads = 128, kUnroll = 8, kMinBlocksPerSM = 8, kUnitElems = 8;
  static constexpr bool kPrefetchRounds = true;  // measured: paged Q6 dequantize 0.86 -> 0.97 of peak
};

template <class Op>
constexpr int ldg_tile_elems() {
  return LdgCfg<Op>::kThreads * LdgCfg<Op>::kUnroll * LdgCfg<Op>::kUnitElems;
}

// Ask L2 for the input bytes of this CTA's first round of loads before
// waiting on the previous grid, so that this grid's DRAM reads start while the
// previous one drains.  Only CTAs of the first wave (those that can be
// resident before the previous grid ends) do it; later CTAs start after it
// has finished anyway.  A prefetch only fills L2, which is also where every
// write of the previous grid lands, so it can never make a later load see
// stale data.  Paged tiles need the sequence length and the block-table
// entry: warp 0 reads them at L2 (bypassing L1, which other SMs' writes do
// not refresh), and since they may be stale they only steer the hint; the
// page index is range checked, so every prefetched address lies inside the
// cache.
template <class Op, bool kPaged>
__device__ __forceinline__ void prefetch_first_round(const Params& p, int kv) {
  using C = LdgCfg<Op>;
  const long long cta =
      blockIdx.x + static_cast<long long>(gridDim.x) * (blockIdx.y + static_cast<long long>(gridDim.y) * blockIdx.z);
  const int seq = blockIdx.y;
  if (cta >= p.prefetch_ctas || seq >= p.g.batch) return;
  long long row0 = 0;
  int nrows = 0;
  int tid = threadIdx.x, nthreads = C::kThreads;
  if (!kPaged) {
    if (!contiguous_tile(p.g, seq, blockIdx.x, row0, nrows)) return;
  } else {
    if (threadIdx.x >= 32) return;
    nthreads = 32;
    if (!paged_tile(p.g, seq, blockIdx.x, __ldcg(p.g.seqlens + seq), nullptr, false, row0, nrows, true)) return;
  }
  const long long elems = min(static_cast<long long>(nrows) * p.g.hd, static_cast<long long>(ldg_tile_elems<Op>()));
  prefetch_l2_range(static_cast<const uint8_t*>(p.in[kv]) + row0 * p.g.hd * Op::kInNum / Op::kInDen,
                    elems * Op::kInNum / Op::kInDen, tid, nthreads);
  if (Op::kReadsScales)
    prefetch_l2_range(static_cast<const __half*>(p.scales[kv]) + row0 * p.g.hd / kBlockElems,
                      elems / kBlockElems * 2, tid, nthreads);
}

// One instantiation per mode: contiguous grids carry no paging code at all.
template <class Op, bool kPaged>
__global__ void __launch_bounds__(LdgCfg<Op>::kThreads, LdgCfg<Op>::kMinBlocksPerSM)
    convert_kernel(const __grid_constant__ Params p) {
  using C = LdgCfg<Op>;
  prefetch_first_round<Op, kPaged>(p, blockIdx.z);
  // Programmatic dependent launch: this grid may be launched while the
  // previous kernel on the stream is still running; wait for it to finish (and
  // its writes to become visible) before loading anything it may have written,
  // and let the next kernel start launching as soon as every CTA of this grid
  // has started.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int s_bt[kPaged ? C::kThreads : 1];
  __shared__ int s_seqlen;
  const int kv = blockIdx.z;
  for (int seq = blockIdx.y; seq < p.g.batch; seq += gridDim.y) {
    long long row0 = 0;
    int nrows = 0;
    bool ok;
    if (!kPaged) {
      ok = contiguous_tile(p.g, seq, blockIdx.x, row0, nrows);
    } else {
      // Stage the sequence's block-table row (when it fits) together with its
      // length, so the page lookup costs one memory round trip, not two.
      const bool staged = p.g.bt_stride <= C::kThreads;
      if (staged && static_cast<int>(threadIdx.x) < p.g.bt_stride)
        s_bt[threadIdx.x] = p.g.block_table[static_cast<long long>(seq) * p.g.bt_stride + threadIdx.x];
      if (threadIdx.x == 0) s_seqlen = p.g.seqlens[seq];
      __syncthreads();
      ok = paged_tile(p.g, seq, blockIdx.x, s_seqlen, staged ? s_bt : nullptr, threadIdx.x == 0, row0, nrows);
      __syncthreads();  // s_bt and s_seqlen are rewritten for the next sequence
    }
    if (ok) {
      const uint8_t* in = static_cast<const uint8_t*>(p.in[kv]) + row0 * p.g.hd * Op::kInNum / Op::kInDen;
      Op::template body<GlobalSrc, C::kThreads, C::kUnroll, kPaged && C::kPrefetchRounds>(p, kv, row0, nrows, in,
                                                                                          threadIdx.x);
    }
  }
}

}  // namespace kvq
