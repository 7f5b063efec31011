// ldg_engine.cuh -- the plain-load engine: one tile per CTA, every thread
// issues its 16-byte (or 8/4-byte) global loads for the whole tile before it
// computes.  Grid: x = tiles of a sequence's window, y = sequences, z = K / V.
#pragma once

#include "ops.cuh"

namespace kvq {

// CTA size, loads in flight per thread, the occupancy the register budget is
// sized for, and elements per load unit, per operation.
template <class Op>
struct LdgCfg;
template <>
struct LdgCfg<Fp8Encode> {
  static constexpr int kThreads = 128, kUnroll = 8, kMinBlocksPerSM = 8, kUnitElems = 8;
};
template <>
struct LdgCfg<Fp8Decode> {
  static constexpr int kThreads = 128, kUnroll = 8, kMinBlocksPerSM = 8, kUnitElems = 8;
};
template <int B>
struct LdgCfg<QEncode<B>> {
  static constexpr int kThreads = 256, kUnroll = 2, kMinBlocksPerSM = 4, kUnitElems = kBlockElems;
};
template <int B>
struct LdgCfg<QDecode<B>> {
  static constexpr int kThreads = 256, kUnroll = 4, kMinBlocksPerSM = 5, kUnitElems = 8;
};

template <class Op>
constexpr int ldg_tile_elems() {
  return LdgCfg<Op>::kThreads * LdgCfg<Op>::kUnroll * LdgCfg<Op>::kUnitElems;
}

template <class Op>
__global__ void __launch_bounds__(LdgCfg<Op>::kThreads, LdgCfg<Op>::kMinBlocksPerSM)
    convert_kernel(const __grid_constant__ Params p) {
  using C = LdgCfg<Op>;
  // Programmatic dependent launch: this grid may be launched while the
  // previous kernel on the stream is still running; wait for it to finish (and
  // its writes to become visible) before touching global memory, and let the
  // next kernel start launching as soon as every CTA of this grid has started.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int s_bt[C::kThreads];
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
      Op::template body<GlobalSrc, C::kThreads, C::kUnroll>(p, kv, row0, nrows, in, threadIdx.x);
    }
  }
}

}  // namespace kvq
