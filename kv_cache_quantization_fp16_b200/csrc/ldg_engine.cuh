// ldg_engine.cuh -- the plain-load engine: every thread issues its 16-byte (or
// 8/4-byte) global loads for a whole round before it computes.  Two grids:
// convert_kernel, one tile per CTA (x = tiles of a sequence's window, y =
// sequences, z = K / V); and, in paged mode, convert_balanced_kernel, one
// wave of CTAs that split the flattened windows of all sequences (K, then V)
// into equal ranges of positions.
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

// ---------------------------------------------------------------------------
// Balanced paged grid.  The windows of all sequences (clipped at 0, as
// paged_tile does) are laid end to end, K's and then V's: T positions.  One
// wave of G CTAs walks them in rounds of G units of `unit` positions (one
// round of loads per thread): in round r CTA c converts positions
// [(r G + c) unit, (r G + c + 1) unit), so the CTAs of a round cover one
// contiguous stretch of the caches (as consecutive tiles do), and the last,
// partial round is split into G equal pieces.  Every CTA moves the same bytes
// to within one position, and one wave has no tail.  (Giving each CTA one
// contiguous range instead spread the concurrent accesses over the whole cache
// and measured 15-25% slower.)  Each CTA finds the windows itself: the batch's
// lengths and their running sums are staged in shared memory (no device->host
// sync); a unit is converted in segments that stay inside one page of one
// sequence.
// ---------------------------------------------------------------------------

constexpr int kBalancedMaxBatch = 1024;

struct BalancedShared {
  int pref[kBalancedMaxBatch + 1];  // pref[i] = positions in the windows of sequences < i
  long long lo[kBalancedMaxBatch];  // first position of sequence i's window
  int warp_sum[32];
  int changed;
};

// Window of a paged sequence with length `seqlen`: first position and length.
__device__ __forceinline__ void paged_window(const Geometry& g, int seqlen, long long& lo, int& len) {
  const long long start = static_cast<long long>(seqlen) + g.offset;
  lo = start < 0 ? 0 : start;
  const long long h = start + g.width;
  len = static_cast<int>(h > lo ? h - lo : 0);
}

// Stage the windows of the batch: every thread takes `per` consecutive
// sequences, then a block-wide exclusive scan of the per-thread totals.  With
// `l2_only`, lengths are read at L2 (a hint before the grid dependency wait).
// The host guarantees batch <= kBalancedMaxBatch and batch * width < 2^31.
template <int NT>
__device__ __forceinline__ void stage_windows(const Geometry& g, BalancedShared& sh, bool l2_only) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = NT / 32;
  const int per = (g.batch + NT - 1) / NT;
  int total = 0;
  for (int k = 0; k < per; ++k) {
    const int i = tid * per + k;
    if (i < g.batch) {
      const int L = l2_only ? __ldcg(g.seqlens + i) : g.seqlens[i];
      long long lo;
      int len;
      paged_window(g, L, lo, len);
      sh.lo[i] = lo;
      sh.pref[i] = len;  // lengths for now, running sums below
      total += len;
    }
  }
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh.warp_sum[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += sh.warp_sum[w];
  int run = base + incl - total;  // exclusive prefix of this thread's first sequence
  for (int k = 0; k < per; ++k) {
    const int i = tid * per + k;
    if (i < g.batch) {
      const int len = sh.pref[i];
      sh.pref[i] = run;
      run += len;
    }
  }
  if (tid == NT - 1) {
    int all = 0;
    for (int w = 0; w < kWarps; ++w) all += sh.warp_sum[w];
    sh.pref[g.batch] = all;
  }
  __syncthreads();
}

// The segment of the flattened windows starting at position r (< end): which
// K/V stream, physical first row and positions (within one page of one
// sequence).  Returns false, after recording the error from thread `report`,
// when the block table cannot place it (the segment is skipped).
__device__ __forceinline__ bool balanced_segment(const Geometry& g, const BalancedShared& sh, uint32_t r,
                                                 uint32_t end, int& kv, long long& row0, int& n, bool report,
                                                 bool l2_only = false) {
  // positions count in 32 bits: the host guarantees batch * width < 2^31, and
  // K's and V's windows together stay below 2^32
  const uint32_t total = static_cast<uint32_t>(sh.pref[g.batch]);
  kv = r >= total ? 1 : 0;
  const uint32_t rr = r - (kv ? total : 0u);
  int lo = 0, hi = g.batch - 1;  // the last sequence whose running sum is <= rr
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<uint32_t>(sh.pref[mid]) <= rr) lo = mid;
    else hi = mid - 1;
  }
  const int seq = lo;
  const long long pos = sh.lo[seq] + static_cast<long long>(rr - static_cast<uint32_t>(sh.pref[seq]));
  if (pos >= static_cast<long long>(g.bt_stride) * g.page_size) {
    n = static_cast<int>(min(end - r, static_cast<uint32_t>(sh.pref[seq + 1]) - rr));
    if (report) record_error(KVQ_DEV_BAD_PAGE_INDEX);
    return false;
  }
  const uint32_t p32 = static_cast<uint32_t>(pos);  // < bt_stride * page_size < 2^32
  const uint32_t ps = static_cast<uint32_t>(g.page_size);
  const uint32_t lp = p32 / ps;
  const uint32_t in_page = p32 - lp * ps;
  uint32_t m = end - r;
  m = min(m, static_cast<uint32_t>(sh.pref[seq + 1]) - rr);
  m = min(m, ps - in_page);
  n = static_cast<int>(m);
  const int32_t* entry = g.block_table + static_cast<long long>(seq) * g.bt_stride + lp;
  const int page = l2_only ? __ldcg(entry) : *entry;
  if (page < 0 || page >= g.dim0) {
    if (report) record_error(KVQ_DEV_BAD_PAGE);
    return false;
  }
  row0 = static_cast<long long>(page) * g.page_size + in_page;
  return true;
}

// Piece k of this CTA: unit k of the full rounds (k < R), or its share of the
// last round (k == R); false past the last piece.  Everything is recomputed
// from shared memory, the launch parameters and the block index, so that
// nothing of it stays live across a unit's loads.
__device__ __forceinline__ bool balanced_piece(const BalancedShared& sh, const Geometry& g, int nkv, int unit,
                                               uint32_t k, uint32_t& b, uint32_t& e) {
  const uint32_t T = static_cast<uint32_t>(sh.pref[g.batch]) * static_cast<uint32_t>(nkv);
  const uint32_t G = gridDim.x, c = blockIdx.x;
  const uint32_t GU = G * static_cast<uint32_t>(unit);
  const uint32_t R = T / GU;
  if (k < R) {
    b = k * GU + c * static_cast<uint32_t>(unit);
    e = b + static_cast<uint32_t>(unit);
    return true;
  }
  if (k > R) return false;
  const unsigned long long rem = T - R * GU;
  b = R * GU + static_cast<uint32_t>(c * rem / G);
  e = R * GU + static_cast<uint32_t>((c + 1) * rem / G);
  return true;
}

template <class Op>
__global__ void __launch_bounds__(LdgCfg<Op>::kThreads, LdgCfg<Op>::kMinBlocksPerSM)
    convert_balanced_kernel(const __grid_constant__ Params p, int nkv, int unit) {
  using C = LdgCfg<Op>;
  __shared__ BalancedShared sh;
  const int tid = threadIdx.x;
  // Before the grid dependency wait: the windows from lengths read at L2 (a hint:
  // the previous grid may still be writing), and an L2 prefetch of this CTA's
  // first unit, so that its DRAM reads start under the previous grid's tail.  A
  // prefetch never changes what a later load returns.
  stage_windows<C::kThreads>(p.g, sh, true);
  {
    uint32_t b, e;
    int kv, n;
    long long row0;
    if (balanced_piece(sh, p.g, nkv, unit, 0, b, e) && b < e &&
        balanced_segment(p.g, sh, b, e, kv, row0, n, false, true)) {
      const long long elems = static_cast<long long>(n) * p.g.hd;
      prefetch_l2_range(static_cast<const uint8_t*>(p.in[kv]) + row0 * p.g.hd * Op::kInNum / Op::kInDen,
                        elems * Op::kInNum / Op::kInDen, tid, C::kThreads);
      if (Op::kReadsScales)
        prefetch_l2_range(static_cast<const __half*>(p.scales[kv]) + row0 * p.g.hd / kBlockElems,
                          elems / kBlockElems * 2, tid, C::kThreads);
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // The lengths again, now that the previous grid's writes are visible; stage
  // them anew only if one changed.
  {
    const int per = (p.g.batch + C::kThreads - 1) / C::kThreads;
    int diff = 0;
    for (int k = 0; k < per; ++k) {
      const int i = tid * per + k;
      if (i < p.g.batch) {
        long long lo;
        int len;
        paged_window(p.g, p.g.seqlens[i], lo, len);
        diff |= (lo != sh.lo[i]) || (len != sh.pref[i + 1] - sh.pref[i]);
      }
    }
    if (__syncthreads_or(diff)) stage_windows<C::kThreads>(p.g, sh, false);
  }
  uint32_t b, e;
  for (uint32_t k = 0; balanced_piece(sh, p.g, nkv, unit, k, b, e); ++k) {
    // the piece in segments that stay inside one page of one sequence
    for (uint32_t r = b; r < e;) {
      int kv, n;
      long long row0;
      if (balanced_segment(p.g, sh, r, e, kv, row0, n, tid == 0)) {
        const uint8_t* in = static_cast<const uint8_t*>(p.in[kv]) + row0 * p.g.hd * Op::kInNum / Op::kInDen;
        Op::template body<GlobalSrc, C::kThreads, C::kUnroll, false>(p, kv, row0, n, in, tid);
      }
      r += static_cast<uint32_t>(n);
    }
  }
}

}  // namespace kvq
