// bulk_engine.cuh -- the TMA bulk-copy engine: persistent CTAs, one producer
// warp and eight consumer warps.  The producer's elected lane resolves each
// tile (window clipping, block-table lookup) and moves the tile's main input
// stream into a 4-stage shared-memory ring with one-dimensional
// cp.async.bulk copies (no cluster multicast) that complete on per-stage
// mbarriers; the consumer warps convert from shared memory and store their
// results with ordinary coalesced stores.  Every wait is bounded by a wall
// clock limit; a wait that runs out records KVQ_DEV_TIMEOUT in the device
// error word, stops the CTA's loop, and the producer then waits (again
// bounded) for the copies it issued before the CTA exits.
//
// Requirements checked on the host: the bytes of one position of the input
// stream are a multiple of 16 (so every tile starts 16-byte aligned and has a
// size that is a multiple of 16), and one tile fits a stage.
#pragma once

#include "ops.cuh"

namespace kvq {

constexpr int kBulkStages = 4;
constexpr int kBulkConsumerWarps = 8;
constexpr int kBulkConsumers = 32 * kBulkConsumerWarps;
constexpr int kBulkThreads = kBulkConsumers + 32;
constexpr int kBulkStageBytes = 16384;
constexpr int kBulkTileElems = 8192;  // at most 2 input bytes per element: one stage
constexpr int kBulkSmemBytes = kBulkStages * kBulkStageBytes;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

// Consumer loads in flight per thread (each tile is one round at 8192 elements).
template <class Op>
struct BulkCfg;
template <>
struct BulkCfg<Fp8Encode> { static constexpr int kUnroll = 4; };
template <>
struct BulkCfg<Fp8Decode> { static constexpr int kUnroll = 4; };
template <int B>
struct BulkCfg<QEncode<B>> { static constexpr int kUnroll = 1; };
template <int B>
struct BulkCfg<QDecode<B>> { static constexpr int kUnroll = 4; };

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for the phase with the given parity to complete.  Gives up when
// `abort_flag` is raised by another warp, or after kWaitLimitNs, in which case
// it raises the flag itself and records KVQ_DEV_TIMEOUT.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort_flag && *abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      if (abort_flag) *abort_flag = 1;
      record_error(KVQ_DEV_TIMEOUT);
      return false;
    }
  }
}

// Global -> shared bulk copy completing on `bar` (no multicast).
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Before the grid dependency wait: an L2-only bulk prefetch of the input of
// this CTA's first tile, so that its DRAM reads start while the previous grid
// on the stream drains (every CTA of this persistent grid is in the first
// wave).  The window and page metadata are read at L2 and only steer the hint
// (the previous grid may still be writing them); the page is range checked,
// so the prefetched range lies inside the cache.  Nothing is copied into
// shared memory before the wait, and a prefetch never changes what a later
// load returns.
template <class Op>
__device__ __forceinline__ void bulk_prefetch_first_tile(const Params& p, int tiles_x, long long total) {
  const long long t = blockIdx.x;
  if (t >= total) return;
  const int x = static_cast<int>(t % tiles_x);
  const long long rest = t / tiles_x;
  const int seq = static_cast<int>(rest % p.g.batch);
  const int kv = static_cast<int>(rest / p.g.batch);
  long long row0 = 0;
  int nrows = 0;
  const bool ok = p.g.page_size == 0
                      ? contiguous_tile(p.g, seq, x, row0, nrows)
                      : paged_tile(p.g, seq, x, __ldcg(p.g.seqlens + seq), nullptr, false, row0, nrows, true);
  if (!ok) return;
  const long long in_off = row0 * p.g.hd * Op::kInNum / Op::kInDen;
  const uint32_t bytes = static_cast<uint32_t>(nrows * p.g.hd * Op::kInNum / Op::kInDen);
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(static_cast<const uint8_t*>(p.in[kv]) + in_off),
               "r"(bytes)
               : "memory");
}

template <class Op>
__global__ void __launch_bounds__(kBulkThreads, 1)
    bulk_kernel(const __grid_constant__ Params p, int tiles_x, int nkv) {
  if (threadIdx.x == 0)
    bulk_prefetch_first_tile<Op>(p, tiles_x, static_cast<long long>(tiles_x) * p.g.batch * nkv);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t full_bar[kBulkStages];
  __shared__ __align__(8) uint64_t empty_bar[kBulkStages];
  __shared__ long long meta_row0[kBulkStages];
  __shared__ int meta_nrows[kBulkStages];
  __shared__ int meta_kv[kBulkStages];
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long total = static_cast<long long>(tiles_x) * p.g.batch * nkv;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBulkStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kBulkConsumerWarps);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    if (lane != 0) return;
    // ---- producer ----
    long long it = 0;
    for (long long t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const int s = static_cast<int>(it % kBulkStages);
      if (it >= kBulkStages &&
          !mbar_wait(&empty_bar[s], static_cast<uint32_t>((it / kBulkStages - 1) & 1), &abort_flag))
        break;
      const int x = static_cast<int>(t % tiles_x);
      const long long rest = t / tiles_x;
      const int seq = static_cast<int>(rest % p.g.batch);
      const int kv = static_cast<int>(rest / p.g.batch);
      long long row0 = 0;
      int nrows = 0;
      const bool ok = p.g.page_size == 0
                          ? contiguous_tile(p.g, seq, x, row0, nrows)
                          : paged_tile(p.g, seq, x, p.g.seqlens[seq], nullptr, true, row0, nrows);
      meta_row0[s] = ok ? row0 : -1;
      meta_nrows[s] = nrows;
      meta_kv[s] = kv;
      if (ok) {
        const long long in_off = row0 * p.g.hd * Op::kInNum / Op::kInDen;
        const uint32_t bytes = static_cast<uint32_t>(nrows * p.g.hd * Op::kInNum / Op::kInDen);
        mbar_arrive_expect_tx(&full_bar[s], bytes);
        bulk_copy_g2s(stage_mem + s * kBulkStageBytes, static_cast<const uint8_t*>(p.in[kv]) + in_off, bytes,
                      &full_bar[s]);
      } else {
        mbar_arrive(&full_bar[s]);
      }
    }
    if (abort_flag) {
      // Do not leave while copies into this CTA's shared memory are in flight.
      for (long long j = it - 1; j >= 0 && j >= it - kBulkStages; --j)
        mbar_wait(&full_bar[j % kBulkStages], static_cast<uint32_t>((j / kBulkStages) & 1), nullptr);
    }
    return;
  }

  // ---- consumers ----
  const int ctid = threadIdx.x - 32;
  long long it = 0;
  for (long long t = blockIdx.x; t < total; t += gridDim.x, ++it) {
    const int s = static_cast<int>(it % kBulkStages);
    if (!mbar_wait(&full_bar[s], static_cast<uint32_t>((it / kBulkStages) & 1), &abort_flag)) break;
    const long long row0 = meta_row0[s];
    if (row0 >= 0) {
      Op::template body<SharedSrc, kBulkConsumers, BulkCfg<Op>::kUnroll, false>(p, meta_kv[s], row0, meta_nrows[s],
                                                                           stage_mem + s * kBulkStageBytes, ctid);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }
}

}  // namespace kvq

// ---------------------------------------------------------------------------
// Self-check of the bounded pipeline wait: one thread waits on an mbarrier
// that expects one arrival that never comes; mbar_wait gives up after its
// limit and records KVQ_DEV_TIMEOUT.
// ---------------------------------------------------------------------------

namespace kvq {

__global__ void selfcheck_wait_timeout_kernel(int32_t* waited_out) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  *waited_out = mbar_wait(&bar, 0, nullptr) ? 0 : 1;
}

}  // namespace kvq

extern "C" kvq_status kvq_selfcheck_wait_timeout(int32_t* waited_out, void* stream) {
  if (!waited_out) return KVQ_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(waited_out, 0, sizeof(int32_t), s) != cudaSuccess) return KVQ_ERR_CUDA;
  kvq::selfcheck_wait_timeout_kernel<<<1, 32, 0, s>>>(waited_out);
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}
