// tiles.cuh -- shared geometry of the KV-cache conversions: window and
// page resolution of one tile, kernel parameters, the device error word.
//
// Windows follow the page "Implementation: Turboderp org Exllamav2 Ext
// Cache" (Description: batch_size / offset / width partial updates; paged
// mode through cache_seqlens and block_table): contiguous sequences cover
// [offset, offset + width); paged sequence i covers logical positions
// [max(0, seqlens[i] + offset), seqlens[i] + offset + width), position p in
// page block_table[i][p / page_size] at row p % page_size.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvq.h"

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
// With `l2_only` the block-table entry is read at L2 (bypassing L1).
__device__ __forceinline__ bool paged_tile(const Geometry& g, int seq, int tile_x, int seqlen,
                                           const int* bt_row, bool report, long long& row0, int& nrows,
                                           bool l2_only = false) {
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
  const int32_t* entry = g.block_table + static_cast<long long>(seq) * g.bt_stride + lp;
  const int page = bt_row ? bt_row[lp] : (l2_only ? __ldcg(entry) : *entry);
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
  // CTAs (in launch order) that can be resident while the previous grid on the
  // stream is still draining: only they prefetch before the dependency wait.
  long long prefetch_ctas;
};

}  // namespace kvq
