// ep_scan.cuh -- single-pass column scan with decoupled look-back.
//
// Tiles of 128 tokens are numbered in (source rank, token) order by a ticket
// drawn when the CTA starts, so a tile only ever waits on tiles that are
// already running.  Each tile publishes, per column, a 64-bit word
// (flag << 32 | value): flag 1 = the tile's own count, flag 2 = the inclusive
// prefix up to and including the tile.  A tile sums its predecessors' words
// backwards until it meets an inclusive prefix (single-pass prefix scan with
// decoupled look-back, Merrill & Garland 2016).  Every wait is bounded by
// %globaltimer; when the limit runs out the tile reports
// EP_STATUS_WAIT_TIMEOUT and continues with what it has (all stores that use
// the resulting positions are bounds-checked).
#pragma once

#include "ep_common.cuh"

namespace ep {

constexpr int kScanTile = 128;                 // tokens per tile == threads per CTA
constexpr int kScanWarps = kScanTile / 32;

struct ScanHeader {
  uint32_t ticket;  // next tile number
  uint32_t done;    // tiles finished
  uint32_t pad[2];
};

// Workspace: header, then `counters` int32 (rounded to 4), then the
// descriptors [num_tiles][columns] uint64.
__host__ __device__ inline size_t scan_workspace_bytes(long num_tiles, int columns,
                                                       int counters) {
  const size_t head = sizeof(ScanHeader) + static_cast<size_t>((counters + 3) & ~3) * 4;
  const size_t bytes = head + static_cast<size_t>(num_tiles) * columns * sizeof(uint64_t);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

// Returns the exclusive prefix of column `c` before tile `tile`, and publishes
// the tile's inclusive prefix (unless `publish` is false, a debug mode).
__device__ __forceinline__ uint32_t lookback_column(uint64_t *desc, int tile, int columns, int c,
                                                    uint32_t agg, bool publish,
                                                    unsigned long long timeout_ns,
                                                    int32_t *status) {
  uint64_t *mine = desc + static_cast<size_t>(tile) * columns + c;
  if (tile == 0) {
    if (publish) st_relaxed_gpu(mine, (2ull << 32) | agg);
    return 0u;
  }
  if (publish) st_relaxed_gpu(mine, (1ull << 32) | agg);
  uint32_t excl = 0;
  for (int j = tile - 1; j >= 0; --j) {
    const uint64_t *p = desc + static_cast<size_t>(j) * columns + c;
    uint64_t w = ld_relaxed_gpu(p);
    if ((w >> 32) == 0) {
      const uint64_t t0 = globaltimer();
      bool ok = false;
      while (true) {
        __nanosleep(100);
        w = ld_relaxed_gpu(p);
        if ((w >> 32) != 0) {
          ok = true;
          break;
        }
        if (globaltimer() - t0 > timeout_ns) break;
      }
      if (!ok) {
        report(status, EP_STATUS_WAIT_TIMEOUT);
        break;
      }
    }
    excl += static_cast<uint32_t>(w);
    if ((w >> 32) == 2) break;
  }
  if (publish) st_relaxed_gpu(mine, (2ull << 32) | (excl + agg));
  return excl;
}

// Last-CTA election: every CTA calls this once at its end (all threads).
// Returns true in exactly one CTA, after all others have finished their
// global writes (they fence before counting themselves done).
__device__ __forceinline__ bool elect_last_cta(uint32_t *done, uint32_t num_ctas, int *s_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(done, 1u);
    *s_flag = (prev == num_ctas - 1) ? 1 : 0;
  }
  __syncthreads();
  const bool last = *s_flag != 0;
  if (last) __threadfence();
  return last;
}

}  // namespace ep
