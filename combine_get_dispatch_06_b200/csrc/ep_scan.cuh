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
  uint32_t claim;   // work counter of a kernel that runs after the scan
  uint32_t pad;
};

// Workspace: header, then `counters` int32 (rounded to 4), then the
// descriptors [num_tiles][columns] uint64.
__host__ __device__ inline size_t scan_workspace_bytes(long num_tiles, int columns,
                                                       long counters) {
  const size_t head = sizeof(ScanHeader) + static_cast<size_t>((counters + 3) & ~3) * 4;
  const size_t bytes = head + static_cast<size_t>(num_tiles) * columns * sizeof(uint64_t);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

// Publishes the tile's own count of column `c` (an inclusive prefix for tile 0).
__device__ __forceinline__ void publish_aggregate(uint64_t *desc, int tile, int columns, int c,
                                                  uint32_t agg) {
  st_relaxed_gpu(desc + static_cast<size_t>(tile) * columns + c,
                 ((tile == 0 ? 2ull : 1ull) << 32) | agg);
}

// Windowed look-back for column `c` of tile `tile`, run by an aligned group of
// G lanes (G a power of two <= 32; all G lanes call it with the same
// arguments).  Each round the group reads a window of G*U predecessor
// descriptors at once (lane l, slot u -> tile - 1 - (l + G*u)), finds the
// nearest inclusive prefix in it, and adds every value up to that one; if
// the window holds none, it adds all of them and moves on.  A descriptor that
// is not yet published makes the group re-read the window, at most
// `timeout_ns` in total.  Returns the exclusive prefix to every lane of the
// group and publishes the tile's inclusive prefix (lane 0 of the group).
// `agg_published`: the caller has already published the tile's own count
// with publish_aggregate().
template <int G, int U>
__device__ __forceinline__ uint32_t lookback_window(uint64_t *desc, int tile, int columns, int c,
                                                    uint32_t agg, bool publish,
                                                    unsigned long long timeout_ns,
                                                    int32_t *status, bool agg_published = false) {
  static_assert(G >= 1 && G <= 32 && (G & (G - 1)) == 0, "G must be a power of two");
  constexpr int W = G * U;
  const int lane = threadIdx.x & 31;
  const int gl = lane & (G - 1);
  const int gbase = lane & ~(G - 1);
  const uint32_t gmask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << gbase);
  uint64_t *mine = desc + static_cast<size_t>(tile) * columns + c;
  if (tile == 0) {
    if (publish && !agg_published && gl == 0) st_relaxed_gpu(mine, (2ull << 32) | agg);
    return 0u;
  }
  if (publish && !agg_published && gl == 0) st_relaxed_gpu(mine, (1ull << 32) | agg);

  uint32_t excl = 0;
  int base = tile - 1;
  uint64_t t0 = 0;
  bool timed_out = false;
  while (true) {
    uint32_t flag[U], val[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = base - (gl + G * u);
      if (j >= 0) {
        const uint64_t w = ld_relaxed_gpu(desc + static_cast<size_t>(j) * columns + c);
        flag[u] = static_cast<uint32_t>(w >> 32);
        val[u] = static_cast<uint32_t>(w);
      } else {  // before tile 0: an inclusive prefix of 0
        flag[u] = 2u;
        val[u] = 0u;
      }
    }
    // nearest inclusive prefix in the window (position gl + G*u)
    int pstar = W;
#pragma unroll
    for (int u = U - 1; u >= 0; --u)
      if (flag[u] == 2u) pstar = gl + G * u;
#pragma unroll
    for (int o = 1; o < G; o <<= 1) pstar = min(pstar, __shfl_xor_sync(gmask, pstar, o));
    bool missing = false;
    uint32_t sum = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int pos = gl + G * u;
      if (pos <= pstar) {
        missing |= (flag[u] == 0u);
        sum += val[u];
      }
    }
    if (__ballot_sync(gmask, missing) & gmask) {
      const uint64_t now = __shfl_sync(gmask, globaltimer(), gbase);
      if (t0 == 0) t0 = now;
      if (now - t0 > timeout_ns) {
        timed_out = true;
        break;
      }
      __nanosleep(64);
      continue;
    }
#pragma unroll
    for (int o = 1; o < G; o <<= 1) sum += __shfl_xor_sync(gmask, sum, o);
    excl += sum;
    if (pstar < W) break;
    base -= W;
  }
  if (timed_out && gl == 0) report(status, EP_STATUS_WAIT_TIMEOUT);
  if (publish && gl == 0) st_relaxed_gpu(mine, (2ull << 32) | (excl + agg));
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
