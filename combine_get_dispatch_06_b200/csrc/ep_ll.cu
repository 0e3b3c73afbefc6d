// ep_ll.cu -- A5 + A6: low-latency dispatch (fused FP8 e4m3 quantisation into
// per-expert slabs) and low-latency combine (top-k weighted gather).
//
// Semantics (DeepEP legacy-test analysis page: low_latency_dispatch with
// use_fp8, its handle (recv_src_info, recv_layout_range), the check that each
// expert's count equals (topk_idx == expert).sum(), and low_latency_combine
// with the check against x * sum of masked weights):
//   - one slab row per (token, expert); rows of expert e ordered by source
//     rank, then token: row = exclusive prefix over the flattened (s, t) order
//     of "token has e", computed here by a tile scan that looks back over the
//     earlier tiles' counts, as in normal dispatch, with experts as columns;
//   - per 128-channel block: amax' = max(max|x|, 1e-4), inv = 448 / amax'
//     (IEEE division), q = e4m3(x * inv) rounded to nearest even and
//     saturated (cvt.rn.satfinite), scale = amax' / 448;
//   - combine: acc = fmaf(y, w_k, acc) over slots k ascending, one bf16
//     rounding at the end.
//
// Kernels (after zero_prefetch clears the workspace words the call uses):
//   ll_scan_kernel      positions, recv_src_info, layout_range, counts, and
//                       a mirror of the positions for the dispatch kernel
//   ll_dispatch_kernel  runs concurrently with the scan; one CTA per token at
//                       a time (tokens claimed from a counter): read the row
//                       once by a bulk copy, quantise it in registers (8
//                       threads per 128-channel block, amax by xor-shuffles)
//                       and store each 16-byte chunk of codes straight to every
//                       destination slab row once the scan has written its
//                       position
//   ll_combine_kernel   one warp per (token, channel segment), up to 8 rows
//                       in flight per lane
// One rank per GPU (ep_shard_ll_*): ll_count_kernel counts the rank's rows
// per expert, shard_ll_prefix_kernel turns every rank's counts into its row
// offsets, its layout_range entries and its experts' receive counts, and the
// three kernels above run in their peer-table forms.
#include <algorithm>

#include "ep_scan.cuh"

namespace ep {
namespace {

// Largest tiles x E for which a tile reads every predecessor's counts at once;
// above it, the windowed decoupled look-back.
constexpr int kLLFullLookback = 16384;

struct LLScanParams {
  const int64_t *topk_idx;
  const int32_t *mask;   // [R], non-zero = failed rank; nullptr = none
  int32_t *stats;        // [E] cumulative received rows, or nullptr
  int R, T, K, E, El, cap, tiles_per_src, num_tiles;
  int32_t *ll_pos;
  int32_t *recv_src_info;
  int32_t *layout_range;
  int32_t *recv_count;
  ScanHeader *head;
  uint64_t *desc;
  int32_t *pos_mirror;  // [R*T][K] ll_pos + 2 (0 = not written yet), for the dispatch kernel
  // One source rank of a sharded job (the call's tokens are rank s0's): rows
  // of each expert that earlier ranks send (base[E]) and the destination
  // ranks' recv_src_info ([R] -> [El][cap]); nullptr and s0 = 0 otherwise.
  // layout_range, recv_count and stats then come from the gathered counts.
  int s0;
  const int32_t *base;
  int32_t *const *rsi_tab;
  int32_t *status;
  unsigned long long timeout_ns;
  unsigned flags;
};

// MAXK: compile-time bound on the top-k slots (8 or 16), chosen per call.
//
// Threads 0..kScanTile-1 hold one token each; the other kScanTile threads
// run the look-back.  As soon as its ids are read, every token thread sets
// its lane's bit in the word of each of its experts (one word per warp and
// expert, shared atomicOr): the popcounts of those words are the tile's rows
// per expert, which the look-back warps publish at once, and a token's rank
// among the warp's tokens with the same expert is the number of lower lanes
// in the word -- token order, whatever slot the expert is in.  Up to
// kLLFullLookback tiles x experts, a tile reads every predecessor's count of
// every expert in one pass (32-bit words, count + 1, 0 = not yet published;
// four experts per 16-byte load where E % 4 == 0; a batch of loads that
// found words not yet published is read again as a whole); above it, the
// windowed decoupled look-back on 64-bit descriptors.
//
// The dispatch kernel that follows runs concurrently with this one: it is
// scheduled once every tile has passed pdl_trigger(), which comes after
// pdl_wait(), so everything before this kernel in the stream is complete by
// then.  It takes each token's slab rows from a mirror of ll_pos in the
// workspace, zeroed before this kernel and written here as ll_pos + 2, so
// that a non-zero word is its own proof of being written.
constexpr int kLLScanThreads = 2 * kScanTile;

// kShard: one rank of a sharded job (p.s0, p.base and p.rsi_tab set).
template <int MAXK, bool kShard>
__global__ void __launch_bounds__(kLLScanThreads, 2) ll_scan_kernel(LLScanParams p) {
  pdl_wait();
  pdl_trigger();  // after the wait: see above
  __shared__ int s_tile;
  __shared__ uint32_t s_lanes[kScanWarps][kMaxExperts];  // lanes of the warp holding expert c
  __shared__ int s_whist[kScanWarps][kMaxExperts];       // rows of expert c in earlier warps
  __shared__ int s_cnt[kMaxExperts];                     // the tile's rows of expert c
  __shared__ int s_excl[kMaxExperts];                    // rows of expert c in earlier tiles
  __shared__ int s_mask[kMaxRanks];  // failed ranks (non-zero), if a mask is given

  const int tid = threadIdx.x;
  const bool tok = tid < kScanTile;  // a token thread (warps 0..kScanWarps-1)
  const int lane = tid & 31;
  const int warp = tid >> 5;
  if (tid == 0) s_tile = static_cast<int>(atomicAdd(&p.head->ticket, 1u));
  // Tiles are usually handed out in block order: the ids of tile blockIdx.x
  // are loaded while the ticket is on its way, and loaded again in the rare
  // case the ticket names another tile.
  auto load_ids = [&](int tl, int64_t (&ids)[MAXK]) {
    const int s_ = tl / p.tiles_per_src;
    const int t_ = (tl % p.tiles_per_src) * kScanTile + tid;
    const size_t st_ = static_cast<size_t>(s_) * p.T + t_;
#pragma unroll
    for (int k = 0; k < MAXK; ++k)
      ids[k] = (t_ < p.T && k < p.K) ? p.topk_idx[st_ * p.K + k] : -1;
  };
  int64_t ids[MAXK];
  if (tok) load_ids(static_cast<int>(blockIdx.x), ids);
  for (int i = tid; i < kScanWarps * kMaxExperts; i += kLLScanThreads) (&s_lanes[0][0])[i] = 0u;
  for (int i = tid; i < p.E; i += kLLScanThreads) {
    s_cnt[i] = 0;
    s_excl[i] = 0;
  }
  if (p.mask != nullptr)
    for (int i = tid; i < p.R; i += kLLScanThreads) s_mask[i] = p.mask[i];
  __syncthreads();

  const int tile = s_tile;
  if (tok && tile != static_cast<int>(blockIdx.x)) load_ids(tile, ids);
  const int s = tile / p.tiles_per_src;  // the call's source index (rank p.s0 + s)
  const int t = (tile % p.tiles_per_src) * kScanTile + tid;
  const bool valid = tok && t < p.T;
  const size_t st = static_cast<size_t>(s) * p.T + t;
  // a failed (masked) source rank sends nothing
  const bool src_ok = p.mask == nullptr || s_mask[(kShard ? p.s0 : 0) + s] == 0;

  // Distinct valid experts of this token (a repeated expert keeps only its
  // first slot in `col`; `ev` keeps every valid id).  Experts on a failed
  // rank are dropped.
  int ev[MAXK], col[MAXK], rnk[MAXK];
  bool bad = false;
#pragma unroll
  for (int k = 0; k < MAXK; ++k) {
    ev[k] = -1;
    col[k] = -1;
    rnk[k] = 0;
    if (valid && k < p.K) {
      const int64_t e = ids[k];
      if (e >= 0 && e < p.E) {
        if (!src_ok || (p.mask != nullptr && s_mask[static_cast<int>(e) / p.El] != 0)) continue;
        ev[k] = static_cast<int>(e);
        bool dup = false;
#pragma unroll
        for (int k2 = 0; k2 < k; ++k2) dup |= (col[k2] == ev[k]);
        if (!dup) {
          col[k] = ev[k];
          atomicOr(&s_lanes[warp][ev[k]], 1u << lane);
        }
      } else if (e != -1) {
        bad = true;
      }
    }
  }
  if (bad) report(p.status, EP_STATUS_BAD_EXPERT);
  __syncthreads();  // every warp's lane words are complete

  const bool publish = (p.flags & EP_DEBUG_SUPPRESS_PUBLISH) == 0;
  const bool full = static_cast<long>(p.num_tiles) * p.E <= kLLFullLookback;
  if (!tok) {
    // ---- look-back warps: publish the tile's counts, then sum the earlier tiles'
    const int lt = tid - kScanTile;
    uint32_t *cnt32 = reinterpret_cast<uint32_t *>(p.desc);  // [num_tiles][E]: rows + 1
    for (int c = lt; c < p.E; c += kScanTile) {
      int n = 0;
#pragma unroll
      for (int w = 0; w < kScanWarps; ++w) n += __popc(s_lanes[w][c]);
      s_cnt[c] = n;
      if (!publish) continue;
      if (full)
        st_relaxed_gpu(reinterpret_cast<int32_t *>(cnt32) + static_cast<size_t>(tile) * p.E + c,
                       n + 1);
      else
        publish_aggregate(p.desc, tile, p.E, c, static_cast<uint32_t>(n));
    }
    if (full) {
      // item i = (predecessor j, group g of cw experts), i = j * G + g; this
      // thread takes i = lt, lt + kScanTile, ... with kB loads in flight,
      // and keeps the sums of one group in registers until the group changes
      const int cw = (p.E & 3) == 0 ? 4 : 1;
      const int G = p.E / cw;
      const int items = tile * G;
      constexpr int kB = 16;
      uint32_t acc[4] = {0u, 0u, 0u, 0u};
      int cur = -1;
      bool timed_out = false;
      auto flush = [&]() {
        if (cur < 0) return;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < cw && acc[q] != 0u) atomicAdd(&s_excl[cur * cw + q], static_cast<int>(acc[q]));
      };
      auto load_item = [&](int i) -> uint4 {
        const int j = i / G, g = i - j * G;
        const uint32_t *a = cnt32 + static_cast<size_t>(j) * p.E + g * cw;
        if (cw == 4) return ld_relaxed_gpu_v4(a);
        return make_uint4(static_cast<uint32_t>(ld_relaxed_gpu(reinterpret_cast<const int32_t *>(a))),
                          1u, 1u, 1u);
      };
      auto unpublished = [](const uint4 &w) {
        return w.x == 0u || w.y == 0u || w.z == 0u || w.w == 0u;
      };
      for (int i0 = lt; i0 < items; i0 += kScanTile * kB) {
        uint4 v[kB];
        uint32_t pend = 0u;  // loads of this batch that found a word not yet published
#pragma unroll
        for (int b = 0; b < kB; ++b) {
          const int i = i0 + b * kScanTile;
          v[b] = i < items ? load_item(i) : make_uint4(1u, 1u, 1u, 1u);
        }
#pragma unroll
        for (int b = 0; b < kB; ++b)
          if (unpublished(v[b])) pend |= 1u << b;
        if (pend != 0u && !timed_out) {
          // read them again, all at once, until every word is there (bounded)
          const uint64_t ts = globaltimer();
          do {
            __nanosleep(64);
#pragma unroll
            for (int b = 0; b < kB; ++b)
              if ((pend >> b) & 1u) v[b] = load_item(i0 + b * kScanTile);
#pragma unroll
            for (int b = 0; b < kB; ++b)
              if (((pend >> b) & 1u) && !unpublished(v[b])) pend &= ~(1u << b);
            if (pend != 0u && globaltimer() - ts > p.timeout_ns) timed_out = true;
          } while (pend != 0u && !timed_out);
        }
#pragma unroll
        for (int b = 0; b < kB; ++b) {
          const int i = i0 + b * kScanTile;
          if (i >= items) break;
          const int g = i % G;
          if (g != cur) {
            flush();
            cur = g;
            acc[0] = acc[1] = acc[2] = acc[3] = 0u;
          }
          acc[0] += v[b].x != 0u ? v[b].x - 1u : 0u;
          acc[1] += v[b].y != 0u ? v[b].y - 1u : 0u;
          acc[2] += v[b].z != 0u ? v[b].z - 1u : 0u;
          acc[3] += v[b].w != 0u ? v[b].w - 1u : 0u;
        }
      }
      flush();
      if (timed_out) report(p.status, EP_STATUS_WAIT_TIMEOUT);
    } else {
      for (int c = lt; c < p.E; c += kScanTile)
        s_excl[c] = static_cast<int>(lookback_window<1, 32>(p.desc, tile, p.E, c,
                                                             static_cast<uint32_t>(s_cnt[c]),
                                                             publish, p.timeout_ns, p.status,
                                                             true));
    }
  } else {
    // ---- token warps: each token's rank among the warp's tokens with its
    // expert, and every expert's rows in the tile's earlier warps
    const uint32_t lt = lanemask_lt();
#pragma unroll
    for (int k = 0; k < MAXK; ++k)
      if (col[k] >= 0) rnk[k] = __popc(s_lanes[warp][col[k]] & lt);
    for (int c = tid; c < p.E; c += kScanTile) {
      int run = 0;
#pragma unroll
      for (int w = 0; w < kScanWarps; ++w) {
        const int n = __popc(s_lanes[w][c]);
        s_whist[w][c] = run;
        run += n;
      }
    }
  }
  __syncthreads();  // s_excl and s_whist are complete

  if (valid) {
    int pos[MAXK];
    bool oob = false;
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
      pos[k] = -1;
      if (col[k] >= 0) {
        const int r = s_excl[col[k]] + s_whist[warp][col[k]] + rnk[k] +
                      (kShard ? p.base[col[k]] : 0);
        if (r >= 0 && r < p.cap)
          pos[k] = r;
        else
          oob = true;  // only reachable after a timed-out look-back
      }
    }
    // a repeated expert's slot takes the row of its first slot
    int v[MAXK];
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
      v[k] = pos[k];
      if (col[k] < 0 && ev[k] >= 0) {
#pragma unroll
        for (int k2 = 0; k2 < MAXK; ++k2)
          if (k2 < k && col[k2] == ev[k]) v[k] = pos[k2];
      }
    }
    // the mirror first (the dispatch kernel waits on it), then ll_pos and
    // recv_src_info; 16 bytes per store where K % 4 == 0 and the row allows
    int32_t *mrow = p.pos_mirror + st * p.K;
    int32_t *prow = p.ll_pos + st * p.K;
    const bool v4m = (p.K & 3) == 0 && (reinterpret_cast<uintptr_t>(mrow) & 15u) == 0;
    const bool v4p = (p.K & 3) == 0 && (reinterpret_cast<uintptr_t>(prow) & 15u) == 0;
#pragma unroll
    for (int k = 0; k < MAXK; k += 4) {
      if (k >= p.K) break;
      if (v4m) {
        st_relaxed_gpu_v4(mrow + k, v[k] + 2, v[k + 1] + 2, v[k + 2] + 2, v[k + 3] + 2);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (k + q < p.K) st_relaxed_gpu(mrow + k + q, v[k + q] + 2);
      }
    }
#pragma unroll
    for (int k = 0; k < MAXK; k += 4) {
      if (k >= p.K) break;
      if (v4p) {
        *reinterpret_cast<int4 *>(prow + k) = make_int4(v[k], v[k + 1], v[k + 2], v[k + 3]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (k + q < p.K) prow[k + q] = v[k + q];
      }
    }
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
      if (pos[k] < 0) continue;
      if constexpr (kShard) {  // the destination's slab handle, in peer memory
        const int d = col[k] / p.El;
        p.rsi_tab[d][static_cast<size_t>(col[k] - d * p.El) * p.cap + pos[k]] = t;
      } else {
        p.recv_src_info[static_cast<size_t>(col[k]) * p.cap + pos[k]] = t;
      }
    }
    if (oob) report(p.status, EP_STATUS_BAD_POSITION);
  }

  if constexpr (kShard) {  // the counts' outputs come from the gathered counts
    __threadfence_system();  // handle entries stored into peers' memory
    return;
  }
  const bool first_of_src = (tile % p.tiles_per_src) == 0;
  for (int c = tid; c < p.E; c += kLLScanThreads) {
    const int run = s_cnt[c];
    const int excl = s_excl[c];
    const size_t o = (static_cast<size_t>(c) * p.R + s) * 2;
    if (first_of_src) p.layout_range[o] = excl;
    // rows source s owns: its only tile stores the count; several tiles add
    // theirs (zeroed on the host)
    if (p.tiles_per_src == 1)
      p.layout_range[o + 1] = run;
    else if (run != 0)
      atomicAdd(&p.layout_range[o + 1], run);
    if (run != 0 && p.stats != nullptr) atomicAdd(&p.stats[c], run);
    if (tile == p.num_tiles - 1) p.recv_count[c] = excl + run;
  }
}

// ---------------------------------------------------------------------------

constexpr int kLLThreads = 256;     // 8 warps quantise one token row together
constexpr int kLLMaxStages = 4;     // input rows in flight per CTA (fewer when H is large)
constexpr int kLLMaxCtasPerSm = 3;
constexpr int kLLMaxDynSmem = 227 * 1024 - 1024;  // the CTA's limit, less its static arrays

__device__ __forceinline__ uint32_t cvt_e4m3x4(float a, float b, float c, float d) {
  // element order in memory: a, b, c, d (a in the lowest byte)
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Shared-memory plan of one CTA: 128 bytes of mbarriers, then `stages` input
// rows (bf16, filled by bulk copies), as many as fit (at most kLLMaxStages,
// at least 2).
struct LLSmem {
  int in_stride;  // bytes per input stage (multiple of 128)
  int stages;     // input stages; 0 if not even 2 fit
  int bytes;      // total
};

__host__ __device__ inline LLSmem ll_smem_plan(int H) {
  LLSmem m;
  m.in_stride = (2 * H + 127) & ~127;
  const long fit = (static_cast<long>(kLLMaxDynSmem) - 128) / m.in_stride;
  m.stages = fit >= 2 ? static_cast<int>(fit < kLLMaxStages ? fit : kLLMaxStages) : 0;
  m.bytes = 128 + m.stages * m.in_stride;
  return m;
}

// One CTA per token at a time.  Tokens are claimed from a shared counter
// (`claim`, zeroed with the workspace), so CTAs that run faster take more of
// them and the grid finishes together.  Thread 0 keeps `stages` claimed rows
// in flight as bulk loads and claims one more token ahead, to hide the
// atomic's round trip.  Warp 0 turns the token's mirrored slab positions into
// one destination row per distinct expert (in shared memory); then every
// thread quantises its 16-channel chunks (8 threads per 128-channel block,
// amax by xor-shuffles) in registers and stores each 16-byte chunk of e4m3
// codes straight to every destination row, and the block's first thread
// stores the block's scale there.  (bf16 payload: 8-channel chunks copied
// unchanged.)  Nothing waits for the stores: a stage is refilled as soon as
// every thread has read it.
//
// The kernel runs concurrently with ll_scan_kernel (see there): rows and
// expert ids are inputs and are read at once; a token's slab rows come from
// the scan's mirror of ll_pos, read a token ahead and read again while a
// word is still zero (not written yet).  The kernel waits for the scan grid
// to complete before it exits, so later work in the stream sees both.
//
// kTab: one rank of a sharded job; the slabs of destination d are recv_tab[d]
// ([El][cap] rows) and scales_tab[d] in peer memory, and warp 0 turns each
// slot's row into the two row pointers.
template <bool kFP8, bool kTab, bool kTimed>
__global__ void __launch_bounds__(kLLThreads)
    ll_dispatch_kernel(const uint8_t *__restrict__ x, const int64_t *__restrict__ topk_idx,
                       const int32_t *pos_mirror, long num_tok, int H, int K, int E, int cap,
                       int round_scale, int ue8m0, LLSmem plan, uint8_t *__restrict__ recv,
                       void *__restrict__ scales_out, uint32_t *claim, int32_t *status,
                       unsigned long long timeout_ns, uint8_t *const *recv_tab,
                       uint8_t *const *scales_tab, int El, PhaseTimer *tm) {
  pdl_trigger();  // the next kernel may take the room this grid leaves
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ long s_tok[kLLMaxStages];  // token in each input stage, -1 = none
  __shared__ long s_dst[kMaxTopk];      // slab row (e * cap + pos) per slot, -1 = none
  __shared__ uint8_t *s_qp[kTab ? kMaxTopk : 1];  // kTab: payload row per slot, or nullptr
  __shared__ uint8_t *s_sp[kTab ? kMaxTopk : 1];  // kTab: scale row per slot
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int nst = plan.stages;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
  uint8_t *inb = smem + 128;
  const int row_in = 2 * H;
  const int pay = kFP8 ? H : 2 * H;             // bytes per slab row
  const int nchunk = kFP8 ? (H >> 4) : (H >> 3);  // 16 (FP8) or 8 (bf16) channels per chunk
  const int nblk = H >> 7;
  float *scales = static_cast<float *>(scales_out);
  uint8_t *scales8 = static_cast<uint8_t *>(scales_out);

  // Token blockIdx.x is this CTA's first (the grid is at most num_tok wide),
  // so every CTA starts on the earliest tokens, whose positions the scan
  // writes first; the rest are claimed from the counter, past the grid.
  auto take = [&]() -> long {  // thread 0: the next unclaimed token, or -1
    const long c = static_cast<long>(atomicAdd(claim, 1u)) + gridDim.x;
    return c < num_tok ? c : -1L;
  };
  auto issue = [&](int stg, long u) {  // thread 0
    s_tok[stg] = u;
    if (u < 0) return;
    mbar_arrive_expect_tx(&bars[stg], static_cast<uint32_t>(row_in));
    bulk_g2s_hint(inb + stg * plan.in_stride, x + u * row_in, static_cast<uint32_t>(row_in),
                  &bars[stg], l2_evict_first_policy());
  };
  auto expert_of = [&](long u) -> int {  // expert of slot `lane` of token u, or -1
    if (u < 0 || lane >= K) return -1;
    const int64_t ee = __ldg(topk_idx + u * K + lane);
    return (ee >= 0 && ee < E) ? static_cast<int>(ee) : -1;
  };
  auto mirror_of = [&](long u) -> int32_t {  // slot `lane` of token u: ll_pos + 2, 0 = not yet
    if (u < 0 || lane >= K) return 1;          // no slot: reads as ll_pos -1
    return ld_relaxed_gpu(pos_mirror + u * K + lane);
  };

  long ahead = -1;  // thread 0: the token claimed for the next issue
  if (tid == 0) {
    for (int i = 0; i < nst; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    for (int i = 0; i < nst; ++i) issue(i, i == 0 ? static_cast<long>(blockIdx.x) : take());
    ahead = take();
  }
  __syncthreads();
  // warp 0: the next token's experts and mirrored slab rows
  int e_next = -1;
  int32_t m_next = 0;
  bool failed = false;
  if (tid < 32) {
    e_next = expert_of(s_tok[0]);
    m_next = mirror_of(s_tok[0]);
  }

  bool all_ok = true;
  int stop = -1;      // stage whose load was the first not waited for, on failure
  int stg = 0;
  uint32_t phase = 0;
  while (true) {
    const long u = s_tok[stg];
    if (u < 0) break;  // claims are ordered: every later stage is empty too
    const uint8_t *in = inb + stg * plan.in_stride;
    const int nxt = stg + 1 == nst ? 0 : stg + 1;

    // warp 0: this token's destination rows (read a token ahead); start
    // reading the next token's
    if (tid < 32) {
      __syncwarp();  // lane 0's last issue() wrote s_tok[nxt]
      const int e = e_next;
      int32_t m = m_next;
      const long un = s_tok[nxt];
      e_next = expert_of(un);
      m_next = mirror_of(un);
      // words still zero are read again (bounded); after a wait ran out,
      // this and later tokens are dropped
      if (!failed) {
        uint64_t t0 = 0;
        while (!__all_sync(0xffffffffu, m != 0)) {
          const uint64_t now = __shfl_sync(0xffffffffu, globaltimer(), 0);
          if (t0 == 0) t0 = now;
          if (now - t0 > timeout_ns) {
            failed = true;
            if (lane == 0) report(status, EP_STATUS_WAIT_TIMEOUT);
            break;
          }
          __nanosleep(64);
          if (m == 0) m = mirror_of(u);
        }
      }
      const int pos = m - 2;
      // one row per distinct expert
      bool dup = false;
      for (int k2 = 0; k2 < K; ++k2) {
        const int e2 = __shfl_sync(0xffffffffu, e, k2);
        dup |= (k2 < lane && e2 == e);
      }
      long dst = -1;
      if (!failed && e >= 0 && !dup) {  // pos -1: the slot was dropped (failed rank)
        if (pos >= 0 && pos < cap)
          dst = static_cast<long>(e) * cap + pos;
        else if (pos != -1)
          report(status, EP_STATUS_BAD_POSITION);
      }
      if (lane < K) s_dst[lane] = dst;
      if constexpr (kTab) {
        if (lane < K) {
          uint8_t *qp = nullptr, *sp = nullptr;
          if (dst >= 0) {
            const int d = e / El;
            const long row = static_cast<long>(e - d * El) * cap + pos;
            qp = recv_tab[d] + row * pay;
            if (kFP8) sp = scales_tab[d] + row * nblk * (ue8m0 ? 1 : 4);
          }
          s_qp[lane] = qp;
          s_sp[lane] = sp;
        }
      }
    }
    const bool ok = mbar_wait_bounded(&bars[stg], phase, timeout_ns);
    if (__syncthreads_and(ok) == 0) {
      all_ok = false;
      stop = stg;
      break;
    }

    if constexpr (kFP8) {
      for (int c0 = 0; c0 < nchunk; c0 += kLLThreads) {
        const int c = c0 + tid;
        const bool act = c < nchunk;
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (act) {
          v0 = reinterpret_cast<const uint4 *>(in)[2 * c];
          v1 = reinterpret_cast<const uint4 *>(in)[2 * c + 1];
        }
        float f[16] = {bf16lo(v0.x), bf16hi(v0.x), bf16lo(v0.y), bf16hi(v0.y),
                       bf16lo(v0.z), bf16hi(v0.z), bf16lo(v0.w), bf16hi(v0.w),
                       bf16lo(v1.x), bf16hi(v1.x), bf16lo(v1.y), bf16hi(v1.y),
                       bf16lo(v1.z), bf16hi(v1.z), bf16lo(v1.w), bf16hi(v1.w)};
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(f[j]));
        // 8 consecutive threads hold one 128-channel block (nchunk % 8 == 0)
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        amax = fmaxf(amax, 1e-4f);
        float inv, scale;
        uint32_t ebits = 0;
        if (round_scale) {
          // smallest power of two >= amax / 448, and its exact reciprocal
          const uint32_t b = __float_as_uint(__fdiv_rn(amax, 448.0f));
          ebits = (b >> 23) + ((b & 0x7FFFFFu) != 0u ? 1u : 0u);
          scale = __uint_as_float(ebits << 23);
          inv = __uint_as_float((254u - ebits) << 23);
        } else {
          inv = __fdiv_rn(448.0f, amax);
          scale = __fdiv_rn(amax, 448.0f);
        }
        if (act) {
          uint4 q;
          q.x = cvt_e4m3x4(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv), __fmul_rn(f[2], inv),
                           __fmul_rn(f[3], inv));
          q.y = cvt_e4m3x4(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv), __fmul_rn(f[6], inv),
                           __fmul_rn(f[7], inv));
          q.z = cvt_e4m3x4(__fmul_rn(f[8], inv), __fmul_rn(f[9], inv), __fmul_rn(f[10], inv),
                           __fmul_rn(f[11], inv));
          q.w = cvt_e4m3x4(__fmul_rn(f[12], inv), __fmul_rn(f[13], inv), __fmul_rn(f[14], inv),
                           __fmul_rn(f[15], inv));
          const bool first = (c & 7) == 0;
          for (int k = 0; k < K; ++k) {
            if constexpr (kTab) {
              uint8_t *qr = s_qp[k];
              if (qr == nullptr) continue;
              st_stream_v4(qr + c * 16L, q);
              if (first) {
                if (ue8m0)
                  s_sp[k][c >> 3] = static_cast<uint8_t>(ebits);
                else
                  reinterpret_cast<float *>(s_sp[k])[c >> 3] = scale;
              }
            } else {
              const long dst = s_dst[k];
              if (dst < 0) continue;
              st_stream_v4(recv + dst * pay + c * 16L, q);
              if (first) {
                if (ue8m0)
                  scales8[dst * nblk + (c >> 3)] = static_cast<uint8_t>(ebits);
                else
                  scales[dst * nblk + (c >> 3)] = scale;
              }
            }
          }
        }
      }
    } else {
      for (int c = tid; c < nchunk; c += kLLThreads) {
        const uint4 v = reinterpret_cast<const uint4 *>(in)[c];
        for (int k = 0; k < K; ++k) {
          if constexpr (kTab) {
            if (s_qp[k] != nullptr) st_stream_v4(s_qp[k] + c * 16L, v);
          } else {
            const long dst = s_dst[k];
            if (dst >= 0) st_stream_v4(recv + dst * pay + c * 16L, v);
          }
        }
      }
    }
    __syncthreads();  // every thread has read the stage and the rows
    if (tid == 0) {
      fence_proxy_async_smem();
      const long next = ahead;
      ahead = next >= 0 ? take() : -1L;
      issue(stg, next);
    }
    stg = nxt;
    if (stg == 0) phase ^= 1u;
  }
  if (!all_ok) {
    report(status, EP_STATUS_WAIT_TIMEOUT);
    if (tid == 0) {
      // drain the loads still in flight before the CTA's shared memory goes
      // away: every stage from the failed one on holds one in flight
      int sg = stop;
      uint32_t ph = phase;
      for (int n = 0; n < nst; ++n) {
        if (s_tok[sg] >= 0) (void)mbar_wait_bounded(&bars[sg], ph, timeout_ns);
        if (++sg == nst) {
          sg = 0;
          ph ^= 1u;
        }
      }
    }
  }
  if constexpr (kTab) __threadfence_system();  // rows stored into peers' memory
  // the scan grid completes before this one does
  pdl_wait();
  if constexpr (kTimed) timer_end(tm, 0ull);  // begun by the zeroing kernel
}

// ---------------------------------------------------------------------------

// One rank of a sharded LL dispatch: the rows it sends to each expert (its
// tokens whose distinct valid slots hold the expert; nothing from a failed
// source rank, nothing to a failed rank's experts), the same count the
// single-GPU scan takes per source rank.  A thread per token; counts zeroed
// before.
__global__ void __launch_bounds__(256)
    ll_count_kernel(const int64_t *__restrict__ topk_idx, const int32_t *__restrict__ mask,
                    int rank, int T, int K, int E, int El, int32_t *counts, int32_t *status) {
  pdl_wait();
  pdl_trigger();
  const long t = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= T || (mask != nullptr && mask[rank] != 0)) return;
  int seen[kMaxTopk];
  int n = 0;
  bool bad = false;
  for (int k = 0; k < K; ++k) {
    const int64_t e = topk_idx[t * K + k];
    if (e == -1) continue;
    if (e < -1 || e >= E) {
      bad = true;
      continue;
    }
    if (mask != nullptr && mask[static_cast<int>(e) / El] != 0) continue;
    bool dup = false;
    for (int i = 0; i < n; ++i) dup |= seen[i] == static_cast<int>(e);
    if (dup) continue;
    seen[n++] = static_cast<int>(e);
    atomicAdd(&counts[e], 1);
  }
  if (bad) report(status, EP_STATUS_BAD_EXPERT);
}

// One rank of a sharded LL dispatch, from every rank's counts (gathered,
// [R][E]): base[e] = rows of expert e that the ranks before `rank` send (its
// own rows follow them, as source ranks are in order in a slab); this rank's
// (first row, rows) entry of every destination's layout_range ([El][R][2],
// in peer memory); and for its own experts the rows received from all ranks
// and the cumulative counter.
__global__ void __launch_bounds__(256)
    shard_ll_prefix_kernel(const int32_t *__restrict__ counts, int rank, int R, int E, int El,
                           int32_t *base, int32_t *const *lr_tab, int32_t *recv_count,
                           int32_t *stats) {
  pdl_wait();
  pdl_trigger();  // the scan's CTAs may start; they wait for this grid to complete
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
    int b = 0;
    for (int s = 0; s < rank; ++s) b += counts[static_cast<size_t>(s) * E + e];
    const int mine = counts[static_cast<size_t>(rank) * E + e];
    base[e] = b;
    const int d = e / El, j = e - d * El;
    int32_t *lr = lr_tab[d] + (static_cast<size_t>(j) * R + rank) * 2;
    lr[0] = b;
    lr[1] = mine;
    if (d == rank) {
      int tot = b + mine;
      for (int s = rank + 1; s < R; ++s) tot += counts[static_cast<size_t>(s) * E + e];
      recv_count[j] = tot;
      if (stats != nullptr) stats[j] += tot;
    }
  }
  __threadfence_system();  // layout_range entries stored into peers' memory
}

constexpr int kLLCombineWarps = 8;

// One warp per (token, channel segment): the token's up-to-K slab rows are
// listed in slot order, then each lane accumulates 16-byte chunks of the
// segment with fmaf in that order.  Splitting rows into `nseg` segments gives
// enough work items to keep every warp busy to the end.  y_tab: one rank of
// a sharded job (its tokens are source rank s0's); expert e's rows are in
// destination e / El's slab y_tab[e / El] in peer memory, read with plain
// loads.  Otherwise y holds every destination's slabs and s0 = 0.
template <bool kTimed>
__global__ void __launch_bounds__(kLLCombineWarps * 32)
    ll_combine_kernel(const uint8_t *__restrict__ y, const uint8_t *const *y_tab, int s0,
                      const int64_t *__restrict__ topk_idx,
                      const float *__restrict__ topk_w, const int32_t *__restrict__ ll_pos,
                      const int32_t *__restrict__ mask, long num_tok, int T, int H, int K, int E,
                      int cap, int nseg, uint8_t *__restrict__ out, int32_t *status,
                      PhaseTimer *tm) {
  pdl_wait();
  unsigned long long begun = 0ull;
  if constexpr (kTimed) begun = timer_begin(tm);
  __shared__ const uint8_t *s_row[kLLCombineWarps][kMaxTopk];
  __shared__ float s_w[kLLCombineWarps][kMaxTopk];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint32_t lt = lanemask_lt();
  const int nvec = H >> 3;
  const int seg_vec = (nvec + nseg - 1) / nseg;
  const int El = E / (cap / T);  // cap = R * T
  const long row_bytes = static_cast<long>(H) * 2;
  const long items = num_tok * nseg;
  for (long it = static_cast<long>(blockIdx.x) * kLLCombineWarps + warp; it < items;
       it += static_cast<long>(gridDim.x) * kLLCombineWarps) {
    const long u = it / nseg;
    const int sg = static_cast<int>(it % nseg);
    bool take = false;
    const uint8_t *row = nullptr;
    float w = 0.f;
    const bool src_ok = mask == nullptr || mask[s0 + u / T] == 0;
    if (lane < K && src_ok) {
      const int64_t e = topk_idx[u * K + lane];
      if (e >= 0 && e < E && (mask == nullptr || mask[e / El] == 0)) {
        const int pos = ll_pos[u * K + lane];
        if (pos >= 0 && pos < cap) {
          take = true;
          if (y_tab != nullptr) {
            const int d = static_cast<int>(e) / El;
            row = y_tab[d] + (static_cast<long>(static_cast<int>(e) - d * El) * cap + pos) *
                                 row_bytes;
          } else {
            row = y + (e * cap + pos) * row_bytes;
          }
          w = topk_w[u * K + lane];
        } else if (sg == 0 && pos != -1) {  // -1: dropped at dispatch
          report(status, EP_STATUS_BAD_POSITION);
        }
      }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int i = __popc(bal & lt);
      s_row[warp][i] = row;
      s_w[warp][i] = w;
    }
    const int n = __popc(bal);
    __syncwarp();

    uint8_t *orow = out + u * row_bytes;
    const int c_end = min(nvec, (sg + 1) * seg_vec);
    for (int c = sg * seg_vec + lane; c < c_end; c += 32) {
      float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < n; i += 8) {
        uint4 v[8];
#pragma unroll
        for (int b = 0; b < 8; ++b)
          if (i + b < n) v[b] = ld_stream_v4(s_row[warp][i + b] + c * 16L);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if (i + b < n) {
            const float wk = s_w[warp][i + b];
            a[0] = __fmaf_rn(bf16lo(v[b].x), wk, a[0]);
            a[1] = __fmaf_rn(bf16hi(v[b].x), wk, a[1]);
            a[2] = __fmaf_rn(bf16lo(v[b].y), wk, a[2]);
            a[3] = __fmaf_rn(bf16hi(v[b].y), wk, a[3]);
            a[4] = __fmaf_rn(bf16lo(v[b].z), wk, a[4]);
            a[5] = __fmaf_rn(bf16hi(v[b].z), wk, a[5]);
            a[6] = __fmaf_rn(bf16lo(v[b].w), wk, a[6]);
            a[7] = __fmaf_rn(bf16hi(v[b].w), wk, a[7]);
          }
        }
      }
      uint4 r;
      r.x = pack_bf16x2(a[0], a[1]);
      r.y = pack_bf16x2(a[2], a[3]);
      r.z = pack_bf16x2(a[4], a[5]);
      r.w = pack_bf16x2(a[6], a[7]);
      st_stream_v4(orow + c * 16L, r);
    }
    __syncwarp();
  }
  if constexpr (kTimed) timer_end(tm, begun);
}

}  // namespace
}  // namespace ep

namespace ep {
namespace {
// LL workspace: scan header, descriptors [tiles][E] (64-bit), then the
// position mirror [R*T][K] int32 (room for K up to kMaxTopk).
size_t ll_mirror_offset(long tiles, int E) {  // 16-byte aligned
  return (sizeof(ScanHeader) + static_cast<size_t>(tiles) * E * sizeof(uint64_t) + 15) &
         ~static_cast<size_t>(15);
}

// LL combine of num_tok tokens (arguments already checked): from y, or from
// the destinations' slabs y_tab (one rank's tokens, source rank s0).
int ll_combine_launch(const uint8_t *y, const uint8_t *const *y_tab, int s0,
                      const int64_t *topk_idx, const float *topk_weights, const int32_t *ll_pos,
                      const int32_t *rank_mask, long num_tok, int T, int H, int K, int E,
                      long cap, void *out, int32_t *status, cudaStream_t stream,
                      PhaseTimer *tm = nullptr) {
  const int threads = kLLCombineWarps * 32;
  auto *kernel = tm != nullptr ? ll_combine_kernel<true> : ll_combine_kernel<false>;
  const void *fn = reinterpret_cast<const void *>(kernel);
  const long resident = static_cast<long>(ctas_per_sm(fn, threads, 0)) * num_sms();
  // split rows into segments until there are >= 4 work items per resident warp
  const int nvec = H / 8;
  int nseg = static_cast<int>((4 * resident * kLLCombineWarps + num_tok - 1) / num_tok);
  nseg = std::max(1, std::min(nseg, std::max(1, nvec / 32)));
  const long items = num_tok * nseg;
  const long grid = std::min<long>((items + kLLCombineWarps - 1) / kLLCombineWarps, resident);
  const cudaError_t launched = launch_pdl(kernel,
      dim3(static_cast<unsigned>(grid)), dim3(threads), 0, stream, y, y_tab, s0, topk_idx,
      topk_weights, ll_pos, rank_mask, num_tok, T, H, K, E, static_cast<int>(cap), nseg,
      static_cast<uint8_t *>(out), status, tm);
  return launch_status(launched);
}

// The scan, then the dispatch kernel that runs alongside it (arguments
// already checked, the workspace words zeroed).  recv_tab / scales_tab: the
// destinations' slabs in peer memory (one rank of a sharded job), else
// recv_x / recv_scales hold every destination's slabs.
int ll_scan_and_dispatch(const LLScanParams &p, const void *x, int H, int use_fp8,
                         int round_scale, int ue8m0, const LLSmem &plan, void *recv_x,
                         void *recv_scales, uint8_t *const *recv_tab, uint8_t *const *scales_tab,
                         long num_tok, cudaStream_t stream, PhaseTimer *tm = nullptr) {
  cudaError_t launched;
  const dim3 sg(static_cast<unsigned>(p.num_tiles)), sb(kLLScanThreads);
  const bool shard = p.rsi_tab != nullptr;
  if (p.K > 8)
    launched = shard ? launch_pdl(ll_scan_kernel<16, true>, sg, sb, 0, stream, p)
                     : launch_pdl(ll_scan_kernel<16, false>, sg, sb, 0, stream, p);
  else
    launched = shard ? launch_pdl(ll_scan_kernel<8, true>, sg, sb, 0, stream, p)
                     : launch_pdl(ll_scan_kernel<8, false>, sg, sb, 0, stream, p);
  if (launch_status(launched) != EP_OK) return EP_ERR_CUDA;

  const bool tab = recv_tab != nullptr;
  if (tab) tm = nullptr;  // the sharded form is never timed
  const size_t smem = spread_smem(static_cast<size_t>(plan.bytes), kLLMaxCtasPerSm);
  const void *fn =
      use_fp8 ? (tab  ? reinterpret_cast<const void *>(ll_dispatch_kernel<true, true, false>)
                 : tm ? reinterpret_cast<const void *>(ll_dispatch_kernel<true, false, true>)
                      : reinterpret_cast<const void *>(ll_dispatch_kernel<true, false, false>))
              : (tab  ? reinterpret_cast<const void *>(ll_dispatch_kernel<false, true, false>)
                 : tm ? reinterpret_cast<const void *>(ll_dispatch_kernel<false, false, true>)
                      : reinterpret_cast<const void *>(ll_dispatch_kernel<false, false, false>));
  if (ensure_dynamic_smem(fn, smem) != EP_OK) return EP_ERR_CUDA;
  const long grid = std::min<long>(
      num_tok,
      static_cast<long>(std::min(kLLMaxCtasPerSm, ctas_per_sm(fn, kLLThreads, smem))) *
          num_sms());
  const dim3 g(static_cast<unsigned>(grid)), b(kLLThreads);
  const uint8_t *xb = static_cast<const uint8_t *>(x);
  uint8_t *rx = static_cast<uint8_t *>(recv_x);
  uint32_t *claim = &p.head->claim;
  const unsigned long long to = p.timeout_ns;
  uint8_t *const *no_tab = nullptr;
  if (use_fp8 && tab)
    launched = launch_pdl(ll_dispatch_kernel<true, true, false>, g, b, smem, stream, xb,
                          p.topk_idx, p.pos_mirror, num_tok, H, p.K, p.E, p.cap, round_scale,
                          ue8m0, plan, rx, recv_scales, claim, p.status, to, recv_tab,
                          scales_tab, p.El, tm);
  else if (use_fp8 && tm != nullptr)
    launched = launch_pdl(ll_dispatch_kernel<true, false, true>, g, b, smem, stream, xb,
                          p.topk_idx, p.pos_mirror, num_tok, H, p.K, p.E, p.cap, round_scale,
                          ue8m0, plan, rx, recv_scales, claim, p.status, to, no_tab, no_tab,
                          p.El, tm);
  else if (use_fp8)
    launched = launch_pdl(ll_dispatch_kernel<true, false, false>, g, b, smem, stream, xb,
                          p.topk_idx, p.pos_mirror, num_tok, H, p.K, p.E, p.cap, round_scale,
                          ue8m0, plan, rx, recv_scales, claim, p.status, to, no_tab, no_tab,
                          p.El, tm);
  else if (tab)
    launched = launch_pdl(ll_dispatch_kernel<false, true, false>, g, b, smem, stream, xb,
                          p.topk_idx, p.pos_mirror, num_tok, H, p.K, p.E, p.cap, 0, 0, plan, rx,
                          static_cast<void *>(nullptr), claim, p.status, to, recv_tab, no_tab,
                          p.El, tm);
  else if (tm != nullptr)
    launched = launch_pdl(ll_dispatch_kernel<false, false, true>, g, b, smem, stream, xb,
                          p.topk_idx, p.pos_mirror, num_tok, H, p.K, p.E, p.cap, 0, 0, plan, rx,
                          static_cast<void *>(nullptr), claim, p.status, to, no_tab, no_tab,
                          p.El, tm);
  else
    launched = launch_pdl(ll_dispatch_kernel<false, false, false>, g, b, smem, stream, xb,
                          p.topk_idx, p.pos_mirror, num_tok, H, p.K, p.E, p.cap, 0, 0, plan, rx,
                          static_cast<void *>(nullptr), claim, p.status, to, no_tab, no_tab,
                          p.El, tm);
  return launch_status(launched);
}
}  // namespace
}  // namespace ep

extern "C" EP_API size_t ep_ll_workspace_bytes(int num_ranks, int num_tokens, int num_experts) {
  using namespace ep;
  if (num_ranks < 1 || num_tokens < 0 || num_experts < 1) return 0;
  const long tiles = static_cast<long>(num_ranks) * ((num_tokens + kScanTile - 1) / kScanTile);
  const size_t bytes = ll_mirror_offset(tiles, num_experts) +
                       static_cast<size_t>(num_ranks) * num_tokens * kMaxTopk * sizeof(int32_t);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

extern "C" EP_API int ep_ll_dispatch(const void *x, const int64_t *topk_idx,
                                     const int32_t *rank_mask, int num_ranks, int num_tokens,
                                     int hidden, int num_topk, int num_experts, int fp8_flags,
                                     void *recv_x, void *recv_scales, int32_t *recv_count,
                                     int32_t *recv_src_info, int32_t *layout_range,
                                     int32_t *ll_pos, int32_t *cumulative_local_expert_recv_stats,
                                     void *workspace, size_t workspace_bytes, int32_t *status,
                                     cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, K = num_topk, E = num_experts;
  const int use_fp8 = (fp8_flags & EP_LL_FP8) != 0;
  const int round_scale = (fp8_flags & EP_LL_ROUND_SCALE) != 0;
  const int ue8m0 = (fp8_flags & EP_LL_UE8M0) != 0;
  if ((fp8_flags & ~(EP_LL_FP8 | EP_LL_ROUND_SCALE | EP_LL_UE8M0)) != 0 ||
      (round_scale && !use_fp8) || (ue8m0 && !round_scale))
    return EP_ERR_INVALID_ARG;
  if (R < 1 || R > kMaxRanks || T < 0 || K < 1 || K > kMaxTopk || E < 1 || E > kMaxExperts ||
      E % R != 0 || H < 8 || (use_fp8 ? (H % 128 != 0) : (H % 8 != 0)))
    return EP_ERR_INVALID_ARG;
  if (recv_count == nullptr || layout_range == nullptr) return EP_ERR_INVALID_ARG;
  if (T == 0) {
    if (cudaMemsetAsync(recv_count, 0, sizeof(int32_t) * E, stream) != cudaSuccess ||
        cudaMemsetAsync(layout_range, 0, sizeof(int32_t) * 2 * static_cast<size_t>(E) * R,
                        stream) != cudaSuccess)
      return EP_ERR_CUDA;
    return EP_OK;
  }
  if (x == nullptr || topk_idx == nullptr || recv_x == nullptr || recv_src_info == nullptr ||
      ll_pos == nullptr || (use_fp8 && recv_scales == nullptr))
    return EP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(recv_x) & 15u) ||
      (use_fp8 && (reinterpret_cast<uintptr_t>(recv_scales) & 15u)))
    return EP_ERR_INVALID_ARG;
  if (cumulative_local_expert_recv_stats != nullptr &&
      (reinterpret_cast<uintptr_t>(cumulative_local_expert_recv_stats) & 3u))
    return EP_ERR_INVALID_ARG;
  const size_t need = ep_ll_workspace_bytes(R, T, E);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return EP_ERR_INVALID_ARG;
  const long cap = static_cast<long>(R) * T;
  const int tiles_per_src = (T + kScanTile - 1) / kScanTile;
  const long num_tiles = static_cast<long>(R) * tiles_per_src;
  if (cap > 0x7ffffffdL) return EP_ERR_UNSUPPORTED;  // mirror words hold ll_pos + 2
  const LLSmem plan = ll_smem_plan(H);               // input rows staged whole
  if (plan.stages < 2) return EP_ERR_UNSUPPORTED;
  // header, descriptors and the mirror words this call uses start at zero
  const size_t used = ll_mirror_offset(num_tiles, E) + static_cast<size_t>(cap) * K * sizeof(int32_t);
  // the call's first kernel zeroes them (the workspace is at least
  // ep_ll_workspace_bytes, a multiple of 256 bytes past `used`, so whole
  // 16-byte words stay inside it), prefetching the ids the scan reads first
  PhaseTimer *const tm = phase_timer(kPhaseLLDispatch);
  if (zero_prefetch(workspace, (used + 15) & ~static_cast<size_t>(15), layout_range,
                    tiles_per_src > 1 ? 2L * E * R : 0L, topk_idx,
                    static_cast<long>(R) * T * K * 8, stream, tm) != EP_OK)
    return EP_ERR_CUDA;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  LLScanParams p;
  p.s0 = 0;
  p.base = nullptr;
  p.rsi_tab = nullptr;
  p.topk_idx = topk_idx;
  p.mask = rank_mask;
  p.stats = cumulative_local_expert_recv_stats;
  p.El = E / R;
  p.R = R;
  p.T = T;
  p.K = K;
  p.E = E;
  p.cap = static_cast<int>(cap);
  p.tiles_per_src = tiles_per_src;
  p.num_tiles = static_cast<int>(num_tiles);
  p.ll_pos = ll_pos;
  p.recv_src_info = recv_src_info;
  p.layout_range = layout_range;
  p.recv_count = recv_count;
  p.head = reinterpret_cast<ScanHeader *>(ws);
  p.desc = reinterpret_cast<uint64_t *>(ws + sizeof(ScanHeader));
  p.pos_mirror = reinterpret_cast<int32_t *>(ws + ll_mirror_offset(num_tiles, E));
  p.status = status;
  const WaitConfig wc = wait_config();
  p.timeout_ns = wc.timeout_ns;
  p.flags = wc.flags;
  return ll_scan_and_dispatch(p, x, H, use_fp8, round_scale, ue8m0, plan, recv_x, recv_scales,
                              nullptr, nullptr, static_cast<long>(R) * T, stream, tm);
}

extern "C" EP_API int ep_ll_combine(const void *y, const int64_t *topk_idx,
                                    const float *topk_weights, const int32_t *ll_pos,
                                    const int32_t *rank_mask, int num_ranks, int num_tokens,
                                    int hidden, int num_topk, int num_experts, void *out,
                                    int32_t *status, cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, K = num_topk, E = num_experts;
  if (R < 1 || R > kMaxRanks || T < 0 || K < 1 || K > kMaxTopk || E < 1 || E > kMaxExperts ||
      E % R != 0 || H < 8 || H % 8 != 0)
    return EP_ERR_INVALID_ARG;
  if (T == 0) return EP_OK;
  if (y == nullptr || topk_idx == nullptr || topk_weights == nullptr || ll_pos == nullptr ||
      out == nullptr)
    return EP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(y) & 15u) || (reinterpret_cast<uintptr_t>(out) & 15u))
    return EP_ERR_INVALID_ARG;
  const long cap = static_cast<long>(R) * T;
  if (cap > 0x7fffffffL) return EP_ERR_UNSUPPORTED;
  return ll_combine_launch(static_cast<const uint8_t *>(y), nullptr, 0, topk_idx, topk_weights,
                           ll_pos, rank_mask, static_cast<long>(R) * T, T, H, K, E, cap, out,
                           status, stream, phase_timer(kPhaseLLCombine));
}

// ---------------------------------------------------------------------------
// One rank per GPU: the low-latency pair with each rank's tokens on its own
// GPU and every destination's slabs in that destination's memory.

extern "C" EP_API size_t ep_shard_ll_workspace_bytes(int num_ranks, int num_tokens,
                                                     int num_experts) {
  using namespace ep;
  if (num_ranks < 1 || num_tokens < 0 || num_experts < 1) return 0;
  // the scan's words for one source rank's tokens, then base[E]
  return ep_ll_workspace_bytes(1, num_tokens, num_experts) +
         ((static_cast<size_t>(num_experts) * sizeof(int32_t) + 255) & ~static_cast<size_t>(255));
}

extern "C" EP_API int ep_shard_ll_counts(const int64_t *topk_idx, const int32_t *rank_mask,
                                         int rank, int num_ranks, int num_tokens, int num_topk,
                                         int num_experts, int32_t *counts, int32_t *status,
                                         cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, K = num_topk, E = num_experts;
  if (R < 1 || R > kMaxRanks || rank < 0 || rank >= R || T < 0 || K < 1 || K > kMaxTopk ||
      E < 1 || E > kMaxExperts || E % R != 0 || counts == nullptr ||
      (T > 0 && topk_idx == nullptr))
    return EP_ERR_INVALID_ARG;
  if (zero_prefetch(nullptr, 0, counts, E, topk_idx, static_cast<long>(T) * K * 8, stream) !=
      EP_OK)
    return EP_ERR_CUDA;
  if (T == 0) return EP_OK;
  return launch_status(launch_pdl(ll_count_kernel, dim3(static_cast<unsigned>((T + 255) / 256)),
                                  dim3(256), 0, stream, topk_idx, rank_mask, rank, T, K, E, E / R,
                                  counts, status));
}

extern "C" EP_API int ep_shard_ll_dispatch(
    const void *x, const int64_t *topk_idx, const int32_t *rank_mask, const int32_t *counts,
    int rank, int num_ranks, int num_tokens, int hidden, int num_topk, int num_experts,
    int fp8_flags, void *const *recv_x_peers, void *const *recv_scales_peers,
    int32_t *const *recv_src_info_peers, int32_t *const *layout_range_peers, int32_t *recv_count,
    int32_t *ll_pos, int32_t *cumulative_local_expert_recv_stats, void *workspace,
    size_t workspace_bytes, int32_t *status, cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, K = num_topk, E = num_experts;
  const int use_fp8 = (fp8_flags & EP_LL_FP8) != 0;
  const int round_scale = (fp8_flags & EP_LL_ROUND_SCALE) != 0;
  const int ue8m0 = (fp8_flags & EP_LL_UE8M0) != 0;
  if ((fp8_flags & ~(EP_LL_FP8 | EP_LL_ROUND_SCALE | EP_LL_UE8M0)) != 0 ||
      (round_scale && !use_fp8) || (ue8m0 && !round_scale))
    return EP_ERR_INVALID_ARG;
  if (R < 1 || R > kMaxRanks || rank < 0 || rank >= R || T < 0 || K < 1 || K > kMaxTopk ||
      E < 1 || E > kMaxExperts || E % R != 0 || H < 8 ||
      (use_fp8 ? (H % 128 != 0) : (H % 8 != 0)))
    return EP_ERR_INVALID_ARG;
  if (counts == nullptr || layout_range_peers == nullptr || recv_count == nullptr)
    return EP_ERR_INVALID_ARG;
  if (T > 0 && (x == nullptr || topk_idx == nullptr || recv_x_peers == nullptr ||
                recv_src_info_peers == nullptr || ll_pos == nullptr ||
                (use_fp8 && recv_scales_peers == nullptr)))
    return EP_ERR_INVALID_ARG;
  if (x != nullptr && (reinterpret_cast<uintptr_t>(x) & 15u)) return EP_ERR_INVALID_ARG;
  if (cumulative_local_expert_recv_stats != nullptr &&
      (reinterpret_cast<uintptr_t>(cumulative_local_expert_recv_stats) & 3u))
    return EP_ERR_INVALID_ARG;
  const size_t need = ep_shard_ll_workspace_bytes(R, T, E);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return EP_ERR_INVALID_ARG;
  const long cap = static_cast<long>(R) * T;
  if (cap > 0x7ffffffdL) return EP_ERR_UNSUPPORTED;  // mirror words hold ll_pos + 2
  const LLSmem plan = ll_smem_plan(H);
  if (plan.stages < 2) return EP_ERR_UNSUPPORTED;
  const int tiles = (T + kScanTile - 1) / kScanTile;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *base = reinterpret_cast<int32_t *>(ws + ep_ll_workspace_bytes(1, T, E));
  // header, descriptors and this call's mirror words start at zero
  const size_t used = ll_mirror_offset(tiles, E) + static_cast<size_t>(T) * K * sizeof(int32_t);
  if (zero_prefetch(workspace, (used + 15) & ~static_cast<size_t>(15), nullptr, 0, topk_idx,
                    static_cast<long>(T) * K * 8, stream) != EP_OK)
    return EP_ERR_CUDA;
  if (launch_status(launch_pdl(shard_ll_prefix_kernel, dim3(static_cast<unsigned>((E + 255) / 256)),
                               dim3(256), 0, stream, counts, rank, R, E, E / R, base,
                               layout_range_peers, recv_count,
                               cumulative_local_expert_recv_stats)) != EP_OK)
    return EP_ERR_CUDA;
  if (T == 0) return EP_OK;

  LLScanParams p;
  p.s0 = rank;
  p.base = base;
  p.rsi_tab = recv_src_info_peers;
  p.topk_idx = topk_idx;
  p.mask = rank_mask;
  p.stats = nullptr;
  p.El = E / R;
  p.R = R;
  p.T = T;
  p.K = K;
  p.E = E;
  p.cap = static_cast<int>(cap);
  p.tiles_per_src = tiles;
  p.num_tiles = tiles;  // one source rank
  p.ll_pos = ll_pos;
  p.recv_src_info = nullptr;
  p.layout_range = nullptr;
  p.recv_count = nullptr;
  p.head = reinterpret_cast<ScanHeader *>(ws);
  p.desc = reinterpret_cast<uint64_t *>(ws + sizeof(ScanHeader));
  p.pos_mirror = reinterpret_cast<int32_t *>(ws + ll_mirror_offset(tiles, E));
  p.status = status;
  const WaitConfig wc = wait_config();
  p.timeout_ns = wc.timeout_ns;
  p.flags = wc.flags;
  return ll_scan_and_dispatch(p, x, H, use_fp8, round_scale, ue8m0, plan, nullptr, nullptr,
                              reinterpret_cast<uint8_t *const *>(recv_x_peers),
                              reinterpret_cast<uint8_t *const *>(recv_scales_peers), T, stream);
}

extern "C" EP_API int ep_shard_ll_combine(const void *const *y_peers, const int64_t *topk_idx,
                                          const float *topk_weights, const int32_t *ll_pos,
                                          const int32_t *rank_mask, int rank, int num_ranks,
                                          int num_tokens, int hidden, int num_topk,
                                          int num_experts, void *out, int32_t *status,
                                          cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, K = num_topk, E = num_experts;
  if (R < 1 || R > kMaxRanks || rank < 0 || rank >= R || T < 0 || K < 1 || K > kMaxTopk ||
      E < 1 || E > kMaxExperts || E % R != 0 || H < 8 || H % 8 != 0)
    return EP_ERR_INVALID_ARG;
  if (T == 0) return EP_OK;
  if (y_peers == nullptr || topk_idx == nullptr || topk_weights == nullptr ||
      ll_pos == nullptr || out == nullptr)
    return EP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(out) & 15u) return EP_ERR_INVALID_ARG;
  const long cap = static_cast<long>(R) * T;
  if (cap > 0x7fffffffL) return EP_ERR_UNSUPPORTED;
  return ll_combine_launch(nullptr, reinterpret_cast<const uint8_t *const *>(y_peers), rank,
                           topk_idx, topk_weights, ll_pos, rank_mask, T, T, H, K, E, cap, out,
                           status, stream);
}
