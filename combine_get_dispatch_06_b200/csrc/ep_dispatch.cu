// ep_dispatch.cu -- A2 + A3: rank prefix matrix, positions, dispatch scatter.
//
// Semantics (DeepEP "Python 接口" page, Dispatch API; legacy-test analysis
// page, intranode handle tuple and check_data): the copy of token (s, t) to
// rank d lands at row send_pos[s][t][d] of d's receive buffer, rows ordered by
// source rank then token.  That row number is the exclusive prefix, over the
// flattened (s, t) order, of is_token_in_rank[.][.][d]; its value at the end
// of source rank s is the rank prefix matrix P[s][d].
//
// Kernels:
//   dispatch_scan_kernel  one CTA per 128-token tile: routing bits -> warp
//                         ballots -> per-rank tile counts -> look-back ->
//                         send_pos, recv_src_idx, received top-k metadata, P,
//                         recv_count; expert counts are reduced with shared +
//                         global atomics.  Small (a few MB of traffic).
//   notify_finish_kernel  after the scan: -1 padding of the received ids past
//                         each rank's count, and the gathered counts turned
//                         into the outputs over the whole grid.
//   shard_prefix_kernel   one rank of a sharded job: P, its destination bases
//                         and receive counts from the all-gathered counts.
//   dispatch_copy_rows_kernel  the data movement: each token row is read ONCE from
//                         HBM into shared memory by a bulk (TMA) copy and
//                         written to each destination by bulk shared->global
//                         copies, S stages deep.  HBM-bound: R*T*H*2 bytes
//                         read, N*H*2 bytes written (N = number of copies).
//   dispatch_copy_planes_kernel  the same for e4m3 rows plus their scales.
// With the phase timers on (ep_set_phase_timers), the notify's finish kernel
// and the bf16 row copy run their timed instances (template flag kTimed).
#include <algorithm>
#include <mutex>

#include "ep_scan.cuh"

namespace ep {
namespace {

constexpr int kMaskWords = (kMaxRanks + 31) / 32;
// Largest tiles x R for which a tile reads every predecessor's counts at once
// (R must divide the tile); above it, the windowed decoupled look-back.
constexpr int kFullLookback = 8192;

struct DispatchScanParams {
  const int64_t *topk_idx;
  const float *topk_w;
  const uint8_t *in_rank;
  int R, T, K, E, El, cap, align, tiles_per_src, num_tiles, W;
  FastDiv el_div;  // division by El
  int32_t *send_pos;
  int32_t *recv_src_idx;
  int64_t *recv_idx;
  float *recv_w;
  int32_t *P;            // or nullptr (one rank of a sharded job: P comes from the counts)
  int32_t *recv_count;   // or nullptr (likewise)
  int32_t *nrte;
  int32_t *ntpr_out;     // optional layout outputs (routing from topk_idx only)
  int32_t *ntpe_out;
  uint8_t *in_rank_out;
  // One rank of a sharded job (the call's tokens are one source rank's):
  // row of the first of its tokens in each destination, and the destination
  // ranks' receive buffers in peer memory.  All nullptr for the simulated
  // ranks of one GPU (rows start at 0, buffers are slices d * cap).
  const int32_t *dst_base;   // [R]
  int32_t *const *rsi_tab;   // [R] -> recv_src_idx rows of rank d
  int64_t *const *ridx_tab;  // [R] -> recv_topk_idx rows of rank d (or nullptr)
  float *const *rw_tab;      // [R] -> recv_topk_weights rows of rank d (or nullptr)
  // Full-grid timer of the launch (or nullptr): complemented earliest block
  // start in the workspace; cumulative [ns, launches, last start, last end].
  unsigned long long *probe_state;
  unsigned long long *probe;
  int finalise;  // the last CTA writes nrte / ntpe_out / ntpr_out (else notify_finish_kernel)
  int idx32, w32, sp32;  // 32-byte stores of received ids / weights / send_pos rows
  ScanHeader *head;
  int32_t *expert_cnt;   // [E] all sources, then [R][E] per source
  uint64_t *desc;
  int32_t *status;
  unsigned long long timeout_ns;
  unsigned flags;
};

// Received top-k metadata of the copy held by rank d: the local id of every
// slot whose expert lives on d (dk[k] == d, lk[k] its local id), -1 and 0.0
// for the others.  32-bit compares and selects; 16-byte stores when K allows
// them (rows of K int64 / K fp32 are then 16-byte aligned).
template <int MAXK>
__device__ __forceinline__ void write_meta(int64_t *idx_row, float *w_row, int K, int d,
                                           const int (&dk)[MAXK], const int (&lk)[MAXK],
                                           const float (&wk)[MAXK], bool idx32, bool w32) {
  if (idx_row != nullptr) {
    int64_t *dst = idx_row;
    if (idx32) {  // K % 4 == 0, rows 32-byte aligned: one whole sector per store
#pragma unroll
      for (int k = 0; k < MAXK; k += 4) {
        if (k < K)
          st_v4_b64(dst + k, dk[k] == d ? static_cast<int64_t>(lk[k]) : -1ll,
                    dk[k + 1] == d ? static_cast<int64_t>(lk[k + 1]) : -1ll,
                    dk[k + 2] == d ? static_cast<int64_t>(lk[k + 2]) : -1ll,
                    dk[k + 3] == d ? static_cast<int64_t>(lk[k + 3]) : -1ll);
      }
    } else if ((K & 1) == 0) {
#pragma unroll
      for (int k = 0; k < MAXK; k += 2) {
        if (k < K) {
          longlong2 v;
          v.x = dk[k] == d ? static_cast<int64_t>(lk[k]) : -1ll;
          v.y = dk[k + 1] == d ? static_cast<int64_t>(lk[k + 1]) : -1ll;
          *reinterpret_cast<longlong2 *>(dst + k) = v;
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < MAXK; ++k)
        if (k < K) dst[k] = dk[k] == d ? static_cast<int64_t>(lk[k]) : -1ll;
    }
  }
  if (w_row != nullptr) {
    float *dst = w_row;
    if (w32) {  // K % 8 == 0, rows 32-byte aligned
#pragma unroll
      for (int k = 0; k < MAXK; k += 8) {
        if (k < K) {
          float v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = dk[k + j] == d ? wk[k + j] : 0.f;
          st_v8_b32(dst + k, v);
        }
      }
    } else if ((K & 3) == 0) {
#pragma unroll
      for (int k = 0; k < MAXK; k += 4) {
        if (k < K) {
          float4 v;
          v.x = dk[k] == d ? wk[k] : 0.f;
          v.y = dk[k + 1] == d ? wk[k + 1] : 0.f;
          v.z = dk[k + 2] == d ? wk[k + 2] : 0.f;
          v.w = dk[k + 3] == d ? wk[k + 3] : 0.f;
          *reinterpret_cast<float4 *>(dst + k) = v;
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < MAXK; ++k)
        if (k < K) dst[k] = dk[k] == d ? wk[k] : 0.f;
    }
  }
}

// MAXK: compile-time bound on the top-k slots (8 or 16), chosen per call.
template <int MAXK>
__global__ void __launch_bounds__(kScanTile) dispatch_scan_kernel(DispatchScanParams p) {
  pdl_wait();
  if (p.probe != nullptr && threadIdx.x == 0) atomicMax(p.probe_state, ~globaltimer());
  __shared__ int s_tile;
  __shared__ int s_last;
  __shared__ uint32_t s_mask[kScanTile * kMaskWords];
  __shared__ int s_woff[kScanWarps][kMaxRanks];
  __shared__ uint32_t s_bal[kScanWarps][kMaxRanks];  // lanes of the warp whose token goes to d
  __shared__ int s_excl[kMaxRanks];
  __shared__ int s_agg[kMaxRanks];
  __shared__ int s_ehist[kMaxExperts];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const bool count_experts = p.nrte != nullptr || p.ntpe_out != nullptr;

  if (tid == 0) s_tile = static_cast<int>(atomicAdd(&p.head->ticket, 1u));
  if (count_experts)
    for (int e = tid; e < p.E; e += kScanTile) s_ehist[e] = 0;
  __syncthreads();

  const int tile = s_tile;
  const int s = tile / p.tiles_per_src;
  const int t = (tile % p.tiles_per_src) * kScanTile + tid;
  const bool valid = t < p.T;
  const size_t st = static_cast<size_t>(s) * p.T + t;

  // ---- the token's top-k ids and weights, loaded once, all at once --------
  const bool want_w = p.recv_w != nullptr || p.rw_tab != nullptr;
  const bool meta = valid && p.topk_idx != nullptr &&
                    (p.recv_idx != nullptr || p.ridx_tab != nullptr || want_w);
  const bool need_idx = valid && p.topk_idx != nullptr;
  int64_t ek[MAXK];
  float wk[MAXK];
#pragma unroll
  for (int k = 0; k < MAXK; ++k) {
    ek[k] = -1;
    wk[k] = 0.f;
    if (need_idx && k < p.K) {
      ek[k] = p.topk_idx[st * p.K + k];
      if (meta && want_w) wk[k] = p.topk_w[st * p.K + k];
    }
  }

  // destination rank and local id of every valid slot (-1: none)
  int dk[MAXK], lk[MAXK];
#pragma unroll
  for (int k = 0; k < MAXK; ++k) {
    const int64_t e = ek[k];
    const bool ok = k < p.K && e >= 0 && e < p.E;
    dk[k] = ok ? fastdiv(static_cast<int>(e), p.el_div) : -1;
    lk[k] = ok ? static_cast<int>(e) - dk[k] * p.El : 0;
  }

  // ---- routing bits of this token --------------------------------------
  uint32_t *my_mask = s_mask + tid * p.W;
  for (int w = 0; w < p.W; ++w) my_mask[w] = 0u;
  if (valid) {
    if (p.in_rank != nullptr) {
      const uint8_t *ir = p.in_rank + st * p.R;
      for (int d = 0; d < p.R; ++d)
        if (ir[d]) my_mask[d >> 5] |= 1u << (d & 31);
    }
    if (p.topk_idx != nullptr && (p.in_rank == nullptr || count_experts)) {
      bool bad = false;
#pragma unroll
      for (int k = 0; k < MAXK; ++k) {
        if (k >= p.K) break;
        const int64_t e = ek[k];
        if (e == -1) continue;
        if (e < -1 || e >= p.E) {
          bad = true;
          continue;
        }
        if (p.in_rank == nullptr) my_mask[dk[k] >> 5] |= 1u << (dk[k] & 31);
        if (count_experts) atomicAdd(&s_ehist[static_cast<int>(e)], 1);
      }
      if (bad) report(p.status, EP_STATUS_BAD_EXPERT);
    }
  }
  // fused layout output: this token's row of is_token_in_rank
  if (valid && p.in_rank_out != nullptr) {
    uint8_t *row = p.in_rank_out + st * p.R;
    if ((p.R & 3) == 0 && (reinterpret_cast<uintptr_t>(p.in_rank_out) & 3u) == 0) {
      for (int d = 0; d < p.R; d += 4) {  // four 0/1 bytes per 32-bit store
        const uint32_t b = my_mask[d >> 5] >> (d & 31);
        reinterpret_cast<uint32_t *>(row)[d >> 2] =
            (b & 1u) | ((b >> 1) & 1u) << 8 | ((b >> 2) & 1u) << 16 | ((b >> 3) & 1u) << 24;
      }
    } else {
      for (int d = 0; d < p.R; ++d) row[d] = (my_mask[d >> 5] >> (d & 31)) & 1u;
    }
  }
  __syncthreads();

  // ---- pass 1: per-warp count of tokens going to each rank ---------------
  for (int d0 = 0; d0 < p.R; d0 += 32) {
    const uint32_t word = my_mask[d0 >> 5];
    const int nb = min(32, p.R - d0);
    for (int b = 0; b < nb; ++b) {
      const uint32_t bal = __ballot_sync(0xffffffffu, (word >> b) & 1u);
      if (lane == 0) {
        s_woff[warp][d0 + b] = __popc(bal);
        s_bal[warp][d0 + b] = bal;
      }
    }
  }
  __syncthreads();

  // ---- tile totals -------------------------------------------------------
  for (int d = tid; d < p.R; d += kScanTile) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kScanWarps; ++w) {
      const int c = s_woff[w][d];
      s_woff[w][d] = run;
      run += c;
    }
    s_agg[d] = run;
  }
  __syncthreads();

  // ---- look-back (a group of 16 lanes per rank column), prefix matrix ----
  const bool publish = (p.flags & EP_DEBUG_SUPPRESS_PUBLISH) == 0;
  const bool last_of_src = (tile % p.tiles_per_src) == p.tiles_per_src - 1;
  if (kScanTile % p.R == 0 && static_cast<long>(p.num_tiles) * p.R <= kFullLookback) {
    // Every tile publishes its counts, and each tile adds up all of its
    // predecessors' counts at once: no tile waits for another's inclusive
    // prefix, only for its counts, which every running tile publishes
    // before it waits on anything.  Tickets order the tiles, so every
    // predecessor is running or done.  Counts are 32-bit words (count + 1,
    // 0 = not yet published), [tile][R] flat; thread tid reads the groups
    // of four words 4 * tid + 512 * m, so (R dividing the tile and hence
    // 512) its word q always belongs to column (4 * tid + q) % R.  A batch
    // that found words not yet published is read again as a whole.
    uint32_t *cnt32 = reinterpret_cast<uint32_t *>(p.desc);
    for (int d = tid; d < p.R; d += kScanTile) {
      s_excl[d] = 0;
      if (publish)
        st_relaxed_gpu(reinterpret_cast<int32_t *>(cnt32) + static_cast<size_t>(tile) * p.R + d,
                       s_agg[d] + 1);
    }
    __syncthreads();
    const int n = tile * p.R;
    const int ngroups = (n + 3) >> 2;
    const bool vec = (reinterpret_cast<uintptr_t>(cnt32) & 15u) == 0;
    auto load_group = [&](int gi) -> uint4 {
      const int f = gi * 4;
      if (vec && f + 3 < n) return ld_relaxed_gpu_v4(cnt32 + f);
      uint4 v = make_uint4(1u, 1u, 1u, 1u);  // words past n count as published zeros
      const int32_t *w32 = reinterpret_cast<const int32_t *>(cnt32) + f;
      v.x = static_cast<uint32_t>(ld_relaxed_gpu(w32));
      if (f + 1 < n) v.y = static_cast<uint32_t>(ld_relaxed_gpu(w32 + 1));
      if (f + 2 < n) v.z = static_cast<uint32_t>(ld_relaxed_gpu(w32 + 2));
      if (f + 3 < n) v.w = static_cast<uint32_t>(ld_relaxed_gpu(w32 + 3));
      return v;
    };
    auto unpublished = [](const uint4 &w) {
      return w.x == 0u || w.y == 0u || w.z == 0u || w.w == 0u;
    };
    uint32_t acc[4] = {0u, 0u, 0u, 0u};
    bool timed_out = false;
    constexpr int kB = 8;
    for (int g0 = tid; g0 < ngroups; g0 += kScanTile * kB) {
      uint4 v[kB];
      uint32_t pend = 0u;
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int gi = g0 + b * kScanTile;
        v[b] = gi < ngroups ? load_group(gi) : make_uint4(1u, 1u, 1u, 1u);
      }
#pragma unroll
      for (int b = 0; b < kB; ++b)
        if (unpublished(v[b])) pend |= 1u << b;
      if (pend != 0u && !timed_out) {
        const uint64_t ts = globaltimer();
        do {
          __nanosleep(64);
#pragma unroll
          for (int b = 0; b < kB; ++b)
            if ((pend >> b) & 1u) v[b] = load_group(g0 + b * kScanTile);
#pragma unroll
          for (int b = 0; b < kB; ++b)
            if (((pend >> b) & 1u) && !unpublished(v[b])) pend &= ~(1u << b);
          if (pend != 0u && globaltimer() - ts > p.timeout_ns) timed_out = true;
        } while (pend != 0u && !timed_out);
      }
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        acc[0] += v[b].x != 0u ? v[b].x - 1u : 0u;
        acc[1] += v[b].y != 0u ? v[b].y - 1u : 0u;
        acc[2] += v[b].z != 0u ? v[b].z - 1u : 0u;
        acc[3] += v[b].w != 0u ? v[b].w - 1u : 0u;
      }
    }
    if (timed_out) report(p.status, EP_STATUS_WAIT_TIMEOUT);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (acc[q] != 0u) atomicAdd(&s_excl[(4 * tid + q) % p.R], static_cast<int>(acc[q]));
    __syncthreads();
    for (int d = tid; d < p.R; d += kScanTile) {
      const int excl = s_excl[d];
      const int run = s_agg[d];
      if (last_of_src && p.P != nullptr) {
        p.P[static_cast<size_t>(s) * p.R + d] = excl + run;
        if (tile == p.num_tiles - 1) p.recv_count[d] = excl + run;
      }
      s_excl[d] = excl + (p.dst_base != nullptr ? p.dst_base[d] : 0);
    }
  } else {
    constexpr int G = 16;
    const int grp = tid / G;
    for (int d = grp; d < p.R; d += kScanTile / G) {
      const int run = s_agg[d];
      const uint32_t excl = lookback_window<G, 4>(p.desc, tile, p.R, d, static_cast<uint32_t>(run),
                                                  publish, p.timeout_ns, p.status);
      if ((tid & (G - 1)) == 0) {
        s_excl[d] = static_cast<int>(excl) + (p.dst_base != nullptr ? p.dst_base[d] : 0);
        if (last_of_src && p.P != nullptr) {
          p.P[static_cast<size_t>(s) * p.R + d] = static_cast<int>(excl) + run;
          if (tile == p.num_tiles - 1) p.recv_count[d] = static_cast<int>(excl) + run;
        }
      }
    }
  }
  __syncthreads();

  // ---- pass 2: positions, handle and received metadata -------------------
  // The token's row in destination d (where it goes): rows of earlier tiles,
  // of earlier warps of this tile, then of lower lanes of this warp.  Each
  // thread writes its own send_pos row, then one row of handle and metadata
  // per destination it goes to (its set routing bits), so the work follows
  // the token's copies, not R.
  const uint32_t lt = lanemask_lt();
  bool overflow = false;
  auto goes = [&](int d) { return ((my_mask[d >> 5] >> (d & 31)) & 1u) != 0u; };
  auto pos_of = [&](int d) { return s_excl[d] + s_woff[warp][d] + __popc(s_bal[warp][d] & lt); };
  if (valid) {
    if (p.sp32) {  // R % 8 == 0, rows 32-byte aligned: a whole sector per 8 ranks
      for (int d0 = 0; d0 < p.R; d0 += 8) {
        int32_t q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = goes(d0 + j) ? pos_of(d0 + j) : -1;
        st_v8_b32(p.send_pos + st * p.R + d0, q);
      }
    } else {
      for (int d = 0; d < p.R; ++d) p.send_pos[st * p.R + d] = goes(d) ? pos_of(d) : -1;
    }
    for (int w = 0; w < p.W; ++w) {
      uint32_t word = my_mask[w];
      while (word != 0u) {
        const int d = w * 32 + __ffs(word) - 1;
        word &= word - 1u;
        const int pos = pos_of(d);
        if (pos < 0 || pos >= p.cap) {  // pos < 0 only after a timed-out look-back
          overflow = true;
          continue;
        }
        if (p.rsi_tab != nullptr) {  // the destination's buffers, in peer memory
          p.rsi_tab[d][pos] = t;
          if (meta)
            write_meta(p.ridx_tab != nullptr ? p.ridx_tab[d] + static_cast<size_t>(pos) * p.K
                                             : nullptr,
                       p.rw_tab != nullptr ? p.rw_tab[d] + static_cast<size_t>(pos) * p.K
                                           : nullptr,
                       p.K, d, dk, lk, wk, p.idx32 != 0, p.w32 != 0);
        } else {
          const size_t row = static_cast<size_t>(d) * p.cap + pos;
          p.recv_src_idx[row] = t;
          if (meta)
            write_meta(p.recv_idx != nullptr ? p.recv_idx + row * p.K : nullptr,
                       p.recv_w != nullptr ? p.recv_w + row * p.K : nullptr, p.K, d, dk, lk, wk,
                       p.idx32 != 0, p.w32 != 0);
        }
      }
    }
  }
  if (overflow) report(p.status, EP_STATUS_CAPACITY);

  // ---- expert counts -> num_recv_tokens_per_expert (+ fused layout) -------
  if (count_experts)
    for (int e = tid; e < p.E; e += kScanTile) {
      const int c = s_ehist[e];
      if (c != 0) {
        atomicAdd(&p.expert_cnt[e], c);
        if (p.ntpe_out != nullptr) atomicAdd(&p.expert_cnt[p.E + s * p.E + e], c);
      }
    }
  pdl_trigger();
  if ((p.finalise != 0 || p.probe != nullptr) &&
      elect_last_cta(&p.head->done, static_cast<uint32_t>(p.num_tiles), &s_last)) {
    // one CTA finalises: loads are issued in batches of 8 so that the loop
    // does not wait one L2 round trip per element
    constexpr int B = 8;
    if (p.finalise != 0 && p.nrte != nullptr)
      for (int e0 = 0; e0 < p.E; e0 += kScanTile * B) {
        int v[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int e = e0 + b * kScanTile + tid;
          v[b] = e < p.E ? __ldcg(&p.expert_cnt[e]) : 0;
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int e = e0 + b * kScanTile + tid;
          int n = v[b];
          if (p.align > 1) n = (n + p.align - 1) / p.align * p.align;
          if (e < p.E) p.nrte[e] = n;
        }
      }
    if (p.finalise != 0 && p.ntpe_out != nullptr)
      for (int i0 = 0; i0 < p.R * p.E; i0 += kScanTile * B) {
        int v[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int i = i0 + b * kScanTile + tid;
          v[b] = i < p.R * p.E ? __ldcg(&p.expert_cnt[p.E + i]) : 0;
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int i = i0 + b * kScanTile + tid;
          if (i < p.R * p.E) p.ntpe_out[i] = v[b];
        }
      }
    if (p.finalise != 0 && p.ntpr_out != nullptr)  // tokens of s to d = P[s][d] - P[s-1][d]
      for (int i = tid; i < p.R * p.R; i += kScanTile) {
        const int prev = i >= p.R ? __ldcg(&p.P[i - p.R]) : 0;
        p.ntpr_out[i] = __ldcg(&p.P[i]) - prev;
      }
    if (p.probe != nullptr && tid == 0) {  // full-grid time of this launch
      const unsigned long long end = globaltimer();
      const unsigned long long start = ~atomicAdd(p.probe_state, 0ull);
      atomicAdd(&p.probe[0], end - start);
      atomicAdd(&p.probe[1], 1ull);
      p.probe[2] = start;
      p.probe[3] = end;
    }
  }
  if (p.rsi_tab != nullptr) __threadfence_system();  // stores into peers' memory
}

// ---------------------------------------------------------------------------
// Row scatter.  One thread per destination rank (blockDim = 32 * ceil(R/32)),
// thread 0 also drives the loads.  Each token is cut into items: `nchunks`
// chunks of its data row and, for FP8 input, one item for its scales row.
// CTA b owns tokens b, b + grid, b + 2*grid, ...; stage i % S holds item i.
// Loads run S - 1 items ahead; before a stage is reloaded every thread waits
// until its own bulk stores from that stage have finished reading it.
// ---------------------------------------------------------------------------

// Launch shape, from sweeps on B200 (stages x chunk x CTAs per SM), 2 CTAs
// per SM in both cases:
//  - rows > 8 KB (R=8, H=7168): ~3.5 KB chunks, 4 stages (~28 KB in flight per
//    SM); deeper pipelines oversubscribe HBM with this write-heavy mix (-1..7%);
//  - rows <= 8 KB (R=16, H=4096, skewed routing): one chunk per row, 8 stages;
//    20% faster there than the long-row shape.
constexpr int kCopyStages = 4;
constexpr int kCopyStagesShort = 8;
constexpr int kCopyChunkMax = 4096;
constexpr int kCopyShortRow = 8192;
constexpr int kCopyMaxCtasPerSm = 2;

// bf16 rows only (the headline path): the row scatter described above.
//
// kTab: the destinations' receive buffers are given by a table of R pointers
// (one rank of a sharded job: peers' memory); else they are slices d * cap of
// recv_x.  kTimed: the kernel is the row-copy phase of the phase timers (tm);
// the untimed form never reads tm.
template <int S, bool kTab, bool kTimed>
__global__ void __launch_bounds__(kMaxRanks)
    dispatch_copy_rows_kernel(const uint8_t *__restrict__ x, const int32_t *__restrict__ send_pos,
                         uint8_t *__restrict__ recv_x, uint8_t *const *recv_tab, int R,
                         long num_tok, int row_bytes, int chunk_bytes, int nchunks,
                         int stage_stride, int cap, int32_t *status,
                         unsigned long long timeout_ns, PhaseTimer *tm) {
  pdl_wait();
  unsigned long long begun = 0ull;
  if constexpr (kTimed) begun = timer_begin(tm);
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
  uint8_t *buf = smem + 128;
  const int tid = threadIdx.x;
  const int d = tid;
  uint8_t *my_rows = nullptr;  // this thread's destination buffer
  if (kTab) {
    if (d < R) my_rows = recv_tab[d];
  } else {
    my_rows = recv_x + static_cast<long>(d) * cap * row_bytes;
  }

  const long ntok_cta =
      static_cast<long>(blockIdx.x) < num_tok ? (num_tok - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const long nitems = ntok_cta * nchunks;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < S; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto token_of = [&](long i) -> long {
    return static_cast<long>(blockIdx.x) + (i / nchunks) * static_cast<long>(gridDim.x);
  };
  auto issue_load = [&](long i, int stg) {
    const long u = token_of(i);
    const int off = static_cast<int>(i % nchunks) * chunk_bytes;
    const int nb = min(chunk_bytes, row_bytes - off);
    mbar_arrive_expect_tx(&bars[stg], static_cast<uint32_t>(nb));
    bulk_g2s_hint(buf + stg * stage_stride, x + u * row_bytes + off, static_cast<uint32_t>(nb),
                  &bars[stg], l2_evict_first_policy());
  };
  auto load_pos = [&](long i) -> int {
    return d < R ? __ldg(send_pos + token_of(i) * R + d) : -1;
  };

  int sp[S];
#pragma unroll
  for (int k = 0; k < S; ++k) sp[k] = -1;
#pragma unroll
  for (int k = 0; k < S - 1; ++k) {
    if (k < nitems) {
      if (tid == 0) issue_load(k, k);
      sp[k] = load_pos(k);
    }
  }

  bool all_ok = true;
  long stop = nitems;  // first item whose load may still be in flight on failure
  for (long base = 0; base < nitems && all_ok; base += S) {
    const uint32_t parity = static_cast<uint32_t>((base / S) & 1);
#pragma unroll
    for (int st = 0; st < S; ++st) {
      const long i = base + st;
      if (i >= nitems) break;
      const bool ok = mbar_wait_bounded(&bars[st], parity, timeout_ns);
      const int chunk = static_cast<int>(i % nchunks);
      if (ok && sp[st] >= 0) {  // sp < 0: no copy to this rank
        if (sp[st] < cap) {
          const int off = chunk * chunk_bytes;
          const int nb = min(chunk_bytes, row_bytes - off);
          bulk_s2g(my_rows + static_cast<long>(sp[st]) * row_bytes + off,
                   buf + st * stage_stride, static_cast<uint32_t>(nb));
        } else if (chunk == 0) {
          report(status, EP_STATUS_CAPACITY);
        }
      }
      bulk_commit();
      bulk_wait_read<1>();
      all_ok = __syncthreads_and(ok) != 0;
      if (!all_ok) {
        stop = i;
        break;
      }
      const long j = i + S - 1;
      const int ps = (st + S - 1) % S;
      if (j < nitems) {
        if (tid == 0) issue_load(j, ps);
        sp[ps] = load_pos(j);
      }
    }
  }
  pdl_trigger();
  bulk_wait_all<0>();
  if (kTab) __threadfence_system();  // the rows went to peers' memory
  if (!all_ok) {
    report(status, EP_STATUS_WAIT_TIMEOUT);
    if (tid == 0) {
      // drain loads still in flight before the CTA's shared memory goes away
      const long end = min(nitems, stop + S - 1);
      for (long k = stop; k < end; ++k)
        (void)mbar_wait_bounded(&bars[k % S], static_cast<uint32_t>((k / S) & 1), timeout_ns);
    }
  }
  if constexpr (kTimed) timer_end(tm, begun);
}


// How the scales row of a token reaches shared memory.
enum ScaleMode : int {
  kScalesNone = 0,      // bf16 input: no scales
  kScalesBulk = 1,      // row-major, rows a multiple of 16 bytes: bulk copy
  kScalesGatherRow = 2, // row-major, other sizes: threads load
  kScalesGatherCol = 3  // column-major [R][H/128][T]: threads gather
};

struct CopyArgs {
  const uint8_t *x;       // data rows [R*T][row_bytes]
  const float *xs;        // scales (FP8 input) or nullptr
  const int32_t *send_pos;
  uint8_t *recv_x;        // [R][cap][row_bytes]
  float *recv_s;          // [R][cap][nblk] or nullptr
  int R, T, cap;
  long num_tok;
  int row_bytes, chunk_bytes, nchunks, stage_stride;
  int nblk, sc_mode, sc_store_bulk;
  int32_t *status;
  unsigned long long timeout_ns;
  PhaseTimer *tm;  // the row-copy phase timer (or nullptr)
};

template <int S, bool kScales>
__global__ void __launch_bounds__(kMaxRanks) dispatch_copy_planes_kernel(CopyArgs a) {
  pdl_wait();
  const unsigned long long begun = timer_begin(a.tm);
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
  uint8_t *buf = smem + 128;
  const int tid = threadIdx.x;
  const int d = tid;
  const int ipt = a.nchunks + (kScales ? 1 : 0);  // items per token
  const int sc_bytes = a.nblk * 4;

  const long ntok_cta = static_cast<long>(blockIdx.x) < a.num_tok
                            ? (a.num_tok - 1 - blockIdx.x) / gridDim.x + 1
                            : 0;
  const long nitems = ntok_cta * ipt;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < S; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // Item cursors, advanced one item at a time (no divisions on the path):
  // `is_*` for the next item to load, `cs_*` for the next item to use.
  long is_tok = blockIdx.x;  // global token index of the item to load
  int is_sub = 0;
  long cs_tok = blockIdx.x;
  int cs_sub = 0;
  int sp[S];                 // send_pos of the item held by each stage
  // Threads past R read rank R-1's entry and ignore it: the load then needs
  // no select, so its result lands in sp[] untouched until S-1 items later
  // (a select or a register copy would stall the warp on the load).
  const bool mine = d < a.R;
  const int dd = mine ? d : a.R - 1;

  auto issue_next = [&](int stg) -> int {  // all threads; returns this thread's pos
    if (tid == 0) {
      if (!kScales || is_sub < a.nchunks) {
        const int off = is_sub * a.chunk_bytes;
        const int nb = min(a.chunk_bytes, a.row_bytes - off);
        mbar_arrive_expect_tx(&bars[stg], static_cast<uint32_t>(nb));
        bulk_g2s_hint(buf + stg * a.stage_stride, a.x + is_tok * a.row_bytes + off,
                      static_cast<uint32_t>(nb), &bars[stg], l2_evict_first_policy());
      } else if (a.sc_mode == kScalesBulk) {
        mbar_arrive_expect_tx(&bars[stg], static_cast<uint32_t>(sc_bytes));
        bulk_g2s(buf + stg * a.stage_stride, a.xs + is_tok * a.nblk,
                 static_cast<uint32_t>(sc_bytes), &bars[stg]);
      } else {
        mbar_arrive(&bars[stg]);  // gathered by the threads when the item is used
      }
    }
    const int pos = __ldg(a.send_pos + is_tok * a.R + dd);
    if (++is_sub == ipt) {
      is_sub = 0;
      is_tok += gridDim.x;
    }
    return pos;
  };

#pragma unroll
  for (int k = 0; k < S; ++k) sp[k] = -1;
#pragma unroll
  for (int k = 0; k < S - 1; ++k)
    if (k < nitems) sp[k] = issue_next(k);

  bool all_ok = true;
  long stop = nitems;  // first item whose load may still be in flight on failure
  for (long base = 0; base < nitems && all_ok; base += S) {
    const uint32_t parity = static_cast<uint32_t>((base / S) & 1);
#pragma unroll
    for (int st = 0; st < S; ++st) {
      const long i = base + st;
      if (i >= nitems) break;
      const bool ok = mbar_wait_bounded(&bars[st], parity, a.timeout_ns);
      const int sub = cs_sub;
      uint8_t *stage = buf + st * a.stage_stride;
      if (kScales && sub == a.nchunks && a.sc_mode >= kScalesGatherRow) {  // uniform in CTA
        float *f = reinterpret_cast<float *>(stage);
        for (int j = tid; j < a.nblk; j += blockDim.x) {
          if (a.sc_mode == kScalesGatherRow) {
            f[j] = __ldg(a.xs + cs_tok * a.nblk + j);
          } else {
            const long s = cs_tok / a.T, t = cs_tok % a.T;
            f[j] = __ldg(a.xs + (s * a.nblk + j) * a.T + t);
          }
        }
        fence_proxy_async_smem();
        __syncthreads();
      }
      const int pos = sp[st];
      if (ok && mine && pos >= 0) {  // pos < 0: no copy to this rank
        const long row = static_cast<long>(d) * a.cap + pos;
        if (pos >= a.cap) {
          if (sub == 0) report(a.status, EP_STATUS_CAPACITY);
        } else if (!kScales || sub < a.nchunks) {
          const int off = sub * a.chunk_bytes;
          const int nb = min(a.chunk_bytes, a.row_bytes - off);
          bulk_s2g(a.recv_x + row * a.row_bytes + off, stage, static_cast<uint32_t>(nb));
        } else if (a.sc_store_bulk) {
          bulk_s2g(a.recv_s + row * a.nblk, stage, static_cast<uint32_t>(sc_bytes));
        } else {
          const float *f = reinterpret_cast<const float *>(stage);
          for (int j = 0; j < a.nblk; ++j) a.recv_s[row * a.nblk + j] = f[j];
        }
      }
      bulk_commit();
      if (++cs_sub == ipt) {
        cs_sub = 0;
        cs_tok += gridDim.x;
      }
      bulk_wait_read<1>();
      all_ok = __syncthreads_and(ok) != 0;
      if (!all_ok) {
        stop = i;
        break;
      }
      const int ps = (st + S - 1) % S;
      if (i + S - 1 < nitems) sp[ps] = issue_next(ps);
    }
  }
  pdl_trigger();
  bulk_wait_all<0>();
  if (!all_ok) {
    report(a.status, EP_STATUS_WAIT_TIMEOUT);
    if (tid == 0) {
      // drain loads still in flight before the CTA's shared memory goes away
      const long end = min(nitems, stop + S - 1);
      for (long k = stop; k < end; ++k)
        (void)mbar_wait_bounded(&bars[k % S], static_cast<uint32_t>((k / S) & 1), a.timeout_ns);
    }
  }
  timer_end(a.tm, begun);
}

}  // namespace
}  // namespace ep

extern "C" EP_API size_t ep_dispatch_workspace_bytes(int num_ranks, int num_tokens,
                                                     int num_experts) {
  using namespace ep;
  if (num_ranks < 1 || num_tokens < 0 || num_experts < 0) return 0;
  const long tiles = static_cast<long>(num_ranks) * ((num_tokens + kScanTile - 1) / kScanTile);
  // expert counters: all sources [E], then per source [R][E] (fused layout)
  return scan_workspace_bytes(tiles, num_ranks,
                              static_cast<long>(num_experts) * (1L + num_ranks));
}

namespace ep {
namespace {

// After the scan.  recv_topk_idx rows from recv_count[d] to cap - 1 := -1
// (grid: x over the rows, y over the destination ranks; 16-byte stores when
// a row of K int64 is a multiple of 16 bytes), and the counts the scan
// gathered become the call's outputs, spread over the whole grid: aligned
// per-expert receive counts (nrte) and, for the fused layout, every source's
// tokens per expert (ntpe_out) and per rank (ntpr_out = P[s] - P[s-1]).
// Any of recv_idx, nrte, ntpe_out, ntpr_out may be nullptr.
struct NotifyFinishParams {
  const int32_t *recv_count;
  int cap, K;
  int64_t *recv_idx;
  const int32_t *expert_cnt;  // [E] all sources, then [R][E] per source
  const int32_t *P;
  int R, E, align;
  int32_t *nrte, *ntpe_out, *ntpr_out;
  PhaseTimer *tm;  // ends the notify phase timer (or nullptr)
};

template <bool kTimed>
__global__ void __launch_bounds__(256) notify_finish_kernel(NotifyFinishParams f) {
  pdl_wait();
  pdl_trigger();
  if (f.recv_idx != nullptr) {
    const int d = blockIdx.y;
    const long first = min(max(f.recv_count[d], 0), f.cap);
    int64_t *base = f.recv_idx + static_cast<long>(d) * f.cap * f.K;
    const long lo = first * f.K, hi = static_cast<long>(f.cap) * f.K;  // in int64 elements
    const long step = static_cast<long>(gridDim.x) * blockDim.x;
    if ((f.K & 1) == 0) {
      const longlong2 v = make_longlong2(-1, -1);
      for (long i = lo / 2 + static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
           i < hi / 2; i += step)
        reinterpret_cast<longlong2 *>(base)[i] = v;
    } else {
      for (long i = lo + static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; i < hi;
           i += step)
        base[i] = -1;
    }
  }
  const long nthr = static_cast<long>(gridDim.x) * gridDim.y * blockDim.x;
  const long me = (static_cast<long>(blockIdx.y) * gridDim.x + blockIdx.x) * blockDim.x +
                  threadIdx.x;
  if (f.nrte != nullptr)
    for (long e = me; e < f.E; e += nthr) {
      int n = __ldcg(&f.expert_cnt[e]);
      if (f.align > 1) n = (n + f.align - 1) / f.align * f.align;
      f.nrte[e] = n;
    }
  if (f.ntpe_out != nullptr)
    for (long i = me; i < static_cast<long>(f.R) * f.E; i += nthr)
      f.ntpe_out[i] = __ldcg(&f.expert_cnt[f.E + i]);
  if (f.ntpr_out != nullptr)
    for (long i = me; i < static_cast<long>(f.R) * f.R; i += nthr)
      f.ntpr_out[i] = __ldcg(&f.P[i]) - (i >= f.R ? __ldcg(&f.P[i - f.R]) : 0);
  if constexpr (kTimed) timer_end(f.tm, 0ull);  // begun by the zeroing kernel
}

// 32-byte stores need rows that are whole multiples of 32 bytes and a
// 32-byte-aligned base (peer buffers are allocation-aligned).
void set_store_widths(DispatchScanParams &p) {
  auto al32 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 31u) == 0; };
  p.idx32 = (p.K % 4 == 0) && (p.ridx_tab != nullptr || (p.recv_idx != nullptr && al32(p.recv_idx)));
  p.w32 = (p.K % 8 == 0) && (p.rw_tab != nullptr || (p.recv_w != nullptr && al32(p.recv_w)));
  p.sp32 = (p.R % 8 == 0) && al32(p.send_pos);
}

// A2 (+ received metadata): the scan kernel.  Arguments already checked.
int notify_impl(const int64_t *topk_idx, const float *topk_weights,
                const uint8_t *is_token_in_rank, int R, int T, int K, int E, int align, int cap,
                int64_t *recv_topk_idx, float *recv_topk_weights, int32_t *recv_src_idx,
                int32_t *rank_prefix_matrix, int32_t *recv_count,
                int32_t *num_recv_tokens_per_expert, int32_t *send_pos, int32_t *ntpr_out,
                int32_t *ntpe_out, uint8_t *in_rank_out, void *workspace, int32_t *status,
                cudaStream_t stream) {
  if (T == 0) {  // nothing to route
    if ((ntpr_out != nullptr &&
         cudaMemsetAsync(ntpr_out, 0, sizeof(int32_t) * R * R, stream) != cudaSuccess) ||
        (ntpe_out != nullptr &&
         cudaMemsetAsync(ntpe_out, 0, sizeof(int32_t) * R * static_cast<size_t>(E), stream) !=
             cudaSuccess))
      return EP_ERR_CUDA;
    if (cudaMemsetAsync(rank_prefix_matrix, 0, sizeof(int32_t) * R * R, stream) != cudaSuccess ||
        cudaMemsetAsync(recv_count, 0, sizeof(int32_t) * R, stream) != cudaSuccess)
      return EP_ERR_CUDA;
    if (num_recv_tokens_per_expert != nullptr &&
        cudaMemsetAsync(num_recv_tokens_per_expert, 0, sizeof(int32_t) * E, stream) !=
            cudaSuccess)
      return EP_ERR_CUDA;
    if (recv_topk_idx != nullptr && cap > 0 &&
        cudaMemsetAsync(recv_topk_idx, 0xFF, sizeof(int64_t) * R * static_cast<size_t>(cap) * K,
                        stream) != cudaSuccess)
      return EP_ERR_CUDA;
    return EP_OK;
  }
  const int Ectr = topk_idx != nullptr ? E : 0;
  const size_t need = ep_dispatch_workspace_bytes(R, T, Ectr);
  // zeroed by a kernel chained to the scan, which first asks L2 for the ids
  PhaseTimer *const tm = phase_timer(kPhaseNotify);
  if (zero_prefetch(workspace, need, nullptr, 0, topk_idx,
                    topk_idx != nullptr ? static_cast<long>(R) * T * K * 8 : 0L, stream,
                    tm) != EP_OK)
    return EP_ERR_CUDA;

  const int tiles_per_src = (T + kScanTile - 1) / kScanTile;
  const long num_tiles = static_cast<long>(R) * tiles_per_src;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  DispatchScanParams p;
  p.topk_idx = topk_idx;
  p.topk_w = topk_weights;
  p.in_rank = is_token_in_rank;
  p.R = R;
  p.T = T;
  p.K = K;
  p.E = E;
  p.El = topk_idx != nullptr ? E / R : 1;
  p.el_div = make_fastdiv(p.El);
  p.cap = cap;
  p.align = align;
  p.tiles_per_src = tiles_per_src;
  p.num_tiles = static_cast<int>(num_tiles);
  p.W = (R + 31) / 32;
  p.send_pos = send_pos;
  p.recv_src_idx = recv_src_idx;
  p.recv_idx = recv_topk_idx;
  p.recv_w = recv_topk_weights;
  p.P = rank_prefix_matrix;
  p.recv_count = recv_count;
  p.nrte = num_recv_tokens_per_expert;
  p.ntpr_out = ntpr_out;
  p.ntpe_out = ntpe_out;
  p.in_rank_out = in_rank_out;
  p.dst_base = nullptr;
  p.rsi_tab = nullptr;
  p.ridx_tab = nullptr;
  p.rw_tab = nullptr;
  p.probe_state = nullptr;
  p.probe = nullptr;
  p.finalise = 0;  // notify_finish_kernel writes the counts after the scan
  p.head = reinterpret_cast<ScanHeader *>(ws);
  p.expert_cnt = reinterpret_cast<int32_t *>(ws + sizeof(ScanHeader));
  const int counters = Ectr * (1 + R);
  p.desc = reinterpret_cast<uint64_t *>(ws + sizeof(ScanHeader) +
                                        static_cast<size_t>((counters + 3) & ~3) * 4);
  p.status = status;
  const WaitConfig wc = wait_config();
  p.timeout_ns = wc.timeout_ns;
  p.flags = wc.flags;
  set_store_widths(p);
  cudaError_t launched;
  if (topk_idx != nullptr && K > 8)
    launched = launch_pdl(dispatch_scan_kernel<16>,
        dim3(static_cast<unsigned>(num_tiles)), dim3(kScanTile), 0, stream,
        p);
  else
    launched = launch_pdl(dispatch_scan_kernel<8>,
        dim3(static_cast<unsigned>(num_tiles)), dim3(kScanTile), 0, stream,
        p);
  if (launch_status(launched) != EP_OK) return EP_ERR_CUDA;
  // rows past the receive count read -1 (fixed worst-case capacity), and the
  // gathered counts become the outputs
  NotifyFinishParams f;
  f.recv_count = recv_count;
  f.cap = cap;
  f.K = K;
  f.recv_idx = cap > 0 ? recv_topk_idx : nullptr;
  f.expert_cnt = p.expert_cnt;
  f.P = rank_prefix_matrix;
  f.R = R;
  f.E = E;
  f.align = align;
  f.nrte = num_recv_tokens_per_expert;
  f.ntpe_out = ntpe_out;
  f.ntpr_out = ntpr_out;
  f.tm = tm;
  const long words = f.recv_idx != nullptr ? static_cast<long>(cap) * K / ((K & 1) == 0 ? 2 : 1)
                                           : 0L;
  const int bx = static_cast<int>(std::max<long>(1L, std::min<long>((words + 255) / 256, 64)));
  launched = tm != nullptr
                 ? launch_pdl(notify_finish_kernel<true>, dim3(bx, R), dim3(256), 0, stream, f)
                 : launch_pdl(notify_finish_kernel<false>, dim3(bx, R), dim3(256), 0, stream, f);
  return launch_status(launched);
}

// A3 rows: the bulk-copy kernel.  Arguments already checked.  `xs` (FP8
// scales, [R][T][nblk] or, col_major, [R][nblk][T]) may be nullptr.
int copy_impl(const void *x, const float *xs, int col_major, int nblk, const int32_t *send_pos,
              int R, int T, int row_bytes, int cap, void *recv_x, float *recv_s,
              int32_t *status, cudaStream_t stream, void *const *recv_tab = nullptr,
              int num_src = -1) {
  if (T == 0 || cap == 0) return EP_OK;
  CopyArgs a;
  a.x = static_cast<const uint8_t *>(x);
  a.xs = xs;
  a.send_pos = send_pos;
  a.recv_x = static_cast<uint8_t *>(recv_x);
  a.recv_s = recv_s;
  a.R = R;
  a.T = T;
  a.cap = cap;
  a.num_tok = static_cast<long>(num_src < 0 ? R : num_src) * T;  // source tokens of the call
  a.row_bytes = row_bytes;
  const bool short_rows = row_bytes <= kCopyShortRow;
  a.nchunks = short_rows ? 1 : (row_bytes + kCopyChunkMax - 1) / kCopyChunkMax;
  a.chunk_bytes = ((row_bytes + a.nchunks - 1) / a.nchunks + 15) & ~15;
  a.nblk = xs != nullptr ? nblk : 0;
  const int sc_bytes = a.nblk * 4;
  const bool rows16 = (sc_bytes % 16) == 0;
  if (xs == nullptr)
    a.sc_mode = kScalesNone;
  else if (col_major)
    a.sc_mode = kScalesGatherCol;
  else if (rows16 && (reinterpret_cast<uintptr_t>(xs) & 15u) == 0)
    a.sc_mode = kScalesBulk;
  else
    a.sc_mode = kScalesGatherRow;
  a.sc_store_bulk = xs != nullptr && rows16 && (reinterpret_cast<uintptr_t>(recv_s) & 15u) == 0;
  a.stage_stride = (std::max(a.chunk_bytes, sc_bytes) + 127) & ~127;
  a.status = status;
  a.timeout_ns = wait_config().timeout_ns;
  a.tm = recv_tab == nullptr ? phase_timer(kPhaseCopy) : nullptr;
  const int stages = short_rows ? kCopyStagesShort : kCopyStages;
  // at most kCopyMaxCtasPerSm CTAs on an SM, also when scheduled early
  const size_t smem =
      spread_smem(128 + static_cast<size_t>(stages) * a.stage_stride, kCopyMaxCtasPerSm);
  const int threads = 32 * ((R + 31) / 32);
  const void *fn;
  if (xs != nullptr)
    fn = short_rows ? reinterpret_cast<const void *>(dispatch_copy_planes_kernel<kCopyStagesShort, true>)
                    : reinterpret_cast<const void *>(dispatch_copy_planes_kernel<kCopyStages, true>);
  else if (recv_tab != nullptr)
    fn = short_rows
             ? reinterpret_cast<const void *>(dispatch_copy_rows_kernel<kCopyStagesShort, true, false>)
             : reinterpret_cast<const void *>(dispatch_copy_rows_kernel<kCopyStages, true, false>);
  else if (a.tm != nullptr)
    fn = short_rows
             ? reinterpret_cast<const void *>(dispatch_copy_rows_kernel<kCopyStagesShort, false, true>)
             : reinterpret_cast<const void *>(dispatch_copy_rows_kernel<kCopyStages, false, true>);
  else
    fn = short_rows
             ? reinterpret_cast<const void *>(dispatch_copy_rows_kernel<kCopyStagesShort, false, false>)
             : reinterpret_cast<const void *>(dispatch_copy_rows_kernel<kCopyStages, false, false>);
  if (ensure_dynamic_smem(fn, smem) != EP_OK) return EP_ERR_CUDA;
  const long grid = std::min<long>(
      a.num_tok,
      static_cast<long>(std::min(kCopyMaxCtasPerSm, ctas_per_sm(fn, threads, smem))) * num_sms());
  const dim3 g(static_cast<unsigned>(grid)), b(threads);
  cudaError_t launched;
  if (xs != nullptr) {
    if (short_rows)
      launched = launch_pdl(dispatch_copy_planes_kernel<kCopyStagesShort, true>,
          dim3(g), dim3(b), smem, stream,
        a);
    else
      launched = launch_pdl(dispatch_copy_planes_kernel<kCopyStages, true>,
          dim3(g), dim3(b), smem, stream,
        a);
  } else {
    auto *tab = reinterpret_cast<uint8_t *const *>(recv_tab);
    if (recv_tab != nullptr && short_rows)
      launched = launch_pdl(dispatch_copy_rows_kernel<kCopyStagesShort, true, false>, g, b, smem, stream,
          a.x, a.send_pos, a.recv_x, tab, a.R, a.num_tok, a.row_bytes, a.chunk_bytes, a.nchunks,
          a.stage_stride, a.cap, a.status, a.timeout_ns, a.tm);
    else if (recv_tab != nullptr)
      launched = launch_pdl(dispatch_copy_rows_kernel<kCopyStages, true, false>, g, b, smem, stream,
          a.x, a.send_pos, a.recv_x, tab, a.R, a.num_tok, a.row_bytes, a.chunk_bytes, a.nchunks,
          a.stage_stride, a.cap, a.status, a.timeout_ns, a.tm);
    else if (short_rows && a.tm != nullptr)
      launched = launch_pdl(dispatch_copy_rows_kernel<kCopyStagesShort, false, true>, g, b, smem,
          stream, a.x, a.send_pos, a.recv_x, tab, a.R, a.num_tok, a.row_bytes, a.chunk_bytes,
          a.nchunks, a.stage_stride, a.cap, a.status, a.timeout_ns, a.tm);
    else if (short_rows)
      launched = launch_pdl(dispatch_copy_rows_kernel<kCopyStagesShort, false, false>, g, b, smem,
          stream, a.x, a.send_pos, a.recv_x, tab, a.R, a.num_tok, a.row_bytes, a.chunk_bytes,
          a.nchunks, a.stage_stride, a.cap, a.status, a.timeout_ns, a.tm);
    else if (a.tm != nullptr)
      launched = launch_pdl(dispatch_copy_rows_kernel<kCopyStages, false, true>, g, b, smem,
          stream, a.x, a.send_pos, a.recv_x, tab, a.R, a.num_tok, a.row_bytes, a.chunk_bytes,
          a.nchunks, a.stage_stride, a.cap, a.status, a.timeout_ns, a.tm);
    else
      launched = launch_pdl(dispatch_copy_rows_kernel<kCopyStages, false, false>, g, b, smem,
          stream, a.x, a.send_pos, a.recv_x, tab, a.R, a.num_tok, a.row_bytes, a.chunk_bytes,
          a.nchunks, a.stage_stride, a.cap, a.status, a.timeout_ns, a.tm);
  }
  return launch_status(launched);
}

// Checks shared by ep_dispatch, ep_notify_dispatch and ep_dispatch_noalloc,
// except the workspace (check_workspace).
int check_notify_shape(const int64_t *topk_idx, const float *topk_weights,
                       const uint8_t *is_token_in_rank, int R, int T, int K, int E, int align,
                       int cap, const int64_t *recv_topk_idx, const float *recv_topk_weights,
                       const int32_t *recv_src_idx, const int32_t *rank_prefix_matrix,
                       const int32_t *recv_count, const int32_t *nrte, const int32_t *send_pos) {
  if (R < 1 || R > kMaxRanks || T < 0 || cap < 0 || align < 1) return EP_ERR_INVALID_ARG;
  if (rank_prefix_matrix == nullptr || recv_count == nullptr) return EP_ERR_INVALID_ARG;
  const bool meta = recv_topk_idx != nullptr || recv_topk_weights != nullptr || nrte != nullptr;
  if (meta && (K < 1 || K > kMaxTopk || E < 1 || E > kMaxExperts || E % R != 0))
    return EP_ERR_INVALID_ARG;
  if (T == 0) return EP_OK;  // an empty tensor's pointers may be NULL
  if (topk_idx == nullptr && is_token_in_rank == nullptr) return EP_ERR_INVALID_ARG;
  if (topk_idx != nullptr && (K < 1 || K > kMaxTopk || E < 1 || E > kMaxExperts || E % R != 0))
    return EP_ERR_INVALID_ARG;
  if (meta && topk_idx == nullptr) return EP_ERR_INVALID_ARG;
  if (recv_topk_weights != nullptr && topk_weights == nullptr) return EP_ERR_INVALID_ARG;
  if (send_pos == nullptr || recv_src_idx == nullptr) return EP_ERR_INVALID_ARG;
  if (static_cast<long>(R) * ((T + kScanTile - 1) / kScanTile) > 0x7fffffffL ||
      static_cast<long>(R) * T > 0x7fffffffL)
    return EP_ERR_UNSUPPORTED;
  return EP_OK;
}

// The caller's workspace of a call that passed check_notify_shape.
int check_workspace(const int64_t *topk_idx, int R, int T, int E, const void *workspace,
                    size_t workspace_bytes) {
  if (T == 0) return EP_OK;
  const size_t need = ep_dispatch_workspace_bytes(R, T, topk_idx != nullptr ? E : 0);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return EP_ERR_INVALID_ARG;
  return EP_OK;
}

int check_notify_args(const int64_t *topk_idx, const float *topk_weights,
                      const uint8_t *is_token_in_rank, int R, int T, int K, int E, int align,
                      int cap, const int64_t *recv_topk_idx, const float *recv_topk_weights,
                      const int32_t *recv_src_idx, const int32_t *rank_prefix_matrix,
                      const int32_t *recv_count, const int32_t *nrte, const int32_t *send_pos,
                      const void *workspace, size_t workspace_bytes) {
  const int rc = check_notify_shape(topk_idx, topk_weights, is_token_in_rank, R, T, K, E, align,
                                    cap, recv_topk_idx, recv_topk_weights, recv_src_idx,
                                    rank_prefix_matrix, recv_count, nrte, send_pos);
  if (rc != EP_OK) return rc;
  return check_workspace(topk_idx, R, T, E, workspace, workspace_bytes);
}

int check_copy_args(const void *x, const int32_t *send_pos, int R, int T, int H, int cap,
                    const void *recv_x) {
  if (R < 1 || R > kMaxRanks || T < 0 || H < 8 || H % 8 != 0 || cap < 0)
    return EP_ERR_INVALID_ARG;
  if (T == 0 || cap == 0) return EP_OK;
  if (x == nullptr || send_pos == nullptr || recv_x == nullptr) return EP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(recv_x) & 15u))
    return EP_ERR_INVALID_ARG;
  if (static_cast<long>(R) * T > 0x7fffffffL) return EP_ERR_UNSUPPORTED;
  return EP_OK;
}

}  // namespace
}  // namespace ep

extern "C" EP_API int ep_notify_dispatch(const int64_t *topk_idx, const float *topk_weights,
                                         const uint8_t *is_token_in_rank, int num_ranks,
                                         int num_tokens, int num_topk, int num_experts,
                                         int expert_alignment, int capacity,
                                         int64_t *recv_topk_idx, float *recv_topk_weights,
                                         int32_t *recv_src_idx, int32_t *rank_prefix_matrix,
                                         int32_t *recv_count,
                                         int32_t *num_recv_tokens_per_expert, int32_t *send_pos,
                                         int32_t *num_tokens_per_rank,
                                         int32_t *num_tokens_per_expert,
                                         uint8_t *is_token_in_rank_out, void *workspace,
                                         size_t workspace_bytes, int32_t *status,
                                         cudaStream_t stream) {
  using namespace ep;
  // the fused layout needs the routing to come from topk_idx
  if ((num_tokens_per_rank != nullptr || num_tokens_per_expert != nullptr ||
       is_token_in_rank_out != nullptr) &&
      (topk_idx == nullptr || is_token_in_rank != nullptr || num_topk < 1 ||
       num_topk > kMaxTopk || num_experts < 1 || num_experts > kMaxExperts ||
       num_ranks < 1 || num_experts % num_ranks != 0))
    return EP_ERR_INVALID_ARG;
  const int rc = check_notify_args(topk_idx, topk_weights, is_token_in_rank, num_ranks,
                                   num_tokens, num_topk, num_experts, expert_alignment, capacity,
                                   recv_topk_idx, recv_topk_weights, recv_src_idx,
                                   rank_prefix_matrix, recv_count, num_recv_tokens_per_expert,
                                   send_pos, workspace, workspace_bytes);
  if (rc != EP_OK) return rc;
  return notify_impl(topk_idx, topk_weights, is_token_in_rank, num_ranks, num_tokens, num_topk,
                     num_experts, expert_alignment, capacity, recv_topk_idx, recv_topk_weights,
                     recv_src_idx, rank_prefix_matrix, recv_count, num_recv_tokens_per_expert,
                     send_pos, num_tokens_per_rank, num_tokens_per_expert, is_token_in_rank_out,
                     workspace, status, stream);
}

extern "C" EP_API int ep_dispatch_cached(const void *x, const int32_t *send_pos, int num_ranks,
                                         int num_tokens, int hidden, int capacity, void *recv_x,
                                         int32_t *status, cudaStream_t stream) {
  using namespace ep;
  const int rc = check_copy_args(x, send_pos, num_ranks, num_tokens, hidden, capacity, recv_x);
  if (rc != EP_OK) return rc;
  return copy_impl(x, nullptr, 0, 0, send_pos, num_ranks, num_tokens, hidden * 2, capacity,
                   recv_x, nullptr, status, stream);
}

extern "C" EP_API int ep_dispatch_cached_fp8(const void *x_e4m3, const float *x_scales,
                                             int scales_col_major, const int32_t *send_pos,
                                             int num_ranks, int num_tokens, int hidden,
                                             int capacity, void *recv_x, float *recv_scales,
                                             int32_t *status, cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, cap = capacity;
  if (R < 1 || R > kMaxRanks || T < 0 || H < 128 || H % 128 != 0 || cap < 0)
    return EP_ERR_INVALID_ARG;
  if (T == 0 || cap == 0) return EP_OK;
  if (x_e4m3 == nullptr || x_scales == nullptr || send_pos == nullptr || recv_x == nullptr ||
      recv_scales == nullptr)
    return EP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x_e4m3) & 15u) || (reinterpret_cast<uintptr_t>(recv_x) & 15u) ||
      (reinterpret_cast<uintptr_t>(x_scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(recv_scales) & 3u))
    return EP_ERR_INVALID_ARG;
  if (static_cast<long>(R) * T > 0x7fffffffL) return EP_ERR_UNSUPPORTED;
  return copy_impl(x_e4m3, x_scales, scales_col_major, H / 128, send_pos, R, T, H, cap, recv_x,
                   recv_scales, status, stream);
}

extern "C" EP_API int ep_dispatch(const void *x, const int64_t *topk_idx,
                                  const float *topk_weights, const uint8_t *is_token_in_rank,
                                  int num_ranks, int num_tokens, int hidden, int num_topk,
                                  int num_experts, int expert_alignment, int capacity,
                                  void *recv_x, int64_t *recv_topk_idx, float *recv_topk_weights,
                                  int32_t *recv_src_idx, int32_t *rank_prefix_matrix,
                                  int32_t *recv_count, int32_t *num_recv_tokens_per_expert,
                                  int32_t *send_pos, void *workspace, size_t workspace_bytes,
                                  int32_t *status, cudaStream_t stream) {
  using namespace ep;
  int rc = check_notify_args(topk_idx, topk_weights, is_token_in_rank, num_ranks, num_tokens,
                             num_topk, num_experts, expert_alignment, capacity, recv_topk_idx,
                             recv_topk_weights, recv_src_idx, rank_prefix_matrix, recv_count,
                             num_recv_tokens_per_expert, send_pos, workspace, workspace_bytes);
  if (rc != EP_OK) return rc;
  rc = check_copy_args(x, send_pos, num_ranks, num_tokens, hidden, capacity, recv_x);
  if (rc != EP_OK) return rc;
  rc = notify_impl(topk_idx, topk_weights, is_token_in_rank, num_ranks, num_tokens, num_topk,
                   num_experts, expert_alignment, capacity, recv_topk_idx, recv_topk_weights,
                   recv_src_idx, rank_prefix_matrix, recv_count, num_recv_tokens_per_expert,
                   send_pos, nullptr, nullptr, nullptr, workspace, status, stream);
  if (rc != EP_OK) return rc;
  return copy_impl(x, nullptr, 0, 0, send_pos, num_ranks, num_tokens, hidden * 2, capacity,
                   recv_x, nullptr, status, stream);
}

// ---------------------------------------------------------------------------
// One rank per GPU (sharded job).  The calling process holds one source rank
// `rank` of R; the counts every rank sends to every destination, gathered by
// the caller's collective, give the rank prefix matrix (the notify step of
// the pages' dispatch); the scan above then runs over this rank's tokens
// alone, offset by the rows lower ranks take in each destination, and writes
// the received metadata and the rows straight into the destinations' receive
// buffers in peer memory.
// ---------------------------------------------------------------------------

namespace ep {
namespace {

// Workspace of a sharded notify: header, the probe's complemented earliest
// start (8 bytes) and the R destination bases, then the look-back
// descriptors of this rank's tiles.
struct ShardWs {
  ScanHeader *head;
  unsigned long long *probe_state;
  int32_t *base;
  uint64_t *desc;
};

ShardWs shard_ws(void *workspace, int R) {
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  ShardWs w;
  w.head = reinterpret_cast<ScanHeader *>(ws);
  w.probe_state = reinterpret_cast<unsigned long long *>(ws + sizeof(ScanHeader));
  w.base = reinterpret_cast<int32_t *>(ws + sizeof(ScanHeader) + 16);
  const long counters = 4 + R;  // probe state (2 ints, padded to 4), bases
  w.desc = reinterpret_cast<uint64_t *>(ws + sizeof(ScanHeader) +
                                        static_cast<size_t>((counters + 3) & ~3L) * 4);
  return w;
}

// P[s][d] = sum over s' <= s of counts[s'][d] (inclusive over source ranks),
// base[d] = P[rank - 1][d] (0 for rank 0), recv_count = P[R - 1][rank], and
// the received slots of each local expert, sum over s of
// expert_counts[s][rank * E_l + j], rounded up to the alignment.
__global__ void __launch_bounds__(256)
    shard_prefix_kernel(const int32_t *__restrict__ counts, const int32_t *__restrict__ ecounts,
                        int R, int E, int rank, int align, int32_t *__restrict__ P,
                        int32_t *__restrict__ base, int32_t *__restrict__ recv_count,
                        int32_t *__restrict__ nrte) {
  pdl_wait();
  pdl_trigger();
  for (int d = threadIdx.x; d < R; d += blockDim.x) {
    int run = 0;
    if (rank == 0) base[d] = 0;
    for (int s = 0; s < R; ++s) {
      run += counts[static_cast<size_t>(s) * R + d];
      P[static_cast<size_t>(s) * R + d] = run;
      if (s == rank - 1) base[d] = run;
    }
    if (d == rank) recv_count[0] = run;
  }
  if (nrte != nullptr) {
    const int El = E / R;
    for (int j = threadIdx.x; j < El; j += blockDim.x) {
      int n = 0;
      for (int s = 0; s < R; ++s) n += ecounts[static_cast<size_t>(s) * E + rank * El + j];
      if (align > 1) n = (n + align - 1) / align * align;
      nrte[j] = n;
    }
  }
}

}  // namespace
}  // namespace ep

extern "C" EP_API size_t ep_shard_workspace_bytes(int num_ranks, int num_tokens) {
  using namespace ep;
  if (num_ranks < 1 || num_tokens < 0) return 0;
  const long tiles = (num_tokens + kScanTile - 1) / kScanTile;
  return scan_workspace_bytes(tiles, num_ranks, 4L + num_ranks);
}

extern "C" EP_API int ep_shard_notify(
    const int64_t *topk_idx, const float *topk_weights, const int32_t *counts,
    const int32_t *expert_counts, int rank, int num_ranks, int num_tokens, int num_topk,
    int num_experts, int expert_alignment, int capacity, int32_t *const *recv_src_idx_peers,
    int64_t *const *recv_topk_idx_peers, float *const *recv_topk_weights_peers,
    int64_t *recv_topk_idx, int32_t *rank_prefix_matrix, int32_t *recv_count,
    int32_t *num_recv_tokens_per_expert, int32_t *send_pos, unsigned long long *notify_probe,
    void *workspace, size_t workspace_bytes, int32_t *status, cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, K = num_topk, E = num_experts;
  const int cap = capacity, align = expert_alignment;
  if (R < 1 || R > kMaxRanks || rank < 0 || rank >= R || T < 0 || cap < 0 || align < 1)
    return EP_ERR_INVALID_ARG;
  if (K < 1 || K > kMaxTopk || E < 1 || E > kMaxExperts || E % R != 0) return EP_ERR_INVALID_ARG;
  if (counts == nullptr || rank_prefix_matrix == nullptr || recv_count == nullptr)
    return EP_ERR_INVALID_ARG;
  if (num_recv_tokens_per_expert != nullptr && expert_counts == nullptr) return EP_ERR_INVALID_ARG;
  if ((recv_topk_idx_peers != nullptr) != (recv_topk_idx != nullptr)) return EP_ERR_INVALID_ARG;
  if (T > 0 && (topk_idx == nullptr || recv_src_idx_peers == nullptr || send_pos == nullptr))
    return EP_ERR_INVALID_ARG;
  if (T > 0 && recv_topk_weights_peers != nullptr && topk_weights == nullptr)
    return EP_ERR_INVALID_ARG;
  const size_t need = ep_shard_workspace_bytes(R, T);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) ||
      (reinterpret_cast<uintptr_t>(notify_probe) & 7u))
    return EP_ERR_INVALID_ARG;

  if (zero_prefetch(workspace, need, nullptr, 0, nullptr, 0, stream) != EP_OK) return EP_ERR_CUDA;
  const ShardWs w = shard_ws(workspace, R);
  cudaError_t launched = launch_pdl(shard_prefix_kernel, dim3(1), dim3(256), 0, stream, counts,
                                    expert_counts, R, E, rank, align, rank_prefix_matrix,
                                    w.base, recv_count, num_recv_tokens_per_expert);
  if (launch_status(launched) != EP_OK) return EP_ERR_CUDA;
  if (T > 0) {
    const int tiles = (T + kScanTile - 1) / kScanTile;
    DispatchScanParams p = {};
    p.topk_idx = topk_idx;
    p.topk_w = topk_weights;
    p.in_rank = nullptr;
    p.R = R;
    p.T = T;
    p.K = K;
    p.E = E;
    p.El = E / R;
    p.el_div = make_fastdiv(p.El);
    p.cap = cap;
    p.align = align;
    p.tiles_per_src = tiles;
    p.num_tiles = tiles;  // one source rank
    p.W = (R + 31) / 32;
    p.send_pos = send_pos;
    p.dst_base = w.base;
    p.rsi_tab = recv_src_idx_peers;
    p.ridx_tab = recv_topk_idx_peers;
    p.rw_tab = recv_topk_weights_peers;
    p.probe_state = notify_probe != nullptr ? w.probe_state : nullptr;
    p.probe = notify_probe;
    p.head = w.head;
    p.desc = w.desc;
    p.status = status;
    const WaitConfig wc = wait_config();
    p.timeout_ns = wc.timeout_ns;
    p.flags = wc.flags;
    set_store_widths(p);
    if (K > 8)
      launched = launch_pdl(dispatch_scan_kernel<16>, dim3(tiles), dim3(kScanTile), 0, stream, p);
    else
      launched = launch_pdl(dispatch_scan_kernel<8>, dim3(tiles), dim3(kScanTile), 0, stream, p);
    if (launch_status(launched) != EP_OK) return EP_ERR_CUDA;
  }
  // this rank's own receive rows past its count read -1 (fixed capacity)
  if (recv_topk_idx != nullptr && cap > 0) {
    NotifyFinishParams f = {};
    f.recv_count = recv_count;
    f.cap = cap;
    f.K = K;
    f.recv_idx = recv_topk_idx;
    const long words = static_cast<long>(cap) * K / ((K & 1) == 0 ? 2 : 1);
    const int bx = static_cast<int>(std::min<long>((words + 255) / 256, 64));
    launched = launch_pdl(notify_finish_kernel<false>, dim3(bx, 1), dim3(256), 0, stream, f);
    return launch_status(launched);
  }
  return EP_OK;
}

extern "C" EP_API int ep_shard_dispatch(const void *x, const int32_t *send_pos, int num_ranks,
                                        int num_tokens, int hidden, int capacity,
                                        void *const *recv_x_peers, int32_t *status,
                                        cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, cap = capacity;
  if (R < 1 || R > kMaxRanks || T < 0 || H < 8 || H % 8 != 0 || cap < 0)
    return EP_ERR_INVALID_ARG;
  if (T == 0 || cap == 0) return EP_OK;
  if (x == nullptr || send_pos == nullptr || recv_x_peers == nullptr) return EP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) & 15u) return EP_ERR_INVALID_ARG;
  return copy_impl(x, nullptr, 0, 0, send_pos, R, T, H * 2, cap, nullptr, nullptr, status, stream,
                   recv_x_peers, 1);
}

// ---------------------------------------------------------------------------
// ep_dispatch_noalloc: ep_dispatch with its scratch in a static device array.
//
// Some callers cannot hand the library a workspace: a host program whose
// device memory is owned by another allocator (a raw cudaMalloc next to that
// pool fails or fragments it), or a latency-critical loop that cannot afford
// cudaMalloc/cudaFree, which may synchronise the device.  For them this entry
// point keeps the look-back scratch in a file-scope __device__ array of
// kNoAllocScratchBytes, which every GPU that loads this library holds until
// the process exits.  It allocates nothing and calls nothing that allocates.
//
// The array's name is only a host-side stand-in in host code; the kernels get
// its device address, looked up with cudaGetSymbolAddress with the device
// current.  The first call on a device does that set-up (make it before any
// stream capture).  Later calls made outside stream capture look the address
// up again, so a device reset (after which the module, and the array, may
// load elsewhere) is harmless; a call made while its stream is capturing uses
// the address of the last call outside capture.  The array is shared by every
// call on a device and keeps the last call's contents; ep_dispatch clears the
// part it uses on the stream before its kernels run, so calls on one stream
// are safe, but calls that overlap on the GPU (other streams, other threads)
// race on it.
// ---------------------------------------------------------------------------

namespace ep {
namespace {

constexpr size_t kNoAllocScratchBytes = 2u << 20;  // 2 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
void *g_noalloc_ptr[kNoAllocMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, or nullptr.
void *noalloc_scratch(cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const bool capturing =
      cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!capturing || g_noalloc_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      g_noalloc_ptr[dev] = nullptr;
      return nullptr;
    }
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace ep

extern "C" EP_API int ep_dispatch_noalloc(
    const void *x, const int64_t *topk_idx, const float *topk_weights,
    const uint8_t *is_token_in_rank, int num_ranks, int num_tokens, int hidden, int num_topk,
    int num_experts, int expert_alignment, int capacity, void *recv_x, int64_t *recv_topk_idx,
    float *recv_topk_weights, int32_t *recv_src_idx, int32_t *rank_prefix_matrix,
    int32_t *recv_count, int32_t *num_recv_tokens_per_expert, int32_t *send_pos,
    int32_t *status, cudaStream_t stream) {
  using namespace ep;
  // ep_dispatch's argument checks first: an invalid call is reported as
  // invalid whatever its size
  int rc = check_notify_shape(topk_idx, topk_weights, is_token_in_rank, num_ranks, num_tokens,
                              num_topk, num_experts, expert_alignment, capacity, recv_topk_idx,
                              recv_topk_weights, recv_src_idx, rank_prefix_matrix, recv_count,
                              num_recv_tokens_per_expert, send_pos);
  if (rc != EP_OK) return rc;
  rc = check_copy_args(x, send_pos, num_ranks, num_tokens, hidden, capacity, recv_x);
  if (rc != EP_OK) return rc;
  const size_t need =
      ep_dispatch_workspace_bytes(num_ranks, num_tokens, topk_idx != nullptr ? num_experts : 0);
  if (need > kNoAllocScratchBytes) return EP_ERR_UNSUPPORTED;  // beyond the static scratch
  void *scratch = noalloc_scratch(stream);
  if (scratch == nullptr) return EP_ERR_CUDA;
  rc = notify_impl(topk_idx, topk_weights, is_token_in_rank, num_ranks, num_tokens, num_topk,
                   num_experts, expert_alignment, capacity, recv_topk_idx, recv_topk_weights,
                   recv_src_idx, rank_prefix_matrix, recv_count, num_recv_tokens_per_expert,
                   send_pos, nullptr, nullptr, nullptr, scratch, status, stream);
  if (rc != EP_OK) return rc;
  return copy_impl(x, nullptr, 0, 0, send_pos, num_ranks, num_tokens, hidden * 2, capacity,
                   recv_x, nullptr, status, stream);
}
