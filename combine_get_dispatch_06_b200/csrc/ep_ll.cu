// ep_ll.cu -- A5 + A6: low-latency dispatch (fused FP8 e4m3 quantisation into
// per-expert slabs) and low-latency combine (top-k weighted gather).
//
// Semantics (DeepEP legacy-test analysis page: low_latency_dispatch with
// use_fp8, its handle (recv_src_info, recv_layout_range), the check that each
// expert's count equals (topk_idx == expert).sum(), and low_latency_combine
// with the check against x * sum of masked weights):
//   - one slab row per (token, expert); rows of expert e ordered by source
//     rank, then token: row = exclusive prefix over the flattened (s, t) order
//     of "token has e", computed here by the same decoupled look-back scan as
//     normal dispatch, with experts as the columns;
//   - per 128-channel block: amax' = max(max|x|, 1e-4), inv = 448 / amax'
//     (IEEE division), q = e4m3(x * inv) rounded to nearest even and
//     saturated (cvt.rn.satfinite), scale = amax' / 448;
//   - combine: acc = fmaf(y, w_k, acc) over slots k ascending, one bf16
//     rounding at the end.
//
// Kernels:
//   ll_scan_kernel      positions, recv_src_info, layout_range, counts
//   ll_dispatch_kernel  one warp per token: read the row once, quantise in
//                       registers (16 lanes per 128-channel block, amax by
//                       xor-shuffles), stage it in shared memory, then one
//                       bulk (TMA) store per destination slab row
//   ll_combine_kernel   one warp per token, up to 16 rows in flight per lane
#include <algorithm>

#include "ep_scan.cuh"

namespace ep {
namespace {

struct LLScanParams {
  const int64_t *topk_idx;
  int R, T, K, E, cap, tiles_per_src, num_tiles;
  int32_t *ll_pos;
  int32_t *recv_src_info;
  int32_t *layout_range;
  int32_t *recv_count;
  ScanHeader *head;
  uint64_t *desc;
  int32_t *status;
  unsigned long long timeout_ns;
  unsigned flags;
};

__global__ void __launch_bounds__(kScanTile) ll_scan_kernel(LLScanParams p) {
  __shared__ int s_tile;
  __shared__ int s_last;
  __shared__ int s_whist[kScanWarps][kMaxExperts];
  __shared__ int s_excl[kMaxExperts];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  if (tid == 0) s_tile = static_cast<int>(atomicAdd(&p.head->ticket, 1u));
  for (int i = tid; i < kScanWarps * kMaxExperts; i += kScanTile) (&s_whist[0][0])[i] = 0;
  __syncthreads();

  const int tile = s_tile;
  const int s = tile / p.tiles_per_src;
  const int t = (tile % p.tiles_per_src) * kScanTile + tid;
  const bool valid = t < p.T;
  const size_t st = static_cast<size_t>(s) * p.T + t;

  // Distinct valid experts of this token (a repeated expert keeps only its
  // first slot in `col`; `ev` keeps every valid id).
  int ev[kMaxTopk], col[kMaxTopk], rnk[kMaxTopk];
  uint32_t pending = 0;
  bool bad = false;
#pragma unroll
  for (int k = 0; k < kMaxTopk; ++k) {
    ev[k] = -1;
    col[k] = -1;
    rnk[k] = 0;
    if (valid && k < p.K) {
      const int64_t e = p.topk_idx[st * p.K + k];
      if (e >= 0 && e < p.E) {
        ev[k] = static_cast<int>(e);
        bool dup = false;
#pragma unroll
        for (int k2 = 0; k2 < k; ++k2) dup |= (col[k2] == ev[k]);
        if (!dup) {
          col[k] = ev[k];
          pending |= 1u << k;
        }
      } else if (e != -1) {
        bad = true;
      }
    }
  }
  if (bad) report(p.status, EP_STATUS_BAD_EXPERT);

  // Rank of each (token, expert) among the warp's tokens that hold that
  // expert: one ballot per distinct expert present in the warp.
  const uint32_t lt = lanemask_lt();
  while (true) {
    const uint32_t any = __ballot_sync(0xffffffffu, pending != 0u);
    if (any == 0u) break;
    const int leader = __ffs(any) - 1;
    int mine = -1;
    if (pending != 0u) {
      const int kf = __ffs(pending) - 1;
#pragma unroll
      for (int k = 0; k < kMaxTopk; ++k)
        if (k == kf) mine = col[k];
    }
    const int c = __shfl_sync(0xffffffffu, mine, leader);
    int kk = -1;
#pragma unroll
    for (int k = 0; k < kMaxTopk; ++k)
      if (col[k] == c && ((pending >> k) & 1u)) kk = k;
    const uint32_t bal = __ballot_sync(0xffffffffu, kk >= 0);
    if (kk >= 0) {
      const int r = __popc(bal & lt);
#pragma unroll
      for (int k = 0; k < kMaxTopk; ++k)
        if (k == kk) rnk[k] = r;
      pending &= ~(1u << kk);
    }
    if (lane == 0) s_whist[warp][c] = __popc(bal);
  }
  __syncthreads();

  const bool publish = (p.flags & EP_DEBUG_SUPPRESS_PUBLISH) == 0;
  const bool first_of_src = (tile % p.tiles_per_src) == 0;
  for (int c = tid; c < p.E; c += kScanTile) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kScanWarps; ++w) {
      const int n = s_whist[w][c];
      s_whist[w][c] = run;
      run += n;
    }
    const uint32_t excl = lookback_column(p.desc, tile, p.E, c, static_cast<uint32_t>(run),
                                          publish, p.timeout_ns, p.status);
    s_excl[c] = static_cast<int>(excl);
    if (first_of_src) p.layout_range[(static_cast<size_t>(c) * p.R + s) * 2] = static_cast<int>(excl);
    if (tile == p.num_tiles - 1) p.recv_count[c] = static_cast<int>(excl) + run;
  }
  __syncthreads();

  if (valid) {
    int pos[kMaxTopk];
    bool oob = false;
#pragma unroll
    for (int k = 0; k < kMaxTopk; ++k) {
      pos[k] = -1;
      if (col[k] >= 0) {
        const int c = col[k];
        const int r = s_excl[c] + s_whist[warp][c] + rnk[k];
        if (r >= 0 && r < p.cap) {
          pos[k] = r;
          p.recv_src_info[static_cast<size_t>(c) * p.cap + r] = t;
        } else {
          oob = true;  // only reachable after a timed-out look-back
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kMaxTopk; ++k) {
      if (k >= p.K) break;
      int v = pos[k];
      if (col[k] < 0 && ev[k] >= 0) {
#pragma unroll
        for (int k2 = 0; k2 < kMaxTopk; ++k2)
          if (k2 < k && col[k2] == ev[k]) v = pos[k2];
      }
      p.ll_pos[st * p.K + k] = v;
    }
    if (oob) report(p.status, EP_STATUS_BAD_POSITION);
  }

  if (elect_last_cta(&p.head->done, static_cast<uint32_t>(p.num_tiles), &s_last)) {
    // rows per (expert, source rank) = next source's first row - this one's
    const int n = p.E * p.R;
    for (int i = tid; i < n; i += kScanTile) {
      const int c = i / p.R;
      const int s2 = i % p.R;
      const size_t o = (static_cast<size_t>(c) * p.R + s2) * 2;
      const int begin = __ldcg(&p.layout_range[o]);
      const int end = (s2 + 1 < p.R) ? __ldcg(&p.layout_range[o + 2]) : __ldcg(&p.recv_count[c]);
      p.layout_range[o + 1] = end - begin;
    }
  }
}

// ---------------------------------------------------------------------------

constexpr int kLLWarps = 4;

__device__ __forceinline__ uint32_t cvt_e4m3x4(float a, float b, float c, float d) {
  // element order in memory: a, b, c, d (a in the lowest byte)
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

template <bool kFP8>
__global__ void __launch_bounds__(kLLWarps * 32)
    ll_dispatch_kernel(const uint8_t *__restrict__ x, const int64_t *__restrict__ topk_idx,
                       const int32_t *__restrict__ ll_pos, long num_tok, int H, int K, int E,
                       int cap, int buf_stride, int pay_bytes, int sc_bytes, int sc_off,
                       uint8_t *__restrict__ recv, float *__restrict__ scales,
                       int32_t *status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint8_t *wbuf = smem + static_cast<size_t>(warp) * 2 * buf_stride;
  const int nvec = H >> 3;
  const int nblk = H >> 7;
  const bool bulk_scales = (sc_bytes & 15) == 0;
  int it = 0;
  for (long u = static_cast<long>(blockIdx.x) * kLLWarps + warp; u < num_tok;
       u += static_cast<long>(gridDim.x) * kLLWarps, ++it) {
    uint8_t *b = wbuf + (it & 1) * buf_stride;
    // the buffer was last used two tokens ago: its stores must have read it
    bulk_wait_read<1>();
    __syncwarp();

    // destination of slot `lane`: one row per distinct expert
    long dst = -1;
    {
      int e = -1, pos = -1;
      if (lane < K) {
        const int64_t ee = topk_idx[u * K + lane];
        if (ee >= 0 && ee < E) {
          e = static_cast<int>(ee);
          pos = ll_pos[u * K + lane];
        }
      }
      bool dup = false;
      for (int k2 = 0; k2 < K; ++k2) {
        const int e2 = __shfl_sync(0xffffffffu, e, k2);
        dup |= (k2 < lane && e2 == e);
      }
      if (e >= 0 && !dup) {
        if (pos >= 0 && pos < cap)
          dst = static_cast<long>(e) * cap + pos;
        else
          report(status, EP_STATUS_BAD_POSITION);
      }
    }

    const uint8_t *xr = x + u * static_cast<long>(H) * 2;
    for (int c0 = 0; c0 < nvec; c0 += 32) {
      const int c = c0 + lane;
      const bool act = c < nvec;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (act) v = __ldg(reinterpret_cast<const uint4 *>(xr) + c);
      if constexpr (kFP8) {
        float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                      bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
        // 16 lanes hold one 128-channel block (nvec is a multiple of 16)
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        amax = fmaxf(amax, 1e-4f);
        const float inv = __fdiv_rn(448.0f, amax);
        if (act) {
          uint2 q;
          q.x = cvt_e4m3x4(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv), __fmul_rn(f[2], inv),
                           __fmul_rn(f[3], inv));
          q.y = cvt_e4m3x4(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv), __fmul_rn(f[6], inv),
                           __fmul_rn(f[7], inv));
          *reinterpret_cast<uint2 *>(b + static_cast<size_t>(c) * 8) = q;
          if ((lane & 15) == 0)
            reinterpret_cast<float *>(b + sc_off)[c >> 4] = __fdiv_rn(amax, 448.0f);
        }
      } else {
        if (act) *reinterpret_cast<uint4 *>(b + static_cast<size_t>(c) * 16) = v;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (dst >= 0) {
      bulk_s2g(recv + dst * pay_bytes, b, static_cast<uint32_t>(pay_bytes));
      if constexpr (kFP8) {
        if (bulk_scales) {
          bulk_s2g(scales + dst * nblk, b + sc_off, static_cast<uint32_t>(sc_bytes));
        } else {
          const float *sb = reinterpret_cast<const float *>(b + sc_off);
          for (int j = 0; j < nblk; ++j) scales[dst * nblk + j] = sb[j];
        }
      }
    }
    bulk_commit();
  }
  bulk_wait_all<0>();
}

// ---------------------------------------------------------------------------

constexpr int kLLCombineWarps = 8;

__global__ void __launch_bounds__(kLLCombineWarps * 32)
    ll_combine_kernel(const uint8_t *__restrict__ y, const int64_t *__restrict__ topk_idx,
                      const float *__restrict__ topk_w, const int32_t *__restrict__ ll_pos,
                      long num_tok, int H, int K, int E, int cap, uint8_t *__restrict__ out,
                      int32_t *status) {
  __shared__ int64_t s_row[kLLCombineWarps][kMaxTopk];
  __shared__ float s_w[kLLCombineWarps][kMaxTopk];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint32_t lt = lanemask_lt();
  const int nvec = H >> 3;
  const long row_bytes = static_cast<long>(H) * 2;
  for (long u = static_cast<long>(blockIdx.x) * kLLCombineWarps + warp; u < num_tok;
       u += static_cast<long>(gridDim.x) * kLLCombineWarps) {
    bool take = false;
    long row = 0;
    float w = 0.f;
    if (lane < K) {
      const int64_t e = topk_idx[u * K + lane];
      if (e >= 0 && e < E) {
        const int pos = ll_pos[u * K + lane];
        if (pos >= 0 && pos < cap) {
          take = true;
          row = e * cap + pos;
          w = topk_w[u * K + lane];
        } else {
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
    for (int c = lane; c < nvec; c += 32) {
      float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < n; i += 8) {
        uint4 v[8];
#pragma unroll
        for (int b = 0; b < 8; ++b)
          if (i + b < n) v[b] = ld_stream_v4(y + s_row[warp][i + b] * row_bytes + c * 16L);
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
}

}  // namespace
}  // namespace ep

extern "C" EP_API size_t ep_ll_workspace_bytes(int num_ranks, int num_tokens, int num_experts) {
  using namespace ep;
  if (num_ranks < 1 || num_tokens < 0 || num_experts < 1) return 0;
  const long tiles = static_cast<long>(num_ranks) * ((num_tokens + kScanTile - 1) / kScanTile);
  return scan_workspace_bytes(tiles, num_experts, 0);
}

extern "C" EP_API int ep_ll_dispatch(const void *x, const int64_t *topk_idx, int num_ranks,
                                     int num_tokens, int hidden, int num_topk, int num_experts,
                                     int use_fp8, void *recv_x, float *recv_scales,
                                     int32_t *recv_count, int32_t *recv_src_info,
                                     int32_t *layout_range, int32_t *ll_pos, void *workspace,
                                     size_t workspace_bytes, int32_t *status,
                                     cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, K = num_topk, E = num_experts;
  if (R < 1 || R > kMaxRanks || T < 0 || K < 1 || K > kMaxTopk || E < 1 || E > kMaxExperts ||
      E % R != 0 || H < 8 || (use_fp8 ? (H % 128 != 0) : (H % 8 != 0)))
    return EP_ERR_INVALID_ARG;
  if (H > 65536) return EP_ERR_UNSUPPORTED;
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
  const size_t need = ep_ll_workspace_bytes(R, T, E);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return EP_ERR_INVALID_ARG;
  const long cap = static_cast<long>(R) * T;
  const int tiles_per_src = (T + kScanTile - 1) / kScanTile;
  const long num_tiles = static_cast<long>(R) * tiles_per_src;
  if (cap > 0x7fffffffL) return EP_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(workspace, 0, need, stream) != cudaSuccess) return EP_ERR_CUDA;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  LLScanParams p;
  p.topk_idx = topk_idx;
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
  p.status = status;
  const WaitConfig wc = wait_config();
  p.timeout_ns = wc.timeout_ns;
  p.flags = wc.flags;
  ll_scan_kernel<<<static_cast<unsigned>(num_tiles), kScanTile, 0, stream>>>(p);
  if (launch_status() != EP_OK) return EP_ERR_CUDA;

  const int pay = use_fp8 ? H : 2 * H;
  const int sc_bytes = use_fp8 ? (H / 128) * 4 : 0;
  const int sc_off = (pay + 127) & ~127;
  const int buf_stride = sc_off + ((sc_bytes + 127) & ~127);
  const size_t smem = static_cast<size_t>(kLLWarps) * 2 * buf_stride;
  const int threads = kLLWarps * 32;
  const long num_tok = static_cast<long>(R) * T;
  const void *fn = use_fp8 ? reinterpret_cast<const void *>(ll_dispatch_kernel<true>)
                           : reinterpret_cast<const void *>(ll_dispatch_kernel<false>);
  if (ensure_dynamic_smem(fn, smem) != EP_OK) return EP_ERR_CUDA;
  const long want = (num_tok + kLLWarps - 1) / kLLWarps;
  const long grid =
      std::min<long>(want, static_cast<long>(ctas_per_sm(fn, threads, smem)) * num_sms());
  if (use_fp8)
    ll_dispatch_kernel<true><<<static_cast<unsigned>(grid), threads, smem, stream>>>(
        static_cast<const uint8_t *>(x), topk_idx, ll_pos, num_tok, H, K, E,
        static_cast<int>(cap), buf_stride, pay, sc_bytes, sc_off,
        static_cast<uint8_t *>(recv_x), recv_scales, status);
  else
    ll_dispatch_kernel<false><<<static_cast<unsigned>(grid), threads, smem, stream>>>(
        static_cast<const uint8_t *>(x), topk_idx, ll_pos, num_tok, H, K, E,
        static_cast<int>(cap), buf_stride, pay, sc_bytes, sc_off,
        static_cast<uint8_t *>(recv_x), nullptr, status);
  return launch_status();
}

extern "C" EP_API int ep_ll_combine(const void *y, const int64_t *topk_idx,
                                    const float *topk_weights, const int32_t *ll_pos,
                                    int num_ranks, int num_tokens, int hidden, int num_topk,
                                    int num_experts, void *out, int32_t *status,
                                    cudaStream_t stream) {
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
  const long num_tok = static_cast<long>(R) * T;
  const int threads = kLLCombineWarps * 32;
  const void *fn = reinterpret_cast<const void *>(ll_combine_kernel);
  const long want = (num_tok + kLLCombineWarps - 1) / kLLCombineWarps;
  const long grid = std::min<long>(want, static_cast<long>(ctas_per_sm(fn, threads, 0)) * num_sms());
  ll_combine_kernel<<<static_cast<unsigned>(grid), threads, 0, stream>>>(
      static_cast<const uint8_t *>(y), topk_idx, topk_weights, ll_pos, num_tok, H, K, E,
      static_cast<int>(cap), static_cast<uint8_t *>(out), status);
  return launch_status();
}
