// ep_combine.cu -- A4: combine (gather-reduce of the dispatched copies).
//
// Semantics (DeepEP legacy-test analysis page, combine call and its check
// (combined_x - bias_0 - bias_1) / is_token_in_rank.sum(1) == x): every
// source token gets back the sum of the rows its destinations return, summed
// in fp32 in ascending destination rank, plus bias_0 then bias_1 if given,
// then rounded once to bf16 (nearest even).
//
// One warp per source token.  The warp reads send_pos[s][t][0..R), compacts
// the valid (d, row) pairs in ascending d into shared memory with a ballot,
// then each lane owns 16-byte chunks (8 channels) of the hidden row: it issues
// the loads of two chunks from up to 8 rows at once (16 loads in flight per
// lane), accumulates in fp32 in list order and writes 16 bytes back.
// HBM-bound: N*H*2 bytes read, R*T*H*2 bytes written.  With the phase timers
// on (ep_set_phase_timers) the single-GPU form runs its timed instance.
#include <algorithm>

#include "ep_common.cuh"

namespace ep {
namespace {

constexpr int kCombineWarps = 8;

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 &v) {
  acc[0] += bf16lo(v.x);
  acc[1] += bf16hi(v.x);
  acc[2] += bf16lo(v.y);
  acc[3] += bf16hi(v.y);
  acc[4] += bf16lo(v.z);
  acc[5] += bf16hi(v.z);
  acc[6] += bf16lo(v.w);
  acc[7] += bf16hi(v.w);
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&a)[8]) {
  uint4 r;
  r.x = pack_bf16x2(a[0], a[1]);
  r.y = pack_bf16x2(a[2], a[3]);
  r.z = pack_bf16x2(a[4], a[5]);
  r.w = pack_bf16x2(a[6], a[7]);
  return r;
}

// kTab: the destinations' buffers are given by tables of R pointers (one
// rank of a sharded job: peers' memory, read with plain loads); else they
// are slices d * cap of y and recv_w.  kBatch: rows whose chunks are loaded
// at once; kMinCtas: CTAs per SM the registers are sized for.  Two shapes:
// 8 rows at 2 CTAs per SM, and -- when no token can have more than 6
// copies -- 6 rows at 3 CTAs per SM, where the extra warps put more loads in
// flight than the rows of one token can.  kTimed: the kernel is the combine
// phase of the phase timers (tm); the untimed form never reads tm.
template <bool kTab, int kBatch, int kMinCtas, bool kTimed>
__global__ void __launch_bounds__(kCombineWarps * 32, kMinCtas)
    combine_kernel(const uint8_t *__restrict__ y, const float *__restrict__ recv_w,
                   const uint8_t *const *y_tab, const float *const *w_tab,
                   const int32_t *__restrict__ send_pos, const uint8_t *__restrict__ bias0,
                   const uint8_t *__restrict__ bias1, int R, long num_tok, int H, int K,
                   int cap, bool want_w, uint8_t *__restrict__ out, float *__restrict__ out_w,
                   int32_t *status, PhaseTimer *tm) {
  pdl_wait();
  unsigned long long begun = 0ull;
  if constexpr (kTimed) begun = timer_begin(tm);
  // per warp: [R] row pointers of y, then [R] row pointers of recv_w
  extern __shared__ __align__(16) const uint8_t *s_ptr[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint8_t **rows = s_ptr + static_cast<size_t>(warp) * 2 * R;
  const float **wrows = reinterpret_cast<const float **>(rows + R);
  const uint32_t lt = lanemask_lt();
  const int nvec = H >> 3;
  const long row_bytes = static_cast<long>(H) * 2;

  for (long u = static_cast<long>(blockIdx.x) * kCombineWarps + warp; u < num_tok;
       u += static_cast<long>(gridDim.x) * kCombineWarps) {
    int n = 0;
    bool bad = false;
    for (int d0 = 0; d0 < R; d0 += 32) {
      const int d = d0 + lane;
      int pos = -1;
      if (d < R) pos = __ldg(send_pos + u * R + d);
      bad |= (pos < -1 || pos >= cap);
      const bool take = pos >= 0 && pos < cap;
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      if (take) {
        const int i = n + __popc(bal & lt);
        if (kTab) {
          rows[i] = y_tab[d] + static_cast<long>(pos) * row_bytes;
          if (want_w) wrows[i] = w_tab[d] + static_cast<long>(pos) * K;
        } else {
          const long row = static_cast<long>(d) * cap + pos;
          rows[i] = y + row * row_bytes;
          if (want_w) wrows[i] = recv_w + row * K;
        }
      }
      n += __popc(bal);
    }
    if (bad) report(status, EP_STATUS_BAD_POSITION);
    __syncwarp();

    uint8_t *orow = out + u * row_bytes;
    for (int c = lane; c < nvec; c += 64) {
      const bool two = c + 32 < nvec;
      float a0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float a1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < n; i += kBatch) {
        uint4 v0[kBatch], v1[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          if (i + b < n) {
            const uint8_t *r = rows[i + b];
            v0[b] = ld_stream_v4(r + static_cast<long>(c) * 16);
            if (two) v1[b] = ld_stream_v4(r + static_cast<long>(c + 32) * 16);
          }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          if (i + b < n) {
            add_bf16x8(a0, v0[b]);
            if (two) add_bf16x8(a1, v1[b]);
          }
        }
      }
      // bias terms come after the sum of the copies: first bias_0, then bias_1
      if (bias0 != nullptr) {
        add_bf16x8(a0, ld_stream_v4(bias0 + u * row_bytes + static_cast<long>(c) * 16));
        if (two) add_bf16x8(a1, ld_stream_v4(bias0 + u * row_bytes + static_cast<long>(c + 32) * 16));
      }
      if (bias1 != nullptr) {
        add_bf16x8(a0, ld_stream_v4(bias1 + u * row_bytes + static_cast<long>(c) * 16));
        if (two) add_bf16x8(a1, ld_stream_v4(bias1 + u * row_bytes + static_cast<long>(c + 32) * 16));
      }
      st_stream_v4(orow + static_cast<long>(c) * 16, pack_bf16x8(a0));
      if (two) st_stream_v4(orow + static_cast<long>(c + 32) * 16, pack_bf16x8(a1));
    }
    if (want_w && lane < K) {
      float a = 0.f;
      for (int i = 0; i < n; ++i) a += __ldg(wrows[i] + lane);
      out_w[u * K + lane] = a;
    }
    __syncwarp();
  }
  if constexpr (kTimed) timer_end(tm, begun);
}

// Launch of one instantiation (arguments already checked).
template <bool kTab, int kBatch, int kMinCtas>
int combine_launch_as(const void *y, const float *recv_w, const uint8_t *const *y_tab,
                      const float *const *w_tab, const int32_t *send_pos, const void *bias_0,
                      const void *bias_1, int R, long num_tok, int H, int K, int cap,
                      void *combined_x, float *combined_w, int32_t *status,
                      cudaStream_t stream) {
  const int threads = kCombineWarps * 32;
  const size_t smem = static_cast<size_t>(kCombineWarps) * 2 * R * sizeof(void *);
  PhaseTimer *const tm = kTab ? nullptr : phase_timer(kPhaseCombine);
  auto *kernel = tm != nullptr ? combine_kernel<kTab, kBatch, kMinCtas, !kTab>
                               : combine_kernel<kTab, kBatch, kMinCtas, false>;
  const void *fn = reinterpret_cast<const void *>(kernel);
  if (ensure_dynamic_smem(fn, smem) != EP_OK) return EP_ERR_CUDA;
  const long want = (num_tok + kCombineWarps - 1) / kCombineWarps;
  const long grid =
      std::min<long>(want, static_cast<long>(ctas_per_sm(fn, threads, smem)) * num_sms());
  const cudaError_t launched = launch_pdl(
      kernel, dim3(static_cast<unsigned>(grid)), dim3(threads), smem, stream,
      static_cast<const uint8_t *>(y), recv_w, y_tab, w_tab, send_pos,
      static_cast<const uint8_t *>(bias_0), static_cast<const uint8_t *>(bias_1), R, num_tok, H,
      K, cap, combined_w != nullptr, static_cast<uint8_t *>(combined_x), combined_w, status, tm);
  return launch_status(launched);
}

// Launch of either form.  A token has at most min(K, R) copies (one per
// destination rank of its experts); when that is at most 6, the 6-row,
// 3-CTA shape reads every token's copies in one batch.  (K only bounds the
// copies when it is the routing's top-k; any K gives the same results.)
int combine_launch(const void *y, const float *recv_w, const uint8_t *const *y_tab,
                   const float *const *w_tab, const int32_t *send_pos, const void *bias_0,
                   const void *bias_1, int R, long num_tok, int H, int K, int cap,
                   void *combined_x, float *combined_w, int32_t *status, cudaStream_t stream) {
  const bool narrow = R <= 6 || (K >= 1 && K <= 6);
  if (y_tab != nullptr)
    return narrow ? combine_launch_as<true, 6, 3>(y, recv_w, y_tab, w_tab, send_pos, bias_0,
                                                  bias_1, R, num_tok, H, K, cap, combined_x,
                                                  combined_w, status, stream)
                  : combine_launch_as<true, 8, 2>(y, recv_w, y_tab, w_tab, send_pos, bias_0,
                                                  bias_1, R, num_tok, H, K, cap, combined_x,
                                                  combined_w, status, stream);
  return narrow ? combine_launch_as<false, 6, 3>(y, recv_w, y_tab, w_tab, send_pos, bias_0, bias_1,
                                                 R, num_tok, H, K, cap, combined_x, combined_w,
                                                 status, stream)
                : combine_launch_as<false, 8, 2>(y, recv_w, y_tab, w_tab, send_pos, bias_0, bias_1,
                                                 R, num_tok, H, K, cap, combined_x, combined_w,
                                                 status, stream);
}

}  // namespace
}  // namespace ep

extern "C" EP_API int ep_combine(const void *y, const float *recv_topk_weights,
                                 const int32_t *send_pos, const void *bias_0, const void *bias_1,
                                 int num_ranks, int num_tokens, int hidden, int num_topk,
                                 int capacity, void *combined_x, float *combined_topk_weights,
                                 int32_t *status, cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, K = num_topk, cap = capacity;
  if (R < 1 || R > kMaxRanks || T < 0 || H < 8 || H % 8 != 0 || cap < 0) return EP_ERR_INVALID_ARG;
  if (combined_topk_weights != nullptr &&
      (recv_topk_weights == nullptr || K < 1 || K > kMaxTopk))
    return EP_ERR_INVALID_ARG;
  if (T == 0) return EP_OK;
  if (y == nullptr || send_pos == nullptr || combined_x == nullptr) return EP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(y) & 15u) || (reinterpret_cast<uintptr_t>(combined_x) & 15u) ||
      (reinterpret_cast<uintptr_t>(bias_0) & 15u) || (reinterpret_cast<uintptr_t>(bias_1) & 15u))
    return EP_ERR_INVALID_ARG;
  const long num_tok = static_cast<long>(R) * T;
  return combine_launch(y, combined_topk_weights != nullptr ? recv_topk_weights : nullptr, nullptr,
                        nullptr, send_pos, bias_0, bias_1, R, num_tok, H, K, cap, combined_x,
                        combined_topk_weights, status, stream);
}

extern "C" EP_API int ep_shard_combine(const void *const *y_peers,
                                       const float *const *recv_topk_weights_peers,
                                       const int32_t *send_pos, const void *bias_0,
                                       const void *bias_1, int num_ranks, int num_tokens,
                                       int hidden, int num_topk, int capacity, void *combined_x,
                                       float *combined_topk_weights, int32_t *status,
                                       cudaStream_t stream) {
  using namespace ep;
  const int R = num_ranks, T = num_tokens, H = hidden, K = num_topk, cap = capacity;
  if (R < 1 || R > kMaxRanks || T < 0 || H < 8 || H % 8 != 0 || cap < 0) return EP_ERR_INVALID_ARG;
  if (combined_topk_weights != nullptr &&
      (recv_topk_weights_peers == nullptr || K < 1 || K > kMaxTopk))
    return EP_ERR_INVALID_ARG;
  if (T == 0) return EP_OK;
  if (y_peers == nullptr || send_pos == nullptr || combined_x == nullptr) return EP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(combined_x) & 15u) ||
      (reinterpret_cast<uintptr_t>(bias_0) & 15u) || (reinterpret_cast<uintptr_t>(bias_1) & 15u))
    return EP_ERR_INVALID_ARG;
  return combine_launch(nullptr, nullptr, reinterpret_cast<const uint8_t *const *>(y_peers),
                        recv_topk_weights_peers, send_pos, bias_0, bias_1, R, T, H, K, cap,
                        combined_x, combined_topk_weights, status, stream);
}
