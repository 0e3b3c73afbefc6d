// ep_layout.cu -- A1: get_dispatch_layout.
//
// From topk_idx [S, T, K] compute num_tokens_per_rank [S, R],
// num_tokens_per_expert [S, E] and is_token_in_rank [S, T, R]
// (GET_DISPATCH_LAYOUT_API page, "Parameters" / "Return Values"; the Ascend
// port there splits tokens evenly over cores, which is the data-parallel
// split used here: one CTA per tile of 128 tokens of one source rank).
//
// Per tile: each thread owns a token and marks its ranks in a shared-memory
// [tile, R] byte matrix and its experts in a shared histogram; the tile's
// counts are then added to the outputs with one global atomic per non-zero
// bin, and the byte matrix is written out with 16-byte stores.  Integer
// atomics make the result independent of the order in which tiles finish.
// Bound: latency (the whole input of the 4096 x 8 case is 256 KiB).
#include "ep_common.cuh"

namespace ep {
namespace {

constexpr int kLayoutTile = 128;

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kLayoutTile)
    layout_kernel(const int64_t *__restrict__ topk_idx, int T, int K, int E, int R, FastDiv El,
                  int tiles_per_src, int32_t *__restrict__ ntpr, int32_t *__restrict__ ntpe,
                  uint8_t *__restrict__ in_rank, int32_t *status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem[];
  int32_t *s_exp = reinterpret_cast<int32_t *>(smem);  // [E]
  uint8_t *s_row = smem + ((E * 4 + 15) & ~15);         // [tile, R]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int s = blockIdx.x / tiles_per_src;
  const int t0 = (blockIdx.x % tiles_per_src) * kLayoutTile;
  const int ntok = min(kLayoutTile, T - t0);

  for (int i = tid; i < E; i += kLayoutTile) s_exp[i] = 0;
  uint32_t *row32 = reinterpret_cast<uint32_t *>(s_row);
  for (int i = tid; i < (ntok * R + 3) / 4; i += kLayoutTile) row32[i] = 0u;
  __syncthreads();

  if (tid < ntok) {
    const int64_t *idx = topk_idx + (static_cast<size_t>(s) * T + t0 + tid) * K;
    bool bad = false;
    for (int k = 0; k < K; ++k) {
      const int64_t e = idx[k];
      if (e == -1) continue;
      if (e < -1 || e >= E) {
        bad = true;
        continue;
      }
      s_row[tid * R + fastdiv(static_cast<int>(e), El)] = 1;
      atomicAdd(&s_exp[static_cast<int>(e)], 1);
    }
    if (bad) report(status, EP_STATUS_BAD_EXPERT);
  }
  __syncthreads();

  // tokens per rank: one warp per rank column
  for (int d = warp; d < R; d += kLayoutTile / 32) {
    int c = 0;
    for (int i = lane; i < ntok; i += 32) c += s_row[i * R + d];
    c = warp_sum(c);
    if (lane == 0 && c != 0) atomicAdd(&ntpr[static_cast<size_t>(s) * R + d], c);
  }
  for (int e = tid; e < E; e += kLayoutTile) {
    const int c = s_exp[e];
    if (c != 0) atomicAdd(&ntpe[static_cast<size_t>(s) * E + e], c);
  }

  // is_token_in_rank rows of this tile are contiguous in global memory
  uint8_t *dst = in_rank + (static_cast<size_t>(s) * T + t0) * R;
  const int nbytes = ntok * R;
  if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
    const int n16 = nbytes >> 4;
    for (int i = tid; i < n16; i += kLayoutTile)
      reinterpret_cast<uint4 *>(dst)[i] = reinterpret_cast<const uint4 *>(s_row)[i];
    for (int i = (n16 << 4) + tid; i < nbytes; i += kLayoutTile) dst[i] = s_row[i];
  } else {
    for (int i = tid; i < nbytes; i += kLayoutTile) dst[i] = s_row[i];
  }
}

}  // namespace
}  // namespace ep

extern "C" EP_API int ep_get_dispatch_layout(const int64_t *topk_idx, int num_src_ranks,
                                             int num_tokens, int num_topk, int num_experts,
                                             int num_ranks, int32_t *num_tokens_per_rank,
                                             int32_t *num_tokens_per_expert,
                                             uint8_t *is_token_in_rank, int32_t *status,
                                             cudaStream_t stream) {
  using namespace ep;
  const int S = num_src_ranks, T = num_tokens, K = num_topk, E = num_experts, R = num_ranks;
  if (S < 1 || T < 0 || K < 1 || K > kMaxTopk || R < 1 || R > kMaxRanks || E < 1 ||
      E > kMaxExperts || E % R != 0)
    return EP_ERR_INVALID_ARG;
  if (num_tokens_per_rank == nullptr || num_tokens_per_expert == nullptr)
    return EP_ERR_INVALID_ARG;
  if (T > 0 && (topk_idx == nullptr || is_token_in_rank == nullptr)) return EP_ERR_INVALID_ARG;
  if (cudaMemsetAsync(num_tokens_per_rank, 0, sizeof(int32_t) * S * R, stream) != cudaSuccess ||
      cudaMemsetAsync(num_tokens_per_expert, 0, sizeof(int32_t) * static_cast<size_t>(S) * E,
                      stream) != cudaSuccess)
    return EP_ERR_CUDA;
  if (T == 0) return EP_OK;
  const int tiles_per_src = (T + kLayoutTile - 1) / kLayoutTile;
  const size_t smem = static_cast<size_t>((E * 4 + 15) & ~15) + kLayoutTile * R;
  if (ensure_dynamic_smem(reinterpret_cast<const void *>(layout_kernel), smem) != EP_OK)
    return EP_ERR_CUDA;
  const long grid = static_cast<long>(S) * tiles_per_src;
  if (grid > 0x7fffffffL) return EP_ERR_UNSUPPORTED;
  const cudaError_t launched = launch_pdl(layout_kernel,
      dim3(static_cast<unsigned>(grid)), dim3(kLayoutTile), smem, stream,
      topk_idx, T, K, E, R, make_fastdiv(E / R), tiles_per_src, num_tokens_per_rank,
      num_tokens_per_expert,
      is_token_in_rank, status);
  return launch_status(launched);
}
