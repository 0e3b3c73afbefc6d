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
//
// Up to 4096 tokens per source rank and 32 ranks, one thread-block cluster of
// 8 CTAs (512 tokens each) takes a whole source rank instead: each CTA counts
// its tokens in shared memory, adds the counts into CTA 0's shared memory
// through the cluster's distributed shared memory, and CTA 0 stores every
// count of the source rank -- no global atomics and no zeroing of the outputs
// beforehand.
#include <cooperative_groups.h>

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

constexpr int kClusterCtas = 8;
constexpr int kClusterThreads = 512;                            // one token per thread
constexpr int kClusterTokens = kClusterCtas * kClusterThreads;  // per source rank
constexpr int kClusterMaxRanks = 32;                            // rank set in one word

__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kClusterThreads)
    layout_cluster_kernel(const int64_t *__restrict__ topk_idx, int T, int K, int E, int R,
                          FastDiv El, int32_t *__restrict__ ntpr, int32_t *__restrict__ ntpe,
                          uint8_t *__restrict__ in_rank, int32_t *status) {
  namespace cg = cooperative_groups;
  pdl_wait();
  pdl_trigger();
  __shared__ int s_exp[kMaxExperts];         // this CTA's counts; CTA 0: the source's
  __shared__ int s_rank[kClusterMaxRanks];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int s = blockIdx.x / kClusterCtas;
  const int t = crank * kClusterThreads + tid;

  for (int i = tid; i < E; i += kClusterThreads) s_exp[i] = 0;
  if (tid < R) s_rank[tid] = 0;
  cluster.sync();  // CTA 0's counters are zero before any CTA adds to them

  uint32_t ranks = 0;  // bit d: the token goes to rank d
  if (t < T) {
    const int64_t *idx = topk_idx + (static_cast<size_t>(s) * T + t) * K;
    int64_t ek[kMaxTopk];
#pragma unroll
    for (int k = 0; k < kMaxTopk; ++k) ek[k] = k < K ? __ldg(idx + k) : -1;
    bool bad = false;
#pragma unroll
    for (int k = 0; k < kMaxTopk; ++k) {
      const int64_t e = ek[k];
      if (k >= K || e == -1) continue;
      if (e < -1 || e >= E) {
        bad = true;
        continue;
      }
      ranks |= 1u << fastdiv(static_cast<int>(e), El);
      atomicAdd(&s_exp[static_cast<int>(e)], 1);
    }
    if (bad) report(status, EP_STATUS_BAD_EXPERT);
    uint8_t *row = in_rank + (static_cast<size_t>(s) * T + t) * R;
    if ((R & 3) == 0 && (reinterpret_cast<uintptr_t>(in_rank) & 3u) == 0) {
      for (int d = 0; d < R; d += 4) {  // four 0/1 bytes per 32-bit store
        const uint32_t b = ranks >> d;
        reinterpret_cast<uint32_t *>(row)[d >> 2] =
            (b & 1u) | ((b >> 1) & 1u) << 8 | ((b >> 2) & 1u) << 16 | ((b >> 3) & 1u) << 24;
      }
    } else {
      for (int d = 0; d < R; ++d) row[d] = (ranks >> d) & 1u;
    }
  }
  for (int d = 0; d < R; ++d) {  // tokens per rank, a warp at a time
    const int c = __popc(__ballot_sync(0xffffffffu, (ranks >> d) & 1u));
    if (lane == 0 && c != 0) atomicAdd(&s_rank[d], c);
  }
  __syncthreads();
  if (crank != 0) {  // into CTA 0's shared memory
    int *r_exp = cluster.map_shared_rank(s_exp, 0);
    int *r_rank = cluster.map_shared_rank(s_rank, 0);
    for (int e = tid; e < E; e += kClusterThreads)
      if (s_exp[e] != 0) atomicAdd(&r_exp[e], s_exp[e]);
    if (tid < R && s_rank[tid] != 0) atomicAdd(&r_rank[tid], s_rank[tid]);
  }
  cluster.sync();  // every CTA's counts are in CTA 0
  if (crank == 0) {
    for (int e = tid; e < E; e += kClusterThreads) ntpe[static_cast<size_t>(s) * E + e] = s_exp[e];
    if (tid < R) ntpr[static_cast<size_t>(s) * R + tid] = s_rank[tid];
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
  if (T > 0 && T <= kClusterTokens && R <= kClusterMaxRanks) {
    // one cluster per source rank; it stores every count, nothing to zero
    if (static_cast<long>(S) * kClusterCtas > 0x7fffffffL) return EP_ERR_UNSUPPORTED;
    const cudaError_t launched = launch_pdl(layout_cluster_kernel,
        dim3(static_cast<unsigned>(S) * kClusterCtas), dim3(kClusterThreads), 0, stream,
        topk_idx, T, K, E, R, make_fastdiv(E / R), num_tokens_per_rank, num_tokens_per_expert,
        is_token_in_rank, status);
    return launch_status(launched);
  }
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
