// ep_common.cuh -- device helpers shared by the routing kernels (sm_100a).
//
// Thin wrappers over documented PTX: mbarrier, bulk (TMA) copies, relaxed
// device-scope loads/stores for the scan descriptors, %globaltimer for the
// bounded waits.  Nothing here is numerical.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ep.h"

namespace ep {

constexpr int kMaxTopk = 16;
constexpr int kMaxExperts = 512;
constexpr int kMaxRanks = 384;

// Launch-time settings of the bounded waits (set by ep_set_wait_timeout_ns /
// ep_set_debug_flags, read on the host when a kernel is launched).
struct WaitConfig {
  unsigned long long timeout_ns;
  unsigned flags;
};
WaitConfig wait_config();

// Number of SMs of the current device (cached per device).
int num_sms();

// Opt-in full-grid timers of the single-GPU entry points (the "Notify
// full-kernel duration" timer of the DeepEP PR #720 page, widened to a phase
// of one or more chained kernels): the earliest block start of the phase's
// first kernel, taken after its programmatic-dependency wait, to the last
// block end of its last kernel, both by %globaltimer.  Blocks publish their
// start as ~t with atomicMax (so the largest complement is the earliest
// start); the last block of the last kernel to finish adds the interval to
// the cumulative sum and clears the working slots for the next launch.
// Layout and use: ep_set_phase_timers in ep.h.
struct PhaseTimer {
  unsigned long long start_c;    // ~earliest block start of the launch in progress (0: none)
  unsigned long long done;       // blocks of the last kernel that have finished
  unsigned long long sum_ns;     // cumulative phase duration
  unsigned long long launches;   // phases timed
  unsigned long long last_start, last_end;
  unsigned long long reserved[2];
};
enum : int {
  kPhaseNotify = 0,
  kPhaseCopy = 1,
  kPhaseCombine = 2,
  kPhaseLLDispatch = 3,
  kPhaseLLCombine = 4,
  kNumPhases = 5
};

// Host: the timer of `phase` for kernels launched now, or nullptr while the
// timers are off or the caller's array has no room for that phase.
PhaseTimer *phase_timer(int phase);

// EP_OK for a launch that returned cudaSuccess, else EP_ERR_CUDA.  The
// launch's own return value is used, not cudaGetLastError(), which would
// also report (and clear) an error some other code left behind.
inline int launch_status(cudaError_t launched) {
  return launched == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

// Raise the dynamic shared-memory limit of `func` on the current device to at
// least `bytes` (needed above 48 KiB).  Cached per (function, device).
int ensure_dynamic_smem(const void *func, size_t bytes);

// Resident CTAs per SM of `func` for `threads` threads and `smem` bytes of
// dynamic shared memory (at least 1).  Cached per (function, device, smem).
int ctas_per_sm(const void *func, int threads, size_t smem);

// Dynamic shared memory to request so that at most `n` CTAs of a kernel fit
// on one SM: max(smem, the smallest size of which n + 1 CTAs overflow the
// SM).  A grid of n CTAs per SM then lands evenly on the SMs even when it is
// scheduled while another kernel still holds part of them.
size_t spread_smem(size_t smem, int n);

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialization.  It calls pdl_wait() before it reads
// or writes any global memory: that waits until the previous grid in the
// stream has completed and its writes are visible, so results keep stream
// order.  (One exception, argued where it is made: the LL dispatch kernel runs
// alongside the LL scan and waits for it only before it exits.)  It calls
// pdl_trigger() once its main work is issued: the next kernel may then be
// scheduled (its CTAs start and block in their own pdl_wait()), which hides
// its launch latency behind this kernel's tail.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// Zeroes a[0, a_bytes) and b[0, b_words) on `stream` with a kernel chained
// to its neighbours by programmatic launch (a memset node would break that
// chain): it waits for the previous kernel in the stream before it stores,
// and lets the next one start.  Before that wait it asks L2 for
// pf[0, pf_bytes) (a hint only; pf may be nullptr).  Falls back to memsets
// where `a` is not 16-byte aligned or a_bytes not a multiple of 16.
// `begin`: a phase timer this kernel starts (nullptr: none).
int zero_prefetch(void *a, size_t a_bytes, int32_t *b, long b_words, const void *pf,
                  long pf_bytes, cudaStream_t stream, PhaseTimer *begin = nullptr);

__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// n / d by one multiply-high, for 0 <= n and n * d < 2^32 (expert ids and
// experts per rank are at most 512).  m = ceil(2^32 / d) exceeds 2^32 / d by
// less than 1, so n * m / 2^32 = n / d + err with 0 <= err < n / 2^32 < 1 / d:
// never enough to reach the next integer.  d == 1 has no 32-bit m.
struct FastDiv {
  uint32_t m;
  int d;
};

inline FastDiv make_fastdiv(int d) {
  FastDiv f;
  f.d = d;
  f.m = d > 1 ? static_cast<uint32_t>((0x100000000ull + static_cast<uint64_t>(d) - 1) / d) : 0u;
  return f;
}

__device__ __forceinline__ int fastdiv(int n, FastDiv f) {
  return f.d == 1 ? n : static_cast<int>(__umulhi(static_cast<uint32_t>(n), f.m));
}

__device__ __forceinline__ void report(int32_t *status, int bits) {
  if (status != nullptr) atomicOr(status, bits);
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Phase timers (see PhaseTimer).  timer_begin: thread 0 of each block of the
// phase's first kernel, after pdl_wait(); it returns the stamp's old value.
// timer_end: every thread of each block of the phase's last kernel, at its
// end (t is uniform); one atomic per block counts the blocks done.  When the
// stamp was taken in the same kernel, thread 0 passes the value timer_begin
// returned: it stores that value before it counts the block, so the stamp
// (whose result it is) has been performed before the count is issued -- no
// fence, which delayed every block's exit.  A stamp taken in an earlier
// kernel of the stream is complete when this kernel passes pdl_wait (pass
// 0).  The last block reads only the timer's own words, through atomics.
__device__ __forceinline__ unsigned long long timer_begin(PhaseTimer *t) {
  if (t == nullptr || threadIdx.x != 0) return 0ull;
  return atomicMax(&t->start_c, ~globaltimer());
}

__device__ __forceinline__ void timer_end(PhaseTimer *t, unsigned long long begun) {
  __shared__ unsigned long long s_begun;
  if (t == nullptr) return;
  __syncthreads();
  if (threadIdx.x != 0) return;
  asm volatile("st.volatile.shared.u64 [%0], %1;" ::"r"(static_cast<uint32_t>(
                   __cvta_generic_to_shared(&s_begun))), "l"(begun)
               : "memory");
  const unsigned long long blocks =
      static_cast<unsigned long long>(gridDim.x) * gridDim.y * gridDim.z;
  if (atomicAdd(&t->done, 1ull) + 1ull != blocks) return;
  const unsigned long long end = globaltimer();
  const unsigned long long start = ~atomicExch(&t->start_c, 0ull);
  t->sum_ns += end - start;
  t->launches += 1ull;
  t->last_start = start;
  t->last_end = end;
  atomicExch(&t->done, 0ull);
}

__device__ __forceinline__ uint64_t ld_relaxed_gpu(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_gpu(uint64_t *p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed_gpu(int32_t *p, int32_t v) {
  asm volatile("st.relaxed.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int32_t ld_relaxed_gpu(const int32_t *p) {
  int32_t v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// four consecutive 32-bit words (16-byte aligned) with one relaxed store
__device__ __forceinline__ void st_relaxed_gpu_v4(int32_t *p, int a, int b, int c, int d) {
  asm volatile("st.relaxed.gpu.global.v4.s32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}

// four consecutive 32-bit words (16-byte aligned) with one relaxed load
__device__ __forceinline__ uint4 ld_relaxed_gpu_v4(const uint32_t *p) {
  uint4 v;
  asm volatile("ld.relaxed.gpu.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Plain arrival (no transaction bytes): completes a phase that expects one.
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, at most `timeout_ns`.
// Returns false if the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > timeout_ns) return false;
  }
}

// ---- bulk (TMA, non-tensor) copies -----------------------------------------

// global -> shared, completion counted on `bar` (bytes % 16 == 0, both ends
// 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gsrc, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// L2 policy for data read once: evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// global -> shared bulk copy with an L2 cache policy (see bulk_g2s).
__device__ __forceinline__ void bulk_g2s_hint(void *smem_dst, const void *gsrc, uint32_t bytes,
                                              uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// shared -> global, tracked by this thread's bulk groups.
__device__ __forceinline__ void bulk_s2g(void *gdst, const void *smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_addr(smem_src)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until at most N of this thread's bulk groups are still in flight.
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Make generic-proxy writes to shared memory visible to the bulk-copy engine.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- vector memory access ------------------------------------------------

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream_v4(void *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// 32-byte stores (one whole L2 sector per thread; address 32-byte aligned).
__device__ __forceinline__ void st_v4_b64(void *p, int64_t a, int64_t b, int64_t c, int64_t d) {
  asm volatile("st.global.v4.b64 [%0], {%1, %2, %3, %4};" ::"l"(p), "l"(a), "l"(b), "l"(c),
               "l"(d)
               : "memory");
}

template <typename T>
__device__ __forceinline__ void st_v8_b32(void *p, const T (&v)[8]) {
  static_assert(sizeof(T) == 4, "32-bit elements");
  uint32_t u[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) u[j] = __builtin_bit_cast(uint32_t, v[j]);
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(u[0]),
               "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
               : "memory");
}

// bf16 pair (packed in a u32, element 0 in the low half) -> two floats.
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Two floats -> packed bf16 pair, round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

}  // namespace ep
