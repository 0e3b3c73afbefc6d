// ep_api.cu -- host-side helpers of the C ABI: status text, version, the
// process-wide limits of the bounded device waits and the phase-timer switch,
// device properties, and the zeroing kernel chained ahead of a notify or an
// LL dispatch.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "ep_common.cuh"

namespace ep {

namespace {
std::atomic<unsigned long long> g_timeout_ns{1000000000ull};
std::atomic<unsigned> g_flags{0u};
constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {0};
std::mutex g_sms_mu;
}  // namespace

WaitConfig wait_config() {
  WaitConfig c;
  c.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  c.flags = g_flags.load(std::memory_order_relaxed);
  return c;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_sms_mu);
  if (g_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

namespace {
std::mutex g_attr_mu;
std::map<std::pair<const void *, int>, size_t> g_smem_set;
std::map<std::tuple<const void *, int, int, size_t>, int> g_occ;
}  // namespace

int ensure_dynamic_smem(const void *func, size_t bytes) {
  if (bytes <= 48 * 1024) return EP_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EP_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  size_t &cur = g_smem_set[{func, dev}];
  if (cur >= bytes) return EP_OK;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess)
    return EP_ERR_CUDA;
  cur = bytes;
  return EP_OK;
}

namespace {
std::mutex g_smem_attr_mu;
int g_smem_per_sm[kMaxDevices] = {0};
int g_smem_reserved[kMaxDevices] = {0};
}  // namespace

size_t spread_smem(size_t smem, int n) {
  int dev = 0;
  if (n < 1 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return smem;
  int per_sm, reserved;
  {
    std::lock_guard<std::mutex> lk(g_smem_attr_mu);
    if (g_smem_per_sm[dev] == 0) {
      int a = 0, b = 0;
      if (cudaDeviceGetAttribute(&a, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
              cudaSuccess ||
          cudaDeviceGetAttribute(&b, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
              cudaSuccess ||
          a <= 0)
        return smem;
      g_smem_per_sm[dev] = a;
      g_smem_reserved[dev] = b;
    }
    per_sm = g_smem_per_sm[dev];
    reserved = g_smem_reserved[dev];
  }
  // n + 1 CTAs of (s + reserved) bytes overflow per_sm once s exceeds this
  const long lo = static_cast<long>(per_sm) / (n + 1) - reserved + 16;
  const size_t want = static_cast<size_t>((std::max<long>(lo, 0) + 15) & ~15L);
  // only if n CTAs of that size still fit
  if (static_cast<long>(n) * (static_cast<long>(want) + reserved) > per_sm) return smem;
  return std::max(smem, want);
}

int ctas_per_sm(const void *func, int threads, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  auto key = std::make_tuple(func, dev, threads, smem);
  auto it = g_occ.find(key);
  if (it != g_occ.end()) return it->second;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem) != cudaSuccess ||
      n < 1)
    n = 1;
  g_occ[key] = n;
  return n;
}

namespace {

template <bool kTimed>
__global__ void __launch_bounds__(256) zero_prefetch_kernel(uint4 *a, long a16, int32_t *b,
                                                            long b_words, const char *pf,
                                                            long pf_bytes, PhaseTimer *begin) {
  const long nthr = static_cast<long>(gridDim.x) * blockDim.x;
  const long me = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (long off = me * 128; off < pf_bytes; off += nthr * 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(pf + off));
  pdl_wait();
  if constexpr (kTimed) timer_begin(begin);
  pdl_trigger();  // the next kernel's CTAs may start; they wait for this grid to complete
  for (long i = me; i < a16; i += nthr) a[i] = make_uint4(0u, 0u, 0u, 0u);
  for (long i = me; i < b_words; i += nthr) b[i] = 0;
}

}  // namespace

int zero_prefetch(void *a, size_t a_bytes, int32_t *b, long b_words, const void *pf,
                  long pf_bytes, cudaStream_t stream, PhaseTimer *begin) {
  if ((reinterpret_cast<uintptr_t>(a) & 15u) != 0 || (a_bytes & 15u) != 0) {
    if (a_bytes > 0 && cudaMemsetAsync(a, 0, a_bytes, stream) != cudaSuccess) return EP_ERR_CUDA;
    if (b_words > 0 &&
        cudaMemsetAsync(b, 0, sizeof(int32_t) * static_cast<size_t>(b_words), stream) !=
            cudaSuccess)
      return EP_ERR_CUDA;
    if (begin == nullptr) return EP_OK;
    a_bytes = 0;  // the kernel only starts the timer
    b_words = 0;
  }
  const long a16 = static_cast<long>(a_bytes / 16);
  if (pf == nullptr) pf_bytes = 0;
  const long want = (std::max({a16, b_words, (pf_bytes + 127) / 128}) + 255) / 256;
  const long grid = std::max(1L, std::min<long>(want, num_sms()));
  auto *kernel = begin != nullptr ? zero_prefetch_kernel<true> : zero_prefetch_kernel<false>;
  return launch_status(launch_pdl(kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, stream,
                                  static_cast<uint4 *>(a), a16, b, b_words,
                                  static_cast<const char *>(pf), pf_bytes, begin));
}

namespace {
std::atomic<PhaseTimer *> g_phase_timers{nullptr};
std::atomic<int> g_phase_count{0};
}  // namespace

PhaseTimer *phase_timer(int phase) {
  PhaseTimer *t = g_phase_timers.load(std::memory_order_relaxed);
  if (t == nullptr || phase < 0 || phase >= g_phase_count.load(std::memory_order_relaxed))
    return nullptr;
  return t + phase;
}

}  // namespace ep

extern "C" {

EP_API const char *ep_status_string(int code) {
  switch (code) {
    case EP_OK: return "ok";
    case EP_ERR_INVALID_ARG: return "invalid argument";
    case EP_ERR_CUDA: return "CUDA launch error";
    case EP_ERR_UNSUPPORTED: return "unsupported shape";
    default: return "unknown status";
  }
}

EP_API int ep_version(void) { return 100; }

EP_API int ep_set_phase_timers(unsigned long long *timers, int num_phases) {
  if (timers == nullptr) {
    ep::g_phase_timers.store(nullptr, std::memory_order_relaxed);
    ep::g_phase_count.store(0, std::memory_order_relaxed);
    return EP_OK;
  }
  if ((reinterpret_cast<uintptr_t>(timers) & 7u) != 0 || num_phases < 1 ||
      num_phases > ep::kNumPhases)
    return EP_ERR_INVALID_ARG;
  ep::g_phase_timers.store(nullptr, std::memory_order_relaxed);
  ep::g_phase_count.store(num_phases, std::memory_order_relaxed);
  ep::g_phase_timers.store(reinterpret_cast<ep::PhaseTimer *>(timers), std::memory_order_relaxed);
  return EP_OK;
}

EP_API int ep_set_wait_timeout_ns(long long ns) {
  if (ns < 0) return EP_ERR_INVALID_ARG;
  ep::g_timeout_ns.store(static_cast<unsigned long long>(ns), std::memory_order_relaxed);
  return EP_OK;
}

EP_API int ep_set_debug_flags(unsigned flags) {
  ep::g_flags.store(flags, std::memory_order_relaxed);
  return EP_OK;
}

// ---- memory shared between the ranks of a sharded job ----------------------

EP_API int ep_shard_alloc(size_t bytes, void **ptr) {
  if (ptr == nullptr || bytes == 0) return EP_ERR_INVALID_ARG;
  *ptr = nullptr;
  void *p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return EP_ERR_CUDA;
  if (cudaMemset(p, 0, bytes) != cudaSuccess) {
    cudaFree(p);
    return EP_ERR_CUDA;
  }
  *ptr = p;
  return EP_OK;
}

EP_API int ep_shard_free(void *ptr) {
  if (ptr == nullptr) return EP_OK;
  return cudaFree(ptr) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

EP_API int ep_ipc_handle(const void *ptr, void *handle) {
  static_assert(sizeof(cudaIpcMemHandle_t) == EP_IPC_HANDLE_BYTES, "IPC handle size");
  if (ptr == nullptr || handle == nullptr) return EP_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, const_cast<void *>(ptr)) != cudaSuccess) return EP_ERR_CUDA;
  memcpy(handle, &h, sizeof h);
  return EP_OK;
}

EP_API int ep_ipc_open(const void *handle, void **ptr) {
  if (handle == nullptr || ptr == nullptr) return EP_ERR_INVALID_ARG;
  *ptr = nullptr;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof h);
  void *p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
    return EP_ERR_CUDA;
  *ptr = p;
  return EP_OK;
}

EP_API int ep_ipc_close(void *ptr) {
  if (ptr == nullptr) return EP_OK;
  return cudaIpcCloseMemHandle(ptr) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // extern "C"
