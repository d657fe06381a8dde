// Status strings, device status read-back, launch accounting and per-kernel timing.
#include "bd_internal.cuh"
#include "bd_tc.cuh"

#include <atomic>
#include <mutex>
#include <vector>

namespace bd {

static const char* const kKernelNames[K_KIND_COUNT] = {
    "delta_stats",       "scale_signpack", "col_scale_signpack",
    "scale_final",       "reconstruct",  "tenant_bucket",  "base_gemv",
    "base_tc",           "delta_lut",    "prepare",
    "tc_gather",         "delta_tc",     "selftest_wait",
    "quant_fp8",         "x_limbs",      "base_fp8",
};

const char* kernel_name(int32_t kind) {
  return (kind >= 0 && kind < K_KIND_COUNT) ? kKernelNames[kind] : "unknown";
}

namespace {
std::atomic<int64_t> g_launches{0};

struct Rec {
  int32_t kind;
  cudaEvent_t e0, e1;
};

struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;  // 2 per record
  std::vector<Rec> recs;
  size_t capacity = 0;
  int64_t dropped[K_KIND_COUNT] = {0};
  // pending begin event for the launch in progress (launch_begin / launch_end pair)
  int32_t open_kind = -1;
  cudaEvent_t open_e0 = nullptr;
};
Profiler g_prof;

int g_sm_cache[64] = {0};
}  // namespace

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (g_sm_cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_cache[dev] = n;
  }
  return g_sm_cache[dev];
}

void launch_begin(int32_t kind, cudaStream_t s) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_prof.on) return;
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (!g_prof.on) return;
  if (g_prof.recs.size() >= g_prof.capacity) {
    if (kind >= 0 && kind < K_KIND_COUNT) g_prof.dropped[kind]++;
    g_prof.open_kind = -1;
    return;
  }
  const size_t i = g_prof.recs.size();
  g_prof.open_kind = kind;
  g_prof.open_e0 = g_prof.pool[2 * i];
  cudaEventRecord(g_prof.open_e0, s);
}

void launch_end(int32_t kind, cudaStream_t s) {
  if (!g_prof.on) return;
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (g_prof.open_kind != kind || g_prof.open_e0 == nullptr) return;
  const size_t i = g_prof.recs.size();
  cudaEvent_t e1 = g_prof.pool[2 * i + 1];
  cudaEventRecord(e1, s);
  g_prof.recs.push_back(Rec{kind, g_prof.open_e0, e1});
  g_prof.open_kind = -1;
  g_prof.open_e0 = nullptr;
}

}  // namespace bd

using namespace bd;

extern "C" const char* bd_status_string(int32_t st) {
  switch (st) {
    case BD_OK: return "ok";
    case BD_ERR_NULL: return "a required pointer is NULL";
    case BD_ERR_SHAPE: return "shape out of range or not divisible as required";
    case BD_ERR_DTYPE: return "dtype not accepted by this call";
    case BD_ERR_ALIGN: return "pointer not 16-byte aligned";
    case BD_ERR_CONFIG: return "bad config (scale mode, group size, clip)";
    case BD_ERR_CUDA: return "CUDA runtime error";
    case BD_ERR_TENANT_RANGE: return "tenant id outside [-1, n_tenants)";
    case BD_ERR_TIMEOUT: return "a bounded wait inside a kernel gave up";
    case BD_ERR_WORKSPACE: return "workspace missing or too small";
    case BD_ERR_TENANT_RECORD: return "a bd_tenant record is invalid";
    case BD_ERR_INTERNAL: return "a kernel's layout self-check failed";
    default: return "unknown status";
  }
}

extern "C" bd_status bd_get_status(const void* workspace, uint32_t* flags, void* stream) {
  if (!workspace) return BD_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t f = 0;
  BD_CUDA_TRY(cudaMemcpyAsync(&f, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s));
  BD_CUDA_TRY(cudaStreamSynchronize(s));
  if (flags) *flags = f;
  if (f & BD_DEV_INTERNAL) return BD_ERR_INTERNAL;
  if (f & BD_DEV_TIMEOUT) return BD_ERR_TIMEOUT;
  if (f & BD_DEV_TENANT_RECORD) return BD_ERR_TENANT_RECORD;
  if (f & BD_DEV_TENANT_RANGE) return BD_ERR_TENANT_RANGE;
  return BD_OK;
}

extern "C" int64_t bd_launch_count(void) { return g_launches.load(); }

namespace bd {
// One thread waits on an mbarrier that nothing ever arrives on, through the same bounded
// wait the tensor-core kernels use: the wait must give up after limit_cycles, set
// BD_DEV_TIMEOUT and let the kernel end normally.
__global__ void k_selftest_wait(long long limit_cycles, uint32_t* __restrict__ status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;  // never raised
  if (threadIdx.x == 0) {
    status[0] = 0;
    abort_flag = 0;
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 &&
      !mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), limit_cycles))
    atomicOr(status, BD_DEV_TIMEOUT);
}
}  // namespace bd

extern "C" bd_status bd_selftest_wait_timeout(void* workspace, size_t ws_bytes,
                                              int64_t limit_cycles, void* stream) {
  if (!workspace) return BD_ERR_NULL;
  if (ws_bytes < kStatusBytes) return BD_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return BD_ERR_ALIGN;
  if (limit_cycles < 1 || limit_cycles > kWaitCycles) return BD_ERR_CONFIG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  launch_begin(K_SELFTEST_WAIT, s);
  k_selftest_wait<<<1, 32, 0, s>>>((long long)limit_cycles, static_cast<uint32_t*>(workspace));
  launch_end(K_SELFTEST_WAIT, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}

extern "C" bd_status bd_profile_enable(int32_t on, int32_t capacity) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (on) {
    if (capacity < 1) capacity = 1;
    const size_t need = 2 * (size_t)capacity;
    while (g_prof.pool.size() < need) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) {
        (void)cudaGetLastError();
        return BD_ERR_CUDA;
      }
      g_prof.pool.push_back(e);
    }
    g_prof.capacity = (size_t)capacity;
    g_prof.recs.clear();
    for (auto& d : g_prof.dropped) d = 0;
    g_prof.on = true;
  } else {
    g_prof.on = false;
  }
  return BD_OK;
}

extern "C" int32_t bd_profile_collect(int64_t* launches, double* total_ms, int32_t max_kinds) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  const int n = max_kinds < K_KIND_COUNT ? max_kinds : K_KIND_COUNT;
  for (int k = 0; k < n; ++k) {
    if (launches) launches[k] = 0;
    if (total_ms) total_ms[k] = 0.0;
  }
  for (const Rec& r : g_prof.recs) {
    cudaEventSynchronize(r.e1);
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.e0, r.e1) != cudaSuccess) {
      (void)cudaGetLastError();
      continue;
    }
    if (r.kind >= 0 && r.kind < n) {
      if (launches) launches[r.kind] += 1;
      if (total_ms) total_ms[r.kind] += ms;
    }
  }
  g_prof.recs.clear();
  return n;
}

extern "C" const char* bd_kernel_name(int32_t kind) { return kernel_name(kind); }
