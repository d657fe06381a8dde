// Internal helpers shared by the library's translation units (not part of the ABI).
#pragma once

#include <atomic>

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/bitdelta.h"

namespace bd {

// ------------------------------------------------------------------------------------
// kernel kinds (for launch accounting and per-kernel timing)
// ------------------------------------------------------------------------------------
// Tokens per tensor-core delta segment (the MMA's N, rounded up to 16). 64 keeps one
// window of a segment's activations at 32 KB, so four windows fit the shared-memory ring.
constexpr int kTcSegTokens = 64;

// Plan written by the tenant-bucket kernel into the apply workspace (int32 words):
// [0] lookup groups, [1] tensor-core segments, [2..6] lookup groups per class (NT = 4, 3,
// 2, 1 tokens of a tenant, then base-only groups), [7] K chunks of the lookup kernel's
// tenant units (1: every unit covers all of d_in); then the arrays.
constexpr int kSegHeader = 8;
constexpr int kLutTokens = 4;   // tokens of one tenant served by one pass of the lookup kernel
constexpr int kLutClasses = 5;
constexpr int kLutTileRows = 512;   // rows of one lookup-kernel tile (and of the serving layout)
constexpr int kLutWindow = 256;     // columns of one lookup-kernel window
constexpr int kLutMaxChunks = 8;    // most K chunks a lookup unit is cut into
// Split budget: the planner cuts the lookup kernel's tenant units into K chunks only while
// (units x chunks) stays within this many per SM; each such chunk keeps a 512-row x
// 4-token fp32 partial sum in the workspace (8 KB).
constexpr int kLutSplitPerSm = 32;
// ... and only when there are fewer whole units than this per CTA of the lookup kernel:
// then whole units split unevenly over the SMs. With more, cutting costs more than it
// evens out (measured on B200: the 1792 one-token units of the decode call cut in two
// took 22% longer; the 616 units of the serving workload's down call, 56 windows long,
// cut in seven took 24% less).
constexpr int kLutMinUnitsPerCta = 8;

enum KernelKind : int32_t {
  K_DELTA_STATS = 0,     // fused delta + whole-matrix shifted sums for the clip
  K_SCALE_SIGNPACK,      // clip + abs-mean (group / row / tensor partials) + sign pack
  K_COL_SCALE_SIGNPACK,  // clip + per-column partial abs sums + sign pack
  K_SCALE_FINAL,         // fixed-order row / column / tensor scale reduction
  K_RECONSTRUCT,         // signs * scales (+ W_base)
  K_TENANT_BUCKET,       // counting sort of tenant ids -> segments
  K_BASE_GEMV,           // CUDA-core base product for small batches / fp32
  K_BASE_TC,             // tcgen05 base product (bf16, fp32 accumulation in TMEM)
  K_DELTA_LUT,           // per-tenant sign-LUT delta product + combine
  K_PREPARE,             // re-tiling of a tenant into the serving layout
  K_TC_GATHER,           // gather + fp16 scaling of the tensor-core segments' tokens
  K_DELTA_TC,            // tcgen05 delta product of many-token tenants + combine
  K_SELFTEST_WAIT,       // failure-detection self test: a bounded wait that runs out
  K_QUANT_FP8,           // per-row e4m3 quantization of a base matrix
  K_X_LIMBS,             // activations -> two e4m3 limbs per value + a power-of-two per token
  K_BASE_FP8,            // tcgen05 base product from e4m3 weights (fp32 accumulation in TMEM)
  K_KIND_COUNT
};

const char* kernel_name(int32_t kind);

// Launch plans of the two base products (bd_base_tc.cu, bd_base_fp8.cu), used by the
// apply call to size its workspace and launch them.
struct TcPlan {
  int n_tile, tiles_n, tiles_m, kblocks, kb_per_split, ksplit, stages;
  size_t smem;
};
struct Fp8Plan {
  int h, n_tile, tiles_n, tiles_m, kblocks, kb_per_split, ksplit, stages;  // h tokens per N tile
  size_t smem, x8_bytes;
  int xmul_count;
};
TcPlan plan_base_tc(int64_t d_out, int64_t d_in, int64_t batch);
bd_status launch_base_tc(const TcPlan& p, const void* w_base, const void* x, int64_t d_out,
                         int64_t d_in, int64_t batch, float* y_part, uint32_t* status,
                         cudaStream_t s);
Fp8Plan plan_base_fp8(int64_t d_out, int64_t d_in, int64_t batch);
bd_status launch_base_fp8(const Fp8Plan& p, const uint8_t* codes, const float* w_scales, const void* x,
                          int64_t d_out, int64_t d_in, int64_t batch, uint8_t* x8, float* xmul, float* y_part,
                          uint32_t* status, cudaStream_t s);

// Called around every kernel launch of the library (bd_abi.cu).
void launch_begin(int32_t kind, cudaStream_t s);
void launch_end(int32_t kind, cudaStream_t s);

int sm_count();  // multiprocessors of the current device (cached per device)

// Lets `fn` use `bytes` of dynamic shared memory on the current device. The attribute is
// per device, so it is set once per device (tracked in `done`, one bit per device
// ordinal < 64; higher ordinals set it on every call). False on a CUDA error (cleared).
template <typename F>
inline bool ensure_dyn_smem(F* fn, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  if (bit) done.fetch_or(bit, std::memory_order_release);
  return true;
}

// Device status word, the first 16 bytes of every workspace.
struct DevStatus {
  uint32_t flags;
  uint32_t pad[3];
};
constexpr size_t kStatusBytes = 256;  // keeps what follows 256-byte aligned

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// A scale mode and group size valid for d_in: GROUP and BLOCK need a power of two >= 32
// that divides d_in.
__host__ __device__ inline bool scale_mode_ok(int32_t mode, int32_t G, int64_t d_in) {
  if (mode < BD_SCALE_GROUP || mode > BD_SCALE_BLOCK) return false;
  if (mode == BD_SCALE_GROUP || mode == BD_SCALE_BLOCK)
    return G >= 32 && (G & (G - 1)) == 0 && (d_in % G) == 0;
  return true;
}
// number of scales of a mode
__host__ __device__ inline int64_t scale_count(int32_t mode, int32_t G, int64_t d_out, int64_t d_in) {
  switch (mode) {
    case BD_SCALE_GROUP: return d_out * (d_in / G);
    case BD_SCALE_ROW: return d_out;
    case BD_SCALE_COL: return d_in;
    case BD_SCALE_BLOCK: return ((d_out + G - 1) / G) * (d_in / G);
    default: return 1;
  }
}
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

#define BD_CUDA_TRY(expr)                           \
  do {                                              \
    cudaError_t _e = (expr);                        \
    if (_e != cudaSuccess) {                        \
      (void)cudaGetLastError();                     \
      return BD_ERR_CUDA;                           \
    }                                               \
  } while (0)

// Launch `kernel` on `s` with programmatic stream serialization allowed: its blocks may be
// scheduled while the previous kernel on the stream drains (the kernel calls pdl_wait()
// before reading anything).
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

#define BD_LAUNCH_CHECK()                           \
  do {                                              \
    cudaError_t _e = cudaGetLastError();            \
    if (_e != cudaSuccess) return BD_ERR_CUDA;      \
  } while (0)

// ------------------------------------------------------------------------------------
// device helpers
// ------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// round-to-nearest-even float -> bf16 bits (finite inputs)
__device__ __forceinline__ uint32_t f2bf_bits(float f) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Programmatic dependent launch (sm_90+). A kernel launched with launch_pdl may start while
// the previous kernel on its stream is still running; pdl_wait() blocks until that kernel
// has completed and its writes are visible, so it comes before any read of data another
// kernel may have produced. pdl_trigger() lets the next kernel on the stream start
// launching (it still waits for this one in its own pdl_wait). Both are no-ops for a
// kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  // 16-byte global load that is not kept in L1 (each byte is read once)
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

}  // namespace bd
