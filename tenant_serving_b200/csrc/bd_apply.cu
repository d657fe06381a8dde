// bd_apply_multi: y_t = W_base x_t + Delta_hat_{u(t)} x_t for a batch of mixed tenants.
//
// "BitDelta Guide", "Systems Mechanics: 1. Decoupled Forward Pass" (shared base product,
// per-tenant delta product) and "2. Fused Dequantization ..." (sign bits stay packed in
// HBM and are expanded on chip). The pages give no kernel for this GPU; the design here:
//
//   k_tenant_bucket  one CTA: counting sort of the tenant ids and the token permutation.
//                    A tenant with enough tokens (and a record the tensor-core kernel
//                    supports) gets segments of <= kTcSegTokens tokens for k_delta_tc;
//                    every other tenant's tokens, and the base-only ones, are cut into
//                    groups of <= 2 for k_delta_lut. Invalid ids set a status bit and
//                    join the base-only tokens. No host synchronisation.
//   base product     bf16: tcgen05 tensor-core GEMM (bd_base_tc.cu), fp32: k_base_gemv.
//                    Both write fp32 partial sums y_part[kz][t][row].
//   k_delta_tc       (bd_delta_tc.cu) the many-token tenants' delta as a tcgen05
//                    contraction with the +/-s matrix expanded into tensor memory.
//   k_delta_lut      persistent CTAs split the (token group, 512-row tile) space evenly.
//                    A CTA streams the tenant's sign words through shared memory 256
//                    columns at a time and, per token, turns every byte of signs into ONE
//                    table lookup: for each 8-column chunk a 256-entry table holds
//                    sum_j (+/-) x_j for every sign pattern (built per window from two
//                    16-entry nibble tables). The lookup order is rotated by row so the
//                    lanes of a warp hit distinct banks. Group-128 scales multiply once per
//                    128 columns, column scales are folded into x before the tables are
//                    built, row / tensor scales multiply at the end.
//   Both delta kernels add the base partial sums in a fixed order and write y (bf16 or
//   fp32) in request order.
#include "bd_internal.cuh"

namespace bd {

struct TcPlan {
  int n_tile, tiles_n, tiles_m, kblocks, kb_per_split, ksplit, stages;
  size_t smem;
};
TcPlan plan_base_tc(int64_t d_out, int64_t d_in, int64_t batch);
bd_status launch_base_tc(const TcPlan& p, const void* w_base, const void* x, int64_t d_out,
                         int64_t d_in, int64_t batch, float* y_part, uint32_t* status,
                         cudaStream_t s);

constexpr int kMaxTenants = 16384;
constexpr int kMaxBatch = 65536;

// ------------------------------------------------------------------------------------
// planning: token groups for the lookup-table kernel, segments for the tensor-core one
// ------------------------------------------------------------------------------------
// Tokens are grouped by tenant (a counting sort). A tenant with at least tc_min tokens
// whose record the tensor-core path supports gets tensor-core segments of <= kTcSegTokens tokens;
// every other tenant's tokens (and the base-only tokens) are cut into lookup-table groups
// of <= kGroupTokens.
// Workspace layout (int32): [0] n_groups, [1] n_tc, [2..3] pad, grp_tenant[max_groups],
// grp_start[max_groups], grp_len[max_groups], tc_tenant[max_tc], tc_start[max_tc],
// tc_count[max_tc], tc_xrow[max_tc] (first row in the gathered X), perm[batch]; and, in
// a region of its own, a copy of each tensor-core segment's tenant record.
constexpr int kGroupTokens = 2;
constexpr int kTcMaxTokens = kTcSegTokens;

inline int max_groups_for(int64_t batch, int32_t n_tenants) {
  const int64_t keys = batch < (int64_t)n_tenants + 1 ? batch : (int64_t)n_tenants + 1;
  return (int)((batch + kGroupTokens - 1) / kGroupTokens + keys);
}

__device__ __forceinline__ bool tc_eligible(const bd_tenant& T, int64_t d_in) {
  const bool mode_ok = (T.mode == BD_SCALE_GROUP && T.group_size >= 64 &&
                        (T.group_size & (T.group_size - 1)) == 0 && (d_in % T.group_size) == 0) ||
                       T.mode == BD_SCALE_ROW || T.mode == BD_SCALE_TENSOR;
  const bool ptr_ok = T.signs != nullptr && T.scales != nullptr &&
                      ((reinterpret_cast<uintptr_t>(T.signs) | reinterpret_cast<uintptr_t>(T.scales)) & 15u) == 0;
  // the tensor-core kernel streams whole tiles of the serving layout
  return mode_ok && ptr_ok && T.layout == BD_LAYOUT_TILED && T.reserved == 0;
}

__global__ void __launch_bounds__(1024) k_tenant_bucket(const int32_t* __restrict__ ids, int batch,
                                                        int n_tenants, int max_groups, int max_tc,
                                                        const bd_tenant* __restrict__ tenants,
                                                        int tc_min, int64_t d_in,
                                                        int32_t* __restrict__ seg_base,
                                                        bd_tenant* __restrict__ tc_rec,
                                                        uint32_t* __restrict__ status) {
  extern __shared__ int32_t cnt[];  // n_tenants + 1 counters (last = base only)
  __shared__ int32_t wsum[5][32];
  __shared__ int32_t bad;
  const int nkeys = n_tenants + 1;
  int32_t* grp_tenant = seg_base + 4;
  int32_t* grp_start = grp_tenant + max_groups;
  int32_t* grp_len = grp_start + max_groups;
  int32_t* tc_tenant = grp_len + max_groups;
  int32_t* tc_start = tc_tenant + max_tc;
  int32_t* tc_count = tc_start + max_tc;
  int32_t* tc_xrow = tc_count + max_tc;
  int32_t* perm = tc_xrow + max_tc;
  if (threadIdx.x == 0) {
    status[0] = 0;  // the status word reports this call
    bad = 0;
  }
  for (int k = threadIdx.x; k < nkeys; k += blockDim.x) cnt[k] = 0;
  __syncthreads();
  for (int t = threadIdx.x; t < batch; t += blockDim.x) {
    int u = ids[t];
    if (u < -1 || u >= n_tenants) {
      bad = 1;
      u = -1;
    }
    atomicAdd(&cnt[u < 0 ? n_tenants : u], 1);
  }
  __syncthreads();
  // per key: tokens, full lookup groups (kGroupTokens tokens), remainder groups, tensor-core
  // segments, gathered-X rows. All full groups are numbered before all remainder groups,
  // so that the lookup-table kernel meets one kind of group for long stretches.
  auto plan = [&](int k, int c, int& ng, int& nr, int& nt, int& nx) {
    ng = nr = nt = nx = 0;
    if (c == 0) return;
    const bool tc = max_tc > 0 && k < n_tenants && c >= tc_min && tc_eligible(tenants[k], d_in);
    if (tc) {
      nt = (c + kTcMaxTokens - 1) / kTcMaxTokens;
      for (int j = 0; j < c; j += kTcMaxTokens) nx += (min(kTcMaxTokens, c - j) + 15) & ~15;
    } else {
      ng = c / kGroupTokens;
      nr = (c % kGroupTokens) ? 1 : 0;
    }
  };
  const int per = (nkeys + blockDim.x - 1) / blockDim.x;
  const int k0 = threadIdx.x * per, k1 = min(nkeys, k0 + per);
  int v[5] = {0, 0, 0, 0, 0};  // tokens, full groups, tc segments, X rows, remainder groups
  for (int k = k0; k < k1; ++k) {
    int ng, nr, nt, nx;
    plan(k, cnt[k], ng, nr, nt, nx);
    v[0] += cnt[k];
    v[1] += ng;
    v[2] += nt;
    v[3] += nx;
    v[4] += nr;
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int inc[5] = {v[0], v[1], v[2], v[3], v[4]};
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const int a = __shfl_up_sync(0xffffffffu, inc[i], o);
      if (lane >= o) inc[i] += a;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int i = 0; i < 5; ++i) wsum[i][w] = inc[i];
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      int a = lane < nw ? wsum[i][lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int c = __shfl_up_sync(0xffffffffu, a, o);
        if (lane >= o) a += c;
      }
      if (lane < nw) wsum[i][lane] = a;
    }
  }
  __syncthreads();
  int off = inc[0] - v[0] + (w > 0 ? wsum[0][w - 1] : 0);
  int gidx = inc[1] - v[1] + (w > 0 ? wsum[1][w - 1] : 0);
  int tidx = inc[2] - v[2] + (w > 0 ? wsum[2][w - 1] : 0);
  int xrow = inc[3] - v[3] + (w > 0 ? wsum[3][w - 1] : 0);
  const int n_full = wsum[1][(blockDim.x >> 5) - 1];  // all full groups come first
  int ridx = n_full + inc[4] - v[4] + (w > 0 ? wsum[4][w - 1] : 0);
  for (int k = k0; k < k1; ++k) {
    const int c = cnt[k];
    int ng, nr, nt, nx;
    plan(k, c, ng, nr, nt, nx);
    if (nt > 0) {
      for (int j = 0; j < c; j += kTcMaxTokens) {
        const int n = min(kTcMaxTokens, c - j);
        tc_tenant[tidx] = k;
        tc_rec[tidx] = tenants[k];
        tc_start[tidx] = off + j;
        tc_count[tidx] = n;
        tc_xrow[tidx] = xrow;
        xrow += (n + 15) & ~15;
        ++tidx;
      }
    } else {
      for (int j = 0; j < c; j += kGroupTokens) {
        const bool full = c - j >= kGroupTokens;
        const int gi = full ? gidx++ : ridx++;
        grp_tenant[gi] = (k == n_tenants) ? -1 : k;
        grp_start[gi] = off + j;
        grp_len[gi] = min(kGroupTokens, c - j);
      }
    }
    cnt[k] = off;  // becomes the scatter cursor
    off += c;
  }
  if (threadIdx.x == blockDim.x - 1) {  // the last thread holds the totals
    seg_base[0] = ridx;
    seg_base[1] = tidx;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < batch; t += blockDim.x) {
    int u = ids[t];
    if (u < -1 || u >= n_tenants) u = -1;
    const int pos = atomicAdd(&cnt[u < 0 ? n_tenants : u], 1);
    perm[pos] = t;
  }
  if (threadIdx.x == 0 && bad) atomicOr(status, BD_DEV_TENANT_RANGE);
}

// ------------------------------------------------------------------------------------
// fp32 base product on CUDA cores (small problems; the bf16 path uses tensor cores)
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_base_gemv_f32(const float* __restrict__ W,
                                                       const float* __restrict__ X, int64_t d_out,
                                                       int64_t d_in, int batch,
                                                       float* __restrict__ y_part) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= d_out) return;
  const float* wr = W + row * d_in;
  for (int t0 = 0; t0 < batch; t0 += 8) {
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int64_t k = lane * 4; k < d_in; k += 128) {
      const float4 w = *reinterpret_cast<const float4*>(wr + k);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (t0 + j < batch) {
          const float4 x = *reinterpret_cast<const float4*>(X + (int64_t)(t0 + j) * d_in + k);
          acc[j] = fmaf(w.x, x.x, fmaf(w.y, x.y, fmaf(w.z, x.z, fmaf(w.w, x.w, acc[j]))));
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float v = warp_sum_f(acc[j]);
      if (lane == 0 && t0 + j < batch) y_part[(int64_t)(t0 + j) * d_out + row] = v;
    }
  }
}

// ------------------------------------------------------------------------------------
// delta product with per-chunk sign lookup tables
// ------------------------------------------------------------------------------------
// Persistent CTAs (one per SM, 8 warps) split the flattened (token group, 512-row tile)
// space evenly; a CTA walks its share in pieces of at most 2048 rows of one group
// (<= 2 tokens of one tenant). A tenant split over several groups has its sign words
// streamed once per group.
//
// A piece streams the tenant's sign words 256 columns (8 words) x 512 rows per stage
// through a 6-deep cp.async ring. Per 256-column window and token, a table
// T[v][c] = sum_j (bit j of v ? +x : -x)[8c + j] over the 8 columns of chunk c is built
// in shared memory for every sign byte v; then one byte of signs costs one table read
// per token.
//   lanes: q = lane >> 1 picks one of 16 rows, wp = lane & 1 one half of the window
//   (words 4wp..4wp+3). At step (k, j) a lane reads word 4wp + ((k + q/4 + 2wp) & 3)
//   and its byte (j + q) & 3: the 32 lanes read 32 different staged words (32 banks),
//   and each half-warp reads 16 different table chunks modulo 16.
//   table page: it sits at shared address 0x10000. For a 2-token group entry
//   (v, chunk, token) is at 0x10000 + v * 256 + 8 * chunk + 4 * token: the two tokens sit
//   side by side, one 8-byte ld.shared returns both, and each half-warp's 16 lanes cover
//   the 32 banks once. For a 1-token group entry (v, chunk) is at 0x10000 + v * 256 +
//   4 * chunk, and the 32 lanes' 4-byte reads cover the 32 banks once. One PRMT of the
//   sign word with the lane's slot constant (entry stride x chunk, plus the 0x1 of
//   0x10000 in its upper half) yields the whole 32-bit shared address of the entry.
//   A lookup is PRMT + ld.shared(.v2) + FADD per token.
//   Group-128 scales are one per lane per row (words 4wp..4wp+3 are one group) and are
//   staged next to the sign words.
constexpr int LUT_THREADS = 256;    // 8 warps, 64 rows each per stage
constexpr int LUT_RG = 4;           // 16-row groups per warp per stage
constexpr int LUT_WARPS = LUT_THREADS / 32;
constexpr int LUT_W = 256;          // columns per window
constexpr int LUT_SB = 512;         // rows per stage: one 16-row slice per warp
constexpr int LUT_NSB = 4;          // stages (sub-blocks) per window of a piece
constexpr int LUT_PASS = LUT_SB * LUT_NSB;  // rows per piece
constexpr int LUT_STAGES = 6;       // cp.async ring depth
constexpr int LUT_SC = 8;           // staged scale bytes per row per window
constexpr uint32_t LUT_BITS_STAGE = LUT_SB * 32;
constexpr uint32_t LUT_SC_STAGE = LUT_SB * LUT_SC;
constexpr uint32_t LUT_ADDR = 0x10000;  // shared address of the table page
constexpr uint32_t LUT_HALF = 3 * (LUT_BITS_STAGE + LUT_SC_STAGE);  // ring stages below / above
constexpr uint32_t LUT_LOW = LUT_ADDR - LUT_HALF;    // first ring byte; dynamic smem must start <=
constexpr uint32_t LUT_X_STAGE = 4096;  // per ring slot: x of 2 tokens + column scales
constexpr uint32_t LUT_XBASE = 0x20000 + LUT_HALF;   // x slots of the ring
constexpr uint32_t LUT_PIECE = LUT_XBASE + LUT_STAGES * LUT_X_STAGE;  // piece descriptor
constexpr size_t LUT_SMEM = LUT_PIECE + 128;  // requested from the dynamic base

__device__ __forceinline__ uint32_t sh_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float2 lds_f32x2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_f32x2(uint32_t a, float x, float y) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(x), "f"(y) : "memory");
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_f16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return __half2float(__ushort_as_half(v));
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float ld_scale(const void* s, bool f16, int64_t i) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(s)[i]) : reinterpret_cast<const float*>(s)[i];
}

struct LutPiece {
  bd_tenant T;
  int u, mode, G, ntok, t0, t1, rows, sc_kind, layout, pos_step, scale_f16;
  int64_t rb0;      // first 512-row tile of the piece
  int64_t r0;
  int64_t bstride;  // sign words between consecutive 512-row stages
  int64_t half_stride;  // sign words between rows r and r + 256
  int64_t sstride;  // staged-scale bytes between consecutive stages
  int whole;
};

__device__ __forceinline__ uint32_t lut_bits_stage(int b) {
  return b < 3 ? LUT_LOW + (uint32_t)b * LUT_BITS_STAGE
               : 0x20000u + (uint32_t)(b - 3) * LUT_BITS_STAGE;
}
__device__ __forceinline__ uint32_t lut_sc_stage(int b) {
  return b < 3 ? LUT_LOW + 3 * LUT_BITS_STAGE + (uint32_t)b * LUT_SC_STAGE
               : 0x20000u + 3 * LUT_BITS_STAGE + (uint32_t)(b - 3) * LUT_SC_STAGE;
}

__device__ __forceinline__ uint32_t lut_x_stage(int b) { return LUT_XBASE + (uint32_t)b * LUT_X_STAGE; }

// Issue the copies of stage (win, sb) into ring buffer b. Staged scales are 2 per row
// (2 * ssz bytes, row stride 2 * ssz).
__device__ __forceinline__ void lut_stage(const LutPiece& P, int win, int sb,
                                          int b, int64_t d_in, bool scale_f16, const void* x,
                                          bool xbf16, int nwin) {
  const int tid = threadIdx.x;
  const int rb = sb * LUT_SB;
  const int ssz = scale_f16 ? 2 : 4;
  if (P.layout == BD_LAYOUT_TILED) {
    // one contiguous 16 KB tile of sign words and (group-128) a 2 / 4 KB tile of scales
    const int64_t tile = (P.rb0 + sb) * nwin + win;
    const uint32_t* src = P.T.signs + tile * 4096;
#pragma unroll
    for (int c = 0; c < 1024; c += LUT_THREADS)
      cp_async16(lut_bits_stage(b) + (uint32_t)(c + tid) * 16u, src + (c + tid) * 4);
    if (P.sc_kind == 1) {
      const uint8_t* ssrc = reinterpret_cast<const uint8_t*>(P.T.scales) + tile * 1024 * ssz;
      for (int c = tid; c * 16 < 1024 * ssz; c += LUT_THREADS)
        cp_async16(lut_sc_stage(b) + (uint32_t)c * 16u, ssrc + c * 16);
    }
  } else {
    if (P.whole) {
      // two 16-byte copies per thread: rows tid/2 and tid/2 + 256 of the stage, half tid & 1
      const int64_t wpr = d_in >> 5;
      // 16-byte copies: copy c = row (c >> 1), half (c & 1) of the stage
      for (int c = tid; c < 1024; c += LUT_THREADS) {
        const int row = c >> 1;
        if (rb + row < P.rows)
          cp_async16(lut_bits_stage(b) + (uint32_t)c * 16u,
                     P.T.signs + (P.r0 + rb + row) * wpr + (c & 1) * 4 + win * 8);
      }
    } else {
      const int64_t wpr = d_in >> 5;
      const int64_t w0 = (int64_t)win * (LUT_W / 32);
      const int nr = min(LUT_SB, P.rows - rb);
      const uint32_t* src = P.T.signs + (P.r0 + rb) * wpr + w0;
      for (int i = tid; i < nr * 8; i += LUT_THREADS) {
        const int rl = i >> 3, k = i & 7;
        if (w0 + k < wpr) cp_async4(lut_bits_stage(b) + rl * 32 + k * 4, src + rl * wpr + k);
      }
    }
    if (P.sc_kind == 1) {
      const int64_t per_row = (d_in / 128) * ssz;
      for (int r = tid; r < LUT_SB && rb + r < P.rows; r += LUT_THREADS) {
        const uint8_t* sp = reinterpret_cast<const uint8_t*>(P.T.scales) + (P.r0 + rb + r) * per_row +
                            win * 2 * ssz;
        const uint32_t sd = lut_sc_stage(b) + (uint32_t)(r * 2 * ssz);
        if (scale_f16) cp_async4(sd, sp);
        else cp_async8(sd, sp);
      }
    }
  }
  // the first stage of a window also brings the window's slice of x (both tokens) and,
  // for column scales, the window's scales: [x0 1 KB][x1 1 KB][col scales 1 KB]
  if (sb == 0 && tid < 3 * 64) {
    const int part = tid >> 6, k = tid & 63;  // 64 x 16 B per part (LUT_THREADS >= 192)
    const int64_t col0 = (int64_t)win * LUT_W;
    const int xb = xbf16 ? 2 : 4;
    const uint32_t dst = lut_x_stage(b) + (uint32_t)(part * 1024 + k * 16);
    if (part < 2) {
      const int64_t col = col0 + (int64_t)k * (16 / xb);
      if (part < P.ntok && k * 16 < LUT_W * xb && col < d_in) {
        const int t = part == 0 ? P.t0 : P.t1;
        cp_async16(dst, reinterpret_cast<const uint8_t*>(x) + ((int64_t)t * d_in + col) * xb);
      }
    } else if (P.mode == BD_SCALE_COL) {
      const int64_t col = col0 + (int64_t)k * (16 / ssz);
      if (k * 16 < LUT_W * ssz && col < d_in)
        cp_async16(dst, reinterpret_cast<const uint8_t*>(P.T.scales) + col * ssz);
    }
  }
}

// Build the sign tables of one window for the piece's tokens from the x slice (and
// column scales) staged in ring slot b.
template <bool XBF16>
__device__ __forceinline__ void lut_build(const LutPiece& P, int win, int b, int64_t d_in,
                                          bool scale_f16) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = lane;  // chunk of the window
  // this thread fills the sign patterns with high nibble h and h + 8 (h = warp, 8 warps)
  const int64_t col = (int64_t)win * LUT_W + 8 * c;
  const uint32_t xs = lut_x_stage(b);
  float sc[8];
  if (P.mode == BD_SCALE_COL) {
    if (scale_f16) {
      uint4 v;
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(xs + 2048 + 16 * c));
      const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 hh = *reinterpret_cast<const __half2*>(&a[k]);
        sc[2 * k] = __low2float(hh);
        sc[2 * k + 1] = __high2float(hh);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) sc[k] = lds_f32(xs + 2048 + 32 * c + 4 * k);
    }
  }
  // both tokens' 16 low-nibble sums (a second token of 0 for single-token groups)
  float lo16[2][16];
  float xv[2][8];
#pragma unroll
  for (int tt = 0; tt < 2; ++tt) {
    if (tt < P.ntok && col < d_in) {
      if (XBF16) {
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(xs + 1024 * tt + 16 * c));
        const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          xv[tt][2 * k] = bf16lo(a[k]);
          xv[tt][2 * k + 1] = bf16hi(a[k]);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) xv[tt][k] = lds_f32(xs + 1024 * tt + 32 * c + 4 * k);
      }
      if (P.mode == BD_SCALE_COL) {
#pragma unroll
        for (int k = 0; k < 8; ++k) xv[tt][k] *= sc[k];
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) xv[tt][k] = 0.f;
    }
    float p01[4], p23[4];
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      p01[n] = ((n & 1) ? xv[tt][0] : -xv[tt][0]) + ((n & 2) ? xv[tt][1] : -xv[tt][1]);
      p23[n] = ((n & 1) ? xv[tt][2] : -xv[tt][2]) + ((n & 2) ? xv[tt][3] : -xv[tt][3]);
    }
#pragma unroll
    for (int lo = 0; lo < 16; ++lo) lo16[tt][lo] = p01[lo & 3] + p23[lo >> 2];
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int h = warp + 8 * hh;
    float hi[2];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
      hi[tt] = (((h & 1) ? xv[tt][4] : -xv[tt][4]) + ((h & 2) ? xv[tt][5] : -xv[tt][5])) +
               (((h & 4) ? xv[tt][6] : -xv[tt][6]) + ((h & 8) ? xv[tt][7] : -xv[tt][7]));
    if (P.ntok == 2) {
      const uint32_t base = LUT_ADDR + (uint32_t)(h << 12) + 8u * (uint32_t)c;
#pragma unroll
      for (int lo = 0; lo < 16; ++lo)
        sts_f32x2(base + (uint32_t)lo * 256u, lo16[0][lo] + hi[0], lo16[1][lo] + hi[1]);
    } else {
      const uint32_t base = LUT_ADDR + (uint32_t)(h << 12) + 4u * (uint32_t)c;
#pragma unroll
      for (int lo = 0; lo < 16; ++lo) sts_f32(base + (uint32_t)lo * 256u, lo16[0][lo] + hi[0]);
    }
  }
}

// Generic path: group sizes other than 128 (one scale per word from global memory) and
// windows that run past d_in. Recomputes the lane constants itself (slow path).
template <int NT>
__device__ __forceinline__ float2 lut_rows_generic(uint32_t wrow, uint32_t srow, const LutPiece& P,
                                                int sb, int i, int win, int64_t d_in,
                                                bool scale_f16) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane >> 1, wp = lane & 1;
  const int rl = sb * LUT_SB + warp * (16 * LUT_RG) + i * 16 + q;  // row inside the piece
  float a0 = 0.f, a1 = 0.f;
  if (rl >= P.rows) return make_float2(0.f, 0.f);
#pragma unroll 1
  for (int k = 0; k < 4; ++k) {
    const int wi = 4 * wp + ((k + (q >> 2) + 2 * wp) & 3);
    const int64_t col = (int64_t)win * LUT_W + 32 * wi;
    if (col >= d_in) continue;
    const uint32_t word = lds_u32(wrow + 4u * (uint32_t)wi);
    float p0 = 0.f, p1 = 0.f;
    for (int j = 0; j < 4; ++j) {
      const int b = (j + q) & 3;
      const uint32_t idx = LUT_ADDR + (((word >> (8 * b)) & 0xFFu) << 8) +
                           (NT == 2 ? 8u : 4u) * (uint32_t)(4 * wi + b);
      p0 += lds_f32(idx);
      if (NT == 2) p1 += lds_f32(idx + 4u);
    }
    float sw = 1.f;
    if (P.sc_kind == 1) {  // staged group-128 scales: group (wi >> 2) of the window
      const uint32_t a = srow + (uint32_t)((wi >> 2) * (scale_f16 ? 2 : 4));
      sw = scale_f16 ? lds_f16(a) : lds_f32(a);
    } else if (P.sc_kind == 2) {
      sw = ld_scale(P.T.scales, scale_f16, (P.r0 + rl) * (d_in / P.G) + col / P.G);
    }
    a0 = fmaf(sw, p0, a0);
    if (NT == 2) a1 = fmaf(sw, p1, a1);
  }
  return make_float2(a0, a1);
}

// The stage loop of one piece. SC: 0 = no per-word scale (row / col / tensor modes, or
// the generic path, which handles scales itself), 1 = staged fp16 group-128 scales,
// 2 = staged fp32 group-128 scales. GENERIC: group sizes other than 128 or a last window
// that runs past d_in.
template <bool XBF16, int NT, int SC, bool GENERIC>
__device__ __forceinline__ void lut_piece(const LutPiece& P, float (&acc)[LUT_NSB][LUT_RG][2], int nwin,
                                          int64_t d_in, const void* x, const uint32_t (&sel)[4],
                                          const uint32_t (&slot2)[4][2], const uint32_t (&wofs)[4],
                                          int warp, int q, int wp) {
  const bool f16s = P.scale_f16 != 0;
  const int ssz = GENERIC ? (f16s ? 2 : 4) : (SC == 2 ? 4 : 2);
  // 2-token tables have 8-byte entries: the slot bytes (entry stride x chunk, <= 124 for
  // the 4-byte stride) double, the 0x1 of 0x10000 in the upper half stays
  uint32_t sl[4][2];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
      sl[k][hh] = NT == 2 ? (((slot2[k][hh] & 0xFFFFu) << 1) | (slot2[k][hh] & 0xFFFF0000u))
                          : slot2[k][hh];
  const int rows = P.rows;
  const int nsb = (rows + LUT_SB - 1) / LUT_SB;  // 1..4
  int pw = 0, ps = 0;
#pragma unroll
  for (int i = 0; i < LUT_STAGES - 1; ++i) {
    if (pw < nwin) {
      lut_stage(P, pw, ps, i, d_in, P.scale_f16 != 0, x, XBF16, nwin);
      if (++ps == nsb) { ps = 0; ++pw; }
    }
    cp_async_commit();
  }
  int bcur = 0, bnext = LUT_STAGES - 1;
  for (int win = 0; win < nwin; ++win) {
#pragma unroll
    for (int sb = 0; sb < LUT_NSB; ++sb) {
      if (sb < nsb) {
        // this stage's copies (the oldest group still pending) have landed for this thread;
        // the barrier makes them visible to all and also tells that every warp is done with
        // the previous stage, whose ring slot (bnext) is refilled right after it
        cp_async_wait<LUT_STAGES - 2>();
        __syncthreads();
        if (pw < nwin) {
          lut_stage(P, pw, ps, bnext, d_in, P.scale_f16 != 0, x, XBF16, nwin);
          if (++ps == nsb) { ps = 0; ++pw; }
        }
        cp_async_commit();
        if (sb == 0) {  // new window: build its tables from the staged x slice
          lut_build<XBF16>(P, win, bcur, d_in, P.scale_f16 != 0);
          __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < LUT_RG; ++i) {  // the warp's 16-row groups of this stage
          const int rs = warp * (16 * LUT_RG) + i * 16;  // first row of the group in the stage
          const uint32_t wrow = lut_bits_stage(bcur) + (uint32_t)((rs + q) * 32);
          // the fast path runs every row group unconditionally (no branch, so the groups'
          // loads interleave); rows past the piece read stale staging data and their
          // results are never written out
          if (!GENERIC || sb * LUT_SB + rs < rows) {
            if (!GENERIC) {
              float s_ = 1.f;
              if (SC != 0) {
                const uint32_t sa = lut_sc_stage(bcur) + (uint32_t)((rs + q) * 2 * ssz + wp * ssz);
                s_ = SC == 1 ? lds_f16(sa) : lds_f32(sa);
              }
              // 16 independent table reads per token, summed as a tree (depth 4)
              uint32_t wd[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) wd[k] = lds_u32(wrow + wofs[k]);
              float w0[4], w1[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                float v0[4], v1[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const uint32_t idx = __byte_perm(wd[k], sl[k][j >> 1], sel[j]);
                  if (NT == 2) {
                    const float2 e = lds_f32x2(idx);
                    v0[j] = e.x;
                    v1[j] = e.y;
                  } else {
                    v0[j] = lds_f32(idx);
                  }
                }
                w0[k] = (v0[0] + v0[1]) + (v0[2] + v0[3]);
                if (NT == 2) w1[k] = (v1[0] + v1[1]) + (v1[2] + v1[3]);
              }
              acc[sb][i][0] = fmaf(s_, (w0[0] + w0[1]) + (w0[2] + w0[3]), acc[sb][i][0]);
              if (NT == 2) acc[sb][i][1] = fmaf(s_, (w1[0] + w1[1]) + (w1[2] + w1[3]), acc[sb][i][1]);
            } else {
              const uint32_t srow = lut_sc_stage(bcur) + (uint32_t)((rs + q) * 2 * ssz);
              const float2 r = lut_rows_generic<NT>(wrow, srow, P, sb, i, win, d_in, f16s);
              acc[sb][i][0] += r.x;
              acc[sb][i][1] += r.y;
            }
          }
        }
        bcur = bcur + 1 == LUT_STAGES ? 0 : bcur + 1;
        bnext = bnext + 1 == LUT_STAGES ? 0 : bnext + 1;
      }
    }
  }
}

// Per-lane lookup constants (see the comment above k_delta_lut's lookup loop).
__device__ __forceinline__ void lut_lane_constants(int q, int wp, uint32_t estride, uint32_t (&sel)[4],
                                                   uint32_t (&slot2)[4][2], uint32_t (&wofs)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int b = (j + q) & 3;
    sel[j] = 0x7600u | ((uint32_t)b << 4) | (uint32_t)(4 + (j & 1));
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int wi = 4 * wp + ((k + (q >> 2) + 2 * wp) & 3);
    wofs[k] = 4u * (uint32_t)wi;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t s0 = estride * (uint32_t)(4 * wi + ((2 * hh + q) & 3));
      const uint32_t s1 = estride * (uint32_t)(4 * wi + ((2 * hh + 1 + q) & 3));
      slot2[k][hh] = s0 | (s1 << 8) | (LUT_ADDR & 0xFFFF0000u);
    }
  }
}

template <bool XBF16>
__global__ void __launch_bounds__(LUT_THREADS, 1) k_delta_lut(
    const bd_tenant* __restrict__ tenants, bool scale_f16, const int32_t* __restrict__ seg_base,
    int max_groups, int max_tc, const void* __restrict__ x, const float* __restrict__ y_part,
    int ksplit, int64_t d_out, int64_t d_in, int batch, void* __restrict__ y, bool y_bf16,
    uint32_t* __restrict__ status) {
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t base = sh_addr(smem);
  if (base > LUT_LOW) {  // the fixed layout needs the dynamic window to start low enough
    if (threadIdx.x == 0) atomicOr(status, BD_DEV_INTERNAL);
    return;
  }
  LutPiece& piece = *reinterpret_cast<LutPiece*>(smem + (LUT_PIECE - base));
  float* out_s = reinterpret_cast<float*>(smem + (LUT_ADDR - base));  // after the last window

  const int32_t* grp_tenant = seg_base + 4;
  const int32_t* grp_start = grp_tenant + max_groups;
  const int32_t* grp_len = grp_start + max_groups;
  const int32_t* perm = grp_len + max_groups + 4 * max_tc;
  // the (token group, 512-row tile) space is split evenly over the CTAs; a piece is up to
  // LUT_NSB consecutive tiles of one group
  const int n_groups = seg_base[0];
  const int64_t n_rt = (d_out + LUT_SB - 1) / LUT_SB;
  const int64_t total = (int64_t)n_groups * n_rt;
  const int64_t share = (total + gridDim.x - 1) / gridDim.x;
  int64_t pos = (int64_t)blockIdx.x * share;
  const int64_t end = min(total, pos + share);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = lane >> 1, wp = lane & 1;
  const int nwin = (int)((d_in + LUT_W - 1) / LUT_W);
  // per-lane lookup constants. sel[j]: byte 0 <- slot byte (j & 1) of slot2[k][j >> 1],
  // byte 1 <- sign byte (j + q) & 3, bytes 2-3 <- 0x0001 (the table's 0x10000).
  uint32_t sel[4], slot2[4][2], wofs[4];
  lut_lane_constants(q, wp, 4u, sel, slot2, wofs);  // 1-token entry stride; lut_piece doubles it

  while (pos < end) {
    if (tid == 0) {
      LutPiece Q;
      const int g = (int)(pos / n_rt);
      Q.rb0 = pos - (int64_t)g * n_rt;
      const int64_t ntiles = min((int64_t)LUT_NSB, min(n_rt - Q.rb0, end - pos));
      Q.r0 = Q.rb0 * LUT_SB;
      Q.rows = (int)min(ntiles * LUT_SB, d_out - Q.r0);
      Q.pos_step = (int)ntiles;
      Q.u = grp_tenant[g];
      Q.ntok = grp_len[g];
      Q.t0 = perm[grp_start[g]];
      Q.t1 = Q.ntok > 1 ? perm[grp_start[g] + 1] : Q.t0;
      Q.mode = BD_SCALE_GROUP;
      Q.G = 128;
      Q.T.signs = nullptr;
      Q.T.scales = nullptr;
      if (Q.u >= 0) {
        Q.T = tenants[Q.u];
        Q.mode = Q.T.mode;
        Q.G = Q.T.group_size;
        // the table lives in device memory, so its records are checked here
        const bool ok_mode = Q.mode >= BD_SCALE_GROUP && Q.mode <= BD_SCALE_TENSOR;
        const bool ok_group = Q.mode != BD_SCALE_GROUP ||
                              (Q.G >= 32 && (Q.G & (Q.G - 1)) == 0 && (d_in % Q.G) == 0);
        const bool ok_ptr = Q.T.signs != nullptr && Q.T.scales != nullptr &&
                            ((reinterpret_cast<uintptr_t>(Q.T.signs) |
                              reinterpret_cast<uintptr_t>(Q.T.scales)) & 15u) == 0;
        const bool ok_layout = (Q.T.layout == BD_LAYOUT_ROWMAJOR || Q.T.layout == BD_LAYOUT_TILED) &&
                               Q.T.reserved == 0;
        if (!(ok_mode && ok_group && ok_ptr && ok_layout)) {
          atomicOr(status, BD_DEV_TENANT_RECORD);
          Q.u = -1;  // base product only
        }
      }
      Q.whole = (d_in % LUT_W) == 0;
      Q.layout = Q.u >= 0 ? Q.T.layout : BD_LAYOUT_ROWMAJOR;
      // 0: no per-word scale; 1: staged group-128 scales (tiled, or row-major with whole
      // windows); 2: group scales read from global memory per word
      Q.sc_kind = Q.mode != BD_SCALE_GROUP
                      ? 0
                      : ((Q.G == 128 && (Q.whole || Q.layout == BD_LAYOUT_TILED)) ? 1 : 2);
      Q.scale_f16 = scale_f16 ? 1 : 0;
      Q.bstride = (int64_t)LUT_SB * (d_in >> 5);
      Q.half_stride = (int64_t)256 * (d_in >> 5);
      Q.sstride = (int64_t)LUT_SB * (d_in / 128) * (scale_f16 ? 2 : 4);
      piece = Q;
    }
    __syncthreads();
    const LutPiece& P = piece;
    pos += P.pos_step;

    float acc[LUT_NSB][LUT_RG][2];  // [sub-block][16-row group][token]
#pragma unroll
    for (int i = 0; i < LUT_NSB; ++i)
#pragma unroll
      for (int j = 0; j < LUT_RG; ++j) acc[i][j][0] = acc[i][j][1] = 0.f;

    if (P.u >= 0) {
      // one specialised stage loop per (tokens, scale kind, path), chosen once per piece
      const bool generic = P.sc_kind == 2 || !P.whole;
      const int ntok = P.ntok;
#define BD_PIECE(NT, SC, GEN) \
  lut_piece<XBF16, NT, SC, GEN>(P, acc, nwin, d_in, x, sel, slot2, wofs, warp, q, wp)
      if (generic) {
        if (ntok == 2) BD_PIECE(2, 0, true); else BD_PIECE(1, 0, true);
      } else if (P.sc_kind == 1) {
        if (scale_f16) { if (ntok == 2) BD_PIECE(2, 1, false); else BD_PIECE(1, 1, false); }
        else { if (ntok == 2) BD_PIECE(2, 2, false); else BD_PIECE(1, 2, false); }
      } else {
        if (ntok == 2) BD_PIECE(2, 0, false); else BD_PIECE(1, 0, false);
      }
#undef BD_PIECE
    }
    // the staged results reuse the table page: every warp must be done with its lookups
    __syncthreads();
    // ---- reduce the two lanes of each row, stage per-token results
#pragma unroll
    for (int sb = 0; sb < LUT_NSB; ++sb) {
#pragma unroll
      for (int i = 0; i < LUT_RG; ++i) {
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          const float v = acc[sb][i][tt] + __shfl_xor_sync(0xffffffffu, acc[sb][i][tt], 1);
          const int rl = sb * LUT_SB + warp * (16 * LUT_RG) + i * 16 + q;
          if (wp == 0) out_s[tt * LUT_PASS + rl] = v;
        }
      }
    }
    __syncthreads();
    // ---- combine with the base product, write y in request order
    // each thread owns up to LUT_RPT rows x 2 tokens; the split-K partials of all of them
    // are loaded together (independent loads) before any is added
    constexpr int LUT_RPT = (LUT_PASS + LUT_THREADS - 1) / LUT_THREADS;
    float rs = 1.f;
    if (P.u >= 0 && P.mode == BD_SCALE_TENSOR) rs = ld_scale(P.T.scales, scale_f16, 0);
    float bsum[2][LUT_RPT];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
      for (int k = 0; k < LUT_RPT; ++k) bsum[tt][k] = 0.f;
    for (int kz = 0; kz < ksplit; ++kz) {
      const float* part = y_part + (int64_t)kz * batch * d_out + P.r0 + tid;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const int t = tt == 0 ? P.t0 : P.t1;
#pragma unroll
        for (int k = 0; k < LUT_RPT; ++k)
          if (tt < P.ntok && tid + k * LUT_THREADS < P.rows)
            bsum[tt][k] += part[(int64_t)t * d_out + k * LUT_THREADS];
      }
    }
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      const int t = tt == 0 ? P.t0 : P.t1;
#pragma unroll
      for (int k = 0; k < LUT_RPT; ++k) {
        const int rl = tid + k * LUT_THREADS;
        if (tt < P.ntok && rl < P.rows) {
          const int64_t row = P.r0 + rl;
          float d = 0.f;
          if (P.u >= 0) {
            float sc = rs;
            if (P.mode == BD_SCALE_ROW) sc = ld_scale(P.T.scales, scale_f16, row);
            d = sc * out_s[tt * LUT_PASS + rl];
          }
          const float v = bsum[tt][k] + d;
          if (y_bf16)
            reinterpret_cast<uint16_t*>(y)[(int64_t)t * d_out + row] = (uint16_t)f2bf_bits(v);
          else
            reinterpret_cast<float*>(y)[(int64_t)t * d_out + row] = v;
        }
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
bd_status launch_delta_tc(const bd_tenant* tenants, const int32_t* seg, int max_groups, int max_tc,
                          const void* x, int64_t d_out, int64_t d_in, int64_t batch, __half* xg,
                          int64_t xg_rows, float* xinv, const float* y_part, int ksplit, void* y,
                          bool y_bf16, uint32_t* status, cudaStream_t s);

// A tenant with at least this many tokens in a batch (and a supported record) goes to the
// tensor-core delta kernel; below it the lookup-table kernel is cheaper per token (6 is
// the crossover measured on B200; both kernels compute the same product, so a build may
// set another value with -DBD_TC_MIN_TOKENS=n, n >= 1, to re-tune it).
#ifndef BD_TC_MIN_TOKENS
#define BD_TC_MIN_TOKENS 6
#endif
constexpr int kTcMinTokens = BD_TC_MIN_TOKENS;

namespace {
struct ApplyLayout {
  int max_groups, max_tc;
  TcPlan tc;
  int ksplit;
  int64_t xg_rows;
  size_t off_seg, off_tcrec, off_part, off_xg, off_xinv, total;
};

ApplyLayout layout_apply(int64_t d_out, int64_t d_in, int64_t batch, int32_t n_tenants, bool tc,
                         bool tc_delta) {
  ApplyLayout L;
  L.max_groups = max_groups_for(batch, n_tenants);
  if (L.max_groups < 1) L.max_groups = 1;
  // a batch smaller than the many-token threshold has no tensor-core segment at all
  if (tc_delta && batch >= kTcMinTokens) {
    // segments: at most one per many-token tenant plus one per extra kTcSegTokens tokens
    int64_t by_tokens = batch / kTcMinTokens, by_tenants = n_tenants;
    L.max_tc = (int)((by_tokens < by_tenants ? by_tokens : by_tenants) + batch / kTcMaxTokens + 1);
  } else {
    L.max_tc = 0;
  }
  L.xg_rows = tc_delta ? batch + 15 * (int64_t)L.max_tc : 0;
  L.ksplit = 1;
  if (tc) {
    L.tc = plan_base_tc(d_out, d_in, batch);
    L.ksplit = L.tc.ksplit;
  }
  size_t off = kStatusBytes;
  L.off_seg = off;
  off = align_up(off + (16 + 3 * (size_t)L.max_groups * 4 + 4 * (size_t)L.max_tc * 4 + (size_t)batch * 4), 256);
  L.off_tcrec = off;
  off = align_up(off + (size_t)L.max_tc * sizeof(bd_tenant), 256);
  L.off_part = off;
  off = align_up(off + (size_t)L.ksplit * batch * d_out * sizeof(float), 256);
  L.off_xg = off;
  off = align_up(off + (size_t)L.xg_rows * d_in * 2, 256);
  L.off_xinv = off;
  off = align_up(off + (size_t)L.xg_rows * sizeof(float), 256);
  L.total = off;
  return L;
}

}  // namespace

size_t apply_workspace_size(int64_t d_out, int64_t d_in, int64_t batch, int32_t n_tenants) {
  if (d_out < 1 || d_in < 32 || batch < 0 || n_tenants < 0) return 0;
  const size_t a = layout_apply(d_out, d_in, batch, n_tenants, true, (d_in % 64) == 0).total;
  const size_t b = layout_apply(d_out, d_in, batch, n_tenants, false, false).total;
  return a > b ? a : b;
}

bd_status apply_impl(const void* w_base, int32_t w_dtype, int64_t d_out, int64_t d_in,
                     const bd_tenant* tenants, int32_t n_tenants, int32_t scale_dtype,
                     const int32_t* tenant_ids, const void* x, int64_t batch, void* y,
                     int32_t y_dtype, void* workspace, size_t ws_bytes, cudaStream_t s) {
  if (w_dtype != BD_BF16 && w_dtype != BD_F32) return BD_ERR_DTYPE;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return BD_ERR_DTYPE;
  if (y_dtype != BD_BF16 && y_dtype != BD_F32) return BD_ERR_DTYPE;
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return BD_ERR_SHAPE;
  if (batch < 0 || batch > kMaxBatch || n_tenants < 0 || n_tenants > kMaxTenants) return BD_ERR_SHAPE;
  if (batch == 0) return BD_OK;
  if (!w_base || !x || !y || !tenant_ids) return BD_ERR_NULL;
  if (n_tenants > 0 && !tenants) return BD_ERR_NULL;
  if (!aligned16(w_base) || !aligned16(x) || !aligned16(y) || !aligned16(tenant_ids) ||
      (tenants && (reinterpret_cast<uintptr_t>(tenants) & 7u)))
    return BD_ERR_ALIGN;
  const bool tc = w_dtype == BD_BF16;
  // the tensor-core delta path needs bf16 activations, fp16 scales and 64-column stages
  const bool tc_delta = tc && scale_dtype == BD_F16 && (d_in % 64) == 0;
  ApplyLayout L = layout_apply(d_out, d_in, batch, n_tenants, tc, tc_delta);
  if (!workspace || ws_bytes < L.total) return BD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BD_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  int32_t* seg = reinterpret_cast<int32_t*>(ws + L.off_seg);
  float* y_part = reinterpret_cast<float*>(ws + L.off_part);

  // 1. bucket tokens by tenant into groups
  const size_t bucket_smem = (size_t)(n_tenants + 1) * sizeof(int32_t);
  static std::atomic<uint64_t> bucket_attr{0};
  if (!ensure_dyn_smem(k_tenant_bucket, (kMaxTenants + 1) * (int)sizeof(int32_t), bucket_attr))
    return BD_ERR_CUDA;
  launch_begin(K_TENANT_BUCKET, s);
  k_tenant_bucket<<<1, 1024, bucket_smem, s>>>(tenant_ids, (int)batch, n_tenants, L.max_groups,
                                               L.max_tc, tenants, kTcMinTokens, d_in, seg,
                                               reinterpret_cast<bd_tenant*>(ws + L.off_tcrec), status);
  launch_end(K_TENANT_BUCKET, s);
  BD_LAUNCH_CHECK();

  // 2. base product (fp32 partial sums)
  if (tc) {
    bd_status st = launch_base_tc(L.tc, w_base, x, d_out, d_in, batch, y_part, status, s);
    if (st != BD_OK) return st;
  } else {
    const int64_t blocks = (d_out * 32 + 255) / 256;
    launch_begin(K_BASE_GEMV, s);
    k_base_gemv_f32<<<(unsigned)blocks, 256, 0, s>>>((const float*)w_base, (const float*)x, d_out,
                                                     d_in, (int)batch, y_part);
    launch_end(K_BASE_GEMV, s);
    BD_LAUNCH_CHECK();
  }

  // 3. tensor-core delta for the many-token tenants, fused with the combine
  if (L.max_tc > 0) {
    bd_status st = launch_delta_tc(reinterpret_cast<const bd_tenant*>(ws + L.off_tcrec), seg,
                                   L.max_groups, L.max_tc, x, d_out, d_in, batch,
                                   reinterpret_cast<__half*>(ws + L.off_xg), L.xg_rows,
                                   reinterpret_cast<float*>(ws + L.off_xinv), y_part, L.ksplit, y,
                                   y_dtype == BD_BF16, status, s);
    if (st != BD_OK) return st;
  }

  // 4. lookup-table delta over the (token group, row) space, fused with the combine
  auto kfn = tc ? k_delta_lut<true> : k_delta_lut<false>;
  static std::atomic<uint64_t> lut_attr[2];
  if (!ensure_dyn_smem(kfn, (int)LUT_SMEM, lut_attr[tc ? 1 : 0])) return BD_ERR_CUDA;

  launch_begin(K_DELTA_LUT, s);
  kfn<<<(unsigned)sm_count(), LUT_THREADS, LUT_SMEM, s>>>(tenants, scale_dtype == BD_F16, seg,
                                                         L.max_groups, L.max_tc, x, y_part, L.ksplit,
                                                         d_out, d_in, (int)batch, y,
                                                         y_dtype == BD_BF16, status);
  launch_end(K_DELTA_LUT, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}

}  // namespace bd

extern "C" size_t bd_apply_workspace_size(int64_t d_out, int64_t d_in, int64_t batch,
                                          int32_t n_tenants) {
  return bd::apply_workspace_size(d_out, d_in, batch, n_tenants);
}

extern "C" bd_status bd_apply_multi(const void* w_base, int32_t w_dtype, int64_t d_out,
                                    int64_t d_in, const bd_tenant* tenants, int32_t n_tenants,
                                    int32_t scale_dtype, const int32_t* tenant_ids, const void* x,
                                    int64_t batch, void* y, int32_t y_dtype, void* workspace,
                                    size_t ws_bytes, void* stream) {
  return bd::apply_impl(w_base, w_dtype, d_out, d_in, tenants, n_tenants, scale_dtype, tenant_ids,
                        x, batch, y, y_dtype, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}
