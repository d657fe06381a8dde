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
//                    lookup groups of <= 4 for k_delta_lut. Invalid ids set a status bit
//                    and join the base-only tokens. No host synchronisation.
//   base product     bf16: tcgen05 tensor-core GEMM (bd_base_tc.cu), fp32: k_base_gemv.
//                    Both write fp32 partial sums y_part[kz][t][row].
//   k_delta_tc       (bd_delta_tc.cu) the many-token tenants' delta as a tcgen05
//                    contraction with the +/-s matrix expanded into tensor memory.
//   k_delta_lut      (bd_delta_lut.cu) the few-token tenants' delta through per-chunk
//                    sign lookup tables in shared memory, all tokens of a group served by
//                    one pass over the tenant's bits.
//   Both delta kernels add the base partial sums in a fixed order and write y (bf16 or
//   fp32) in request order.
#include "bd_internal.cuh"

namespace bd {

constexpr int kMaxTenants = 16384;
constexpr int kMaxBatch = 65536;

// ------------------------------------------------------------------------------------
// planning: lookup groups for the lookup-table kernel, segments for the tensor-core one
// ------------------------------------------------------------------------------------
// Tokens are grouped by tenant (a counting sort). A tenant with at least tc_min tokens
// whose record the tensor-core path supports gets tensor-core segments of <= kTcSegTokens
// tokens; every other tenant's tokens are cut into lookup groups of <= kLutTokens (one pass
// over the tenant's bits per group), and the base-only tokens into groups of the same size.
// Groups are numbered by class: all groups of 4 tokens first, then 3, 2, 1, then the
// base-only groups, so that the lookup kernel meets one kind of group for long stretches.
// Workspace layout (int32): the kSegHeader words, grp_tenant[max_groups],
// grp_start[max_groups], grp_len[max_groups], tc_tenant[max_tc], tc_start[max_tc],
// tc_count[max_tc], tc_xrow[max_tc] (first row in the gathered X), perm[batch]; and, in a
// region of its own, a copy of each tensor-core segment's tenant record.
constexpr int kTcMaxTokens = kTcSegTokens;

inline int max_groups_for(int64_t batch, int32_t n_tenants) {
  const int64_t keys = batch < (int64_t)n_tenants + 1 ? batch : (int64_t)n_tenants + 1;
  return (int)((batch + kLutTokens - 1) / kLutTokens + keys);
}

__device__ __forceinline__ bool tc_eligible(const bd_tenant& T, int64_t d_in) {
  const bool mode_ok = ((T.mode == BD_SCALE_GROUP || T.mode == BD_SCALE_BLOCK) && T.group_size >= 64 &&
                        scale_mode_ok(T.mode, T.group_size, d_in)) ||
                       T.mode == BD_SCALE_ROW || T.mode == BD_SCALE_COL || T.mode == BD_SCALE_TENSOR;
  const bool ptr_ok = T.signs != nullptr && T.scales != nullptr &&
                      ((reinterpret_cast<uintptr_t>(T.signs) | reinterpret_cast<uintptr_t>(T.scales)) & 15u) == 0;
  // the tensor-core kernel streams whole tiles of the serving layout
  return mode_ok && ptr_ok && T.layout == BD_LAYOUT_TILED && T.reserved == 0;
}

constexpr int kPlanQ = 3 + kLutClasses;  // tokens, tc segments, gathered X rows, groups per class

__global__ void __launch_bounds__(1024) k_tenant_bucket(const int32_t* __restrict__ ids, int batch,
                                                        int n_tenants, int max_groups, int max_tc,
                                                        const bd_tenant* __restrict__ tenants,
                                                        int tc_min, int64_t d_in, int64_t lut_tiles,
                                                        int split_cap, int lut_ctas,
                                                        int32_t* __restrict__ lut_cnt,
                                                        int32_t* __restrict__ seg_base,
                                                        bd_tenant* __restrict__ tc_rec,
                                                        uint32_t* __restrict__ status) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  extern __shared__ int32_t cnt[];  // n_tenants + 1 counters (last = base only)
  __shared__ int32_t wsum[kPlanQ][32];
  __shared__ int32_t bad;
  const int nkeys = n_tenants + 1;
  int32_t* grp_tenant = seg_base + kSegHeader;
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
  // per key: q[0] tokens, q[1] tensor-core segments, q[2] gathered-X rows, q[3 + k] lookup
  // groups of class k (k = 0..3: tenant groups of 4 - k tokens; k = 4: base-only groups)
  auto plan = [&](int k, int c, int (&q)[kPlanQ]) {
#pragma unroll
    for (int i = 0; i < kPlanQ; ++i) q[i] = 0;
    q[0] = c;
    if (c == 0) return;
    const bool tc = max_tc > 0 && k < n_tenants && c >= tc_min && tc_eligible(tenants[k], d_in);
    if (tc) {
      q[1] = (c + kTcMaxTokens - 1) / kTcMaxTokens;
      for (int j = 0; j < c; j += kTcMaxTokens) q[2] += (min(kTcMaxTokens, c - j) + 15) & ~15;
    } else if (k == n_tenants) {
      q[3 + 4] = (c + kLutTokens - 1) / kLutTokens;
    } else {
      q[3 + 0] = c / kLutTokens;
      const int rem = c % kLutTokens;
      if (rem) q[3 + (kLutTokens - rem)] = 1;
    }
  };
  const int per = (nkeys + blockDim.x - 1) / blockDim.x;
  const int k0 = threadIdx.x * per, k1 = min(nkeys, k0 + per);
  int v[kPlanQ];
#pragma unroll
  for (int i = 0; i < kPlanQ; ++i) v[i] = 0;
  for (int k = k0; k < k1; ++k) {
    int q[kPlanQ];
    plan(k, cnt[k], q);
#pragma unroll
    for (int i = 0; i < kPlanQ; ++i) v[i] += q[i];
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int inc[kPlanQ];
#pragma unroll
  for (int i = 0; i < kPlanQ; ++i) inc[i] = v[i];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int i = 0; i < kPlanQ; ++i) {
      const int a = __shfl_up_sync(0xffffffffu, inc[i], o);
      if (lane >= o) inc[i] += a;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int i = 0; i < kPlanQ; ++i) wsum[i][w] = inc[i];
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
#pragma unroll
    for (int i = 0; i < kPlanQ; ++i) {
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
  const int last = (blockDim.x >> 5) - 1;
  int ex[kPlanQ];  // this thread's exclusive prefix of each quantity
#pragma unroll
  for (int i = 0; i < kPlanQ; ++i) ex[i] = inc[i] - v[i] + (w > 0 ? wsum[i][w - 1] : 0);
  int off = ex[0], tidx = ex[1], xrow = ex[2];
  int gnext[kLutClasses];  // next group index of each class
  int cstart = 0;
#pragma unroll
  for (int k = 0; k < kLutClasses; ++k) {
    gnext[k] = cstart + ex[3 + k];
    cstart += wsum[3 + k][last];
  }
  for (int k = k0; k < k1; ++k) {
    const int c = cnt[k];
    int q[kPlanQ];
    plan(k, c, q);
    if (q[1] > 0) {
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
      for (int j = 0; j < c; j += kLutTokens) {
        const int len = min(kLutTokens, c - j);
        const int cls = k == n_tenants ? 4 : kLutTokens - len;
        const int gi = gnext[cls]++;
        grp_tenant[gi] = (k == n_tenants) ? -1 : k;
        grp_start[gi] = off + j;
        grp_len[gi] = len;
      }
    }
    cnt[k] = off;  // becomes the scatter cursor
    off += c;
  }
  if (threadIdx.x == blockDim.x - 1) {  // the last thread holds the totals
    seg_base[0] = cstart;
    seg_base[1] = tidx;
#pragma unroll
    for (int k = 0; k < kLutClasses; ++k) seg_base[2 + k] = wsum[3 + k][last];
    // K chunks of the lookup kernel's tenant units: when there are fewer (group, tile)
    // units than kLutMinUnitsPerCta per CTA of the lookup kernel, whole units would split
    // unevenly over the SMs, so each is cut into kc chunks of d_in (kc divides the windows,
    // >= 2 windows per chunk), as many as the partial-sum budget allows
    int64_t units = 0;
#pragma unroll
    for (int k = 0; k < kLutClasses - 1; ++k) units += wsum[3 + k][last];
    units *= lut_tiles;
    const int64_t nwin = (d_in + kLutWindow - 1) / kLutWindow;
    int kc = 1;
    if (units > 0 && units < (int64_t)kLutMinUnitsPerCta * lut_ctas)
      for (int c = kLutMaxChunks; c >= 2; --c)
        if (nwin % c == 0 && nwin / c >= 2 && units * c <= (int64_t)split_cap) {
          kc = c;
          break;
        }
    seg_base[2 + kLutClasses] = kc;
  }
  // the split units' arrival counters and the lookup kernel's piece counter (the word
  // after them) start from zero in every call
  for (int i = threadIdx.x; i <= split_cap / 2; i += blockDim.x) lut_cnt[i] = 0;
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
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
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
// host side
// ------------------------------------------------------------------------------------
bd_status launch_delta_tc(const bd_tenant* tenants, const int32_t* seg, int max_groups, int max_tc,
                          const void* x, int64_t d_out, int64_t d_in, int64_t batch, __half* xg,
                          int64_t xg_rows, float* xinv, const float* y_part, int ksplit, void* y,
                          bool y_bf16, uint32_t* status, cudaStream_t s);
bd_status launch_delta_lut(bool xbf16, const bd_tenant* tenants, bool scale_f16, const int32_t* seg,
                           int max_groups, int max_tc, const void* x, const float* y_part, int ksplit,
                           int64_t d_out, int64_t d_in, int64_t batch, void* y, bool y_bf16,
                           float* lut_part, int32_t* lut_cnt, int split_cap, uint32_t* status,
                           cudaStream_t s);

// A tenant with at least this many tokens in a batch (and a supported record) goes to the
// tensor-core delta kernel; below it the lookup-table kernel serves the tenant's tokens,
// kLutTokens of them per pass over its bits (one pass up to 4 tokens, two up to 8). 9 is
// the crossover measured on B200 over the fused Llama-3-8B calls of the serving workload
// (a layer took 2.36 ms with 9, 2.52 ms with 5). Both kernels compute the same product, so
// a build may set another value with -DBD_TC_MIN_TOKENS=n, n >= 1, to re-tune it;
// bd_tc_min_tokens() reports the value built in.
#ifndef BD_TC_MIN_TOKENS
#define BD_TC_MIN_TOKENS 9
#endif
constexpr int kTcMinTokens = BD_TC_MIN_TOKENS;
static_assert(kTcMinTokens >= 1, "the many-token threshold is a token count");

namespace {
struct ApplyLayout {
  int max_groups, max_tc;
  TcPlan tc;
  Fp8Plan f8;
  int ksplit;
  int split_cap;  // lookup units (x K chunks) that may keep partial sums
  int64_t xg_rows;
  size_t off_seg, off_tcrec, off_part, off_xg, off_xinv, off_x8, off_xmul, off_lpart, off_lcnt, total;
};

// tc: the base product on the tensor cores (bf16 weights, or e4m3 ones when fp8)
ApplyLayout layout_apply(int64_t d_out, int64_t d_in, int64_t batch, int32_t n_tenants, bool tc,
                         bool tc_delta, bool fp8 = false) {
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
  if (fp8) {
    L.f8 = plan_base_fp8(d_out, d_in, batch);
    L.ksplit = L.f8.ksplit;
  } else if (tc) {
    L.tc = plan_base_tc(d_out, d_in, batch);
    L.ksplit = L.tc.ksplit;
  }
  size_t off = kStatusBytes;
  L.off_seg = off;
  off = align_up(off + (kSegHeader * 4 + 3 * (size_t)L.max_groups * 4 + 4 * (size_t)L.max_tc * 4 + (size_t)batch * 4), 256);
  L.off_tcrec = off;
  off = align_up(off + (size_t)L.max_tc * sizeof(bd_tenant), 256);
  L.off_part = off;
  off = align_up(off + (size_t)L.ksplit * batch * d_out * sizeof(float), 256);
  L.off_xg = off;
  off = align_up(off + (size_t)L.xg_rows * d_in * 2, 256);
  L.off_xinv = off;
  off = align_up(off + (size_t)L.xg_rows * sizeof(float), 256);
  L.off_x8 = off;
  off = align_up(off + (fp8 ? L.f8.x8_bytes : 0), 256);
  L.off_xmul = off;
  off = align_up(off + (fp8 ? (size_t)L.f8.xmul_count * sizeof(float) : 0), 256);
  // lookup-kernel K split: partial sums [unit][512 rows][4 tokens] and arrival counters
  {
    const int64_t tiles = (d_out + kLutTileRows - 1) / kLutTileRows;
    int64_t cap = (int64_t)kLutSplitPerSm * sm_count();
    const int64_t most = (int64_t)L.max_groups * tiles * kLutMaxChunks;
    if (cap > most) cap = most;
    L.split_cap = (int)cap;
  }
  L.off_lpart = off;
  off = align_up(off + (size_t)L.split_cap * kLutTileRows * 4 * sizeof(float), 256);
  L.off_lcnt = off;
  off = align_up(off + (size_t)(L.split_cap / 2 + 1) * sizeof(int32_t), 256);
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

size_t apply_fp8_workspace_size(int64_t d_out, int64_t d_in, int64_t batch, int32_t n_tenants) {
  if (d_out < 1 || d_in < 32 || batch < 0 || n_tenants < 0) return 0;
  return layout_apply(d_out, d_in, batch, n_tenants, true, (d_in % 64) == 0, true).total;
}

// w_scales != nullptr: w_base holds e4m3 codes with per-row fp32 scales w_scales (x bf16)
bd_status apply_impl(const void* w_base, int32_t w_dtype, int64_t d_out, int64_t d_in,
                     const bd_tenant* tenants, int32_t n_tenants, int32_t scale_dtype,
                     const int32_t* tenant_ids, const void* x, int64_t batch, void* y,
                     int32_t y_dtype, void* workspace, size_t ws_bytes, cudaStream_t s,
                     const float* w_scales = nullptr) {
  const bool fp8 = w_scales != nullptr;
  if (w_dtype != BD_BF16 && w_dtype != BD_F32) return BD_ERR_DTYPE;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return BD_ERR_DTYPE;
  if (y_dtype != BD_BF16 && y_dtype != BD_F32) return BD_ERR_DTYPE;
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return BD_ERR_SHAPE;
  if (batch < 0 || batch > kMaxBatch || n_tenants < 0 || n_tenants > kMaxTenants) return BD_ERR_SHAPE;
  if (batch == 0) return BD_OK;
  if (!w_base || !x || !y || !tenant_ids) return BD_ERR_NULL;
  if (n_tenants > 0 && !tenants) return BD_ERR_NULL;
  if (!aligned16(w_base) || !aligned16(x) || !aligned16(y) || !aligned16(tenant_ids) ||
      (tenants && (reinterpret_cast<uintptr_t>(tenants) & 7u)) ||
      (fp8 && (reinterpret_cast<uintptr_t>(w_scales) & 3u)))
    return BD_ERR_ALIGN;
  const bool tc = w_dtype == BD_BF16;  // with an e4m3 base, w_dtype is the activations' bf16
  // the tensor-core delta path needs bf16 activations, fp16 scales and 64-column stages
  const bool tc_delta = tc && scale_dtype == BD_F16 && (d_in % 64) == 0;
  ApplyLayout L = layout_apply(d_out, d_in, batch, n_tenants, tc, tc_delta, fp8);
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
  BD_CUDA_TRY(launch_pdl(k_tenant_bucket, dim3(1), dim3(1024), bucket_smem, s, tenant_ids, (int)batch, n_tenants,
                         L.max_groups, L.max_tc, tenants, (int)kTcMinTokens, d_in,
                         (int64_t)((d_out + kLutTileRows - 1) / kLutTileRows), L.split_cap, sm_count(),
                         reinterpret_cast<int32_t*>(ws + L.off_lcnt), seg,
                         reinterpret_cast<bd_tenant*>(ws + L.off_tcrec), status));
  launch_end(K_TENANT_BUCKET, s);
  BD_LAUNCH_CHECK();

  // 2. base product (fp32 partial sums)
  if (fp8) {
    bd_status st = launch_base_fp8(L.f8, static_cast<const uint8_t*>(w_base), w_scales, x, d_out, d_in, batch,
                                   ws + L.off_x8, reinterpret_cast<float*>(ws + L.off_xmul), y_part, status, s);
    if (st != BD_OK) return st;
  } else if (tc) {
    bd_status st = launch_base_tc(L.tc, w_base, x, d_out, d_in, batch, y_part, status, s);
    if (st != BD_OK) return st;
  } else {
    const int64_t blocks = (d_out * 32 + 255) / 256;
    launch_begin(K_BASE_GEMV, s);
    BD_CUDA_TRY(launch_pdl(k_base_gemv_f32, dim3((unsigned)blocks), dim3(256), 0, s, (const float*)w_base,
                           (const float*)x, d_out, d_in, (int)batch, y_part));
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

  // 4. lookup-table delta over the (lookup group, row tile) space, fused with the combine
  return launch_delta_lut(tc, tenants, scale_dtype == BD_F16, seg, L.max_groups, L.max_tc, x, y_part,
                          L.ksplit, d_out, d_in, batch, y, y_dtype == BD_BF16,
                          reinterpret_cast<float*>(ws + L.off_lpart), reinterpret_cast<int32_t*>(ws + L.off_lcnt),
                          L.split_cap, status, s);
}

}  // namespace bd

extern "C" int32_t bd_tc_min_tokens(void) { return bd::kTcMinTokens; }

extern "C" size_t bd_apply_workspace_size(int64_t d_out, int64_t d_in, int64_t batch,
                                          int32_t n_tenants) {
  return bd::apply_workspace_size(d_out, d_in, batch, n_tenants);
}

extern "C" size_t bd_apply_fp8_workspace_size(int64_t d_out, int64_t d_in, int64_t batch,
                                              int32_t n_tenants) {
  return bd::apply_fp8_workspace_size(d_out, d_in, batch, n_tenants);
}

extern "C" bd_status bd_apply_multi_fp8(const uint8_t* w_codes, const float* w_scales, int64_t d_out,
                                        int64_t d_in, const bd_tenant* tenants, int32_t n_tenants,
                                        int32_t scale_dtype, const int32_t* tenant_ids, const void* x,
                                        int64_t batch, void* y, int32_t y_dtype, void* workspace,
                                        size_t ws_bytes, void* stream) {
  if (batch > 0 && !w_scales) return BD_ERR_NULL;  // (batch 0: shapes checked, nothing launched)
  return bd::apply_impl(w_codes, BD_BF16, d_out, d_in, tenants, n_tenants, scale_dtype, tenant_ids, x, batch, y,
                        y_dtype, workspace, ws_bytes, static_cast<cudaStream_t>(stream), w_scales);
}

extern "C" bd_status bd_apply_multi(const void* w_base, int32_t w_dtype, int64_t d_out,
                                    int64_t d_in, const bd_tenant* tenants, int32_t n_tenants,
                                    int32_t scale_dtype, const int32_t* tenant_ids, const void* x,
                                    int64_t batch, void* y, int32_t y_dtype, void* workspace,
                                    size_t ws_bytes, void* stream) {
  return bd::apply_impl(w_base, w_dtype, d_out, d_in, tenants, n_tenants, scale_dtype, tenant_ids,
                        x, batch, y, y_dtype, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}
